/*
 * vc.h -- C ABI of the VeriCache hot-path library (libvc_b200.so, sm_100a).
 *
 * VeriCache drafts tokens from a compressed KV cache and verifies them against
 * the full KV cache, keeping exactly the tokens full-cache greedy decoding
 * would produce ("VeriCache: making lossy KV compression exact", devshah.ca,
 * section "The Core Idea"; "VeriCache: Turning Lossy KV Cache into Lossless
 * LLM Inference", menfem.com, section "Key Contributions").  This library is
 * the data-parallel hot path of one round:
 *
 *   draft attention   one query token per request over the compressed cache,
 *                     either quantised (vc_draft_attn_quant) or token-dropped
 *                     (vc_draft_attn_sparse);
 *   verify attention  nq = K + 1 causal query rows per request over the full
 *                     bf16 cache (vc_verify_attn);
 *   acceptance        argmax of the K + 1 verifier logit rows, first mismatch,
 *                     accepted length and correction token (vc_accept).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - Pointers are DEVICE pointers unless a parameter says "host".  The caller
 *   owns all memory; the library never allocates device memory in these
 *   calls.  Element types are given per argument: bf16 and fp16 arrays are
 *   passed as `const void*` holding IEEE binary16 / bfloat16 bit patterns.
 * - Layouts are dense, row-major, with the shapes written in brackets
 *   (last index fastest).  Every device pointer must be 16-byte aligned.
 * - `stream` is a cudaStream_t passed as `void*` (NULL = legacy default
 *   stream).  Calls only enqueue work on that stream and return; nothing
 *   blocks the host.
 * - Workspace: each kernel that splits the context across thread blocks
 *   needs a caller-owned workspace of at least the size its
 *   *_workspace_size() function returns.  The workspace must be zero-filled
 *   once before its first use (e.g. cudaMemsetAsync); every call leaves it
 *   ready for the next call.  Calls that share one workspace must not
 *   overlap on the GPU (use one workspace per stream in flight).
 * - Errors: invalid shapes, sizes, alignments or null pointers are detected
 *   on the host before any launch and return VC_ERR_INVALID_ARG (nothing is
 *   enqueued); unsupported but well-formed configurations return
 *   VC_ERR_UNSUPPORTED; a failed launch returns VC_ERR_CUDA.  A thread-local
 *   message for the last error is available from vc_last_error().  Data
 *   errors that only the device can see (an out-of-range kept position, a
 *   bounded wait that timed out) skip the offending access and set a flag
 *   in the workspace, readable with vc_workspace_flags().
 */
#ifndef VC_H_
#define VC_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define VC_ABI_VERSION 2

#if defined(__GNUC__)
#define VC_API __attribute__((visibility("default")))
#else
#define VC_API
#endif

typedef enum vc_status {
  VC_OK = 0,
  VC_ERR_INVALID_ARG = -1,
  VC_ERR_UNSUPPORTED = -2,
  VC_ERR_CUDA = -3,
  VC_ERR_TIMEOUT = -4,
  VC_ERR_WORKSPACE = -5
} vc_status;

typedef enum vc_dtype { VC_F32 = 0, VC_BF16 = 1, VC_F16 = 2 } vc_dtype;

/* Device-side flags reported through the workspace (bit mask). */
#define VC_FLAG_BAD_INDEX 1u   /* a kept position was outside [0, T_store) */
#define VC_FLAG_WAIT_TIMEOUT 2u /* a bounded on-chip wait gave up */
#define VC_FLAG_RANGE 4u        /* a quantisation scale or zero fell outside the fp16 range */
#define VC_FLAG_BAD_LENGTH 8u   /* a per-request length or accepted length was invalid; that request was skipped */

/* Message for the last error returned on the calling thread ("" if none). */
VC_API const char* vc_last_error(void);
/* ABI version of the loaded library (VC_ABI_VERSION at build time). */
VC_API int vc_abi_version(void);

/* Attention geometry of one call (one layer).
 *   B    requests in the batch, >= 1
 *   Hq   query heads, Hkv KV heads; Hq % Hkv == 0 and g = Hq / Hkv <= 8.
 *        Query head hq reads KV head hq / g (grouped-query attention).
 *   D    head dimension, 64 or 128
 *   sm_scale  softmax scale; a value <= 0 selects 1 / sqrt(D). */
typedef struct vc_attn_shape {
  int B;
  int Hq;
  int Hkv;
  int D;
  float sm_scale;
} vc_attn_shape;

/* One layer of a quantised draft cache.  Quantisation keeps every position
 * and lowers the precision of each stored number (devshah.ca page, section
 * "The Tradeoff VeriCache Is Trying to Escape"); the system sees a compressor
 * only through its bit width and its dropped positions (menfem.com source
 * page, section "Key Contributions").  The pages fix no format; this one is
 * KIVI-style asymmetric uniform quantisation:
 *
 *   keys:   per channel over groups of `group` consecutive tokens,
 *           k_hat[t][c] = code * k_scale[t / group][c] + k_zero[t / group][c]
 *   values: per token over groups of `group` consecutive channels,
 *           v_hat[t][c] = code * v_scale[t][c / group] + v_zero[t][c / group]
 *
 * evaluated as one fp32 fused multiply-add.  The oldest L_q tokens are
 * quantised; the newest R tokens are kept in bf16 (the residual window, rows
 * 0..R-1 of a buffer of R_cap rows).
 *
 * Storage (this library's choice; the pages fix none).  Everything one group
 * of `group` quantised tokens needs is one contiguous RECORD, so a stage of
 * the draft kernel is a single bulk copy:
 *
 *   records   uint8 [B][Hkv][L_q / group][REC],  REC = 2 * CB + 8 * D,
 *             CB = group * D * bits / 8
 *   record:   [0, CB)            key codes of the group (block order below)
 *             [CB, 2CB)          value codes of the group (block order below)
 *             [2CB, +2D)         key scales, D fp16 in key-parameter order
 *             [2CB + 2D, +2D)    key zeros, same order
 *             [2CB + 4D, +2D)    value scales of the group's tokens, fp16
 *                                [group/2][D/group][2]: for token pair
 *                                (2p, 2p+1) and value group v, the two
 *                                tokens' entries side by side
 *             [2CB + 6D, +2D)    value zeros, same shape
 *   k_res, v_res      bf16  [B][Hkv][R_cap][D]
 *
 * Key-parameter order: channel c = 16 kt + 8 h + 2 t + e (h, e in {0,1},
 * t in 0..3) sits at fp16 slot 2 (t * 2 (D/16) + 2 kt + h) + e, so the
 * channel pairs one MMA lane multiplies form one contiguous run.
 *
 * Code blocks are stored in fragment-native order, the order in which the
 * tensor-core tiles of the draft kernel consume them.  For one group (a
 * group x D code matrix C[t][c]) split tokens and channels into tiles of 16;
 * lane L = 4 gid + tig (gid 0..7, tig 0..3) owns, per (token tile, channel
 * tile), four registers of two codes:
 *   keys:   reg0 = C[16tt+gid][16ct+2tig+{0,1}],  reg1 = same with token +8,
 *           reg2 = C[16tt+gid][16ct+2tig+8+{0,1}], reg3 = reg2 with token +8
 *   values: reg0 = C[16tt+2tig+{0,1}][16ct+gid],  reg1 = same with channel +8,
 *           reg2 = C[16tt+2tig+8+{0,1}][16ct+gid], reg3 = reg2 with channel +8
 * Words X_j / Y_j (j = 0 .. NW/2 - 1, NW = 2 (D/16) / TPW, TPW = 8 / bits)
 * cover the channel tiles ct = TPW j + i; keys: X_j = (reg0, reg1), Y_j =
 * (reg2, reg3); values: X_j = (reg0, reg2), Y_j = (reg1, reg3).  In a word,
 * local tile i puts the first register's two codes at bits [bits*i, +bits)
 * and [16 + bits*i, +bits), the second register's at [8 + bits*i, +bits) and
 * [24 + bits*i, +bits).  Lane L's word w of token tile tt is 32-bit word
 * (tt * 32 + L) * NW + w of the group's block.
 *
 *   bits in {2, 4}; group in {32, 64}; L_q >= 0 and a multiple of group;
 *   0 <= R <= R_cap; L_q + R >= 1; records, k_res and v_res 16-byte
 *   aligned.  Scales, zeros and codes must be finite and q * scale must stay
 *   inside the fp16 range (|q * scale| < 65504). */
typedef struct vc_quant_cache {
  const void* records;
  const void* k_res;
  const void* v_res;
  int bits;
  int group;
  int64_t L_q;
  int R;
  int R_cap;
  /* Optional device int32 [B][2]: the (L_q, R) of each request, for caches
   * maintained on the device across rounds (vc_cache_commit).  When set, L_q
   * above is the record capacity in tokens (records holds L_q / group records
   * per (request, KV head)), R above is ignored, and request b uses its own
   * lens[b] = (L_q_b, R_b) with L_q_b a multiple of group, L_q_b <= L_q and
   * R_b <= R_cap.  NULL: every request has L_q and R. */
  const int32_t* lens;
  /* VC_CACHE_STATIC: the records, residual rows and lens are not written by
   * the kernel that precedes this call in the stream (e.g. the previous
   * layer's draft call), so the draft kernel may start copying its first
   * records before that kernel has finished.  0: it waits first (always
   * safe; required right after vc_cache_commit or any other writer). */
  int flags;
} vc_quant_cache;
#define VC_CACHE_STATIC 1

/* One layer of a token-dropped draft cache: every (request, KV head) keeps
 * the same number n_keep of positions (the pages restrict the method to equal
 * drop counts per layer and head, menfem.com source page, section
 * "Limitations"; a dropping compressor is described by its positions,
 * section "Key Contributions").
 *   k, v   bf16  [B][Hkv][T_store][D]   rows addressed by idx
 *   idx    int32 [B][Hkv][n_keep]       each in [0, T_store); order free
 *   n_keep >= 1. */
typedef struct vc_sparse_cache {
  const void* k;
  const void* v;
  int64_t T_store;
  const int32_t* idx;
  int n_keep;
} vc_sparse_cache;

/* ---- draft attention over a quantised cache --------------------------------
 * out[b][hq][:] = softmax(q[b][hq] . K_hat^T * sm_scale) . V_hat over the
 * L_q dequantised tokens followed by the R residual tokens of KV head hq / g.
 * Drafting decodes one token per step against the compressed cache held in
 * HBM (menfem.com source page, "Key Contributions").
 *   q    bf16 [B][Hq][D]        (|q| < 65504)
 *   out  fp32 [B][Hq][D]
 *   ws   workspace of vc_draft_attn_quant_workspace_size() bytes. */
VC_API size_t vc_draft_attn_quant_workspace_size(const vc_attn_shape* shape, const vc_quant_cache* cache);
VC_API vc_status vc_draft_attn_quant(const vc_attn_shape* shape, const vc_quant_cache* cache, const void* q,
                              float* out, void* ws, size_t ws_bytes, void* stream);

/* ---- allocation-free quantised draft attention -----------------------------
 * The pages have no counterpart to this entry point; it serves callers that
 * cannot allocate device memory or pass a workspace -- code running inside a
 * host framework whose memory pool owns all device memory, or latency-
 * critical paths that must never reach an allocator.  It computes exactly
 * what vc_draft_attn_quant computes, with the same arguments minus the
 * workspace: the split-K scratch lives in a fixed device array of
 * VC_NOALLOC_SCRATCH_BYTES inside the library, which every GPU that loads the
 * library holds until the process exits.  Nothing is allocated.
 *   - The first call on a device looks up that array's address (with the
 *     device current); make that first call before any stream capture.
 *   - All calls share the one array and leave in it whatever they wrote;
 *     nothing in it has to start at zero except the flag word below, which
 *     is zero when the library loads.  Calls that overlap on the GPU
 *     (different streams or host threads) race on the array and must be
 *     serialised by the caller.
 *   - Device-side errors (a bounded on-chip wait that gave up: that call's
 *     output is incomplete) are ORed into the array's flag word and stay
 *     there across calls until vc_draft_attn_quant_noalloc_flags() reads
 *     and clears them.
 *   - The array's address is cached per device for the life of the process:
 *     cudaDeviceReset() while the library is in use is not supported.
 *   - A call whose scratch would exceed VC_NOALLOC_SCRATCH_BYTES returns
 *     VC_ERR_WORKSPACE with a message and enqueues nothing. */
#define VC_NOALLOC_SCRATCH_BYTES (4u << 20)
VC_API vc_status vc_draft_attn_quant_noalloc(const vc_attn_shape* shape, const vc_quant_cache* cache,
                                             const void* q, float* out, void* stream);
/* Reads the VC_FLAG_* bits that vc_draft_attn_quant_noalloc calls on the
 * current device have set since the last read, writes them to *host_flags
 * (host memory) and clears them.  Enqueues the read and the clear on
 * `stream` and waits for that stream.  No counterpart in the pages; it is
 * the allocation-free path's version of vc_workspace_flags(). */
VC_API vc_status vc_draft_attn_quant_noalloc_flags(uint32_t* host_flags, void* stream);

/* ---- draft attention over a token-dropped cache ----------------------------
 * out[b][hq][:] = softmax(q . K[idx]^T * sm_scale) . V[idx] over the n_keep
 * kept rows of KV head hq / g.
 *   q    bf16 [B][Hq][D];  out fp32 [B][Hq][D]. */
VC_API size_t vc_draft_attn_sparse_workspace_size(const vc_attn_shape* shape, const vc_sparse_cache* cache);
VC_API vc_status vc_draft_attn_sparse(const vc_attn_shape* shape, const vc_sparse_cache* cache, const void* q,
                               float* out, void* ws, size_t ws_bytes, void* stream);

/* ---- building the compressed caches on the GPU -------------------------------
 * A compressor is known to the system only through the positions it drops and
 * the bit width it stores (menfem.com source page, "Key Contributions"); these
 * calls produce both kinds of draft cache from one layer's full bf16 cache.
 *
 * vc_quantize_cache: the oldest L_q rows of every (request, KV head) of
 * k, v (bf16 [B][Hkv][T][D]) become group records in the layout of
 * vc_quant_cache (records uint8 [B][Hkv][L_q / group][REC]), the newest
 * T - L_q rows are copied to rows 0 .. T - L_q - 1 of k_res, v_res (bf16
 * [B][Hkv][R_cap][D]).  Rule (the library's reading of KIVI-style
 * quantisation): per group s = fp16((max - min) / (2^bits - 1)) and
 * z = fp16(min), rounded to nearest even; code = clamp(rint((x - z) / s),
 * 0, 2^bits - 1) with the stored s and z, half to even, as an exact
 * division decides; s == 0 gives code 0.  The records equal the oracle's
 * byte for byte.  A scale or zero outside the fp16 range raises
 * VC_FLAG_RANGE in the workspace's flag word.  bits 2|4, group 32|64,
 * D 64|128, L_q a multiple of group, T - L_q <= R_cap.
 * vc_compact_kept: for each (request, KV head) the rows idx[..][j] of k, v
 * (bf16 [B][Hkv][T_store][D]) go to row j of k_out, v_out (bf16
 * [B][Hkv][n_keep][D]): the kept-row pool the token-dropped draft reads with
 * slots 0 .. n_keep - 1.  An index outside [0, T_store) writes a zero row and
 * raises VC_FLAG_BAD_INDEX (ws may be NULL).
 * Both need a workspace of vc_compress_workspace_size() bytes (a flag word,
 * zeroed once). */
VC_API size_t vc_compress_workspace_size(void);
VC_API vc_status vc_quantize_cache(const vc_attn_shape* shape, const void* k, const void* v, int64_t T, int bits,
                                   int group, int64_t L_q, void* records, void* k_res, void* v_res, int R_cap,
                                   void* ws, size_t ws_bytes, void* stream);
VC_API vc_status vc_compact_kept(const vc_attn_shape* shape, const void* k, const void* v, int64_t T_store,
                                 const int32_t* idx, int n_keep, void* k_out, void* v_out, void* ws,
                                 size_t ws_bytes, void* stream);

/* ---- cache maintenance around a round -----------------------------------------
 * After acceptance, a round keeps the accepted prefix plus the verifier's
 * correction and discards the rest of the draft (devshah.ca page, "The Core
 * Idea", the worked example's Emit / Discard lines).  The library's reading:
 * before a round the caches hold every committed token but the newest (x);
 * the verification block is (x, d_1 .. d_K), nq = K + 1 rows whose exact K, V
 * the verifier computes; with a = accept_len[b] the rows x, d_1 .. d_a
 * (a + 1 rows) are committed and d_(a+1) .. d_K rolled back.
 * vc_cache_commit appends those rows of k_new, v_new (bf16 [B][Hkv][nq][D],
 * this layer's block rows) to the bf16 residual of each request's quantised
 * cache; when the residual would exceed R_cap, its oldest `group` rows first
 * become one group record (vc_quantize_cache's rule, byte-identical to it)
 * at index L_q_b / group and the residual keeps the rest.  cache->lens (device
 * [B][2]) is required and is updated in place; accept_len is a device int32
 * [B] (vc_accept's output): nothing is read back to the host.  Needs
 * nq <= group and R_cap >= group + nq - 1.  A request with an accepted length
 * outside [0, nq), invalid lengths or no record capacity left is left
 * unchanged and raises VC_FLAG_BAD_LENGTH.  The full bf16 cache needs no data
 * movement: its committed length simply grows by a + 1.  Workspace: a flag
 * word of vc_compress_workspace_size() bytes. */
VC_API vc_status vc_cache_commit(const vc_attn_shape* shape, const vc_quant_cache* cache, const void* k_new,
                                 const void* v_new, int nq, const int32_t* accept_len, void* ws, size_t ws_bytes,
                                 void* stream);

/* ---- block verification attention -----------------------------------------
 * One pass over the full cache scores every drafted position at once and
 * yields one extra prediction past the last drafted token (devshah.ca page,
 * "The Core Idea").  Row i (0 <= i < nq) of
 * query head hq attends causally to keys 0 .. T - nq + i of KV head hq / g;
 * the block's own keys are the last nq rows of the cache.
 *   q    bf16 [B][nq][Hq][D]
 *   k, v bf16 [B][Hkv][T][D]   (HBM-resident or a staging buffer)
 *   out  fp32 [B][nq][Hq][D]
 *   lse  fp32 [B][nq][Hq] natural-log softmax denominators, or NULL
 *   1 <= nq <= 32, nq <= T < 2^31, g = Hq / Hkv <= 8, D = 64 or 128,
 *   B * Hkv <= 65535 (VC_ERR_INVALID_ARG otherwise).  q, k and v are read
 *   through TMA tensor maps encoded per call; a map the driver refuses
 *   returns VC_ERR_CUDA before any launch. */
VC_API size_t vc_verify_attn_workspace_size(const vc_attn_shape* shape, int64_t T, int nq);
VC_API vc_status vc_verify_attn(const vc_attn_shape* shape, const void* q, const void* k, const void* v, int64_t T,
                         int nq, float* out, float* lse, void* ws, size_t ws_bytes, void* stream);

/* ---- greedy acceptance -----------------------------------------------------
 * target[b][i] = argmax_v logits[b][i][v] for i = 0..K (lowest index wins a
 * tie, +0 and -0 tie, the first NaN counts as the maximum).  accept_len[b] =
 * the first i < K with draft[b][i] != target[b][i], or K when all match;
 * correction[b] = target[b][accept_len[b]] (the bonus token when all match).
 * The emitted run is draft[b][0 .. a-1] followed by correction[b]
 * (devshah.ca page, "The Core Idea": accept until the first mismatch, insert
 * the full-cache correction, keep the bonus token when everything matches).
 *   logits  fp32 or bf16 [B][K+1][V] (dtype VC_F32 or VC_BF16)
 *   draft   int32 [B][K]; target int32 [B][K+1];
 *   accept_len, correction int32 [B].   B >= 1, 0 <= K <= 64, V >= 1. */
VC_API size_t vc_accept_workspace_size(int B, int K, int V);
VC_API vc_status vc_accept(const void* logits, int dtype, int B, int K, int V, const int32_t* draft, int32_t* target,
                    int32_t* accept_len, int32_t* correction, void* ws, size_t ws_bytes, void* stream);

/* ---- host -> HBM streaming of the full KV for verification ----------------
 * The full cache may live in host memory and be brought to the GPU only for
 * verification (devshah.ca page, "Verifying Without Giving Back the
 * Speedup"; menfem.com source page, "Key Contributions": the verifier reads
 * the full KV from CPU memory over the interconnect).  A vc_kvstream moves one
 * layer at a time into one of two caller-owned device staging slots with
 * cudaMemcpyAsync on a copy stream, so the copy of layer l + 1 overlaps the
 * verification of layer l.  Layer l always uses slot l % 2.  Everything is
 * stream-ordered with events; no call blocks the host except destroy.
 *   host_k[l], host_v[l]  pinned host memory, bytes_per_layer each (caller-owned)
 *   dev_k[0..1], dev_v[0..1]  device staging slots, bytes_per_layer each
 *   copy_stream  the stream that carries the copies (caller-owned)
 * Protocol per layer l: prefetch(l) (enqueues the copies once the slot's
 * previous layer was released), acquire(l, compute) (the compute stream
 * waits for the copies; returns the slot's pointers), launch the work,
 * release(l, compute) (the slot may be overwritten after the work).  Calling
 * acquire on a layer that was not prefetched, or prefetch on a slot whose
 * previous layer was not yet released, returns VC_ERR_INVALID_ARG. */
typedef struct vc_kvstream vc_kvstream;
VC_API vc_status vc_kvstream_create(vc_kvstream** out, int n_layers, const void* const* host_k,
                                    const void* const* host_v, size_t bytes_per_layer, void* const* dev_k,
                                    void* const* dev_v, void* copy_stream);
VC_API vc_status vc_kvstream_prefetch(vc_kvstream* s, int layer);
VC_API vc_status vc_kvstream_acquire(vc_kvstream* s, int layer, void* compute_stream, const void** k,
                                     const void** v);
VC_API vc_status vc_kvstream_release(vc_kvstream* s, int layer, void* compute_stream);
VC_API vc_status vc_kvstream_destroy(vc_kvstream* s);

/* ---- one verifier decoder layer on caller-given weights --------------------
 * Verification is one pass of the same model over the drafted block with the
 * full cache (devshah.ca page, "The Core Idea"; drafter and verifier share
 * the weights, menfem.com source page, "Methodology").  vc_verify_layer runs
 * one Llama-style pre-norm decoder layer over the block:
 *   h = RMSNorm(x) w1; [q | k | v] = h Wqkv^T; rotary embedding (rotate-half
 *   pairs j, j + D/2, angle = position * rope_theta^(-2j/D)) of q and k at
 *   positions T - nq + i; the block's k and v written into the full cache
 *   rows T - nq .. T - 1; o = vc_verify_attn; x += o Wo^T;
 *   h2 = RMSNorm(x) w2; [g | u] = h2 Wgu^T; x += (silu(g) u) Wd^T.
 * Activations are bf16 between the steps (each step's result is rounded to
 * bf16 once); the projections are cuBLAS bf16 GEMMs with fp32 accumulation.
 *   x        bf16 [B][nq][d_model], read and overwritten with the layer output
 *   k_cache, v_cache  bf16 [B][Hkv][T][D] (full cache, resident); rows
 *            T - nq .. T - 1 are overwritten with the block's k and v
 *   weights  bf16 row-major [out][in]: w1, w2 [d_model]; wqkv
 *            [(Hq + 2 Hkv) D][d_model]; wo [d_model][Hq D]; wgu
 *            [2 d_ff][d_model] (gate rows, then up rows); wd [d_model][d_ff]
 * D in {64, 128}, Hq/Hkv <= 8, nq <= 32, d_model and d_ff multiples of 8,
 * every pointer 16-byte aligned.  The workspace (size from the query) also
 * holds cuBLAS's scratch.  Returns VC_ERR_INVALID_ARG on bad arguments
 * before any launch. */
typedef struct vc_layer_shape {
  int d_model, d_ff, Hq, Hkv, D;
  float rms_eps;     /* e.g. 1e-5 */
  float rope_theta;  /* e.g. 500000 */
} vc_layer_shape;
typedef struct vc_layer_weights {
  const void *w1, *wqkv, *wo, *w2, *wgu, *wd;
} vc_layer_weights;
VC_API size_t vc_verify_layer_workspace_size(const vc_layer_shape* shape, int B, int nq, int64_t T);
VC_API vc_status vc_verify_layer(const vc_layer_shape* shape, const vc_layer_weights* weights, int B, int nq,
                                 int64_t T, void* x, void* k_cache, void* v_cache, void* ws, size_t ws_bytes,
                                 void* stream);

/* ---- bandwidth-limited links ---------------------------------------------------
 * Remote prefix caching sends the compressed cache to the serving GPU over a
 * slow network while the full cache stays reachable over a fast local link
 * (menfem.com source page, "Key Contributions" (two deployment pipelines),
 * "Methodology": 1.2 GB/s remote against 40 GB/s local).  A vc_link emulates
 * a host -> device link of `gbps` GB/s on the GPU's own bus: copies run on
 * `stream` in chunks of chunk_bytes (0: 8 MiB), each released no sooner than
 * its size / gbps after the previous one started (a one-thread kernel sleeps
 * on the device clock; bounded at 60 s per chunk, after which it sets
 * VC_FLAG_WAIT_TIMEOUT and lets the copy proceed).  gbps == 0: unpaced.
 *   vc_link_copy   asynchronous host -> device copy on the link's stream
 *                  (src should be pinned host memory); returns at once.
 *   vc_link_flags  reads and clears the link's flag word (synchronous).
 *   vc_link_destroy waits for the link's stream, then frees the link.
 * The link allocates 64 bytes of device memory for its clock. */
typedef struct vc_link vc_link;
VC_API vc_status vc_link_create(vc_link** out, void* stream, double gbps, size_t chunk_bytes);
VC_API vc_status vc_link_copy(vc_link* link, void* dst, const void* src, size_t bytes);
VC_API vc_status vc_link_flags(vc_link* link, uint32_t* host_flags);
VC_API vc_status vc_link_destroy(vc_link* link);

/* ---- cross-request staggering scheduler -------------------------------------
 * Drafting is bound by HBM bandwidth and verification by the host link, so
 * the pages interleave different requests' draft and verify phases instead
 * of running all drafts and then all verifications (devshah.ca page,
 * "Verifying Without Giving Back the Speedup", Figure 2; menfem.com source
 * page, "Key Contributions").  vc_sched runs rounds for n requests:
 *   draft   draft_len x n_layers calls of the request's draft attention on the
 *           request's stream;
 *   verify  n_layers of host-streamed verification (vc_kvstream over the
 *           shared copy stream, kernels on the request's stream);
 *   accept  one vc_accept call.
 * VC_SCHED_LOCKSTEP: every request drafts, then (after all drafts) the
 * verifications run one after another; the next round starts when all are
 * done.  VC_SCHED_STAGGER: a request starts verifying as soon as its own
 * draft is done and the link is free, and starts its next round's draft as
 * soon as its own round is done, so one request's verification overlaps
 * other requests' drafting.  The host polls events (never blocks a device)
 * and gives up with VC_ERR_TIMEOUT once timeout_ms pass without progress
 * (no draft, verification or round of any request completing or starting);
 * a run that keeps progressing may last any time.  Inputs and outputs
 * of every call are the caller's (device pointers, as in the calls above);
 * the round's synthetic inputs do not change between rounds. */
#define VC_DRAFT_QUANT 0
#define VC_DRAFT_SPARSE 1
#define VC_SCHED_LOCKSTEP 0
#define VC_SCHED_STAGGER 1
typedef struct vc_sched_request {
  vc_attn_shape shape;               /* B, Hq, Hkv, D, sm_scale of the request */
  int draft_kind;                    /* VC_DRAFT_QUANT or VC_DRAFT_SPARSE */
  const vc_quant_cache* qcaches;     /* host array [n_layers] (quant) */
  const vc_sparse_cache* scaches;    /* host array [n_layers] (sparse) */
  const void* draft_q;               /* bf16 [draft_len][n_layers][B][Hq][D] */
  float* draft_out;                  /* fp32 [B][Hq][D] */
  void* draft_ws;
  size_t draft_ws_bytes;
  const void* const* host_k;         /* host array [n_layers] of pinned host pointers */
  const void* const* host_v;
  size_t kv_bytes_per_layer;         /* B * Hkv * T * D * 2 */
  void* stage_k[2];                  /* device staging slots, kv_bytes_per_layer each */
  void* stage_v[2];
  const void* verify_q;              /* bf16 [n_layers][B][nq][Hq][D] */
  float* verify_out;                 /* fp32 [B][nq][Hq][D] (last layer's result remains) */
  void* verify_ws;
  size_t verify_ws_bytes;
  int64_t T;
  int nq;
  const void* logits;                /* [B][draft_len + 1][V], dtype logits_dtype */
  int logits_dtype;
  int V;
  const int32_t* draft_tokens;       /* [B][draft_len] */
  int32_t* target;                   /* [B][draft_len + 1] */
  int32_t* accept_len;               /* [B] */
  int32_t* correction;               /* [B] */
  void* accept_ws;
  size_t accept_ws_bytes;
  void* stream;                      /* the request's compute stream */
} vc_sched_request;
typedef struct vc_sched_stats {
  double elapsed_ms;      /* device time from the first enqueued work to the last completion */
  double link_busy_ms;    /* device time the copy stream spent copying (verification streaming) */
  double draft_ms;        /* summed device time of the draft phases */
  double verify_ms;       /* summed device time of the verify + accept phases */
  int rounds;
  int requests;
  double fetch_ms;        /* summed device time of the requests' fetches over the remote link */
  double first_draft_ms;  /* device time from the start to the last request's first draft */
} vc_sched_stats;
typedef struct vc_sched vc_sched;
VC_API vc_status vc_sched_create(vc_sched** out, int n_requests, const vc_sched_request* reqs, int n_layers,
                                 int draft_len, int policy, void* copy_stream, int timeout_ms);
VC_API vc_status vc_sched_run_rounds(vc_sched* s, int n_rounds, vc_sched_stats* stats);
VC_API vc_status vc_sched_destroy(vc_sched* s);

/* Remote prefix caching (the pages' second deployment pipeline; see the
 * links above).  vc_sched_set_links paces the scheduler's transfers:
 *   remote_stream, remote_gbps  the link that fetches requests' compressed
 *                               caches (vc_sched_set_fetch); gbps 0: unpaced
 *   local_gbps                  the verification streaming on copy_stream
 *                               (0: unpaced, the bus's own speed)
 *   chunk_bytes                 pacing chunk (0: 8 MiB)
 * vc_sched_set_fetch gives request r a list of n host -> device copies
 * (src pinned host, dst device, bytes each; the arrays are copied) that
 * every vc_sched_run_rounds call performs over the remote link, in request
 * order, before r's first draft of that call.  VC_SCHED_STAGGER lets r draft
 * as soon as its own fetch is done (other requests' fetches continue on the
 * remote link while r drafts and verifies); VC_SCHED_LOCKSTEP starts the
 * first drafts only when every fetch is done.  Both return
 * VC_ERR_INVALID_ARG for bad arguments. */
VC_API vc_status vc_sched_set_links(vc_sched* s, void* remote_stream, double remote_gbps, double local_gbps,
                                    size_t chunk_bytes);
VC_API vc_status vc_sched_set_fetch(vc_sched* s, int request, int n, const void* const* src, void* const* dst,
                                    const size_t* bytes);

/* Host-only model of the same policy on a simulated timeline (no GPU): each
 * request's fetch takes fetch_ms of the remote link (fetch_ms may be NULL:
 * no fetches; fetches run one at a time in request order, all enqueued at
 * the start), its draft draft_ms of the GPU (drafts share the GPU one at a
 * time) and its verification verify_ms of the local link (one at a time).
 * Writes the finishing time of the last round to *makespan_ms.  A request
 * index `never_done` >= 0 makes that request's first verification never
 * complete, which exercises the timeout path (VC_ERR_TIMEOUT after
 * timeout_ms of simulated time without progress).  Used by the CPU tests
 * of the policy. */
VC_API vc_status vc_sched_simulate(int n_requests, int n_rounds, int policy, const double* fetch_ms,
                                   const double* draft_ms, const double* verify_ms, int never_done,
                                   double timeout_ms, double* makespan_ms);

/* ---- workspace flags -------------------------------------------------------
 * Copies the device-side flag word of a workspace to *host_flags and clears
 * it (a synchronous read on `stream`).  Returns VC_OK or VC_ERR_CUDA. */
VC_API vc_status vc_workspace_flags(void* ws, size_t ws_bytes, uint32_t* host_flags, void* stream);

/* ---- test exports ------------------------------------------------------------
 * vc_debug_dequant writes the dequantised L_q rows of every (request, head)
 * in natural [token][channel] order, extracting the codes with the same
 * word layout and masks the draft kernel uses:
 *   k_out, v_out fp32 [B][Hkv][L_q][D]   (R residual rows are not included)
 * vc_debug_gather writes the kept rows the sparse draft kernel reads:
 *   k_out, v_out bf16 [B][Hkv][n_keep][D]; out-of-range positions write
 *   zeros and raise VC_FLAG_BAD_INDEX in `ws` (which may be NULL). */
VC_API vc_status vc_debug_dequant(const vc_attn_shape* shape, const vc_quant_cache* cache, float* k_out, float* v_out,
                           void* stream);
VC_API vc_status vc_debug_gather(const vc_attn_shape* shape, const vc_sparse_cache* cache, void* k_out, void* v_out,
                          void* ws, size_t ws_bytes, void* stream);

/* vc_debug_wait_timeout runs the bounded on-chip wait every hot-path kernel
 * uses on an mbarrier that nothing ever completes, giving up after limit_ns
 * (1 us .. 100 ms): the wait must return, OR VC_FLAG_WAIT_TIMEOUT into
 * *flags (device uint32) and write 2 to *result (device uint32; 1 would mean
 * the wait completed).  The kernel ends normally and the context stays
 * usable; this is how the library's device-side failure path is tested
 * without faulting or hanging a GPU. */
VC_API vc_status vc_debug_wait_timeout(uint32_t* flags, uint32_t* result, int64_t limit_ns, void* stream);

/* vc_debug_verify_abort is vc_verify_attn with its failure path forced: in
 * every block the K tile with block-local index skip_tile (>= 0) is never
 * requested, and the tile loop's waits give up after limit_ns (1 us ..
 * 100 ms) instead of 2 s.  A block that has that tile stops: the wait on it
 * ORs VC_FLAG_WAIT_TIMEOUT into the workspace's flag word and raises the
 * block's abort flag, every other wait of the block then gives up, the
 * block drains its MMAs and copies, releases its tensor memory and returns;
 * its output rows are not valid.  Blocks with fewer tiles finish normally.
 * Same arguments and checks as vc_verify_attn otherwise.  Test only: it
 * shows a timed-out wait ending the kernel and leaving the context usable
 * without faulting or hanging a GPU. */
VC_API vc_status vc_debug_verify_abort(const vc_attn_shape* shape, const void* q, const void* k, const void* v,
                                       int64_t T, int nq, float* out, float* lse, void* ws, size_t ws_bytes,
                                       int skip_tile, int64_t limit_ns, void* stream);

/* vc_debug_quant_partition reports, without touching a GPU, how
 * vc_draft_attn_quant cuts one call into blocks when at most target_blocks
 * blocks are allowed (the real call uses SMs x resident blocks).  Each
 * (request, KV head) unit is an axis of *residual_tiles tiles of 16 residual
 * rows followed by *quant_stages quantised stages.  With
 * *blocks_per_unit >= 1 every unit is cut into that many contiguous pieces of
 * equal cost, one per block; with *blocks_per_unit == 0 (more units than
 * blocks) each block takes whole units.  Every unit ends up in
 * *partials_per_unit block partials.  block_ranges may be NULL; else it
 * needs max_blocks >= *n_blocks rows of six int32: first unit, end unit,
 * residual tiles [r0, r1) and quantised stages [q0, q1) of that block
 * (unit-local indices, the same for every unit of the block). */
VC_API vc_status vc_debug_quant_partition(const vc_attn_shape* shape, const vc_quant_cache* cache,
                                          int target_blocks, int32_t* block_ranges, int max_blocks, int* n_blocks,
                                          int* blocks_per_unit, int* partials_per_unit, int* residual_tiles,
                                          int* quant_stages);

#ifdef __cplusplus
}
#endif

#endif /* VC_H_ */
