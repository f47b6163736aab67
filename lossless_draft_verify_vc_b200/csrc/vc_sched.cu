// vc_sched.cu -- cross-request staggering of draft (HBM-bound) and verify
// (host-link-bound) phases.
//
// The pages observe that drafting from the compressed cache is limited by HBM
// bandwidth while verifying against the full cache is limited by the
// CPU-GPU link, and interleave the phases of different requests instead of
// running all drafts and then all verifications ("VeriCache: making lossy KV
// compression exact", devshah.ca, section "Verifying Without Giving Back the
// Speedup" and its Figure 2; "VeriCache: Turning Lossy KV Cache into Lossless
// LLM Inference", menfem.com, "Key Contributions").
//
// Remote prefix caching adds a third resource: a request's compressed cache
// first arrives over a slow remote link, and only then can it draft, while
// verification streams the full cache over the fast local link (menfem.com,
// "Key Contributions", the two deployment pipelines).  Fetches run one at a
// time on the remote link in request order; staggering lets a fetched
// request draft and verify while later requests are still arriving.
//
// The policy below is written once against a small Backend interface.  The
// CUDA backend enqueues the real work (draft launches on the request's
// stream, host-streamed verification over the shared copy stream, acceptance)
// and answers completion queries with cudaEventQuery -- the host polls and
// never blocks a device.  The simulated backend replays the same policy on a
// virtual clock (GPU and link as one-at-a-time servers); it backs
// vc_sched_simulate, which the host-only tests use.
#include <chrono>
#include <deque>
#include <memory>
#include <thread>
#include <vector>

#include "vc_kvstream.h"

namespace vc {
namespace sched {

struct Backend {
  virtual ~Backend() = default;
  virtual bool has_fetch(int r) { (void)r; return false; }
  virtual vc_status enqueue_fetch(int r) { (void)r; return VC_OK; }  // over the remote link, in call order
  virtual int fetch_done(int r) { (void)r; return 1; }
  virtual vc_status enqueue_draft(int r) = 0;
  virtual vc_status enqueue_verify(int r) = 0;  // verification + acceptance of the round
  virtual int draft_done(int r) = 0;             // 1 done, 0 pending, < 0 error
  virtual int round_done(int r) = 0;
  virtual void on_round_done(int r) { (void)r; }
  virtual double now_ms() = 0;
  virtual void idle() = 0;
};

enum Phase { kFetching, kIdle, kDrafting, kReady, kVerifying, kFinished };

// Runs n_rounds rounds for n requests, each first fetching its compressed
// cache if it has a fetch list (all fetches are enqueued at the start, in
// request order, on the remote link).
//   LOCKSTEP: round k's drafts start only when every request finished round
//   k - 1 (for k = 0: when every fetch is done); verifications start only
//   when no request is still drafting.
//   STAGGER: a request drafts as soon as its fetch or previous round is done
//   and verifies as soon as its draft is done and the link is free.
// In both, one verification holds the link at a time (first ready, first
// served).  timeout_ms bounds the time WITHOUT progress (no phase of any
// request changed): a long run that keeps completing phases never times out,
// one whose outstanding work stops completing fails after timeout_ms.
vc_status run_policy(Backend& be, int n, int n_rounds, int policy, double timeout_ms) {
  std::vector<Phase> ph(n, kIdle);
  std::vector<int> rnd(n, 0);
  std::deque<int> ready;
  int link_owner = -1;
  int finished = 0;
  double t_progress = be.now_ms();
  if (n_rounds <= 0) return VC_OK;
  for (int r = 0; r < n; ++r)
    if (be.has_fetch(r)) {
      vc_status st = be.enqueue_fetch(r);
      if (st != VC_OK) return st;
      ph[r] = kFetching;
    }
  while (finished < n) {
    bool progressed = false;
    for (int r = 0; r < n; ++r) {
      if (ph[r] == kFetching) {
        const int q = be.fetch_done(r);
        if (q < 0) return set_error(VC_ERR_CUDA, "vc_sched: fetch of request %d failed", r);
        if (q > 0) {
          ph[r] = kIdle;
          progressed = true;
        }
      }
      if (ph[r] == kIdle) {
        bool allowed = true;
        if (policy == VC_SCHED_LOCKSTEP)
          for (int o = 0; o < n; ++o)
            if (ph[o] != kFinished && (rnd[o] != rnd[r] || (ph[o] != kIdle && ph[o] != kDrafting))) allowed = false;
        if (allowed) {
          vc_status st = be.enqueue_draft(r);
          if (st != VC_OK) return st;
          ph[r] = kDrafting;
          progressed = true;
        }
      }
      if (ph[r] == kDrafting) {
        const int q = be.draft_done(r);
        if (q < 0) return set_error(VC_ERR_CUDA, "vc_sched: draft of request %d failed", r);
        if (q > 0) {
          ph[r] = kReady;
          ready.push_back(r);
          progressed = true;
        }
      }
      if (ph[r] == kVerifying) {
        const int q = be.round_done(r);
        if (q < 0) return set_error(VC_ERR_CUDA, "vc_sched: verification of request %d failed", r);
        if (q > 0) {
          be.on_round_done(r);
          if (link_owner == r) link_owner = -1;
          if (++rnd[r] >= n_rounds) {
            ph[r] = kFinished;
            ++finished;
          } else {
            ph[r] = kIdle;
          }
          progressed = true;
        }
      }
    }
    if (link_owner < 0 && !ready.empty()) {
      bool allowed = true;
      if (policy == VC_SCHED_LOCKSTEP)
        for (int o = 0; o < n; ++o)
          if (ph[o] == kDrafting) allowed = false;
      if (allowed) {
        const int r = ready.front();
        ready.pop_front();
        vc_status st = be.enqueue_verify(r);
        if (st != VC_OK) return st;
        ph[r] = kVerifying;
        link_owner = r;
        progressed = true;
      }
    }
    if (progressed) {
      t_progress = be.now_ms();
    } else {
      if (be.now_ms() - t_progress > timeout_ms)
        return set_error(VC_ERR_TIMEOUT, "vc_sched: no progress within %.0f ms", timeout_ms);
      be.idle();
    }
  }
  return VC_OK;
}

// ------------------------------------------------------------ simulated backend
struct SimBackend final : Backend {
  int n;
  std::vector<double> fetch_ms, draft_ms, verify_ms;
  int never_done;
  double t = 0, gpu_free = 0, link_free = 0, remote_free = 0;
  std::vector<double> fetch_end, draft_end, round_end;
  std::vector<int> verifies;
  double makespan = 0;
  SimBackend(int n_, const double* f, const double* d, const double* v, int nd)
      : n(n_), fetch_ms(f ? std::vector<double>(f, f + n_) : std::vector<double>()), draft_ms(d, d + n_),
        verify_ms(v, v + n_), never_done(nd), fetch_end(n_, 0), draft_end(n_, 0), round_end(n_, 0),
        verifies(n_, 0) {}
  bool has_fetch(int r) override { return !fetch_ms.empty() && fetch_ms[r] > 0; }
  vc_status enqueue_fetch(int r) override {
    const double start = std::max(t, remote_free);
    fetch_end[r] = start + fetch_ms[r];
    remote_free = fetch_end[r];
    return VC_OK;
  }
  int fetch_done(int r) override { return t >= fetch_end[r] ? 1 : 0; }
  vc_status enqueue_draft(int r) override {
    const double start = std::max(t, gpu_free);
    draft_end[r] = start + draft_ms[r];
    gpu_free = draft_end[r];
    return VC_OK;
  }
  vc_status enqueue_verify(int r) override {
    const double start = std::max(std::max(t, link_free), draft_end[r]);
    const bool stuck = (r == never_done && verifies[r] == 0);
    round_end[r] = stuck ? 1e300 : start + verify_ms[r];
    link_free = round_end[r];
    ++verifies[r];
    return VC_OK;
  }
  int draft_done(int r) override { return t >= draft_end[r] ? 1 : 0; }
  int round_done(int r) override { return t >= round_end[r] ? 1 : 0; }
  void on_round_done(int r) override { makespan = std::max(makespan, round_end[r]); }
  double now_ms() override { return t; }
  void idle() override {
    double next = 1e300;
    for (int r = 0; r < n; ++r) {
      if (fetch_end[r] > t) next = std::min(next, fetch_end[r]);
      if (draft_end[r] > t) next = std::min(next, draft_end[r]);
      if (round_end[r] > t) next = std::min(next, round_end[r]);
    }
    t = next < 1e299 ? next : t + 1.0;
  }
};

// ----------------------------------------------------------------- CUDA backend
struct RequestState {
  vc_sched_request req;
  std::vector<vc_quant_cache> qc;
  std::vector<vc_sparse_cache> sc;
  std::vector<const void*> hk, hv;
  std::unique_ptr<KvStream> ks;
  cudaEvent_t ev_draft0 = nullptr, ev_draft1 = nullptr, ev_ver0 = nullptr, ev_round1 = nullptr;
  cudaEvent_t ev_fetch0 = nullptr, ev_fetch1 = nullptr, ev_first = nullptr;
  std::vector<cudaEvent_t> copy_t0, copy_t1;
  // the compressed cache's copies over the remote link (remote prefix caching)
  std::vector<const void*> fetch_src;
  std::vector<void*> fetch_dst;
  std::vector<size_t> fetch_bytes;
  bool first_draft = true;  // the call's first draft waits for the fetch and stamps ev_first
};

struct CudaBackend final : Backend {
  int n_layers = 0, draft_len = 0;
  cudaStream_t copy_stream = nullptr;
  std::vector<std::unique_ptr<RequestState>> rs;
  std::unique_ptr<PacedLink> remote, local;  // optional links (vc_sched_set_links)
  cudaEvent_t ev_begin = nullptr;
  bool begun = false;
  double draft_ms = 0, verify_ms = 0, link_ms = 0, fetch_ms = 0;
  std::chrono::steady_clock::time_point clock0 = std::chrono::steady_clock::now();

  ~CudaBackend() override {
    for (auto& r : rs) {
      r->ks.reset();  // before the local link it may copy through
      for (cudaEvent_t e : {r->ev_draft0, r->ev_draft1, r->ev_ver0, r->ev_round1, r->ev_fetch0, r->ev_fetch1,
                            r->ev_first})
        if (e) cudaEventDestroy(e);
      for (auto e : r->copy_t0) cudaEventDestroy(e);
      for (auto e : r->copy_t1) cudaEventDestroy(e);
    }
    if (ev_begin) cudaEventDestroy(ev_begin);
  }

  bool has_fetch(int i) override { return !rs[i]->fetch_src.empty(); }
  vc_status enqueue_fetch(int i) override {
    RequestState& r = *rs[i];
    if (!remote) return set_error(VC_ERR_INVALID_ARG, "vc_sched: request %d has a fetch but no remote link", i);
    if (!begun) {
      cudaEventRecord(ev_begin, remote->stream);
      begun = true;
    }
    cudaEventRecord(r.ev_fetch0, remote->stream);
    for (size_t k = 0; k < r.fetch_src.size(); ++k) {
      vc_status st = remote->copy(r.fetch_dst[k], r.fetch_src[k], r.fetch_bytes[k]);
      if (st != VC_OK) return st;
    }
    if (cudaEventRecord(r.ev_fetch1, remote->stream) != cudaSuccess)
      return set_error(VC_ERR_CUDA, "vc_sched: event record failed");
    return VC_OK;
  }
  int fetch_done(int i) override {
    const int q = query(rs[i]->ev_fetch1);
    if (q > 0) {
      float ms = 0;
      if (cudaEventElapsedTime(&ms, rs[i]->ev_fetch0, rs[i]->ev_fetch1) == cudaSuccess) fetch_ms += ms;
    }
    return q;
  }

  vc_status enqueue_draft(int i) override {
    RequestState& r = *rs[i];
    const vc_sched_request& q = r.req;
    cudaStream_t s = static_cast<cudaStream_t>(q.stream);
    if (!begun) {
      cudaEventRecord(ev_begin, s);
      begun = true;
    }
    if (r.first_draft) {
      // the cache this draft reads arrived over the remote link
      if (!r.fetch_src.empty() && cudaStreamWaitEvent(s, r.ev_fetch1, 0) != cudaSuccess)
        return set_error(VC_ERR_CUDA, "vc_sched: wait for the fetch failed");
      cudaEventRecord(r.ev_first, s);
      r.first_draft = false;
    }
    cudaEventRecord(r.ev_draft0, s);
    const size_t qstride = static_cast<size_t>(q.shape.B) * q.shape.Hq * q.shape.D;  // elements per (step, layer)
    const auto* qbase = static_cast<const uint16_t*>(q.draft_q);
    for (int t = 0; t < draft_len; ++t)
      for (int l = 0; l < n_layers; ++l) {
        const void* qp = qbase + (static_cast<size_t>(t) * n_layers + l) * qstride;
        vc_status st = q.draft_kind == VC_DRAFT_QUANT
                           ? vc_draft_attn_quant(&q.shape, &r.qc[l], qp, q.draft_out, q.draft_ws, q.draft_ws_bytes, s)
                           : vc_draft_attn_sparse(&q.shape, &r.sc[l], qp, q.draft_out, q.draft_ws,
                                                  q.draft_ws_bytes, s);
        if (st != VC_OK) return st;
      }
    if (cudaEventRecord(r.ev_draft1, s) != cudaSuccess)
      return set_error(VC_ERR_CUDA, "vc_sched: event record failed");
    return VC_OK;
  }

  vc_status enqueue_verify(int i) override {
    RequestState& r = *rs[i];
    const vc_sched_request& q = r.req;
    cudaStream_t s = static_cast<cudaStream_t>(q.stream);
    cudaEventRecord(r.ev_ver0, s);
    const size_t qstride = static_cast<size_t>(q.shape.B) * q.nq * q.shape.Hq * q.shape.D;
    const auto* qbase = static_cast<const uint16_t*>(q.verify_q);
    vc_status st = r.ks->prefetch(0, r.copy_t0[0], r.copy_t1[0]);
    if (st == VC_OK && n_layers > 1) st = r.ks->prefetch(1, r.copy_t0[1], r.copy_t1[1]);
    for (int l = 0; l < n_layers && st == VC_OK; ++l) {
      const void *k = nullptr, *v = nullptr;
      st = r.ks->acquire(l, s, &k, &v);
      if (st == VC_OK)
        st = vc_verify_attn(&q.shape, qbase + l * qstride, k, v, q.T, q.nq, q.verify_out, nullptr, q.verify_ws,
                            q.verify_ws_bytes, s);
      if (st == VC_OK) st = r.ks->release(l, s);
      if (st == VC_OK && l + 2 < n_layers) st = r.ks->prefetch(l + 2, r.copy_t0[l + 2], r.copy_t1[l + 2]);
    }
    if (st == VC_OK)
      st = vc_accept(q.logits, q.logits_dtype, q.shape.B, draft_len, q.V, q.draft_tokens, q.target, q.accept_len,
                     q.correction, q.accept_ws, q.accept_ws_bytes, s);
    if (st != VC_OK) return st;
    if (cudaEventRecord(r.ev_round1, s) != cudaSuccess)
      return set_error(VC_ERR_CUDA, "vc_sched: event record failed");
    return VC_OK;
  }

  static int query(cudaEvent_t e) {
    const cudaError_t q = cudaEventQuery(e);
    if (q == cudaSuccess) return 1;
    if (q == cudaErrorNotReady) return 0;
    return -1;
  }
  int draft_done(int i) override {
    const int q = query(rs[i]->ev_draft1);
    if (q > 0) {
      float ms = 0;
      cudaEventElapsedTime(&ms, rs[i]->ev_draft0, rs[i]->ev_draft1);
      draft_ms += ms;
    }
    return q;
  }
  int round_done(int i) override { return query(rs[i]->ev_round1); }
  void on_round_done(int i) override {
    RequestState& r = *rs[i];
    float ms = 0;
    cudaEventElapsedTime(&ms, r.ev_ver0, r.ev_round1);
    verify_ms += ms;
    for (int l = 0; l < n_layers; ++l) {
      float c = 0;
      if (cudaEventElapsedTime(&c, r.copy_t0[l], r.copy_t1[l]) == cudaSuccess) link_ms += c;
    }
  }
  double now_ms() override {
    return std::chrono::duration<double, std::milli>(std::chrono::steady_clock::now() - clock0).count();
  }
  void idle() override { std::this_thread::sleep_for(std::chrono::microseconds(20)); }
};

}  // namespace sched

struct Sched {
  sched::CudaBackend be;
  int policy = VC_SCHED_STAGGER;
  double timeout_ms = 60000;
};

}  // namespace vc

extern "C" {

vc_status vc_sched_create(vc_sched** out, int n_requests, const vc_sched_request* reqs, int n_layers, int draft_len,
                          int policy, void* copy_stream, int timeout_ms) {
  VC_REQUIRE(out && reqs, "vc_sched_create: null argument");
  VC_REQUIRE(n_requests >= 1 && n_layers >= 1 && draft_len >= 0 && draft_len <= 64,
             "vc_sched_create: need n_requests >= 1, n_layers >= 1, 0 <= draft_len <= 64");
  VC_REQUIRE(policy == VC_SCHED_LOCKSTEP || policy == VC_SCHED_STAGGER, "vc_sched_create: unknown policy %d", policy);
  VC_REQUIRE(timeout_ms > 0, "vc_sched_create: timeout must be positive");
  for (int i = 0; i < n_requests; ++i) {
    const vc_sched_request& q = reqs[i];
    VC_REQUIRE(q.draft_kind == VC_DRAFT_QUANT ? q.qcaches != nullptr : (q.draft_kind == VC_DRAFT_SPARSE && q.scaches),
               "vc_sched_create: request %d has no draft caches for its kind", i);
    VC_REQUIRE(q.host_k && q.host_v && q.stage_k[0] && q.stage_k[1] && q.stage_v[0] && q.stage_v[1],
               "vc_sched_create: request %d lacks host KV or staging slots", i);
    VC_REQUIRE(q.kv_bytes_per_layer == static_cast<size_t>(q.shape.B) * q.shape.Hkv * q.T * q.shape.D * 2,
               "vc_sched_create: request %d: kv_bytes_per_layer must equal B*Hkv*T*D*2", i);
    VC_REQUIRE(q.draft_q && q.draft_out && q.verify_q && q.verify_out && q.logits && q.target && q.accept_len &&
                   q.correction && (draft_len == 0 || q.draft_tokens),
               "vc_sched_create: request %d has a null input or output", i);
  }
  auto* s = new vc::Sched();
  s->policy = policy;
  s->timeout_ms = timeout_ms;
  auto& be = s->be;
  be.n_layers = n_layers;
  be.draft_len = draft_len;
  be.copy_stream = static_cast<cudaStream_t>(copy_stream);
  bool ok = cudaEventCreate(&be.ev_begin) == cudaSuccess;
  for (int i = 0; i < n_requests && ok; ++i) {
    auto r = std::make_unique<vc::sched::RequestState>();
    r->req = reqs[i];
    if (reqs[i].draft_kind == VC_DRAFT_QUANT)
      r->qc.assign(reqs[i].qcaches, reqs[i].qcaches + n_layers);
    else
      r->sc.assign(reqs[i].scaches, reqs[i].scaches + n_layers);
    r->ks = std::make_unique<vc::KvStream>();
    void* dk[2] = {reqs[i].stage_k[0], reqs[i].stage_k[1]};
    void* dv[2] = {reqs[i].stage_v[0], reqs[i].stage_v[1]};
    ok = r->ks->init(n_layers, reqs[i].host_k, reqs[i].host_v, reqs[i].kv_bytes_per_layer, dk, dv,
                     be.copy_stream) == VC_OK;
    for (cudaEvent_t* e : {&r->ev_draft0, &r->ev_draft1, &r->ev_ver0, &r->ev_round1, &r->ev_fetch0, &r->ev_fetch1,
                           &r->ev_first})
      ok = ok && cudaEventCreate(e) == cudaSuccess;
    r->copy_t0.assign(n_layers, nullptr);
    r->copy_t1.assign(n_layers, nullptr);
    for (int l = 0; l < n_layers && ok; ++l)
      ok = cudaEventCreate(&r->copy_t0[l]) == cudaSuccess && cudaEventCreate(&r->copy_t1[l]) == cudaSuccess;
    be.rs.push_back(std::move(r));
  }
  if (!ok) {
    delete s;
    return vc::set_error(VC_ERR_CUDA, "vc_sched_create: could not create events");
  }
  *out = reinterpret_cast<vc_sched*>(s);
  vc::clear_error();
  return VC_OK;
}

vc_status vc_sched_run_rounds(vc_sched* sp, int n_rounds, vc_sched_stats* stats) {
  VC_REQUIRE(sp && n_rounds >= 0, "vc_sched_run_rounds: null scheduler or negative round count");
  auto* s = reinterpret_cast<vc::Sched*>(sp);
  auto& be = s->be;
  be.begun = false;
  be.draft_ms = be.verify_ms = be.link_ms = 0;
  be.clock0 = std::chrono::steady_clock::now();
  const int n = static_cast<int>(be.rs.size());
  be.fetch_ms = 0;
  for (auto& r : be.rs) r->first_draft = true;
  vc_status st = vc::sched::run_policy(be, n, n_rounds, s->policy, s->timeout_ms);
  if (st != VC_OK) return st;
  if (stats) {
    stats->rounds = n_rounds;
    stats->requests = n;
    stats->draft_ms = be.draft_ms;
    stats->verify_ms = be.verify_ms;
    stats->link_busy_ms = be.link_ms;
    stats->fetch_ms = be.fetch_ms;
    stats->elapsed_ms = 0;
    stats->first_draft_ms = 0;
    for (auto& r : be.rs) {
      float ms = 0;
      if (n_rounds > 0 && cudaEventElapsedTime(&ms, be.ev_begin, r->ev_round1) == cudaSuccess)
        stats->elapsed_ms = std::max(stats->elapsed_ms, static_cast<double>(ms));
      if (n_rounds > 0 && cudaEventElapsedTime(&ms, be.ev_begin, r->ev_first) == cudaSuccess)
        stats->first_draft_ms = std::max(stats->first_draft_ms, static_cast<double>(ms));
    }
  }
  vc::clear_error();
  return VC_OK;
}

vc_status vc_sched_destroy(vc_sched* sp) {
  if (!sp) return VC_OK;
  auto* s = reinterpret_cast<vc::Sched*>(sp);
  cudaError_t e = cudaSuccess;
  for (auto& r : s->be.rs) {
    const cudaError_t e1 = cudaStreamSynchronize(static_cast<cudaStream_t>(r->req.stream));
    if (e1 != cudaSuccess) e = e1;
  }
  const cudaError_t e2 = cudaStreamSynchronize(s->be.copy_stream);
  if (e2 != cudaSuccess) e = e2;
  delete s;
  if (e != cudaSuccess) return vc::set_error(VC_ERR_CUDA, "vc_sched_destroy: %s", cudaGetErrorString(e));
  vc::clear_error();
  return VC_OK;
}

vc_status vc_sched_set_links(vc_sched* sp, void* remote_stream, double remote_gbps, double local_gbps,
                             size_t chunk_bytes) {
  VC_REQUIRE(sp, "vc_sched_set_links: null scheduler");
  VC_REQUIRE(remote_gbps >= 0 && remote_gbps <= 1e4 && local_gbps >= 0 && local_gbps <= 1e4,
             "vc_sched_set_links: rates must be in [0, 1e4] GB/s");
  VC_REQUIRE(chunk_bytes == 0 || (chunk_bytes >= 4096 && chunk_bytes <= (size_t(1) << 32)),
             "vc_sched_set_links: chunk must be 0 (default 8 MiB) or 4 KiB .. 4 GiB");
  auto& be = reinterpret_cast<vc::Sched*>(sp)->be;
  for (auto& r : be.rs) r->ks->link = nullptr;
  be.remote.reset();
  be.local.reset();
  be.remote = std::make_unique<vc::PacedLink>();
  vc_status st = be.remote->init(static_cast<cudaStream_t>(remote_stream), remote_gbps, chunk_bytes);
  if (st != VC_OK) {
    be.remote.reset();
    return st;
  }
  if (local_gbps > 0) {
    be.local = std::make_unique<vc::PacedLink>();
    st = be.local->init(be.copy_stream, local_gbps, chunk_bytes);
    if (st != VC_OK) {
      be.local.reset();
      return st;
    }
    for (auto& r : be.rs) r->ks->link = be.local.get();
  }
  vc::clear_error();
  return VC_OK;
}

vc_status vc_sched_set_fetch(vc_sched* sp, int request, int n, const void* const* src, void* const* dst,
                             const size_t* bytes) {
  VC_REQUIRE(sp, "vc_sched_set_fetch: null scheduler");
  auto& be = reinterpret_cast<vc::Sched*>(sp)->be;
  VC_REQUIRE(request >= 0 && request < static_cast<int>(be.rs.size()), "vc_sched_set_fetch: request %d out of range",
             request);
  VC_REQUIRE(n >= 0 && (n == 0 || (src && dst && bytes)), "vc_sched_set_fetch: null list");
  for (int k = 0; k < n; ++k)
    VC_REQUIRE(src[k] && dst[k] && bytes[k] > 0, "vc_sched_set_fetch: copy %d is empty or null", k);
  auto& r = *be.rs[request];
  r.fetch_src.assign(src, src + n);
  r.fetch_dst.assign(dst, dst + n);
  r.fetch_bytes.assign(bytes, bytes + n);
  vc::clear_error();
  return VC_OK;
}

vc_status vc_sched_simulate(int n_requests, int n_rounds, int policy, const double* fetch_ms, const double* draft_ms,
                            const double* verify_ms, int never_done, double timeout_ms, double* makespan_ms) {
  VC_REQUIRE(n_requests >= 1 && n_rounds >= 0 && draft_ms && verify_ms && makespan_ms && timeout_ms > 0,
             "vc_sched_simulate: invalid argument");
  VC_REQUIRE(policy == VC_SCHED_LOCKSTEP || policy == VC_SCHED_STAGGER, "vc_sched_simulate: unknown policy %d",
             policy);
  for (int i = 0; i < n_requests; ++i)
    VC_REQUIRE(draft_ms[i] >= 0 && verify_ms[i] >= 0 && (!fetch_ms || fetch_ms[i] >= 0),
               "vc_sched_simulate: durations must be non-negative");
  vc::sched::SimBackend be(n_requests, fetch_ms, draft_ms, verify_ms, never_done);
  vc_status st = vc::sched::run_policy(be, n_requests, n_rounds, policy, timeout_ms);
  *makespan_ms = be.makespan;
  if (st == VC_OK) vc::clear_error();
  return st;
}

}  // extern "C"
