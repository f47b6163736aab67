"""Seeded synthetic inputs for tests and the benchmark.

This module only draws random tensors with the shapes and distributions of
the workloads (random KV rows, queries, kept-position lists, draft tokens,
logits with a planted argmax, random quantised caches for throughput runs).
It holds none of the method's arithmetic: no quantisation rule, no attention,
no acceptance.  Both the CUDA-path tests and the oracle-side tests draw their
inputs from here; the oracle never imports the CUDA path and vice versa.

Every generator takes an explicit ``seed`` and ``device`` and is
deterministic for a given (seed, device).  Inputs drawn on the GPU (for the
full-size benchmark) differ from CPU draws of the same seed; a test that
compares with the oracle always copies the exact GPU tensors to the host.
"""

from __future__ import annotations

import torch


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed) & 0x7FFFFFFFFFFFFFFF)
    return g


def normal(shape, seed: int, device="cpu", dtype=torch.bfloat16) -> torch.Tensor:
    """~N(0, 1), rounded to ``dtype``."""
    g = _gen(seed, device)
    return torch.randn(shape, generator=g, device=device, dtype=torch.float32).to(dtype)


def kv_full(B: int, Hkv: int, T: int, D: int, seed: int, device="cpu", key_outliers: bool = True,
            dtype=torch.bfloat16):
    """Full bf16 KV for one layer, [B, Hkv, T, D] each.

    Values ~N(0, 1).  Keys ~N(0, 1) times a per-(request, head, channel)
    multiplier exp(N(0, 1)) when ``key_outliers`` (lognormal channel
    outliers, the structure that motivates per-channel key groups)."""
    g = _gen(seed, device)
    k = torch.randn((B, Hkv, T, D), generator=g, device=device, dtype=torch.float32)
    if key_outliers:
        mult = torch.exp(torch.randn((B, Hkv, 1, D), generator=g, device=device, dtype=torch.float32))
        k = k * mult
    v = torch.randn((B, Hkv, T, D), generator=g, device=device, dtype=torch.float32)
    return k.to(dtype), v.to(dtype)


def kept_positions(B: int, Hkv: int, T: int, n_keep: int, seed: int, device="cpu") -> torch.Tensor:
    """Token-drop kept positions: top-n_keep of U(0, 1) scores per (request,
    head), sorted ascending, int32 [B, Hkv, n_keep].  Every head keeps the
    same count."""
    if not 0 < n_keep <= T:
        raise ValueError("need 0 < n_keep <= T")
    g = _gen(seed, device)
    scores = torch.rand((B, Hkv, T), generator=g, device=device)
    idx = torch.topk(scores, n_keep, dim=-1, sorted=False).indices
    return torch.sort(idx, dim=-1).values.to(torch.int32)


def tokens(shape, vocab: int, seed: int, device="cpu") -> torch.Tensor:
    g = _gen(seed, device)
    return torch.randint(0, vocab, shape, generator=g, device=device, dtype=torch.int64).to(torch.int32)


def geometric_accept_lengths(B: int, K: int, p_mismatch: float, seed: int) -> list:
    """Accepted-prefix lengths: each drafted position mismatches with
    probability p_mismatch independently, capped at K (host ints)."""
    g = _gen(seed, "cpu")
    u = torch.rand((B, K), generator=g)
    out = []
    for b in range(B):
        a = 0
        while a < K and float(u[b, a]) >= p_mismatch:
            a += 1
        out.append(a)
    return out


def planted_logits(B: int, K: int, V: int, draft: torch.Tensor, accept_lens, seed: int,
                   device="cpu", dtype=torch.float32) -> torch.Tensor:
    """Logits [B, K + 1, V] with a planted unique argmax: rows i < a_b peak at
    draft[b, i], row a_b (when a_b < K) peaks at a token different from
    draft[b, a_b]; other rows are noise.  Noise ~N(0, 1); a planted peak is
    max(noise) + 1, exactly representable in bf16 for these magnitudes."""
    g = _gen(seed, device)
    x = torch.randn((B, K + 1, V), generator=g, device=device, dtype=torch.float32).to(dtype)
    draft_h = draft.detach().to("cpu", torch.int64)
    alt = torch.randint(1, max(V, 2), (B,), generator=_gen(seed + 1, "cpu")).tolist()
    for b in range(B):
        a = int(accept_lens[b])
        for i in range(min(a, K)):
            t = int(draft_h[b, i])
            x[b, i, t] = (x[b, i].float().max() + 1.0).to(dtype)
        if a < K and V > 1:
            t = (int(draft_h[b, a]) + int(alt[b])) % V
            if t == int(draft_h[b, a]):
                t = (t + 1) % V
            x[b, a, t] = (x[b, a].float().max() + 1.0).to(dtype)
    return x


def random_quant_cache(B: int, Hkv: int, L_q: int, R_cap: int, D: int, bits: int, group: int,
                       seed: int, device="cpu") -> dict:
    """A quantised cache drawn directly in compressed form for throughput runs:
    group records (the library's descriptor layout: two code blocks of
    group * D * bits / 8 uniform random bytes, then four parameter rows of D
    fp16 each -- key scales, key zeros, value scales, value zeros), scales
    ~U(0.05, 1.5), zeros ~U(-3, -0.5) (magnitudes of 2/4-bit groups of N(0, 1)
    data), bf16 residual ~N(0, 1)."""
    g = _gen(seed, device)
    ng = L_q // group
    cb = group * D * bits // 8

    def u(shape, lo, hi):
        return (torch.rand(shape, generator=g, device=device) * (hi - lo) + lo).to(torch.float16)

    codes = torch.randint(0, 256, (B, Hkv, ng, 2 * cb), generator=g, device=device, dtype=torch.int32)
    params = torch.cat([u((B, Hkv, ng, D), 0.05, 1.5), u((B, Hkv, ng, D), -3.0, -0.5),
                        u((B, Hkv, ng, D), 0.05, 1.5), u((B, Hkv, ng, D), -3.0, -0.5)], dim=-1)
    records = torch.cat([codes.to(torch.uint8), params.view(torch.uint8)], dim=-1).contiguous()
    return dict(
        bits=bits, group=group, L_q=L_q, R=R_cap, R_cap=R_cap, D=D, records=records,
        k_res=normal((B, Hkv, R_cap, D), seed + 11, device),
        v_res=normal((B, Hkv, R_cap, D), seed + 12, device),
    )
