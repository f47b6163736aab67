"""The work partition of vc_draft_attn_quant, checked on the CPU through
vc_debug_quant_partition (no GPU call).  Each (request, KV head) unit is an
axis of residual tiles (16 rows each) followed by quantised stages; the call
either cuts every unit into the same number of contiguous, cost-balanced,
non-empty pieces (one per block) or gives each block whole units.  Checked:
every tile and stage of every unit is covered exactly once, the pieces'
costs are balanced, and the reported partials per unit match the pieces
that hold residual tiles plus the pieces that hold quantised stages."""

import pytest

from lossless_draft_verify_vc_b200 import build as B
from lossless_draft_verify_vc_b200 import vc


@pytest.fixture(scope="module", autouse=True)
def _lib():
    B.build()
    vc.lib()


def _cache(bits, G, L_q, R):
    qc = vc.vc_quant_cache()
    qc.records = 16 if L_q else None
    qc.k_res = qc.v_res = 16 if R else None
    qc.bits, qc.group, qc.L_q, qc.R, qc.R_cap = bits, G, L_q, R, max(R, 1)
    return qc


def _rec_bytes(bits, G, D):
    return 2 * G * D * bits // 8 + 8 * D


def _stage_groups(bits, G, D, g):
    rec = _rec_bytes(bits, G, D)
    ng_stage = max(1, 3072 // rec) if rec < 3072 else 1
    # a stage slot also holds one warp's fp32 state of 4 (g <= 4) or 8 heads at a segment end
    state = (4 if g <= 4 else 8) * D * 4
    if ng_stage * rec < state:
        ng_stage = -(-state // rec)
    return ng_stage, rec


CASES = [
    # B, Hq, Hkv, D, L_q, R, bits, G, target blocks
    (8, 32, 8, 128, 32640, 128, 2, 32, 592),     # Llama-3.1-8B, 8 x 32K, KIVI-2
    (1, 32, 8, 128, 499872, 128, 2, 32, 592),    # 500K context
    (1, 64, 8, 128, 131008, 64, 4, 64, 296),     # Llama-70B shape, 4-bit group 64
    (1, 4, 2, 64, 480, 32, 2, 32, 592),          # tiny: more blocks asked than stages
    (3, 3, 3, 64, 160, 0, 2, 32, 7),             # no residual
    (1, 4, 2, 64, 0, 40, 2, 32, 50),             # residual only
    (200, 64, 8, 128, 64, 0, 2, 32, 296),        # many small units: whole units per block
    (2, 8, 2, 128, 32 * 37, 3, 2, 32, 13),       # ragged residual, odd block count
    (7, 28, 7, 128, 32 * 100, 128, 2, 32, 20),   # fewer blocks than units, with residual
]


@pytest.mark.parametrize("Bq,Hq,Hkv,D,L_q,R,bits,G,target", CASES)
def test_partition_covers_every_tile_and_stage_once_in_balanced_pieces(Bq, Hq, Hkv, D, L_q, R, bits, G, target):
    sh = vc.shape(Bq, Hq, Hkv, D)
    p = vc.vc_debug_quant_partition(sh, _cache(bits, G, L_q, R), target)
    U = Bq * Hkv
    ng_stage, rec = _stage_groups(bits, G, D, Hq // Hkv)
    sq = -(-(L_q // G) // ng_stage)
    sr = -(-R // 16)
    assert (p["quant_stages"], p["residual_tiles"]) == (sq, sr)
    n, bpu = p["n_blocks"], p["blocks_per_unit"]
    assert 1 <= n <= target
    res_cov = [[0] * sr for _ in range(U)]
    q_cov = [[0] * sq for _ in range(U)]
    partials = [0] * U
    for (u0, u1, r0, r1, q0, q1) in p["blocks"]:
        assert 0 <= u0 < u1 <= U
        assert r1 > r0 or q1 > q0, "a block without work"
        for u in range(u0, u1):
            for t in range(r0, r1):
                res_cov[u][t] += 1
            for s in range(q0, q1):
                q_cov[u][s] += 1
            partials[u] += (r1 > r0) + (q1 > q0)
    assert all(c == 1 for row in res_cov for c in row)
    assert all(c == 1 for row in q_cov for c in row)
    assert all(x == p["partials_per_unit"] for x in partials)
    # cost model: a stage costs its bytes, a residual tile 4/3 of its bf16 bytes
    cq, cr = ng_stage * rec, 16 * 4 * D * 4 // 3
    if bpu >= 1:
        assert n == U * bpu
        unit_cost = sr * cr + sq * cq
        for k, (u0, u1, r0, r1, q0, q1) in enumerate(p["blocks"]):
            assert (u0, u1) == (k // bpu, k // bpu + 1)
            c = (r1 - r0) * cr + (q1 - q0) * cq
            assert abs(c - unit_cost / bpu) <= max(cq if sq else 0, cr if sr else 0) + 1, (k, c, unit_cost / bpu)
        # as many blocks as fit, up to one piece per tile or stage, and at least 8
        # quantised stages per warp (4 warps per block) when the unit has any
        want = min(target // U, unit_cost // max(cq if sq else 0, cr if sr else 0))
        if sq:
            want = min(want, sq // (4 * 8))
        assert bpu == max(1, want)
    else:
        assert U > target and n == target
        per = [u1 - u0 for (u0, u1, *_rest) in p["blocks"]]
        assert max(per) - min(per) <= 1


def test_partition_rejects_bad_arguments():
    sh = vc.shape(1, 4, 2, 64)
    with pytest.raises(vc.VcError):
        vc.vc_debug_quant_partition(sh, _cache(2, 32, 480, 32), 0)
    with pytest.raises(vc.VcError):
        vc.vc_debug_quant_partition(sh, _cache(3, 32, 480, 32), 4)
