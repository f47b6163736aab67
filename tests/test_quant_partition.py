"""The work partition of vc_draft_attn_quant, checked on the CPU through
vc_debug_quant_partition (no GPU call): the stages of one call -- every
(request, head) unit's residual rows, 16 per stage, then every unit's
quantised groups -- are cut into contiguous, non-empty, cost-balanced block
ranges, and the segment bound the workspace is sized with holds."""

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


CASES = [
    # B, Hq, Hkv, D, L_q, R, bits, G, target blocks
    (8, 32, 8, 128, 32640, 128, 2, 32, 592),     # Llama-3.1-8B, 8 x 32K, KIVI-2
    (1, 32, 8, 128, 499872, 128, 2, 32, 592),    # 500K context
    (1, 64, 8, 128, 131008, 64, 4, 64, 296),     # Llama-70B shape, 4-bit group 64
    (1, 4, 2, 64, 480, 32, 2, 32, 592),          # tiny: more blocks asked than stages
    (3, 3, 3, 64, 160, 0, 2, 32, 7),             # no residual
    (1, 4, 2, 64, 0, 40, 2, 32, 50),             # residual only
    (200, 64, 8, 128, 64, 0, 2, 32, 296),        # many small units
    (2, 8, 2, 128, 32 * 37, 3, 2, 32, 13),       # ragged residual, odd block count
]


@pytest.mark.parametrize("Bq,Hq,Hkv,D,L_q,R,bits,G,target", CASES)
def test_partition_covers_every_stage_once_in_balanced_ranges(Bq, Hq, Hkv, D, L_q, R, bits, G, target):
    sh = vc.shape(Bq, Hq, Hkv, D)
    qc = _cache(bits, G, L_q, R)
    p = vc.vc_debug_quant_partition(sh, qc, target)
    U = Bq * Hkv
    rec = _rec_bytes(bits, G, D)
    ng_stage = max(1, 3072 // rec) if rec < 3072 else 1
    ng = L_q // G
    sq = -(-ng // ng_stage)
    sr = -(-R // 16)
    assert p["n_quant_stages"] == U * sq
    assert p["n_stages"] == U * (sq + sr)
    first, n = p["first"], p["n_blocks"]
    assert 1 <= n <= target
    assert first[0] == 0 and first[n] == p["n_stages"]
    assert all(first[k] < first[k + 1] for k in range(n)), "a block without a stage"
    # cost of a stage: its bytes (records), or twice its bytes (16 bf16 K and V
    # rows, fetched without a pipeline)
    cq, cr = ng_stage * rec, 16 * 4 * D * 2
    RZ = U * sr

    def cost(s):
        return s * cr if s < RZ else RZ * cr + (s - RZ) * cq

    total = cost(p["n_stages"])
    for k in range(n):
        c = cost(first[k + 1]) - cost(first[k])
        assert abs(c - total / n) <= max(cq, cr) + 1, (k, c, total / n)

    def seg(s):
        return s // sr if s < RZ else U + (s - RZ) // sq

    segs = max(seg(first[k + 1] - 1) - seg(first[k]) + 1 for k in range(n))
    assert p["max_segments"] == segs


def test_partition_rejects_bad_arguments():
    sh = vc.shape(1, 4, 2, 64)
    with pytest.raises(vc.VcError):
        vc.vc_debug_quant_partition(sh, _cache(2, 32, 480, 32), 0)
    with pytest.raises(vc.VcError):
        vc.vc_debug_quant_partition(sh, _cache(3, 32, 480, 32), 4)
