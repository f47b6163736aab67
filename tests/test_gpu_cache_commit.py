"""Cache maintenance on the GPU (vc_cache_commit) against the oracle.

Rounds are driven as a server would drive them: the verifier's planted
logits go through vc_accept, whose device-side accepted lengths feed
vc_cache_commit directly (nothing is read back to decide the commit).  After
every round the device cache -- per-request lengths, group records and
residual rows -- must equal the oracle's maintained cache byte for byte, and
the draft attention over the maintained cache (per-request lengths read by
the kernel) must match the oracle's attention on its cache."""

import numpy as np
import pytest
import torch

from lossless_draft_verify_vc_b200 import synth
from lossless_draft_verify_vc_b200 import vc
from oracle import attention as A
from oracle import cache as CM
from oracle import quant as Q
from tests.vcutil import ATTN_TOL, np32, row_rel_err

pytestmark = pytest.mark.gpu
dev = "cuda"


@pytest.mark.parametrize("bits,G,D,Hq,Hkv,R_cap,K", [(2, 32, 128, 8, 2, 128, 30), (4, 64, 128, 16, 2, 96, 30),
                                                    (2, 32, 64, 4, 1, 40, 8)])
def test_rounds_of_commits_match_the_oracle(bits, G, D, Hq, Hkv, R_cap, K):
    B, nq, V = 3, K + 1, 512
    rounds = 14
    T0 = 4 * G + 21
    R0 = 21
    cap_groups = 4 + rounds  # room for one new record per round
    rec_b = 2 * G * D * bits // 8 + 8 * D
    sh = vc.shape(B, Hq, Hkv, D)
    # the prompt: quantised on the GPU into capacity-sized buffers
    k0, v0 = synth.kv_full(B, Hkv, T0, D, seed=bits + G + D)
    records = torch.zeros((B, Hkv, cap_groups, rec_b), dtype=torch.uint8, device=dev)
    k_res = torch.zeros((B, Hkv, R_cap, D), dtype=torch.bfloat16, device=dev)
    v_res = torch.zeros_like(k_res)
    wsq = vc.workspace(vc.vc_compress_workspace_size())
    L0 = T0 - R0
    tmp = torch.zeros((B, Hkv, L0 // G, rec_b), dtype=torch.uint8, device=dev)
    vc.vc_quantize_cache(sh, k0.to(dev), v0.to(dev), T0, bits, G, L0, tmp, k_res, v_res, R_cap, wsq)
    records[:, :, :L0 // G] = tmp
    lens = torch.tensor([[L0, R0]] * B, dtype=torch.int32, device=dev)
    tc = dict(bits=bits, group=G, L_q=cap_groups * G, R=0, R_cap=R_cap, records=records, k_res=k_res, v_res=v_res,
              lens=lens)
    qc = vc.quant_cache(tc)
    states = []
    for b in range(B):
        c = Q.build_quant_cache(np32(k0[b:b + 1]), np32(v0[b:b + 1]), bits, G, R0)
        states.append(dict(bits=bits, group=G, D=D, L_q=L0, R=R0, records=c["records"][0], k_res=c["k_res"][0],
                           v_res=c["v_res"][0]))
    ws_acc = vc.workspace(vc.vc_accept_workspace_size(B, K, V))
    ws_c = vc.workspace(vc.vc_compress_workspace_size())
    ws_d = vc.workspace(vc.vc_draft_attn_quant_workspace_size(sh, qc))
    tgt = torch.empty((B, K + 1), dtype=torch.int32, device=dev)
    acc = torch.empty(B, dtype=torch.int32, device=dev)
    cor = torch.empty(B, dtype=torch.int32, device=dev)
    for r in range(rounds):
        draft = synth.tokens((B, K), V, seed=500 + r)
        lens_planted = synth.geometric_accept_lengths(B, K, 0.15, seed=600 + r)
        logits = synth.planted_logits(B, K, V, draft, lens_planted, seed=700 + r)
        vc.vc_accept(logits.to(dev), B, K, V, draft.to(dev), tgt, acc, cor, ws_acc)
        kb, vb = synth.kv_full(B, Hkv, nq, D, seed=800 + r)
        vc.vc_cache_commit(sh, qc, kb.to(dev), vb.to(dev), nq, acc, ws_c)
        torch.cuda.synchronize()
        assert vc.vc_workspace_flags(ws_c) == 0
        for b in range(B):
            states[b] = CM.commit(states[b], np32(kb[b]), np32(vb[b]), lens_planted[b], R_cap)
        got_lens = lens.cpu().numpy()
        for b in range(B):
            st = states[b]
            assert tuple(got_lens[b]) == (st["L_q"], st["R"]), (r, b)
            assert np.array_equal(records[b, :, :st["L_q"] // G].cpu().numpy(), st["records"]), (r, b)
            assert np.array_equal(np32(k_res[b, :, :st["R"]]), st["k_res"]), (r, b)
            assert np.array_equal(np32(v_res[b, :, :st["R"]]), st["v_res"]), (r, b)
        if r % 4 == 3 or r == rounds - 1:
            q = synth.normal((B, Hq, D), seed=900 + r)
            out = torch.full((B, Hq, D), float("nan"), device=dev)
            vc.vc_draft_attn_quant(sh, qc, q.to(dev), out, ws_d)
            torch.cuda.synchronize()
            for b in range(B):
                want = A.draft_attention_quant(np32(q[b:b + 1]), CM.as_cache(states[b]))
                assert row_rel_err(np32(out[b:b + 1]), want) <= ATTN_TOL, (r, b)


def test_invalid_accept_length_and_full_capacity_leave_the_request_unchanged():
    B, Hkv, D, G, bits, R_cap, nq = 2, 1, 64, 32, 2, 40, 9
    sh = vc.shape(B, 4, Hkv, D)
    rec_b = 2 * G * D * bits // 8 + 8 * D
    records = torch.zeros((B, Hkv, 1, rec_b), dtype=torch.uint8, device=dev)
    k_res = torch.zeros((B, Hkv, R_cap, D), dtype=torch.bfloat16, device=dev)
    v_res = torch.zeros_like(k_res)
    # request 0: residual full, no record capacity left (L_q = capacity); request 1: fine
    lens = torch.tensor([[32, 40], [0, 3]], dtype=torch.int32, device=dev)
    qc = vc.quant_cache(dict(bits=bits, group=G, L_q=32, R=0, R_cap=R_cap, records=records, k_res=k_res,
                             v_res=v_res, lens=lens))
    kb, vb = synth.kv_full(B, Hkv, nq, D, seed=1, device=dev)
    ws = vc.workspace(vc.vc_compress_workspace_size())
    acc = torch.tensor([2, 4], dtype=torch.int32, device=dev)
    vc.vc_cache_commit(sh, qc, kb, vb, nq, acc, ws)
    torch.cuda.synchronize()
    assert vc.vc_workspace_flags(ws) & vc.VC_FLAG_BAD_LENGTH
    assert lens.cpu().tolist() == [[32, 40], [0, 8]]
    assert np.array_equal(np32(k_res[1, 0, 3:8]), np32(kb[1, 0, :5]))
    acc = torch.tensor([9, 0], dtype=torch.int32, device=dev)  # 9 = nq: outside the block
    lens[0, 0] = 0
    vc.vc_cache_commit(sh, qc, kb, vb, nq, acc, ws)
    torch.cuda.synchronize()
    assert vc.vc_workspace_flags(ws) & vc.VC_FLAG_BAD_LENGTH
    assert lens.cpu().tolist() == [[0, 40], [0, 9]]
