"""Parity of the CUDA acceptance kernel with the oracle (bit-exact)."""

import numpy as np
import pytest
import torch

from lossless_draft_verify_vc_b200 import synth
from lossless_draft_verify_vc_b200 import vc
from oracle import accept as ACC

pytestmark = pytest.mark.gpu
dev = "cuda"


def run_accept(logits: torch.Tensor, draft: torch.Tensor):
    B, K1, V = logits.shape
    K = K1 - 1
    ws = vc.workspace(vc.vc_accept_workspace_size(B, K, V))
    target = torch.full((B, K1), -7, dtype=torch.int32, device=dev)
    acc = torch.full((B,), -7, dtype=torch.int32, device=dev)
    cor = torch.full((B,), -7, dtype=torch.int32, device=dev)
    d = draft.to(dev, torch.int32).contiguous() if K else torch.zeros((B, 1), dtype=torch.int32, device=dev)
    vc.vc_accept(logits.contiguous(), B, K, V, d, target, acc, cor, ws)
    torch.cuda.synchronize()
    return target.cpu().numpy(), acc.cpu().numpy(), cor.cpu().numpy(), ws


def check(logits, draft):
    t, a, c, ws = run_accept(logits.to(dev), draft)
    tw, aw, cw = ACC.accept(logits.float().cpu().numpy(), draft.cpu().numpy().reshape(logits.shape[0], -1))
    assert np.array_equal(t, tw)
    assert np.array_equal(a, aw)
    assert np.array_equal(c, cw)
    return a


def test_tiny_planted_prefix_of_five():
    """One request, K = 8 drafted tokens, vocabulary 1024 fp32, argmax planted
    to agree with the draft on the first 5 positions."""
    K, V = 8, 1024
    draft = synth.tokens((1, K), V, seed=2)
    logits = synth.planted_logits(1, K, V, draft, [5], seed=2)
    a = check(logits, draft)
    assert a[0] == 5


def test_llama8b_vocab_bf16_geometric_prefixes():
    B, K, V = 8, 30, 128256
    draft = synth.tokens((B, K), V, seed=3)
    lens = synth.geometric_accept_lengths(B, K, 0.2, seed=3)
    logits = synth.planted_logits(B, K, V, draft, lens, seed=3, dtype=torch.bfloat16)
    a = check(logits, draft)
    assert a.tolist() == lens


@pytest.mark.parametrize("V", [1, 3, 5, 1001, 16385, 152064])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_ties_nans_and_unaligned_rows(V, dtype):
    """Integer-valued logits force many ties; some NaNs; V not a multiple of
    the vector width makes rows start unaligned."""
    g = torch.Generator().manual_seed(V)
    B, K = 5, 4
    logits = torch.randint(-2, 3, (B, K + 1, V), generator=g).to(dtype)
    if V > 4:
        logits[1, 2, V // 2] = float("nan")
        logits[1, 2, V // 3] = float("nan")
        logits[2, 0, :] = float("-inf")
        logits[3, 1, :] = 0.0
        logits[3, 1, V - 1] = -0.0
    draft = torch.randint(0, V, (B, K), generator=g, dtype=torch.int32)
    tgt = ACC.greedy_predictions(logits.float().numpy())
    draft[0] = torch.from_numpy(tgt[0, :K])  # request 0 accepts all and takes the bonus
    check(logits, draft)


def test_zero_draft_length():
    logits = torch.randn(3, 1, 77)
    t, a, c, _ = run_accept(logits.to(dev), torch.zeros(3, 0, dtype=torch.int32))
    assert a.tolist() == [0, 0, 0]
    assert c.tolist() == logits.argmax(-1)[:, 0].tolist()


def test_workspace_reuse_is_stable():
    B, K, V = 4, 6, 40000
    draft = synth.tokens((B, K), V, seed=9)
    logits = synth.planted_logits(B, K, V, draft, [0, 3, 6, 2], seed=9).to(dev)
    ws = vc.workspace(vc.vc_accept_workspace_size(B, K, V))
    outs = []
    for _ in range(3):
        target = torch.empty((B, K + 1), dtype=torch.int32, device=dev)
        acc = torch.empty(B, dtype=torch.int32, device=dev)
        cor = torch.empty(B, dtype=torch.int32, device=dev)
        vc.vc_accept(logits, B, K, V, draft.to(dev), target, acc, cor, ws)
        outs.append((target.cpu(), acc.cpu(), cor.cpu()))
    for o in outs[1:]:
        assert all(torch.equal(x, y) for x, y in zip(o, outs[0]))
    assert outs[0][1].tolist() == [0, 3, 6, 2]


def test_invalid_arguments_are_refused():
    ws = vc.workspace(1 << 16)
    x = torch.zeros(1, 2, 8, device=dev)
    i = torch.zeros(4, dtype=torch.int32, device=dev)
    with pytest.raises(vc.VcError) as e:
        vc.vc_accept(x, 1, 1, 0, i, i, i, i, ws)
    assert e.value.status == vc.VC_ERR_INVALID_ARG
