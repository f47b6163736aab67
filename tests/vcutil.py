"""Shared helpers for the tests: dtype marshalling between torch tensors and
the oracle's numpy arrays, and the attention tolerance metric.

Tolerance (one reading of "max relative error 2e-3" for attention outputs,
which cluster near zero so an element-wise ratio is ill-posed): for every
output row, max_c |o_c - o*_c| / max_c |o*_c| must be <= 2e-3."""

from __future__ import annotations

import numpy as np
import torch

ATTN_TOL = 2e-3


def np32(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float32).numpy()


def row_rel_err(got, want) -> float:
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    D = want.shape[-1]
    g = got.reshape(-1, D)
    w = want.reshape(-1, D)
    num = np.abs(g - w).max(axis=1)
    den = np.maximum(np.abs(w).max(axis=1), 1e-30)
    return float((num / den).max())


def quant_cache_to_torch(cache: dict, device, R_cap: int | None = None, pad_value: float = float("nan")) -> dict:
    """The oracle's quantised cache (numpy) as device tensors in the library's
    layout.  Residual rows beyond R (up to R_cap) are filled with pad_value so
    a kernel that reads them produces NaN."""
    R = cache["R"]
    R_cap = R if R_cap is None else R_cap
    B, H = cache["records"].shape[:2]
    D = cache["D"]

    def res(x):
        out = torch.full((B, H, max(R_cap, 1), D), pad_value, dtype=torch.float32)
        if R:
            out[:, :, :R] = torch.from_numpy(np.ascontiguousarray(x[:, :, :R]))
        return out.to(torch.bfloat16).to(device)

    rec = torch.from_numpy(np.ascontiguousarray(cache["records"]).astype(np.uint8)).to(device)
    return dict(bits=cache["bits"], group=cache["group"], L_q=cache["L_q"], R=R, R_cap=max(R_cap, 1),
                records=rec, k_res=res(cache["k_res"]), v_res=res(cache["v_res"]))


def quant_cache_from_torch(t: dict) -> dict:
    """Device quantised cache (e.g. drawn on the GPU for a full-size run) as the
    oracle's numpy dict; only rows 0..R-1 of the residual are kept."""
    R = int(t["R"])
    D = int(t["k_res"].shape[-1])
    return dict(bits=int(t["bits"]), group=int(t["group"]), L_q=int(t["L_q"]), R=R, D=D,
                records=t["records"].detach().cpu().numpy(),
                k_res=np32(t["k_res"][:, :, :R]), v_res=np32(t["v_res"][:, :, :R]))
