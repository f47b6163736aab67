"""Cache maintenance around a VeriCache round (oracle; test infrastructure only).

What the pages fix
------------------
[P1] "The Core Idea": a round drafts K tokens from the compressed cache, one
verification pass with the full cache scores all of them, the accepted
prefix plus the verifier's correction is kept and everything after the first
mismatch is discarded (the worked example's Emit / Discard lines).  [P2]
"Key Contributions": the compressed cache is described by the bit width it
stores; recent tokens are kept at full precision.

Readings taken where the pages are silent
-----------------------------------------
* Before a round, both caches hold the rows of every committed token except
  the newest one (x): it has no K and V yet.  The verification block is
  (x, d_1 .. d_K), nq = K + 1 rows, and the verifier computes their exact K
  and V.  With a accepted drafts the committed sequence gains x, d_1 .. d_a
  (a + 1 rows, the verifier's exact K and V), the correction becomes the new
  x, and the rows of d_(a+1) .. d_K are discarded (rolled back).
* The compressed cache receives the same a + 1 exact rows, appended to its
  bf16 residual window, so after every round it holds exactly the committed
  sequence (the drafter's own approximate rows of the round are not kept).
* When the residual would hold more than R_cap rows, its oldest `group` rows
  become one quantised group record (the rule of quant.py, per channel for
  keys and per token for values) appended after the existing records, and
  the residual keeps the rest.  With a + 1 <= group (K + 1 <= group: K <= 31
  at group 32), one record per commit always suffices.
* Consequence used as the pin: after any sequence of commits the maintained
  cache equals the cache built at once from the committed rows,
  build_quant_cache(committed, residual = R), record for record and row for
  row, because every record is the quantisation of one fixed group of G
  consecutive committed rows.
"""

from __future__ import annotations

import numpy as np

from . import quant


def empty_state(Hkv: int, D: int, bits: int, group: int) -> dict:
    """A request's quantised cache with no rows (per KV head)."""
    lay = quant.record_layout(bits, group, D)
    return dict(bits=bits, group=group, D=D, L_q=0, R=0,
                records=np.zeros((Hkv, 0, lay["size"]), np.uint8),
                k_res=np.zeros((Hkv, 0, D), np.float32), v_res=np.zeros((Hkv, 0, D), np.float32))


def commit(state: dict, k_block: np.ndarray, v_block: np.ndarray, accept_len: int, R_cap: int) -> dict:
    """One round's maintenance of one request's quantised cache.

    k_block, v_block: [Hkv, nq, D] bf16 values (float32) -- the verifier's
    exact rows of the block (x, d_1 .. d_(nq-1)).  accept_len a in
    [0, nq - 1]: rows 0 .. a are committed, the rest discarded.
    Returns the new state (the input is not modified)."""
    G, bits = state["group"], state["bits"]
    k_block = np.asarray(k_block, np.float32)
    v_block = np.asarray(v_block, np.float32)
    nq = k_block.shape[1]
    if not 0 <= accept_len < nq:
        raise ValueError("accepted length outside the block")
    n = accept_len + 1
    k_res = np.concatenate([state["k_res"], k_block[:, :n]], axis=1)
    v_res = np.concatenate([state["v_res"], v_block[:, :n]], axis=1)
    records, L_q = state["records"], state["L_q"]
    if k_res.shape[1] > R_cap:
        if k_res.shape[1] - G > R_cap:
            raise ValueError("more new rows than one group record can absorb")
        # the oldest G residual rows become one record (quant.py's rule)
        kc, sk, zk = quant.quantize_keys(k_res[:, :G], bits, G)
        vc, sv, zv = quant.quantize_values(v_res[:, :G], bits, G)
        rec = quant.pack_group_records(quant.pack_group_blocks(kc, bits, G, values=False),
                                       quant.pack_group_blocks(vc, bits, G, values=True),
                                       sk, zk, quant.pair_interleave(sv), quant.pair_interleave(zv), bits, G)
        records = np.concatenate([records, rec], axis=1)
        L_q += G
        k_res, v_res = k_res[:, G:], v_res[:, G:]
    return dict(bits=bits, group=G, D=state["D"], L_q=L_q, R=k_res.shape[1], records=records,
                k_res=k_res, v_res=v_res)


def as_cache(state: dict) -> dict:
    """One request's state as build_quant_cache's dict (B = 1)."""
    return dict(bits=state["bits"], group=state["group"], L_q=state["L_q"], R=state["R"], D=state["D"],
                records=state["records"][None], k_res=state["k_res"][None], v_res=state["v_res"][None])
