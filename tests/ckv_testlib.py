"""Helpers shared by the tests: build oracle state from the seeded inputs, compare results.

Nothing here computes the method: the oracle and the CUDA binding each do their own arithmetic.
"""

from __future__ import annotations

import numpy as np
import torch

from oracle import ckv_oracle as O
from synth import workloads as S


def oracle_cfg(w: S.Workload, ls: S.LayerSpec) -> O.LayerCfg:
    return O.LayerCfg(num_heads=w.num_heads, head_dim=w.head_dim, rope_dim=w.rope_dim,
                      ratio=ls.ratio, window=w.window, comp_dtype=ls.comp_dtype,
                      win_dtype=ls.win_dtype)


def _np(t):
    return None if t is None else t.detach().cpu().numpy().copy()


def oracle_cache(lay: dict) -> O.LayerCache:
    return O.LayerCache(comp_codes=_np(lay["comp_codes"]), comp_scales=_np(lay["comp_scales"]),
                        win_codes=_np(lay["win_codes"]), win_scales=_np(lay["win_scales"]),
                        comp_table=_np(lay["comp_table"]), win_table=_np(lay["win_table"]))


def oracle_setup(cfg: O.LayerCfg, cache: O.LayerCache, lay: dict, batch: int) -> None:
    """The appends that precede the decode step (unfinished group, or the whole context)."""
    start = _np(lay["setup_start"])
    cu = _np(lay["cu_setup"])
    kv = _np(lay["kv_setup"])
    lg = _np(lay["logit_setup"])
    for b in range(batch):
        # tokens before setup_start sit in completed groups (setup_start is a group boundary)
        while len(cache.residue) <= b:
            cache.residue.append([])
        O.append_tokens(cfg, cache, b, int(start[b]), kv[cu[b]:cu[b + 1]], lg[cu[b]:cu[b + 1]])


def oracle_append_decode_token(cfg, cache, lay, seq_lens) -> None:
    kv = _np(lay["kv_new"])
    lg = _np(lay["logit_new"])
    for b, L in enumerate(seq_lens):
        O.append_tokens(cfg, cache, b, int(L) - 1, kv[b:b + 1], lg[b:b + 1])


def topk_sets_match(gpu_idx, gpu_cnt, oracle_scores, k, rel_band=1e-5):
    """Compare a selected set against the oracle's fp32 scores.

    The sets must be equal except for candidates whose oracle score lies within rel_band*|tau|
    of tau, the oracle's k-th largest fp32 score (such candidates are interchangeable).
    Returns (ok, message)."""
    s32 = np.asarray(oracle_scores, dtype=np.float32).astype(np.float64)
    n = s32.shape[0]
    k_eff = min(k, n)
    ref = O.topk_select(oracle_scores, k)
    if int(gpu_cnt) != k_eff:
        return False, f"count {int(gpu_cnt)} != {k_eff}"
    g = np.asarray(gpu_idx[:k_eff], dtype=np.int64)
    if np.any(np.diff(g) <= 0):
        return False, "indices not strictly ascending"
    if np.any(g < 0) or np.any(g >= n):
        return False, "index out of range"
    if np.any(np.asarray(gpu_idx[k_eff:]) != -1):
        return False, "padding is not -1"
    if k_eff == 0:
        return True, "empty"
    tau = np.sort(s32)[::-1][k_eff - 1]
    diff = np.setxor1d(g, ref)
    bad = diff[np.abs(s32[diff] - tau) > rel_band * abs(tau)]
    if bad.size:
        return False, f"{bad.size} non-interchangeable differences, e.g. {bad[:5]} (tau={tau})"
    return True, f"{diff.size} interchangeable differences"


def max_rel_err(out, ref):
    """Per (request, head) row: max_d |o - ref| / max_d |ref|; the max over rows."""
    out = np.asarray(out, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    num = np.max(np.abs(out - ref), axis=-1)
    den = np.maximum(np.max(np.abs(ref), axis=-1), 1e-30)
    return float(np.max(num / den))


# ------------------------------------------------------------------------------------------------
# CUDA side (through the Python binding of the C ABI)
# ------------------------------------------------------------------------------------------------

def gpu_layer(ckv, w: S.Workload, lay: dict, ls: S.LayerSpec, max_seq_len=None, top_k="spec"):
    """A DecodeLayer over copies of the generated pools (the tables are shared)."""
    cfg = ckv.LayerConfig(w.num_heads, w.head_dim, w.rope_dim, ls.ratio, w.window, ls.comp_dtype,
                          ls.win_dtype)
    clone = lambda t: None if t is None else t.clone()  # noqa: E731
    cache = ckv.cache_from_tensors(cfg, w.batch, clone(lay["comp_codes"]), clone(lay["comp_scales"]),
                                   clone(lay["win_codes"]), clone(lay["win_scales"]),
                                   lay["comp_table"], lay["win_table"])
    msl = max(w.seq_lens) if max_seq_len is None else max_seq_len
    return ckv.DecodeLayer(cfg, cache, w.batch, msl, ls.top_k if top_k == "spec" else top_k)


def gpu_setup(dl, lay: dict) -> None:
    cu = lay["cu_setup"]
    n = (cu[1:] - cu[:-1]).max().item()
    if n > 0:
        dl.append(lay["setup_start"].to(torch.int32), lay["kv_setup"], lay["logit_setup"],
                  cu_new=cu, max_new=int(n))


def gpu_append_decode_token(dl, lay: dict, seq_len) -> None:
    dl.append((seq_len - 1).to(torch.int32), lay["kv_new"], lay["logit_new"])


def status_word(dl) -> int:
    torch.cuda.synchronize()
    return int(dl.status[0].item()) & 0xffffffff

