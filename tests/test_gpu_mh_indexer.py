"""Parity of the multi-head indexer (kv_index_append, sparse_mh_indexer_topk) with the oracle.

Bars: scores within 1e-5 of the request's largest |score| (the FP8 query codes are bit-identical
on both sides and e4m3 products are exact; the error is fp32 accumulation); top-k sets equal except for
candidates whose oracle score lies within 1e-5*|tau| of the k-th score; forced ties resolved to
the lowest indices exactly; appended index entries within one e4m3 step of the oracle's (both
sides quantise an fp32 fold, the device's summed in another order) and the residue ring
bit-exact (a copy of the input).
"""

import numpy as np
import pytest
import torch

from oracle import ckv_oracle as O
from synth import workloads as S
from tests import ckv_testlib as T

pytestmark = pytest.mark.gpu

SCORE_TOL = 1e-5


def _np(t):
    return t.detach().cpu().numpy()


def _layer_cfg(ckv, w, ls):
    return ckv.LayerConfig(w.num_heads, w.head_dim, w.rope_dim, ls.ratio, w.window, ls.comp_dtype, ls.win_dtype)


def _layer_cache(ckv, cfg, w, lay):
    return ckv.cache_from_tensors(cfg, w.batch, lay["comp_codes"], lay["comp_scales"], lay["win_codes"],
                                  lay["win_scales"], lay["comp_table"], lay["win_table"])


def _select(ckv, w, gen, ix, heads, dim, top_k, layer=0, q_index=None):
    """Runs sparse_mh_indexer_topk on the generated index plane; returns idx, cnt, scores, status."""
    lay, ls = gen["layers"][layer], w.layers[layer]
    cfg = _layer_cfg(ckv, w, ls)
    cache = _layer_cache(ckv, cfg, w, lay)
    icfg = ckv.IndexConfig(heads, dim)
    icache = ckv.IndexCache(ix["codes"], ix["scales"])
    msl = max(w.seq_lens)
    ws = torch.empty(ckv.mh_indexer_workspace_bytes(cfg, icfg, w.batch, msl, top_k), dtype=torch.uint8,
                     device="cuda")
    idx = torch.empty((w.batch, top_k), dtype=torch.int32, device="cuda")
    cnt = torch.empty(w.batch, dtype=torch.int32, device="cuda")
    scores = torch.full((w.batch, ckv.score_stride(cfg, msl)), float("nan"), device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    qi = ix["q_index"] if q_index is None else q_index
    ckv.sparse_mh_indexer_topk(cfg, cache, icfg, icache, gen["seq_len"], msl, qi, ix["weights"], top_k, idx, cnt,
                               ws, status, scores=scores)
    torch.cuda.synchronize()
    return _np(idx), _np(cnt), _np(scores), int(status.item())


def _check_against_oracle(w, gen, ix, idx, cnt, sc, top_k, layer=0, requests=None):
    ls = w.layers[layer]
    ocfg = T.oracle_cfg(w, ls)
    ic = O.IndexCache(_np(ix["codes"]), _np(ix["scales"]))
    table = _np(gen["layers"][layer]["comp_table"])
    qi, wt = _np(ix["q_index"]), _np(ix["weights"])
    for b in (range(w.batch) if requests is None else requests):
        L = w.seq_lens[b]
        s64 = O.mh_indexer_scores(ocfg, ic, table, b, qi[b], wt[b], L)
        n_c = s64.shape[0]
        if n_c:
            err = np.max(np.abs(sc[b, :n_c] - s64)) / max(np.max(np.abs(s64)), 1e-30)
            assert err <= SCORE_TOL, f"{w.name} b={b}: score error {err:.2e}"
        ok, msg = T.topk_sets_match(idx[b], cnt[b], s64, top_k, SCORE_TOL)
        assert ok, f"{w.name} b={b}: {msg}"


SMALL = [
    # (workload, index heads, index dim, top_k)
    (S.scaled(S.csa_b8_ctx32k(), (1000, 2999, 5001, 9, 4100, 515), "mh"), 64, 128, 512),
    (S.scaled(S.csa_b8_ctx32k(), (700, 3, 20001), "mh16"), 16, 128, 64),
    (S.scaled(S.csa_b8_ctx32k(), (4099, 1537), "mh48"), 48, 128, 100),
    (S.scaled(S.mixed_64req(), (1025, 3000, 70001, 5, 777), "mh128"), 128, 256, 2048),
    (S.scaled(S.csa_b4_ctx1m(), (131072, 65537), "mh"), 64, 128, 2048),  # > 16384 candidates
]


@pytest.mark.parametrize("case", SMALL, ids=lambda c: f"{c[0].name}_h{c[1]}_d{c[2]}")
def test_mh_scores_and_selection_match_the_oracle(cuda_lib, case):
    w, heads, dim, k = case
    gen = S.generate(w, "cuda")
    ix = S.generate_index(w, gen, heads=heads, dim=dim, device="cuda")
    idx, cnt, sc, st = _select(cuda_lib, w, gen, ix, heads, dim, k)
    assert st == 0, f"status {st:#x}"
    _check_against_oracle(w, gen, ix, idx, cnt, sc, k)


@pytest.mark.parametrize("n,base", [(2048, 512), (1200, 200)], ids=["one_epilogue_group", "two_epilogue_groups"])
def test_mh_many_short_requests_per_cta(cuda_lib, n, base):
    # n requests of 1 or 2 tiles (every 7th with no candidate): each persistent CTA walks several
    # requests, so both query-image slots and the per-warp weight slots are reused and the
    # producer waits for the MMAs of the request two switches back. 2048 requests of 2 tiles take
    # the one-group kernel (3 CTAs per SM), 1200 of 1 tile the two-group kernel, whose groups
    # take alternate tiles and so see alternate requests
    lens = tuple((base + 100 * (i % 3)) if i % 7 else 3 for i in range(n))
    w = S.Workload(f"mh_{n}req", lens, 64, 512, 64, 128, (S.LayerSpec(4, 16, "bf16", "fp8"),),
                   paged=True, from_scratch=False, seed=7100)
    gen = S.generate(w, "cuda")
    ix = S.generate_index(w, gen, device="cuda")
    idx, cnt, sc, st = _select(cuda_lib, w, gen, ix, 64, 128, 16)
    assert st == 0, f"status {st:#x}"
    _check_against_oracle(w, gen, ix, idx, cnt, sc, 16)


@pytest.mark.parametrize("lens,k", [((4000, 3001), 50), ((100000, 70001), 300)],
                         ids=["one_cta_selection", "bitmap_selection"])
def test_mh_zero_query_ties_select_the_lowest_indices(cuda_lib, lens, k):
    # a zero index query scores every candidate 0: the selection is the first k entries
    w = S.scaled(S.csa_b8_ctx32k(), lens, "mhtie")
    gen = S.generate(w, "cuda")
    ix = S.generate_index(w, gen, device="cuda")
    idx, cnt, sc, st = _select(cuda_lib, w, gen, ix, 64, 128, k, q_index=torch.zeros_like(ix["q_index"]))
    assert st == 0
    for b, L in enumerate(lens):
        n_c = L // 4
        assert int(cnt[b]) == min(k, n_c)
        assert np.array_equal(idx[b, :cnt[b]], np.arange(min(k, n_c)))
        assert np.all(sc[b, :n_c] == 0.0)


def test_mh_bad_block_and_length_set_status(cuda_lib):
    w = S.scaled(S.csa_b8_ctx32k(), (3000, 2000), "mhbad")
    gen = S.generate(w, "cuda")
    ix = S.generate_index(w, gen, device="cuda")
    gen["layers"][0]["comp_table"][1, 2] = 10 ** 6     # entries 128 .. 191 of request 1 unmapped
    idx, cnt, sc, st = _select(cuda_lib, w, gen, ix, 64, 128, 64)
    assert st & cuda_lib.CKV_DEV_BAD_BLOCK
    assert np.all(sc[1, 128:192] == 0.0)
    gen["layers"][0]["comp_table"][1, 2] = 0
    gen["seq_len"][0] = 5000                           # above max_seq_len = 3000
    idx, cnt, sc, st = _select(cuda_lib, w, gen, ix, 64, 128, 64)
    assert st & cuda_lib.CKV_DEV_BAD_LENGTH
    assert int(cnt[0]) == 0 and np.all(idx[0] == -1)


def test_mh_full_size_32k_and_1m(cuda_lib):
    for w, k in ((S.csa_b8_ctx32k(), 512), (S.csa_b4_ctx1m(), 2048)):
        gen = S.generate(w, "cuda")
        ix = S.generate_index(w, gen, device="cuda")
        idx, cnt, sc, st = _select(cuda_lib, w, gen, ix, 64, 128, k)
        assert st == 0
        _check_against_oracle(w, gen, ix, idx, cnt, sc, k, requests=(0, w.batch - 1))
        del gen, ix
        torch.cuda.empty_cache()


# ------------------------------------------------------------------------------------------------
# index-key compressor
# ------------------------------------------------------------------------------------------------

def _append_index(ckv, w, gen, ix, dim, layer=0):
    """GPU: the set-up append (multi-token) then the decode token; returns the device plane."""
    lay, ls = gen["layers"][layer], w.layers[layer]
    cfg = _layer_cfg(ckv, w, ls)
    cache = _layer_cache(ckv, cfg, w, lay)
    icfg = ckv.IndexConfig(64, dim)
    icache = ckv.IndexCache(torch.zeros_like(ix["codes"]), torch.zeros_like(ix["scales"]),
                            torch.zeros((w.batch, ls.ratio, dim), device="cuda"),
                            torch.zeros((w.batch, ls.ratio), device="cuda"))
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    cu = lay["cu_setup"]
    n = int((cu[1:] - cu[:-1]).max().item())
    if n > 0:
        ckv.kv_index_append(cfg, cache, icfg, icache, lay["setup_start"].to(torch.int32), ix["k_setup"],
                            lay["logit_setup"], status, cu_new=cu, max_new=n, max_seq_len=max(w.seq_lens))
    ckv.kv_index_append(cfg, cache, icfg, icache, (gen["seq_len"] - 1).to(torch.int32), ix["k_new"],
                        lay["logit_new"], status, max_seq_len=max(w.seq_lens))
    torch.cuda.synchronize()
    return icache, int(status.item())


def _oracle_append_index(w, gen, ix, dim, layer=0):
    lay, ls = gen["layers"][layer], w.layers[layer]
    ocfg = T.oracle_cfg(w, ls)
    ic = O.IndexCache(np.zeros_like(_np(ix["codes"])), np.zeros_like(_np(ix["scales"])))
    table = _np(lay["comp_table"])
    start, cu = _np(lay["setup_start"]), _np(lay["cu_setup"])
    ks, lg = _np(ix["k_setup"]), _np(lay["logit_setup"])
    kn, ln = _np(ix["k_new"]), _np(lay["logit_new"])
    for b, L in enumerate(w.seq_lens):
        while len(ic.residue) <= b:
            ic.residue.append([])
        O.index_append_tokens(ocfg, ic, table, b, int(start[b]), ks[cu[b]:cu[b + 1]], lg[cu[b]:cu[b + 1]])
        O.index_append_tokens(ocfg, ic, table, b, L - 1, kn[b:b + 1], ln[b:b + 1])
    return ic


APPEND = [
    S.Workload("mh_scratch_r4", (777, 1500, 130, 4), 8, 512, 64, 128, (S.LayerSpec(4, 16, "bf16", "fp8"),),
               paged=True, from_scratch=True, seed=2300),
    S.Workload("mh_scratch_r128", (777, 1500, 130), 8, 512, 64, 128, (S.LayerSpec(128, 16, "bf16", "fp8"),),
               paged=True, from_scratch=True, seed=2301),
    S.scaled(S.csa_b8_ctx32k(), (32768, 20001, 4099, 9, 700, 131), "mhdecode", seed=2302),
]


@pytest.mark.parametrize("w", APPEND, ids=lambda w: w.name)
@pytest.mark.parametrize("dim", [128, 256])
def test_index_append_matches_the_oracle(cuda_lib, w, dim):
    gen = S.generate(w, "cuda")
    ix = S.generate_index(w, gen, dim=dim, device="cuda")
    icache, st = _append_index(cuda_lib, w, gen, ix, dim)
    assert st == 0
    ic = _oracle_append_index(w, gen, ix, dim)
    ls = w.layers[0]
    gs, os_ = _np(icache.scales).reshape(-1), ic.scales.reshape(-1)
    assert np.allclose(gs, os_, rtol=1e-6, atol=0), "index entry scales"
    gc, oc = _np(icache.codes).astype(np.int64), ic.codes.astype(np.int64)
    bad = gc != oc
    # a differing code is a neighbour: same sign, magnitude code +-1
    assert np.all((gc[bad] & 0x80) == (oc[bad] & 0x80)), "index code signs"
    assert np.all(np.abs((gc[bad] & 0x7F) - (oc[bad] & 0x7F)) <= 1), "index codes beyond one step"
    assert int(bad.sum()) <= max(4, gc.size // 1000), f"{int(bad.sum())} index codes differ"
    # the ring holds the unfinished group's keys and logits as given
    ring, ring_lg = _np(icache.residue_k), _np(icache.residue_logit)
    for b in range(w.batch):
        for pos, key, logit in ic.residue[b]:
            assert np.array_equal(ring[b, pos % ls.ratio], key)
            assert ring_lg[b, pos % ls.ratio] == logit


def test_append_then_select_matches_the_oracle_end_to_end(cuda_lib):
    # index plane built by the appends on both sides, then scored and selected
    w = APPEND[0]
    gen = S.generate(w, "cuda")
    ix = S.generate_index(w, gen, device="cuda")
    icache, st = _append_index(cuda_lib, w, gen, ix, 128)
    assert st == 0
    ic = _oracle_append_index(w, gen, ix, 128)
    ix_dev = dict(ix, codes=icache.codes, scales=icache.scales)
    idx, cnt, sc, st = _select(cuda_lib, w, gen, ix_dev, 64, 128, 16)
    assert st == 0
    ocfg = T.oracle_cfg(w, w.layers[0])
    table = _np(gen["layers"][0]["comp_table"])
    qi, wt = _np(ix["q_index"]), _np(ix["weights"])
    for b, L in enumerate(w.seq_lens):
        s64 = O.mh_indexer_scores(ocfg, ic, table, b, qi[b], wt[b], L)
        if s64.size:
            # entries may differ by one e4m3 step where the two folds round differently
            err = np.max(np.abs(sc[b, :s64.size] - s64)) / np.max(np.abs(s64))
            assert err <= 0.07, f"b={b}: score error {err:.2e}"
        # the selection is exact against the scores of the device's own entries
        s_dev = O.mh_indexer_scores(ocfg, O.IndexCache(_np(icache.codes), _np(icache.scales)), table, b,
                                    qi[b], wt[b], L)
        ok, msg = T.topk_sets_match(idx[b], cnt[b], s_dev, 16, SCORE_TOL)
        assert ok, f"b={b}: {msg}"
