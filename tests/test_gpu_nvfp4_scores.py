"""The head-averaged indexer over an NVFP4 compressed cache at D = 512 against the oracle, through
the C ABI: scores within 1e-5 of the largest, top-k sets by the set
rule, on batches whose requests switch inside a CTA's range of tiles, ragged last tiles, queries
of very different magnitudes, and an unmapped block (flagged, its entries score 0)."""

import numpy as np
import pytest
import torch

from oracle import ckv_oracle as O
from synth import workloads as S
from tests import ckv_testlib as T

pytestmark = pytest.mark.gpu


def _layer(lens, seed, top_k=64):
    w = S.Workload("nvfp4_scores", tuple(lens), 64, 512, 64, 128, (S.LayerSpec(4, top_k, "nvfp4", "fp8"),),
                   paged=True, from_scratch=False, seed=seed)
    gen = S.generate(w, "cuda")
    return w, gen, gen["layers"][0], w.layers[0]


def _check(cuda_lib, w, gen, lay, ls, q, skip=()):
    dl = T.gpu_layer(cuda_lib, w, lay, ls)
    seq = gen["seq_len"]
    scores = torch.full((w.batch, cuda_lib.score_stride(dl.cfg, dl.max_seq_len)), float("nan"), device="cuda")
    dl.select(seq, q, scores=scores)
    st = T.status_word(dl)
    sc, idx, cnt = scores.cpu().numpy(), dl.idx.cpu().numpy(), dl.cnt.cpu().numpy()
    ocfg, oc = T.oracle_cfg(w, ls), T.oracle_cache(lay)
    qn = q.cpu().numpy()
    for b, L in enumerate(w.seq_lens):
        if b in skip:
            continue
        n_c = L // 4
        s64 = O.indexer_scores(ocfg, oc, b, qn[b], L)
        if n_c:
            err = np.max(np.abs(sc[b, :n_c] - s64)) / max(np.max(np.abs(s64)), 1e-30)
            assert err <= 1e-5, f"b={b}: score error {err:.2e}"
        ok, msg = T.topk_sets_match(idx[b], cnt[b], s64, ls.top_k, 1e-5)
        assert ok, f"b={b}: {msg}"
    return st, sc


def test_many_short_and_long_requests(cuda_lib):
    rng = np.random.default_rng(9000)
    lens = [int(x) for x in rng.integers(1, 40000, size=300)] + [131072, 5, 513, 129 * 4]
    w, gen, lay, ls = _layer(lens, 9001)
    st, _ = _check(cuda_lib, w, gen, lay, ls, lay["q"])
    assert st == 0


@pytest.mark.parametrize("scale", [1e-4, 1.0, 3e4])
def test_query_magnitudes(cuda_lib, scale):
    w, gen, lay, ls = _layer((20000, 777, 65537), 9002)
    q = (lay["q"] * scale).contiguous()
    st, _ = _check(cuda_lib, w, gen, lay, ls, q)
    assert st == 0


def test_unmapped_block_is_flagged_and_scores_zero(cuda_lib):
    w, gen, lay, ls = _layer((5000, 3000), 9003)
    lay["comp_table"][0, 3] = -1           # entries 192 .. 255 of request 0
    st, sc = _check(cuda_lib, w, gen, lay, ls, lay["q"], skip=(0,))
    assert st & cuda_lib.CKV_DEV_BAD_BLOCK
    assert np.all(sc[0, 192:256] == 0.0)
    assert np.all(np.isfinite(sc[0, :5000 // 4]))
