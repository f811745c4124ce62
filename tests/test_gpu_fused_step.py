"""ckv_decode_step: append, select and attend of one layer in one call.

The fused call runs the same kernels as the three calls except that the indexer's query pass runs
beside the append on sparse layers (and also writes the cos/sin table of the rotary pairs with the
prep kernel's arithmetic), and that on dense layers of large batches one front kernel runs the
append beside the attention's query preparation, so every result must be bit-identical to the
three calls': the output, the selection and every byte the append writes. Each side works on its
own copy of the same generated pools.
"""

import numpy as np
import pytest
import torch

from oracle import ckv_oracle as O
from synth import workloads as S
from tests import ckv_testlib as T

pytestmark = pytest.mark.gpu

CACHE_PLANES = ("comp_codes", "comp_scales", "win_codes", "win_scales", "residue_kv", "residue_logit")

# sparse layers launch the append and the query pass as two kernels; dense layers of more than 18
# requests (more (request, slice) CTAs than SMs) one front kernel: both forms are covered
_LENS24 = tuple(1000 + (7919 * i) % 30000 for i in range(24))
SMALL = [
    S.scaled(S.csa_b8_ctx32k(), (32768, 20001, 4099, 9, 700, 131), "fused", seed=6000),
    S.scaled(S.hca_b32_ctx128k(), (131072, 60000, 129, 1000), "fused", seed=6001),
    S.scaled(S.mixed_64req(), (16385, 5000, 1025, 70000), "fused", seed=6002),
    S.csa_b1_ctx4k_fp32(),
    S.scaled(S.csa_b8_ctx32k(), _LENS24, "fused_front", seed=6003),
    S.scaled(S.hca_b32_ctx128k(), tuple(4 * x for x in _LENS24), "fused_front", seed=6004),
]


def _bytes(t):
    return t.contiguous().view(torch.uint8)


def _check_fused_equals_three_calls(cuda_lib, w):
    gen = S.generate(w, "cuda")
    seq = gen["seq_len"]
    for li, (lay, ls) in enumerate(zip(gen["layers"], w.layers)):
        three = T.gpu_layer(cuda_lib, w, lay, ls)
        fused = T.gpu_layer(cuda_lib, w, lay, ls)
        T.gpu_setup(three, lay)
        T.gpu_setup(fused, lay)
        out3 = three.step(seq, (seq - 1).to(torch.int32), lay["q"], lay["kv_new"], lay["logit_new"]).clone()
        out1 = fused.fused_step(seq, lay["q"], lay["kv_new"], lay["logit_new"]).clone()
        assert T.status_word(three) == 0 and T.status_word(fused) == 0
        assert torch.equal(_bytes(out1), _bytes(out3)), f"{w.name} layer {li}: outputs differ"
        if ls.top_k is not None:
            assert torch.equal(fused.cnt, three.cnt)
            assert torch.equal(fused.idx, three.idx)
        for name in CACHE_PLANES:
            a, b = getattr(three.cache, name), getattr(fused.cache, name)
            if a is not None:
                assert torch.equal(_bytes(a), _bytes(b)), f"{w.name} layer {li}: {name} differs"


@pytest.mark.parametrize("w", SMALL, ids=lambda w: w.name)
def test_fused_step_is_bit_identical_to_the_three_calls(cuda_lib, w):
    _check_fused_equals_three_calls(cuda_lib, w)


def test_fused_step_at_full_size(cuda_lib):
    _check_fused_equals_three_calls(cuda_lib, S.csa_b8_ctx32k())
    torch.cuda.empty_cache()


def test_fused_step_sets_the_status_of_a_bad_length(cuda_lib):
    w = SMALL[0]
    gen = S.generate(w, "cuda")
    lay, ls = gen["layers"][0], w.layers[0]
    dl = T.gpu_layer(cuda_lib, w, lay, ls)
    seq = gen["seq_len"].clone()
    seq[2] = max(w.seq_lens) + 5  # above max_seq_len: flagged, that request skipped
    out = dl.fused_step(seq, lay["q"], lay["kv_new"], lay["logit_new"])
    assert T.status_word(dl) & cuda_lib.CKV_DEV_BAD_LENGTH
    assert torch.count_nonzero(out[2]) == 0


FULL = [S.csa_b1_ctx4k_fp32, S.csa_b8_ctx32k, S.hca_b32_ctx128k, S.csa_b4_ctx1m, S.mixed_64req]


@pytest.mark.parametrize("make", FULL, ids=lambda f: f.__name__)
def test_fused_step_matches_the_oracle_at_full_size(cuda_lib, make):
    """The call the bench times, at every named workload's full size, against the oracle (not
    against the three calls): the unfinished group is appended first (both sides), then one
    ckv_decode_step per layer appends the decode token, selects and attends. Selections follow
    the set rule on the oracle's scores; outputs are within 2e-3 (2e-2 NVFP4) of the oracle on
    the GPU's selection, and on the oracle's own selection when the two are equal; the caches
    the step appended to hold the oracle's bytes within the append's rounding rules (all but the
    1 GiB pool of the 1M-context workload)."""
    from tests.test_gpu_parity import ATT_TOL, _compare_caches
    w = make()
    gen = S.generate(w, "cuda")
    seq = gen["seq_len"]
    for li, (lay, ls) in enumerate(zip(gen["layers"], w.layers)):
        dl = T.gpu_layer(cuda_lib, w, lay, ls)
        T.gpu_setup(dl, lay)
        out = dl.fused_step(seq, lay["q"], lay["kv_new"], lay["logit_new"]).cpu().numpy()
        assert T.status_word(dl) == 0, f"{w.name} layer {li}: device status"
        ocfg = T.oracle_cfg(w, ls)
        oc = T.oracle_cache(lay)
        T.oracle_setup(ocfg, oc, lay, w.batch)
        T.oracle_append_decode_token(ocfg, oc, lay, w.seq_lens)
        if lay["comp_codes"].numel() <= 256 << 20:   # the 1 GiB pool of the 1M workload: outputs only
            _compare_caches(f"{w.name} layer {li}", ocfg, oc, dl, lay, w, ls)
        qn = lay["q"].cpu().numpy()
        idx, cnt = dl.idx.cpu().numpy() if dl.idx is not None else None, \
            dl.cnt.cpu().numpy() if dl.cnt is not None else None
        worst = 0.0
        for b, L in enumerate(w.seq_lens):
            n_c = L // ls.ratio
            if ls.top_k is not None:
                s64 = O.indexer_scores(ocfg, oc, b, qn[b], L)
                ok, msg = T.topk_sets_match(idx[b], cnt[b], s64, ls.top_k, 1e-5)
                assert ok, f"{w.name} layer {li} b={b}: {msg}"
                sel_gpu = idx[b, :cnt[b]].astype(np.int64)
                sel_ref = O.topk_select(s64, ls.top_k)
            else:
                sel_gpu = sel_ref = np.arange(n_c)
            ref = O.attention(ocfg, oc, b, qn[b], L, sel_gpu)
            e = T.max_rel_err(out[b], ref)
            assert e <= ATT_TOL[ls.comp_dtype], f"{w.name} layer {li} b={b}: rel err {e:.2e}"
            if np.array_equal(sel_gpu, sel_ref):
                e1 = T.max_rel_err(out[b], O.attention(ocfg, oc, b, qn[b], L, sel_ref))
                assert e1 <= ATT_TOL[ls.comp_dtype], f"{w.name} layer {li} b={b}: rel err {e1:.2e} (oracle set)"
            worst = max(worst, e)
        print(f"{w.name} layer {li}: max attention rel err {worst:.2e}")
        del dl
    del gen
    torch.cuda.empty_cache()
