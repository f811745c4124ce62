"""sparse_indexer_topk_noalloc: the indexer for callers that cannot allocate device memory.

Such callers (an extension inside a host program that owns all device memory and gives it no
allocator, or a latency-critical path where an allocation would synchronize the device) pass no
workspace; the library uses its own fixed 16 MiB scratch array. These tests call the entry point
through the C ABI and check that it returns what the workspace entry point returns, on two calls
in a row with different queries (the shared scratch keeps the previous call's contents), and that
sizes beyond the scratch are refused before anything runs. This file is collected last.
"""

import ctypes

import numpy as np
import pytest
import torch

from synth import workloads as S
from tests import ckv_testlib as T

pytestmark = pytest.mark.gpu


def _noalloc(ckv, dl, seq, q, idx, cnt, scores):
    """One call of the entry point through the C ABI; scores=None leaves the scores in the
    library's scratch array."""
    lib = ckv.load_library()
    st = lib.sparse_indexer_topk_noalloc(
        ctypes.byref(dl.cfg.c()), ctypes.byref(dl.cache.c()), int(seq.shape[0]), seq.data_ptr(),
        dl.max_seq_len, q.data_ptr(), dl.top_k, idx.data_ptr(), cnt.data_ptr(),
        None if scores is None else scores.data_ptr(), dl.status.data_ptr(),
        torch.cuda.current_stream().cuda_stream)
    return st


def test_noalloc_matches_the_workspace_entry_point_on_two_calls(cuda_lib):
    w = S.scaled(S.csa_b8_ctx32k(), (32768, 20001, 4099, 9), "noalloc", seed=5000)
    gen = S.generate(w, "cuda")
    lay, ls = gen["layers"][0], w.layers[0]
    seq = gen["seq_len"]
    dl = T.gpu_layer(cuda_lib, w, lay, ls)
    stride = cuda_lib.score_stride(dl.cfg, dl.max_seq_len)
    for call in range(2):
        q = lay["q"] if call == 0 else (lay["q"] * -1.5 + 0.25).contiguous()
        ref_scores = torch.full((w.batch, stride), float("nan"), device="cuda")
        dl.select(seq, q, scores=ref_scores)
        ref_idx, ref_cnt = dl.idx.clone(), dl.cnt.clone()
        idx = torch.full_like(dl.idx, -7)
        cnt = torch.full_like(dl.cnt, -7)
        scores = torch.full((w.batch, stride), float("nan"), device="cuda")
        assert _noalloc(cuda_lib, dl, seq, q, idx, cnt, scores) == cuda_lib.CKV_OK
        assert T.status_word(dl) == 0
        assert torch.equal(cnt, ref_cnt)
        assert torch.equal(idx, ref_idx)          # index output: bit-exact
        for b, L in enumerate(w.seq_lens):
            n = L // ls.ratio
            a, r = scores[b, :n].cpu().numpy(), ref_scores[b, :n].cpu().numpy()
            if n:
                assert np.max(np.abs(a - r)) <= 1e-5 * max(np.max(np.abs(r)), 1e-30)


def test_noalloc_without_a_score_buffer_matches_on_two_calls(cuda_lib):
    """With no score buffer the scores themselves live in the shared scratch array (its largest
    region). The selection must equal the workspace entry point's, bit for bit, on two calls in a
    row with different queries and lengths."""
    w = S.scaled(S.csa_b8_ctx32k(), (65536, 40001, 131, 12289, 5), "noalloc_noscores", seed=5002)
    gen = S.generate(w, "cuda")
    lay, ls = gen["layers"][0], w.layers[0]
    dl = T.gpu_layer(cuda_lib, w, lay, ls)
    for call in range(2):
        seq = gen["seq_len"] if call == 0 else (gen["seq_len"] - 3).clamp(min=1).to(torch.int32)
        q = lay["q"] if call == 0 else (lay["q"] * 0.75 - 0.5).contiguous()
        dl.select(seq, q)
        ref_idx, ref_cnt = dl.idx.clone(), dl.cnt.clone()
        idx = torch.full_like(dl.idx, -7)
        cnt = torch.full_like(dl.cnt, -7)
        assert _noalloc(cuda_lib, dl, seq, q, idx, cnt, None) == cuda_lib.CKV_OK
        assert T.status_word(dl) == 0
        assert torch.equal(cnt, ref_cnt), f"call {call}: counts differ"
        assert torch.equal(idx, ref_idx), f"call {call}: selections differ"


def test_noalloc_refuses_sizes_beyond_its_scratch(cuda_lib):
    # 64 requests of 1M tokens need far more than 16 MiB of selection scratch
    w = S.scaled(S.csa_b8_ctx32k(), (1000,) * 2, "noalloc_small", seed=5001)
    gen = S.generate(w, "cuda")
    lay, ls = gen["layers"][0], w.layers[0]
    dl = T.gpu_layer(cuda_lib, w, lay, ls)
    cfg = dl.cfg.c()
    need = cuda_lib.indexer_workspace_bytes(dl.cfg, 64, 1 << 20, 2048)
    assert need > 16 << 20
    big = cuda_lib.load_library().sparse_indexer_topk_noalloc(
        ctypes.byref(cfg), ctypes.byref(dl.cache.c()), 64, gen["seq_len"].data_ptr(), 1 << 20,
        lay["q"].data_ptr(), 2048, dl.idx.data_ptr(), dl.cnt.data_ptr(), None, dl.status.data_ptr(),
        None)
    assert big == cuda_lib.CKV_ERR_WORKSPACE
