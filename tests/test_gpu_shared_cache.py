"""One compressed cache written by one layer and read by several.

aidevelopers.cz "DeepSeek-V4.1-Flash ve vLLM", section "Polovina vrstev nemusí číst celý prompt":
a global compressed cache is produced once and read by many layers. With this library that is a
matter of passing the same pools, tables and residue to the calls: one layer (the owner) appends,
the others only select and attend with their own queries (one sparse reader with its own top-k,
one dense reader). Every reader must match the oracle on the cache the owner built.
"""

import numpy as np
import pytest
import torch

import compressed_kv_sparse_compress_b200 as ckv
from oracle import ckv_oracle as O
from synth import workloads as S
from tests import ckv_testlib as T

pytestmark = pytest.mark.gpu


def test_layers_sharing_one_nvfp4_cache_match_the_oracle(cuda_lib):
    lens = (20001, 4099, 16385, 777)
    w = S.Workload("shared_cache", lens, 64, 512, 64, 128, (S.LayerSpec(4, 256, "nvfp4", "fp8"),),
                   paged=True, from_scratch=False, seed=7000)
    gen = S.generate(w, "cuda")
    lay, ls = gen["layers"][0], w.layers[0]
    seq = gen["seq_len"]
    owner = T.gpu_layer(cuda_lib, w, lay, ls)
    T.gpu_setup(owner, lay)
    owner.step(seq, (seq - 1).to(torch.int32), lay["q"], lay["kv_new"], lay["logit_new"])
    assert T.status_word(owner) == 0

    # readers: the owner's cache object, their own buffers and queries
    g = torch.Generator(device="cuda").manual_seed(7001)
    sparse = ckv.DecodeLayer(owner.cfg, owner.cache, w.batch, max(lens), 64)
    dense = ckv.DecodeLayer(owner.cfg, owner.cache, w.batch, max(lens), None)
    q_sparse = torch.randn(lay["q"].shape, generator=g, device="cuda")
    q_dense = torch.randn(lay["q"].shape, generator=g, device="cuda")
    sparse.select(seq, q_sparse)
    out_sparse = sparse.attend(seq, q_sparse).cpu().numpy()
    out_dense = dense.attend(seq, q_dense).cpu().numpy()
    assert T.status_word(sparse) == 0 and T.status_word(dense) == 0

    cfg = T.oracle_cfg(w, ls)
    oc = T.oracle_cache(lay)
    T.oracle_setup(cfg, oc, lay, w.batch)
    T.oracle_append_decode_token(cfg, oc, lay, lens)
    qs, qd = q_sparse.cpu().numpy(), q_dense.cpu().numpy()
    idx, cnt = sparse.idx.cpu().numpy(), sparse.cnt.cpu().numpy()
    for b, L in enumerate(lens):
        s64 = O.indexer_scores(cfg, oc, b, qs[b], L)
        ok, msg = T.topk_sets_match(idx[b], int(cnt[b]), s64, 64)
        assert ok, msg
        ref = O.attention(cfg, oc, b, qs[b], L, idx[b, :cnt[b]])
        assert T.max_rel_err(out_sparse[b], ref) <= 2e-2, b
        ref = O.attention(cfg, oc, b, qd[b], L, np.arange(L // 4))
        assert T.max_rel_err(out_dense[b], ref) <= 2e-2, b
