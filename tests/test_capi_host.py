"""Host-side tests of libckv: exports, block pools, sizes and argument validation (no GPU)."""

import ctypes
import os
import re

import numpy as np
import pytest

import compressed_kv_sparse_compress_b200 as ckv
from oracle import ckv_oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    src = open(os.path.join(ROOT, "include", "ckv.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\**\s+\**\s*([a-z_][a-z0-9_]*)\s*\(",
                                 src, flags=re.M)))


def test_library_exports_every_declared_symbol():
    lib = ckv.load_library()
    names = declared_functions()
    assert len(names) >= 14
    assert set(names) == set(ckv.EXPORTS)
    for n in names:
        assert hasattr(lib, n), n


def test_pool_matches_oracle_pool_on_random_sequences():
    rng = np.random.default_rng(0)
    for trial in range(20):
        n = int(rng.integers(1, 64))
        a = ckv.BlockPool(n)
        b = O.BlockPool(n)
        held = []
        for _ in range(200):
            if rng.random() < 0.55:
                k = int(rng.integers(0, 6))
                ra, rb = a.alloc(k), b.alloc(k)
                assert ra == rb
                if ra:
                    held.extend(ra)
            elif held:
                k = int(rng.integers(1, min(len(held), 5) + 1))
                pick = [held.pop(int(rng.integers(0, len(held)))) for _ in range(k)]
                a.free(pick)
                b.free(pick)
            assert a.num_free == b.num_free
        a.close()


def test_pool_errors():
    p = ckv.BlockPool(3)
    assert p.alloc(0) == []
    ids = p.alloc(3)
    assert ids == [0, 1, 2] and p.alloc(1) is None
    with pytest.raises(ckv.CkvError) as e:
        p.free([3])
    assert e.value.status == ckv.CKV_ERR_INVALID_ARG
    p.free([2])
    with pytest.raises(ckv.CkvError):
        p.free([2])          # double free
    with pytest.raises(ckv.CkvError):
        p.free([0, 0])       # repeated id: nothing freed
    assert p.num_free == 1
    with pytest.raises(ckv.CkvError):
        ckv.BlockPool(0)


@pytest.mark.parametrize("comp,win,d", [("f32", "f32", 128), ("bf16", "fp8", 512), ("nvfp4", "fp8", 512),
                                        ("nvfp4", "f32", 64)])
def test_row_bytes_match_the_oracle_layout(comp, win, d):
    cfg = ckv.LayerConfig(8, d, 16, 4, 128, comp, win)
    ocfg = O.LayerCfg(8, d, 16, 4, 128, comp, win)
    cb, cs, wb, ws = cfg.row_bytes()
    assert cb == O.comp_entry_code_bytes(ocfg)
    assert cs == (d // 16 if comp == "nvfp4" else 0)
    assert wb == O.win_token_code_bytes(ocfg)
    assert ws == (4 if win == "fp8" else 0)


def test_score_stride_and_workspace_sizes():
    cfg = ckv.LayerConfig(64, 512, 64, 4, 128, "bf16", "fp8")
    assert ckv.score_stride(cfg, 1048576) == 262144
    assert ckv.score_stride(cfg, 4099) == 1024          # floor(4099/4) = 1024, a multiple of 64
    assert ckv.score_stride(cfg, 4100) == 1088          # 1025 rounded up to 64
    small = ckv.indexer_workspace_bytes(cfg, 8, 32768, 512)
    big = ckv.indexer_workspace_bytes(cfg, 8, 1048576, 512)
    assert 0 < small < big
    assert ckv.attention_workspace_bytes(cfg, 8, 32768, 512) > 0
    assert ckv.attention_workspace_bytes(cfg, 8, 32768, 0) >= ckv.attention_workspace_bytes(cfg, 8, 32768, 512)


@pytest.mark.parametrize("field,value", [("ratio", 3), ("ratio", 512), ("window", 300), ("rope_dim", 7),
                                         ("rope_dim", 1024), ("head_dim", 100), ("num_heads", 0)])
def test_bad_configs_are_rejected(field, value):
    cfg = ckv.LayerConfig(8, 128, 32, 4, 128, "bf16", "fp8")
    setattr(cfg, field, value)
    with pytest.raises(ckv.CkvError) as e:
        cfg.row_bytes()
    assert e.value.status in (ckv.CKV_ERR_INVALID_ARG, ckv.CKV_ERR_UNSUPPORTED)
    assert ckv.indexer_workspace_bytes(cfg, 1, 1024, 16) == 0


def test_bad_dtype_pairs_are_unsupported():
    for comp, win in [("fp8", "fp8"), ("bf16", "nvfp4"), ("bf16", "bf16")]:
        cfg = ckv.LayerConfig(8, 128, 32, 4, 128, comp, win)
        with pytest.raises(ckv.CkvError) as e:
            cfg.row_bytes()
        assert e.value.status == ckv.CKV_ERR_UNSUPPORTED


def test_entry_points_reject_null_arguments_before_any_device_work():
    lib = ckv.load_library()
    cfg = ckv.LayerConfig(8, 128, 32, 4, 128, "bf16", "fp8").c()
    cache = ckv.LayerCacheC()  # all NULL
    st = lib.kv_compress_append(ctypes.byref(cfg), ctypes.byref(cache), 1, None, None, 1, 1024, None,
                                None, None, None)
    assert st == ckv.CKV_ERR_INVALID_ARG
    st = lib.sparse_indexer_topk(ctypes.byref(cfg), ctypes.byref(cache), 1, None, 1024, None, 4, None,
                                 None, None, None, 0, None, None)
    assert st == ckv.CKV_ERR_INVALID_ARG
    st = lib.compressed_window_attention(ctypes.byref(cfg), ctypes.byref(cache), 1, None, 1024, None,
                                         None, None, 0, None, None, 0, None, None)
    assert st == ckv.CKV_ERR_INVALID_ARG
    assert ckv.status_str(ckv.CKV_ERR_WORKSPACE) == "workspace too small"
    assert ckv.launch_count() == 0


def test_fused_step_workspace_and_argument_checks():
    cfg = ckv.LayerConfig(64, 512, 64, 4, 128, "bf16", "fp8")
    sparse = ckv.decode_step_workspace_bytes(cfg, 8, 32768, 512)
    dense = ckv.decode_step_workspace_bytes(cfg, 8, 32768, 0)
    # the fused step's workspace holds the indexer's and the attention's, each 256-byte aligned
    assert sparse >= ckv.indexer_workspace_bytes(cfg, 8, 32768, 512) + ckv.attention_workspace_bytes(cfg, 8, 32768, 512)
    assert dense == ckv.attention_workspace_bytes(cfg, 8, 32768, 0)
    assert ckv.decode_step_workspace_bytes(cfg, 8, 32768, -1) == 0
    bad = ckv.LayerConfig(8, 100, 32, 4, 128, "bf16", "fp8")
    assert ckv.decode_step_workspace_bytes(bad, 1, 1024, 16) == 0
    lib = ckv.load_library()
    cache = ckv.LayerCacheC()  # all NULL
    st = lib.ckv_decode_step(ctypes.byref(cfg.c()), ctypes.byref(cache), 1, None, 1024, None, None, None, 4,
                             None, None, None, None, 0, None, None)
    assert st == ckv.CKV_ERR_INVALID_ARG
    assert ckv.launch_count() == 0


def test_mh_indexer_workspace_and_argument_checks():
    cfg = ckv.LayerConfig(64, 512, 64, 4, 128, "bf16", "fp8")
    icfg = ckv.IndexConfig(64, 128)
    ws = ckv.mh_indexer_workspace_bytes(cfg, icfg, 8, 32768, 512)
    # the FP8 query images (8 x 64 x 128) and scaled head weights (8 x 64 fp32) ahead of the
    # head-averaged indexer's selection state
    assert ws == 8 * 64 * 128 + 8 * 64 * 4 + ckv.indexer_workspace_bytes(cfg, 8, 32768, 512)
    for heads, dim in [(8, 128), (72, 128), (144, 128), (64, 64), (64, 96), (64, 512), (0, 128)]:
        assert ckv.mh_indexer_workspace_bytes(cfg, ckv.IndexConfig(heads, dim), 8, 32768, 512) == 0
    assert ckv.mh_indexer_workspace_bytes(cfg, icfg, 8, 32768, 0) == 0
    lib = ckv.load_library()
    null_cache = ckv.LayerCacheC()
    null_icache = ckv.IndexCacheC()
    st = lib.sparse_mh_indexer_topk(ctypes.byref(cfg.c()), ctypes.byref(null_cache), ctypes.byref(icfg.c()),
                                    ctypes.byref(null_icache), 1, None, 1024, None, None, 4, None, None, None,
                                    None, 0, None, None)
    assert st == ckv.CKV_ERR_INVALID_ARG
    st = lib.kv_index_append(ctypes.byref(cfg.c()), ctypes.byref(null_cache), ctypes.byref(icfg.c()),
                             ctypes.byref(null_icache), 1, None, None, 1, 1024, None, None, None, None)
    assert st == ckv.CKV_ERR_INVALID_ARG
    # a layer cache that passes the host checks (16-byte aligned host buffers; nothing launches
    # because the index config is refused first)
    buf = np.zeros(64, dtype=np.uint8)
    base = (buf.ctypes.data + 15) // 16 * 16
    cache = ckv.LayerCacheC(base, None, base, base, base, base, base, base, 8, 1, 1)
    icache = ckv.IndexCacheC(base, base, base, base)
    for heads, dim, want in [(72, 128, ckv.CKV_ERR_UNSUPPORTED), (64, 100, ckv.CKV_ERR_UNSUPPORTED)]:
        st = lib.sparse_mh_indexer_topk(ctypes.byref(cfg.c()), ctypes.byref(cache),
                                        ctypes.byref(ckv.IndexConfig(heads, dim).c()), ctypes.byref(icache), 1,
                                        base, 1024, base, base, 4, base, base, None, base, 1 << 30, base, None)
        assert st == want
    st = lib.kv_index_append(ctypes.byref(cfg.c()), ctypes.byref(cache), ctypes.byref(icfg.c()),
                             ctypes.byref(ckv.IndexCacheC(base, base, None, None)), 1, base, None, 1, 1024, base,
                             base, base, None)
    assert st == ckv.CKV_ERR_INVALID_ARG  # the append needs the index rings
    st = lib.sparse_mh_indexer_topk(ctypes.byref(cfg.c()), ctypes.byref(cache), ctypes.byref(icfg.c()),
                                    ctypes.byref(icache), 4096, base, 1024, base, base, 4, base, base, None,
                                    base, 1 << 30, base, None)
    assert st == ckv.CKV_ERR_UNSUPPORTED  # batch above 2048
    hca = ckv.LayerConfig(64, 512, 64, 128, 128, "bf16", "fp8")
    st = lib.sparse_mh_indexer_topk(ctypes.byref(hca.c()), ctypes.byref(cache), ctypes.byref(icfg.c()),
                                    ctypes.byref(icache), 1, base, 1024, base, base, 4, base, base, None,
                                    base, 1 << 30, base, None)
    assert st == ckv.CKV_ERR_UNSUPPORTED  # 2 entries per pool block: runs of 64 do not fit
    assert ckv.launch_count() == 0
