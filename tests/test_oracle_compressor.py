"""Pins of the oracle's compressor and append: special cases with exact answers."""

import numpy as np
import pytest
import scipy.special

from oracle import ckv_oracle as O
from tests.test_oracle_rope_paging import rope_complex


def empty_cache(cfg, n_tokens, batch=1):
    n_blk = -(-n_tokens // 256)
    epb = cfg.entries_per_block
    cb = O.comp_entry_code_bytes(cfg)
    wb = O.win_token_code_bytes(cfg)
    comp = np.zeros((batch * n_blk, epb, cb), dtype=np.uint8)
    scales = np.zeros((batch * n_blk, epb, cfg.head_dim // 16), dtype=np.uint8) \
        if cfg.comp_dtype == "nvfp4" else None
    win = np.zeros((batch * n_blk, 256, wb), dtype=np.uint8)
    wsc = np.zeros((batch * n_blk, 256), dtype=np.float32) if cfg.win_dtype == "fp8" else None
    table = np.arange(batch * n_blk, dtype=np.int32).reshape(batch, n_blk)
    return O.LayerCache(comp, scales, win, wsc, table, table.copy())


def stored_rotated(kv, pos, d_r):
    return rope_complex(kv.astype(np.float64), pos, d_r, 10000.0).astype(np.float32)


def test_softmax_weights_match_scipy():
    rng = np.random.default_rng(0)
    for r in [1, 4, 128]:
        lg = rng.normal(size=r) * 3
        w = O.softmax_weights(lg)
        assert np.allclose(w, scipy.special.softmax(lg), rtol=1e-14, atol=0)
        assert np.sum(w) == pytest.approx(1.0, abs=1e-15)


def test_ratio_one_stores_each_rotated_token():
    cfg = O.LayerCfg(2, 32, 16, 1, 8, "f32", "f32")
    rng = np.random.default_rng(1)
    L = 300
    kv = rng.normal(size=(L, 32)).astype(np.float32)
    lg = rng.normal(size=L).astype(np.float32)
    c = empty_cache(cfg, L)
    O.append_tokens(cfg, c, 0, 0, kv, lg)
    got = O.decode_comp_entries(cfg, c, 0, np.arange(L))
    ref = stored_rotated(kv, np.arange(L), 16).astype(np.float64)
    assert np.array_equal(got, ref)
    assert c.residue[0] == []


@pytest.mark.parametrize("ratio", [4, 128])
def test_one_hot_weights_select_a_token(ratio):
    cfg = O.LayerCfg(2, 64, 32, ratio, 0, "f32", "f32")
    rng = np.random.default_rng(ratio)
    groups = 3
    L = groups * ratio
    kv = rng.normal(size=(L, 64)).astype(np.float32)
    chosen = rng.integers(0, ratio, size=groups)
    lg = np.full(L, -np.inf, dtype=np.float32)
    for g, t in enumerate(chosen):
        lg[g * ratio + t] = 0.0
    c = empty_cache(cfg, L)
    O.append_tokens(cfg, c, 0, 0, kv, lg)
    for g, t in enumerate(chosen):
        p = g * ratio + t
        got = O.decode_comp_entries(cfg, c, 0, [g])[0]
        assert np.array_equal(got, stored_rotated(kv[p], p, 32).astype(np.float64))


def test_equal_logits_give_the_group_mean():
    cfg = O.LayerCfg(2, 64, 32, 4, 0, "f32", "f32")
    rng = np.random.default_rng(2)
    kv = rng.normal(size=(8, 64)).astype(np.float32)
    lg = np.full(8, 0.7, dtype=np.float32)
    c = empty_cache(cfg, 8)
    O.append_tokens(cfg, c, 0, 0, kv, lg)
    for g in range(2):
        rot = rope_complex(kv[4 * g:4 * g + 4].astype(np.float64), np.arange(4 * g, 4 * g + 4),
                           32, 10000.0)
        mean = rot.mean(axis=0).astype(np.float32).astype(np.float64)
        assert np.allclose(O.decode_comp_entries(cfg, c, 0, [g])[0], mean, rtol=0, atol=1e-6)


def test_compress_group_is_the_weighted_sum():
    rng = np.random.default_rng(3)
    x = rng.normal(size=(4, 16))
    lg = rng.normal(size=4)
    w = scipy.special.softmax(lg)
    ref = [sum(w[t] * x[t, d] for t in range(4)) for d in range(16)]
    assert np.allclose(O.compress_group(x, lg), ref, rtol=0, atol=1e-14)


@pytest.mark.parametrize("comp,win", [("f32", "f32"), ("bf16", "fp8"), ("nvfp4", "fp8")])
def test_split_appends_equal_one_append(comp, win):
    cfg = O.LayerCfg(2, 64, 16, 4, 16, comp, win)
    rng = np.random.default_rng(4)
    L = 523
    kv = rng.normal(size=(L, 64)).astype(np.float32)
    lg = rng.normal(size=L).astype(np.float32)
    a = empty_cache(cfg, L)
    O.append_tokens(cfg, a, 0, 0, kv, lg)
    b = empty_cache(cfg, L)
    cuts = [0, 1, 2, 7, 100, 101, 400, 522, L]
    for s, e in zip(cuts[:-1], cuts[1:]):
        O.append_tokens(cfg, b, 0, s, kv[s:e], lg[s:e])
    # the window writes differ only for tokens that fell out of the window in between
    assert np.array_equal(a.comp_codes, b.comp_codes)
    if comp == "nvfp4":
        assert np.array_equal(a.comp_scales, b.comp_scales)
    t = np.arange(L - 16, L)
    assert np.array_equal(O.decode_window_tokens(cfg, a, 0, t), O.decode_window_tokens(cfg, b, 0, t))
    assert len(a.residue[0]) == L % 4 and [p for p, _, _ in a.residue[0]] == [520, 521, 522]


def test_window_holds_the_last_w_rotated_tokens():
    cfg = O.LayerCfg(2, 64, 16, 4, 10, "f32", "fp8")
    rng = np.random.default_rng(5)
    L = 37
    kv = rng.normal(size=(L, 64)).astype(np.float32)
    lg = rng.normal(size=L).astype(np.float32)
    c = empty_cache(cfg, L)
    O.append_tokens(cfg, c, 0, 0, kv, lg)
    rows = O.window_token_rows(c.win_table[0], np.arange(L))
    flat = c.win_codes.reshape(-1, 64)
    for t in range(L):
        if t < L - 10:
            assert not np.any(flat[rows[t]])
        else:
            codes, s = O.quantize_fp8_token(stored_rotated(kv[t], t, 16))
            assert np.array_equal(flat[rows[t]], codes)
            assert c.win_scales.reshape(-1)[rows[t]] == s


def test_residue_mismatch_is_rejected():
    cfg = O.LayerCfg(2, 16, 0, 4, 0, "f32", "f32")
    c = empty_cache(cfg, 16)
    O.append_tokens(cfg, c, 0, 0, np.zeros((3, 16), np.float32), np.zeros(3, np.float32))
    with pytest.raises(ValueError):
        O.append_tokens(cfg, c, 0, 4, np.zeros((1, 16), np.float32), np.zeros(1, np.float32))
