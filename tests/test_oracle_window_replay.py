"""Pins of the oracle's SWA bounded replay (aidevelopers.cz "DeepSeek-V4.1-Flash ve vLLM", section
"Proč je obnova sliding-window cache drahá": after a prefix-cache hit only the last window is
replayed and its dependence on older positions is cut).

Each pin is an invariant or a value computed here independently of the oracle's own helpers:
replaying the tokens a full append already wrote changes no byte; replaying other tokens leaves
every compressed byte and every window row outside the window as it was, and stores the new
tokens' rotations (complex-number rotary embedding) within the FP8 step; the residue it rebuilds
is the one the next append folds (weights and sum written out here)."""

import copy

import numpy as np
import pytest

from oracle import ckv_oracle as O
from tests.test_oracle_compressor import empty_cache
from tests.test_oracle_rope_paging import rope_complex


def _filled(cfg, L, seed, batch=1):
    """A cache of `batch` requests with L tokens each appended from scratch, and the raw tokens."""
    rng = np.random.default_rng(seed)
    c = empty_cache(cfg, L + 1, batch)
    kv = rng.normal(size=(batch, L, cfg.head_dim)).astype(np.float32)
    lg = rng.normal(size=(batch, L)).astype(np.float32)
    for b in range(batch):
        O.append_tokens(cfg, c, b, 0, kv[b], lg[b])
    return c, kv, lg


CFGS = [
    O.LayerCfg(4, 64, 32, 4, 128, "bf16", "fp8"),
    O.LayerCfg(4, 64, 32, 128, 128, "nvfp4", "fp8"),
    O.LayerCfg(2, 32, 16, 4, 16, "f32", "f32"),
    O.LayerCfg(2, 32, 16, 8, 128, "bf16", "f32"),
]


@pytest.mark.parametrize("cfg", CFGS, ids=lambda c: f"r{c.ratio}_w{c.window}_{c.comp_dtype}_{c.win_dtype}")
@pytest.mark.parametrize("L", [1000, 1027, 77, 3])
def test_replaying_the_appended_tokens_changes_nothing(cfg, L):
    c, kv, lg = _filled(cfg, L, 10 + L, batch=2)
    before = copy.deepcopy(c)
    n_w = min(cfg.window, L)
    for b in range(2):
        O.window_replay(cfg, c, b, L, kv[b, L - n_w:], lg[b, L - n_w:])
    assert np.array_equal(c.comp_codes, before.comp_codes)
    if c.comp_scales is not None:
        assert np.array_equal(c.comp_scales, before.comp_scales)
    assert np.array_equal(c.win_codes, before.win_codes)
    if c.win_scales is not None:
        assert np.array_equal(c.win_scales, before.win_scales)
    for b in range(2):
        assert [p for p, _, _ in c.residue[b]] == [p for p, _, _ in before.residue[b]]
        for (p0, x0, l0), (p1, x1, l1) in zip(c.residue[b], before.residue[b]):
            assert np.array_equal(x0, x1) and l0 == l1
        # the residue is exactly the unfinished group
        assert [p for p, _, _ in c.residue[b]] == list(range((L // cfg.ratio) * cfg.ratio, L))


@pytest.mark.parametrize("cfg", CFGS[:3], ids=lambda c: f"r{c.ratio}_{c.comp_dtype}_{c.win_dtype}")
def test_replaying_other_tokens_rewrites_only_the_window(cfg):
    L = 1000
    c, kv, lg = _filled(cfg, L, 20)
    before = copy.deepcopy(c)
    rng = np.random.default_rng(21)
    n_w = min(cfg.window, L)
    new_kv = (rng.normal(size=(n_w, cfg.head_dim)) * 3.0).astype(np.float32)
    new_lg = rng.normal(size=n_w).astype(np.float32)
    O.window_replay(cfg, c, 0, L, new_kv, new_lg)
    # compressed entries come from the prefix cache: untouched
    assert np.array_equal(c.comp_codes, before.comp_codes)
    if c.comp_scales is not None:
        assert np.array_equal(c.comp_scales, before.comp_scales)
    # window positions [L - n_w, L) hold the new tokens rotated at their positions
    got = O.decode_window_tokens(cfg, c, 0, np.arange(L - n_w, L))
    want = np.stack([rope_complex(new_kv[i].astype(np.float64), L - n_w + i, cfg.rope_dim, 10000.0)
                     for i in range(n_w)])
    if cfg.win_dtype == "f32":
        assert np.array_equal(got, want.astype(np.float32).astype(np.float64))
    else:  # within half of e4m3's step (1/16 relative) of each element, relative to the token max
        amax = np.max(np.abs(want), axis=1, keepdims=True)
        assert np.all(np.abs(got - want) <= amax / 448.0 * 16.0 + 1e-6 * amax)
    # the window rows of older positions are the ones the appends wrote
    older = np.arange(max(0, L - 256), L - n_w)
    if older.size:
        assert np.array_equal(O.decode_window_tokens(cfg, c, 0, older), O.decode_window_tokens(cfg, before, 0, older))


def test_the_next_append_folds_the_replayed_residue():
    """L = 1023 leaves positions 1020..1022 unfinished (r = 4). After a replay with new tokens, the
    append of position 1023 completes the group: its entry is the softmax-weighted sum of the
    three replayed tokens and the new one, each rotated at its position (f32 storage: exact up to
    the fp64 -> fp32 rounding)."""
    cfg = O.LayerCfg(2, 32, 16, 4, 128, "f32", "f32")
    L = 1023
    c, kv, lg = _filled(cfg, L, 30)
    rng = np.random.default_rng(31)
    new_kv = rng.normal(size=(128, 32)).astype(np.float32)
    new_lg = rng.normal(size=128).astype(np.float32)
    O.window_replay(cfg, c, 0, L, new_kv, new_lg)
    tok = rng.normal(size=(1, 32)).astype(np.float32)
    tlg = np.array([0.7], dtype=np.float32)
    O.append_tokens(cfg, c, 0, L, tok, tlg)
    xs = [new_kv[125], new_kv[126], new_kv[127], tok[0]]
    ls = np.array([new_lg[125], new_lg[126], new_lg[127], tlg[0]], dtype=np.float64)
    e = np.exp(ls - ls.max())
    w = e / e.sum()
    want = sum(w[i] * rope_complex(xs[i].astype(np.float64), 1020 + i, 16, 10000.0) for i in range(4))
    got = O.decode_comp_entries(cfg, c, 0, [255])[0]
    assert np.array_equal(got, want.astype(np.float32).astype(np.float64))
    # the entries before it are the prefix's
    assert np.array_equal(O.decode_comp_entries(cfg, c, 0, np.arange(255)),
                          O.decode_comp_entries(cfg, _filled(cfg, L, 30)[0], 0, np.arange(255)))


def test_a_context_shorter_than_the_window_is_replayed_whole():
    cfg = O.LayerCfg(2, 32, 16, 4, 128, "bf16", "fp8")
    L = 10
    c, kv, lg = _filled(cfg, L, 40)
    rng = np.random.default_rng(41)
    new_kv = rng.normal(size=(L, 32)).astype(np.float32)
    O.window_replay(cfg, c, 0, L, new_kv, rng.normal(size=L).astype(np.float32))
    assert [p for p, _, _ in c.residue[0]] == [8, 9]
    assert np.array_equal(c.residue[0][0][1], new_kv[8]) and np.array_equal(c.residue[0][1][1], new_kv[9])
