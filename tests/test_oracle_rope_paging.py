"""Pins of the oracle's rotary embedding, paged addressing and block pool."""

import numpy as np
import pytest

from oracle import ckv_oracle as O


def rope_complex(x, pos, d_r, base, inverse=False):
    """Independent formulation: pair (a, b) is the complex number a + ib, multiplied by
    exp(i * pos * base^(-2i/d_r))."""
    x = np.array(x, dtype=np.float64, copy=True)
    if d_r == 0:
        return x
    d = x.shape[-1]
    z = x[..., d - d_r::2] + 1j * x[..., d - d_r + 1::2]
    k = np.arange(d_r // 2)
    theta = np.array([base ** (-(2.0 * i) / d_r) for i in k])
    ang = np.multiply.outer(np.asarray(pos, dtype=np.float64), theta) * (-1 if inverse else 1)
    z = z * np.exp(1j * ang)
    x[..., d - d_r::2] = z.real
    x[..., d - d_r + 1::2] = z.imag
    return x


@pytest.mark.parametrize("d,d_r", [(16, 8), (128, 32), (512, 64)])
def test_rope_matches_complex_formulation(d, d_r):
    rng = np.random.default_rng(d)
    x = rng.normal(size=(5, d))
    pos = np.array([0, 1, 77, 4095, 1048575])
    got = O.rope_apply(x, pos, d_r, 10000.0)
    ref = rope_complex(x, pos, d_r, 10000.0)
    # an fp64 angle near 2^20 rad has an ulp of 2^-32 ~ 2.3e-10 rad: the two formulations may
    # round the angle (and reduce it for cos/sin) one ulp apart
    assert np.allclose(got, ref, rtol=0, atol=1e-9)
    assert np.array_equal(got[:, : d - d_r], x[:, : d - d_r])


def test_rope_inverse_norm_and_identities():
    rng = np.random.default_rng(1)
    x = rng.normal(size=(7, 64))
    pos = rng.integers(0, 2 ** 20, size=7)
    y = O.rope_apply(x, pos, 32, 10000.0)
    assert np.allclose(O.rope_apply(y, pos, 32, 10000.0, inverse=True), x, atol=1e-12)
    assert np.allclose(np.linalg.norm(y, axis=1), np.linalg.norm(x, axis=1), rtol=1e-13)
    assert np.array_equal(O.rope_apply(x, pos, 0, 10000.0), x)
    assert np.allclose(O.rope_apply(x, 0, 32, 10000.0), x, atol=0)


def test_rope_relative_position_property():
    rng = np.random.default_rng(2)
    q = rng.normal(size=64)
    k = rng.normal(size=64)
    for p, s, shift in [(10, 3, 1000), (4095, 17, 12345), (70000, 69999, 5)]:
        a = O.rope_apply(q, p, 64, 10000.0) @ O.rope_apply(k, s, 64, 10000.0)
        b = O.rope_apply(q, p + shift, 64, 10000.0) @ O.rope_apply(k, s + shift, 64, 10000.0)
        assert a == pytest.approx(b, abs=1e-9)


def test_rope_inv_freq_endpoints():
    f = O.rope_inv_freq(64, 10000.0)
    assert f[0] == 1.0
    assert f[-1] == pytest.approx(10000.0 ** (-62 / 64), rel=1e-15)
    assert np.all(np.diff(f) < 0)


@pytest.mark.parametrize("ratio", [1, 2, 4, 8, 64, 128, 256])
def test_comp_entry_rows_brute_force(ratio):
    # brute force from token positions: entry i holds tokens [i*r, (i+1)*r), all in logical
    # block (i*r)//256; within a physical block entries are stored in order of first token.
    rng = np.random.default_rng(ratio)
    n_lblk = 6
    table = rng.permutation(20)[:n_lblk].astype(np.int32)
    epb = 256 // ratio
    n_entries = n_lblk * 256 // ratio
    for i in range(n_entries):
        first_tok = i * ratio
        lblk = first_tok // 256
        assert all((t // 256) == lblk for t in range(first_tok, first_tok + ratio))
        slot = (first_tok % 256) // ratio
        assert O.comp_entry_rows(table, [i], ratio)[0] == table[lblk] * epb + slot


def test_window_rows_and_identity_table():
    table = np.arange(8, dtype=np.int32)
    t = np.arange(8 * 256)
    assert np.array_equal(O.window_token_rows(table, t), t)
    assert np.array_equal(O.comp_entry_rows(table, np.arange(512), 4), np.arange(512))
    with pytest.raises(ValueError):
        O.window_token_rows(np.array([-1, 3], dtype=np.int32), [10])


def test_relocated_blocks_decode_identically():
    rng = np.random.default_rng(3)
    cfg = O.LayerCfg(4, 32, 8, 4, 16, "bf16", "fp8")
    n_blk = 5
    codes = rng.integers(0, 2 ** 16, size=(n_blk, 64, 32), dtype=np.uint16).view(np.uint8)
    codes = codes.reshape(n_blk, 64, 64)
    wcodes = rng.integers(0, 0x7E, size=(n_blk, 256, 32), dtype=np.uint8)
    wsc = rng.uniform(0.5, 1.5, size=(n_blk, 256)).astype(np.float32)
    ident = np.arange(n_blk, dtype=np.int32)[None]
    a = O.LayerCache(codes, None, wcodes, wsc, ident, ident)
    perm = rng.permutation(n_blk).astype(np.int32)          # logical l -> physical perm[l]
    codes2 = np.empty_like(codes)
    wcodes2 = np.empty_like(wcodes)
    wsc2 = np.empty_like(wsc)
    codes2[perm] = codes
    wcodes2[perm] = wcodes
    wsc2[perm] = wsc
    b = O.LayerCache(codes2, None, wcodes2, wsc2, perm[None], perm[None])
    e = np.arange(n_blk * 64)
    assert np.array_equal(O.decode_comp_entries(cfg, a, 0, e), O.decode_comp_entries(cfg, b, 0, e),
                          equal_nan=True)  # random 16-bit patterns include bf16 NaNs
    t = np.arange(n_blk * 256)
    assert np.array_equal(O.decode_window_tokens(cfg, a, 0, t), O.decode_window_tokens(cfg, b, 0, t))


def test_block_pool_lifo_and_errors():
    p = O.BlockPool(5)
    assert p.alloc(2) == [0, 1]
    assert p.alloc(1) == [2]
    p.free([1, 0])
    assert p.alloc(1) == [0]          # last freed comes back first
    assert p.alloc(3) == [1, 3, 4]
    assert p.alloc(1) is None         # exhausted: all-or-nothing
    assert p.num_free == 0
    with pytest.raises(ValueError):
        p.free([7])
    p.free([4])
    with pytest.raises(ValueError):
        p.free([4])                   # double free
    with pytest.raises(ValueError):
        p.free([2, 2])
    assert p.alloc(2) is None and p.num_free == 1
