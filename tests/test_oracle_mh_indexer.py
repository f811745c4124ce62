"""Pins of the oracle's multi-head indexer: special cases whose scores are known in closed form.

The multi-head score is s_j = sum_h w_h * max(0, q^_h . k_j) with each head's index query stored
as FP8 (scale amax/448) and k_j an FP8 entry times its scale; the index keys of a group are folded with the softmax of
the group's logits. Each case below fails for one plausible slip: a dropped or misplaced ReLU,
weights indexed by the wrong axis, a query not quantised (or with the wrong scale), the entry
scale left out, the wrong group or weights in the fold, a residue lost between calls.
"""

import math

import numpy as np
import pytest

from oracle import ckv_oracle as O


def _cfg(ratio=4):
    return O.LayerCfg(4, 64, 0, ratio, 0, "f32", "f32")


def _pool(n_entries, d_i, ratio=4, batch=1):
    epb = 256 // ratio
    n_blk = -(-n_entries // epb)
    codes = np.zeros((batch * n_blk, epb, d_i), dtype=np.uint8)
    scales = np.ones((batch * n_blk, epb), dtype=np.float32)
    table = np.arange(batch * n_blk, dtype=np.int32).reshape(batch, n_blk)
    return O.IndexCache(codes, scales), table


def _store(ic, table, cfg, b, j, x, scale):
    """Entry j of request b := e4m3 codes of x (exactly representable values) with `scale`."""
    row = int(O.comp_entry_rows(table[b], [j], cfg.ratio)[0])
    ic.codes.reshape(-1, ic.codes.shape[-1])[row] = O.e4m3_encode_satfinite(np.asarray(x, np.float32))
    ic.scales.reshape(-1)[row] = scale


def test_one_hot_heads_pick_their_own_weight():
    # entry j = 2 * e_(j mod 16); head h looks only along e_h with strength c_h: the score of entry
    # j is w_m * c_m * 2 * scale for m = j mod 16, so a weight or query taken from the wrong head
    # gives another value
    cfg, d_i, n = _cfg(), 64, 48
    ic, table = _pool(n, d_i)
    for j in range(n):
        x = np.zeros(d_i)
        x[j % 16] = 2.0
        _store(ic, table, cfg, 0, j, x, 0.5)
    c = np.array([1 + h for h in range(16)], dtype=np.float32)         # one value per head: exact
    w = np.array([0.25 * (h + 3) for h in range(16)], dtype=np.float32)
    q = np.zeros((16, d_i), dtype=np.float32)
    q[np.arange(16), np.arange(16)] = c
    s = O.mh_indexer_scores(cfg, ic, table, 0, q, w, 4 * n)
    ref = np.array([w[j % 16] * c[j % 16] * 2.0 * 0.5 for j in range(n)])
    assert np.allclose(s, ref, rtol=1e-6, atol=0)   # c_h is 448 times its fp32 scale


def test_relu_drops_negative_dots_before_the_weights():
    # two heads with opposite queries and equal weights: sum_h max(0, .) = |q . k|, where a score
    # without the ReLU would be 0; a negative weight turns the clipped dot negative, where a ReLU
    # applied after the weight would give 0
    cfg, d_i = _cfg(), 64
    ic, table = _pool(8, d_i)
    rng = np.random.default_rng(5)
    xs = []
    for j in range(8):
        x = O.e4m3_decode(O.e4m3_encode_satfinite(rng.normal(size=d_i).astype(np.float32) * 4))
        xs.append(x)
        _store(ic, table, cfg, 0, j, x, 1.0)
    q1 = np.asarray(rng.integers(-8, 9, size=d_i), dtype=np.float32) * 32   # e4m3 values: scale 1 exact
    q1[0] = 448.0
    q = np.stack([q1, -q1])
    s = O.mh_indexer_scores(cfg, ic, table, 0, q, np.array([1.0, 1.0], np.float32), 32)
    dots = [float(np.dot(q1.astype(np.float64), x)) for x in xs]
    assert np.allclose(s, [abs(d) for d in dots], rtol=1e-15, atol=0)
    assert any(d < 0 for d in dots) and any(d > 0 for d in dots)
    s_neg = O.mh_indexer_scores(cfg, ic, table, 0, q[:1], np.array([-2.0], np.float32), 32)
    assert np.allclose(s_neg, [-2.0 * max(d, 0.0) for d in dots], rtol=1e-15, atol=0)


def test_query_is_stored_as_fp8_per_head():
    # head 0's query (1, 0.3, 0, ...) has scale 1/448: 0.3 * 448 = 134.4 lies between the e4m3
    # values 128 and 144 and rounds to 128, so the key e_1 scores 128/448, not 0.3; head 1's query
    # 0.3 e_1 alone has scale 0.3/448 and is exact. The scale is per head: a shared one would
    # round head 1 as well
    cfg, d_i = _cfg(), 64
    ic, table = _pool(4, d_i)
    x = np.zeros(d_i)
    x[1] = 1.0
    _store(ic, table, cfg, 0, 0, x, 1.0)
    q = np.zeros((2, d_i), dtype=np.float32)
    q[0, 0], q[0, 1], q[1, 1] = 1.0, 0.3, 0.3
    s0 = O.mh_indexer_scores(cfg, ic, table, 0, q[:1], np.array([1.0], np.float32), 4)
    assert s0[0] == pytest.approx(128.0 / 448.0, rel=1e-6)
    s1 = O.mh_indexer_scores(cfg, ic, table, 0, q, np.array([0.0, 1.0], np.float32), 4)
    assert s1[0] == pytest.approx(float(np.float32(0.3)), rel=1e-6)


def test_entry_scale_multiplies_the_score():
    cfg, d_i = _cfg(), 128
    ic, table = _pool(4, d_i)
    x = np.full(d_i, 0.5)
    _store(ic, table, cfg, 0, 0, x, 0.125)
    _store(ic, table, cfg, 0, 1, x, 3.0)
    q = np.ones((2, d_i), dtype=np.float32)
    s = O.mh_indexer_scores(cfg, ic, table, 0, q, np.array([1.0, 0.5], np.float32), 8)
    assert s[0] == pytest.approx(1.5 * 64 * 0.125, rel=1e-6)
    assert s[1] == pytest.approx(1.5 * 64 * 3.0, rel=1e-6)


def test_all_positive_dots_collapse_to_one_weighted_query():
    # when every dot is positive the ReLU is the identity and s_j = (sum_h w_h q^_h) . k_j
    cfg, d_i = _cfg(), 64
    ic, table = _pool(64, d_i)
    rng = np.random.default_rng(9)
    xs = []
    for j in range(64):
        x = O.e4m3_decode(O.e4m3_encode_satfinite(rng.uniform(0.5, 4.0, size=d_i).astype(np.float32)))
        xs.append(x)
        _store(ic, table, cfg, 0, j, x, 0.25)
    q = rng.uniform(0.1, 1.0, size=(8, d_i)).astype(np.float32)
    w = rng.uniform(-1.0, 1.0, size=8).astype(np.float32)
    s = O.mh_indexer_scores(cfg, ic, table, 0, q, w, 256)
    qhat = np.stack([O.dequant_fp8_token(*O.quantize_fp8_token(qh)) for qh in q])
    qbar = (w.astype(np.float64)[:, None] * qhat).sum(axis=0)
    ref = np.array([0.25 * float(qbar @ x) for x in xs])
    assert np.allclose(s, ref, rtol=1e-12, atol=1e-12)


def test_candidates_stop_at_the_last_completed_group():
    cfg, d_i = _cfg(), 64
    ic, table = _pool(16, d_i)
    q = np.ones((1, d_i), dtype=np.float32)
    for L in (1, 3, 4, 7, 8, 63):
        assert O.mh_indexer_scores(cfg, ic, table, 0, q, np.ones(1, np.float32), L).shape == (L // 4,)


# ------------------------------------------------------------------------------------------------
# index-key compressor
# ------------------------------------------------------------------------------------------------

@pytest.mark.parametrize("ratio", [4, 128])
def test_fold_uses_the_softmax_of_each_groups_logits(ratio):
    # keys and logits chosen so the folded entry is known: group g's keys are a_t * u with
    # logits l_t, so the entry is (sum_t softmax(l)_t a_t) * u
    cfg, d_i = _cfg(ratio), 64
    groups = 3
    ic, table = _pool(groups, d_i, ratio)
    rng = np.random.default_rng(ratio)
    u = np.zeros(d_i, dtype=np.float32)
    u[:4] = [1.0, -2.0, 0.5, 4.0]
    a = rng.uniform(-1, 1, size=groups * ratio)
    lg = rng.normal(size=groups * ratio).astype(np.float32)
    keys = (a[:, None] * u[None, :]).astype(np.float32)
    O.index_append_tokens(cfg, ic, table, 0, 0, keys, lg)
    got = O.decode_index_entries(cfg, ic, table, 0, np.arange(groups))
    for g in range(groups):
        sl = slice(g * ratio, (g + 1) * ratio)
        e = [math.exp(float(v)) for v in lg[sl].astype(np.float64)]
        coef = sum(ei * float(np.float32(a_t)) for ei, a_t in
                   zip(e, keys[sl, 0].astype(np.float64))) / sum(e)
        ref = coef * u.astype(np.float64)
        amax = np.max(np.abs(ref))
        # FP8 with scale amax/448: relative step 2^-3 at most, exact for the largest element
        assert np.all(np.abs(got[g] - ref) <= 2.0 ** -4 * np.abs(ref) + 1e-6 * amax)
        assert abs(abs(got[g][3]) - amax) <= 1e-6 * amax


def test_index_residue_carries_across_calls():
    cfg, d_i = _cfg(4), 64
    rng = np.random.default_rng(11)
    n = 4 * 25 + 3
    keys = rng.normal(size=(n, d_i)).astype(np.float32)
    lg = rng.normal(size=n).astype(np.float32)
    one, table = _pool(26, d_i)
    O.index_append_tokens(cfg, one, table, 0, 0, keys, lg)
    many, _ = _pool(26, d_i)
    pos = 0
    for step in (1, 2, 5, 1, 30, 7, 57):
        step = min(step, n - pos)
        O.index_append_tokens(cfg, many, table, 0, pos, keys[pos:pos + step], lg[pos:pos + step])
        pos += step
    assert pos == n
    assert np.array_equal(one.codes, many.codes) and np.array_equal(one.scales, many.scales)
    assert [p for p, _, _ in many.residue[0]] == [100, 101, 102]
    with pytest.raises(ValueError):
        O.index_append_tokens(cfg, many, table, 0, 104, keys[:1], lg[:1])


def test_index_entries_land_in_the_paged_rows():
    # a permuted table: entry i of request b lives in row table[b][(4 i) // 256] * 64 + i % 64
    cfg, d_i = _cfg(4), 64
    ic, _ = _pool(128, d_i, batch=2)
    table = np.array([[3, 1], [0, 2]], dtype=np.int32)
    keys = np.zeros((512, d_i), dtype=np.float32)
    keys[:, 0] = np.repeat(np.arange(128, dtype=np.float32) + 1, 4)  # entry i = (i + 1) e_0
    O.index_append_tokens(cfg, ic, table, 1, 0, keys, np.zeros(512, np.float32))
    flat = ic.codes.reshape(-1, d_i)
    sc = ic.scales.reshape(-1)
    for i in (0, 63, 64, 127):
        row = int(table[1][(4 * i) // 256]) * 64 + i % 64
        assert O.e4m3_decode(flat[row:row + 1])[0, 0] * sc[row] == pytest.approx(i + 1, rel=1e-6)
    assert not flat[table[0][0] * 64:(table[0][0] + 1) * 64].any()


def test_fp8_query_matches_torchs_e4m3_cast():
    # library pin of the query quantiser: codes from torch's float8_e4m3fn cast of q / s
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(21)
    q = rng.normal(size=(16, 128)).astype(np.float32) * rng.uniform(0.01, 100, size=(16, 1)).astype(np.float32)
    q[3] = 0.0
    got = O.index_query_fp8(q)
    for h in range(q.shape[0]):
        amax = np.float32(np.max(np.abs(q[h])))
        s = np.float32(amax / np.float32(448.0)) if amax > 0 else np.float32(1.0)
        x = torch.from_numpy(q[h] / s).to(torch.float8_e4m3fn).to(torch.float64).numpy()
        assert np.array_equal(got[h], x * np.float64(s))


def test_ratio_one_index_append_stores_each_key():
    # r = 1: every key is its own group (weight 1), so each entry is the key's FP8 storage
    cfg, d_i = _cfg(1), 128
    ic, table = _pool(300, d_i, ratio=1)
    rng = np.random.default_rng(23)
    keys = rng.normal(size=(300, d_i)).astype(np.float32)
    O.index_append_tokens(cfg, ic, table, 0, 0, keys, rng.normal(size=300).astype(np.float32))
    got = O.decode_index_entries(cfg, ic, table, 0, np.arange(300))
    for t in range(300):
        codes, s = O.quantize_fp8_token(keys[t])
        assert np.array_equal(got[t], O.dequant_fp8_token(codes, s))
    assert ic.residue[0] == []
