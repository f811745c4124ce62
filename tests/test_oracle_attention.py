"""Pins of the oracle's indexer, top-k and attention: library routines, brute force and
closed forms."""

import math

import numpy as np
import pytest
import torch

from oracle import ckv_oracle as O
from tests.test_oracle_compressor import empty_cache, stored_rotated
from tests.test_oracle_rope_paging import rope_complex


def built_cache(cfg, L, seed):
    rng = np.random.default_rng(seed)
    kv = rng.normal(size=(L, cfg.head_dim)).astype(np.float32)
    lg = rng.normal(size=L).astype(np.float32)
    c = empty_cache(cfg, L)
    O.append_tokens(cfg, c, 0, 0, kv, lg)
    q = rng.normal(size=(cfg.num_heads, cfg.head_dim)).astype(np.float32)
    return c, kv, lg, q


# ---------------------------------------------------------------------------------- indexer


def test_indexer_scores_brute_force():
    cfg = O.LayerCfg(3, 16, 8, 2, 4, "bf16", "fp8")
    c, kv, lg, q = built_cache(cfg, 23, 0)
    L = 23
    got = O.indexer_scores(cfg, c, 0, q, L)
    qr = rope_complex(q.astype(np.float64), L - 1, 8, 10000.0)
    n = L // 2
    assert got.shape == (n,)
    for j in range(n):
        k = O.decode_comp_entries(cfg, c, 0, [j])[0]
        s = 0.0
        for h in range(3):
            s += sum(float(qr[h, d]) * float(k[d]) for d in range(16))
        s = s / 3 / math.sqrt(16)
        assert got[j] == pytest.approx(s, rel=1e-12, abs=1e-14)


def test_indexer_head_mean_collapses_to_one_dot():
    cfg = O.LayerCfg(64, 128, 32, 4, 0, "f32", "f32")
    c, kv, lg, q = built_cache(cfg, 1024, 1)
    s = O.indexer_scores(cfg, c, 0, q, 1024)
    qbar = rope_complex(q.astype(np.float64), 1023, 32, 10000.0).mean(axis=0)
    k = O.decode_comp_entries(cfg, c, 0, np.arange(256))
    assert np.allclose(s, (k @ qbar) / math.sqrt(128), rtol=1e-12, atol=1e-14)


def test_topk_matches_full_sort_brute_force():
    rng = np.random.default_rng(2)
    s = rng.normal(size=500).astype(np.float32)
    s[10] = s[20] = s[30] = np.float32(5.0)      # ties at the top
    for k in [0, 1, 2, 3, 64, 499, 500, 600]:
        ref = sorted(sorted(range(500), key=lambda j: (-float(s[j]), j))[:k])
        assert list(O.topk_select(s, k)) == ref
    assert list(O.topk_select(s, 2)) == [10, 20]     # the lower index wins a tie


def test_topk_decides_on_fp32_scores():
    # two fp64 scores that round to the same fp32 value tie, and the lower index wins
    s = np.array([1.0, 1.0 + 1e-12, 0.5])
    assert list(O.topk_select(s, 1)) == [0]


# -------------------------------------------------------------------------------- attention


def sdpa_mqa(q_rot, keys, scale, bias=None):
    """Plain multi-query attention by torch's reference SDPA in fp64 (keys are also values)."""
    qt = torch.from_numpy(np.asarray(q_rot, dtype=np.float64))[None, :, None, :]   # [1,H,1,D]
    k = torch.from_numpy(np.asarray(keys, dtype=np.float64))[None, None].expand(1, qt.shape[1], -1, -1)
    mask = None
    if bias is not None:
        mask = torch.from_numpy(np.asarray(bias, dtype=np.float64))[None, None, None, :]
    with torch.no_grad():
        o = torch.nn.functional.scaled_dot_product_attention(qt, k, k, attn_mask=mask, scale=scale)
    return o[0, :, 0, :].numpy()


@pytest.mark.parametrize("L", [1, 5, 64, 300])
def test_ratio_one_all_selected_no_window_is_plain_mqa(L):
    cfg = O.LayerCfg(4, 32, 16, 1, 0, "f32", "f32")
    c, kv, lg, q = built_cache(cfg, L, 10 + L)
    sel, scores, out = O.decode_layer(cfg, c, 0, q, L, top_k=L)
    assert list(sel) == list(range(L))
    keys = stored_rotated(kv, np.arange(L), 16).astype(np.float64)
    q_rot = rope_complex(q.astype(np.float64), L - 1, 16, 10000.0)
    ref = rope_complex(sdpa_mqa(q_rot, keys, 1 / math.sqrt(32)), L - 1, 16, 10000.0, inverse=True)
    assert np.allclose(out, ref, rtol=0, atol=1e-12)


@pytest.mark.parametrize("L,W", [(50, 8), (300, 128), (20, 128)])
def test_window_duplicates_add_ln2_to_their_logits(L, W):
    # r=1, every entry selected and a window of W: each of the last min(L, W) tokens is a key
    # twice, which is plain MQA with +ln 2 on those tokens' logits.
    cfg = O.LayerCfg(4, 32, 16, 1, W, "f32", "f32")
    c, kv, lg, q = built_cache(cfg, L, 20 + L)
    _, _, out = O.decode_layer(cfg, c, 0, q, L, top_k=None)
    keys = stored_rotated(kv, np.arange(L), 16).astype(np.float64)
    bias = np.zeros(L)
    bias[L - min(L, W):] = math.log(2.0)
    q_rot = rope_complex(q.astype(np.float64), L - 1, 16, 10000.0)
    ref = rope_complex(sdpa_mqa(q_rot, keys, 1 / math.sqrt(32), bias), L - 1, 16, 10000.0, inverse=True)
    assert np.allclose(out, ref, rtol=0, atol=1e-12)


def test_single_key_returns_the_token():
    # no completed entry (r > L) and a window of one: the only key is the decode token, whose
    # rotation is undone by the inverse rotation of the output.
    cfg = O.LayerCfg(3, 64, 32, 8, 1, "f32", "f32")
    c, kv, lg, q = built_cache(cfg, 5, 3)
    _, _, out = O.decode_layer(cfg, c, 0, q, 5, top_k=4)
    for h in range(3):
        assert np.allclose(out[h], kv[4].astype(np.float64), rtol=0, atol=1e-6)


def test_attention_brute_force_paged_quantized():
    cfg = O.LayerCfg(2, 16, 8, 2, 3, "bf16", "fp8")
    c, kv, lg, q = built_cache(cfg, 21, 4)
    L = 21
    sel, scores, out = O.decode_layer(cfg, c, 0, q, L, top_k=4)
    ref_sel = sorted(sorted(range(10), key=lambda j: (-float(np.float32(scores[j])), j))[:4])
    assert list(sel) == ref_sel
    keys = [O.decode_comp_entries(cfg, c, 0, [j])[0] for j in sel]
    keys += [O.decode_window_tokens(cfg, c, 0, [t])[0] for t in range(L - 3, L)]
    qr = rope_complex(q.astype(np.float64), L - 1, 8, 10000.0)
    for h in range(2):
        logit = [sum(qr[h, d] * k[d] for d in range(16)) / 4.0 for k in keys]
        m = max(logit)
        e = [math.exp(x - m) for x in logit]
        z = sum(e)
        o = [sum(e[j] * keys[j][d] for j in range(len(keys))) / z for d in range(16)]
        o = rope_complex(np.array(o), L - 1, 8, 10000.0, inverse=True)
        assert np.allclose(out[h], o, rtol=0, atol=1e-12)


def test_entry_order_does_not_matter():
    cfg = O.LayerCfg(4, 64, 32, 4, 16, "nvfp4", "fp8")
    c, kv, lg, q = built_cache(cfg, 400, 5)
    e = np.array([3, 17, 40, 41, 99])
    a = O.attention(cfg, c, 0, q, 400, e)
    b = O.attention(cfg, c, 0, q, 400, e[::-1])
    assert np.allclose(a, b, rtol=0, atol=1e-13)


def test_split_softmax_merged_by_log_sum_exp_is_the_joint_softmax():
    # the identity a split-KV kernel relies on: partial (max, sum, unnormalised output) over
    # disjoint key sets, merged, equal the one softmax over their union
    cfg = O.LayerCfg(4, 64, 32, 4, 16, "bf16", "fp8")
    c, kv, lg, q = built_cache(cfg, 500, 6)
    L = 500
    e = np.arange(0, 125, 3)
    joint = O.attention(cfg, c, 0, q, L, e)
    qr = rope_complex(q.astype(np.float64), L - 1, 32, 10000.0)
    x = np.concatenate([O.decode_comp_entries(cfg, c, 0, e),
                        O.decode_window_tokens(cfg, c, 0, np.arange(L - 16, L))])
    parts = [x[:10], x[10:30], x[30:]]
    ms, ls, os_ = [], [], []
    for p in parts:
        lo = (qr @ p.T) / 8.0
        m = lo.max(axis=1)
        w = np.exp(lo - m[:, None])
        ms.append(m)
        ls.append(w.sum(axis=1))
        os_.append(w @ p)
    M = np.max(ms, axis=0)
    Z = sum(l * np.exp(m - M) for m, l in zip(ms, ls))
    o = sum(oo * np.exp(m - M)[:, None] for m, oo in zip(ms, os_)) / Z[:, None]
    o = rope_complex(o, L - 1, 32, 10000.0, inverse=True)
    assert np.allclose(joint, o, rtol=0, atol=1e-12)


def test_csa_with_all_selected_equals_dense():
    cfg = O.LayerCfg(4, 64, 32, 4, 16, "bf16", "fp8")
    c, kv, lg, q = built_cache(cfg, 333, 7)
    _, _, dense = O.decode_layer(cfg, c, 0, q, 333, top_k=None)
    _, _, full = O.decode_layer(cfg, c, 0, q, 333, top_k=10 ** 6)
    assert np.array_equal(dense, full)


def test_no_keys_gives_zero_output():
    cfg = O.LayerCfg(2, 16, 8, 4, 0, "f32", "f32")
    c, kv, lg, q = built_cache(cfg, 3, 8)
    _, _, out = O.decode_layer(cfg, c, 0, q, 3, top_k=4)
    assert not np.any(out)
