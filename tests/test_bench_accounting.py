"""The bench's algorithmic byte and flop counts (the roofline numerators), checked against the
stored formats on CPU: they must follow from the row sizes and the workload, not from a timing."""

import math
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from synth import workloads as S  # noqa: E402


def test_head_averaged_indexer_reads_every_entry_once():
    w = S.csa_b8_ctx32k()
    ls = w.layers[0]
    b = bench.layer_bytes(w, ls)
    n_c = 32768 // 4
    # bf16 entries of 512 dims and the block table of each request (the score kernel reads the
    # head-averaged query; the raw [64][512] query is read by the query pass before it)
    assert b["indexer"] == 8 * (n_c * 1024 + 4 * 128)
    assert b["indexer"] == 67112960
    # attention: 512 selected entries + 128 FP8 window tokens (512 codes + a scale) + q in, o out
    assert b["attention"] == 8 * (512 * 1024 + 128 * (512 + 4) + 2 * 4 * 64 * 512)


def test_multi_head_indexer_reads_index_rows_not_kv_entries():
    w = S.csa_b4_ctx1m()
    ls = w.layers[0]
    b = bench.layer_bytes(w, ls, "mh")
    n_c = 1048576 // 4
    per_req = n_c * (bench.MH_DIM + 4) + 4 * math.ceil(1048576 / 256) + 4 * bench.MH_HEADS * (bench.MH_DIM + 1)
    assert b["indexer"] == 4 * per_req
    # the index rows are 132 B against 1024 B per bf16 entry
    assert b["indexer"] < bench.layer_bytes(w, ls)["indexer"] / 7
    # the append also writes the index entry and reads the index ring
    assert b["append"] > bench.layer_bytes(w, ls)["append"]


def test_dense_layer_has_no_indexer_bytes():
    w = S.hca_b32_ctx128k()
    b = bench.layer_bytes(w, w.layers[0])
    assert b["indexer"] == 0
    assert b["attention"] == 32 * (1024 * 1024 + 128 * (512 + 4) + 2 * 4 * 64 * 512)


def test_multi_head_tensor_record_counts_two_flops_per_head_dim_and_entry():
    w = S.csa_b8_ctx32k()
    r = bench.tensor_record(w, "mh", 0.010)  # 10 us per launch
    flops = 2.0 * bench.MH_HEADS * bench.MH_DIM * 8 * (32768 // 4)
    assert r["flops_per_launch"] == flops
    assert r["achieved_tflops"] == pytest.approx(flops / 1e-5 / 1e12)
    assert r["frac"] == pytest.approx(r["achieved_tflops"] / r["peak_tflops"])


def test_attention_flops_count_both_products_per_key():
    w = S.csa_b4_ctx1m()
    # 2048 selected entries + 128 window tokens per request, 2 H D flops each for the logits and
    # for the weighted sum
    assert bench.attention_flops(w, w.layers[0]) == 4 * 4.0 * 64 * 512 * (2048 + 128)
    h = S.hca_b32_ctx128k()
    assert bench.attention_flops(h, h.layers[0]) == 32 * 4.0 * 64 * 512 * (1024 + 128)


def test_roofline_record_divides_bytes_by_the_average_launch():
    r = bench.roofline_record("attention_kernel", 1e9, [1.0, 3.0], 6425.6, "measured", "none",
                              flops_per_launch=2e12)
    assert r["achieved"] == pytest.approx(1e9 / 2e-3 / 1e9)
    assert r["frac"] == pytest.approx(r["achieved"] / 6425.6)
    assert r["tensor"]["achieved_tflops"] == pytest.approx(2e12 / 2e-3 / 1e12)
    assert r["traffic"] is None


def test_default_workload_is_the_largest_single_gpu_config():
    assert bench.DEFAULT_WORKLOAD == "csa_b4_ctx1m"
    assert set(bench.CONFIGS) == {"csa_b1_ctx4k_fp32", "csa_b8_ctx32k", "hca_b32_ctx128k", "csa_b4_ctx1m",
                                  "mixed_64req"}
