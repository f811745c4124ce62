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
    # bf16 entries of 512 dims, the block table of each request, the raw query [64][512] fp32
    assert b["indexer"] == 8 * (n_c * 1024 + 4 * 128 + 4 * 64 * 512)
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
