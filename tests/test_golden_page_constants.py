"""The structural constants the pages state (tests/golden/page_constants.txt), checked against
the oracle's layout and the library's sizes."""

import os

import numpy as np
import pytest

import compressed_kv_sparse_compress_b200 as ckv
from oracle import ckv_oracle as O

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "page_constants.txt")


def constants():
    out = {}
    for line in open(GOLDEN):
        if line.strip() and not line.startswith("#"):
            name, value = line.split()[:2]
            out[name] = float(value)
    return out


def test_logical_block_and_ratios():
    c = constants()
    assert O.LOGICAL_BLOCK_TOKENS == c["logical_block_tokens"]
    for r in (int(c["csa_ratio"]), int(c["hca_ratio"])):
        cfg = O.LayerCfg(64, 512, 64, r, int(c["window_tokens"]), "bf16", "fp8")
        assert cfg.entries_per_block * r == c["logical_block_tokens"]
        # a 1M-token context holds 1M / r completed entries (4x and 128x fewer than tokens)
        assert O.num_compressed(1 << 20, r) == (1 << 20) // r
        lib = ckv.LayerConfig(64, 512, 64, r, int(c["window_tokens"]), "bf16", "fp8")
        assert lib.row_bytes()[0] == 1024


def test_window_of_128_is_accepted_and_attended():
    c = constants()
    cfg = ckv.LayerConfig(64, 512, 64, 4, int(c["window_tokens"]), "nvfp4", "fp8")
    assert cfg.row_bytes()[2] == 512


def test_nvfp4_cache_is_about_45_percent_smaller_than_fp8():
    c = constants()
    nv = ckv.LayerConfig(64, 512, 64, 4, 128, "nvfp4", "fp8").row_bytes()
    codes, scales, fp8_codes, fp8_scale = nv
    saving = 1 - (codes + scales) / (fp8_codes + fp8_scale)
    assert saving == pytest.approx(c["nvfp4_saving_vs_fp8"], abs=0.01)
