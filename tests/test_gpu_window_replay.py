"""kv_window_replay (SWA bounded replay: aidevelopers.cz "DeepSeek-V4.1-Flash ve vLLM", section
"Proč je obnova sliding-window cache drahá") against the oracle, through the C ABI.

A context is appended from scratch on both sides; the last min(W, L) positions are then replayed
with different (recomputed) tokens. The window, the residue ring and the untouched compressed
entries must hold the oracle's bytes under the append's rounding rules, and the next decode step
(whose append completes the unfinished group from the replayed ring) must select and attend as
the oracle does."""

import numpy as np
import pytest
import torch

from oracle import ckv_oracle as O
from synth import workloads as S
from tests import ckv_testlib as T
from tests.test_gpu_parity import ATT_TOL, _compare_caches

pytestmark = pytest.mark.gpu

# every length leaves an unfinished group that the next token completes (L % r == r - 1) and
# keeps position L inside the last mapped block (L % 256 != 0)
CASES = [
    ("bf16_fp8_r4", (1027, 515, 79, 3), 64, 512, 64, 4, 32, "bf16", "fp8"),
    ("nvfp4_fp8_r128", (1023, 383, 127), 64, 512, 64, 128, None, "nvfp4", "fp8"),
    ("f32_f32_r4_d128", (1027, 99, 7), 16, 128, 32, 4, 16, "f32", "f32"),
    ("bf16_f32_r8", (1031, 135), 8, 256, 64, 8, 16, "bf16", "f32"),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: c[0])
def test_window_replay_matches_the_oracle(cuda_lib, case):
    name, lens, H, D, d_r, r, k, comp, win = case
    w = S.Workload("replay_" + name, lens, H, D, d_r, 128, (S.LayerSpec(r, k, comp, win),), paged=True,
                   from_scratch=True, seed=8100 + r)
    gen = S.generate(w, "cuda")
    lay, ls = gen["layers"][0], w.layers[0]
    seq = gen["seq_len"]
    dl = T.gpu_layer(cuda_lib, w, lay, ls, max_seq_len=max(lens) + 1)
    T.gpu_setup(dl, lay)
    T.gpu_append_decode_token(dl, lay, seq)
    ocfg = T.oracle_cfg(w, ls)
    oc = T.oracle_cache(lay)
    T.oracle_setup(ocfg, oc, lay, w.batch)
    T.oracle_append_decode_token(ocfg, oc, lay, w.seq_lens)
    comp_before = dl.cache.comp_codes.clone()

    g = torch.Generator(device="cuda")
    g.manual_seed(8200 + r)
    kv = (torch.randn((w.batch, 128, D), generator=g, device="cuda") * 2.0).contiguous()
    lg = torch.randn((w.batch, 128), generator=g, device="cuda").contiguous()
    dl.replay_window(seq, kv, lg)
    assert T.status_word(dl) == 0
    assert torch.equal(dl.cache.comp_codes, comp_before), "the replay wrote compressed entries"
    kvh, lgh = kv.cpu().numpy(), lg.cpu().numpy()
    for b, L in enumerate(lens):
        n_w = min(128, L)
        O.window_replay(ocfg, oc, b, L, kvh[b, :n_w], lgh[b, :n_w])
    _compare_caches(name, ocfg, oc, dl, lay, w, ls)

    # the next decode step: its append completes the unfinished group from the replayed ring
    kv1 = torch.randn((w.batch, D), generator=g, device="cuda")
    lg1 = torch.randn((w.batch,), generator=g, device="cuda")
    dl.append(seq.clone(), kv1, lg1)
    seq1 = (seq + 1).to(torch.int32)
    if k is not None:
        dl.select(seq1, lay["q"])
    out = dl.attend(seq1, lay["q"]).cpu().numpy()
    assert T.status_word(dl) == 0
    kv1h, lg1h, qn = kv1.cpu().numpy(), lg1.cpu().numpy(), lay["q"].cpu().numpy()
    for b, L in enumerate(lens):
        O.append_tokens(ocfg, oc, b, L, kv1h[b:b + 1], lg1h[b:b + 1])
    for b, L in enumerate(lens):
        L1 = L + 1
        if k is not None:
            s64 = O.indexer_scores(ocfg, oc, b, qn[b], L1)
            ok, msg = T.topk_sets_match(dl.idx[b].cpu().numpy(), int(dl.cnt[b]), s64, k, 1e-5)
            assert ok, f"{name} b={b}: {msg}"
            sel = dl.idx[b, :int(dl.cnt[b])].cpu().numpy().astype(np.int64)
        else:
            sel = np.arange(L1 // r)
        ref = O.attention(ocfg, oc, b, qn[b], L1, sel)
        e = T.max_rel_err(out[b], ref)
        assert e <= ATT_TOL[comp], f"{name} b={b}: rel err {e:.2e}"


def test_window_replay_flags_a_bad_length(cuda_lib):
    w = S.Workload("replay_bad", (300, 200), 8, 128, 32, 128, (S.LayerSpec(4, 8, "bf16", "fp8"),), paged=True,
                   from_scratch=True, seed=8300)
    gen = S.generate(w, "cuda")
    lay, ls = gen["layers"][0], w.layers[0]
    dl = T.gpu_layer(cuda_lib, w, lay, ls)
    win_before = dl.cache.win_codes.clone()
    seq = gen["seq_len"].clone()
    seq[1] = 10 ** 6
    kv = torch.zeros((2, 128, 128), device="cuda")
    lg = torch.zeros((2, 128), device="cuda")
    dl.replay_window(seq, kv, lg)
    assert T.status_word(dl) & cuda_lib.CKV_DEV_BAD_LENGTH
    # request 1 was skipped: its window rows are as they were
    rows = [int(lay["win_table"][1, lb]) for lb in range(lay["win_table"].shape[1]) if int(lay["win_table"][1, lb]) >= 0]
    for row in rows:
        assert torch.equal(dl.cache.win_codes[row], win_before[row])
