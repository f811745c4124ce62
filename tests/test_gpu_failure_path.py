"""The device failure path without a fault: a bounded wait that nothing completes.

ckv_debug_force_timeout makes the MMA-issuing lane of every tensor-core attention CTA of one
request wait on a barrier that no one arrives on. The wait gives up after its bound; the CTA frees
its tensor memory without having issued anything, marks its partial empty and sets
CKV_DEV_TIMEOUT. The call returns, the forced request's output is zero, the other requests match
the oracle, and the next call (hook off) is correct again on the same context."""

import numpy as np
import pytest
import torch

from oracle import ckv_oracle as O
from synth import workloads as S
from tests import ckv_testlib as T

pytestmark = pytest.mark.gpu


def test_attention_wait_that_never_completes_sets_the_timeout_bit(cuda_lib):
    w = S.scaled(S.csa_b8_ctx32k(), (9000, 20001, 4099), "failure_path", seed=8400)
    gen = S.generate(w, "cuda")
    lay, ls = gen["layers"][0], w.layers[0]
    seq = gen["seq_len"]
    dl = T.gpu_layer(cuda_lib, w, lay, ls)
    dl.select(seq, lay["q"])
    assert T.status_word(dl) == 0
    cuda_lib.debug_force_timeout(1)
    try:
        out = dl.attend(seq, lay["q"]).cpu().numpy()
        st = T.status_word(dl)
    finally:
        cuda_lib.debug_force_timeout(-1)
    assert st & cuda_lib.CKV_DEV_TIMEOUT
    assert np.all(np.isfinite(out))
    assert not np.any(out[1])
    ocfg, oc = T.oracle_cfg(w, ls), T.oracle_cache(lay)
    qn = lay["q"].cpu().numpy()
    idx, cnt = dl.idx.cpu().numpy(), dl.cnt.cpu().numpy()

    def check(out, requests):
        for b in requests:
            ref = O.attention(ocfg, oc, b, qn[b], w.seq_lens[b], idx[b, :cnt[b]].astype(np.int64))
            assert T.max_rel_err(out[b], ref) <= 2e-3, b

    check(out, [0, 2])
    # the same context, hook off: every request is attended again
    dl.status.zero_()
    out2 = dl.attend(seq, lay["q"]).cpu().numpy()
    assert T.status_word(dl) == 0
    check(out2, [0, 1, 2])
