"""An expired bounded device wait is reported, not hung: the library's mbarrier
wait, run on a barrier that nothing arrives at with a 0.2 s limit, writes
FLIDE_ERR_TIMEOUT to the status word; the CUDA context stays usable for the
hot path right after."""
import time

import numpy as np
import pytest
import torch

from tree_forked_decision_b200 import flide, inputs

from gpu_helpers import assert_close, oracle_attn, run_attn

pytestmark = pytest.mark.gpu


def test_bounded_wait_expires_with_timeout_status():
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    t0 = time.perf_counter()
    flide.selftest_wait_timeout(st, 200_000)
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t0
    assert int(st.item()) == flide.ERR_TIMEOUT
    assert 0.15 < elapsed < 5.0  # the limit, not an open-ended spin


def test_bounded_wait_completes_when_arrived():
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    flide.selftest_wait_timeout(st, 200_000, arrive=True)
    torch.cuda.synchronize()
    assert int(st.item()) == flide.OK


def test_context_usable_after_expired_wait():
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    flide.selftest_wait_timeout(st, 50_000)
    torch.cuda.synchronize()
    assert int(st.item()) == flide.ERR_TIMEOUT
    tree = inputs.fanout_tree(1, 100, 3, 5)
    a = inputs.attn_inputs(tree, 8, 2, 128, torch.bfloat16, np.random.default_rng(2))
    got, scale = run_attn(tree, a)
    assert_close(got, oracle_attn(tree, a, scale), torch.bfloat16)


def test_selftest_rejects_bad_arguments():
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    with pytest.raises(flide.FlideError):
        flide.selftest_wait_timeout(st, 0)
