"""Failure detection on the GPU without faulting it: every wait inside the
fused kernel is bounded; a wait that runs out reports DT_ERR_TIMEOUT through
the device status word and the kernel drains and exits, leaving the context
usable.  The test makes the waits run out by setting their limit to 0 ns."""

import numpy as np
import pytest
import torch

import oracle as orc
import partitioned_attention_state_b200 as dt
from partitioned_attention_state_b200 import workloads as wl
from partitioned_attention_state_b200.session import Session

from parity import check_lse, check_out, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    yield
    dt.dt_set_wait_limit_ns(2_000_000_000)


def test_wait_limit_zero_reports_timeout_and_context_survives():
    H, S, D, P = 4, 1024, 72, 8
    q, k, v = wl.InputStream(H, S, D, 0.05, seed=1).next_step()
    sess = Session(H, S, D, P)
    sess.set_inputs(q, k, v)
    dt.dt_set_wait_limit_ns(0)
    sess.step(1)
    torch.cuda.synchronize()
    assert int(sess.status[0].item()) == dt.DT_ERR_TIMEOUT
    # the context is intact: a normal launch afterwards is correct
    dt.dt_set_wait_limit_ns(2_000_000_000)
    sess.status.zero_()
    sess.stamps[:] = -1
    sess.step(1)
    sess.check()
    Q, K, V = (orc.widen_bf16(x) for x in (q, k, v))
    ref_o, ref_l = orc.attention_state(Q[2], K[2], V[2], orc.softmax_scale(D))
    check_out(to_np(sess.O[2]), ref_o)
    check_lse(to_np(sess.L[2]), ref_l)


def test_invalid_arguments_launch_nothing():
    sess = Session(1, 256, 64, 2)
    p = dt.params(1, 256, 96, 2, dt.DT_MODE_ALL_COMPUTE, 0, 0, 1)
    with pytest.raises(dt.DtError) as e:
        dt.dt_attn_partial_fused(p, sess.d_plan, sess.Q, sess.K, sess.V, sess.cache_O, sess.cache_L, None, sess.O,
                                 sess.L, sess.counters, sess.status)
    assert e.value.status == dt.DT_ERR_UNSUPPORTED
    p.D = 64
    with pytest.raises(dt.DtError) as e:
        dt.dt_attn_partial_fused(p, sess.d_plan, sess.Q[:, :, 1:], sess.K, sess.V, sess.cache_O, sess.cache_L,
                                 None, sess.O, sess.L, sess.counters, sess.status)
    assert e.value.status == dt.DT_ERR_UNSUPPORTED
    torch.cuda.synchronize()
    assert int(sess.status[0].item()) == 0
