"""GPU parity of the HBM-bound state kernels (N-way composition, plan-driven
cache scatter, window residual) against the oracle, through the C ABI."""

import numpy as np
import pytest
import torch

import oracle as orc
import partitioned_attention_state_b200 as dt

from parity import check_lse, check_out, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def rand_states(N, H, S, D, seed, empty_frac=0.1):
    rng = np.random.Generator(np.random.PCG64(seed))
    O = rng.standard_normal((N, H, S, D)).astype(np.float32)
    L = (rng.standard_normal((N, H, S)) * 6).astype(np.float32)
    L[rng.random((N, H, S)) < empty_frac] = -np.inf
    L[:, 0, :3] = -np.inf            # a few rows with every input empty
    O[np.isneginf(L)] = 0.0
    return O, L


@pytest.mark.parametrize("N,H,S,D", [(16, 3, 333, 128), (4, 2, 1024, 72), (1, 1, 17, 64), (9, 2, 500, 8)])
def test_state_merge_matches_compose_n(N, H, S, D):
    O, L = rand_states(N, H, S, D, seed=N * 7 + D)
    o_in, l_in = torch.from_numpy(O).cuda(), torch.from_numpy(L).cuda()
    o_out = torch.empty((H, S, D), device="cuda")
    l_out = torch.empty((H, S), device="cuda")
    dt.dt_state_merge(N, H, S, D, o_in, l_in, o_out, l_out)
    torch.cuda.synchronize()
    for h in range(H):
        ref_o, ref_l = orc.compose_n([(O[n, h].astype(np.float64), L[n, h].astype(np.float64)) for n in range(N)])
        check_out(to_np(o_out[h]), ref_o, max_abs=1e-5, rel=1e-6)
        check_lse(to_np(l_out[h]), ref_l, max_abs=1e-5)


@pytest.mark.parametrize("H,S,D,P", [(2, 1000, 72, 3), (3, 4096, 128, 16), (1, 5, 64, 4)])
def test_cache_update_scatters_exactly_the_compute_slots(H, S, D, P):
    nqt = len(orc.query_tiles(S, P))
    rng = np.random.Generator(np.random.PCG64(S))
    plan = (rng.random((nqt, P)) < 0.5).astype(np.uint8)
    p = dt.params(H, S, D, P, dt.DT_MODE_EXPLICIT, 0, 0, 1)
    fresh_O = torch.randn((P, H, S, D), device="cuda")
    fresh_L = torch.randn((P, H, S), device="cuda")
    cache_O = torch.randn((P, H, S, D), device="cuda")
    cache_L = torch.randn((P, H, S), device="cuda")
    want_O, want_L = cache_O.clone(), cache_L.clone()
    for t, (_, q0, q1) in enumerate(orc.query_tiles(S, P)):
        for k in range(P):
            if plan[t, k] == orc.COMPUTE:
                want_O[k, :, q0:q1] = fresh_O[k, :, q0:q1]
                want_L[k, :, q0:q1] = fresh_L[k, :, q0:q1]
    d_plan = torch.from_numpy(plan).cuda()
    dt.dt_state_cache_update(p, d_plan, fresh_O, fresh_L, cache_O, cache_L)
    torch.cuda.synchronize()
    assert torch.equal(cache_O, want_O) and torch.equal(cache_L, want_L)


@pytest.mark.parametrize("H,S,D", [(2, 1000, 72), (16, 16384, 72)])
def test_window_residual_make_and_apply(H, S, D):
    of = torch.randn((H, S, D), device="cuda")
    ow = torch.randn((H, S, D), device="cuda")
    R = torch.empty_like(of)
    O = torch.empty((H, S, D), dtype=torch.bfloat16, device="cuda")
    dt.dt_window_residual(dt.DT_WR_MAKE, H, S, D, of, ow, R, None)
    dt.dt_window_residual(dt.DT_WR_APPLY, H, S, D, None, ow, R, O)
    torch.cuda.synchronize()
    r_ref = to_np(of) - to_np(ow)
    np.testing.assert_allclose(to_np(R), r_ref, rtol=0, atol=1e-6)
    # both sides round the same fp32 sum to bf16 (nearest even)
    s32 = (ow.cpu().numpy() + R.cpu().numpy()).astype(np.float32)
    o_ref = orc.round_bf16(s32.astype(np.float64))
    np.testing.assert_array_equal(to_np(O), o_ref)
