"""Failure detection on the GPU without a fault: the library's bounded waits
(the grid barrier of the cooperative kernels, the mbarrier wait of the tcgen05
kernels) are made to run out on a condition nothing satisfies.  Each must give
up within its budget, leave MOE_ERR_TIMEOUT in the sticky status word and
return, after which the context is still usable: a normal layer call that
follows passes its oracle check."""
import time

import numpy as np
import pytest

import oracle as O
from synthetic import workloads as W

from inputs import dev_experts, dev_router, dev_u, host_expert, host_router, host_u, rel_err

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import sparse_mixture_experts_15_b200 as moe

MOE_ERR_TIMEOUT = -4


def _layer_still_correct():
    wl = W.small(T=256)
    s = moe.shape(wl.T, wl.d, wl.N, wl.k, wl.h, 1, 0)
    u = dev_u(wl)
    w, b = dev_router(wl)
    wg, wu, wd = dev_experts(wl)
    y = torch.empty((wl.T, wl.d), dtype=torch.bfloat16, device="cuda")
    moe.moe_layer_fwd(s, w, wg, wu, wd, u, y)
    torch.cuda.synchronize()
    assert moe.moe_device_status() == 0
    uh = host_u(wl)
    wr, _ = host_router(wl)
    _, _, idx, tw = O.route(O.as_f32(O.BF16, uh), wr, wl.k)
    mats = [host_expert(wl, e) for e in range(wl.N)]
    ref = O.moe_tokens([m[0] for m in mats], [m[1] for m in mats], [m[2] for m in mats],
                       O.decode(O.BF16, uh), idx, tw, round_h=1)
    assert rel_err(y.float().cpu().numpy(), ref) < 2e-2


@pytest.mark.parametrize("kind", ["grid_barrier", "mbarrier"])
def test_bounded_wait_runs_out_and_reports_timeout(kind):
    code = moe.WAIT_GRID_BARRIER if kind == "grid_barrier" else moe.WAIT_MBARRIER
    moe.moe_reset_device_status()
    torch.cuda.synchronize()
    assert moe.moe_device_status() == 0
    budget_ns = 2_000_000  # 2 ms
    t0 = time.perf_counter()
    moe.moe_wait_check(code, budget_ns)
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t0
    assert moe.moe_device_status() == MOE_ERR_TIMEOUT
    assert elapsed < 2.0, f"the wait took {elapsed:.3f} s for a 2 ms budget"
    # the status word is sticky until reset, and the context is still usable
    assert moe.moe_device_status() == MOE_ERR_TIMEOUT
    moe.moe_reset_device_status()
    _layer_still_correct()


def test_wait_check_rejects_bad_arguments():
    with pytest.raises(moe.MoeError):
        moe.moe_wait_check(7, 1_000_000)
    with pytest.raises(moe.MoeError):
        moe.moe_wait_check(moe.WAIT_MBARRIER, 10)
    assert moe.moe_device_status() == 0
