"""GPU parity of quantile balancing ("Stable LatentMoE interactive demo
document", Quantile Balancing) against the CPU oracle, through the C ABI:
cutoffs, the exact q-th smallest required bias, the histogram estimate and
the loads, all bit-exact."""
import numpy as np
import pytest

import oracle as O

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import sparse_mixture_experts_15_b200 as moe


@pytest.fixture(autouse=True)
def _clean_status():
    moe.moe_reset_device_status()
    yield
    assert moe.moe_device_status() == 0


def _run(scores, k, q, bias=None, bins=0):
    T, N = scores.shape
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    s = dev(scores)
    b = None if bias is None else dev(bias)
    cut = torch.empty(T, dtype=torch.float32, device="cuda")
    bx = torch.empty(N, dtype=torch.float32, device="cuda")
    bh = torch.empty(N, dtype=torch.float32, device="cuda") if bins else None
    loads = torch.empty(N, dtype=torch.int32, device="cuda")
    moe.moe_quantile_balance(s, k, q, bx, bias=b, bins=bins, cutoff=cut, bias_hist=bh,
                             loads=loads)
    torch.cuda.synchronize()
    return (cut.cpu().numpy(), bx.cpu().numpy(), None if bh is None else bh.cpu().numpy(),
            loads.cpu().numpy())


def _check(scores, k, q, bias=None, bins=0):
    cut, bx, bh, loads = _run(scores, k, q, bias, bins)
    a = O.qb_cutoffs(scores, k, bias)
    ref_b, ref_loads = O.qb_exact(scores, a, q)
    assert np.array_equal(cut.view(np.uint32), a.view(np.uint32))
    assert np.array_equal(bx.view(np.uint32), ref_b.view(np.uint32))
    assert np.array_equal(loads, ref_loads)
    assert np.all(loads >= q)
    if bins:
        ref_h = O.qb_hist(scores, a, q, bins)
        assert np.array_equal(bh.view(np.uint32), ref_h.view(np.uint32))
    return bx, loads


def test_qb_random_with_bias():
    rng = np.random.default_rng(21)
    T, N, k = 600, 13, 3
    scores = rng.standard_normal((T, N)).astype(np.float32)
    bias = (0.2 * rng.standard_normal(N)).astype(np.float32)
    _check(scores, k, q=130, bias=bias, bins=64)


def test_qb_latent_shape_hot_experts():
    """896 experts, top-16, 4096 tokens, target q = 73 (k T / N): six hot
    experts get most of the routing before balancing; with the balancing bias
    and the cutoffs fixed every expert takes q tokens, more only through
    ties (a token's k-th expert has required = 0 exactly)."""
    rng = np.random.default_rng(1004)
    T, N, k = 4096, 896, 16
    q = (k * T) // N
    scores = (0.02 * rng.standard_normal((T, N))).astype(np.float32)
    scores[:, :6] += np.float32(0.05)
    a = O.qb_cutoffs(scores, k)
    before = (scores >= a[:, None]).sum(0)
    assert before[:6].min() > 4 * q  # the hot experts are overloaded
    bx, loads = _check(scores, k, q, bins=256)
    req = (a[:, None] - scores).astype(np.float32)
    below = (req < bx[None, :]).sum(0)
    assert np.all(below <= q - 1) and np.all(loads >= q)
    assert np.all(loads[:6] == q)  # the hot experts' q-th required bias is untied


def test_qb_ties():
    """Integer-valued scores: many equal required biases; still bit-exact."""
    rng = np.random.default_rng(3)
    T, N, k = 777, 40, 5
    scores = rng.integers(-3, 4, size=(T, N)).astype(np.float32)
    _check(scores, k, q=50, bins=16)
    _check(scores, k, q=1, bins=1)
    _check(scores, k, q=T, bins=4096)
