"""GPU parity of the routing-side steps against the CPU oracle, through the C ABI:
generator, router (bit-exact logits and top-k), aux statistics, permutation
(bit-exact), gather (bit-exact) and combine."""
import numpy as np
import pytest

import oracle as O
import synthetic as S
from synthetic import workloads as W

from inputs import (dev_normal, dev_router, dev_u, host_router, host_u, to_numpy_codes, ORACLE_DT,
                    rel_err)

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import sparse_mixture_experts_15_b200 as moe


@pytest.fixture(autouse=True)
def _clean_status():
    moe.moe_reset_device_status()
    yield
    assert moe.moe_device_status() == 0


# ------------------------------------------------------------------ inputs
@pytest.mark.parametrize("dtype", [S.DT_F32, S.DT_BF16, S.DT_F16])
def test_generator_device_matches_host(dtype):
    d = dev_normal(5, 9, (1000, 24), 0.7, dtype, offset=123)
    h = S.normal(5, 9, (1000, 24), 0.7, dtype, offset=123)
    assert np.array_equal(to_numpy_codes(d).view(h.dtype), h)
    wl = W.small(T=300)
    assert np.array_equal(to_numpy_codes(dev_u(wl)), host_u(wl))
    qs = torch.empty((40, 256), dtype=torch.uint8, device="cuda")
    sc = torch.empty((40, 16), dtype=torch.int16, device="cuda")
    S.q4_dev(3, 11, 40, 512, qs.data_ptr(), sc.data_ptr(), torch.cuda.current_stream().cuda_stream,
             row0=7)
    hq, hs = S.q4(3, 11, 40, 512, row0=7)
    assert np.array_equal(qs.cpu().numpy(), hq)
    assert np.array_equal(sc.cpu().numpy().view(np.uint16), hs)


# ------------------------------------------------------------------ router
def _route_gpu(wl, T=None, probs=True):
    T = wl.T if T is None else T
    s = moe.shape(T, wl.d, wl.N, wl.k, wl.h, wl.renorm, 0)
    u = dev_u(wl, T)
    w, b = dev_router(wl)
    idx = torch.empty((T, wl.k), dtype=torch.int32, device="cuda")
    tw = torch.empty((T, wl.k), dtype=torch.float32, device="cuda")
    pr = torch.empty((T, wl.N), dtype=torch.float32, device="cuda") if probs else None
    z = torch.empty((T, wl.N), dtype=torch.float32, device="cuda")
    moe.moe_route(s, u, w, idx, tw, bias=b, probs=pr, logits=z)
    torch.cuda.synchronize()
    return (z.cpu().numpy(), None if pr is None else pr.cpu().numpy(), idx.cpu().numpy(),
            tw.cpu().numpy())


def _route_oracle(wl, rows):
    u = host_u(wl, max(rows) + 1)[rows]
    w, b = host_router(wl)
    return O.route(O.as_f32(ORACLE_DT[wl.act_dtype], u), w, wl.k, wl.renorm, b)


@pytest.mark.parametrize("name,T,sample", [("tiny", None, None), ("small", None, None),
                                           ("small", 1001, None), ("mixtral", None, 512),
                                           ("latent", 1024, 96), ("decode", 32, None)])
def test_route_bit_exact(name, T, sample):
    wl = W.ALL[name]() if T is None else W.ALL[name](T=T) if name != "tiny" else W.tiny()
    z, pr, idx, tw = _route_gpu(wl)
    Tn = wl.T
    rng = np.random.default_rng(1)
    rows = np.arange(Tn) if sample is None else np.sort(rng.choice(Tn, sample, replace=False))
    lz, lp, lidx, ltw = _route_oracle(wl, rows)
    assert np.array_equal(z[rows].view(np.uint32), lz.view(np.uint32)), "logits not bit-exact"
    assert np.array_equal(idx[rows], lidx), "top-k indices differ"
    assert np.allclose(tw[rows], ltw, rtol=2e-6, atol=1e-7)
    assert np.allclose(pr[rows], lp, rtol=2e-6, atol=1e-7)
    if wl.renorm:
        assert np.allclose(tw.sum(1), 1.0, atol=2e-6)


def test_route_ties_and_controlled_logits():
    """Tutorial §3.4 controlled logits, built as u . W so the GPU router sees them:
    balanced (2.0 at expert t mod 4) and collapsed (2.0 at expert 0)."""
    T, d, N = 16, 8, 4
    for case in ("balanced", "collapsed"):
        u = np.zeros((T, d), np.float32)
        Wr = np.zeros((N, d), np.float32)
        if case == "balanced":
            u[np.arange(T), np.arange(T) % N] = 2.0
            Wr[np.arange(N), np.arange(N)] = 1.0
        else:
            u[:, 0] = 2.0
            Wr[0, 0] = 1.0
        s = moe.shape(T, d, N, 1, 64, 1, 0)
        idx = torch.empty((T, 1), dtype=torch.int32, device="cuda")
        tw = torch.empty((T, 1), dtype=torch.float32, device="cuda")
        pr = torch.empty((T, N), dtype=torch.float32, device="cuda")
        moe.moe_route(s, torch.from_numpy(u).cuda(), torch.from_numpy(Wr).cuda(), idx, tw, probs=pr)
        f = torch.empty(N, device="cuda")
        P = torch.empty(N, device="cuda")
        ns = torch.empty(1, device="cuda")
        loads = torch.empty(N, dtype=torch.int32, device="cuda")
        moe.moe_aux_stats(pr, idx, f, P, ns, loads)
        torch.cuda.synchronize()
        lp, lidx, _ = O.route_from_logits(u @ Wr.T, 1)
        of, oP, ons, oloads = O.aux_stats(lp, lidx)
        assert np.array_equal(idx.cpu().numpy(), lidx)
        assert np.allclose(f.cpu().numpy(), of, atol=0)
        assert np.allclose(P.cpu().numpy(), oP, rtol=1e-6)
        assert abs(ns.item() - ons) < 1e-5
        assert f"{ns.item():.4f}" == ("1.0000" if case == "balanced" else "2.8449")
    # ties: equal logits go to the lower expert index
    u = np.ones((3, 8), np.float32)
    Wr = np.zeros((6, 8), np.float32)
    Wr[[1, 2, 4]] = 0.25
    s = moe.shape(3, 8, 6, 3, 64, 1, 0)
    idx = torch.empty((3, 3), dtype=torch.int32, device="cuda")
    tw = torch.empty((3, 3), dtype=torch.float32, device="cuda")
    moe.moe_route(s, torch.from_numpy(u).cuda(), torch.from_numpy(Wr).cuda(), idx, tw)
    assert idx.cpu().numpy().tolist() == [[1, 2, 4]] * 3


def _block_order_router(N, d=256):
    """Router rows whose fp32 logit depends on the summation order (u = 1):
    expert 0: 2^25 at 0, -2^25 at 128, 1 at 129 (blocked order 0, one chain 1);
    expert 1: 1 at 0, 2^25 at 128, -2^25 at 129 (blocked 1, one chain 0);
    expert 2: 2^25 at 0, 1 at 8, -2^25 at 128 (blocked 0, a pairwise tree 1);
    expert 3: 0.5 at 0; the rest zero."""
    Wr = np.zeros((N, d), np.float32)
    Wr[0, [0, 128, 129]] = [2.0 ** 25, -(2.0 ** 25), 1.0]
    Wr[1, [0, 128, 129]] = [1.0, 2.0 ** 25, -(2.0 ** 25)]
    Wr[2, [0, 8, 128]] = [2.0 ** 25, 1.0, -(2.0 ** 25)]
    Wr[3, 0] = 0.5
    return Wr


@pytest.mark.parametrize("N", [4, 8, 32])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16, torch.float16])
def test_router_block_order_on_gpu(N, dtype):
    """Every router kernel forms the logits in the blocked order of the oracle
    (128-input chains, block sums in order): the hand-worked logits 0, 1, 0,
    0.5 come out exactly and the top-2 is experts 1 and 3."""
    T, d = 40, 256
    Wr = _block_order_router(N, d)
    u = np.ones((T, d), np.float32)
    s = moe.shape(T, d, N, 2, 64, 1, 0)
    idx = torch.empty((T, 2), dtype=torch.int32, device="cuda")
    tw = torch.empty((T, 2), dtype=torch.float32, device="cuda")
    z = torch.empty((T, N), dtype=torch.float32, device="cuda")
    moe.moe_route(s, torch.from_numpy(u).to(dtype).cuda(), torch.from_numpy(Wr).cuda(), idx, tw,
                  logits=z)
    torch.cuda.synchronize()
    zo, _, oidx, _ = O.route(u, Wr, 2, 1)
    zn = z.cpu().numpy()
    assert np.array_equal(zn, zo)
    assert np.array_equal(zn[:, :4], np.tile([0.0, 1.0, 0.0, 0.5], (T, 1)))
    assert np.array_equal(idx.cpu().numpy(), oidx)
    assert np.all(idx.cpu().numpy() == [1, 3])


def test_layer_routing_block_order():
    """The layer path's own router (the fused route+dispatch kernel for few
    experts) picks experts 1 and 3 on the order-sensitive router rows."""
    T, d, N, k, h = 64, 256, 4, 2, 64
    Wr = torch.from_numpy(_block_order_router(N, d)).cuda()
    u = torch.ones((T, d), dtype=torch.bfloat16, device="cuda")
    g = torch.Generator(device="cuda").manual_seed(11)
    w_gate, w_up = ((torch.randn(N, h, d, device="cuda", generator=g) * 0.02).to(torch.bfloat16)
                    for _ in range(2))
    w_down = (torch.randn(N, d, h, device="cuda", generator=g) * 0.02).to(torch.bfloat16)
    y = torch.empty((T, d), dtype=torch.bfloat16, device="cuda")
    top_idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    s = moe.shape(T, d, N, k, h, 1, 0)
    moe.moe_layer_fwd(s, Wr, w_gate, w_up, w_down, u, y, outputs={"top_idx": top_idx})
    torch.cuda.synchronize()
    assert np.all(top_idx.cpu().numpy() == [1, 3])


@pytest.mark.parametrize("name,T", [("small", 4096), ("latent", 2048)])
def test_aux_stats_vs_oracle(name, T):
    wl = W.ALL[name](T=T)
    z, pr, idx, tw = _route_gpu(wl)
    N = wl.N
    f = torch.empty(N, device="cuda")
    P = torch.empty(N, device="cuda")
    ns = torch.empty(1, device="cuda")
    loads = torch.empty(N, dtype=torch.int32, device="cuda")
    moe.moe_aux_stats(torch.from_numpy(pr).cuda(), torch.from_numpy(idx).cuda(), f, P, ns, loads)
    torch.cuda.synchronize()
    # the oracle's statistics from the oracle's own routing of the same tokens
    lz, lp, lidx, ltw = _route_oracle(wl, np.arange(T))
    of, oP, ons, oloads = O.aux_stats(lp, lidx)
    assert np.array_equal(loads.cpu().numpy(), oloads)
    assert np.array_equal(f.cpu().numpy() * T, np.round(of * T))
    assert np.allclose(P.cpu().numpy(), oP, rtol=1e-4, atol=1e-7)
    assert abs(ns.item() - ons) <= 1e-4 * max(1.0, abs(ons))
    assert loads.cpu().numpy().sum() == wl.k * T  # §3.6 conservation


@pytest.mark.parametrize("name,T", [("small", 4096), ("latent", 512)])
def test_aux_grad_vs_oracle(name, T):
    """Tutorial §3.7: dL_aux/dz from the GPU's own probabilities and loads,
    against the oracle's closed form on the same values."""
    wl = W.ALL[name](T=T)
    z, pr, idx, tw = _route_gpu(wl)
    N, alpha = wl.N, 0.01
    f = torch.empty(N, device="cuda")
    P = torch.empty(N, device="cuda")
    ns = torch.empty(1, device="cuda")
    probs = torch.from_numpy(pr).cuda()
    moe.moe_aux_stats(probs, torch.from_numpy(idx).cuda(), f, P, ns)
    dz = torch.empty((T, N), device="cuda")
    moe.moe_aux_grad(probs, f, dz, alpha)
    torch.cuda.synchronize()
    got = dz.cpu().numpy().astype(np.float64)
    ref = O.aux_grad(pr.astype(np.float64), f.cpu().numpy().astype(np.float64), alpha)
    scale = np.abs(ref).max()
    assert scale > 0
    assert np.abs(got - ref).max() <= 1e-5 * scale
    assert np.abs(got.sum(1)).max() <= 1e-5 * scale  # the gradients of a token sum to zero


# ----------------------------------------------------------------- permute
def _permute_gpu(idx_np, N, C):
    T, k = idx_np.shape
    s = moe.shape(T, 64, N, k, 64, 1, C)
    idx = torch.from_numpy(np.ascontiguousarray(idx_np, np.int32)).cuda()
    counts = torch.empty(N, dtype=torch.int32, device="cuda")
    offsets = torch.empty(N + 1, dtype=torch.int32, device="cuda")
    perm = torch.full((max(T * k, 1),), -7, dtype=torch.int32, device="cuda")
    row_of = torch.empty((T, k), dtype=torch.int32, device="cuda")
    overflow = torch.empty(N, dtype=torch.int32, device="cuda")
    totals = torch.empty(3, dtype=torch.int32, device="cuda")
    moe.moe_permute(s, idx, counts, offsets, perm, row_of, overflow, totals)
    torch.cuda.synchronize()
    rows = int(offsets[N].item())
    return dict(counts=counts.cpu().numpy(), offsets=offsets.cpu().numpy(),
                perm_tok=perm.cpu().numpy()[:rows], row_of=row_of.cpu().numpy(),
                overflow=overflow.cpu().numpy(), totals=totals.cpu().numpy())


def _assert_permute_equal(got, ref):
    for key in ("counts", "offsets", "perm_tok", "row_of", "overflow"):
        assert np.array_equal(got[key], ref[key]), key
    assert np.array_equal(got["totals"], ref["totals"].astype(np.int32))


def test_permute_tutorial_capacity_cases(golden):
    """Top-1 loads [10,3,2,1] and [4,4,4,4] at capacity 4/6/10 (tutorial §3.5, §3.8)."""
    for rec in golden("tutorial_capacity.txt"):
        a = (np.array([0] * 10 + [1] * 3 + [2] * 2 + [3]) if rec["case"] == "uneven"
             else np.arange(16) % 4).astype(np.int32)[:, None]
        C = moe.moe_capacity(16, 4, 1, float(rec["factor"]))
        got = _permute_gpu(a, 4, C)
        _assert_permute_equal(got, O.permute(a, 4, C))
        assert int(got["totals"][1]) == int(rec["dropped"])
        assert int(got["totals"][2]) == int(rec["empty"])


@pytest.mark.parametrize("T,N,k,C", [(1, 4, 2, 0), (37, 5, 2, 0), (1000, 8, 2, 211), (4096, 8, 2, 0),
                                     (8192, 8, 2, 2560), (4096, 896, 16, 0), (3001, 64, 6, 300),
                                     (300, 1024, 32, 9), (0, 8, 2, 0)])
def test_permute_bit_exact(T, N, k, C):
    rng = np.random.default_rng(T * 31 + N)
    z = rng.standard_normal((T, N)) + np.linspace(2.0, 0.0, N)[None, :]  # skewed loads
    idx = np.argsort(-z, axis=1, kind="stable")[:, :k].astype(np.int32)
    got = _permute_gpu(idx, N, C)
    ref = O.permute(idx, N, C)
    _assert_permute_equal(got, ref)
    assert int(got["totals"][0]) + int(got["totals"][1]) == T * k


def test_permute_bounds_error_is_recorded():
    """An expert id out of range is caught by the kernel's bounds check (no fault)."""
    idx = np.array([[0, 1], [9, 2]], np.int32)  # 9 >= N = 4
    _permute_gpu(idx, 4, 0)
    assert moe.moe_device_status() == -5
    moe.moe_reset_device_status()


# ------------------------------------------------------------ gather/combine
@pytest.mark.parametrize("dtype,width", [(S.DT_BF16, 512), (S.DT_F32, 64), (S.DT_F16, 136)])
def test_gather_bit_exact(dtype, width):
    T, N, k = 333, 8, 2
    rng = np.random.default_rng(4)
    idx = np.argsort(-rng.standard_normal((T, N)), axis=1)[:, :k].astype(np.int32)
    p = _permute_gpu(idx, N, 50)
    u = dev_normal(3, 1, (T, width), 1.0, dtype)
    s = moe.shape(T, width, N, k, 64, 1, 50)
    xr = torch.zeros((T * k, width), dtype=u.dtype, device="cuda")
    moe.moe_gather(s, width, u, torch.from_numpy(p["perm_tok"]).cuda(),
                   torch.from_numpy(p["offsets"]).cuda(), xr)
    torch.cuda.synchronize()
    rows = len(p["perm_tok"])
    ref = to_numpy_codes(u)[p["perm_tok"]]
    assert np.array_equal(to_numpy_codes(xr)[:rows], ref)


@pytest.mark.parametrize("y_dtype", [S.DT_F32, S.DT_BF16])
def test_combine_vs_oracle(y_dtype):
    T, N, k, width = 257, 6, 3, 384
    rng = np.random.default_rng(5)
    idx = np.argsort(-rng.standard_normal((T, N)), axis=1)[:, :k].astype(np.int32)
    p = _permute_gpu(idx, N, 100)
    rows = len(p["perm_tok"])
    yr = rng.standard_normal((T * k, width)).astype(np.float32)
    tw = rng.random((T, k)).astype(np.float32)
    s = moe.shape(T, width, N, k, 64, 1, 100)
    y = torch.empty((T, width), dtype=getattr(torch, {0: "float32", 1: "bfloat16"}[y_dtype]),
                    device="cuda")
    moe.moe_combine(s, width, torch.from_numpy(yr).cuda(), torch.from_numpy(p["row_of"]).cuda(),
                    torch.from_numpy(tw).cuda(), y)
    ref = O.combine(yr[:rows].astype(np.float64), p["row_of"], tw.astype(np.float64))
    got = y.float().cpu().numpy()
    if y_dtype == S.DT_F32:
        assert rel_err(got, ref) < 1e-6
    else:
        # bf16 output: within the bf16 layers' 2e-2 and one bf16 ulp of each value
        assert rel_err(got, ref) < 2e-2
        assert np.all(np.abs(got - ref) <= np.abs(ref) * 2.0 ** -8 + 1e-6)
    dropped = np.all(p["row_of"] < 0, axis=1)
    assert np.all(got[dropped] == 0.0)
