"""GPU parity of the q4_0 decode path (deployment notes "Kestrel-MCU notes 13",
§2 lookup loading and §4 q4_0 experts) against the CPU oracle, through the C
ABI.  Routing bit-exact; layer outputs within max|d|/rms(y) <= 2e-2.

The 24-layer chain is checked layer by layer with teacher forcing: the GPU
layer runs on the oracle's own input to that layer, so a one-ulp fp16
difference cannot change a later layer's routing.  The fused chain entry
point is then checked against the layer calls made one by one on the GPU."""
import numpy as np
import pytest

import oracle as O
import synthetic as S
from synthetic import workloads as W

from inputs import rel_err

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

TOL_Q4 = 2e-2

if torch.cuda.is_available():
    import sparse_mixture_experts_15_b200 as moe


@pytest.fixture(autouse=True)
def _clean_status():
    moe.moe_reset_device_status()
    yield
    assert moe.moe_device_status() == 0


class Layer:
    """One decode layer's weights on both sides, from the seeded generator."""

    def __init__(self, wl, l):
        N, d, h, st = wl.N, wl.d, wl.h, torch.cuda.current_stream().cuda_stream
        self.w_route_h = S.normal(wl.seed, W.tid(W.TID_WROUTE, l), (N, d), W.SIGMA_W, S.DT_F32)
        self.w_route = torch.from_numpy(self.w_route_h).cuda()
        self.dev, self.mats = [], []
        host = []
        for base, rows, cols in ((W.TID_WGATE, h, d), (W.TID_WUP, h, d), (W.TID_WDOWN, d, h)):
            tid = W.tid(base, l)
            qs = torch.empty((N * rows, cols // 2), dtype=torch.uint8, device="cuda")
            sc = torch.empty((N * rows, cols // 32), dtype=torch.int16, device="cuda")
            S.q4_dev(wl.seed, tid, N * rows, cols, qs.data_ptr(), sc.data_ptr(), st)
            self.dev += [qs, sc]
            hq, hs = S.q4(wl.seed, tid, N * rows, cols)
            host.append([O.Mat(O.Q4_0, rows, cols, qs=hq[e * rows:(e + 1) * rows],
                               scales=hs[e * rows:(e + 1) * rows]) for e in range(N)])
        self.mats = list(zip(*host))
        self.abi = moe.q4_layer(self.w_route, *self.dev)


def _u0(wl):
    return S.normal(wl.seed, W.TID_U, (wl.T, wl.d), 1.0, S.DT_F16)


def _f16(codes):
    return torch.from_numpy(np.ascontiguousarray(codes).view(np.int16)).view(torch.float16).cuda()


def _codes(t):
    return t.cpu().view(torch.int16).numpy().view(np.uint16)


@pytest.mark.parametrize("T", [1, 8, 32])
def test_decode_layer_vs_oracle(T):
    wl = W.decode(T=T, n_layers=1)
    L = Layer(wl, 0)
    u = _u0(wl)
    s = moe.shape(T, wl.d, wl.N, wl.k, wl.h, 1, 0)
    y = torch.empty((T, wl.d), dtype=torch.float16, device="cuda")
    un = torch.empty_like(y)
    idx = torch.empty((T, wl.k), dtype=torch.int32, device="cuda")
    tw = torch.empty((T, wl.k), dtype=torch.float32, device="cuda")
    moe.moe_decode_layer(s, L.abi, _f16(u), y, un, idx, tw)
    torch.cuda.synchronize()
    oidx, otw, oy, oun = O.decode_layer(u, L.w_route_h, L.mats, wl.k)
    assert np.array_equal(idx.cpu().numpy(), oidx)
    assert np.allclose(tw.cpu().numpy(), otw, rtol=2e-6, atol=1e-7)
    assert rel_err(y.float().cpu().numpy(), oy) < TOL_Q4
    # u_next = fp16(u + y): within one fp16 ulp of the oracle's
    got = un.float().cpu().numpy()
    ref = O.decode(O.F16, oun)
    assert np.all(np.abs(got - ref) <= np.abs(ref) * 2.0 ** -10 + 2.0 ** -24)


def test_decode_chain_teacher_forced_and_fused():
    wl = W.decode(T=32, n_layers=24)
    layers = [Layer(wl, l) for l in range(wl.n_layers)]
    s = moe.shape(wl.T, wl.d, wl.N, wl.k, wl.h, 1, 0)
    u = _u0(wl)
    gpu_idx = []
    for l, L in enumerate(layers):
        y = torch.empty((wl.T, wl.d), dtype=torch.float16, device="cuda")
        idx = torch.empty((wl.T, wl.k), dtype=torch.int32, device="cuda")
        moe.moe_decode_layer(s, L.abi, _f16(u), y, None, idx)
        torch.cuda.synchronize()
        oidx, otw, oy, oun = O.decode_layer(u, L.w_route_h, L.mats, wl.k)
        assert np.array_equal(idx.cpu().numpy(), oidx), f"layer {l} routing"
        assert rel_err(y.float().cpu().numpy(), oy) < TOL_Q4, f"layer {l} output"
        u = oun  # teacher forcing: the next layer starts from the oracle's input
    # the chained entry point equals the layer calls made one by one on the GPU
    u0 = _f16(_u0(wl))
    out = torch.empty_like(u0)
    idx_all = torch.empty((wl.n_layers, wl.T, wl.k), dtype=torch.int32, device="cuda")
    moe.moe_decode_step(s, [L.abi for L in layers], u0, out, idx_all)
    cur = u0
    for l, L in enumerate(layers):
        y = torch.empty_like(cur)
        nxt = torch.empty_like(cur)
        idx = torch.empty((wl.T, wl.k), dtype=torch.int32, device="cuda")
        moe.moe_decode_layer(s, L.abi, cur, y, nxt, idx)
        assert torch.equal(idx, idx_all[l])
        cur = nxt
    torch.cuda.synchronize()
    assert np.array_equal(_codes(cur), _codes(out))


def test_decode_reads_only_selected_experts():
    """With every token routed to expert 0 (router rows 1.. zero, row 0 large),
    corrupting the other experts' weights must not change the output."""
    wl = W.decode(T=8, n_layers=1)
    L = Layer(wl, 0)
    N, d = wl.N, wl.d
    wr = torch.zeros((N, d), dtype=torch.float32, device="cuda")
    wr[0] = 1.0
    wr[1] = 0.5
    u = np.abs(_u0(wl).view(np.float16)).astype(np.float16).view(np.uint16)  # positive sums
    s = moe.shape(wl.T, d, N, wl.k, wl.h, 1, 0)
    layer = moe.q4_layer(wr, *L.dev)
    y1 = torch.empty((wl.T, d), dtype=torch.float16, device="cuda")
    moe.moe_decode_layer(s, layer, _f16(u), y1)
    for t in L.dev:  # scribble over experts 2..N-1 (rows of gate/up/down)
        rows = t.shape[0] // N
        t[2 * rows:].fill_(0x55 if t.dtype == torch.uint8 else 0x7BFF)
    y2 = torch.empty_like(y1)
    moe.moe_decode_layer(s, layer, _f16(u), y2)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)


@pytest.mark.parametrize("T,d,N,k,h", [
    (32, 512, 64, 8, 128),   # 64 experts top-8: more items than SMs, the two-phase kernel
    (32, 1024, 8, 2, 256),   # h = 256: the two-phase kernel (the per-token plan is too large)
    (5, 64, 4, 2, 32),       # tiny: one q4 block per hidden row, ragged T
    (3, 96, 4, 3, 64),       # d/32 = 3 blocks: uneven phase-A parts
    (16, 2048, 8, 2, 128),   # wide rows: per-token kernel with 4 hidden slices of 32
])
def test_decode_layer_other_shapes(T, d, N, k, h):
    import dataclasses
    wl = dataclasses.replace(W.decode(T=T, n_layers=1), d=d, N=N, k=k, h=h)
    L = Layer(wl, 0)
    u = _u0(wl)
    s = moe.shape(T, d, N, k, h, 1, 0)
    assert moe.moe_decode_workspace_bytes(s) > 0
    y = torch.empty((T, d), dtype=torch.float16, device="cuda")
    un = torch.empty_like(y)
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    moe.moe_decode_layer(s, L.abi, _f16(u), y, un, idx)
    torch.cuda.synchronize()
    oidx, otw, oy, oun = O.decode_layer(u, L.w_route_h, L.mats, k)
    assert np.array_equal(idx.cpu().numpy(), oidx)
    assert rel_err(y.float().cpu().numpy(), oy) < TOL_Q4


PER_TOKEN, TWO_PHASE = 1, 2  # moe_decode_kernel's answers


@pytest.mark.parametrize("T,d,N,k,h,kind", [
    (32, 1024, 8, 2, 256, TWO_PHASE),  # output units of 256 rows: two router blocks each
    (32, 512, 64, 8, 128, TWO_PHASE),  # 64 experts: 64 block sums per unit
    (16, 512, 8, 2, 128, PER_TOKEN),   # 16 tokens x 2 slots x 4 slices
    (16, 2048, 8, 2, 128, PER_TOKEN),  # wide rows
])
def test_decode_step_equals_layers(T, d, N, k, h, kind):
    """A 3-layer chained step (layers 1.. route from the router block sums
    that the previous layer formed, in either decode kernel, the one the
    shape runs checked by the kernel query) equals the layer calls made one
    by one, which form the block sums from their own input."""
    import dataclasses
    wl = dataclasses.replace(W.decode(T=T, n_layers=3), d=d, N=N, k=k, h=h)
    layers = [Layer(wl, l) for l in range(wl.n_layers)]
    s = moe.shape(T, d, N, k, h, 1, 0)
    assert moe.moe_decode_kernel(s) == kind
    u0 = _f16(_u0(wl))
    out = torch.empty_like(u0)
    idx_all = torch.empty((wl.n_layers, T, k), dtype=torch.int32, device="cuda")
    moe.moe_decode_step(s, [L.abi for L in layers], u0, out, idx_all)
    cur = u0
    for l, L in enumerate(layers):
        y = torch.empty_like(cur)
        nxt = torch.empty_like(cur)
        idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
        moe.moe_decode_layer(s, L.abi, cur, y, nxt, idx)
        assert torch.equal(idx, idx_all[l]), f"layer {l}"
        cur = nxt
    torch.cuda.synchronize()
    assert np.array_equal(_codes(cur), _codes(out))


def test_decode_step_chunks_and_graph_replay():
    """40 layers (more than one launch carries) at T=1: the chained call equals
    the layer calls made one by one, and a CUDA-graph replay of the chained
    call reproduces it bit for bit."""
    wl = W.decode(T=1, n_layers=40)
    layers = [Layer(wl, l) for l in range(wl.n_layers)]
    s = moe.shape(wl.T, wl.d, wl.N, wl.k, wl.h, 1, 0)
    u0 = _f16(_u0(wl))
    out = torch.empty_like(u0)
    idx_all = torch.empty((wl.n_layers, wl.T, wl.k), dtype=torch.int32, device="cuda")
    abis = [L.abi for L in layers]
    moe.moe_decode_step(s, abis, u0, out, idx_all)
    cur = u0
    for l, L in enumerate(layers):
        y = torch.empty_like(cur)
        nxt = torch.empty_like(cur)
        idx = torch.empty((wl.T, wl.k), dtype=torch.int32, device="cuda")
        moe.moe_decode_layer(s, L.abi, cur, y, nxt, idx)
        assert torch.equal(idx, idx_all[l]), f"layer {l}"
        cur = nxt
    torch.cuda.synchronize()
    assert np.array_equal(_codes(cur), _codes(out))
    ws = torch.empty(moe.moe_decode_workspace_bytes(s), dtype=torch.uint8, device="cuda")
    out2 = torch.zeros_like(out)
    g = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        with torch.cuda.graph(g, stream=side):
            moe.moe_decode_step(s, abis, u0, out2, ws=ws)
    torch.cuda.current_stream().wait_stream(side)
    for _ in range(2):
        out2.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert np.array_equal(_codes(out2), _codes(out))


@pytest.mark.parametrize("T", [8, 32])
def test_decode_step_trace_matches_and_stamps_phases(T):
    """The traced step (40 layers, two launches) gives the same output and
    routing as moe_decode_step, and each layer's phase stamps are
    non-decreasing SM cycle counts (block 0 stays on one SM)."""
    wl = W.decode(T=T, n_layers=40)
    layers = [Layer(wl, l) for l in range(wl.n_layers)]
    s = moe.shape(wl.T, wl.d, wl.N, wl.k, wl.h, 1, 0)
    u0 = _f16(_u0(wl))
    abis = [L.abi for L in layers]
    out, out_t = torch.empty_like(u0), torch.empty_like(u0)
    idx, idx_t = (torch.empty((wl.n_layers, wl.T, wl.k), dtype=torch.int32, device="cuda")
                  for _ in range(2))
    moe.moe_decode_step(s, abis, u0, out, idx)
    stamps = torch.zeros((wl.n_layers, moe.DECODE_STAMPS), dtype=torch.int64, device="cuda")
    moe.moe_decode_step_trace(s, abis, u0, out_t, stamps, idx_t)
    torch.cuda.synchronize()
    assert np.array_equal(_codes(out), _codes(out_t))
    assert torch.equal(idx, idx_t)
    st = stamps.cpu().numpy()
    assert np.all(st > 0)
    assert np.all(np.diff(st, axis=1) >= 0)
    assert np.all(st[1:32, 0] >= st[:31, -1])  # layers of one launch follow each other
    with pytest.raises(ValueError):
        moe.moe_decode_step_trace(s, abis, u0, out_t, stamps[:4], idx_t)


def test_decode_empty_batch():
    """T = 0: both decode entry points succeed and launch nothing."""
    wl = W.decode(T=1, n_layers=2)
    layers = [Layer(wl, l) for l in range(2)]
    s = moe.shape(0, wl.d, wl.N, wl.k, wl.h, 1, 0)
    u = torch.empty((0, wl.d), dtype=torch.float16, device="cuda")
    y = torch.empty_like(u)
    moe.moe_decode_layer(s, layers[0].abi, u, y)
    moe.moe_decode_step(s, [L.abi for L in layers], u, y)
    torch.cuda.synchronize()
