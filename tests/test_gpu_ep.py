"""Expert parallelism on the device (the dispatch and combine all-to-alls of
"Mixture of Experts MoE: how sparse activation saves compute", fused with the
gather and the weighted combine), through the C ABI.

R logical ranks share this GPU: every rank's buffers are separate device
allocations and the peer address tables hold them, so the kernels take the
same loads and stores they would take over NVLink.  The ranks' steps run one
after another on one stream (every rank's dispatch, then every owner's
experts, then every combine), so no kernel ever waits for one that has not
finished; the waits are satisfied when they start.  The expert-parallel layer
must equal the single-GPU layer on the ranks' batches laid end to end bit for
bit (same rows per expert in the same order, same kernels), and the oracle
within the bf16 bound."""
import numpy as np
import pytest

import oracle as O
import synthetic as S
from synthetic import workloads as W

from inputs import dev_experts, dev_router, host_expert, host_router, host_u, rel_err

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import sparse_mixture_experts_15_b200 as moe
    from sparse_mixture_experts_15_b200 import ep


@pytest.fixture(autouse=True)
def _clean_status():
    moe.moe_reset_device_status()
    yield
    assert moe.moe_device_status() == 0


def _ptrs(ts):
    return torch.tensor([t.data_ptr() for t in ts], dtype=torch.int64, device="cuda")


def _ep_layer(wl, splits, u_all, w, b, wg, wu, wd, epochs=1):
    """Run the expert-parallel layer over len(splits) logical ranks; rank r
    holds rows [start_r, start_r + splits[r]) of u_all.  Returns the ranks' y
    stacked in rank order and the plans."""
    R, N, k, d, h = len(splits), wl.N, wl.k, wl.d, wl.h
    E = N // R
    i32 = dict(dtype=torch.int32, device="cuda")
    starts = np.concatenate([[0], np.cumsum(splits)])
    ranks = []
    for r in range(R):
        T = int(splits[r])
        s = moe.shape(T, d, N, k, h, 1, 0)
        u = u_all[int(starts[r]):int(starts[r + 1])].contiguous()
        top_idx, top_w = torch.empty((T, k), **i32), torch.empty((T, k), dtype=torch.float32,
                                                                 device="cuda")
        moe.moe_route(s, u, w, top_idx, top_w, bias=b)
        loc = dict(counts=torch.empty(N, **i32), offsets=torch.empty(N + 1, **i32),
                   perm_tok=torch.empty(T * k, **i32), row_of=torch.empty((T, k), **i32),
                   overflow=torch.empty(N, **i32), totals=torch.empty(3, **i32))
        moe.moe_permute(s, top_idx, loc["counts"], loc["offsets"], loc["perm_tok"],
                        loc["row_of"], loc["overflow"], loc["totals"])
        ranks.append(dict(s=s, u=u, top_idx=top_idx, top_w=top_w, **loc))
    counts_all = np.stack([rk["counts"].cpu().numpy() for rk in ranks])
    plans = [ep.plan(counts_all, wl.capacity(int(sum(splits))), r) for r in range(R)]
    cap = max(16, max(p.recv_rows for p in plans))
    bufs = [dict(recv_rows=torch.zeros((cap, d), dtype=torch.bfloat16, device="cuda"),
                 recv_w=torch.zeros(cap, dtype=torch.float32, device="cuda"),
                 out_rows=torch.zeros((cap, d), dtype=torch.float32, device="cuda"),
                 arrive=torch.zeros(R, **i32), done=torch.zeros(4, **i32)) for _ in range(R)]
    peers = {n: _ptrs([bf[n] for bf in bufs]) for n in bufs[0]}
    es = moe.shape(cap, d, E, 1, h, 1, 0)
    for r, (rk, p) in enumerate(zip(ranks, plans)):
        rk["bufs"] = moe.ep_buffers(R, r, cap, bufs[r], peers)
        rk["kept"] = torch.from_numpy(p.kept).cuda()
        rk["send_base"] = torch.from_numpy(p.send_base).cuda()
        rk["recv_offsets"] = torch.from_numpy(p.recv_offsets).cuda()
        rk["ws"] = torch.empty(moe.moe_ep_workspace_bytes(es), dtype=torch.uint8, device="cuda")
        rk["y"] = torch.empty((rk["s"].T, d), dtype=torch.bfloat16, device="cuda")
    act = moe.act()
    for epoch in range(1, epochs + 1):
        for rk in ranks:
            moe.moe_ep_dispatch(rk["s"], rk["bufs"], epoch, rk["u"], rk["perm_tok"],
                                rk["offsets"], rk["row_of"], rk["top_w"], rk["kept"],
                                rk["send_base"], rk["ws"])
        for r, rk in enumerate(ranks):
            moe.moe_ep_expert_ffn(es, rk["bufs"], epoch, rk["recv_offsets"], wg[r * E:(r + 1) * E],
                                  wu[r * E:(r + 1) * E], wd[r * E:(r + 1) * E], rk["ws"], a=act)
        for rk in ranks:
            rk["y"].fill_(float("nan"))
            moe.moe_ep_combine(rk["s"], rk["bufs"], epoch, rk["top_idx"], rk["row_of"],
                               rk["offsets"], rk["kept"], rk["send_base"], rk["y"])
    torch.cuda.synchronize()
    for bf in bufs:  # every flag carries the last epoch
        assert torch.all(bf["arrive"] == epochs) and int(bf["done"][0]) == epochs
    return torch.cat([rk["y"] for rk in ranks]), plans, ranks


@pytest.mark.parametrize("case", ["two_ranks", "four_ranks_capacity", "two_ranks_grouped_gemm"])
def test_ep_layer_equals_single_gpu_layer(case):
    import dataclasses
    if case == "two_ranks":
        wl, splits = W.small(T=700), [413, 287]
    elif case == "four_ranks_capacity":
        wl = dataclasses.replace(W.small(T=900), capacity_factor=1.0, zipf_s=1.2)
        splits = [300, 1, 250, 349]
    else:  # h = 512: the two-launch grouped GEMM path on the owners
        wl, splits = dataclasses.replace(W.small(T=600), h=512), [320, 280]
    T = int(sum(splits))
    wl = dataclasses.replace(wl, T=T)
    u_all = torch.from_numpy(host_u(wl).view(np.int16)).view(torch.bfloat16).cuda()
    w, b = dev_router(wl)
    wg, wu, wd = dev_experts(wl)
    y_ep, plans, ranks = _ep_layer(wl, splits, u_all, w, b, wg, wu, wd, epochs=2)
    # the single-GPU layer on the concatenated batch
    s = moe.shape(T, wl.d, wl.N, wl.k, wl.h, 1, wl.capacity())
    y_one = torch.empty((T, wl.d), dtype=torch.bfloat16, device="cuda")
    row_of = torch.empty((T, wl.k), dtype=torch.int32, device="cuda")
    moe.moe_layer_fwd(s, w, wg, wu, wd, u_all, y_one, bias=b, outputs={"row_of": row_of})
    torch.cuda.synchronize()
    assert torch.equal(y_ep.view(torch.int16), y_one.view(torch.int16))
    # the plan's overflow is the single-GPU layer's (capacity over all ranks)
    idx_all = torch.cat([rk["top_idx"] for rk in ranks]).cpu().numpy()
    perm = O.permute(idx_all, wl.N, wl.capacity())
    assert np.array_equal(plans[0].overflow, perm["overflow"])
    if case == "four_ranks_capacity":
        assert perm["totals"][1] > 0
    # and the oracle, within the bf16 bound (rows the layer computes)
    wr, bias = host_router(wl)
    uh = host_u(wl)
    _, _, idx, tw = O.route(O.as_f32(O.BF16, uh), wr, wl.k, 1, bias)
    assert np.array_equal(idx, idx_all)
    mats = [host_expert(wl, e) for e in range(wl.N)]
    ref = O.moe_tokens([m[0] for m in mats], [m[1] for m in mats], [m[2] for m in mats],
                       O.decode(O.BF16, uh), idx, tw, row_of=perm["row_of"], round_h=1)
    got = y_ep.float().cpu().numpy()
    gone = (perm["row_of"] < 0).all(1)
    assert np.all(got[gone] == 0.0)
    assert rel_err(got[~gone], ref[~gone]) < 2e-2


def test_ep_wait_runs_out_without_arrivals():
    """An owner whose sources never arrived gives up after its bounded wait:
    MOE_ERR_TIMEOUT in the status word, and the call returns."""
    wl = W.small(T=64)
    R, E = 2, wl.N // 2
    i32 = dict(dtype=torch.int32, device="cuda")
    cap = 64
    bufs = [dict(recv_rows=torch.zeros((cap, wl.d), dtype=torch.bfloat16, device="cuda"),
                 recv_w=torch.zeros(cap, dtype=torch.float32, device="cuda"),
                 out_rows=torch.zeros((cap, wl.d), dtype=torch.float32, device="cuda"),
                 arrive=torch.zeros(R, **i32), done=torch.zeros(4, **i32)) for _ in range(R)]
    peers = {n: _ptrs([bf[n] for bf in bufs]) for n in bufs[0]}
    es = moe.shape(cap, wl.d, E, 1, wl.h, 1, 0)
    wg, wu, wd = dev_experts(wl)
    ws = torch.empty(moe.moe_ep_workspace_bytes(es), dtype=torch.uint8, device="cuda")
    recv_offsets = torch.zeros(E + 1, **i32)
    moe.moe_ep_expert_ffn(es, moe.ep_buffers(R, 0, cap, bufs[0], peers), 1, recv_offsets,
                          wg[:E], wu[:E], wd[:E], ws)
    torch.cuda.synchronize()
    assert moe.moe_device_status() == -4  # MOE_ERR_TIMEOUT
    moe.moe_reset_device_status()
