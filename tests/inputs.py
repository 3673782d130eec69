"""Workload inputs for the parity tests, drawn from the shared seeded generator.

Device tensors come from the generator's CUDA implementation, host arrays from
its C implementation; the two are bit-identical (checked in the GPU tests).
Nothing here computes any part of the MoE layer.
"""
from __future__ import annotations

import numpy as np

import oracle as O
import synthetic as S
from synthetic import workloads as W

TORCH_OF = {S.DT_F32: "float32", S.DT_BF16: "bfloat16", S.DT_F16: "float16"}
ORACLE_DT = {S.DT_F32: O.F32, S.DT_BF16: O.BF16, S.DT_F16: O.F16}


def torch_dtype(code):
    import torch
    return getattr(torch, TORCH_OF[code])


def dev_normal(seed, tid, shape, sigma, dtype, device="cuda", offset=0):
    import torch
    t = torch.empty(shape, dtype=torch_dtype(dtype), device=device)
    S.normal_dev(seed, tid, t.numel(), sigma, dtype, t.data_ptr(),
                 torch.cuda.current_stream().cuda_stream, offset)
    return t


def dev_u(wl: W.Workload, T=None, device="cuda"):
    import torch
    T = wl.T if T is None else T
    if wl.rms_inputs:
        t = torch.empty((T, wl.d), dtype=torch_dtype(wl.act_dtype), device=device)
        S.rmsnorm_rows_dev(wl.seed, W.TID_U, T, wl.d, wl.act_dtype, t.data_ptr(),
                           torch.cuda.current_stream().cuda_stream)
        return t
    return dev_normal(wl.seed, W.TID_U, (T, wl.d), wl.u_sigma, wl.act_dtype, device)


def host_u(wl: W.Workload, T=None):
    T = wl.T if T is None else T
    if wl.rms_inputs:
        return S.rmsnorm_rows(wl.seed, W.TID_U, T, wl.d, wl.act_dtype)
    return S.normal(wl.seed, W.TID_U, (T, wl.d), wl.u_sigma, wl.act_dtype)


def dev_router(wl: W.Workload, device="cuda", layer=0):
    import torch
    w = dev_normal(wl.seed, W.tid(W.TID_WROUTE, layer), (wl.N, wl.d), W.SIGMA_W, S.DT_F32, device)
    b = wl.router_bias()
    return w, (None if b is None else torch.from_numpy(b).to(device))


def host_router(wl: W.Workload, layer=0):
    return (S.normal(wl.seed, W.tid(W.TID_WROUTE, layer), (wl.N, wl.d), W.SIGMA_W, S.DT_F32),
            wl.router_bias())


def dev_experts(wl: W.Workload, device="cuda"):
    """W_gate [N][h][w], W_up [N][h][w], W_down [N][w][h] with w the expert width."""
    w, h, N = wl.expert_in, wl.h, wl.N
    dt = W.w_storage(wl)
    return (dev_normal(wl.seed, W.TID_WGATE, (N, h, w), W.SIGMA_W, dt, device),
            dev_normal(wl.seed, W.TID_WUP, (N, h, w), W.SIGMA_W, dt, device),
            dev_normal(wl.seed, W.TID_WDOWN, (N, w, h), W.SIGMA_W, dt, device))


def host_expert(wl: W.Workload, e: int):
    """Oracle matrices of expert e, drawn directly at that expert's offset."""
    w, h = wl.expert_in, wl.h
    dt = W.w_storage(wl)
    od = ORACLE_DT[dt]
    g = S.normal(wl.seed, W.TID_WGATE, (h, w), W.SIGMA_W, dt, offset=e * h * w)
    u = S.normal(wl.seed, W.TID_WUP, (h, w), W.SIGMA_W, dt, offset=e * h * w)
    d = S.normal(wl.seed, W.TID_WDOWN, (w, h), W.SIGMA_W, dt, offset=e * w * h)
    return O.Mat(od, h, w, data=g), O.Mat(od, h, w, data=u), O.Mat(od, w, h, data=d)


def to_numpy_codes(t):
    """Raw storage of a device tensor: uint16 codes for 16-bit types, else values."""
    import torch
    c = t.detach().cpu()
    if c.dtype in (torch.bfloat16, torch.float16):
        return c.view(torch.int16).numpy().view(np.uint16)
    return c.numpy()


def rel_err(got, ref):
    """max |got - ref| / rms(ref), the layer's output tolerance measure."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    rms = float(np.sqrt(np.mean(ref * ref)))
    return float(np.max(np.abs(got - ref))) / (rms if rms > 0 else 1.0)


def fro_err(got, ref):
    """||got - ref|| / ||ref|| (Frobenius), the gradients' tolerance measure."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    n = float(np.linalg.norm(ref))
    return float(np.linalg.norm(got - ref)) / (n if n > 0 else 1.0)


# ------------------------------------------------------------- LatentMoE
def dev_latent(wl: W.Workload, device="cuda"):
    """Device weights of a LatentMoE workload (bf16; router fp32)."""
    import torch
    E, d, l, h, n, sh = wl.N, wl.d, wl.latent, wl.h, wl.n_shared, wl.shared_hidden
    st = torch.cuda.current_stream().cuda_stream
    out = dict(
        w_route=dev_normal(wl.seed, W.TID_WROUTE, (E, d), W.SIGMA_W, S.DT_F32, device),
        w_gate=dev_normal(wl.seed, W.TID_WGATE, (E, h, l), wl.w_sigma, S.DT_BF16, device),
        w_up=dev_normal(wl.seed, W.TID_WUP, (E, h, l), wl.w_sigma, S.DT_BF16, device),
        w_down=dev_normal(wl.seed, W.TID_WDOWN, (E, l, h), wl.w_sigma, S.DT_BF16, device),
        w_dp=dev_normal(wl.seed, W.TID_WDP, (l, d), W.SIGMA_W, S.DT_BF16, device),
        w_upp=dev_normal(wl.seed, W.TID_WUPP, (d, l), W.SIGMA_W, S.DT_BF16, device))
    sg = torch.empty((max(n, 1), sh, d), dtype=torch.bfloat16, device=device)
    su = torch.empty_like(sg)
    sd = torch.empty((max(n, 1), d, sh), dtype=torch.bfloat16, device=device)
    for j in range(n):
        tg, tu, td = W.shared_tids(j)
        S.normal_dev(wl.seed, tg, sh * d, W.SIGMA_W, S.DT_BF16, sg[j].data_ptr(), st)
        S.normal_dev(wl.seed, tu, sh * d, W.SIGMA_W, S.DT_BF16, su[j].data_ptr(), st)
        S.normal_dev(wl.seed, td, d * sh, W.SIGMA_W, S.DT_BF16, sd[j].data_ptr(), st)
    out.update(shared_gate=sg, shared_up=su, shared_down=sd)
    return out


def host_latent_expert(wl: W.Workload, e: int):
    l, h = wl.latent, wl.h
    g = S.normal(wl.seed, W.TID_WGATE, (h, l), wl.w_sigma, S.DT_BF16, offset=e * h * l)
    u = S.normal(wl.seed, W.TID_WUP, (h, l), wl.w_sigma, S.DT_BF16, offset=e * h * l)
    d = S.normal(wl.seed, W.TID_WDOWN, (l, h), wl.w_sigma, S.DT_BF16, offset=e * l * h)
    return O.Mat(O.BF16, h, l, data=g), O.Mat(O.BF16, h, l, data=u), O.Mat(O.BF16, l, h, data=d)


def host_latent_dense(wl: W.Workload):
    d, l, sh = wl.d, wl.latent, wl.shared_hidden
    W_dp = O.Mat(O.BF16, l, d, data=S.normal(wl.seed, W.TID_WDP, (l, d), W.SIGMA_W, S.DT_BF16))
    W_upp = O.Mat(O.BF16, d, l, data=S.normal(wl.seed, W.TID_WUPP, (d, l), W.SIGMA_W, S.DT_BF16))
    shared = []
    for j in range(wl.n_shared):
        tg, tu, td = W.shared_tids(j)
        shared.append((O.Mat(O.BF16, sh, d, data=S.normal(wl.seed, tg, (sh, d), W.SIGMA_W,
                                                            S.DT_BF16)),
                       O.Mat(O.BF16, sh, d, data=S.normal(wl.seed, tu, (sh, d), W.SIGMA_W,
                                                            S.DT_BF16)),
                       O.Mat(O.BF16, d, sh, data=S.normal(wl.seed, td, (d, sh), W.SIGMA_W,
                                                            S.DT_BF16))))
    return W_dp, W_upp, shared
