"""Python binding of the sm_100a sparse-MoE layer library (libmoe.so).

Argument marshalling only: every function here converts torch tensors to
device pointers, calls the C entry point of the same name declared in
include/moe.h, and raises MoeError on a non-zero status.  All compute runs in
the library's CUDA kernels; there is no Python or CPU fallback.  Importing
this package fails loudly when libmoe.so has not been built.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe.so")

F32, BF16, F16, Q4_0, E4M3 = 0, 1, 2, 3, 4
ACT_SWIGLU, ACT_SITU_GLU = 0, 1

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with "
                      "`python sparse_mixture_experts_15_b200/build.py` (nvcc, sm_100a)")
_lib = ctypes.CDLL(LIB_PATH)

_i32, _i64, _sz, _vp, _f32, _f64 = (ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t,
                                    ctypes.c_void_p, ctypes.c_float, ctypes.c_double)


class MoeShape(ctypes.Structure):
    _fields_ = [("T", _i32), ("d", _i32), ("N", _i32), ("k", _i32), ("h", _i32),
                ("renorm", _i32), ("capacity", _i32)]


class MoeAct(ctypes.Structure):
    _fields_ = [("kind", _i32), ("beta_gate", _f32), ("beta_up", _f32)]


class MoeLayerWeights(ctypes.Structure):
    _fields_ = [("w_route", _vp), ("bias", _vp), ("w_gate", _vp), ("w_up", _vp),
                ("w_down", _vp), ("w_dtype", _i32), ("act", MoeAct)]


class MoeLayerOutputs(ctypes.Structure):
    _fields_ = [(n, _vp) for n in ("top_idx", "top_w", "probs", "counts", "offsets", "perm_tok",
                                   "row_of", "overflow", "totals", "f", "P", "n_sum_fP")]


class MoeQ4Layer(ctypes.Structure):
    _fields_ = [(n, _vp) for n in ("w_route", "bias", "gate_qs", "gate_scales", "up_qs",
                                   "up_scales", "down_qs", "down_scales")]


class MoeLatentWeights(ctypes.Structure):
    _fields_ = [("latent", _i32), ("n_shared", _i32), ("shared_hidden", _i32),
                ("w_down_proj", _vp), ("w_up_proj", _vp), ("shared_gate", _vp),
                ("shared_up", _vp), ("shared_down", _vp), ("rms_eps", _f32)]


class MoeLayerGrads(ctypes.Structure):
    _fields_ = [(n, _vp) for n in ("du", "dz", "dw_route", "dw_gate", "dw_up", "dw_down")]


class MoeLatentGrads(ctypes.Structure):
    _fields_ = [(n, _vp) for n in ("dx", "dz", "dw_route", "dw_gate", "dw_up", "dw_down", "dw_dp",
                                   "dw_upp", "dsh_gate", "dsh_up", "dsh_down")]


class MoeE4M3Scales(ctypes.Structure):
    _fields_ = [(n, _vp) for n in ("gate_scale", "up_scale", "down_scale")]


class MoeEpBuffers(ctypes.Structure):
    _fields_ = [("world", _i32), ("rank", _i32), ("recv_capacity", _i32)] + [
        (n, _vp) for n in ("recv_rows", "recv_w", "out_rows", "arrive", "done", "peer_recv_rows",
                           "peer_recv_w", "peer_out_rows", "peer_arrive", "peer_done")]


_P_SHAPE = ctypes.POINTER(MoeShape)
_PROTOS = {
    "moe_capacity": (_i32, [_i64, _i32, _i32, _f64, ctypes.POINTER(_i32)]),
    "moe_route_workspace_bytes": (_sz, [_P_SHAPE]),
    "moe_route": (_i32, [_P_SHAPE, _vp, _i32, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "moe_aux_stats_workspace_bytes": (_sz, [_i32]),
    "moe_aux_stats": (_i32, [_i32, _i32, _i32, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "moe_permute_workspace_bytes": (_sz, [_P_SHAPE]),
    "moe_permute": (_i32, [_P_SHAPE, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "moe_permute_noalloc": (_i32, [_P_SHAPE, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp]),
    "moe_gather": (_i32, [_P_SHAPE, _i32, _vp, _i32, _vp, _vp, _vp, _vp]),
    "moe_expert_ffn_workspace_bytes": (_sz, [_P_SHAPE, _i32, _i32]),
    "moe_expert_ffn": (_i32, [_P_SHAPE, _i32, _vp, _i32, _vp, _vp, _vp, _vp, _i32,
                              ctypes.POINTER(MoeAct), _vp, _vp, _sz, _vp]),
    "moe_combine": (_i32, [_P_SHAPE, _i32, _vp, _vp, _vp, _vp, _i32, _vp]),
    "moe_layer_workspace_bytes": (_sz, [_P_SHAPE, _i32]),
    "moe_layer_fwd": (_i32, [_P_SHAPE, ctypes.POINTER(MoeLayerWeights), _vp, _i32, _vp,
                             ctypes.POINTER(MoeLayerOutputs), _vp, _sz, _vp]),
    "moe_layer_bwd_workspace_bytes": (_sz, [_P_SHAPE]),
    "moe_layer_bwd": (_i32, [_P_SHAPE, ctypes.POINTER(MoeLayerWeights), _vp, _vp,
                             ctypes.POINTER(MoeLayerOutputs), _f32, _vp,
                             ctypes.POINTER(MoeLayerGrads), _vp, _sz, _vp]),
    "moe_latent_workspace_bytes": (_sz, [_P_SHAPE, ctypes.POINTER(MoeLatentWeights)]),
    "moe_latent_fwd": (_i32, [_P_SHAPE, ctypes.POINTER(MoeLayerWeights),
                              ctypes.POINTER(MoeLatentWeights), _vp, _vp,
                              ctypes.POINTER(MoeLayerOutputs), _vp, _sz, _vp]),
    "moe_quantize_e4m3_rows": (_i32, [_i64, _i32, _vp, _i32, _vp, _vp, _vp]),
    "moe_expert_ffn_e4m3_workspace_bytes": (_sz, [_P_SHAPE]),
    "moe_expert_ffn_e4m3": (_i32, [_P_SHAPE, _i32, _vp, _vp, _vp, _vp, _vp, _vp,
                                   ctypes.POINTER(MoeE4M3Scales), ctypes.POINTER(MoeAct), _vp,
                                   _vp, _sz, _vp]),
    "moe_latent_bwd_workspace_bytes": (_sz, [_P_SHAPE, ctypes.POINTER(MoeLatentWeights)]),
    "moe_latent_bwd": (_i32, [_P_SHAPE, ctypes.POINTER(MoeLayerWeights),
                              ctypes.POINTER(MoeLatentWeights), _vp, _vp,
                              ctypes.POINTER(MoeLayerOutputs), ctypes.POINTER(MoeLatentGrads), _vp,
                              _sz, _vp]),
    "moe_latent_fwd_e4m3": (_i32, [_P_SHAPE, ctypes.POINTER(MoeLayerWeights),
                                   ctypes.POINTER(MoeE4M3Scales),
                                   ctypes.POINTER(MoeLatentWeights), _vp, _vp,
                                   ctypes.POINTER(MoeLayerOutputs), _vp, _sz, _vp]),
    "moe_decode_kernel": (_i32, [_P_SHAPE]),
    "moe_decode_workspace_bytes": (_sz, [_P_SHAPE]),
    "moe_decode_layer": (_i32, [_P_SHAPE, ctypes.POINTER(MoeQ4Layer), _vp, _vp, _vp, _vp, _vp,
                                _vp, _sz, _vp]),
    "moe_decode_step": (_i32, [_P_SHAPE, _i32, ctypes.POINTER(MoeQ4Layer), _vp, _vp, _vp, _vp,
                               _sz, _vp]),
    "moe_decode_step_trace": (_i32, [_P_SHAPE, _i32, ctypes.POINTER(MoeQ4Layer), _vp, _vp, _vp,
                                     _vp, _sz, _vp, _vp]),
    "moe_aux_grad": (_i32, [_i32, _i32, _f32, _vp, _vp, _vp, _vp]),
    "moe_quantile_balance_workspace_bytes": (_sz, [_i32, _i32]),
    "moe_quantile_balance": (_i32, [_i32, _i32, _i32, _vp, _vp, _i32, _i32, _vp, _vp, _vp, _vp,
                                    _vp, _sz, _vp]),
    "moe_ep_plan": (_i32, [_i32, _i32, _i32, _i32] + [_vp] * 9),
    "moe_ep_workspace_bytes": (_sz, [_P_SHAPE]),
    "moe_ep_dispatch": (_i32, [_P_SHAPE, ctypes.POINTER(MoeEpBuffers), ctypes.c_uint32] +
                        [_vp] * 7 + [_vp, _sz, _vp]),
    "moe_ep_expert_ffn": (_i32, [_P_SHAPE, ctypes.POINTER(MoeEpBuffers), ctypes.c_uint32, _vp,
                                 _vp, _vp, _vp, ctypes.POINTER(MoeAct), _vp, _sz, _vp]),
    "moe_ep_combine": (_i32, [_P_SHAPE, ctypes.POINTER(MoeEpBuffers), ctypes.c_uint32] +
                       [_vp] * 6 + [_vp]),
    "moe_status_string": (ctypes.c_char_p, [_i32]),
    "moe_device_status": (_i32, [_vp, ctypes.POINTER(_i32)]),
    "moe_reset_device_status": (_i32, [_vp]),
    "moe_wait_check": (_i32, [_i32, _i64, _vp]),
}
for _name, (_res, _args) in _PROTOS.items():
    _fn = getattr(_lib, _name)
    _fn.restype, _fn.argtypes = _res, _args

EXPORTED = tuple(_PROTOS)


class MoeError(RuntimeError):
    def __init__(self, status: int, where: str):
        msg = _lib.moe_status_string(status).decode()
        super().__init__(f"{where}: {msg} ({status})")
        self.status = status


def _check(rc: int, where: str):
    if rc != 0:
        raise MoeError(rc, where)


def _ptr(t):
    """Device address of a tensor the library reads or writes (None -> NULL).
    The kernels take every tensor as a dense row-major array in device
    memory, so a host tensor or a strided view is refused here, before any
    call: its address would point the kernels at the wrong memory."""
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"expected a CUDA tensor, got a tensor on {t.device}")
    if not t.is_contiguous():
        raise ValueError(f"expected a contiguous tensor, got strides {tuple(t.stride())}")
    return t.data_ptr()


_F32, _I32, _F16, _BF16, _U8 = "float32", "int32", "float16", "bfloat16", "uint8"
_ACT = (_F32, _BF16, _F16)  # activation storage types
_Q4_SCALES = ("int16", "uint16")  # fp16 scale codes, any 16-bit integer view


def _need(what, t, n, dtypes=None):
    """Refuse a tensor with fewer than n elements where the call touches n, or
    of another element type than the library reads or writes there.  The
    library sees only the address, so a short or narrower tensor would be read
    or written past its end on the device."""
    if t is None:
        return
    if t.numel() < n:
        raise ValueError(f"{what}: {t.numel()} elements, the call needs at least {n}")
    if dtypes is not None:
        allowed = (dtypes,) if isinstance(dtypes, str) else tuple(dtypes)
        name = str(t.dtype).replace("torch.", "")
        if name not in allowed:
            raise ValueError(f"{what}: dtype {name}, the call needs {' or '.join(allowed)}")


def _outputs(s: MoeShape, outputs):
    """moe_layer_outputs from a dict of tensors, each checked against its
    documented size."""
    Tk, TN, N = s.T * s.k, s.T * s.N, s.N
    sizes = dict(top_idx=(Tk, _I32), top_w=(Tk, _F32), probs=(TN, _F32), counts=(N, _I32),
                 offsets=(N + 1, _I32), perm_tok=(Tk, _I32), row_of=(Tk, _I32),
                 overflow=(N, _I32), totals=(3, _I32), f=(N, _F32), P=(N, _F32),
                 n_sum_fP=(1, _F32))
    for key, t in (outputs or {}).items():
        _need(key, t, *sizes[key])
    return MoeLayerOutputs(**{key: _ptr(t) for key, t in (outputs or {}).items()})


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    return int(stream)


def _dtype_code(t):
    import torch
    return {torch.float32: F32, torch.bfloat16: BF16, torch.float16: F16}[t.dtype]


def _ws(nbytes, device, ws=None):
    import torch
    if ws is not None:
        if ws.numel() * ws.element_size() < nbytes:
            raise MoeError(-6, "workspace")
        return ws, ws.numel() * ws.element_size()
    n = max(int(nbytes), 256)
    return torch.empty(n, dtype=torch.uint8, device=device), n


def shape(T, d, N, k, h=0, renorm=1, capacity=0) -> MoeShape:
    return MoeShape(T, d, N, k, h, renorm, capacity)


def act(kind=ACT_SWIGLU, beta_gate=0.0, beta_up=0.0) -> MoeAct:
    return MoeAct(kind, beta_gate, beta_up)


# ------------------------------------------------------------- entry points
def moe_capacity(T: int, N: int, k: int, factor: float) -> int:
    out = _i32(0)
    _check(_lib.moe_capacity(T, N, k, factor, ctypes.byref(out)), "moe_capacity")
    return out.value


def moe_route(s: MoeShape, u, w_route, top_idx, top_w, bias=None, probs=None, logits=None,
              ws=None, stream=None):
    for args in (("u", u, s.T * s.d, _ACT), ("w_route", w_route, s.N * s.d, _F32),
                 ("bias", bias, s.N, _F32), ("top_idx", top_idx, s.T * s.k, _I32),
                 ("top_w", top_w, s.T * s.k, _F32), ("probs", probs, s.T * s.N, _F32),
                 ("logits", logits, s.T * s.N, _F32)):
        _need(*args)
    nb = _lib.moe_route_workspace_bytes(ctypes.byref(s))
    wbuf, wlen = (None, 0) if logits is not None else _ws(nb, u.device, ws)
    _check(_lib.moe_route(ctypes.byref(s), _ptr(u), _dtype_code(u), _ptr(w_route), _ptr(bias),
                          _ptr(top_idx), _ptr(top_w), _ptr(probs), _ptr(logits), _ptr(wbuf), wlen,
                          _stream(stream)), "moe_route")


def moe_aux_stats(probs, top_idx, f=None, P=None, n_sum_fP=None, loads=None, ws=None,
                  stream=None):
    T, k = top_idx.shape
    N = f.shape[0] if f is not None else (P.shape[0] if P is not None else loads.shape[0])
    for args in (("probs", probs, T * N, _F32), ("top_idx", top_idx, T * k, _I32),
                 ("f", f, N, _F32), ("P", P, N, _F32), ("n_sum_fP", n_sum_fP, 1, _F32),
                 ("loads", loads, N, _I32)):
        _need(*args)
    wbuf, wlen = _ws(_lib.moe_aux_stats_workspace_bytes(N), top_idx.device, ws)
    _check(_lib.moe_aux_stats(T, N, k, _ptr(probs), _ptr(top_idx), _ptr(f), _ptr(P),
                              _ptr(n_sum_fP), _ptr(loads), _ptr(wbuf), wlen, _stream(stream)),
           "moe_aux_stats")


def _permute_sizes(s, top_idx, counts, offsets, perm_tok, row_of, overflow, totals):
    Tk = s.T * s.k
    for what, t, n in (("top_idx", top_idx, Tk), ("counts", counts, s.N),
                       ("offsets", offsets, s.N + 1), ("perm_tok", perm_tok, Tk),
                       ("row_of", row_of, Tk), ("overflow", overflow, s.N), ("totals", totals, 3)):
        _need(what, t, n, _I32)


def moe_permute(s: MoeShape, top_idx, counts, offsets, perm_tok, row_of, overflow, totals,
                ws=None, stream=None):
    _permute_sizes(s, top_idx, counts, offsets, perm_tok, row_of, overflow, totals)
    wbuf, wlen = _ws(_lib.moe_permute_workspace_bytes(ctypes.byref(s)), top_idx.device, ws)
    _check(_lib.moe_permute(ctypes.byref(s), _ptr(top_idx), _ptr(counts), _ptr(offsets),
                            _ptr(perm_tok), _ptr(row_of), _ptr(overflow), _ptr(totals), _ptr(wbuf),
                            wlen, _stream(stream)), "moe_permute")


def moe_permute_noalloc(s: MoeShape, top_idx, counts, offsets, perm_tok, row_of, overflow,
                        totals, stream=None):
    """moe_permute without a workspace (the library's fixed 1 MiB scratch)."""
    _permute_sizes(s, top_idx, counts, offsets, perm_tok, row_of, overflow, totals)
    _check(_lib.moe_permute_noalloc(ctypes.byref(s), _ptr(top_idx), _ptr(counts), _ptr(offsets),
                                    _ptr(perm_tok), _ptr(row_of), _ptr(overflow), _ptr(totals),
                                    _stream(stream)), "moe_permute_noalloc")


def moe_gather(s: MoeShape, width: int, u, perm_tok, offsets, x_rows, stream=None):
    """perm_tok is read for the offsets[N] grouped rows only, a count the
    device holds, so its size is not checked here."""
    _need("u", u, s.T * width, _ACT)
    _need("perm_tok", perm_tok, 0, _I32)
    _need("offsets", offsets, s.N + 1, _I32)
    _need("x_rows", x_rows, s.T * s.k * width, str(u.dtype).replace("torch.", ""))
    _check(_lib.moe_gather(ctypes.byref(s), width, _ptr(u), _dtype_code(u), _ptr(perm_tok),
                           _ptr(offsets), _ptr(x_rows), _stream(stream)), "moe_gather")


def moe_expert_ffn(s: MoeShape, width: int, x_rows, offsets, w_gate, w_up, w_down, y_rows,
                   a: MoeAct | None = None, ws=None, stream=None):
    a = a or act()
    rows = s.T * s.k
    x_dt = str(x_rows.dtype).replace("torch.", "")
    for args in (("x_rows", x_rows, rows * width, (_F32, _BF16)),
                 ("offsets", offsets, s.N + 1, _I32),
                 ("w_gate", w_gate, s.N * s.h * width, x_dt), ("w_up", w_up, s.N * s.h * width, x_dt),
                 ("w_down", w_down, s.N * width * s.h, x_dt),
                 ("y_rows", y_rows, rows * width, _F32)):
        _need(*args)
    dt = _dtype_code(x_rows)
    nb = _lib.moe_expert_ffn_workspace_bytes(ctypes.byref(s), width, dt)
    wbuf, wlen = _ws(nb, x_rows.device, ws)
    _check(_lib.moe_expert_ffn(ctypes.byref(s), width, _ptr(x_rows), dt, _ptr(offsets),
                               _ptr(w_gate), _ptr(w_up), _ptr(w_down), _dtype_code(w_gate),
                               ctypes.byref(a), _ptr(y_rows), _ptr(wbuf), wlen, _stream(stream)),
           "moe_expert_ffn")


def moe_combine(s: MoeShape, width: int, y_rows, row_of, top_w, y, stream=None):
    """y_rows is read at the rows row_of names, so its size is not checked here."""
    for args in (("y_rows", y_rows, 0, _F32), ("row_of", row_of, s.T * s.k, _I32),
                 ("top_w", top_w, s.T * s.k, _F32), ("y", y, s.T * width, _ACT)):
        _need(*args)
    _check(_lib.moe_combine(ctypes.byref(s), width, _ptr(y_rows), _ptr(row_of), _ptr(top_w),
                            _ptr(y), _dtype_code(y), _stream(stream)), "moe_combine")


def moe_layer_workspace_bytes(s: MoeShape, act_dtype: int) -> int:
    return int(_lib.moe_layer_workspace_bytes(ctypes.byref(s), act_dtype))


def moe_layer_fwd(s: MoeShape, w_route, w_gate, w_up, w_down, u, y, bias=None, a=None,
                  outputs: dict | None = None, ws=None, stream=None):
    """The whole layer.  `outputs` maps moe_layer_outputs field names to tensors."""
    a = a or act()
    dt = _dtype_code(u)
    u_dt = str(u.dtype).replace("torch.", "")
    for args in (("u", u, s.T * s.d, (_F32, _BF16)), ("y", y, s.T * s.d, u_dt),
                 ("w_route", w_route, s.N * s.d, _F32), ("bias", bias, s.N, _F32),
                 ("w_gate", w_gate, s.N * s.h * s.d, u_dt), ("w_up", w_up, s.N * s.h * s.d, u_dt),
                 ("w_down", w_down, s.N * s.d * s.h, u_dt)):
        _need(*args)
    O = _outputs(s, outputs)
    W = MoeLayerWeights(_ptr(w_route), _ptr(bias), _ptr(w_gate), _ptr(w_up), _ptr(w_down),
                        _dtype_code(w_gate), a)
    wbuf, wlen = _ws(moe_layer_workspace_bytes(s, dt), u.device, ws)
    _check(_lib.moe_layer_fwd(ctypes.byref(s), ctypes.byref(W), _ptr(u), dt, _ptr(y),
                              ctypes.byref(O), _ptr(wbuf), wlen, _stream(stream)), "moe_layer_fwd")


def moe_layer_bwd_workspace_bytes(s: MoeShape) -> int:
    return int(_lib.moe_layer_bwd_workspace_bytes(ctypes.byref(s)))


def moe_layer_bwd(s: MoeShape, w_route, w_gate, w_up, w_down, u, dy, fwd: dict, grads: dict,
                  bias=None, a=None, alpha: float = 0.0, f=None, ws=None, stream=None):
    """Layer backward (include/moe.h): fwd holds the forward's top_idx, top_w,
    probs, offsets, perm_tok, row_of; grads the fp32 outputs du, dz, dw_route
    (optional), dw_gate, dw_up, dw_down; f (optional) the loads of the
    balancing term."""
    a = a or act()
    Tk = s.T * s.k
    for args in (("u", u, s.T * s.d, _BF16), ("dy", dy, s.T * s.d, _BF16),
                 ("w_route", w_route, s.N * s.d, _F32), ("bias", bias, s.N, _F32),
                 ("w_gate", w_gate, s.N * s.h * s.d, _BF16), ("w_up", w_up, s.N * s.h * s.d, _BF16),
                 ("w_down", w_down, s.N * s.d * s.h, _BF16), ("f", f, s.N, _F32),
                 ("top_idx", fwd.get("top_idx"), Tk, _I32), ("top_w", fwd.get("top_w"), Tk, _F32),
                 ("probs", fwd.get("probs"), s.T * s.N, _F32),
                 ("offsets", fwd.get("offsets"), s.N + 1, _I32),
                 ("perm_tok", fwd.get("perm_tok"), 0, _I32), ("row_of", fwd.get("row_of"), Tk, _I32),
                 ("du", grads.get("du"), s.T * s.d, _F32), ("dz", grads.get("dz"), s.T * s.N, _F32),
                 ("dw_route", grads.get("dw_route"), s.N * s.d, _F32),
                 ("dw_gate", grads.get("dw_gate"), s.N * s.h * s.d, _F32),
                 ("dw_up", grads.get("dw_up"), s.N * s.h * s.d, _F32),
                 ("dw_down", grads.get("dw_down"), s.N * s.d * s.h, _F32)):
        _need(*args)
    W = MoeLayerWeights(_ptr(w_route), _ptr(bias), _ptr(w_gate), _ptr(w_up), _ptr(w_down), BF16, a)
    O = _outputs(s, fwd)
    G = MoeLayerGrads(*(_ptr(grads.get(n)) for n in ("du", "dz", "dw_route", "dw_gate", "dw_up",
                                                     "dw_down")))
    wbuf, wlen = _ws(moe_layer_bwd_workspace_bytes(s), u.device, ws)
    _check(_lib.moe_layer_bwd(ctypes.byref(s), ctypes.byref(W), _ptr(u), _ptr(dy),
                              ctypes.byref(O), alpha, _ptr(f), ctypes.byref(G), _ptr(wbuf), wlen,
                              _stream(stream)), "moe_layer_bwd")


def latent_weights(latent, w_down_proj, w_up_proj, shared_gate=None, shared_up=None,
                   shared_down=None, n_shared=0, shared_hidden=0, rms_eps=1e-6):
    return MoeLatentWeights(latent, n_shared, shared_hidden, _ptr(w_down_proj), _ptr(w_up_proj),
                            _ptr(shared_gate), _ptr(shared_up), _ptr(shared_down), rms_eps)


def moe_latent_workspace_bytes(s: MoeShape, lw: MoeLatentWeights) -> int:
    return int(_lib.moe_latent_workspace_bytes(ctypes.byref(s), ctypes.byref(lw)))


def moe_latent_fwd(s: MoeShape, w_route, w_gate, w_up, w_down, lw: MoeLatentWeights, x, y,
                   bias=None, a=None, outputs: dict | None = None, ws=None, stream=None):
    """The LatentMoE layer; x, y bf16 [T][d]; routed experts at latent width."""
    a = a or act()
    l = lw.latent
    for args in (("x", x, s.T * s.d, _BF16), ("y", y, s.T * s.d, _BF16),
                 ("w_route", w_route, s.N * s.d, _F32), ("bias", bias, s.N, _F32),
                 ("w_gate", w_gate, s.N * s.h * l, _BF16), ("w_up", w_up, s.N * s.h * l, _BF16),
                 ("w_down", w_down, s.N * l * s.h, _BF16)):
        _need(*args)
    O = _outputs(s, outputs)
    W = MoeLayerWeights(_ptr(w_route), _ptr(bias), _ptr(w_gate), _ptr(w_up), _ptr(w_down), BF16,
                        a)
    wbuf, wlen = _ws(moe_latent_workspace_bytes(s, lw), x.device, ws)
    _check(_lib.moe_latent_fwd(ctypes.byref(s), ctypes.byref(W), ctypes.byref(lw), _ptr(x),
                               _ptr(y), ctypes.byref(O), _ptr(wbuf), wlen, _stream(stream)),
           "moe_latent_fwd")


def moe_latent_bwd(s: MoeShape, w_route, w_gate, w_up, w_down, lw: MoeLatentWeights, x, dy,
                   fwd: dict, grads: dict, bias=None, a=None, ws=None, stream=None):
    """LatentMoE backward (include/moe.h): fwd holds the forward's top_idx,
    top_w, probs, offsets, perm_tok, row_of; grads the fp32 outputs."""
    a = a or act()
    l, n, sh = lw.latent, lw.n_shared, lw.shared_hidden
    sizes = dict(dx=s.T * s.d, dz=s.T * s.N, dw_route=s.N * s.d, dw_gate=s.N * s.h * l,
                 dw_up=s.N * s.h * l, dw_down=s.N * l * s.h, dw_dp=l * s.d, dw_upp=s.d * l,
                 dsh_gate=n * sh * s.d, dsh_up=n * sh * s.d, dsh_down=n * s.d * sh)
    for key, t in grads.items():
        _need(key, t, sizes[key], _F32)
    for args in (("x", x, s.T * s.d, _BF16), ("dy", dy, s.T * s.d, _BF16),
                 ("w_route", w_route, s.N * s.d, _F32), ("bias", bias, s.N, _F32),
                 ("w_gate", w_gate, s.N * s.h * l, _BF16), ("w_up", w_up, s.N * s.h * l, _BF16),
                 ("w_down", w_down, s.N * l * s.h, _BF16)):
        _need(*args)
    W = MoeLayerWeights(_ptr(w_route), _ptr(bias), _ptr(w_gate), _ptr(w_up), _ptr(w_down), BF16, a)
    O = _outputs(s, fwd)
    G = MoeLatentGrads(*(_ptr(grads.get(k)) for k in sizes))
    wbuf, wlen = _ws(int(_lib.moe_latent_bwd_workspace_bytes(ctypes.byref(s), ctypes.byref(lw))),
                     x.device, ws)
    _check(_lib.moe_latent_bwd(ctypes.byref(s), ctypes.byref(W), ctypes.byref(lw), _ptr(x),
                               _ptr(dy), ctypes.byref(O), ctypes.byref(G), _ptr(wbuf), wlen,
                               _stream(stream)), "moe_latent_bwd")


_CODES = (_U8, "float8_e4m3fn")


def moe_quantize_e4m3_rows(x, codes, scales, stream=None):
    """Row-wise E4M3 quantisation (include/moe.h): x [rows][cols] bf16 or fp32
    -> codes [rows][cols] (uint8 or float8_e4m3fn), scales [rows] fp32."""
    rows, cols = x.shape[0], x.numel() // max(x.shape[0], 1)
    _need("x", x, rows * cols, (_BF16, _F32))
    _need("codes", codes, rows * cols, _CODES)
    _need("scales", scales, rows, _F32)
    _check(_lib.moe_quantize_e4m3_rows(rows, cols, _ptr(x), _dtype_code(x), _ptr(codes),
                                       _ptr(scales), _stream(stream)), "moe_quantize_e4m3_rows")


def moe_expert_ffn_e4m3_workspace_bytes(s: MoeShape) -> int:
    return int(_lib.moe_expert_ffn_e4m3_workspace_bytes(ctypes.byref(s)))


def moe_expert_ffn_e4m3(s: MoeShape, width: int, x_rows, x_scale, offsets, w_gate, w_up,
                        w_down, gate_scale, up_scale, down_scale, y_rows, a=None, ws=None,
                        stream=None):
    """Grouped expert FFN with E4M3 operands (include/moe.h); y_rows fp32."""
    a = a or act()
    R = s.T * s.k
    for args in (("x_rows", x_rows, R * width, _CODES), ("x_scale", x_scale, R, _F32),
                 ("offsets", offsets, s.N + 1, _I32),
                 ("w_gate", w_gate, s.N * s.h * width, _CODES),
                 ("w_up", w_up, s.N * s.h * width, _CODES),
                 ("w_down", w_down, s.N * width * s.h, _CODES),
                 ("gate_scale", gate_scale, s.N * s.h, _F32), ("up_scale", up_scale, s.N * s.h, _F32),
                 ("down_scale", down_scale, s.N * width, _F32), ("y_rows", y_rows, R * width, _F32)):
        _need(*args)
    sc = MoeE4M3Scales(_ptr(gate_scale), _ptr(up_scale), _ptr(down_scale))
    wbuf, wlen = _ws(int(_lib.moe_expert_ffn_e4m3_workspace_bytes(ctypes.byref(s))),
                     x_rows.device, ws)
    _check(_lib.moe_expert_ffn_e4m3(ctypes.byref(s), width, _ptr(x_rows), _ptr(x_scale),
                                    _ptr(offsets), _ptr(w_gate), _ptr(w_up), _ptr(w_down),
                                    ctypes.byref(sc), ctypes.byref(a), _ptr(y_rows), _ptr(wbuf),
                                    wlen, _stream(stream)), "moe_expert_ffn_e4m3")


def moe_latent_fwd_e4m3(s: MoeShape, w_route, w_gate, w_up, w_down, gate_scale, up_scale,
                        down_scale, lw: MoeLatentWeights, x, y, bias=None, a=None,
                        outputs: dict | None = None, ws=None, stream=None):
    """The LatentMoE layer with E4M3 routed experts (codes + fp32 row scales)."""
    a = a or act()
    l = lw.latent
    for args in (("x", x, s.T * s.d, _BF16), ("y", y, s.T * s.d, _BF16),
                 ("w_route", w_route, s.N * s.d, _F32), ("bias", bias, s.N, _F32),
                 ("w_gate", w_gate, s.N * s.h * l, _CODES), ("w_up", w_up, s.N * s.h * l, _CODES),
                 ("w_down", w_down, s.N * l * s.h, _CODES),
                 ("gate_scale", gate_scale, s.N * s.h, _F32),
                 ("up_scale", up_scale, s.N * s.h, _F32),
                 ("down_scale", down_scale, s.N * l, _F32)):
        _need(*args)
    O = _outputs(s, outputs)
    W = MoeLayerWeights(_ptr(w_route), _ptr(bias), _ptr(w_gate), _ptr(w_up), _ptr(w_down), E4M3,
                        a)
    sc = MoeE4M3Scales(_ptr(gate_scale), _ptr(up_scale), _ptr(down_scale))
    wbuf, wlen = _ws(moe_latent_workspace_bytes(s, lw), x.device, ws)
    _check(_lib.moe_latent_fwd_e4m3(ctypes.byref(s), ctypes.byref(W), ctypes.byref(sc),
                                    ctypes.byref(lw), _ptr(x), _ptr(y), ctypes.byref(O),
                                    _ptr(wbuf), wlen, _stream(stream)), "moe_latent_fwd_e4m3")


def q4_layer(w_route, gate_qs, gate_scales, up_qs, up_scales, down_qs, down_scales,
             bias=None) -> MoeQ4Layer:
    """One q4_0 layer's device pointers (sizes follow the shape of the call
    that uses it, so only the element types are checked here)."""
    for args in (("w_route", w_route, 0, _F32), ("bias", bias, 0, _F32),
                 ("gate_qs", gate_qs, 0, _U8), ("up_qs", up_qs, 0, _U8),
                 ("down_qs", down_qs, 0, _U8), ("gate_scales", gate_scales, 0, _Q4_SCALES),
                 ("up_scales", up_scales, 0, _Q4_SCALES),
                 ("down_scales", down_scales, 0, _Q4_SCALES)):
        _need(*args)
    return MoeQ4Layer(_ptr(w_route), _ptr(bias), _ptr(gate_qs), _ptr(gate_scales), _ptr(up_qs),
                      _ptr(up_scales), _ptr(down_qs), _ptr(down_scales))


DECODE_PER_TOKEN, DECODE_TWO_PHASE = 1, 2  # moe_decode_kernel's answers (0: unsupported)


def moe_decode_kernel(s: MoeShape) -> int:
    return int(_lib.moe_decode_kernel(ctypes.byref(s)))


def moe_decode_workspace_bytes(s: MoeShape) -> int:
    return int(_lib.moe_decode_workspace_bytes(ctypes.byref(s)))


def moe_decode_layer(s: MoeShape, layer: MoeQ4Layer, u, y, u_next=None, top_idx=None,
                     top_w=None, ws=None, stream=None):
    """u, y, u_next: fp16 tensors [T][d]."""
    for args in (("u", u, s.T * s.d, _F16), ("y", y, s.T * s.d, _F16),
                 ("u_next", u_next, s.T * s.d, _F16), ("top_idx", top_idx, s.T * s.k, _I32),
                 ("top_w", top_w, s.T * s.k, _F32)):
        _need(*args)
    wbuf, wlen = _ws(moe_decode_workspace_bytes(s), u.device, ws)
    _check(_lib.moe_decode_layer(ctypes.byref(s), ctypes.byref(layer), _ptr(u), _ptr(y),
                                 _ptr(u_next), _ptr(top_idx), _ptr(top_w), _ptr(wbuf), wlen,
                                 _stream(stream)), "moe_decode_layer")


def moe_decode_step(s: MoeShape, layers, u0, u_out, top_idx_all=None, ws=None, stream=None):
    """`layers`: a sequence of MoeQ4Layer (host structs of device pointers)."""
    for args in (("u0", u0, s.T * s.d, _F16), ("u_out", u_out, s.T * s.d, _F16),
                 ("top_idx_all", top_idx_all, len(layers) * s.T * s.k, _I32)):
        _need(*args)
    arr = (MoeQ4Layer * len(layers))(*layers)
    wbuf, wlen = _ws(moe_decode_workspace_bytes(s), u0.device, ws)
    _check(_lib.moe_decode_step(ctypes.byref(s), len(layers), arr, _ptr(u0), _ptr(u_out),
                                _ptr(top_idx_all), _ptr(wbuf), wlen, _stream(stream)),
           "moe_decode_step")


DECODE_STAMPS = 13  # phase stamps per layer of moe_decode_step_trace


def moe_decode_step_trace(s: MoeShape, layers, u0, u_out, stamps, top_idx_all=None, ws=None,
                          stream=None):
    """moe_decode_step plus per-layer phase stamps: stamps is an int64 device
    tensor of at least DECODE_STAMPS * len(layers) elements (SM cycles, see
    moe.h)."""
    for args in (("u0", u0, s.T * s.d, _F16), ("u_out", u_out, s.T * s.d, _F16),
                 ("top_idx_all", top_idx_all, len(layers) * s.T * s.k, _I32),
                 ("stamps", stamps, DECODE_STAMPS * len(layers), "int64")):
        _need(*args)
    arr = (MoeQ4Layer * len(layers))(*layers)
    wbuf, wlen = _ws(moe_decode_workspace_bytes(s), u0.device, ws)
    _check(_lib.moe_decode_step_trace(ctypes.byref(s), len(layers), arr, _ptr(u0), _ptr(u_out),
                                      _ptr(top_idx_all), _ptr(wbuf), wlen, _ptr(stamps),
                                      _stream(stream)), "moe_decode_step_trace")


def moe_aux_grad(probs, f, dz, alpha: float = 1.0, stream=None):
    """dL_aux/dz [T][N] (fp32 device tensors) with the loads f held constant."""
    T, N = probs.shape
    _need("probs", probs, T * N, _F32)
    _need("f", f, N, _F32)
    _need("dz", dz, T * N, _F32)
    _check(_lib.moe_aux_grad(T, N, alpha, _ptr(probs), _ptr(f), _ptr(dz), _stream(stream)),
           "moe_aux_grad")


def moe_quantile_balance_workspace_bytes(T: int, N: int) -> int:
    return int(_lib.moe_quantile_balance_workspace_bytes(T, N))


def moe_quantile_balance(scores, k: int, q: int, bias_exact, bias=None, bins: int = 0,
                         cutoff=None, bias_hist=None, loads=None, ws=None, stream=None):
    """scores [T][N] fp32 device tensor; outputs are device tensors (see moe.h)."""
    T, N = scores.shape
    for args in (("scores", scores, T * N, _F32), ("bias_exact", bias_exact, N, _F32),
                 ("bias", bias, N, _F32), ("cutoff", cutoff, T, _F32),
                 ("bias_hist", bias_hist, N, _F32), ("loads", loads, N, _I32)):
        _need(*args)
    wbuf, wlen = _ws(moe_quantile_balance_workspace_bytes(T, N), scores.device, ws)
    _check(_lib.moe_quantile_balance(T, N, k, _ptr(scores), _ptr(bias), q, bins, _ptr(cutoff),
                                     _ptr(bias_exact), _ptr(bias_hist), _ptr(loads), _ptr(wbuf),
                                     wlen, _stream(stream)), "moe_quantile_balance")


def moe_ep_plan(counts_all, capacity: int, rank: int) -> dict:
    """Host-only exchange plan of expert parallelism: counts_all [world][N]
    (every rank's dispatches per expert) -> this rank's plan arrays (numpy
    int32): kept, local_offsets, send_base, send_counts, recv_offsets,
    recv_src_base [E][world], recv_counts, overflow."""
    import numpy as np
    c = np.ascontiguousarray(counts_all, dtype=np.int32)
    if c.ndim != 2:
        raise ValueError("counts_all must be [world][N]")
    world, N = c.shape
    E = N // world if world else 0
    out = dict(kept=np.empty(N, np.int32), local_offsets=np.empty(N + 1, np.int32),
               send_base=np.empty(N, np.int32), send_counts=np.empty(world, np.int32),
               recv_offsets=np.empty(E + 1, np.int32),
               recv_src_base=np.empty((E, world), np.int32),
               recv_counts=np.empty(world, np.int32), overflow=np.empty(N, np.int32))
    order = ("kept", "local_offsets", "send_base", "send_counts", "recv_offsets",
             "recv_src_base", "recv_counts", "overflow")
    _check(_lib.moe_ep_plan(world, rank, N, capacity, c.ctypes.data,
                            *[out[key].ctypes.data for key in order]), "moe_ep_plan")
    return out


def ep_buffers(world: int, rank: int, recv_capacity: int, mine: dict, peers: dict):
    """moe_ep_buffers of `rank`: mine holds this rank's tensors (recv_rows,
    recv_w, out_rows, arrive, done); peers holds, per name, an int64 device
    tensor [world] of every rank's addresses of that buffer as this device
    sees them."""
    return MoeEpBuffers(world, rank, recv_capacity, *(_ptr(mine[n]) for n in (
        "recv_rows", "recv_w", "out_rows", "arrive", "done")), *(_ptr(peers[n]) for n in (
            "recv_rows", "recv_w", "out_rows", "arrive", "done")))


def moe_ep_workspace_bytes(expert_shape: MoeShape) -> int:
    return int(_lib.moe_ep_workspace_bytes(ctypes.byref(expert_shape)))


def moe_ep_dispatch(s: MoeShape, bufs: MoeEpBuffers, epoch: int, u, perm_tok, offsets, row_of,
                    top_w, kept, send_base, ws, stream=None):
    """Stores this rank's kept dispatch rows (and combine weights) into their
    owners' receive buffers and raises its arrival flag on every rank."""
    for args in (("u", u, s.T * s.d, _BF16), ("perm_tok", perm_tok, 0, _I32),
                 ("offsets", offsets, s.N + 1, _I32), ("row_of", row_of, s.T * s.k, _I32),
                 ("top_w", top_w, s.T * s.k, _F32), ("kept", kept, s.N, _I32),
                 ("send_base", send_base, s.N, _I32)):
        _need(*args)
    _check(_lib.moe_ep_dispatch(ctypes.byref(s), ctypes.byref(bufs), epoch, _ptr(u),
                                _ptr(perm_tok), _ptr(offsets), _ptr(row_of), _ptr(top_w),
                                _ptr(kept), _ptr(send_base), _ptr(ws), ws.numel(),
                                _stream(stream)), "moe_ep_dispatch")


def moe_ep_expert_ffn(expert_shape: MoeShape, bufs: MoeEpBuffers, epoch: int, recv_offsets,
                      w_gate, w_up, w_down, ws, a=None, stream=None):
    """Waits for every source, runs this rank's experts on the received rows
    and raises its done flag."""
    s, a = expert_shape, a or act()
    for args in (("recv_offsets", recv_offsets, s.N + 1, _I32),
                 ("w_gate", w_gate, s.N * s.h * s.d, _BF16), ("w_up", w_up, s.N * s.h * s.d, _BF16),
                 ("w_down", w_down, s.N * s.d * s.h, _BF16)):
        _need(*args)
    _check(_lib.moe_ep_expert_ffn(ctypes.byref(s), ctypes.byref(bufs), epoch, _ptr(recv_offsets),
                                  _ptr(w_gate), _ptr(w_up), _ptr(w_down), ctypes.byref(a),
                                  _ptr(ws), ws.numel(), _stream(stream)), "moe_ep_expert_ffn")


def moe_ep_combine(s: MoeShape, bufs: MoeEpBuffers, epoch: int, top_idx, row_of, offsets, kept,
                   send_base, y, stream=None):
    """Waits for every owner, then y_t = sum of its kept slots' output rows."""
    for args in (("top_idx", top_idx, s.T * s.k, _I32), ("row_of", row_of, s.T * s.k, _I32),
                 ("offsets", offsets, s.N + 1, _I32), ("kept", kept, s.N, _I32),
                 ("send_base", send_base, s.N, _I32), ("y", y, s.T * s.d, _BF16)):
        _need(*args)
    _check(_lib.moe_ep_combine(ctypes.byref(s), ctypes.byref(bufs), epoch, _ptr(top_idx),
                               _ptr(row_of), _ptr(offsets), _ptr(kept), _ptr(send_base), _ptr(y),
                               _stream(stream)), "moe_ep_combine")


def moe_device_status(stream=None) -> int:
    out = _i32(0)
    _check(_lib.moe_device_status(_stream(stream), ctypes.byref(out)), "moe_device_status")
    return out.value


def moe_reset_device_status(stream=None):
    _check(_lib.moe_reset_device_status(_stream(stream)), "moe_reset_device_status")


WAIT_GRID_BARRIER, WAIT_MBARRIER = 0, 1


def moe_wait_check(kind: int, budget_ns: int, stream=None):
    """Runs one bounded device wait on a condition nothing satisfies (see
    include/moe.h): the wait records MOE_ERR_TIMEOUT and the kernel returns."""
    _check(_lib.moe_wait_check(kind, budget_ns, _stream(stream)), "moe_wait_check")


def status_string(code: int) -> str:
    return _lib.moe_status_string(code).decode()
