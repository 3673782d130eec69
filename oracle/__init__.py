"""CPU oracle for the sparse-MoE SwiGLU layer forward and its backward (ctypes over moe_oracle.c).

TEST INFRASTRUCTURE ONLY: imported by tests/, by the smoke check and by the
CPU-baseline leg of bench.py.  The GPU product path never imports it.

Every numerical function lives in moe_oracle.c; this module only marshals
numpy arrays.  See the C file for the citations of each step.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
SO = os.path.join(_HERE, "_moe_oracle.so")
SRC = os.path.join(_HERE, "moe_oracle.c")

F32, BF16, F16, Q4_0, F64, E4M3 = 0, 1, 2, 3, 4, 5


def build(force: bool = False) -> str:
    if force or not os.path.exists(SO) or os.path.getmtime(SRC) > os.path.getmtime(SO):
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-ffp-contract=off", "-fPIC",
                               "-shared", SRC, "-o", SO + ".tmp", "-lm"])
        os.replace(SO + ".tmp", SO)
    return SO


class OrMat(ctypes.Structure):
    _fields_ = [("dtype", ctypes.c_int), ("rows", ctypes.c_int64), ("cols", ctypes.c_int64),
                ("data", ctypes.c_void_p), ("qs", ctypes.c_void_p), ("scales", ctypes.c_void_p),
                ("row_scale", ctypes.c_void_p)]


_lib = None


def lib():
    global _lib
    if _lib is None:
        L = ctypes.CDLL(build())
        i64, vp, dbl = ctypes.c_int64, ctypes.c_void_p, ctypes.c_double
        L.or_bf16_to_f64.argtypes = [ctypes.c_uint16]
        L.or_bf16_to_f64.restype = dbl
        L.or_f16_to_f64.argtypes = [ctypes.c_uint16]
        L.or_f16_to_f64.restype = dbl
        L.or_round_bf16.argtypes = [dbl]
        L.or_round_bf16.restype = dbl
        L.or_round_bf16_n.argtypes = [i64, vp, vp]
        L.or_round_bf16_n.restype = None
        L.or_round_f16.argtypes = [dbl]
        L.or_round_f16.restype = ctypes.c_uint16
        L.or_mat_decode.argtypes = [ctypes.POINTER(OrMat), vp]
        L.or_router_logit.argtypes = [vp, vp, i64]
        L.or_router_logit.restype = ctypes.c_float
        L.or_route.argtypes = [i64, i64, i64, i64, ctypes.c_int, vp, vp, vp, vp, vp, vp, vp]
        L.or_route_from_logits.argtypes = [i64, i64, i64, ctypes.c_int, vp, vp, vp, vp]
        L.or_aux_stats.argtypes = [i64, i64, i64, vp, vp, vp, vp, vp, vp]
        L.or_capacity.argtypes = [i64, i64, i64, dbl]
        L.or_capacity.restype = i64
        L.or_permute.argtypes = [i64, i64, i64, i64, vp, vp, vp, vp, vp, vp, vp]
        L.or_matvec.argtypes = [ctypes.POINTER(OrMat), vp, vp]
        L.or_expert.argtypes = [ctypes.POINTER(OrMat)] * 3 + [vp, ctypes.c_int, dbl, dbl,
                                                              ctypes.c_int, vp]
        L.or_moe_tokens.argtypes = [i64, vp, vp, vp, vp, i64, vp, vp, vp, ctypes.c_int, dbl, dbl,
                                    ctypes.c_int, vp, i64, vp]
        L.or_moe_dense.argtypes = [i64, i64, i64, vp, vp, vp, vp, i64, vp, vp, ctypes.c_int, dbl,
                                   dbl, ctypes.c_int, vp]
        L.or_rmsnorm.argtypes = [i64, vp, dbl, vp]
        L.or_combine.argtypes = [i64, i64, i64, vp, vp, vp, vp]
        L.or_ledger.argtypes = [i64, i64, i64, i64, vp, vp, vp, vp]
        L.or_bandwidth_gain.argtypes = [i64, i64, i64]
        L.or_bandwidth_gain.restype = dbl
        L.or_qb_cutoffs.argtypes = [i64, i64, i64, vp, vp, vp]
        L.or_qb_exact.argtypes = [i64, i64, vp, vp, i64, vp, vp]
        L.or_qb_hist.argtypes = [i64, i64, vp, vp, i64, i64, vp]
        L.or_aux_grad.argtypes = [i64, i64, dbl, vp, vp, vp]
        L.or_threads.argtypes = []
        L.or_threads.restype = ctypes.c_int
        L.or_set_threads.argtypes = [ctypes.c_int]
        L.or_set_threads.restype = None
        L.or_e4m3_to_f64.argtypes = [ctypes.c_uint8]
        L.or_e4m3_to_f64.restype = dbl
        L.or_round_e4m3.argtypes = [dbl]
        L.or_round_e4m3.restype = ctypes.c_uint8
        L.or_quant_e4m3_rows.argtypes = [i64, i64, vp, vp, vp]
        L.or_quant_e4m3_rows.restype = None
        L.or_latent_loss.argtypes = [i64, i64, i64, ctypes.c_int, vp, vp, vp, dbl, dbl, vp, vp,
                                     vp, i64, vp, vp, vp, dbl, vp, i64, vp, vp, vp]
        L.or_latent_loss.restype = dbl
        L.or_latent_backward.argtypes = [i64, i64, i64, ctypes.c_int, vp, vp, vp, dbl, dbl, vp,
                                         vp, vp, i64, vp, vp, vp, dbl, vp, i64, vp, vp] + [vp] * 11
        L.or_latent_backward.restype = None
        L.or_layer_loss.argtypes = [i64, i64, i64, ctypes.c_int, vp, vp, vp, ctypes.c_int, dbl,
                                    dbl, vp, vp, vp, i64, vp, vp, vp, dbl, vp, vp]
        L.or_layer_loss.restype = dbl
        L.or_layer_backward.argtypes = [i64, i64, i64, ctypes.c_int, vp, vp, vp, ctypes.c_int,
                                        dbl, dbl, vp, vp, vp, i64, vp, vp, vp, dbl, vp, vp, vp,
                                        vp, vp, vp, vp]
        L.or_layer_backward.restype = None
        for f in (L.or_mat_decode, L.or_route, L.or_route_from_logits, L.or_aux_stats,
                  L.or_permute, L.or_matvec, L.or_expert, L.or_moe_tokens, L.or_moe_dense,
                  L.or_rmsnorm, L.or_ledger, L.or_combine, L.or_qb_cutoffs, L.or_qb_exact,
                  L.or_qb_hist, L.or_aux_grad):
            f.restype = None
        _lib = L
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data


def _c(a, dt):
    return np.ascontiguousarray(a, dtype=dt)


# ------------------------------------------------------------------ matrices
class Mat:
    """A [rows][cols] matrix in f32 / bf16 / f16 / q4_0 storage (keeps arrays alive)."""

    def __init__(self, dtype, rows, cols, data=None, qs=None, scales=None):
        self.dtype, self.rows, self.cols = dtype, rows, cols
        self.row_scale = None
        if dtype == F32:
            self.data = _c(data, np.float32)
        elif dtype == F64:
            self.data = _c(data, np.float64)
        elif dtype in (BF16, F16):
            self.data = _c(data, np.uint16)
        elif dtype == E4M3:  # data: uint8 codes [rows][cols]; scales: fp32 per row
            self.data, self.row_scale = _c(data, np.uint8), _c(scales, np.float32)
        else:
            self.qs, self.scales, self.data = _c(qs, np.uint8), _c(scales, np.uint16), None
        self.s = OrMat(dtype, rows, cols, _p(self.data),
                       _p(getattr(self, "qs", None)) if dtype == Q4_0 else None,
                       _p(getattr(self, "scales", None)) if dtype == Q4_0 else None,
                       _p(self.row_scale))

    def decode(self):
        out = np.empty((self.rows, self.cols), dtype=np.float64)
        lib().or_mat_decode(ctypes.byref(self.s), out.ctypes.data)
        return out


def mat_array(mats):
    arr = (OrMat * len(mats))(*[m.s for m in mats])
    return arr


def f16_to_f64(code: int) -> float:
    return lib().or_f16_to_f64(int(code))


def round_bf16(x: float) -> float:
    return lib().or_round_bf16(float(x))


def round_bf16_array(x) -> np.ndarray:
    x = _c(x, np.float64)
    y = np.empty_like(x)
    lib().or_round_bf16_n(x.size, x.ctypes.data, y.ctypes.data)
    return y


def latent_tokens(x_codes, w_route, k, W_dp, get_expert, W_upp, shared, beta_g, beta_u, eps,
                  renorm=1, bias=None, fp8=False):
    """LatentMoE forward for the given token rows (Stable LatentMoE demo document:
    width separation, RMSNorm before the up-projection, SiTU-GLU soft caps):
      routing on the full-width x; x_l = bf16(W_dp x); m = sum_s a_s E_s(x_l) with
      the soft-capped routed experts (hidden stored as bf16);
      m^ = bf16(m / sqrt(mean m^2 + eps)); y = W_upp m^ + sum_j S_j(x) (plain SwiGLU).
    get_expert(e) returns the (gate, up, down) matrices of routed expert e.
    fp8=True is the FP8 form of the routed experts: their matrices are E4M3
    with a scale per row, x_l is quantised to E4M3 with a scale per token
    (quant_e4m3_rows) and H is rounded to E4M3 with no scale.
    Returns (top_idx, top_w, y in float64)."""
    x = decode(BF16, x_codes)
    _, _, idx, tw = route(x.astype(np.float32), w_route, k, renorm, bias)
    y = np.zeros((x.shape[0], W_upp.rows))
    for t in range(x.shape[0]):
        xl = round_bf16_array(matvec(W_dp, x[t]))
        if fp8:
            xc, xs = quant_e4m3_rows(xl)
            xl = e4m3_mat(xc, xs).decode()[0]
        m = np.zeros(W_dp.rows)
        for s_ in range(k):
            g, u, d = get_expert(int(idx[t, s_]))
            m += tw[t, s_] * expert(g, u, d, xl, act=1, beta_g=beta_g, beta_u=beta_u,
                                    round_h=2 if fp8 else 1)
        mh = round_bf16_array(rmsnorm(m, eps))
        yt = matvec(W_upp, mh)
        for (g, u, d) in shared:
            yt = yt + expert(g, u, d, x[t], act=0, round_h=1)
        y[t] = yt
    return idx, tw, y


def latent_tokens_expert_major(x_codes, w_route, k, W_dp, get_expert, W_upp, shared, beta_g,
                               beta_u, eps, renorm=1, bias=None, threads=8):
    """The same LatentMoE forward as latent_tokens, with the routed experts
    visited in ascending expert order, each fetched once through get_expert(e)
    (so that a sample of tokens covering all 896 experts never holds more than
    a few experts' weights).  Every expert output of a (token, slot) pair is
    the same or_expert call as in latent_tokens, and m sums them in slot order,
    so the result is bit-identical; only the loop nest differs.  Expert
    evaluations run on `threads` Python threads (ctypes releases the GIL)."""
    import concurrent.futures as cf

    x = decode(BF16, x_codes)
    _, _, idx, tw = route(x.astype(np.float32), w_route, k, renorm, bias)
    T = x.shape[0]
    xl = np.stack([round_bf16_array(matvec(W_dp, x[t])) for t in range(T)]) if T else \
        np.zeros((0, W_dp.rows))
    outs = np.zeros((T, k, W_dp.rows))
    pairs = {}
    for t in range(T):
        for s_ in range(k):
            pairs.setdefault(int(idx[t, s_]), []).append((t, s_))

    def run(e, mats):
        g, u, d = mats
        for t, s_ in pairs[e]:
            outs[t, s_] = expert(g, u, d, xl[t], act=1, beta_g=beta_g, beta_u=beta_u, round_h=1)

    with cf.ThreadPoolExecutor(max_workers=threads) as ex:
        futs = []
        for e in sorted(pairs):
            futs.append(ex.submit(run, e, get_expert(e)))
            if len(futs) >= 2 * threads:  # bound the experts held at once
                futs.pop(0).result()
        for f in futs:
            f.result()
    y = np.zeros((T, W_upp.rows))
    for t in range(T):
        m = np.zeros(W_dp.rows)
        for s_ in range(k):
            m += tw[t, s_] * outs[t, s_]
        mh = round_bf16_array(rmsnorm(m, eps))
        yt = matvec(W_upp, mh)
        for (g, u, d) in shared:
            yt = yt + expert(g, u, d, x[t], act=0, round_h=1)
        y[t] = yt
    return idx, tw, y


def e4m3_to_f64(code: int) -> float:
    return lib().or_e4m3_to_f64(int(code))


def round_e4m3(x) -> np.ndarray:
    """Nearest FP8 E4M3 codes (uint8) of float64 values, ties to even, saturating at 448."""
    x = np.asarray(x, np.float64)
    out = np.array([lib().or_round_e4m3(float(v)) for v in x.ravel()], np.uint8)
    return out.reshape(x.shape)


def quant_e4m3_rows(x):
    """(codes uint8 [rows][cols], scales fp32 [rows]): per row s = amax / 448,
    codes = nearest E4M3 of the fp32 quotient x / s."""
    x = _c(np.atleast_2d(x), np.float32)
    rows, cols = x.shape
    codes = np.empty((rows, cols), np.uint8)
    scales = np.empty(rows, np.float32)
    lib().or_quant_e4m3_rows(rows, cols, x.ctypes.data, codes.ctypes.data, scales.ctypes.data)
    return codes, scales


def e4m3_mat(codes, scales):
    """An E4M3 matrix with one fp32 scale per row."""
    codes = np.atleast_2d(codes)
    return Mat(E4M3, codes.shape[0], codes.shape[1], data=codes, scales=scales)


def round_f16(x) -> np.ndarray:
    """Round float64 values to fp16 bit patterns (round to nearest even)."""
    x = np.asarray(x, np.float64)
    out = np.array([lib().or_round_f16(float(v)) for v in x.ravel()], np.uint16)
    return out.reshape(x.shape)


def decode_layer(u_codes, w_route, mats, k, renorm=1, bias=None):
    """One q4_0 decode layer on fp16 activations (deployment notes §2, §4):
    routing, then y_t = sum_s a_s F_{e_s}(u_t) with the hidden vector unrounded;
    returns (top_idx, top_w, y in float64, u_next = fp16(u + y) codes)."""
    u = decode(F16, u_codes)
    _, _, idx, tw = route(u.astype(np.float32), w_route, k, renorm, bias)
    y = moe_tokens([m[0] for m in mats], [m[1] for m in mats], [m[2] for m in mats], u, idx, tw)
    return idx, tw, y, round_f16(u + y)


def decode(dtype, arr):
    """Exact decode of an f32/bf16/f16 array to float64 (the oracle's own decoder)."""
    arr = np.asarray(arr)
    m = Mat(dtype, 1, arr.size, data=arr.reshape(-1))
    return m.decode().reshape(arr.shape)


def as_f32(dtype, arr):
    """Exact conversion of an activation array to fp32 for the router dot products."""
    return decode(dtype, arr).astype(np.float32)


# -------------------------------------------------------------------- router
def router_logit(w, u):
    w, u = _c(w, np.float32), _c(u, np.float32)
    return float(lib().or_router_logit(w.ctypes.data, u.ctypes.data, w.size))


def route(u_f32, w_route, k, renorm=1, bias=None):
    u_f32, w_route = _c(u_f32, np.float32), _c(w_route, np.float32)
    T, d = u_f32.shape
    N = w_route.shape[0]
    bias = None if bias is None else _c(bias, np.float32)
    logits = np.empty((T, N), np.float32)
    probs = np.empty((T, N), np.float64)
    idx = np.empty((T, k), np.int32)
    w = np.empty((T, k), np.float64)
    lib().or_route(T, d, N, k, renorm, u_f32.ctypes.data, w_route.ctypes.data, _p(bias),
                   logits.ctypes.data, probs.ctypes.data, idx.ctypes.data, w.ctypes.data)
    return logits, probs, idx, w


def route_from_logits(logits, k, renorm=1):
    logits = _c(logits, np.float32)
    T, N = logits.shape
    probs = np.empty((T, N), np.float64)
    idx = np.empty((T, k), np.int32)
    w = np.empty((T, k), np.float64)
    lib().or_route_from_logits(T, N, k, renorm, logits.ctypes.data, probs.ctypes.data,
                               idx.ctypes.data, w.ctypes.data)
    return probs, idx, w


def aux_stats(probs, idx):
    probs, idx = _c(probs, np.float64), _c(idx, np.int32)
    T, N = probs.shape
    k = idx.shape[1]
    f = np.empty(N, np.float64)
    P = np.empty(N, np.float64)
    nsum = np.empty(1, np.float64)
    loads = np.empty(N, np.int32)
    lib().or_aux_stats(T, N, k, probs.ctypes.data, idx.ctypes.data, f.ctypes.data, P.ctypes.data,
                       nsum.ctypes.data, loads.ctypes.data)
    return f, P, float(nsum[0]), loads


def capacity(T, N, k, factor):
    return int(lib().or_capacity(T, N, k, float(factor)))


def permute(idx, N, C):
    idx = _c(idx, np.int32)
    T, k = idx.shape
    counts = np.empty(N, np.int32)
    offsets = np.empty(N + 1, np.int32)
    perm_tok = np.full(T * k, -7, np.int32)
    row_of = np.empty((T, k), np.int32)
    overflow = np.empty(N, np.int32)
    totals = np.empty(3, np.int64)
    lib().or_permute(T, N, k, C, idx.ctypes.data, counts.ctypes.data, offsets.ctypes.data,
                     perm_tok.ctypes.data, row_of.ctypes.data, overflow.ctypes.data,
                     totals.ctypes.data)
    return dict(counts=counts, offsets=offsets, perm_tok=perm_tok[: int(offsets[N])],
                row_of=row_of, overflow=overflow, totals=totals)


# -------------------------------------------------------------------- experts
def matvec(W: Mat, x):
    x = _c(x, np.float64)
    y = np.empty(W.rows, np.float64)
    lib().or_matvec(ctypes.byref(W.s), x.ctypes.data, y.ctypes.data)
    return y


def expert(Wg: Mat, Wu: Mat, Wd: Mat, u, act=0, beta_g=0.0, beta_u=0.0, round_h=0):
    u = _c(u, np.float64)
    out = np.empty(Wd.rows, np.float64)
    lib().or_expert(ctypes.byref(Wg.s), ctypes.byref(Wu.s), ctypes.byref(Wd.s), u.ctypes.data,
                    act, beta_g, beta_u, round_h, out.ctypes.data)
    return out


def moe_tokens(Wg, Wu, Wd, u, idx, top_w, row_of=None, tokens=None, act=0, beta_g=0.0,
               beta_u=0.0, round_h=0):
    """y_t = sum_kept a_{t,s} F_{idx}(u_t) for the listed tokens (all by default)."""
    u = _c(u, np.float64)
    idx, top_w = _c(idx, np.int32), _c(top_w, np.float64)
    T, d_in = u.shape
    k = idx.shape[1]
    tokens = np.arange(T, dtype=np.int32) if tokens is None else _c(tokens, np.int32)
    d_out = Wd[0].rows
    y = np.empty((len(tokens), d_out), np.float64)
    g, up, dn = mat_array(Wg), mat_array(Wu), mat_array(Wd)
    row_of = None if row_of is None else _c(row_of, np.int32)
    lib().or_moe_tokens(k, g, up, dn, u.ctypes.data, d_in, idx.ctypes.data, top_w.ctypes.data,
                        _p(row_of), act, beta_g, beta_u, round_h, tokens.ctypes.data, len(tokens),
                        y.ctypes.data)
    return y


def moe_dense(Wg, Wu, Wd, u, idx, top_w, act=0, beta_g=0.0, beta_u=0.0, round_h=0):
    u = _c(u, np.float64)
    idx, top_w = _c(idx, np.int32), _c(top_w, np.float64)
    T, d_in = u.shape
    k = idx.shape[1]
    d_out = Wd[0].rows
    y = np.empty((T, d_out), np.float64)
    lib().or_moe_dense(T, len(Wg), k, mat_array(Wg), mat_array(Wu), mat_array(Wd), u.ctypes.data,
                       d_in, idx.ctypes.data, top_w.ctypes.data, act, beta_g, beta_u, round_h,
                       y.ctypes.data)
    return y


def combine(rows, row_of, top_w):
    """y_t = sum over kept slots of a_{t,s} * rows[row_of[t, s]] (float64)."""
    rows = _c(rows, np.float64)
    row_of, top_w = _c(row_of, np.int32), _c(top_w, np.float64)
    T, k = row_of.shape
    width = rows.shape[1]
    y = np.empty((T, width), np.float64)
    lib().or_combine(T, k, width, rows.ctypes.data, row_of.ctypes.data, top_w.ctypes.data,
                     y.ctypes.data)
    return y


def rmsnorm(x, eps=1e-6):
    x = _c(x, np.float64)
    y = np.empty_like(x)
    lib().or_rmsnorm(x.size, x.ctypes.data, eps, y.ctypes.data)
    return y


# -------------------------------------------------------------------- ledgers
def ledger(d, h, N, k):
    out = [np.zeros(1, np.int64) for _ in range(3)] + [np.zeros(1, np.float64)]
    lib().or_ledger(d, h, N, k, *[o.ctypes.data for o in out])
    return dict(one=int(out[0][0]), all=int(out[1][0]), active=int(out[2][0]),
                bf16_gib=float(out[3][0]))


def bandwidth_gain(ffn, top_k, ffn_e):
    return float(lib().or_bandwidth_gain(ffn, top_k, ffn_e))


# ------------------------------------------------------- quantile balancing
def qb_cutoffs(scores, k, bias=None):
    """a_i: the k-th largest s_ij + b_j of each token (Stable LatentMoE demo
    document, Quantile Balancing), fp32."""
    s = _c(scores, np.float32)
    T, N = s.shape
    b = None if bias is None else _c(bias, np.float32)
    a = np.empty(T, np.float32)
    lib().or_qb_cutoffs(T, N, k, s.ctypes.data, _p(b), a.ctypes.data)
    return a


def qb_exact(scores, cutoffs, q):
    """(b, loads): b_j = the q-th smallest required_ij = a_i - s_ij; loads_j =
    #{i : required_ij <= b_j}."""
    s, a = _c(scores, np.float32), _c(cutoffs, np.float32)
    T, N = s.shape
    b = np.empty(N, np.float32)
    loads = np.empty(N, np.int32)
    lib().or_qb_exact(T, N, s.ctypes.data, a.ctypes.data, q, b.ctypes.data, loads.ctypes.data)
    return b, loads


def qb_hist(scores, cutoffs, q, bins):
    """The histogram estimate of the same quantile (bins equal bins over the
    range of required_j, the upper edge of the bin where the count reaches q)."""
    s, a = _c(scores, np.float32), _c(cutoffs, np.float32)
    T, N = s.shape
    b = np.empty(N, np.float32)
    lib().or_qb_hist(T, N, s.ctypes.data, a.ctypes.data, q, bins, b.ctypes.data)
    return b


def aux_grad(probs, f, alpha=1.0):
    """dL_aux/dz [T][N] with the loads f held constant (tutorial §3.7)."""
    p, f = _c(probs, np.float64), _c(f, np.float64)
    T, N = p.shape
    dz = np.empty((T, N), np.float64)
    lib().or_aux_grad(T, N, alpha, p.ctypes.data, f.ctypes.data, dz.ctypes.data)
    return dz


# ----------------------------------------------------------- layer backward
def _layer_args(Wg, Wu, Wd, u, top_idx, row_of, dy, Wr, z, f):
    u = _c(u, np.float64)
    T, d_in = u.shape
    idx = _c(top_idx, np.int32)
    k = idx.shape[1]
    N = len(Wg)
    d_out = Wd[0].rows
    dy = _c(dy, np.float64).reshape(T, d_out)
    Wr = None if Wr is None else _c(Wr, np.float64)
    z = None if z is None else _c(z, np.float64)
    if Wr is None and z is None:
        raise ValueError("give the router weights or the logits")
    row_of = None if row_of is None else _c(row_of, np.int32)
    f = None if f is None else _c(f, np.float64)
    return u, T, d_in, idx, k, N, d_out, dy, Wr, z, row_of, f


def layer_loss(Wg, Wu, Wd, u, top_idx, dy, Wr=None, z=None, row_of=None, renorm=1, act=0,
               beta_g=0.0, beta_u=0.0, alpha=0.0, f=None):
    """(L, y): L = sum dy . y (+ alpha N sum f_i P_i when f is given) with the
    selected sets top_idx and the dropped dispatches (row_of < 0) held fixed,
    everything in double.  z = u Wr^T when Wr is given, else the given logits."""
    u, T, d_in, idx, k, N, d_out, dy, Wr, z, row_of, f = _layer_args(
        Wg, Wu, Wd, u, top_idx, row_of, dy, Wr, z, f)
    y = np.empty((T, d_out), np.float64)
    L = lib().or_layer_loss(T, N, k, renorm, mat_array(Wg), mat_array(Wu), mat_array(Wd), act,
                            beta_g, beta_u, _p(Wr), _p(z), u.ctypes.data, d_in, idx.ctypes.data,
                            _p(row_of), dy.ctypes.data, alpha, _p(f), y.ctypes.data)
    return float(L), y


def layer_backward(Wg, Wu, Wd, u, top_idx, dy, Wr=None, z=None, row_of=None, renorm=1, act=0,
                   beta_g=0.0, beta_u=0.0, alpha=0.0, f=None):
    """Gradients of layer_loss: dict of dz [T][N], du [T][d_in], dWr [N][d_in]
    (None without Wr), dWg, dWu [N][h][d_in], dWd [N][d_out][h]."""
    u, T, d_in, idx, k, N, d_out, dy, Wr, z, row_of, f = _layer_args(
        Wg, Wu, Wd, u, top_idx, row_of, dy, Wr, z, f)
    h = Wg[0].rows
    out = dict(dz=np.empty((T, N)), du=np.empty((T, d_in)),
               dWr=None if Wr is None else np.empty((N, d_in)),
               dWg=np.empty((N, h, d_in)), dWu=np.empty((N, h, d_in)), dWd=np.empty((N, d_out, h)))
    lib().or_layer_backward(T, N, k, renorm, mat_array(Wg), mat_array(Wu), mat_array(Wd), act,
                            beta_g, beta_u, _p(Wr), _p(z), u.ctypes.data, d_in, idx.ctypes.data,
                            _p(row_of), dy.ctypes.data, alpha, _p(f), out["dz"].ctypes.data,
                            out["du"].ctypes.data, _p(out["dWr"]), out["dWg"].ctypes.data,
                            out["dWu"].ctypes.data, out["dWd"].ctypes.data)
    return out


def _latent_args(routed, Wr, W_dp, W_upp, shared, x, top_idx, dy):
    Wg, Wu, Wd = routed
    x = _c(x, np.float64)
    T, d = x.shape
    idx = _c(top_idx, np.int32)
    sg = [m[0] for m in shared]
    su = [m[1] for m in shared]
    sd = [m[2] for m in shared]
    sh_arrays = (mat_array(sg), mat_array(su), mat_array(sd)) if shared else (None, None, None)
    return (Wg, Wu, Wd, _c(Wr, np.float64), x, T, d, idx, idx.shape[1], len(Wg),
            _c(dy, np.float64).reshape(T, d), sh_arrays)


def latent_loss(routed, Wr, W_dp, W_upp, shared, x, top_idx, dy, beta_g, beta_u, eps=1e-6,
                renorm=1):
    """(L, y) of the LatentMoE layer in double (no intermediate rounding) with
    the selected sets top_idx held fixed; routed = (gates, ups, downs) lists of
    Mats at the latent width, shared = [(gate, up, down)] at full width."""
    Wg, Wu, Wd, Wr, x, T, d, idx, k, N, dy, sh = _latent_args(routed, Wr, W_dp, W_upp, shared,
                                                              x, top_idx, dy)
    y = np.empty((T, d), np.float64)
    L = lib().or_latent_loss(T, N, k, renorm, mat_array(Wg), mat_array(Wu), mat_array(Wd), beta_g,
                             beta_u, Wr.ctypes.data, ctypes.byref(W_dp.s), ctypes.byref(W_upp.s),
                             len(shared), *sh, eps, x.ctypes.data, d, idx.ctypes.data,
                             dy.ctypes.data, y.ctypes.data)
    return float(L), y


def latent_backward(routed, Wr, W_dp, W_upp, shared, x, top_idx, dy, beta_g, beta_u, eps=1e-6,
                    renorm=1):
    """Gradients of latent_loss: dict of dz, dx, dWr, dWdp, dWupp, dWg, dWu,
    dWd, dSg, dSu, dSd (the shared ones None without shared experts)."""
    Wg, Wu, Wd, Wr, x, T, d, idx, k, N, dy, sh = _latent_args(routed, Wr, W_dp, W_upp, shared,
                                                              x, top_idx, dy)
    l, h = W_dp.rows, Wg[0].rows
    n = len(shared)
    s_h = shared[0][0].rows if n else 0
    out = dict(dz=np.empty((T, N)), dx=np.empty((T, d)), dWr=np.empty((N, d)),
               dWdp=np.empty((l, d)), dWupp=np.empty((d, l)), dWg=np.empty((N, h, l)),
               dWu=np.empty((N, h, l)), dWd=np.empty((N, l, h)),
               dSg=np.empty((n, s_h, d)) if n else None, dSu=np.empty((n, s_h, d)) if n else None,
               dSd=np.empty((n, d, s_h)) if n else None)
    lib().or_latent_backward(T, N, k, renorm, mat_array(Wg), mat_array(Wu), mat_array(Wd),
                             beta_g, beta_u, Wr.ctypes.data, ctypes.byref(W_dp.s),
                             ctypes.byref(W_upp.s), n, *sh, eps, x.ctypes.data, d,
                             idx.ctypes.data, dy.ctypes.data,
                             *[_p(out[key]) for key in ("dz", "dx", "dWr", "dWdp", "dWupp", "dWg",
                                                        "dWu", "dWd", "dSg", "dSu", "dSd")])
    return out


def threads() -> int:
    """Threads the oracle's OpenMP loops use."""
    return int(lib().or_threads())


def set_threads(n: int):
    lib().or_set_threads(int(n))
