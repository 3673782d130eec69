"""Pins of the CPU oracle to what the pages and the mathematics fix.

Every oracle function is checked here against something other than itself:
values printed on the pages (tests/golden/), closed forms, brute force on
tiny inputs, or an independent library routine (numpy / torch CPU).  The
checks are chosen so that a dropped term, a wrong sign or index, or a
transposed operand in the oracle fails at least one of them.
"""
import math
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle as O

RNG = np.random.default_rng(12345)


# ------------------------------------------------------------------ formats
def test_f16_decode_exhaustive():
    """All 65536 fp16 codes against numpy's float16; subnormals are m * 2^-24."""
    codes = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = codes.view(np.float16).astype(np.float64)
    got = O.decode(O.F16, codes)
    finite = np.isfinite(ref)
    assert np.array_equal(got[finite], ref[finite])
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    assert O.f16_to_f64(0x0001) == 2.0 ** -24
    assert O.f16_to_f64(0x03FF) == 1023 * 2.0 ** -24
    assert O.f16_to_f64(0x0400) == 2.0 ** -14  # smallest normal
    assert O.f16_to_f64(0x8200) == -512 * 2.0 ** -24


def test_bf16_decode_exhaustive():
    codes = np.arange(65536, dtype=np.uint32)
    with np.errstate(invalid="ignore"):
        ref = (codes << 16).view(np.float32).astype(np.float64)
    got = O.decode(O.BF16, codes.astype(np.uint16))
    finite = np.isfinite(ref)
    assert np.array_equal(got[finite], ref[finite])


def test_round_bf16_matches_torch():
    x = np.concatenate([RNG.standard_normal(20000) * 10.0 ** RNG.integers(-6, 6, 20000),
                        [0.0, -0.0, 1.0, 1.00390625, 1.005859375, 3.0e38]])
    ref = torch.tensor(x.astype(np.float32)).to(torch.bfloat16).to(torch.float64).numpy()
    got = np.array([O.round_bf16(v) for v in x])
    assert np.array_equal(got, ref)


def test_q4_decode_layout_and_scales():
    """q4_0: w = (q - 8) * s; byte j holds element j (low) and j+16 (high)."""
    qs = np.zeros((1, 16), np.uint8)
    for j in range(16):
        qs[0, j] = (j & 0xF) | (((15 - j) & 0xF) << 4)
    for code, s in ((0x3C00, 1.0), (0x0001, 2.0 ** -24), (0xC000, -2.0), (0x0000, 0.0)):
        m = O.Mat(O.Q4_0, 1, 32, qs=qs, scales=np.array([[code]], np.uint16))
        w = m.decode()[0]
        exp = [(j - 8) * s for j in range(16)] + [((15 - j) - 8) * s for j in range(16)]
        assert w.tolist() == exp


# --------------------------------------------------------------- router dot
def _exact_dot(w, u):
    return float(sum(Fraction(float(a)) * Fraction(float(b)) for a, b in zip(w, u)))


def test_router_logit_within_fp32_bound():
    """Summation error bound of any order of d fp32 terms: |z - exact| <= d u sum|w u|
    (u = 2^-24); the blocked order of 128-element chains meets the tighter
    (128 + d / 128) u sum|w u|."""
    for d in (8, 64, 512, 4096):
        w = RNG.standard_normal(d).astype(np.float32)
        u = RNG.standard_normal(d).astype(np.float32)
        z = O.router_logit(w, u)
        exact = _exact_dot(w, u)
        mass = float(np.sum(np.abs(w.astype(np.float64) * u)))
        assert abs(z - exact) <= (d + 1) * 2.0 ** -24 * mass
        assert abs(z - exact) <= (min(d, 128) + (d + 127) // 128 + 1) * 2.0 ** -24 * mass


def test_router_logit_integer_inputs_exact():
    w = RNG.integers(-8, 8, 512).astype(np.float32)
    u = RNG.integers(-8, 8, 512).astype(np.float32)
    assert O.router_logit(w, u) == float(np.dot(w.astype(np.int64), u.astype(np.int64)))


def test_router_logit_documented_order():
    """Hand-worked values that only the documented blocked order produces
    (blocks of 128 elements, each an ascending chain from +0, block sums added
    in ascending order).

    Within one block the order is the ascending chain: [2^25, -2^25, 1] gives
    (2^25 - 2^25) + 1 = 1; descending would give (1 - 2^25) -> -2^25 (ulp 4),
    then + 2^25 = 0.
    Across blocks (d = 256, block 0 = positions 0..127, block 1 = 128..255):
    - 2^25 at 0, -2^25 at 128, 1 at 129: P_0 = 2^25, P_1 = -2^25 + 1 -> -2^25,
      z = 0; one ascending chain over all 256 would give 1;
    - 1 at 0, 2^25 at 128, -2^25 at 129: P_0 = 1, P_1 = 0, z = 1; one chain
      would give (1 + 2^25 -> 2^25) - 2^25 = 0;
    - 2^25 at 0, 1 at 8, -2^25 at 128: P_0 = 2^25 + 1 -> 2^25, z = 0; a
      pairwise tree over 8-element chunks would cancel the big terms first
      and give 1.
    """
    w = np.ones(3, np.float32)
    assert O.router_logit(w, np.array([2.0 ** 25, -(2.0 ** 25), 1.0], np.float32)) == 1.0
    assert O.router_logit(w, np.array([1.0, -(2.0 ** 25), 2.0 ** 25], np.float32)) == 1.0 - 1.0
    d = 256
    w = np.ones(d, np.float32)
    for pos, want in (({0: 2.0 ** 25, 128: -(2.0 ** 25), 129: 1.0}, 0.0),
                      ({0: 1.0, 128: 2.0 ** 25, 129: -(2.0 ** 25)}, 1.0),
                      ({0: 2.0 ** 25, 8: 1.0, 128: -(2.0 ** 25)}, 0.0)):
        u = np.zeros(d, np.float32)
        for j, v in pos.items():
            u[j] = v
        assert O.router_logit(w, u) == want
    # a shorter last block: d = 200 = 128 + 72
    u = np.zeros(200, np.float32)
    u[127], u[128], u[199] = 1.0, 2.0 ** 25, -(2.0 ** 25)
    assert O.router_logit(np.ones(200, np.float32), u) == 1.0


def test_router_logit_uses_fused_multiply_add():
    """(1+2^-12)^2 - 1 = 2^-11 + 2^-24 exactly with a fused multiply-add;
    a separately rounded product would give 2^-11."""
    w = np.zeros(8, np.float32)
    u = np.zeros(8, np.float32)
    w[0], u[0] = 1.0, -1.0
    w[1] = u[1] = np.float32(1.0 + 2.0 ** -12)
    assert O.router_logit(w, u) == 2.0 ** -11 + 2.0 ** -24


# ------------------------------------------------------------------ routing
def test_softmax_topk_renorm_against_numpy():
    T, N, k = 64, 8, 2
    logits = RNG.standard_normal((T, N)).astype(np.float32)
    probs, idx, w = O.route_from_logits(logits, k)
    z = logits.astype(np.float64)
    ref_p = np.exp(z - z.max(1, keepdims=True))
    ref_p /= ref_p.sum(1, keepdims=True)
    assert np.allclose(probs, ref_p, rtol=1e-14, atol=0)
    ref_idx = np.argsort(-logits, axis=1, kind="stable")[:, :k]
    assert np.array_equal(idx, ref_idx)
    sel = np.take_along_axis(ref_p, ref_idx, 1)
    assert np.allclose(w, sel / sel.sum(1, keepdims=True), rtol=1e-14)
    assert np.allclose(w.sum(1), 1.0, rtol=0, atol=1e-15)  # §3.6 second relation


def test_topk_ties_go_to_lower_index():
    logits = np.array([[1.0, 3.0, 3.0, 0.0], [5.0, 5.0, 5.0, 5.0], [0.0, 0.0, 1.0, 1.0]],
                      np.float32)
    _, idx, _ = O.route_from_logits(logits, 2)
    assert idx.tolist() == [[1, 2], [0, 1], [2, 3]]


def test_top1_renorm_weight_is_one_and_switch_keeps_p():
    """§3.2 caveat: renormalising one probability gives 1; Switch keeps p."""
    logits = RNG.standard_normal((16, 4)).astype(np.float32)
    probs, idx, w = O.route_from_logits(logits, 1, renorm=1)
    assert idx.shape == (16, 1) and np.all(w == 1.0)
    probs0, idx0, w0 = O.route_from_logits(logits, 1, renorm=0)
    assert np.array_equal(w0[:, 0], probs0[np.arange(16), idx0[:, 0]])


def test_route_logits_are_router_logit_plus_bias():
    T, d, N = 8, 64, 4
    u = RNG.standard_normal((T, d)).astype(np.float32)
    W = RNG.standard_normal((N, d)).astype(np.float32)
    b = np.array([0.0, -0.5, 1.25, -2.0], np.float32)
    logits, probs, idx, w = O.route(u, W, 2, 1, b)
    for t in range(T):
        for i in range(N):
            assert logits[t, i] == np.float32(O.router_logit(W[i], u[t])) + b[i]
            assert abs(logits[t, i] - (_exact_dot(W[i], u[t]) + float(b[i]))) < 1e-4


def test_lab_shapes_and_conservation(golden):
    """§04 / §3.6 / §09 ex. 1: idx shapes and sum L_i = kT."""
    for rec in golden("tutorial_lab_shapes.txt"):
        T, d, N, k = (int(rec[x]) for x in ("T", "d", "N", "k"))
        u = RNG.standard_normal((T, 8)).astype(np.float32)
        W = RNG.standard_normal((N, 8)).astype(np.float32)
        _, probs, idx, w = O.route(u, W, k)
        assert idx.shape == tuple(int(x) for x in rec["top_idx_shape"].split(","))
        _, _, _, loads = O.aux_stats(probs, idx)
        assert loads.sum() == int(rec["dispatches"]) == k * T
        if "example_loads" in rec:
            assert sum(int(x) for x in rec["example_loads"].split(",")) == k * T


# -------------------------------------------------------------- aux stats
def _controlled_logits(case, T=16, N=4):
    z = np.zeros((T, N), np.float32)
    if case == "balanced":
        z[np.arange(T), np.arange(T) % N] = 2.0
    else:
        z[:, 0] = 2.0
    return z


def test_aux_stats_printed_values(golden):
    for rec in golden("tutorial_aux_stats.txt"):
        probs, idx, _ = O.route_from_logits(_controlled_logits(rec["case"]), 1)
        f, P, nsum, loads = O.aux_stats(probs, idx)
        assert np.allclose(f, [float(x) for x in rec["f"].split(",")], atol=0)
        assert [round(v, 4) for v in P] == [float(x) for x in rec["P"].split(",")]
        assert f"{nsum:.4f}" == rec["N_sum_fP"]


def test_aux_stats_closed_form():
    """Collapsed case: P_0 = e^2/(e^2+3), the others 1/(e^2+3); N sum fP = 4 P_0."""
    probs, idx, _ = O.route_from_logits(_controlled_logits("collapsed"), 1)
    f, P, nsum, _ = O.aux_stats(probs, idx)
    e2 = math.exp(2.0)
    assert abs(P[0] - e2 / (e2 + 3)) < 1e-15 and abs(P[1] - 1 / (e2 + 3)) < 1e-15
    assert abs(nsum - 4 * e2 / (e2 + 3)) < 1e-14
    # f counts slot 0 (the argmax) only, not every top-k slot
    logits = np.array([[3, 2, 0, 0], [0, 3, 2, 0]], np.float32)
    probs, idx, _ = O.route_from_logits(logits, 2)
    f, P, nsum, loads = O.aux_stats(probs, idx)
    assert f.tolist() == [0.5, 0.5, 0.0, 0.0] and loads.tolist() == [1, 2, 1, 0]


# -------------------------------------------------------- capacity, permute
def _assign(case, T=16, N=4):
    if case == "uneven":
        return np.array([0] * 10 + [1] * 3 + [2] * 2 + [3], np.int32)
    return (np.arange(T) % N).astype(np.int32)


def test_capacity_overflow_printed_values(golden):
    for rec in golden("tutorial_capacity.txt"):
        a = _assign(rec["case"])
        C = O.capacity(16, 4, 1, float(rec["factor"]))
        assert C == int(rec["capacity"])
        out = O.permute(a[:, None], 4, C)
        assert out["counts"].tolist() == [int(x) for x in rec["loads"].split(",")]
        assert int(out["totals"][1]) == int(rec["dropped"])
        assert int(out["totals"][2]) == int(rec["empty"])
        assert int(out["totals"][0]) + int(out["totals"][1]) == 16


def test_capacity_topk_counts_dispatches():
    """§3.5: for top-k the capacity counts k*T dispatches (1.25 * 2 * 8192 / 8)."""
    assert O.capacity(8192, 8, 2, 1.25) == 2560
    assert O.capacity(16, 4, 2, 1.0) == 8


def _permute_brute(idx, N, C):
    """Independent restatement: walk experts, list their tokens in order."""
    T, k = idx.shape
    rows, row_of = [], -np.ones((T, k), np.int64)
    for e in range(N):
        hits = [(t, s) for t in range(T) for s in range(k) if idx[t, s] == e]
        keep = hits if C == 0 else hits[:C]
        for (t, s) in keep:
            row_of[t, s] = len(rows)
            rows.append(t)
    return np.array(rows, np.int64), row_of


@pytest.mark.parametrize("T,N,k,C", [(37, 5, 2, 0), (64, 8, 2, 9), (50, 6, 3, 20), (12, 4, 1, 2),
                                     (1, 3, 3, 0), (40, 8, 2, 1)])
def test_permute_brute_force(T, N, k, C):
    z = RNG.standard_normal((T, N)).astype(np.float32)
    idx = np.argsort(-z, axis=1, kind="stable")[:, :k].astype(np.int32)
    out = O.permute(idx, N, C)
    rows, row_of = _permute_brute(idx, N, C)
    assert np.array_equal(out["perm_tok"], rows)
    assert np.array_equal(out["row_of"], row_of)
    L = np.bincount(idx.ravel(), minlength=N)
    assert np.array_equal(out["counts"], L)
    kept = np.minimum(L, C) if C else L
    assert np.array_equal(out["offsets"], np.concatenate([[0], np.cumsum(kept)]))
    assert np.array_equal(out["overflow"], np.maximum(L - C, 0) if C else 0 * L)
    assert int(out["totals"][0]) == kept.sum()
    assert int(out["totals"][2]) == (np.maximum(C - L, 0).sum() if C else 0)


def test_permute_brute_force_random_shapes():
    """The same comparison over random shapes, capacities and expert sets
    (distinct experts per token, any order), including empty experts."""
    from hypothesis import given, settings, strategies as st

    @settings(max_examples=150, deadline=None)
    @given(st.integers(1, 60), st.integers(1, 10), st.data())
    def check(T, N, data):
        k = data.draw(st.integers(1, N))
        C = data.draw(st.integers(0, 2 * T))
        seed = data.draw(st.integers(0, 2**31 - 1))
        rng = np.random.default_rng(seed)
        idx = np.stack([rng.permutation(N)[:k] for _ in range(T)]).astype(np.int32)
        out = O.permute(idx, N, C)
        rows, row_of = _permute_brute(idx, N, C)
        assert np.array_equal(out["perm_tok"], rows)
        assert np.array_equal(out["row_of"], row_of)

    check()


# ---------------------------------------------------------------- experts
def _rand_mat(rows, cols, scale=0.3):
    return O.Mat(O.F32, rows, cols, data=(RNG.standard_normal((rows, cols)) * scale)
                 .astype(np.float32))


def _silu(x):
    return x / (1.0 + np.exp(-x))


def test_expert_matches_numpy_swiglu():
    """N=1, k=1: the layer is one dense SwiGLU, W_down (SiLU(W_g u) * W_u u)."""
    d, h = 24, 40
    Wg, Wu, Wd = _rand_mat(h, d), _rand_mat(h, d), _rand_mat(d, h)
    u = RNG.standard_normal(d)
    G, U = Wg.decode() @ u, Wu.decode() @ u
    ref = Wd.decode() @ (_silu(G) * U)
    assert np.allclose(O.expert(Wg, Wu, Wd, u), ref, rtol=1e-12, atol=1e-14)
    # matvec orientation: W is [rows][cols], y = W x (not W^T x)
    assert np.allclose(O.matvec(Wg, u), G, rtol=1e-13, atol=1e-15)
    # the whole layer with N = 1, k = 1 reduces to the same SwiGLU
    y = O.moe_tokens([Wg], [Wu], [Wd], u[None, :], np.zeros((1, 1), np.int32), np.ones((1, 1)))
    assert np.allclose(y[0], ref, rtol=1e-12, atol=1e-14)


def test_expert_zero_down_gives_zero():
    d, h = 16, 8
    Wd = O.Mat(O.F32, d, h, data=np.zeros((d, h), np.float32))
    y = O.expert(_rand_mat(h, d), _rand_mat(h, d), Wd, RNG.standard_normal(d))
    assert np.all(y == 0.0)


def test_situ_glu_soft_caps():
    """SiTU-GLU: huge beta reduces to SwiGLU; the hidden product stays within beta_g*beta_u."""
    d, h = 16, 32
    Wg, Wu = _rand_mat(h, d, 30.0), _rand_mat(h, d, 30.0)
    eye = O.Mat(O.F32, h, h, data=np.eye(h, dtype=np.float32))
    u = RNG.standard_normal(d)
    # identity "down" exposes the hidden vector: [h][h]
    hid = O.expert(Wg, Wu, eye, u, act=1, beta_g=4.0, beta_u=25.0)
    assert np.max(np.abs(hid)) <= 100.0
    G, U = Wg.decode() @ u, Wu.decode() @ u
    assert np.allclose(hid, _silu(4 * np.tanh(G / 4)) * 25 * np.tanh(U / 25), rtol=1e-12)
    Wg2, Wu2 = _rand_mat(h, d), _rand_mat(h, d)
    big = O.expert(Wg2, Wu2, eye, u, act=1, beta_g=1e7, beta_u=1e7)
    plain = O.expert(Wg2, Wu2, eye, u, act=0)
    assert np.allclose(big, plain, rtol=1e-9, atol=1e-12)


def test_situ_glu_gate_and_up_caps_are_not_interchangeable():
    """LatentMoE document, SiTU-GLU: the caps multiply to beta_g * beta_u, given
    as 4 x 25 = 100 (gate cap first, up cap second).  With one hidden unit and
    an identity down projection the hidden value is exposed:
      gate saturated (g -> +inf): H = SiLU(4) * 25 tanh(v / 25);
      up saturated   (v -> +inf): H = SiLU(4 tanh(g / 4)) * 25;
      both saturated:             H = SiLU(4) * 25 = 98.2..., below 100,
    where exchanged caps would give SiLU(25) * 4 = 99.99...  The workload
    constants carry the same assignment."""
    from synthetic import workloads as W
    one = O.Mat(O.F32, 1, 1, data=np.ones((1, 1), np.float32))

    def hidden(g, v):
        Wg = O.Mat(O.F32, 1, 1, data=np.array([[g]], np.float32))
        Wu = O.Mat(O.F32, 1, 1, data=np.array([[v]], np.float32))
        return float(O.expert(Wg, Wu, one, np.ones(1), act=1, beta_g=4.0, beta_u=25.0)[0])

    silu4 = 4.0 / (1.0 + math.exp(-4.0))
    assert math.isclose(hidden(1e4, 5.0), silu4 * 25.0 * math.tanh(5.0 / 25.0), rel_tol=1e-14)
    g = 3.0
    gc = 4.0 * math.tanh(g / 4.0)
    assert math.isclose(hidden(g, 1e4), gc / (1.0 + math.exp(-gc)) * 25.0, rel_tol=1e-14)
    both = hidden(1e4, 1e4)
    assert math.isclose(both, silu4 * 25.0, rel_tol=1e-14) and both < 100.0
    assert abs(both - 25.0 / (1.0 + math.exp(-25.0)) * 4.0) > 1.5
    wl = W.latent()
    assert (wl.beta_gate, wl.beta_up) == (4.0, 25.0)


def test_round_h_rounds_hidden_to_bf16():
    d, h = 16, 32
    Wg, Wu = _rand_mat(h, d), _rand_mat(h, d)
    eye = O.Mat(O.F32, h, h, data=np.eye(h, dtype=np.float32))
    u = RNG.standard_normal(d)
    hid = O.expert(Wg, Wu, eye, u, round_h=1)
    exact = O.expert(Wg, Wu, eye, u, round_h=0)
    ref = torch.tensor(exact.astype(np.float32)).to(torch.bfloat16).double().numpy()
    assert np.array_equal(hid, ref)


def test_sparse_equals_dense_brute_force():
    """Appendix lab: the dense all-experts reference equals the sparse path (max error 0)."""
    T, d, h, N, k = 16, 12, 20, 4, 2
    Wg = [_rand_mat(h, d) for _ in range(N)]
    Wu = [_rand_mat(h, d) for _ in range(N)]
    Wd = [_rand_mat(d, h) for _ in range(N)]
    u = RNG.standard_normal((T, d))
    W_route = RNG.standard_normal((N, d)).astype(np.float32)
    _, probs, idx, w = O.route(u.astype(np.float32), W_route, k)
    ys = O.moe_tokens(Wg, Wu, Wd, u, idx, w)
    yd = O.moe_dense(Wg, Wu, Wd, u, idx, w)
    assert np.max(np.abs(ys - yd)) == 0.0
    # hand restatement with numpy per token
    for t in range(T):
        ref = sum(w[t, s] * (Wd[e].decode() @ (_silu(Wg[e].decode() @ u[t]) * (Wu[e].decode()
                                                                              @ u[t])))
                  for s, e in enumerate(idx[t]))
        assert np.allclose(ys[t], ref, rtol=1e-12, atol=1e-14)


def test_dropped_dispatch_contributes_nothing():
    T, d, h, N, k = 6, 8, 8, 2, 1
    Wg = [_rand_mat(h, d) for _ in range(N)]
    Wu = [_rand_mat(h, d) for _ in range(N)]
    Wd = [_rand_mat(d, h) for _ in range(N)]
    u = RNG.standard_normal((T, d))
    idx = np.zeros((T, 1), np.int32)  # every token to expert 0, capacity 4
    out = O.permute(idx, N, 4)
    y = O.moe_tokens(Wg, Wu, Wd, u, idx, np.ones((T, 1)), row_of=out["row_of"])
    assert np.all(y[4:] == 0.0) and np.all(np.abs(y[:4]).sum(1) > 0)


def test_combine_of_expert_rows_equals_sparse_layer():
    """Grouping rows by expert, running experts per row and combining by row_of
    gives the token-wise sparse layer (§3.6: split into [L_i, d], add back)."""
    T, d, h, N, k, C = 20, 8, 12, 4, 2, 7
    Wg = [_rand_mat(h, d) for _ in range(N)]
    Wu = [_rand_mat(h, d) for _ in range(N)]
    Wd = [_rand_mat(d, h) for _ in range(N)]
    u = RNG.standard_normal((T, d))
    W_route = RNG.standard_normal((N, d)).astype(np.float32)
    _, _, idx, w = O.route(u.astype(np.float32), W_route, k)
    out = O.permute(idx, N, C)
    rows = np.zeros((len(out["perm_tok"]), d))
    for e in range(N):
        for r in range(out["offsets"][e], out["offsets"][e + 1]):
            rows[r] = O.expert(Wg[e], Wu[e], Wd[e], u[out["perm_tok"][r]])
    y = O.combine(rows, out["row_of"], w)
    ref = O.moe_tokens(Wg, Wu, Wd, u, idx, w, row_of=out["row_of"])
    assert np.allclose(y, ref, rtol=1e-13, atol=1e-15)
    # a dropped slot adds nothing; an all-dropped token is exactly zero
    assert np.all(O.combine(rows, -np.ones((T, k), np.int32), w) == 0.0)


def test_q4_expert_equals_dequantised_f64():
    """Per-GEMV emulation with the same quantised weights (deployment notes §6)."""
    d, h = 64, 32
    qs = RNG.integers(0, 256, (h, d // 2)).astype(np.uint8)
    sc = np.array(RNG.choice([0x2000, 0x1C00, 0x0003, 0x83FF, 0x0000], (h, d // 32)), np.uint16)
    m = O.Mat(O.Q4_0, h, d, qs=qs, scales=sc)
    dense = np.zeros((h, d))
    for r in range(h):
        for c in range(d):
            b, j = divmod(c, 32)
            byte = int(qs[r, b * 16 + (j % 16)])
            q = byte & 15 if j < 16 else byte >> 4
            dense[r, c] = (q - 8) * float(np.array([sc[r, b]], np.uint16).view(np.float16)[0])
    x = RNG.standard_normal(d)
    assert np.allclose(O.matvec(m, x), dense @ x, rtol=1e-13, atol=1e-16)


def test_rmsnorm_closed_form_and_scale_invariance():
    x = RNG.standard_normal(3584)
    y = O.rmsnorm(x)
    assert abs(np.sqrt(np.mean(y * y)) - 1.0) < 1e-6
    assert np.allclose(O.rmsnorm(x * 37.0, eps=0.0), O.rmsnorm(x, eps=0.0), rtol=1e-12)
    assert np.allclose(O.rmsnorm(x * 37.0), y, rtol=1e-6)  # eps = 1e-6 only shifts the scale
    c = np.full(10, 0.5)
    assert np.allclose(O.rmsnorm(c, eps=0.0), np.ones(10), rtol=1e-15)


# ---------------------------------------------------------------- ledgers
def test_parameter_ledger_printed_values(golden):
    for rec in golden("tutorial_ledger.txt"):
        led = O.ledger(int(rec["d"]), int(rec["h"]), int(rec["N"]), int(rec["k"]))
        assert led["one"] == int(rec["one"])
        assert led["all"] == int(rec["all"])
        assert led["active"] == int(rec["active"])
        assert f"{led['bf16_gib']:.3f}" == f"{float(rec['bf16_gib']):.3f}"
        assert led["all"] / led["active"] == float(rec["all_over_active"])


def test_bandwidth_gain_printed_values(golden):
    for rec in golden("mcu_bandwidth_gain.txt"):
        g = O.bandwidth_gain(int(rec["ffn"]), int(rec["top_k"]), int(rec["ffn_e"]))
        assert f"{g:.2f}" == rec["gain"]


def test_round_f16_matches_numpy():
    x = np.concatenate([RNG.standard_normal(5000) * 10.0 ** RNG.integers(-8, 4, 5000),
                        [0.0, 65504.0, 6.0e-8, 2.0 ** -25, 3 * 2.0 ** -26, 1.0 + 2.0 ** -11]])
    ref = x.astype(np.float16).view(np.uint16)
    assert np.array_equal(O.round_f16(x), ref)


def test_decode_layer_q4_matches_dequantised_dense():
    """A q4_0 layer equals the same layer with the dequantised weights in
    float64 (the per-GEMV emulation of the deployment notes, §6)."""
    T, d, h, N, k = 5, 64, 32, 4, 2
    mats, dense = [], []
    for e in range(N):
        trip = []
        for rows, cols in ((h, d), (h, d), (d, h)):
            qs = RNG.integers(0, 256, (rows, cols // 2)).astype(np.uint8)
            sc = np.array(RNG.choice([0x2000, 0x1C00, 0x0005, 0x9C00], (rows, cols // 32)),
                          np.uint16)
            trip.append(O.Mat(O.Q4_0, rows, cols, qs=qs, scales=sc))
        mats.append(tuple(trip))
        dense.append(tuple(O.Mat(O.F32, m.rows, m.cols, data=m.decode().astype(np.float32))
                           for m in trip))
    u = RNG.standard_normal((T, d)).astype(np.float16).view(np.uint16)
    w_route = (RNG.standard_normal((N, d)) * 0.1).astype(np.float32)
    idx, tw, y, un = O.decode_layer(u, w_route, mats, k)
    # the q4 values are exactly representable in fp32, so the dense copy is exact
    y2 = O.moe_tokens([m[0] for m in dense], [m[1] for m in dense], [m[2] for m in dense],
                      O.decode(O.F16, u), idx, tw)
    assert np.array_equal(y, y2)
    assert np.array_equal(un, (O.decode(O.F16, u) + y).astype(np.float16).view(np.uint16))


def _latent_case(N=6, d=64, l=32, h=48, sh=40, n_sh=2, T=5, scale_down=1.0):
    rng = np.random.default_rng(77)

    def bf(rows, cols, sig=0.2):
        v = (rng.standard_normal((rows, cols)) * sig).astype(np.float32)
        return O.Mat(O.BF16, rows, cols, data=v.view(np.uint32) >> 16)

    experts = [(bf(h, l), bf(h, l), bf(l, h)) for _ in range(N)]
    if scale_down != 1.0:  # exact power-of-two rescale of every routed down matrix
        experts = [(g, u, O.Mat(O.F32, l, h, data=(dn.decode() * scale_down).astype(np.float32)))
                   for g, u, dn in experts]
    shared = [(bf(sh, d), bf(sh, d), bf(d, sh)) for _ in range(n_sh)]
    W_dp, W_upp = bf(l, d), bf(d, l)
    w_route = rng.standard_normal((N, d)).astype(np.float32)
    x = (rng.standard_normal((T, d)).astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    return x, w_route, W_dp, experts, W_upp, shared


def test_latent_rmsnorm_removes_scale_of_routed_branch():
    """LatentMoE document: RMSNorm before the up-projection makes the output
    insensitive to the routed branch's scale.  An exact x8 on every routed
    down matrix leaves y bit-identical when eps = 0."""
    x, wr, W_dp, ex, W_upp, sh = _latent_case()
    _, _, y1 = O.latent_tokens(x, wr, 2, W_dp, lambda e: ex[e], W_upp, sh, 4.0, 25.0, 0.0)
    x, wr, W_dp, ex8, W_upp, sh = _latent_case(scale_down=8.0)
    _, _, y8 = O.latent_tokens(x, wr, 2, W_dp, lambda e: ex8[e], W_upp, sh, 4.0, 25.0, 0.0)
    assert np.array_equal(y1, y8)


def test_latent_routed_experts_live_in_the_bottleneck():
    """Routed experts see only x_l = W_dp x: with W_dp = 0 the routed branch is
    zero and y is exactly the shared experts' output; routing (on x) is unchanged."""
    x, wr, W_dp, ex, W_upp, sh = _latent_case()
    zero = O.Mat(O.F32, W_dp.rows, W_dp.cols, data=np.zeros((W_dp.rows, W_dp.cols), np.float32))
    idx0, _, y0 = O.latent_tokens(x, wr, 2, zero, lambda e: ex[e], W_upp, sh, 4.0, 25.0, 1e-6)
    idx1, _, _ = O.latent_tokens(x, wr, 2, W_dp, lambda e: ex[e], W_upp, sh, 4.0, 25.0, 1e-6)
    assert np.array_equal(idx0, idx1)
    xd = O.decode(O.BF16, x)
    ref = np.array([sum(O.expert(g, u, d, xd[t], round_h=1) for g, u, d in sh)
                    for t in range(x.shape[0])])
    assert np.array_equal(y0, ref)


def test_latent_single_expert_closed_form():
    """N = 1, k = 1, no shared experts: y = W_upp bf16(rms(F(bf16(W_dp x))))
    restated with numpy and torch's bf16 rounding."""
    x, wr, W_dp, ex, W_upp, sh = _latent_case(N=1, n_sh=0, T=3)
    _, tw, y = O.latent_tokens(x, wr[:1], 1, W_dp, lambda e: ex[e], W_upp, [], 4.0, 25.0, 1e-6)
    assert np.all(tw == 1.0)

    def bf16(v):
        return torch.tensor(v.astype(np.float32)).to(torch.bfloat16).double().numpy()

    g, u, d = (m.decode() for m in ex[0])
    for t, xt in enumerate(O.decode(O.BF16, x)):
        xl = bf16(W_dp.decode() @ xt)
        G, U = 4 * np.tanh(g @ xl / 4), 25 * np.tanh(u @ xl / 25)
        m = d @ bf16(_silu(G) * U)
        mh = bf16(m / np.sqrt(np.mean(m * m) + 1e-6))
        assert np.allclose(y[t], W_upp.decode() @ mh, rtol=1e-11, atol=1e-12)


def test_latent_expert_major_order_is_bit_identical():
    """The expert-major loop nest (each routed expert fetched once, used by the
    full-size GPU parity test) returns exactly the per-token forward."""
    x, wr, W_dp, ex, W_upp, sh = _latent_case(N=9, T=11)
    fetched = []

    def get(e):
        fetched.append(e)
        return ex[e]

    i1, w1, y1 = O.latent_tokens(x, wr, 3, W_dp, lambda e: ex[e], W_upp, sh, 4.0, 25.0, 1e-6)
    i2, w2, y2 = O.latent_tokens_expert_major(x, wr, 3, W_dp, get, W_upp, sh, 4.0, 25.0, 1e-6,
                                              threads=4)
    assert np.array_equal(i1, i2) and np.array_equal(w1, w2) and np.array_equal(y1, y2)
    assert fetched == sorted(set(i1.ravel().tolist()))  # every routed expert once, in order


# ------------------------------------------------------- quantile balancing
# Stable LatentMoE demo document, Quantile Balancing: with every token's top-k
# cutoff a_i fixed, the bias that gives expert j exactly q tokens is the q-th
# smallest required_ij = a_i - s_ij.
def test_qb_hand_example():
    # k = 1: a_i = max_j s_ij = [3, 2, 5, 1.5].
    # expert 0: required = a - s_0 = [0, 2, 0, 0.5] -> sorted [0, 0, 0.5, 2]
    # expert 1: required = a - s_1 = [2, 0, 1, 0]   -> sorted [0, 0, 1, 2]
    s = np.array([[3, 1], [0, 2], [5, 4], [1, 1.5]], np.float32)
    a = O.qb_cutoffs(s, 1)
    assert a.tolist() == [3.0, 2.0, 5.0, 1.5]
    b, loads = O.qb_exact(s, a, 2)
    assert b.tolist() == [0.0, 0.0] and loads.tolist() == [2, 2]
    b, loads = O.qb_exact(s, a, 3)
    assert b.tolist() == [0.5, 1.0] and loads.tolist() == [3, 3]
    # 4 bins over [0, 2] (width 0.5): expert 0 counts [2, 1, 0, 1] reach 3 in
    # bin 1 -> edge 1.0; expert 1 counts [2, 0, 1, 1] reach 3 in bin 2 -> 1.5
    assert O.qb_hist(s, a, 3, 4).tolist() == [1.0, 1.5]


def test_qb_matches_numpy_sort_and_balances():
    rng = np.random.default_rng(11)
    T, N, k, q = 300, 13, 3, 47
    s = rng.standard_normal((T, N)).astype(np.float32)
    bias = (0.1 * rng.standard_normal(N)).astype(np.float32)
    a = O.qb_cutoffs(s, k, bias)
    sel = (s + bias[None, :]).astype(np.float32)  # one fp32 add per score
    assert np.array_equal(a, np.sort(sel, axis=1)[:, N - k])
    req = (a[:, None] - s).astype(np.float32)
    b, loads = O.qb_exact(s, a, q)
    ref = np.sort(req, axis=0)[q - 1]
    assert np.array_equal(b, ref + np.float32(0.0))
    # the q-th order statistic: fewer than q tokens lie strictly below it and
    # at least q clear it (more only through ties, e.g. required = 0 for the
    # tokens whose k-th expert is j itself)
    assert np.all((req < b[None, :]).sum(0) <= q - 1)
    assert np.all(loads >= q)
    assert np.array_equal(loads, (req <= b[None, :]).sum(0))
    ties = (req == b[None, :]).sum(0)
    assert np.all(loads - ties <= q - 1)


def test_qb_histogram_estimate_brackets_the_exact_quantile():
    rng = np.random.default_rng(5)
    T, N, k, q, B = 1000, 7, 2, 250, 64
    s = rng.standard_normal((T, N)).astype(np.float32)
    a = O.qb_cutoffs(s, k)
    exact, _ = O.qb_exact(s, a, q)
    est = O.qb_hist(s, a, q, B)
    req = (a[:, None] - s).astype(np.float32)
    w = (req.max(0) - req.min(0)) / B
    slack = 4 * np.spacing(np.abs(req).max(0))
    assert np.all(est >= exact - slack)
    assert np.all(est - exact <= w + slack)


# ------------------------------------------------------- aux-loss gradient
def _aux_loss(z, f, alpha):
    """alpha N sum_i f_i P_i with P the batch mean of softmax(z) (tutorial §3.4)."""
    e = np.exp(z - z.max(1, keepdims=True))
    p = e / e.sum(1, keepdims=True)
    return alpha * z.shape[1] * float((f * p.mean(0)).sum())


def test_aux_grad_matches_central_differences():
    """Tutorial §3.7 closed form vs a numerical derivative of §3.4's L_aux with
    the loads f held constant."""
    rng = np.random.default_rng(8)
    T, N, alpha = 6, 5, 0.01
    z = rng.standard_normal((T, N))
    f = rng.dirichlet(np.ones(N))
    e = np.exp(z - z.max(1, keepdims=True))
    p = e / e.sum(1, keepdims=True)
    dz = O.aux_grad(p, f, alpha)
    h = 1e-6
    num = np.empty_like(z)
    for t in range(T):
        for j in range(N):
            zp, zm = z.copy(), z.copy()
            zp[t, j] += h
            zm[t, j] -= h
            num[t, j] = (_aux_loss(zp, f, alpha) - _aux_loss(zm, f, alpha)) / (2 * h)
    assert np.allclose(dz, num, rtol=1e-6, atol=1e-11)


def test_aux_grad_invariants():
    rng = np.random.default_rng(9)
    T, N = 50, 8
    p = rng.dirichlet(np.ones(N), size=T)
    f = rng.dirichlet(np.ones(N))
    dz = O.aux_grad(p, f, 1.0)
    assert np.allclose(dz.sum(1), 0.0, atol=1e-15)  # softmax gradients sum to zero per token
    # perfectly balanced loads push no logit
    assert np.allclose(O.aux_grad(p, np.full(N, 1.0 / N), 1.0), 0.0, atol=1e-16)
    # the over-loaded expert of a token with p = f is pushed down (positive gradient)
    f2 = np.array([0.7, 0.1, 0.1, 0.1])
    g = O.aux_grad(np.array([[0.25, 0.25, 0.25, 0.25]]), f2, 1.0)
    assert g[0, 0] > 0 and np.all(g[0, 1:] < 0)
