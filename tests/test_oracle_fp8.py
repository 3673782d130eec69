"""Pins of the oracle's FP8 E4M3 pieces (CPU only).

The Stable LatentMoE demo document bounds the SiTU-GLU product by
beta_g * beta_u = 4 * 25 = 100, under the FP8 E4M3 limit of 448, which is what
lets the routed experts run in E4M3.  The oracle's codec, row quantiser and
E4M3 matrix storage are pinned here against torch's float8_e4m3fn conversions
(a library routine), exhaustively where the domain is small, and the bound
against the closed form of the capped product.
"""
import math

import numpy as np
import pytest
import torch

import oracle


def _torch_decode(codes):
    return torch.from_numpy(np.asarray(codes, np.uint8)).view(torch.float8_e4m3fn).double().numpy()


def _torch_encode(x):
    t = torch.from_numpy(np.asarray(x, np.float64)).to(torch.float8_e4m3fn)
    return t.view(torch.uint8).numpy()


def test_decode_all_codes():
    codes = np.arange(256, dtype=np.uint8)
    ours = np.array([oracle.e4m3_to_f64(c) for c in codes])
    ref = _torch_decode(codes)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan) and nan.sum() == 2  # 0x7F and 0xFF
    assert np.array_equal(ours[~nan], ref[~nan])
    assert np.array_equal(np.signbit(ours[~nan]), np.signbit(ref[~nan]))
    assert ours[0x7E] == 448.0 and ours[0x01] == 2.0 ** -9 and ours[0x08] == 2.0 ** -6


def test_encode_values_midpoints_and_random():
    finite = np.array([oracle.e4m3_to_f64(c) for c in range(0x7F)])
    # every finite value is its own code
    assert np.array_equal(oracle.round_e4m3(finite), np.arange(0x7F, dtype=np.uint8))
    # midpoints go to the even code; a hair above or below goes to the nearer one
    mids = (finite[:-1] + finite[1:]) / 2
    got = oracle.round_e4m3(mids).astype(int)
    lo = np.arange(0x7E)
    assert np.array_equal(got, np.where(lo % 2 == 0, lo, lo + 1))
    assert np.array_equal(oracle.round_e4m3(np.nextafter(mids, 0)).astype(int), lo)
    assert np.array_equal(oracle.round_e4m3(np.nextafter(mids, 1e9)).astype(int), lo + 1)
    assert np.array_equal(oracle.round_e4m3(mids), _torch_encode(mids))
    # random fp32 values over the whole range, both signs, subnormals included
    rng = np.random.default_rng(17)
    mag = 2.0 ** rng.uniform(-12, math.log2(463.9), 20000)
    x = (mag * rng.choice([-1.0, 1.0], mag.size)).astype(np.float32).astype(np.float64)
    assert np.array_equal(oracle.round_e4m3(x), _torch_encode(x))
    # signed zeros and tiny values keep their sign
    assert list(oracle.round_e4m3([0.0, -0.0, 1e-9, -1e-9])) == [0x00, 0x80, 0x00, 0x80]


def test_encode_saturates_above_448():
    """Above 448 the oracle saturates (a 'satfinite' conversion); torch agrees
    up to the tie at 464 and returns NaN beyond it, which the quantiser never
    reaches (its quotients stay within 448 times one fp32 rounding)."""
    x = np.array([448.0, 449.0, 463.9, 464.0, 465.0, 1e6, -1e6, np.inf, -np.inf])
    assert list(oracle.round_e4m3(x)) == [0x7E] * 6 + [0xFE, 0x7E, 0xFE]
    assert oracle.round_e4m3([np.nan])[0] == 0x7F
    assert np.array_equal(oracle.round_e4m3(x[:4]), _torch_encode(x[:4]))


def test_row_quantiser():
    rng = np.random.default_rng(23)
    x = rng.normal(0, 0.02, (64, 96)).astype(np.float32)
    x[5] = 0.0
    x[6, 7] = -3.5  # one large entry sets the row's scale
    codes, scales = oracle.quant_e4m3_rows(x)
    # scale = amax / 448 in fp32; zero rows get scale 1 and zero codes
    amax = np.abs(x).max(1)
    expect = np.where(amax > 0, (amax / np.float32(448.0)).astype(np.float32), np.float32(1.0))
    assert np.array_equal(scales, expect)
    assert not codes[5].any()
    # each row's largest magnitude maps to +-448
    for r in range(64):
        if amax[r] > 0:
            c = codes[r, np.argmax(np.abs(x[r]))]
            assert c in (0x7E, 0xFE)
    # codes are torch's E4M3 rounding of the fp32 quotients
    q = (x / scales[:, None]).astype(np.float32).astype(np.float64)
    assert np.array_equal(codes, _torch_encode(q))
    # the E4M3 matrix decodes to scale * value; error within half a unit in the last place
    deq = oracle.e4m3_mat(codes, scales).decode()
    assert np.array_equal(deq, scales[:, None].astype(np.float64) * _torch_decode(codes))
    v = np.abs(q)
    ulp = np.where(v < 2.0 ** -6, 2.0 ** -9, 2.0 ** (np.floor(np.log2(np.maximum(v, 1e-30))) - 3))
    assert np.all(np.abs(deq - x.astype(np.float64)) <= 0.5 * ulp * scales[:, None] * (1 + 1e-6))


def test_situ_product_stays_under_e4m3_limit():
    """|SiLU(4 tanh(g/4)) * 25 tanh(v/25)| < SiLU(4) * 25 < 100 < 448 for any g, v;
    the oracle's expert with an identity down projection exposes H."""
    h = 64
    g = np.concatenate([np.linspace(-1e4, 1e4, h // 2), np.linspace(-30, 30, h // 2)])
    v = np.concatenate([np.linspace(1e4, -1e4, h // 2), np.linspace(-300, 300, h // 2)])
    mk = lambda a: oracle.Mat(oracle.F64, a.shape[0], a.shape[1], data=a)  # noqa: E731
    Wg, Wu, Wd = mk(g[:, None]), mk(v[:, None]), mk(np.eye(h))
    H = oracle.expert(Wg, Wu, Wd, np.ones(1), act=1, beta_g=4.0, beta_u=25.0)
    bound = 4.0 / (1.0 + math.exp(-4.0)) * 25.0
    assert np.abs(H).max() <= bound and bound < 100.0 < 448.0
    # round_h = 2 is the E4M3 rounding of exactly these H values
    H8 = oracle.expert(Wg, Wu, Wd, np.ones(1), act=1, beta_g=4.0, beta_u=25.0, round_h=2)
    assert np.array_equal(H8, _torch_decode(_torch_encode(H)))


@pytest.mark.parametrize("seed", [1, 2, 3])
def test_fp8_expert_error_matches_the_e4m3_estimate(seed):
    """The E4M3 expert (per-row weight scales, per-token activation scale, H in
    E4M3) against the same expert in double.  E4M3 keeps 4 significant bits:
    a rounded normal value carries a relative error uniform in about +-2^-4 / m
    (m the mantissa in [1, 2)), about 2.6% rms.  A dot product of quantised
    weights and activations then errs by about sqrt(2) * 2.6% = 3.7% of its
    rms, H = SiLU(g') v' by about 5.5% plus its own E4M3 rounding, and the
    down projection adds its weights' 2.6%: about 6.5% of rms(y) in all.  A
    mistake in the scales or in the rounding lands far outside [3%, 10%]."""
    rng = np.random.default_rng(seed)
    d, h = 256, 384
    Wg, Wu = rng.normal(0, 0.05, (h, d)), rng.normal(0, 0.05, (h, d))
    Wd = rng.normal(0, 0.05, (d, h))
    x = rng.normal(0, 1.0, d)
    f64 = lambda a: oracle.Mat(oracle.F64, a.shape[0], a.shape[1], data=a)  # noqa: E731
    q8 = lambda a: oracle.e4m3_mat(*oracle.quant_e4m3_rows(a.astype(np.float32)))  # noqa: E731
    exact = oracle.expert(f64(Wg), f64(Wu), f64(Wd), x, act=1, beta_g=4.0, beta_u=25.0)
    xc, xs = oracle.quant_e4m3_rows(x.astype(np.float32))
    x8 = oracle.e4m3_mat(xc, xs).decode()[0]
    fp8 = oracle.expert(q8(Wg), q8(Wu), q8(Wd), x8, act=1, beta_g=4.0, beta_u=25.0, round_h=2)
    rel = np.sqrt(np.mean((fp8 - exact) ** 2)) / np.sqrt(np.mean(exact ** 2))
    assert 0.03 < rel < 0.10, rel


def test_fp8_latent_layer_routes_the_same_and_stays_within_e4m3_error():
    """The FP8 form of the LatentMoE layer: routing (fp32, on x) is unchanged,
    and the output stays within a few percent of the bf16 layer's rms.  The
    routed branch's E4M3 error (about 6.5% of its rms) is divided by RMSNorm's
    scale and added to the unchanged shared experts."""
    rng = np.random.default_rng(5)
    N, d, l, h, sh, T, k = 6, 64, 32, 48, 40, 6, 2

    def bf(rows, cols, sig=0.2):
        v = (rng.standard_normal((rows, cols)) * sig).astype(np.float32)
        return oracle.Mat(oracle.BF16, rows, cols, data=v.view(np.uint32) >> 16)

    experts = [(bf(h, l), bf(h, l), bf(l, h)) for _ in range(N)]
    q8 = lambda m: oracle.e4m3_mat(*oracle.quant_e4m3_rows(m.decode().astype(np.float32)))  # noqa
    experts8 = [tuple(q8(m) for m in trip) for trip in experts]
    shared = [(bf(sh, d), bf(sh, d), bf(d, sh)) for _ in range(2)]
    W_dp, W_upp = bf(l, d), bf(d, l)
    w_route = rng.standard_normal((N, d)).astype(np.float32)
    x = (rng.standard_normal((T, d)).astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    i16, w16, y16 = oracle.latent_tokens(x, w_route, k, W_dp, lambda e: experts[e], W_upp,
                                         shared, 4.0, 25.0, 1e-6)
    i8, w8, y8 = oracle.latent_tokens(x, w_route, k, W_dp, lambda e: experts8[e], W_upp, shared,
                                      4.0, 25.0, 1e-6, fp8=True)
    assert np.array_equal(i16, i8) and np.array_equal(w16, w8)
    rel = np.sqrt(np.mean((y8 - y16) ** 2)) / np.sqrt(np.mean(y16 ** 2))
    assert 1e-3 < rel < 0.1, rel
