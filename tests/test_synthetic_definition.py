"""The seeded input generator computes what its definition says (CPU only).

The generator is input preparation shared by the oracle and the GPU path (the
GPU tests check that host and device agree bit for bit).  Here its host side
is checked against a Python restatement of the definition: Vigna's splitmix64
(validated against the reference outputs published with it), the key of
(seed, tensor id), Irwin-Hall sums of twelve 16-bit fields, one fp32 multiply
by sigma, and round-to-nearest-even to bf16 (torch) or fp16 (numpy).
"""
import numpy as np
import torch

import synthetic as S

M64 = (1 << 64) - 1
GAMMA = 0x9E3779B97F4A7C15


def splitmix64(x):
    z = (x + GAMMA) & M64
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & M64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & M64
    return z ^ (z >> 31)


def test_splitmix64_reference_outputs():
    """The first outputs of splitmix64 from state 1234567, as published with
    the algorithm's reference implementation."""
    state, out = 1234567, []
    for _ in range(5):
        out.append(splitmix64(state))
        state = (state + GAMMA) & M64
    assert out == [6457827717110365317, 3203168211198807973, 9817491932198370423,
                   4593380528125082431, 16408922859458223821]


def _normals(seed, tid, n, sigma, offset=0):
    key = splitmix64(((seed * GAMMA) & M64) ^ splitmix64(tid))
    out = np.empty(n, np.float32)
    for i in range(n):
        s = 0
        for j in range(3):
            h = splitmix64((key + 3 * (offset + i) + j) & M64)
            s += (h & 0xFFFF) + ((h >> 16) & 0xFFFF) + ((h >> 32) & 0xFFFF) + (h >> 48)
        x = np.float32((s - 393210) / 65536.0)  # exact: |s - 393210| < 2^19
        out[i] = x * np.float32(sigma)           # one fp32 multiply
    return out


def test_host_generator_matches_its_definition():
    for seed, tid, sigma, offset in ((1001, 5, 0.02, 0), (7, 1, 1.0, 12345), (1004, 13, 0.7, 99)):
        ref = _normals(seed, tid, 300, sigma, offset)
        f32 = S.normal(seed, tid, (300,), sigma, S.DT_F32, offset=offset)
        assert np.array_equal(f32.view(np.uint32), ref.view(np.uint32))
        bf = S.normal(seed, tid, (300,), sigma, S.DT_BF16, offset=offset)
        ref_bf = torch.from_numpy(ref).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
        assert np.array_equal(bf, ref_bf)
        f16 = S.normal(seed, tid, (300,), sigma, S.DT_F16, offset=offset)
        assert np.array_equal(f16, ref.astype(np.float16).view(np.uint16))


def test_irwin_hall_moments():
    """Twelve uniforms minus 6 have mean 0 and variance 1 (the Irwin-Hall
    construction of an approximate standard normal)."""
    x = S.normal(3, 9, (200000,), 1.0, S.DT_F32).astype(np.float64)
    assert abs(x.mean()) < 0.01 and abs(x.var() - 1.0) < 0.01
    assert np.abs(x).max() <= 6.0


def test_q4_scale_classes():
    """q4_0 test scales: 1/64 zero, 7/64 subnormal (the fp16 subnormal-decode
    case of the deployment notes), the rest normal in [2^-9, 2^-7), both signs."""
    _, scales = S.q4(1002, 3, 4096, 512)
    c = scales.ravel()
    ex, man = (c >> 10) & 0x1F, c & 0x3FF
    zero = (c & 0x7FFF) == 0
    sub = (ex == 0) & (man != 0)
    normal = (ex == 6) | (ex == 7)
    assert np.all(zero | sub | normal)
    assert abs(zero.mean() - 1 / 64) < 0.005 and abs(sub.mean() - 7 / 64) < 0.01
    assert 0.45 < ((c >> 15) == 1)[normal].mean() < 0.55
