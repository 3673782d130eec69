"""The allocation-free permutation entry point, moe_permute_noalloc.

It serves callers that cannot allocate device memory when they call in (a C
program that loads only this library and has no device allocator, or a
framework whose memory planner forbids allocation at call time): the scratch
comes from a fixed array inside the library.  Checked here through the C ABI
against moe_permute, which takes a caller workspace, on two calls in a row
(the shared array keeps the first call's contents when the second starts).
This file is collected last so a run that stops at the first failure has
already run every other test.
"""
import ctypes

import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import sparse_mixture_experts_15_b200 as moe


def _buffers(T, N, k):
    i32 = dict(dtype=torch.int32, device="cuda")
    return dict(counts=torch.empty(N, **i32), offsets=torch.empty(N + 1, **i32),
                perm_tok=torch.full((T * k,), -1, **i32), row_of=torch.empty((T, k), **i32),
                overflow=torch.empty(N, **i32), totals=torch.empty(3, **i32))


def _call(fn, s, idx, b, *ws):
    args = [ctypes.byref(s), idx.data_ptr(), b["counts"].data_ptr(), b["offsets"].data_ptr(),
            b["perm_tok"].data_ptr(), b["row_of"].data_ptr(), b["overflow"].data_ptr(),
            b["totals"].data_ptr(), *ws, torch.cuda.current_stream().cuda_stream]
    return fn(*args)


@pytest.mark.parametrize("cases", [[(4096, 8, 2, 0), (8192, 8, 2, 2560)],
                                   [(4096, 896, 16, 0), (777, 64, 6, 40)]])
def test_noalloc_permute_matches_workspace_permute(cases):
    lib = moe._lib
    for T, N, k, C in cases:  # two calls in a row on the shared scratch
        rng = np.random.default_rng(T + N)
        z = rng.standard_normal((T, N)) + np.linspace(1.5, 0.0, N)[None, :]
        idx = torch.from_numpy(np.argsort(-z, axis=1)[:, :k].astype(np.int32)).cuda()
        s = moe.shape(T, 64, N, k, 64, 1, C)
        ref, got = _buffers(T, N, k), _buffers(T, N, k)
        nb = lib.moe_permute_workspace_bytes(ctypes.byref(s))
        ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
        assert _call(lib.moe_permute, s, idx, ref, ws.data_ptr(), nb) == 0
        assert _call(lib.moe_permute_noalloc, s, idx, got) == 0
        torch.cuda.synchronize()
        rows = int(ref["offsets"][N].item())
        for key in ("counts", "offsets", "row_of", "overflow", "totals"):
            assert torch.equal(got[key], ref[key]), key
        assert torch.equal(got["perm_tok"][:rows], ref["perm_tok"][:rows])
    assert moe.moe_device_status() == 0


def test_noalloc_permute_rejects_oversize():
    lib = moe._lib
    T, N, k = 65536, 1024, 32  # needs 8192 x 1024 ints of scratch, over the 262144 limit
    s = moe.shape(T, 64, N, k, 64, 1, 0)
    one = torch.zeros(16, dtype=torch.int32, device="cuda")
    p = one.data_ptr()
    rc = lib.moe_permute_noalloc(ctypes.byref(s), p, p, p, p, p, p, p,
                                 torch.cuda.current_stream().cuda_stream)
    assert rc == -6 and moe.status_string(rc).startswith("MOE_ERR_WORKSPACE")


def _one_case_on(stream, T=3000, N=64, k=4, C=0):
    """Both entry points on `stream` (a torch stream of the current device)."""
    lib = moe._lib
    rng = np.random.default_rng(11)
    z = rng.standard_normal((T, N)) + np.linspace(1.0, 0.0, N)[None, :]
    with torch.cuda.stream(stream):
        idx = torch.from_numpy(np.argsort(-z, axis=1)[:, :k].astype(np.int32)).cuda()
        s = moe.shape(T, 64, N, k, 64, 1, C)
        ref, got = _buffers(T, N, k), _buffers(T, N, k)
        nb = lib.moe_permute_workspace_bytes(ctypes.byref(s))
        ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
        assert _call(lib.moe_permute, s, idx, ref, ws.data_ptr(), nb) == 0
        assert _call(lib.moe_permute_noalloc, s, idx, got) == 0
    stream.synchronize()
    rows = int(ref["offsets"][N].item())
    for key in ("counts", "offsets", "row_of", "overflow", "totals"):
        assert torch.equal(got[key], ref[key]), key
    assert torch.equal(got["perm_tok"][:rows], ref["perm_tok"][:rows])


def test_noalloc_permute_on_a_side_stream():
    """The entry point runs on whatever stream the caller passes."""
    _one_case_on(torch.cuda.Stream(), C=30)
    assert moe.moe_device_status() == 0


@pytest.mark.skipif(not torch.cuda.is_available() or torch.cuda.device_count() < 2,
                    reason="needs a second visible GPU")
def test_noalloc_permute_on_a_second_device():
    """The fixed array exists once per device; its address is looked up per
    device, so a call on device 1 uses device 1's copy."""
    with torch.cuda.device(1):
        _one_case_on(torch.cuda.current_stream(), C=30)
        assert moe.moe_device_status() == 0
