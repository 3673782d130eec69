"""The C-ABI boundary without a GPU: the library loads, exports every entry
point include/*.h declares, the Python binding covers them, and host-side
argument checks reject bad calls before any device work."""
import ctypes
import glob
import os
import re
import subprocess

import pytest

from conftest import ROOT

import sparse_mixture_experts_15_b200 as moe


def _declared():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        txt = open(h).read()
        names |= set(re.findall(r"MOE_API\s+[\w\s\*]*?\b(moe_\w+)\s*\(", txt))
    return sorted(names)


def test_header_declares_entry_points():
    names = _declared()
    for required in ("moe_route", "moe_permute", "moe_expert_ffn", "moe_combine",
                     "moe_layer_fwd", "moe_aux_stats", "moe_gather", "moe_capacity"):
        assert required in names


def test_library_exports_every_declared_symbol():
    out = subprocess.run(["nm", "-D", "--defined-only", moe.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = {ln.split()[-1] for ln in out.splitlines() if " T " in ln}
    missing = [n for n in _declared() if n not in exported]
    assert not missing, missing
    lib = ctypes.CDLL(moe.LIB_PATH)
    for n in _declared():
        assert getattr(lib, n) is not None


def test_binding_covers_every_symbol():
    assert set(_declared()) <= set(moe.EXPORTED)


def test_capacity_host_only():
    """Tutorial §3.5: C = ceil(c * dispatches / N)."""
    assert moe.moe_capacity(16, 4, 1, 1.0) == 4
    assert moe.moe_capacity(16, 4, 1, 1.5) == 6
    assert moe.moe_capacity(16, 4, 1, 2.5) == 10
    assert moe.moe_capacity(8192, 8, 2, 1.25) == 2560
    assert moe.moe_capacity(100, 8, 2, 0.0) == 0
    with pytest.raises(moe.MoeError):
        moe.moe_capacity(-1, 8, 2, 1.0)


def test_status_strings():
    assert moe.status_string(0) == "MOE_OK"
    for code in range(-1, -7, -1):
        assert moe.status_string(code).startswith("MOE_ERR_")


def test_host_rejects_bad_shapes_before_device_work():
    lib = moe._lib
    bad = [moe.shape(16, 63, 4, 2, 128),   # d % 8 != 0
           moe.shape(16, 64, 4, 5, 128),   # k > N
           moe.shape(16, 64, 0, 1, 128),   # N = 0
           moe.shape(16, 64, 2000, 2, 128),  # N > 1024
           moe.shape(16, 64, 64, 33, 128)]   # k > 32
    for s in bad:
        assert lib.moe_route_workspace_bytes(ctypes.byref(s)) == 0
        rc = lib.moe_route(ctypes.byref(s), None, 1, None, None, None, None, None, None, None, 0,
                           None)
        assert rc == -1
        rc = lib.moe_permute(ctypes.byref(s), None, None, None, None, None, None, None, None, 0,
                             None)
        assert rc == -1


def test_host_rejects_null_and_misaligned_pointers():
    lib = moe._lib
    s = moe.shape(16, 64, 4, 2, 128)
    # null outputs
    assert lib.moe_route(ctypes.byref(s), 4096, 0, 8192, None, None, None, None, None, None, 0,
                         None) == -1
    # misaligned activation pointer
    assert lib.moe_route(ctypes.byref(s), 4098, 0, 8192, None, 12288, 16384, None, None, 20480,
                         1 << 20, None) == -1
    # workspace too small
    assert lib.moe_route(ctypes.byref(s), 4096, 0, 8192, None, 12288, 16384, None, None, 20480,
                         16, None) == -6
    # unsupported expert dtype combination (fp32 activations, bf16 weights)
    a = moe.act()
    assert lib.moe_expert_ffn(ctypes.byref(s), 64, 4096, 0, 4096, 4096, 4096, 4096, 1,
                              ctypes.byref(a), 4096, None, 0, None) == -2
    # SiTU-GLU needs positive caps
    a2 = moe.act(moe.ACT_SITU_GLU, 0.0, 25.0)
    assert lib.moe_expert_ffn(ctypes.byref(s), 64, 4096, 1, 4096, 4096, 4096, 4096, 1,
                              ctypes.byref(a2), 4096, None, 0, None) == -1


def test_workspace_queries_are_host_only_and_monotone():
    lib = moe._lib
    small = moe.shape(1024, 512, 8, 2, 128)
    big = moe.shape(8192, 512, 8, 2, 128)
    for q in (lambda s: lib.moe_route_workspace_bytes(ctypes.byref(s)),
              lambda s: lib.moe_permute_workspace_bytes(ctypes.byref(s)),
              lambda s: lib.moe_layer_workspace_bytes(ctypes.byref(s), 1),
              lambda s: lib.moe_expert_ffn_workspace_bytes(ctypes.byref(s), 512, 1)):
        assert 0 < q(small) <= q(big)


def test_quantile_balance_rejects_bad_arguments_on_the_host():
    lib = moe._lib
    p = 4096  # any non-null address: the checks run before any device work
    bad = [(0, 8, 2, 1, 0),        # T = 0
           (100, 0, 1, 1, 0),      # N = 0
           (100, 2000, 2, 1, 0),   # N > 1024
           (100, 8, 9, 1, 0),      # k > N
           (100, 64, 33, 1, 0),    # k > 32
           (100, 8, 2, 0, 0),      # q = 0
           (100, 8, 2, 101, 0),    # q > T
           (100, 8, 2, 10, 5000),  # bins > 4096
           (40000, 8, 2, 10, 0)]   # T > 32768
    for T, N, k, q, bins in bad:
        assert lib.moe_quantile_balance(T, N, k, p, None, q, bins, p, p, None, None, p, 1 << 20,
                                        None) == -1
    # a histogram output needs bins >= 1
    assert lib.moe_quantile_balance(100, 8, 2, 10, None, 10, 0, p, p, p, None, p, 1 << 20,
                                    None) == -1
    # no cutoff output and no workspace
    assert lib.moe_quantile_balance(100, 8, 2, p, None, 10, 0, None, p, None, None, None, 0,
                                    None) == -6
    assert lib.moe_quantile_balance_workspace_bytes(100, 8) >= 400


def test_aux_grad_host_checks():
    lib = moe._lib
    assert lib.moe_aux_grad(-1, 8, 1.0, 4096, 4096, 4096, None) == -1
    assert lib.moe_aux_grad(10, 0, 1.0, 4096, 4096, 4096, None) == -1
    assert lib.moe_aux_grad(10, 8, 1.0, None, 4096, 4096, None) == -1
    assert lib.moe_aux_grad(0, 8, 1.0, None, None, None, None) == 0  # empty batch: no-op


def test_binding_refuses_host_tensors_before_the_call():
    """A host tensor's address handed to a kernel would be read as device
    memory; the binding refuses it before calling into the library."""
    import torch
    s = moe.shape(16, 64, 4, 2, 128)
    u = torch.zeros((16, 64), dtype=torch.bfloat16)
    perm = torch.zeros(32, dtype=torch.int32)
    offsets = torch.zeros(5, dtype=torch.int32)
    x_rows = torch.zeros((32, 64), dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA tensor"):
        moe.moe_gather(s, 64, u, perm, offsets, x_rows)
    with pytest.raises(ValueError, match="CUDA tensor"):
        qs, sc = torch.zeros(8, dtype=torch.uint8), torch.zeros(8, dtype=torch.int16)
        moe.q4_layer(torch.zeros((4, 64)), qs, sc, qs, sc, qs, sc)


def test_binding_refuses_short_tensors_before_the_call():
    """The library sees only addresses; the binding checks each tensor against
    the size the header documents, so a short one never reaches a kernel."""
    import torch
    s = moe.shape(16, 64, 4, 2, 128)
    i32 = dict(dtype=torch.int32)
    with pytest.raises(ValueError, match="x_rows: .* at least 2048"):
        moe.moe_gather(s, 64, torch.zeros((16, 64)), torch.zeros(32, **i32),
                       torch.zeros(5, **i32), torch.zeros((31, 64)))
    with pytest.raises(ValueError, match="offsets"):
        moe.moe_permute(s, torch.zeros((16, 2), **i32), torch.zeros(4, **i32),
                        torch.zeros(4, **i32), torch.zeros(32, **i32), torch.zeros((16, 2), **i32),
                        torch.zeros(4, **i32), torch.zeros(3, **i32))
    with pytest.raises(ValueError, match="w_down"):
        moe.moe_layer_fwd(s, torch.zeros((4, 64)), torch.zeros((4, 128, 64)),
                          torch.zeros((4, 128, 64)), torch.zeros((4, 64, 127)),
                          torch.zeros((16, 64)), torch.zeros((16, 64)))
    with pytest.raises(ValueError, match="row_of"):
        moe.moe_layer_fwd(s, torch.zeros((4, 64)), torch.zeros((4, 128, 64)),
                          torch.zeros((4, 128, 64)), torch.zeros((4, 64, 128)),
                          torch.zeros((16, 64)), torch.zeros((16, 64)),
                          outputs={"row_of": torch.zeros(31, **i32)})
    with pytest.raises(ValueError, match="dz"):
        moe.moe_aux_grad(torch.zeros((16, 4)), torch.zeros(4), torch.zeros(63))


def test_binding_refuses_other_element_types():
    """A narrower element type would let the kernels write past the end."""
    import torch
    s = moe.shape(16, 64, 4, 2, 128)
    with pytest.raises(ValueError, match="top_w: dtype bfloat16"):
        moe.moe_route(s, torch.zeros((16, 64)), torch.zeros((4, 64)),
                      torch.zeros((16, 2), dtype=torch.int32),
                      torch.zeros((16, 2), dtype=torch.bfloat16))
    with pytest.raises(ValueError, match="w_up: dtype float32"):
        bf = dict(dtype=torch.bfloat16)
        moe.moe_layer_fwd(s, torch.zeros((4, 64)), torch.zeros((4, 128, 64), **bf),
                          torch.zeros((4, 128, 64)), torch.zeros((4, 64, 128), **bf),
                          torch.zeros((16, 64), **bf), torch.zeros((16, 64), **bf))
    with pytest.raises(ValueError, match="top_idx: dtype int64"):
        moe.moe_permute(s, torch.zeros((16, 2), dtype=torch.int64),
                        *[torch.zeros(64, dtype=torch.int32)] * 6)


def test_ep_plan_host_checks():
    """moe_ep_plan is host only: bad arguments return MOE_ERR_INVALID_ARG."""
    import numpy as np
    lib = moe._lib
    c = np.array([[3, 0, 2, 1], [1, 4, 0, 2]], np.int32)
    bufs = [np.zeros(64, np.int32) for _ in range(8)]
    ptrs = [b.ctypes.data for b in bufs]
    assert lib.moe_ep_plan(2, 0, 4, 3, c.ctypes.data, *ptrs) == 0
    assert lib.moe_ep_plan(3, 0, 4, 3, c.ctypes.data, *ptrs) == -1   # 4 experts over 3 ranks
    assert lib.moe_ep_plan(2, 2, 4, 3, c.ctypes.data, *ptrs) == -1   # rank out of range
    assert lib.moe_ep_plan(2, 0, 4, -1, c.ctypes.data, *ptrs) == -1  # negative capacity
    assert lib.moe_ep_plan(2, 0, 4, 3, None, *ptrs) == -1
    neg = c.copy()
    neg[1, 2] = -1
    assert lib.moe_ep_plan(2, 0, 4, 3, neg.ctypes.data, *ptrs) == -1
    assert lib.moe_ep_plan(2, 0, 4, 3, c.ctypes.data, *ptrs[:7], None) == 0  # overflow optional


def test_wait_check_rejects_bad_arguments_on_the_host():
    """moe_wait_check refuses an unknown wait kind or a budget out of range
    before touching the device."""
    lib = moe._lib
    assert lib.moe_wait_check(2, 1_000_000, None) == -1
    assert lib.moe_wait_check(-1, 1_000_000, None) == -1
    assert lib.moe_wait_check(0, 999, None) == -1
    assert lib.moe_wait_check(1, 2_000_000_001, None) == -1


def test_new_entry_points_reject_bad_arguments_on_the_host():
    """The FP8, expert-parallel and backward entry points refuse NULL or
    ill-sized arguments before touching the device."""
    lib = moe._lib
    s = moe.shape(64, 256, 8, 2, 256)
    # E4M3 quantiser: columns must be a multiple of 16, pointers non-NULL
    assert lib.moe_quantize_e4m3_rows(4, 24, None, moe.BF16, None, None, None) == -1
    assert lib.moe_quantize_e4m3_rows(4, 32, None, moe.BF16, None, None, None) == -1
    assert lib.moe_quantize_e4m3_rows(4, 32, None, 7, None, None, None) == -2
    assert lib.moe_quantize_e4m3_rows(0, 32, None, moe.BF16, None, None, None) == 0
    # FP8 LatentMoE layer: NULL scales
    assert lib.moe_latent_fwd_e4m3(ctypes.byref(s), None, None, None, None, None, None, None, 0,
                                   None) == -1
    # expert parallelism: NULL buffers
    assert lib.moe_ep_dispatch(ctypes.byref(s), None, 1, *([None] * 7), None, 0, None) == -1
    assert lib.moe_ep_combine(ctypes.byref(s), None, 1, *([None] * 6), None) == -1
    es = moe.shape(128, 256, 4, 1, 256)
    assert lib.moe_ep_expert_ffn(ctypes.byref(es), None, 1, None, None, None, None, None, None, 0,
                                 None) == -1
    assert lib.moe_ep_workspace_bytes(ctypes.byref(es)) >= 256
    # layer backward: widths must be multiples of 128; NULL pointers
    assert lib.moe_layer_bwd_workspace_bytes(ctypes.byref(moe.shape(64, 200, 8, 2, 256))) == 0
    assert lib.moe_layer_bwd_workspace_bytes(ctypes.byref(s)) > 0
    assert lib.moe_layer_bwd(ctypes.byref(s), None, None, None, None, 0.0, None, None, None, 0,
                             None) == -1


@pytest.mark.parametrize("T,d,N,k,h,ok", [
    (32, 512, 64, 8, 128, True),    # the decode GPU tests' shapes
    (32, 1024, 8, 2, 256, True),
    (5, 64, 4, 2, 32, True),
    (3, 96, 4, 3, 64, True),
    (1, 512, 8, 2, 128, True),
    (32, 512, 8, 2, 1024, True),    # h / 32 = 32 parts
    (33, 512, 8, 2, 128, False),    # T > 32
    (32, 512, 65, 2, 128, False),   # N > 64
    (32, 512, 64, 9, 128, False),   # k > 8
    (32, 500, 8, 2, 128, False),    # d not a multiple of 32
    (32, 512, 8, 2, 96, False),     # h / 32 = 3 does not divide 32
    (32, 512, 8, 2, 2048, False),   # h / 32 = 64 parts
    (32, 4096, 8, 2, 128, False),   # token rows alone exceed shared memory
])
def test_decode_shape_support_query(T, d, N, k, h, ok):
    """The decode workspace query is the shape-support check: nonzero exactly
    for the shapes the persistent kernel's shared-memory plan can hold."""
    n = moe.moe_decode_workspace_bytes(moe.shape(T, d, N, k, h, 1, 0))
    assert (n > 0) == ok


def test_decode_kernel_query_on_the_host():
    """The decode kernel query answers 0 for a shape outside the limits, and
    0 for every shape where no device is visible; with a device the benchmark
    shapes run the per-token kernel and 64 experts top-8 (more (token, slot)
    pairs than SMs) the two-phase kernel."""
    import torch
    assert moe.moe_decode_kernel(moe.shape(33, 512, 8, 2, 128, 1, 0)) == 0
    assert moe.moe_decode_kernel(moe.shape(32, 500, 8, 2, 128, 1, 0)) == 0
    if not torch.cuda.is_available():
        assert moe.moe_decode_kernel(moe.shape(32, 512, 8, 2, 128, 1, 0)) == 0
        return
    for T in (1, 8, 32):
        assert moe.moe_decode_kernel(moe.shape(T, 512, 8, 2, 128, 1, 0)) == moe.DECODE_PER_TOKEN
    assert moe.moe_decode_kernel(moe.shape(32, 512, 64, 8, 128, 1, 0)) == moe.DECODE_TWO_PHASE


@pytest.mark.parametrize("N,k", [(8, 2), (64, 8)])
def test_decode_plan_for_an_empty_batch(N, k):
    """The decode shape check plans T = 0 too (no items, no units): the
    workspace query answers on the host instead of failing."""
    assert moe.moe_decode_workspace_bytes(moe.shape(0, 512, N, k, 128, 1, 0)) > 0
