"""The C ABI from plain C, without a GPU.

A C11 program that includes include/moe.h is compiled with warnings as errors
(and the header once more as C++), linked against the library, and run.  It
prints the size and every field offset of the header's structs, which must
match the Python binding's ctypes mirrors, and calls the host-only entry
points and the host-side argument checks.
"""
import ctypes
import os
import shutil
import subprocess

import pytest

from conftest import ROOT

import sparse_mixture_experts_15_b200 as moe

STRUCTS = {
    "moe_shape": (moe.MoeShape, ["T", "d", "N", "k", "h", "renorm", "capacity"]),
    "moe_act": (moe.MoeAct, ["kind", "beta_gate", "beta_up"]),
    "moe_layer_weights": (moe.MoeLayerWeights,
                          ["w_route", "bias", "w_gate", "w_up", "w_down", "w_dtype", "act"]),
    "moe_layer_outputs": (moe.MoeLayerOutputs,
                          ["top_idx", "top_w", "probs", "counts", "offsets", "perm_tok",
                           "row_of", "overflow", "totals", "f", "P", "n_sum_fP"]),
    "moe_q4_layer": (moe.MoeQ4Layer, ["w_route", "bias", "gate_qs", "gate_scales", "up_qs",
                                      "up_scales", "down_qs", "down_scales"]),
    "moe_latent_weights": (moe.MoeLatentWeights,
                           ["latent", "n_shared", "shared_hidden", "w_down_proj", "w_up_proj",
                            "shared_gate", "shared_up", "shared_down", "rms_eps"]),
}

PROGRAM = r"""
#include <stddef.h>
#include <stdio.h>
#include <string.h>
#include "moe.h"

#define FIELD(s, f) printf(#s " " #f " %zu\n", offsetof(s, f))

int main(void) {
%FIELDS%
  /* host-only entry points */
  int32_t c = -1;
  if (moe_capacity(8192, 8, 2, 1.25, &c) != MOE_OK || c != 2560) return 10;
  if (moe_capacity(-1, 8, 2, 1.0, &c) != MOE_ERR_INVALID_ARG) return 11;
  if (strncmp(moe_status_string(MOE_ERR_WORKSPACE), "MOE_ERR_WORKSPACE", 17) != 0) return 12;
  /* argument checks run on the host before any device work */
  moe_shape s = {4096, 512, 8, 2, 128, 1, 0};
  if (moe_layer_fwd(NULL, NULL, NULL, MOE_BF16, NULL, NULL, NULL, 0, NULL) != MOE_ERR_INVALID_ARG)
    return 13;
  moe_shape bad = s;
  bad.k = 9;
  if (moe_route_workspace_bytes(&bad) != 0) return 14;
  if (moe_permute_workspace_bytes(&s) == 0) return 15;
  if (moe_quantile_balance(0, 8, 2, NULL, NULL, 1, 0, NULL, NULL, NULL, NULL, NULL, 0, NULL)
      != MOE_ERR_INVALID_ARG) return 16;
  /* the expert-parallel exchange plan is host only */
  const int32_t counts[2][4] = {{3, 0, 2, 1}, {1, 4, 0, 2}};
  int32_t kept[4], loff[5], sbase[4], scnt[2], roff[3], rsrc[2][2], rcnt[2], ovf[4];
  if (moe_ep_plan(2, 1, 4, 3, &counts[0][0], kept, loff, sbase, scnt, roff, &rsrc[0][0], rcnt,
                  ovf) != MOE_OK)
    return 17;
  if (kept[1] != 3 || kept[3] != 2 || sbase[0] != 3 || roff[2] != 5 || rsrc[1][1] != 3 ||
      ovf[0] != 1)
    return 18;
  printf("ok\n");
  return 0;
}
"""


def _fields_c():
    lines = []
    for name, (_, fields) in STRUCTS.items():
        lines.append(f'  printf("{name} sizeof %zu\\n", sizeof({name}));')
        lines += [f"  FIELD({name}, {f});" for f in fields]
    return "\n".join(lines)


@pytest.fixture(scope="module")
def c_program(tmp_path_factory):
    if shutil.which("gcc") is None:
        pytest.skip("gcc not available")
    d = tmp_path_factory.mktemp("cabi")
    src = d / "abi.c"
    src.write_text(PROGRAM.replace("%FIELDS%", _fields_c()))
    exe = d / "abi"
    libdir = os.path.dirname(moe.LIB_PATH)
    subprocess.run(["gcc", "-std=c11", "-Wall", "-Wextra", "-Werror", "-pedantic",
                    "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe),
                    "-L", libdir, "-lmoe", f"-Wl,-rpath,{libdir}"], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True)
    return out


def test_c_program_runs_host_checks(c_program):
    assert c_program.returncode == 0, (c_program.returncode, c_program.stdout, c_program.stderr)
    assert c_program.stdout.strip().endswith("ok")


def test_struct_layout_matches_binding(c_program):
    got = {}
    for ln in c_program.stdout.splitlines():
        parts = ln.split()
        if len(parts) == 3 and parts[0] in STRUCTS:
            got[(parts[0], parts[1])] = int(parts[2])
    for name, (cls, fields) in STRUCTS.items():
        assert got[(name, "sizeof")] == ctypes.sizeof(cls), name
        assert [f for f, _ in cls._fields_] == fields, name
        for f in fields:
            assert got[(name, f)] == getattr(cls, f).offset, (name, f)


def test_header_compiles_as_cpp(tmp_path):
    if shutil.which("g++") is None:
        pytest.skip("g++ not available")
    src = tmp_path / "abi.cpp"
    src.write_text('#include "moe.h"\nint main() { return moe_capacity(1, 1, 1, 1.0, nullptr) '
                   '== MOE_ERR_INVALID_ARG ? 0 : 1; }\n')
    subprocess.run(["g++", "-std=c++17", "-Wall", "-Wextra", "-Werror", "-pedantic",
                    "-I", os.path.join(ROOT, "include"), "-c", str(src), "-o",
                    str(tmp_path / "abi.o")], check=True)
