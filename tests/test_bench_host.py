"""Host-side pieces of bench.py that need no GPU: the oracle CPU baselines of
the decode and LatentMoE workloads (on shrunken shapes) and the LatentMoE
launch count."""
import dataclasses
import os
import sys

from conftest import ROOT

sys.path.insert(0, os.path.join(ROOT, "tests"))

import bench  # noqa: E402
from synthetic import workloads as W  # noqa: E402


def test_decode_cpu_baseline_runs_a_bounded_sample():
    wl = W.decode(T=8, n_layers=2)
    rate, seconds, n = bench.decode_cpu_baseline(wl, budget_s=0.2)
    assert rate > 0 and seconds >= 0.2 and n == 4


def test_latent_cpu_baseline_runs_a_bounded_sample():
    wl = dataclasses.replace(W.latent(T=64), N=32, d=256, latent=128, h=128, shared_hidden=128)
    rate, seconds, n = bench.latent_cpu_baseline(wl, budget_s=0.2)
    assert rate > 0 and seconds >= 0.2 and n == 1


def test_latent_fp8_cpu_baseline_runs_a_bounded_sample():
    wl = dataclasses.replace(W.latent(T=64), N=32, d=256, latent=128, h=128, shared_hidden=128)
    rate, seconds, n = bench.latent_cpu_baseline(wl, budget_s=0.2, fp8=True)
    assert rate > 0 and seconds >= 0.2 and n == 1


def test_latent_launch_count_matches_the_profiled_list():
    # 13 kernels per step in the committed LatentMoE launch list
    assert bench.latent_launches(W.latent()) == 13
    assert bench.latent_launches(dataclasses.replace(W.latent(), n_shared=0)) == 12


def test_oracle_thread_count_is_reported_and_settable():
    import oracle as O
    n = O.threads()
    assert n >= 1 and bench.oracle_threads() == n
    O.set_threads(1)
    try:
        assert O.threads() == 1
    finally:
        O.set_threads(n)
    assert O.threads() == n
    assert isinstance(bench.cpu_model(), str)


def _reference_line(capsys, workload, **kw):
    import argparse
    import json
    wl = W.decode(T=8, n_layers=2) if workload == "decode" else W.ALL[workload](**kw)
    args = argparse.Namespace(gpus=1, steps=1, warmup=3)
    bench.reference_arm(args, wl)
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    return wl, line


def test_reference_arm_line(capsys):
    """--impl reference prints the contract's line: the oracle's rate on the
    same workload label as the GPU arm, with its cpu_baseline and e2e."""
    for workload, kw in (("decode", {}), ("small", {"T": 512})):
        wl, line = _reference_line(capsys, workload, **kw)
        assert line["impl"] == "reference" and line["value"] > 0
        assert line["config"]["workload"] == bench.workload_label(wl)
        assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
        assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["value"] == line["value"]
        assert line["unit"] == "tokens/s" and line["higher_is_better"] is True


def test_decode_step_bytes_match_the_algorithmic_figures():
    """Decode roofline bytes per step: 24 layers x (router 16,384 B + 110,592 B
    per selected q4_0 expert + fp16 activations in and out), so 5.75 MB at one
    token (two experts per layer) and about 23.2 MB at 32 tokens, where the
    batch's union covers all 8 experts in every layer (the oracle's routing of
    the decode batch through each layer's router)."""
    import numpy as np
    import oracle as O
    import synthetic as S
    assert bench.Q4_EXPERT_BYTES(W.decode(T=1)) == 110592
    wl1 = W.decode(T=1)
    sel1 = np.array([[[0, 5]]] * wl1.n_layers)
    assert bench.decode_step_bytes(wl1, sel1) == 24 * (16384 + 2 * 110592 + 2048) == 5750784
    wl = W.decode(T=32)
    sel = []
    u = S.normal(wl.seed, W.TID_U, (wl.T, wl.d), 1.0, S.DT_F16)
    for layer in range(wl.n_layers):
        wr = S.normal(wl.seed, W.tid(W.TID_WROUTE, layer), (wl.N, wl.d), W.SIGMA_W, S.DT_F32)
        sel.append(O.route(O.as_f32(O.F16, u), wr, wl.k)[2])
    sel = np.array(sel)
    assert all(len(np.unique(sel[layer])) == 8 for layer in range(wl.n_layers))
    assert bench.decode_step_bytes(wl, sel) == 24 * (16384 + 8 * 110592 + 65536) == 23199744


def test_small_layer_algorithmic_work():
    """The small layer's work per step: T (2 N d + k 6 d h) = 3.25 GFLOP with
    every dispatch kept (no capacity); the roofline counts the expert part."""
    wl = W.small()
    experts = bench.expert_flops(wl, wl.T * wl.k)
    assert experts == 6 * 512 * 128 * 8192
    router = 2 * wl.T * wl.N * wl.d
    assert abs((router + experts) / 1e9 - 3.25) < 0.01


def test_layer_launch_counts():
    """Kernels per moe_layer_fwd step that bench.py claims: 3 for the small
    layer (one-launch routing, fused FFN, combine: the committed launch list),
    6 for the Mixtral-shaped layer (router with counts, dispatch, gather,
    gate/up GEMM, down GEMM, combine) and 4 for the fp32 layer (one-launch
    routing, two SIMT expert kernels, combine)."""
    assert bench.layer_launches(W.small()) == 3
    assert bench.layer_launches(W.mixtral()) == 6
    assert bench.layer_launches(W.tiny()) == 4
