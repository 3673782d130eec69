"""Benchmark of the sparse-MoE layer forward on B200 (tokens/s).

One step = one full pass of the layer (router -> permutation -> gather ->
grouped tcgen05 SwiGLU experts -> weighted combine) over one batch of seeded
synthetic tokens already resident in HBM.  Default workload: the
Mixtral-shaped layer (T=8192, d=4096, N=8 experts, h=14336, top-2, router
bias b_i = -1.2 ln(i+1), capacity factor 1.25, bf16).  Other workloads:
--workload small | latent | decode | tiny.

Timing: one pass is exactly --steps steps between two CUDA events, bracketed
by a barrier and a device synchronize.  Passes repeat until about one second
of device time has been timed, so that the clock sampler sees the timed
kernels; the reported time is the median pass (max over ranks per pass).

Prints ONE JSON line (rank 0).  With torchrun (N > 1) every rank runs its own
replica of the workload (the layer needs no collective: "replicas only",
weak scaling) and the time is the max over ranks.
--impl reference times the CPU oracle (the reference arm) on a bounded sample.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import synthetic as S  # noqa: E402
from synthetic import workloads as W  # noqa: E402

METRIC = "MoE-layer fwd tokens/s on 1 B200"

# DRAM bytes (read + write) per launch of a workload's dominant kernel, from one
# ncu capture (summary under profiles/).  Reported only while the kernel's
# source still hashes to the captured version; otherwise the value is stale.
PROFILED_TRAFFIC = {
    "small": {"bytes": 11571200 + 0, "src": "sparse_mixture_experts_15_b200/csrc/ffn_fused.cu",
              "sha1": "f01aa212595dfc284b7bf4a906467bdd015125b8", "profile": "profiles/tc_fused_ffn_small.md"},
    # gate/up + down launches of one Mixtral-shaped step (read + write)
    "mixtral": {"bytes": (3195234048 + 350338816) + (2617828096 + 188471808),
                "src": "sparse_mixture_experts_15_b200/csrc/gemm_tc.cu",
                "sha1": "d0e757544daf43d57f078d8fa58c3efd90adb6a8", "profile": "profiles/tc_grouped_gemm_mixtral.md"},
}


def profiled_traffic(workload: str):
    rec = PROFILED_TRAFFIC.get(workload)
    if not rec:
        return None
    import hashlib
    try:
        with open(os.path.join(ROOT, rec["src"]), "rb") as f:
            if hashlib.sha1(f.read()).hexdigest() != rec["sha1"]:
                return None
    except OSError:
        return None
    return rec["bytes"]
L2_BYTES = 126 * 1024 * 1024
# Nominal B200 figures (dense bf16 tensor cores, HBM3e), the second
# denominator next to the measured peaks.
SPEC_BF16_TFLOPS = 2250.0
SPEC_HBM_GBS = 8000.0


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return (float(d["hbm_gbs"]), float(d["bf16_tflops"]), float(d["bf16_tflops_sustained"]),
                "measured")
    return 6650.0, 1590.0, 1400.0, "fallback"


# ------------------------------------------------------------ multi-rank
def max_over_ranks(value: float, dist, device) -> float:
    """The slowest rank's time: every rank's device-timed value, reduced by MAX."""
    if dist is None:
        return value
    import torch
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


MIN_TIMED_MS = 1000.0  # device time covered by the timed passes together
MAX_PASSES = 2000


def set_min_timed_ms(ms: float):
    global MIN_TIMED_MS
    MIN_TIMED_MS = float(ms)


def timed_passes(run_pass, dist, device, min_total_ms: float | None = None):
    """Times passes of exactly `steps` steps until min_total_ms of device time.

    run_pass() launches one pass and returns its two recorded CUDA events.
    Every pass is bracketed by a barrier (N > 1) and a device synchronize, its
    time is the max over ranks, and the number of passes follows from the
    first pass's max-over-ranks time, so that every rank takes the same
    collective steps.  Returns (median pass ms, list of pass ms)."""
    import torch

    def one():
        if dist:
            dist.barrier()
        torch.cuda.synchronize()
        a, b = run_pass()
        torch.cuda.synchronize()
        return max_over_ranks(a.elapsed_time(b), dist, device)

    if min_total_ms is None:
        min_total_ms = MIN_TIMED_MS
    first = one()
    n = int(min(MAX_PASSES, max(3, -(-min_total_ms // max(first, 1e-3)))))
    passes = [first] + [one() for _ in range(n - 1)]
    return statistics.median(passes), passes


def pass_summary(passes, steps: int) -> str:
    """How the timed passes went, for config.timing."""
    return (f"{len(passes)} passes of {steps} steps (median reported; "
            f"min {min(passes):.3f} ms, max {max(passes):.3f} ms per pass)")


def whole_job_rate(tokens_per_rank_step: int, steps: int, world: int, ms: float) -> float:
    """Tokens/s of the whole job: all ranks' tokens over the slowest rank's time."""
    return tokens_per_rank_step * steps * world / (ms / 1e3)


def rank_seed(base_seed: int, rank: int, world: int, replica: int = 0) -> int:
    """Seed of replica `replica` on rank `rank`: every rank draws its own batch."""
    return base_seed + 7919 * (rank + world * replica)


# --------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.out = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"], stdout=self.out,
                stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.out.flush()
        rows = []
        with open(self.out.name) as f:
            for ln in f:
                parts = [x.strip() for x in ln.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.out.name)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": float(rows[0][2]) if rows[0][2].replace(".", "").isdigit() else None,
                "reasons": reasons, "samples": len(rows)}


# ------------------------------------------------------------ workload setup
class Replica:
    """Device inputs and weights of one copy of the workload."""

    def __init__(self, wl: W.Workload, seed: int, torch):
        self.wl = wl
        st = torch.cuda.current_stream().cuda_stream
        T, d, N, h = wl.T, wl.d, wl.N, wl.h
        tdt = {S.DT_F32: torch.float32, S.DT_BF16: torch.bfloat16, S.DT_F16: torch.float16}
        adt = tdt[wl.act_dtype]
        wdt = tdt[W.w_storage(wl)]
        self.u = torch.empty((T, d), dtype=adt, device="cuda")
        if wl.rms_inputs:
            S.rmsnorm_rows_dev(seed, W.TID_U, T, d, wl.act_dtype, self.u.data_ptr(), st)
        else:
            S.normal_dev(seed, W.TID_U, T * d, wl.u_sigma, wl.act_dtype, self.u.data_ptr(), st)
        self.w_route = torch.empty((N, d), dtype=torch.float32, device="cuda")
        S.normal_dev(seed, W.TID_WROUTE, N * d, W.SIGMA_W, S.DT_F32, self.w_route.data_ptr(), st)
        b = wl.router_bias()
        self.bias = None if b is None else torch.from_numpy(b).cuda()
        self.w = []
        for tid, shp in ((W.TID_WGATE, (N, h, d)), (W.TID_WUP, (N, h, d)),
                         (W.TID_WDOWN, (N, d, h))):
            t = torch.empty(shp, dtype=wdt, device="cuda")
            S.normal_dev(seed, tid, t.numel(), W.SIGMA_W, W.w_storage(wl), t.data_ptr(), st)
            self.w.append(t)

    def nbytes(self):
        return sum(t.numel() * t.element_size() for t in [self.u, self.w_route, *self.w])


def layer_launches(wl: W.Workload, sms: int = 148) -> int:
    """Kernels moe_layer_fwd launches for this workload (the library's own
    path choices restated): routing, permutation and row copies in one
    cooperative launch when a CTA's token rows and the router rows fit on chip,
    else router (+counts) / permutation / gather; the expert FFN in one fused
    launch for small h, else gate/up + down; then the combine."""
    T, d, N, k, h = wl.T, wl.d, wl.N, wl.k, wl.h
    el = 4 if wl.act_dtype == S.DT_F32 else 2
    r16 = lambda b: -(-b // 16) * 16
    grid = min(T, sms)
    tpc = -(-T // grid) if T else 0
    smem = (r16(tpc * (d * el + 16)) + r16(N * (d + 4) * 4) + r16(tpc * N * 4) + 2 * r16(tpc * k * 4)
            + 3 * 64 + 80 + 8 * 16 * 4 + r16(-(-T // tpc) * N * 4 if tpc else 0))
    one_launch_routing = (T > 0 and N <= 16 and k <= N and tpc * k <= 256
                          and smem <= 200 * 1024 and wl.act_dtype in (S.DT_F32, S.DT_BF16))
    if one_launch_routing:
        routing = 1
    elif N <= 16 and k <= 16 and (-(-T // (16 if N <= 8 else 8))) * N <= 8192:
        routing = 3  # router with counts, dispatch, gather
    else:
        routing = 6  # logits, top-k, histogram, scan, scatter, gather
    if wl.act_dtype == S.DT_F32:
        ffn = 2
    else:
        ffn = 1 if (h % 64 == 0 and h <= 256 and d % 128 == 0 and (h // 64 + d // 128) * 64 <= 512) else 2
    return routing + ffn + 1


class Step:
    """The layer step through the C ABI, split at the expert FFN so that the
    tcgen05 GEMM launches can be timed on their own stream position."""

    def __init__(self, wl: W.Workload, torch, moe):
        self.wl, self.torch, self.moe = wl, torch, moe
        T, d, N, k, h = wl.T, wl.d, wl.N, wl.k, wl.h
        self.s = moe.shape(T, d, N, k, h, wl.renorm, wl.capacity())
        i32 = dict(dtype=torch.int32, device="cuda")
        adt = {S.DT_F32: torch.float32, S.DT_BF16: torch.bfloat16}[wl.act_dtype]
        self.top_idx = torch.empty((T, k), **i32)
        self.top_w = torch.empty((T, k), dtype=torch.float32, device="cuda")
        self.logits = torch.empty((T, N), dtype=torch.float32, device="cuda")
        self.counts = torch.empty(N, **i32)
        self.offsets = torch.empty(N + 1, **i32)
        self.perm = torch.empty(T * k, **i32)
        self.row_of = torch.empty((T, k), **i32)
        self.overflow = torch.empty(N, **i32)
        self.totals = torch.empty(3, **i32)
        self.x_rows = torch.empty((T * k, d), dtype=adt, device="cuda")
        self.y_rows = torch.empty((T * k, d), dtype=torch.float32, device="cuda")
        self.y = torch.empty((T, d), dtype=adt, device="cuda")
        lib = moe._lib
        import ctypes
        pb = lib.moe_permute_workspace_bytes(ctypes.byref(self.s))
        fb = lib.moe_expert_ffn_workspace_bytes(ctypes.byref(self.s), d, wl.act_dtype)
        self.ws_perm = torch.empty(max(pb, 256), dtype=torch.uint8, device="cuda")
        self.ws_ffn = torch.empty(max(fb, 256), dtype=torch.uint8, device="cuda")
        self.act = moe.act()
        self.lws = torch.empty(moe.moe_layer_workspace_bytes(self.s, wl.act_dtype),
                               dtype=torch.uint8, device="cuda")
        self.outs = {"top_idx": self.top_idx, "top_w": self.top_w, "totals": self.totals}
        self.launches_per_step = layer_launches(wl)

    def layer(self, r: Replica):
        """The product entry point: the whole layer in one C-ABI call."""
        self.moe.moe_layer_fwd(self.s, r.w_route, *r.w, r.u, self.y, bias=r.bias,
                               outputs=self.outs, ws=self.lws)

    def ffn(self, r: Replica):
        """The expert FFN alone on replica r's own grouped rows (filled by
        split(r)), so consecutive replays read rows and weights that are not
        L2-resident."""
        self._ffn(r, r.x_rows, r.offsets)

    def _ffn(self, r: Replica, x_rows, offsets):
        self.moe.moe_expert_ffn(self.s, self.wl.d, x_rows, offsets, *r.w, self.y_rows, self.act,
                                ws=self.ws_ffn)

    def split(self, r: Replica):
        """The step split at the expert FFN; keeps r's grouped rows and offsets."""
        self(r)
        r.x_rows = self.x_rows.clone()
        r.offsets = self.offsets.clone()

    def __call__(self, r: Replica):
        m = self.moe
        m.moe_route(self.s, r.u, r.w_route, self.top_idx, self.top_w, bias=r.bias,
                    logits=self.logits)
        m.moe_permute(self.s, self.top_idx, self.counts, self.offsets, self.perm, self.row_of,
                      self.overflow, self.totals, ws=self.ws_perm)
        m.moe_gather(self.s, self.wl.d, r.u, self.perm, self.offsets, self.x_rows)
        self._ffn(r, self.x_rows, self.offsets)
        m.moe_combine(self.s, self.wl.d, self.y_rows, self.row_of, self.top_w, self.y)


def expert_flops(wl: W.Workload, kept_rows: int) -> float:
    """FLOPs of the expert GEMMs for kept_rows grouped rows: gate, up and down
    are three products of 2 d h FLOPs each per row."""
    return 6.0 * wl.d * wl.h * kept_rows


# --------------------------------------------------------------- oracle legs
def oracle_pass(wl: W.Workload, host, tokens):
    """The oracle on the listed tokens (routing of all tokens when a capacity
    makes drops depend on the whole batch)."""
    import oracle as O
    od = {S.DT_F32: O.F32, S.DT_BF16: O.BF16, S.DT_F16: O.F16}[wl.act_dtype]
    u_codes, w_route, bias, mats = host
    if wl.capacity():
        route_rows = np.arange(wl.T)
    else:
        route_rows = tokens
    _, _, idx, tw = O.route(O.as_f32(od, u_codes[route_rows]), w_route, wl.k, wl.renorm, bias)
    C = wl.capacity()
    perm = O.permute(idx, wl.N, C)
    sel = tokens if wl.capacity() else np.arange(len(tokens))
    O.moe_tokens([m[0] for m in mats], [m[1] for m in mats], [m[2] for m in mats],
                 O.decode(od, u_codes[tokens]), idx[sel], tw[sel], row_of=perm["row_of"][sel],
                 tokens=np.arange(len(tokens), dtype=np.int32),
                 round_h=int(wl.act_dtype == S.DT_BF16))


def oracle_host_inputs(wl: W.Workload):
    import oracle as O
    dt = W.w_storage(wl)
    od = {S.DT_F32: O.F32, S.DT_BF16: O.BF16}[dt]
    u = (S.rmsnorm_rows(wl.seed, W.TID_U, wl.T, wl.d, wl.act_dtype) if wl.rms_inputs
         else S.normal(wl.seed, W.TID_U, (wl.T, wl.d), wl.u_sigma, wl.act_dtype))
    w_route = S.normal(wl.seed, W.TID_WROUTE, (wl.N, wl.d), W.SIGMA_W, S.DT_F32)
    mats = []
    for e in range(wl.N):
        g = S.normal(wl.seed, W.TID_WGATE, (wl.h, wl.d), W.SIGMA_W, dt, offset=e * wl.h * wl.d)
        up = S.normal(wl.seed, W.TID_WUP, (wl.h, wl.d), W.SIGMA_W, dt, offset=e * wl.h * wl.d)
        dn = S.normal(wl.seed, W.TID_WDOWN, (wl.d, wl.h), W.SIGMA_W, dt, offset=e * wl.d * wl.h)
        mats.append((O.Mat(od, wl.h, wl.d, data=g), O.Mat(od, wl.h, wl.d, data=up),
                     O.Mat(od, wl.d, wl.h, data=dn)))
    return u, w_route, wl.router_bias(), mats


def cpu_sample_tokens(wl: W.Workload) -> int:
    """Tokens per oracle sample: about 10 s of host work on 8 cores."""
    per_token = 6.0 * wl.d * wl.h * wl.k
    return int(max(16, min(wl.T, 2.0e10 / per_token)))


def cpu_model() -> str:
    """The host CPU's model name, for the baseline line."""
    try:
        with open("/proc/cpuinfo") as f:
            for ln in f:
                if ln.startswith("model name"):
                    return ln.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def oracle_threads() -> int:
    import oracle as O
    return O.threads()


def run_cpu_baseline(wl: W.Workload, host, budget_s: float = 12.0, n: int = 0):
    n = n or cpu_sample_tokens(wl)
    rng = np.random.default_rng(0)
    done, t0 = 0, time.perf_counter()
    while True:
        tokens = np.sort(rng.choice(wl.T, n, replace=False)).astype(np.int32)
        oracle_pass(wl, host, tokens)
        done += n
        el = time.perf_counter() - t0
        if el >= budget_s:
            break
    return done / el, el, n


def workload_label(wl: W.Workload, fp8: bool = False) -> str:
    """The workload as both bench arms name it in config.workload."""
    if wl.name == "decode":
        return (f"decode: T={wl.T} d={wl.d} N={wl.N} h={wl.h} top-{wl.k}, "
                f"{wl.n_layers} layers per step")
    if wl.name == "latent":
        return (f"latent: T={wl.T} d={wl.d} l={wl.latent} E={wl.N} H={wl.h} top-{wl.k}, "
                f"{wl.n_shared} shared of hidden {wl.shared_hidden}, "
                f"caps {wl.beta_gate:g}/{wl.beta_up:g}"
                + (", E4M3 routed experts" if fp8 else ""))
    return f"{wl.name}: T={wl.T} d={wl.d} N={wl.N} h={wl.h} top-{wl.k}"


class DecodeOracle:
    """The decode workload's host weights (every layer, q4_0) and one oracle
    sample: random tokens of the batch through all layers (the tokens of a
    decode batch are independent of one another)."""

    def __init__(self, wl: W.Workload):
        import oracle as O
        self.O, self.wl = O, wl
        N, d, h = wl.N, wl.d, wl.h
        self.layers = []
        for layer in range(wl.n_layers):
            wr = S.normal(wl.seed, W.tid(W.TID_WROUTE, layer), (N, d), W.SIGMA_W, S.DT_F32)
            planes = []
            for base, rows, cols in ((W.TID_WGATE, h, d), (W.TID_WUP, h, d), (W.TID_WDOWN, d, h)):
                hq, hs = S.q4(wl.seed, W.tid(base, layer), N * rows, cols)
                planes.append([O.Mat(O.Q4_0, rows, cols, qs=hq[e * rows:(e + 1) * rows],
                                     scales=hs[e * rows:(e + 1) * rows]) for e in range(N)])
            self.layers.append((wr, list(zip(*planes))))
        self.u0 = S.normal(wl.seed, W.TID_U, (wl.T, d), 1.0, S.DT_F16)
        self.n = min(wl.T, 4)

    def sample(self, rng) -> int:
        u = self.u0[np.sort(rng.choice(self.wl.T, self.n, replace=False))]
        for wr, mats in self.layers:
            u = self.O.decode_layer(u, wr, mats, self.wl.k)[3]
        return self.n


def _tests_on_path():
    """The host-side input helpers shared with the tests live in tests/."""
    path = os.path.join(ROOT, "tests")
    if path not in sys.path:
        sys.path.insert(0, path)


class LatentOracle:
    """The LatentMoE workload's dense host weights; one oracle sample is one
    random token, whose 16 routed experts prepare() generates untimed
    (generation is not oracle work; 59 GB of experts never sit on the host)."""

    def __init__(self, wl: W.Workload, fp8: bool = False):
        import oracle as O
        _tests_on_path()
        from inputs import host_latent_dense
        self.O, self.wl, self.fp8 = O, wl, fp8
        self.W_dp, self.W_upp, self.shared = host_latent_dense(wl)
        self.w_route = S.normal(wl.seed, W.TID_WROUTE, (wl.N, wl.d), W.SIGMA_W, S.DT_F32)
        self.x_all = S.rmsnorm_rows(wl.seed, W.TID_U, wl.T, wl.d, S.DT_BF16)

    def prepare(self, rng):
        from inputs import host_latent_expert
        x = self.x_all[[int(rng.integers(self.wl.T))]]
        _, _, idx, _ = self.O.route(self.O.as_f32(self.O.BF16, x), self.w_route, self.wl.k)
        experts = {int(e): host_latent_expert(self.wl, int(e)) for e in idx[0]}
        if self.fp8:  # the oracle's own E4M3 quantiser, untimed like the generation
            O = self.O
            experts = {e: tuple(O.e4m3_mat(*O.quant_e4m3_rows(m.decode().astype(np.float32)))
                                for m in mats) for e, mats in experts.items()}
        return x, experts

    def run(self, prepared) -> int:
        x, experts = prepared
        self.O.latent_tokens(x, self.w_route, self.wl.k, self.W_dp, experts.__getitem__,
                             self.W_upp, self.shared, self.wl.beta_gate, self.wl.beta_up, 1e-6,
                             fp8=self.fp8)
        return 1


def decode_cpu_baseline(wl: W.Workload, budget_s: float = 12.0):
    """The oracle on the host cores for the decode workload, DecodeOracle
    samples until the budget is spent.  Returns (tokens/s, seconds, sample)."""
    ora = DecodeOracle(wl)
    rng = np.random.default_rng(0)
    done, t0 = 0, time.perf_counter()
    while True:
        done += ora.sample(rng)
        el = time.perf_counter() - t0
        if el >= budget_s:
            return done / el, el, ora.n


def latent_cpu_baseline(wl: W.Workload, budget_s: float = 12.0, fp8: bool = False):
    """The oracle on the host cores for the LatentMoE workload, one timed
    token per sample (its experts generated before the timed pass)."""
    ora = LatentOracle(wl, fp8)
    rng = np.random.default_rng(0)
    done, timed = 0, 0.0
    while timed < budget_s:
        prepared = ora.prepare(rng)
        t0 = time.perf_counter()
        done += ora.run(prepared)
        timed += time.perf_counter() - t0
    return done / timed, timed, 1


def latent_launches(wl: W.Workload) -> int:
    """Kernels moe_latent_fwd launches for a LatentMoE workload with more than
    16 routed experts (the library's path restated): router logits and top-k,
    the three permutation kernels, x_l = W_dp x, the gather, routed gate/up,
    routed down, the combine, RMSNorm, the shared experts' gate/up when there
    are shared experts, and the output GEMM."""
    assert wl.N > 16
    return 2 + 3 + 1 + 1 + 1 + 1 + 1 + 1 + (1 if wl.n_shared > 0 else 0) + 1


def reference_arm(args, wl):
    """--impl reference: the CPU oracle timed on this machine's host cores, each
    step a bounded sample of the workload (W untimed steps first)."""
    cores = oracle_threads()
    rng = np.random.default_rng(1)
    if wl.name == "decode":
        ora = DecodeOracle(wl)
        for _ in range(args.warmup):
            ora.sample(rng)
        t0 = time.perf_counter()
        n = sum(ora.sample(rng) for _ in range(args.steps))
        el = time.perf_counter() - t0
        cores = min(ora.n, cores)
        sample = f"{ora.n} random tokens through all {wl.n_layers} layers per step"
    elif wl.name == "latent":
        ora = LatentOracle(wl, getattr(args, "fp8", False))
        for _ in range(args.warmup):
            ora.run(ora.prepare(rng))
        n, el = 0, 0.0
        for _ in range(args.steps):
            prepared = ora.prepare(rng)
            t0 = time.perf_counter()
            n += ora.run(prepared)
            el += time.perf_counter() - t0
        cores = 1
        sample = "one random token per step (its 16 routed experts generated untimed)"
    else:
        host = oracle_host_inputs(wl)
        m = cpu_sample_tokens(wl) // 4 or 1
        samples = [np.sort(rng.choice(wl.T, m, replace=False)).astype(np.int32)
                   for _ in range(args.warmup + args.steps)]
        for i in range(args.warmup):
            oracle_pass(wl, host, samples[i])
        t0 = time.perf_counter()
        for i in range(args.steps):
            oracle_pass(wl, host, samples[args.warmup + i])
        el = time.perf_counter() - t0
        n = m * args.steps
        sample = f"{m} random tokens of the {wl.name} batch per step"
    value = n / el
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": el / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": workload_label(wl, getattr(args, "fp8", False))},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores,
                             "kind": "oracle", "cpu": cpu_model(), "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------- main
# ----------------------------------------------------------- decode workload
DECODE_LAYERS_PER_LAUNCH = 32  # layer descriptors one decode launch carries
Q4_EXPERT_BYTES = lambda wl: 3 * wl.h * wl.d // 2 + 3 * wl.h * wl.d // 32 * 2  # qs + fp16 scales


def decode_step_bytes(wl: W.Workload, sel) -> int:
    """Algorithmic HBM bytes of one decode step: per layer the fp32 router,
    the q4_0 weights of the union of the experts the batch selected (each
    read once), and the fp16 activations in and out.  sel: [layers][T][k]."""
    return sum(wl.N * wl.d * 4 + len(np.unique(sel[layer])) * Q4_EXPERT_BYTES(wl)
               + 2 * wl.T * wl.d * 2 for layer in range(wl.n_layers))


class DecodeReplica:
    """24 layers of q4_0 experts (all N experts resident; only selected ones read)."""

    def __init__(self, wl, seed, torch, moe):
        st = torch.cuda.current_stream().cuda_stream
        N, d, h = wl.N, wl.d, wl.h
        self.layers, self.keep = [], []
        for l in range(wl.n_layers):
            wr = torch.empty((N, d), dtype=torch.float32, device="cuda")
            S.normal_dev(seed, W.tid(W.TID_WROUTE, l), N * d, W.SIGMA_W, S.DT_F32,
                         wr.data_ptr(), st)
            mats = []
            for base, rows, cols in ((W.TID_WGATE, h, d), (W.TID_WUP, h, d),
                                     (W.TID_WDOWN, d, h)):
                qs = torch.empty((N * rows, cols // 2), dtype=torch.uint8, device="cuda")
                sc = torch.empty((N * rows, cols // 32), dtype=torch.int16, device="cuda")
                S.q4_dev(seed, W.tid(base, l), N * rows, cols, qs.data_ptr(), sc.data_ptr(), st)
                mats += [qs, sc]
            self.keep += [wr, *mats]
            self.layers.append(moe.q4_layer(wr, *mats))
        self.u = torch.empty((wl.T, d), dtype=torch.float16, device="cuda")
        S.normal_dev(seed, W.TID_U, wl.T * d, 1.0, S.DT_F16, self.u.data_ptr(), st)

    def nbytes(self):
        return sum(t.numel() * t.element_size() for t in self.keep)


# Intervals between the 13 per-layer stamps of each decode kernel (the
# bracketed ones are empty in the per-token kernel).
DECODE_PHASES = {
    1: ("(stamps 0-1)", "route", "(stamps 2-3)", "stage item rows", "(stamps 4-5)",
        "gate/up dots", "H", "(stamps 7-8)", "down columns ready", "down partial row",
        "cluster barrier", "next row"),
    2: ("stage u", "route", "group pairs", "stage gate/up rows", "(stamps 4-5)", "gate/up dots",
        "H store", "grid barrier 1", "down rows ready", "down dots", "combine + u_next",
        "grid barrier 2"),
}
DECODE_KERNELS = {
    1: "decode_token: all layers of the step in one launch, one thread-block cluster per token",
    2: "decode_persistent: all layers of the step in one cooperative launch, two grid barriers "
       "per layer",
}


def decode_phases(wl, moe, s, rep, out, ws, torch, sm_mhz: float):
    """Per-layer phase durations (us, median over layers 1..) of one traced
    decode step: SM-cycle stamps of block 0 converted at the sampled clock."""
    stamps = torch.zeros((wl.n_layers, moe.DECODE_STAMPS), dtype=torch.int64, device="cuda")
    for _ in range(2):  # the second call is warm
        moe.moe_decode_step_trace(s, rep.layers, rep.u, out, stamps, ws=ws)
    torch.cuda.synchronize()
    st = stamps.cpu().numpy().astype(np.float64)
    cyc = np.diff(st, axis=1)[1:] if wl.n_layers > 1 else np.diff(st, axis=1)
    per = np.median(cyc, axis=0) / sm_mhz
    layer = np.median(st[1:, -1] - st[1:, 0] if wl.n_layers > 1 else st[:, -1] - st[:, 0]) / sm_mhz
    return {"layer_us": float(layer), "sm_mhz": sm_mhz,
            **{name: float(v) for name, v in zip(DECODE_PHASES[moe.moe_decode_kernel(s)], per)}}


def decode_main(args, wl, torch, moe, rank, world, dist):
    stream = torch.cuda.current_stream()
    one = DecodeReplica(wl, rank_seed(wl.seed, rank, world), torch, moe)
    n_rep = max(1, -(-2 * L2_BYTES // one.nbytes()))
    reps = [one] + [DecodeReplica(wl, rank_seed(wl.seed, rank, world, i), torch, moe)
                    for i in range(1, n_rep)]
    s = moe.shape(wl.T, wl.d, wl.N, wl.k, wl.h, 1, 0)
    ws = torch.empty(moe.moe_decode_workspace_bytes(s), dtype=torch.uint8, device="cuda")
    out = torch.empty((wl.T, wl.d), dtype=torch.float16, device="cuda")
    idx_all = torch.empty((n_rep, wl.n_layers, wl.T, wl.k), dtype=torch.int32, device="cuda")

    def step(i):
        moe.moe_decode_step(s, reps[i].layers, reps[i].u, out, idx_all[i], ws=ws)

    for i in range(max(args.warmup, n_rep)):
        step(i % n_rep)
    torch.cuda.synchronize()
    assert moe.moe_device_status() == 0
    graphs = []
    cap = torch.cuda.Stream()
    cap.wait_stream(stream)
    with torch.cuda.stream(cap):
        for i in range(n_rep):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=cap):
                step(i)
            graphs.append(g)
    stream.wait_stream(cap)
    for i in range(args.warmup):
        graphs[i % n_rep].replay()
    torch.cuda.synchronize()
    sel = idx_all.cpu().numpy()
    step_bytes = [decode_step_bytes(wl, sel[i]) for i in range(n_rep)]
    sampler = ClockSampler(int(os.environ.get("LOCAL_RANK", "0"))) if rank == 0 else None

    def run_pass():
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for i in range(args.steps):
            graphs[i % n_rep].replay()
        b.record(stream)
        return a, b

    if sampler:
        sampler.start()
        time.sleep(0.3)
    torch.cuda.nvtx.range_push("timed")
    ms, passes = timed_passes(run_pass, dist, "cuda")
    torch.cuda.nvtx.range_pop()
    clocks = sampler.stop() if sampler else None
    hbm, _, _, src = _peaks()
    bytes_timed = sum(step_bytes[i % n_rep] for i in range(args.steps))
    achieved = bytes_timed / (ms / 1e3) / 1e9
    tokens = wl.T * args.steps * world
    # end to end: pinned host u -> device -> 24 layers -> pinned host output
    u_host = reps[0].u.cpu().pin_memory()
    o_host = torch.empty_like(out, device="cpu").pin_memory()
    u_dev = torch.empty_like(reps[0].u)
    for _ in range(args.warmup):
        u_dev.copy_(u_host, non_blocking=True)
        moe.moe_decode_step(s, reps[0].layers, u_dev, out, ws=ws)
        o_host.copy_(out, non_blocking=True)
    torch.cuda.synchronize()
    ea, eb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ea.record(stream)
    for _ in range(args.steps):
        u_dev.copy_(u_host, non_blocking=True)
        moe.moe_decode_step(s, reps[0].layers, u_dev, out, ws=ws)
        o_host.copy_(out, non_blocking=True)
    eb.record(stream)
    torch.cuda.synchronize()
    e_ms = max_over_ranks(ea.elapsed_time(eb), dist, "cuda")
    phases = decode_phases(wl, moe, s, reps[0], out, ws, torch,
                           (clocks or {}).get("sm_mhz") or 1965.0)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, el_s, n = decode_cpu_baseline(wl)
        cpu = {"value": v, "unit": "tokens/s", "cores": min(n, oracle_threads()), "kind": "oracle",
               "cpu": cpu_model(),
               "sample": f"random samples of {n} tokens through all {wl.n_layers} layers, "
                         f"{el_s:.1f} s of CPU work"}
    if rank == 0:
        line = {"metric": METRIC, "value": whole_job_rate(wl.T, args.steps, world, ms),
                "unit": "tokens/s",
                "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": ms / args.steps, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "q4_0 weights, fp16 activations, fp32 math",
                "data": "synthetic",
                "config": {"workload": workload_label(wl),
                           "global_batch": wl.T * world, "parallelism": f"replicas x{world}",
                           "timing": pass_summary(passes, args.steps),
                           "l2": f"weights rotate over {n_rep} replicas "
                                 f"({n_rep * one.nbytes() / 2**20:.0f} MiB > L2)"},
                "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s",
                             "frac": achieved / hbm, "traffic": None,
                             "kernel": DECODE_KERNELS[moe.moe_decode_kernel(s)],
                             "phases_us": phases,
                             "bytes_per_step": bytes_timed / args.steps,
                             "peak_source": f"{src} hbm_gbs",
                             "frac_of_spec": achieved / SPEC_HBM_GBS},
                "cpu_baseline": cpu,
                "e2e": {"value": tokens / (e_ms / 1e3), "unit": "tokens/s",
                        "h2d_bytes_per_step": wl.T * wl.d * 2,
                        "d2h_bytes_per_step": wl.T * wl.d * 2},
                "gpu_launches": -(-wl.n_layers // DECODE_LAYERS_PER_LAUNCH) * args.steps,
                "clocks": clocks}
        print(json.dumps(line), flush=True)


# ----------------------------------------------------------- latent workload
def latent_main(args, wl, torch, moe, rank, world, dist):
    _tests_on_path()
    stream = torch.cuda.current_stream()
    st = stream.cuda_stream
    E, d, l, h, n, sh = wl.N, wl.d, wl.latent, wl.h, wl.n_shared, wl.shared_hidden
    seed = rank_seed(wl.seed, rank, world)

    def normal(tid, shape, dt, tdt):
        t = torch.empty(shape, dtype=tdt, device="cuda")
        S.normal_dev(seed, tid, t.numel(), W.SIGMA_W, dt, t.data_ptr(), st)
        return t

    bf = torch.bfloat16
    w_route = normal(W.TID_WROUTE, (E, d), S.DT_F32, torch.float32)

    def routed(tid, rows, cols):
        """Routed expert weights: bf16, or with --fp8 E4M3 codes and row
        scales made by the library's quantiser from the same bf16 draws (in
        chunks of experts, so the bf16 copy never exists whole)."""
        if not args.fp8:
            return normal(tid, (E, rows, cols), S.DT_BF16, bf), None
        codes = torch.empty((E, rows, cols), dtype=torch.uint8, device="cuda")
        scales = torch.empty(E * rows, dtype=torch.float32, device="cuda")
        chunk = 64
        tmp = torch.empty((chunk, rows, cols), dtype=bf, device="cuda")
        for e0 in range(0, E, chunk):
            m = min(chunk, E - e0)
            S.normal_dev(seed, tid, m * rows * cols, W.SIGMA_W, S.DT_BF16, tmp.data_ptr(), st,
                         offset=e0 * rows * cols)
            moe.moe_quantize_e4m3_rows(tmp[:m].reshape(m * rows, cols), codes[e0:e0 + m],
                                       scales[e0 * rows:(e0 + m) * rows])
        del tmp
        return codes, scales

    wg, wg_s = routed(W.TID_WGATE, h, l)
    wu, wu_s = routed(W.TID_WUP, h, l)
    wd, wd_s = routed(W.TID_WDOWN, l, h)
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    w_dp = normal(W.TID_WDP, (l, d), S.DT_BF16, bf)
    w_upp = normal(W.TID_WUPP, (d, l), S.DT_BF16, bf)
    sg = torch.empty((n, sh, d), dtype=bf, device="cuda")
    su, sd = torch.empty_like(sg), torch.empty((n, d, sh), dtype=bf, device="cuda")
    for j in range(n):
        tg, tu, td = W.shared_tids(j)
        S.normal_dev(seed, tg, sh * d, W.SIGMA_W, S.DT_BF16, sg[j].data_ptr(), st)
        S.normal_dev(seed, tu, sh * d, W.SIGMA_W, S.DT_BF16, su[j].data_ptr(), st)
        S.normal_dev(seed, td, d * sh, W.SIGMA_W, S.DT_BF16, sd[j].data_ptr(), st)
    x = torch.empty((wl.T, d), dtype=bf, device="cuda")
    S.rmsnorm_rows_dev(seed, W.TID_U, wl.T, d, S.DT_BF16, x.data_ptr(), st)
    y = torch.empty_like(x)
    s = moe.shape(wl.T, d, E, wl.k, h, 1, 0)
    lw = moe.latent_weights(l, w_dp, w_upp, sg, su, sd, n, sh, 1e-6)
    ws = torch.empty(moe.moe_latent_workspace_bytes(s, lw), dtype=torch.uint8, device="cuda")
    counts = torch.empty(E, dtype=torch.int32, device="cuda")
    act = moe.act(moe.ACT_SITU_GLU, wl.beta_gate, wl.beta_up)

    def layer(x_in, outputs=None):
        if args.fp8:
            moe.moe_latent_fwd_e4m3(s, w_route, wg, wu, wd, wg_s, wu_s, wd_s, lw, x_in, y, a=act,
                                    outputs=outputs, ws=ws)
        else:
            moe.moe_latent_fwd(s, w_route, wg, wu, wd, lw, x_in, y, a=act, outputs=outputs,
                               ws=ws)

    def step():
        layer(x, {"counts": counts})

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert moe.moe_device_status() == 0
    g = torch.cuda.CUDAGraph()
    cap = torch.cuda.Stream()
    cap.wait_stream(stream)
    with torch.cuda.stream(cap):
        with torch.cuda.graph(g, stream=cap):
            step()
    stream.wait_stream(cap)
    g.replay()
    torch.cuda.synchronize()
    used = int((counts > 0).sum().item())
    # algorithmic HBM bytes: router + touched routed experts + dense weights + activations
    routed_bytes = used * 3 * l * h * 2 if not args.fp8 else used * (3 * l * h + (2 * h + l) * 4)
    wbytes = (E * d * 4 + routed_bytes + 2 * l * d * 2 + n * 3 * sh * d * 2)
    abytes = 2 * wl.T * d * 2
    step_bytes = wbytes + abytes
    flops = (2.0 * wl.T * E * d + 2.0 * wl.T * l * d + 6.0 * l * h * wl.T * wl.k
             + 2.0 * wl.T * d * l + n * 6.0 * wl.T * d * sh)
    sampler = ClockSampler(int(os.environ.get("LOCAL_RANK", "0"))) if rank == 0 else None

    def run_pass():
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(args.steps):
            g.replay()
        b.record(stream)
        return a, b

    if sampler:
        sampler.start()
        time.sleep(0.3)
    torch.cuda.nvtx.range_push("timed")
    ms, passes = timed_passes(run_pass, dist, "cuda")
    torch.cuda.nvtx.range_pop()
    clocks = sampler.stop() if sampler else None
    hbm, tf, _, src = _peaks()
    per_step_s = ms / args.steps / 1e3
    achieved = step_bytes / per_step_s / 1e9
    # end to end: pinned host x -> device -> layer -> pinned host y
    x_host = x.cpu().pin_memory()
    y_host = torch.empty_like(y, device="cpu").pin_memory()
    x_dev = torch.empty_like(x)
    ea, eb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ea.record(stream)
    for _ in range(args.steps):
        x_dev.copy_(x_host, non_blocking=True)
        layer(x_dev)
        y_host.copy_(y, non_blocking=True)
    eb.record(stream)
    torch.cuda.synchronize()
    e_ms = max_over_ranks(ea.elapsed_time(eb), dist, "cuda")
    tokens = wl.T * args.steps * world
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, el_s, n = latent_cpu_baseline(wl, fp8=args.fp8)
        cpu = {"value": v, "unit": "tokens/s", "cores": 1, "kind": "oracle", "cpu": cpu_model(),
               "sample": f"random single tokens of the latent batch, {el_s:.1f} s of "
                         "oracle work (their routed experts generated"
                         f"{' and quantised' if args.fp8 else ''} untimed)"}
    if rank == 0:
        line = {"metric": METRIC, "value": whole_job_rate(wl.T, args.steps, world, ms),
                "unit": "tokens/s",
                "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": ms / args.steps, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None,
                "dtype": "e4m3 routed experts, bf16 elsewhere" if args.fp8 else "bf16",
                "data": "synthetic",
                "config": {"workload": workload_label(wl, args.fp8),
                           "global_batch": wl.T * world, "parallelism": f"replicas x{world}",
                           "timing": pass_summary(passes, args.steps),
                           "l2": (f"routed expert weights {routed_bytes / 1e9:.1f} GB > L2"),
                           "experts_touched": used},
                "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s",
                             "frac": achieved / hbm, "traffic": None,
                             "kernel": "whole layer step (routed tcgen05 GEMMs stream every "
                                       "touched expert once)",
                             "bytes_per_step": step_bytes,
                             "tflops": flops / per_step_s / 1e12,
                             "peak_source": f"{src} hbm_gbs",
                             "frac_of_spec": achieved / SPEC_HBM_GBS},
                "cpu_baseline": cpu,
                "e2e": {"value": tokens / (e_ms / 1e3), "unit": "tokens/s",
                        "h2d_bytes_per_step": wl.T * d * 2, "d2h_bytes_per_step": wl.T * d * 2},
                "gpu_launches": latent_launches(wl) * args.steps, "clocks": clocks}
        print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="mixtral",
                    choices=["small", "mixtral", "tiny", "decode", "latent"])
    ap.add_argument("--decode-T", type=int, default=32, help="decode batch (1, 8 or 32)")
    ap.add_argument("--tokens", type=int, default=0,
                    help="override T (smaller cases for profiling captures)")
    ap.add_argument("--experts", type=int, default=0,
                    help="latent workload: override the routed expert count (profiling captures "
                         "of a few GB with the full-size per-expert shape)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--fp8", action="store_true",
                    help="latent workload: E4M3 routed experts (moe_latent_fwd_e4m3)")
    ap.add_argument("--min-timed-ms", type=float, default=1000.0,
                    help="device time the timed passes cover together (smaller for profiling)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    set_min_timed_ms(args.min_timed_ms)
    wl = W.decode(T=args.decode_T) if args.workload == "decode" else W.ALL[args.workload]()
    if args.tokens > 0 and args.workload != "decode":
        wl.T = args.tokens
    if args.experts > 0:
        if args.workload != "latent":
            ap.error("--experts applies to the latent workload")
        wl.N = args.experts

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank == 0:
            reference_arm(args, wl)
        return

    import torch
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    import sparse_mixture_experts_15_b200 as moe

    if args.workload in ("decode", "latent"):
        (decode_main if args.workload == "decode" else latent_main)(args, wl, torch, moe, rank,
                                                                    world, dist)
        if dist:
            dist.barrier()
            dist.destroy_process_group()
        return

    # replicas rotate so that the inputs of consecutive steps exceed L2
    one = Replica(wl, rank_seed(wl.seed, rank, world), torch)
    n_rep = max(1, min(64, -(-2 * L2_BYTES // max(one.nbytes(), 1))))
    reps = [one] + [Replica(wl, rank_seed(wl.seed, rank, world, i), torch)
                    for i in range(1, n_rep)]
    step = Step(wl, torch, moe)
    stream = torch.cuda.current_stream()

    for i in range(args.warmup):
        step.layer(reps[i % n_rep])
    for r in reps:  # each replica's grouped rows and offsets for the GEMM-only replays
        step.split(r)
    torch.cuda.synchronize()
    kept = [0] * n_rep
    for i in range(n_rep):
        step.layer(reps[i])
        torch.cuda.synchronize()
        kept[i] = int(step.totals[0].item())
    assert moe.moe_device_status() == 0

    # The step (moe_layer_fwd) is device-only work (no host sync), so each
    # replica's step is captured once as a CUDA graph and replayed.
    full_g, ffn_g = [], []
    cap = torch.cuda.Stream()
    cap.wait_stream(stream)
    with torch.cuda.stream(cap):
        for i in range(n_rep):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=cap):
                step.layer(reps[i])
            full_g.append(g)
            g2 = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g2, stream=cap):
                step.ffn(reps[i])
            ffn_g.append(g2)
    stream.wait_stream(cap)
    for i in range(args.warmup):
        full_g[i % n_rep].replay()
    torch.cuda.synchronize()

    sampler = ClockSampler(local) if rank == 0 else None

    def graph_pass(graphs):
        def run():
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            for i in range(args.steps):
                graphs[i % n_rep].replay()
            b.record(stream)
            return a, b
        return run

    if sampler:
        sampler.start()
        time.sleep(0.3)
    torch.cuda.nvtx.range_push("timed")
    ms, passes = timed_passes(graph_pass(full_g), dist, "cuda")
    torch.cuda.nvtx.range_pop()
    clocks = sampler.stop() if sampler else None
    # the dominant kernel alone: the expert FFN launches of each step, timed
    # the same way (median pass)
    f_ms, f_passes = timed_passes(graph_pass(ffn_g), dist, "cuda",
                                  min_total_ms=MIN_TIMED_MS / 2)
    ffn_ms = [f_ms / args.steps] * args.steps
    tokens = wl.T * args.steps * world
    value = whole_job_rate(wl.T, args.steps, world, ms)

    # roofline of the dominant kernel: the tcgen05 grouped GEMM (gate/up + down launches)
    hbm, tf_burst, tf_sust, peak_src = _peaks()
    fused = (wl.h % 64 == 0 and wl.h <= 256 and wl.d % 128 == 0
             and (wl.h // 64 + wl.d // 128) * 64 <= 512)
    kept_timed = [kept[i % n_rep] for i in range(args.steps)]
    gemm_flops = sum(expert_flops(wl, kr) for kr in kept_timed)
    gemm_s = sum(ffn_ms) / 1e3
    achieved_tf = gemm_flops / gemm_s / 1e12
    # The GEMM launches run back to back for half a second or more, long
    # enough for the 1 kW power cap to settle the clocks: the denominator is
    # the measured sustained bf16 GEMM rate (a seconds-long cuBLAS loop under
    # the same cap) when the timed loop is that long, else the burst rate.
    long_loop = sum(f_passes) >= 250.0
    tf_peak = tf_sust if long_loop else tf_burst
    roofline = {"bound": "tensor", "achieved": achieved_tf, "peak": tf_peak, "unit": "TFLOP/s",
                "frac": achieved_tf / tf_peak, "frac_of_burst": achieved_tf / tf_burst,
                "traffic": profiled_traffic(wl.name),
                "kernel": ("tc_fused_ffn (gate/up + SwiGLU + down in one launch, H on chip)"
                           if fused else "tc_grouped_gemm (gate/up + down, 2 launches per step)"),
                "peak_source": (f"{peak_src} bf16_tflops_sustained (GEMM loop of "
                                f"{sum(f_passes):.0f} ms)" if long_loop
                                else f"{peak_src} bf16_tflops (burst)"),
                "frac_of_spec": achieved_tf / SPEC_BF16_TFLOPS,
                "ms_per_launch_pair": gemm_s / args.steps * 1e3}

    # end to end: pinned host input -> device -> layer -> pinned host output
    e2e = None
    if not args.no_e2e:
        u_host = torch.empty_like(reps[0].u, device="cpu").pin_memory()
        u_host.copy_(reps[0].u.cpu())
        y_host = torch.empty_like(step.y, device="cpu").pin_memory()
        u_dev = torch.empty_like(reps[0].u)
        r0 = reps[0]
        outs = {"top_idx": step.top_idx}
        lws = torch.empty(moe.moe_layer_workspace_bytes(step.s, wl.act_dtype), dtype=torch.uint8,
                          device="cuda")

        def e2e_step():
            u_dev.copy_(u_host, non_blocking=True)
            moe.moe_layer_fwd(step.s, r0.w_route, *r0.w, u_dev, step.y, bias=r0.bias,
                              outputs=outs, ws=lws)
            y_host.copy_(step.y, non_blocking=True)

        def serial_ms():
            for _ in range(args.warmup):
                e2e_step()
            torch.cuda.synchronize()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            for _ in range(args.steps):
                e2e_step()
            b.record(stream)
            torch.cuda.synchronize()
            return a.elapsed_time(b)

        def pipelined_ms():
            """Every step uploads its input and downloads its result, on two
            copy streams with double-buffered device tensors, so that step
            i+1's upload and step i-1's download overlap step i's layer on the
            compute stream (PCIe carries both directions at once)."""
            h2d, d2h = torch.cuda.Stream(), torch.cuda.Stream()
            u_b = [torch.empty_like(u_dev) for _ in range(2)]
            y_b = [torch.empty_like(step.y) for _ in range(2)]
            y_h = [torch.empty_like(step.y, device="cpu").pin_memory() for _ in range(2)]
            up, done, down = ([torch.cuda.Event() for _ in range(2)] for _ in range(3))
            for ev in (*up, *done, *down):
                ev.record(stream)

            def one(i):
                j = i % 2
                h2d.wait_event(done[j])            # the layer that last read u_b[j] is done
                with torch.cuda.stream(h2d):
                    u_b[j].copy_(u_host, non_blocking=True)
                    up[j].record(h2d)
                stream.wait_event(up[j])
                stream.wait_event(down[j])          # y_b[j]'s previous download is done
                moe.moe_layer_fwd(step.s, r0.w_route, *r0.w, u_b[j], y_b[j], bias=r0.bias,
                                  outputs=outs, ws=lws)
                done[j].record(stream)
                d2h.wait_event(done[j])
                with torch.cuda.stream(d2h):
                    y_h[j].copy_(y_b[j], non_blocking=True)
                    down[j].record(d2h)

            for i in range(args.warmup):
                one(i)
            torch.cuda.synchronize()

            def run_pass():
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(stream)
                h2d.wait_event(a)
                for i in range(args.steps):
                    one(i)
                for ev in down:
                    stream.wait_event(ev)
                b.record(stream)
                return a, b

            # passes over about half a second, as the device-timed legs, so
            # that the clocks under the power cap match theirs
            e_ms, _ = timed_passes(run_pass, dist, "cuda", min_total_ms=MIN_TIMED_MS / 2)
            return e_ms

        mode = ("pipelined: two copy streams, double-buffered inputs and outputs; median of "
                "passes over about half a second")
        try:
            e_ms = pipelined_ms()
        except Exception as exc:  # measure the plain serial loop instead
            torch.cuda.synchronize()
            mode = f"serial (pipelined run failed: {type(exc).__name__})"
            e_ms = serial_ms()
        if mode.startswith("serial"):
            e_ms = max_over_ranks(e_ms, dist, "cuda")
        el = 2 if wl.act_dtype != S.DT_F32 else 4
        e2e = {"value": tokens / (e_ms / 1e3), "unit": "tokens/s",
               "h2d_bytes_per_step": wl.T * wl.d * el, "d2h_bytes_per_step": wl.T * wl.d * el,
               "mode": mode}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        host = oracle_host_inputs(wl)
        v, el_s, n = run_cpu_baseline(wl, host)
        import oracle as O
        threads = O.threads()
        O.set_threads(1)
        v1, _, _ = run_cpu_baseline(wl, host, budget_s=6.0,
                                    n=max(1, cpu_sample_tokens(wl) // threads))
        O.set_threads(threads)
        cpu = {"value": v, "unit": "tokens/s", "cores": threads, "kind": "oracle",
               "one_thread_value": v1, "cpu": cpu_model(),
               "sample": f"random samples of {n} tokens of the {wl.name} batch, "
                         f"{el_s:.1f} s of CPU work"}

    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms / args.steps,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": "bf16" if wl.act_dtype == S.DT_BF16 else "f32", "data": "synthetic",
                "config": {"workload": workload_label(wl), "global_batch": wl.T * world,
                           "parallelism": f"replicas x{world}",
                           "timing": pass_summary(passes, args.steps),
                           "l2": f"inputs rotate over {n_rep} replicas "
                                 f"({n_rep * one.nbytes() / 2**20:.0f} MiB > L2)",
                           "capacity": wl.capacity()},
                "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
                "gpu_launches": step.launches_per_step * args.steps, "clocks": clocks}
        print(json.dumps(line), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
