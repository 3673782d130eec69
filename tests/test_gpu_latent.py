"""GPU parity of the LatentMoE layer (Stable LatentMoE demo document: width
separation, RMSNorm before the up-projection, SiTU-GLU soft caps) against the
CPU oracle, through the C ABI.  Its test names follow the document's:
forward shape and routing, agreement with an independent reference, routed
experts living in the latent bottleneck."""
import numpy as np
import pytest

import oracle as O
import synthetic as S
from synthetic import workloads as W

from inputs import dev_latent, dev_u, host_latent_dense, host_latent_expert, host_u, rel_err

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

TOL_BF16 = 2e-2

if torch.cuda.is_available():
    import sparse_mixture_experts_15_b200 as moe


@pytest.fixture(autouse=True)
def _clean_status():
    moe.moe_reset_device_status()
    yield
    assert moe.moe_device_status() == 0


def small_latent(T=200):
    return W.Workload("latent_small", T=T, d=256, N=32, k=4, h=128, seed=1005,
                      act_dtype=S.DT_BF16, w_dtype="bf16", rms_inputs=True, latent=128,
                      n_shared=2, shared_hidden=128, beta_gate=4.0, beta_up=25.0)


def _run_gpu(wl, dw=None):
    dw = dw or dev_latent(wl)
    T = wl.T
    s = moe.shape(T, wl.d, wl.N, wl.k, wl.h, 1, 0)
    lw = moe.latent_weights(wl.latent, dw["w_dp"], dw["w_upp"], dw["shared_gate"],
                            dw["shared_up"], dw["shared_down"], wl.n_shared, wl.shared_hidden,
                            1e-6)
    x = dev_u(wl)
    y = torch.empty((T, wl.d), dtype=torch.bfloat16, device="cuda")
    i32 = dict(dtype=torch.int32, device="cuda")
    outs = dict(top_idx=torch.empty((T, wl.k), **i32),
                top_w=torch.empty((T, wl.k), dtype=torch.float32, device="cuda"),
                counts=torch.empty(wl.N, **i32))
    moe.moe_latent_fwd(s, dw["w_route"], dw["w_gate"], dw["w_up"], dw["w_down"], lw, x, y,
                       a=moe.act(moe.ACT_SITU_GLU, wl.beta_gate, wl.beta_up), outputs=outs)
    torch.cuda.synchronize()
    return y, {k: v.cpu().numpy() for k, v in outs.items()}


def _oracle(wl, tokens):
    x_codes = host_u(wl)[tokens]
    w_route = S.normal(wl.seed, W.TID_WROUTE, (wl.N, wl.d), W.SIGMA_W, S.DT_F32)
    W_dp, W_upp, shared = host_latent_dense(wl)
    cache = {}

    def get(e):
        if e not in cache:
            cache[e] = host_latent_expert(wl, e)
        return cache[e]

    return O.latent_tokens(x_codes, w_route, wl.k, W_dp, get, W_upp, shared, wl.beta_gate,
                           wl.beta_up, 1e-6)


def test_forward_shape_and_routing_small():
    wl = small_latent()
    y, outs = _run_gpu(wl)
    assert tuple(y.shape) == (wl.T, wl.d)
    idx, tw, ref = _oracle(wl, np.arange(wl.T))
    assert np.array_equal(outs["top_idx"], idx)
    assert np.allclose(outs["top_w"], tw, rtol=2e-6, atol=1e-7)
    assert outs["counts"].sum() == wl.k * wl.T


def test_matches_an_independent_reference_small():
    wl = small_latent()
    y, _ = _run_gpu(wl)
    _, _, ref = _oracle(wl, np.arange(wl.T))
    assert rel_err(y.float().cpu().numpy(), ref) < TOL_BF16


def test_latent_bottleneck_is_where_routed_experts_live():
    """With W_dp = 0 the routed branch vanishes (x_l = 0 -> m = 0 -> m^ = 0) and
    y equals the shared experts alone; routing (on the full-width x) is unchanged."""
    wl = small_latent(T=96)
    dw = dev_latent(wl)
    y_full, o_full = _run_gpu(wl, dw)
    dw["w_dp"].zero_()
    y0, o0 = _run_gpu(wl, dw)
    assert np.array_equal(o_full["top_idx"], o0["top_idx"])
    _, W_upp, shared = host_latent_dense(wl)
    xd = O.decode(O.BF16, host_u(wl))
    ref = np.array([sum(O.expert(g, u, d, xd[t], round_h=1) for g, u, d in shared)
                    for t in range(wl.T)])
    assert rel_err(y0.float().cpu().numpy(), ref) < TOL_BF16
    assert rel_err(y_full.float().cpu().numpy(), ref) > 0.05  # the routed branch mattered


def expert_cover_tokens(idx, N, seed=5):
    """A few tokens whose top-k sets together contain every expert routed to at
    all: greedy set cover (each step takes the token that adds the most experts
    not yet covered; ties to the lower token index after a seeded shuffle)."""
    rng = np.random.default_rng(seed)
    order = rng.permutation(idx.shape[0])
    sets = [set(idx[t].tolist()) for t in range(idx.shape[0])]
    need = set(idx.ravel().tolist())
    chosen = []
    while need:
        best = max(order, key=lambda t: (len(sets[t] & need), -t))
        chosen.append(int(best))
        need -= sets[best]
    return np.sort(np.array(chosen, dtype=np.int64))


def test_latent_full_size_routing_all_tokens_and_expert_cover():
    """The LatentMoE-shaped layer at full size: T=4096, d=4096, l=3584, 896
    routed experts of hidden 3072, top-16, 2 shared experts.  Routing indices,
    combine weights and per-expert counts against the oracle on all 4096
    tokens; outputs on a set of tokens whose routed experts cover every expert
    that any token selected (each expert generated once on the host)."""
    wl = W.latent()
    y, outs = _run_gpu(wl)
    x_all = host_u(wl)
    w_route = S.normal(wl.seed, W.TID_WROUTE, (wl.N, wl.d), W.SIGMA_W, S.DT_F32)
    _, _, idx, tw = O.route(O.as_f32(O.BF16, x_all), w_route, wl.k)
    assert np.array_equal(outs["top_idx"], idx)
    assert np.allclose(outs["top_w"], tw, rtol=2e-6, atol=1e-7)
    perm = O.permute(idx, wl.N, 0)
    assert np.array_equal(outs["counts"], perm["counts"])
    assert outs["counts"].sum() == wl.k * wl.T
    tokens = expert_cover_tokens(idx, wl.N)
    assert set(idx[tokens].ravel().tolist()) == set(np.nonzero(perm["counts"])[0].tolist())
    W_dp, W_upp, shared = host_latent_dense(wl)
    idx_s, _, ref = O.latent_tokens_expert_major(
        x_all[tokens], w_route, wl.k, W_dp, lambda e: host_latent_expert(wl, e), W_upp, shared,
        wl.beta_gate, wl.beta_up, 1e-6, threads=max(1, min(16, O.threads())))
    assert np.array_equal(idx_s, idx[tokens])
    got = y[torch.from_numpy(tokens).long().cuda()].float().cpu().numpy()
    assert rel_err(got, ref) < TOL_BF16
