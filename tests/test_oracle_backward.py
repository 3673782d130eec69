"""Pins of the oracle's layer backward (CPU only).

The backward is the gradient of L = sum dy . y (+ alpha N sum f_i P_i) with the
selected sets and the capacity drops held fixed ("Mixture of Experts MoE: how
sparse activation saves compute" §3.1, §3.2, §3.4 and §3.7; the Stable LatentMoE
demo document's check that only the selected experts receive gradient).  It is
pinned to things other than itself:

* torch autograd in float64 over an independent torch statement of the forward;
* central finite differences of the oracle's own loss (whose forward is pinned
  to the already-pinned routing and expert functions below);
* closed forms: Euler's identity for the parameters the output is linear in,
  the softmax's shift invariance, k = 1 with renormalisation (a == 1, so the
  router only sees the balancing term of §3.7), dy = 0;
* sparsity: experts with no kept dispatch get exactly zero gradient.
"""
import numpy as np
import pytest
import torch

import oracle

BG, BU = 4.0, 25.0


def _case(seed, T=10, d=12, h=16, N=5, k=2, C=0, scale=0.4):
    rng = np.random.default_rng(seed)
    Wg = rng.normal(0, scale, (N, h, d))
    Wu = rng.normal(0, scale, (N, h, d))
    Wd = rng.normal(0, scale, (N, d, h))
    Wr = rng.normal(0, 0.6, (N, d))
    u = rng.normal(0, 1.0, (T, d))
    z = u @ Wr.T
    idx = np.argsort(-z, axis=1, kind="stable")[:, :k].astype(np.int32)
    row_of = oracle.permute(idx, N, C)["row_of"] if C else None
    dy = rng.normal(0, 1.0, (T, d))
    f = rng.dirichlet(np.ones(N))
    return dict(Wg=Wg, Wu=Wu, Wd=Wd, Wr=Wr, u=u, z=z, idx=idx, row_of=row_of, dy=dy, f=f, k=k)


def _mats(W):
    return [oracle.Mat(oracle.F64, W.shape[1], W.shape[2], data=W[e]) for e in range(W.shape[0])]


def _oracle(c, renorm, act, alpha, use_wr=True):
    kw = dict(Wr=c["Wr"] if use_wr else None, z=None if use_wr else c["z"], row_of=c["row_of"],
              renorm=renorm, act=act, beta_g=BG, beta_u=BU, alpha=alpha,
              f=c["f"] if alpha else None)
    args = (_mats(c["Wg"]), _mats(c["Wu"]), _mats(c["Wd"]), c["u"], c["idx"], c["dy"])
    return oracle.layer_loss(*args, **kw), oracle.layer_backward(*args, **kw)


def _torch_grads(c, renorm, act, alpha, use_wr=True):
    """The same loss stated with torch tensor ops; gradients by autograd."""
    t = {n: torch.tensor(c[n], dtype=torch.float64, requires_grad=True)
         for n in ("Wg", "Wu", "Wd", "Wr", "u", "z")}
    idx = torch.tensor(c["idx"], dtype=torch.long)
    N = c["z"].shape[1]
    if use_wr:
        z = t["u"] @ t["Wr"].T
        z.retain_grad()
    else:
        z = t["z"]
    p = torch.softmax(z, dim=1)
    ps = torch.gather(p, 1, idx)
    a = ps / ps.sum(1, keepdim=True) if renorm else ps
    if c["row_of"] is not None:
        a = a * torch.tensor(c["row_of"] >= 0, dtype=torch.float64)
    g = torch.einsum("tkhd,td->tkh", t["Wg"][idx], t["u"])
    v = torch.einsum("tkhd,td->tkh", t["Wu"][idx], t["u"])
    if act == 1:
        g = BG * torch.tanh(g / BG)
        v = BU * torch.tanh(v / BU)
    H = torch.nn.functional.silu(g) * v
    F = torch.einsum("tkmh,tkh->tkm", t["Wd"][idx], H)
    y = (a.unsqueeze(-1) * F).sum(1)
    L = (torch.tensor(c["dy"]) * y).sum()
    if alpha:
        L = L + alpha * N * (torch.tensor(c["f"]) * p.mean(0)).sum()
    L.backward()
    out = {n: t[n].grad.numpy() for n in ("Wg", "Wu", "Wd", "u")}
    out["Wr"] = t["Wr"].grad.numpy() if use_wr else None
    out["z"] = z.grad.numpy()
    return float(L.detach()), y.detach().numpy(), out


def _close(a, b, rel=1e-11):
    scale = max(np.abs(b).max(), 1e-300)
    assert np.abs(a - b).max() <= rel * scale, (np.abs(a - b).max(), scale)


@pytest.mark.parametrize("act", [0, 1])
@pytest.mark.parametrize("renorm", [1, 0])
@pytest.mark.parametrize("C,alpha,use_wr", [(0, 0.0, True), (3, 0.0, True), (3, 0.01, True),
                                            (4, 0.02, False)])
def test_backward_matches_autograd(act, renorm, C, alpha, use_wr):
    c = _case(11 + C + act, C=C)
    if C:
        assert (c["row_of"] < 0).any(), "the case should drop some dispatches"
    (L, y), g = _oracle(c, renorm, act, alpha, use_wr)
    tL, ty, tg = _torch_grads(c, renorm, act, alpha, use_wr)
    assert abs(L - tL) <= 1e-12 * max(1.0, abs(tL))
    _close(y, ty)
    _close(g["dWg"], tg["Wg"])
    _close(g["dWu"], tg["Wu"])
    _close(g["dWd"], tg["Wd"])
    _close(g["du"], tg["u"])
    _close(g["dz"], tg["z"])
    if use_wr:
        _close(g["dWr"], tg["Wr"])
    else:
        assert g["dWr"] is None


def test_backward_central_differences():
    """Every input's gradient against central differences of the oracle's loss
    at sampled entries (step 1e-5: truncation ~1e-10, rounding ~1e-11)."""
    c = _case(5, T=6, d=8, h=12, N=4, k=2, C=3)
    renorm, act, alpha = 1, 1, 0.05
    _, g = _oracle(c, renorm, act, alpha)
    rng = np.random.default_rng(3)
    eps = 1e-5

    def loss(cc):
        return _oracle(cc, renorm, act, alpha)[0][0]

    for name, gname in (("Wg", "dWg"), ("Wu", "dWu"), ("Wd", "dWd"), ("Wr", "dWr"), ("u", "du")):
        G = g[gname]
        nz = np.argwhere(np.abs(G) > 1e-3 * np.abs(G).max())
        picks = nz[rng.choice(len(nz), size=min(12, len(nz)), replace=False)]
        for pos in map(tuple, picks):
            cp, cm = dict(c), dict(c)
            cp[name] = c[name].copy()
            cm[name] = c[name].copy()
            cp[name][pos] += eps
            cm[name][pos] -= eps
            fd = (loss(cp) - loss(cm)) / (2 * eps)
            assert abs(fd - G[pos]) <= 1e-6 * np.abs(G).max(), (name, pos, fd, G[pos])
    # the logits directly (router given as z)
    _, gz = _oracle(c, renorm, act, alpha, use_wr=False)
    for pos in [(0, 0), (1, 2), (3, 1), (5, 3)]:
        cp, cm = dict(c), dict(c)
        cp["z"] = c["z"].copy()
        cm["z"] = c["z"].copy()
        cp["z"][pos] += eps
        cm["z"][pos] -= eps
        fd = (_oracle(cp, renorm, act, alpha, False)[0][0] -
              _oracle(cm, renorm, act, alpha, False)[0][0]) / (2 * eps)
        assert abs(fd - gz["dz"][pos]) <= 1e-6 * np.abs(gz["dz"]).max()


def test_loss_forward_is_the_pinned_forward():
    """With dyadic inputs the fp32 router chain is exact, so the double logits
    of the loss equal the routing oracle's; the loss's y must then equal the
    pinned routing + expert path (route, permute, moe_tokens)."""
    rng = np.random.default_rng(9)
    T, d, h, N, k = 12, 16, 8, 6, 2
    u = rng.integers(-32, 33, (T, d)) / 8.0
    Wr = rng.integers(-32, 33, (N, d)) / 16.0
    W = [rng.normal(0, 0.3, (N, h, d)), rng.normal(0, 0.3, (N, h, d)), rng.normal(0, 0.3, (N, d, h))]
    logits, _, idx, tw = oracle.route(u.astype(np.float32), Wr.astype(np.float32), k)
    assert np.array_equal(logits.astype(np.float64), u @ Wr.T)
    row_of = oracle.permute(idx, N, 3)["row_of"]
    mats = [_mats(x) for x in W]
    y_ref = oracle.moe_tokens(*mats, u, idx, tw, row_of=row_of)
    dy = np.zeros((T, d))
    for renorm in (1,):
        _, y = oracle.layer_loss(*mats, u, idx, dy, Wr=Wr, row_of=row_of, renorm=renorm)
        _close(y, y_ref, rel=1e-14)


def test_only_selected_experts_receive_gradient():
    """Stable LatentMoE demo document: gradients reach only the selected experts.
    Expert 4 is never selected; expert 3 is selected only by dropped dispatches."""
    c = _case(21, T=8, d=8, h=8, N=5, k=2)
    c["idx"][:, 0] = np.arange(8) % 3
    c["idx"][:, 1] = np.where(np.arange(8) % 2 == 0, 3, (np.arange(8) + 1) % 3)
    row_of = np.zeros((8, 2), np.int32)
    row_of[:, 1] = np.where(c["idx"][:, 1] == 3, -1, 0)
    c["row_of"] = row_of
    for act in (0, 1):
        _, g = _oracle(c, 1, act, 0.0)
        for e in (3, 4):
            for n in ("dWg", "dWu", "dWd"):
                assert not g[n][e].any(), (n, e)
        for e in (0, 1, 2):
            assert np.abs(g["dWd"][e]).max() > 0


def test_euler_identities_and_shift_invariance():
    """y is linear in W_down (and in W_up without the soft caps), so
    sum(dW * W) equals the loss's dy . y term; the softmax is invariant to a
    shift of a token's logits, so each row of dz sums to zero."""
    c = _case(31, C=3)
    for act in (0, 1):
        (L, _), g = _oracle(c, 1, act, 0.0)
        _close(np.array([np.sum(g["dWd"] * c["Wd"])]), np.array([L]), rel=1e-12)
        if act == 0:
            _close(np.array([np.sum(g["dWu"] * c["Wu"])]), np.array([L]), rel=1e-12)
        assert np.abs(g["dz"].sum(1)).max() <= 1e-14 * np.abs(g["dz"]).max() * c["z"].shape[1]


def test_top1_renormalised_router_sees_only_the_balancing_term():
    """k = 1 with renormalisation gives a == 1 (tutorial §3.2's caveat for
    top-1), so dy reaches no logit; with the balancing term dz is exactly the
    closed form of §3.7."""
    c = _case(41, k=1)
    z32 = c["z"].astype(np.float32)
    c["z"] = z32.astype(np.float64)
    probs, _, _ = oracle.route_from_logits(z32, 1)
    _, g0 = _oracle(c, 1, 0, 0.0, use_wr=False)
    assert not g0["dz"].any()
    _, g1 = _oracle(c, 1, 0, 0.3, use_wr=False)
    assert np.array_equal(g1["dz"], oracle.aux_grad(probs, c["f"], 0.3))


def test_zero_upstream_gradient():
    c = _case(51, C=4)
    c["dy"] = np.zeros_like(c["dy"])
    _, g = _oracle(c, 1, 1, 0.1)
    for n in ("dWg", "dWu", "dWd"):
        assert not g[n].any()
    probs = np.exp(c["z"] - c["z"].max(1, keepdims=True))
    probs /= probs.sum(1, keepdims=True)
    _close(g["dz"], oracle.aux_grad(probs, c["f"], 0.1), rel=1e-13)
    _close(g["du"], g["dz"] @ c["Wr"], rel=1e-13)
    _close(g["dWr"], g["dz"].T @ c["u"], rel=1e-13)


# ----------------------------------------------------------- LatentMoE layer
LD, LL, LH, LN, LK, LSH, NSH = 12, 8, 10, 6, 2, 14, 2


def _latent_case(seed, renorm=1):
    rng = np.random.default_rng(seed)
    c = dict(Wg=rng.normal(0, 0.5, (LN, LH, LL)), Wu=rng.normal(0, 0.5, (LN, LH, LL)),
             Wd=rng.normal(0, 0.5, (LN, LL, LH)), Wr=rng.normal(0, 0.6, (LN, LD)),
             Wdp=rng.normal(0, 0.4, (LL, LD)), Wupp=rng.normal(0, 0.4, (LD, LL)),
             Sg=rng.normal(0, 0.3, (NSH, LSH, LD)), Su=rng.normal(0, 0.3, (NSH, LSH, LD)),
             Sd=rng.normal(0, 0.3, (NSH, LD, LSH)), x=rng.normal(0, 1.0, (7, LD)),
             dy=rng.normal(0, 1.0, (7, LD)), renorm=renorm)
    z = c["x"] @ c["Wr"].T
    c["idx"] = np.argsort(-z, axis=1, kind="stable")[:, :LK].astype(np.int32)
    return c


def _m64(a):
    return oracle.Mat(oracle.F64, a.shape[0], a.shape[1], data=a)


def _latent(c, eps, fn):
    routed = (_mats(c["Wg"]), _mats(c["Wu"]), _mats(c["Wd"]))
    shared = [(_m64(c["Sg"][j]), _m64(c["Su"][j]), _m64(c["Sd"][j])) for j in range(NSH)]
    return fn(routed, c["Wr"], _m64(c["Wdp"]), _m64(c["Wupp"]), shared, c["x"], c["idx"],
              c["dy"], BG, BU, eps=eps, renorm=c["renorm"])


def _latent_torch(c, eps):
    t = {n: torch.tensor(c[n], dtype=torch.float64, requires_grad=True)
         for n in ("Wg", "Wu", "Wd", "Wr", "Wdp", "Wupp", "Sg", "Su", "Sd", "x")}
    idx = torch.tensor(c["idx"], dtype=torch.long)
    x = t["x"]
    z = x @ t["Wr"].T
    z.retain_grad()
    p = torch.softmax(z, dim=1)
    ps = torch.gather(p, 1, idx)
    a = ps / ps.sum(1, keepdim=True) if c["renorm"] else ps
    xl = x @ t["Wdp"].T
    g = BG * torch.tanh(torch.einsum("tkhl,tl->tkh", t["Wg"][idx], xl) / BG)
    v = BU * torch.tanh(torch.einsum("tkhl,tl->tkh", t["Wu"][idx], xl) / BU)
    F = torch.einsum("tkmh,tkh->tkm", t["Wd"][idx], torch.nn.functional.silu(g) * v)
    m = (a.unsqueeze(-1) * F).sum(1)
    mh = m / torch.sqrt((m * m).mean(1, keepdim=True) + eps)
    y = mh @ t["Wupp"].T
    for j in range(NSH):
        hs = torch.nn.functional.silu(x @ t["Sg"][j].T) * (x @ t["Su"][j].T)
        y = y + hs @ t["Sd"][j].T
    L = (torch.tensor(c["dy"]) * y).sum()
    L.backward()
    out = {n: t[n].grad.numpy() for n in t}
    out["z"] = z.grad.numpy()
    return float(L.detach()), y.detach().numpy(), out


@pytest.mark.parametrize("renorm", [1, 0])
@pytest.mark.parametrize("eps", [1e-6, 0.3])
def test_latent_backward_matches_autograd(renorm, eps):
    c = _latent_case(61 + renorm, renorm)
    L, y = _latent(c, eps, oracle.latent_loss)
    g = _latent(c, eps, oracle.latent_backward)
    tL, ty, tg = _latent_torch(c, eps)
    assert abs(L - tL) <= 1e-12 * max(1.0, abs(tL))
    _close(y, ty)
    for ours, theirs in (("dz", "z"), ("dx", "x"), ("dWr", "Wr"), ("dWdp", "Wdp"),
                         ("dWupp", "Wupp"), ("dWg", "Wg"), ("dWu", "Wu"), ("dWd", "Wd"),
                         ("dSg", "Sg"), ("dSu", "Su"), ("dSd", "Sd")):
        _close(g[ours], tg[theirs])


def test_latent_loss_forward_is_the_pinned_pieces():
    """The loss's forward composed from the pinned oracle pieces: the matvec,
    the SiTU-GLU expert, RMSNorm and numpy's softmax."""
    c = _latent_case(71)
    eps = 1e-6
    _, y = _latent(c, eps, oracle.latent_loss)
    for t in range(c["x"].shape[0]):
        z = c["Wr"] @ c["x"][t]
        p = np.exp(z - z.max())
        p /= p.sum()
        sel = c["idx"][t]
        a = p[sel] / p[sel].sum()
        xl = oracle.matvec(_m64(c["Wdp"]), c["x"][t])
        m = sum(a[s] * oracle.expert(_m64(c["Wg"][e]), _m64(c["Wu"][e]), _m64(c["Wd"][e]), xl,
                                     act=1, beta_g=BG, beta_u=BU) for s, e in enumerate(sel))
        yt = oracle.matvec(_m64(c["Wupp"]), oracle.rmsnorm(m, eps))
        for j in range(NSH):
            yt = yt + oracle.expert(_m64(c["Sg"][j]), _m64(c["Su"][j]), _m64(c["Sd"][j]), c["x"][t])
        _close(y[t], yt, rel=1e-13)


def test_latent_backward_central_differences():
    c = _latent_case(81)
    eps = 1e-6
    g = _latent(c, eps, oracle.latent_backward)
    rng = np.random.default_rng(4)
    h = 1e-5
    for name, gname in (("Wg", "dWg"), ("Wd", "dWd"), ("Wr", "dWr"), ("Wdp", "dWdp"),
                        ("Wupp", "dWupp"), ("Sd", "dSd"), ("x", "dx")):
        G = g[gname]
        nz = np.argwhere(np.abs(G) > 1e-3 * np.abs(G).max())
        for pos in map(tuple, nz[rng.choice(len(nz), size=min(8, len(nz)), replace=False)]):
            cp, cm = dict(c), dict(c)
            cp[name], cm[name] = c[name].copy(), c[name].copy()
            cp[name][pos] += h
            cm[name][pos] -= h
            fd = (_latent(cp, eps, oracle.latent_loss)[0] -
                  _latent(cm, eps, oracle.latent_loss)[0]) / (2 * h)
            assert abs(fd - G[pos]) <= 1e-6 * np.abs(G).max(), (name, pos, fd, G[pos])


def test_latent_only_selected_experts_receive_gradient():
    """Stable LatentMoE demo document, forward-contract tab: only the selected
    routed experts receive gradient."""
    c = _latent_case(91)
    c["idx"][:, 0] = 0
    c["idx"][:, 1] = np.where(np.arange(7) % 2 == 0, 1, 2)
    g = _latent(c, 1e-6, oracle.latent_backward)
    for e in range(LN):
        used = e in (0, 1, 2)
        for n in ("dWg", "dWu", "dWd"):
            assert bool(np.abs(g[n][e]).max() > 0) == used, (n, e)


def test_latent_rmsnorm_makes_the_routed_scale_a_null_direction():
    """Stable LatentMoE demo document, RMSNorm tab: with RMSNorm before the
    up-projection the output does not depend on the routed experts' scale.
    With eps = 0, y(c W_down) = y(W_down) for every c > 0, so the derivative
    along W_down itself, sum(dW_down * W_down), is zero; W_upp and the shared
    W_down enter linearly, so their Euler sums add up to the loss."""
    c = _latent_case(101)
    L, _ = _latent(c, 0.0, oracle.latent_loss)
    g = _latent(c, 0.0, oracle.latent_backward)
    scale = np.abs(g["dWd"]).max() * np.abs(c["Wd"]).max() * c["Wd"].size
    assert abs(np.sum(g["dWd"] * c["Wd"])) <= 1e-12 * scale
    euler = np.sum(g["dWupp"] * c["Wupp"]) + np.sum(g["dSd"] * c["Sd"])
    assert abs(euler - L) <= 1e-12 * max(1.0, abs(L))
    # with a positive eps the scale is no longer a null direction
    g2 = _latent(c, 0.3, oracle.latent_backward)
    assert abs(np.sum(g2["dWd"] * c["Wd"])) > 1e-6
