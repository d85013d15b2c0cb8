"""Pins for the oracle's backward pass (Key design 4 of the BA notes: QAT with
a straight-through estimator for sign; paper-notes page "BinaryAttention:
One-Bit QK-Attention for Vision and Diffusion Transformers", CVPR 2026).

What pins it, none of it the oracle's own formula:
  - central finite differences of the un-quantised core (softmax attention
    on continuous s, t, mu, V and bias), which is smooth;
  - finite differences of the whole forward in q with the sign pattern held
    fixed, which isolates the mean-|x| scale path;
  - torch autograd (float64) of the quantised forward written with
    straight-through quantisers, an independent reverse-mode derivation;
  - special cases: one key (no gradient reaches q or k), clip = 0 (only the
    scale path), the bias gradient of a rel-pos table against the dense
    expansion.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")


def _rng(seed):
    return np.random.default_rng(seed)


def _loss_core(oracle, s, t, muq, muk, vh, b, dO):
    r = oracle.bwd_core(s, t, muq, muk, vh, b, dO, quantise_p=False)
    return float((r["O"] * dO).sum())


@pytest.mark.parametrize("N,d", [(5, 3), (7, 4)])
def test_core_gradients_match_finite_differences(oracle, N, d):
    rng = _rng(N * 10 + d)
    s, t, vh, dO = (rng.standard_normal((N, d)) for _ in range(4))
    muq, muk = rng.uniform(0.5, 1.5, N), rng.uniform(0.5, 1.5, N)
    b = rng.standard_normal((N, N)) * 0.3
    g = oracle.bwd_core(s, t, muq, muk, vh, b, dO, quantise_p=False)
    eps = 1e-6
    args = dict(s=s, t=t, muq=muq, muk=muk, vh=vh, b=b)
    grads = dict(s="ds", t="dt", muq="dmuq", muk="dmuk", vh="dvh", b="dbias")
    for name, gname in grads.items():
        x = args[name]
        fd = np.zeros_like(x)
        for idx in np.ndindex(*x.shape):
            xp, xm = x.copy(), x.copy()
            xp[idx] += eps
            xm[idx] -= eps
            lp = _loss_core(oracle, **{**args, name: xp}, dO=dO)
            lm = _loss_core(oracle, **{**args, name: xm}, dO=dO)
            fd[idx] = (lp - lm) / (2 * eps)
        np.testing.assert_allclose(g[gname], fd, rtol=1e-5, atol=1e-7, err_msg=name)


def test_scale_path_matches_finite_differences_in_q(oracle):
    """clip = 0 keeps only the mean-|x| path of dq; with the sign pattern
    fixed (no entry within eps of 0) that is the true derivative of the
    un-quantised forward in q."""
    rng = _rng(3)
    B, H, N, d = 1, 1, 6, 5
    q, k, v = (rng.standard_normal((B, H, N, d)).astype(np.float32) for _ in range(3))
    q[np.abs(q) < 0.05] = 0.3
    dO = rng.standard_normal((B, H, N, d))
    r = oracle.attention_bwd(q, k, v, dO, ste_clip=0.0, quantise=False)
    eps = 1e-3            # fp32 inputs: a step well above their rounding
    fd = np.zeros_like(q, dtype=np.float64)
    for idx in np.ndindex(*q.shape):
        qp, qm = q.copy(), q.copy()
        qp[idx] += np.float32(eps)
        qm[idx] -= np.float32(eps)
        step = float(qp[idx]) - float(qm[idx])
        lp = (oracle.attention_bwd(qp, k, v, dO, quantise=False)["O"] * dO).sum()
        lm = (oracle.attention_bwd(qm, k, v, dO, quantise=False)["O"] * dO).sum()
        fd[idx] = (lp - lm) / step
    np.testing.assert_allclose(r["dq"], fd, rtol=1e-4, atol=1e-6)


def _ste(x_value, x):
    """Value of x_value, gradient of x (straight through)."""
    return x + (x_value - x).detach()


def _torch_forward(q, k, v, bias_dense, clip, quantise=True):
    """The method's forward in float64 torch with straight-through quantisers."""
    d = q.shape[-1]
    sq = torch.where(q >= 0, 1.0, -1.0).to(q.dtype)
    sk = torch.where(k >= 0, 1.0, -1.0).to(k.dtype)
    mq = (q.abs() <= clip).to(q.dtype)
    mk = (k.abs() <= clip).to(k.dtype)
    s = _ste(sq, q * mq)
    t = _ste(sk, k * mk)
    muq = q.abs().mean(-1)
    muk = k.abs().mean(-1)
    z = s @ t.transpose(-1, -2)
    S = muq[..., :, None] * muk[..., None, :] * z / np.sqrt(d)
    if bias_dense is not None:
        S = S + bias_dense
    m = S.max(-1, keepdim=True).values.detach()
    Pt = torch.exp(S - m)
    l = Pt.sum(-1, keepdim=True)
    if quantise:
        pq = _ste(torch.round(255.0 * Pt), 255.0 * Pt)     # torch.round: half to even
        # V: per (b, h, channel) absmax / 127 in fp32, codes rint(v / s) in fp32
        v32 = v.detach().float()
        sv = (v32.abs().amax(dim=-2, keepdim=True) / 127.0)
        codes = torch.where(sv > 0, torch.round(v32 / torch.where(sv > 0, sv, torch.ones_like(sv))),
                            torch.zeros_like(v32)).clamp(-127, 127)
        vh = _ste((sv.double() * codes.double()), v)
        return (pq / 255.0) @ vh / l
    return (Pt @ v) / l


@pytest.mark.parametrize("clip", [float("inf"), 1.0])
@pytest.mark.parametrize("bias", ["none", "dense", "relpos", "relpos_cls"])
def test_quantised_backward_matches_torch_autograd(oracle, clip, bias):
    rng = _rng(11)
    B, H, gh, gw, d = 2, 2, 3, 4, 8
    N = gh * gw + (1 if bias == "relpos_cls" else 0)
    q, k, v = (rng.standard_normal((B, H, N, d)).astype(np.float32) for _ in range(3))
    dO = rng.standard_normal((B, H, N, d))
    kind, bias_arr, ld, dense = 0, None, 0, None
    if bias == "dense":
        kind, ld = 1, N + 3
        bias_arr = np.zeros((H, N, ld), np.float32)
        bias_arr[:, :, :N] = rng.standard_normal((H, N, N)).astype(np.float32) * 0.5
        dense = bias_arr[:, :, :N].astype(np.float64)
    elif bias in ("relpos", "relpos_cls"):
        kind = 2 if bias == "relpos" else 3
        G = (2 * gh - 1) * (2 * gw - 1) + (3 if kind == 3 else 0)
        bias_arr = (rng.standard_normal((H, G)) * 0.5).astype(np.float32)
        dense = np.zeros((H, N, N))
        for h in range(H):
            for i in range(N):
                for j in range(N):
                    dense[h, i, j] = oracle.bias_value(kind, bias_arr, 0, h, N, gh, gw, i, j)
    r = oracle.attention_bwd(q, k, v, dO, kind, bias_arr, ld, gh, gw, ste_clip=clip)
    tq, tk, tv = (torch.tensor(x.astype(np.float64), requires_grad=True) for x in (q, k, v))
    tb = None
    if dense is not None:
        tb = torch.tensor(dense, requires_grad=True)
    O = _torch_forward(tq, tk, tv, tb, clip)
    np.testing.assert_allclose(O.detach().numpy(), r["O"], rtol=1e-9, atol=1e-12)
    (O * torch.tensor(dO)).sum().backward()
    for name, t in (("dq", tq), ("dk", tk), ("dv", tv)):
        np.testing.assert_allclose(r[name], t.grad.numpy(), rtol=1e-7, atol=1e-10, err_msg=name)
    if bias == "dense":
        np.testing.assert_allclose(r["dbias"][:, :, :N], tb.grad.numpy(), rtol=1e-7, atol=1e-10)
        assert not r["dbias"][:, :, N:].any()
    if bias == "relpos":
        G = (2 * gh - 1) * (2 * gw - 1)
        want = np.zeros((H, G))
        for h in range(H):
            for i in range(N):
                for j in range(N):
                    ri, ci, rj, cj = i // gw, i % gw, j // gw, j % gw
                    want[h, (ri - rj + gh - 1) * (2 * gw - 1) + (ci - cj + gw - 1)] += tb.grad.numpy()[h, i, j]
        np.testing.assert_allclose(r["dbias"], want, rtol=1e-7, atol=1e-10)
    if bias == "relpos_cls":
        # by hand: the three class entries collect the class row, the class
        # column and the corner; the grid entries collect the patch block
        gd = tb.grad.numpy()
        G = (2 * gh - 1) * (2 * gw - 1)
        want = np.zeros((H, G + 3))
        want[:, G] = gd[:, 0, 1:].sum(-1)
        want[:, G + 1] = gd[:, 1:, 0].sum(-1)
        want[:, G + 2] = gd[:, 0, 0]
        for i in range(1, N):
            for j in range(1, N):
                ri, ci, rj, cj = (i - 1) // gw, (i - 1) % gw, (j - 1) // gw, (j - 1) % gw
                want[:, (ri - rj + gh - 1) * (2 * gw - 1) + (ci - cj + gw - 1)] += gd[:, i, j]
        np.testing.assert_allclose(r["dbias"], want, rtol=1e-7, atol=1e-10)


def test_single_key_passes_no_gradient_to_q_and_k(oracle):
    """N = 1: P = 1 whatever the scores, so dS = 0: dq = dk = 0, dv = dO."""
    rng = _rng(5)
    q, k, v = (rng.standard_normal((2, 3, 1, 16)).astype(np.float32) for _ in range(3))
    dO = rng.standard_normal((2, 3, 1, 16))
    bias = np.zeros((3, 1, 4), np.float32)
    bias[:, 0, 0] = 2.0
    r = oracle.attention_bwd(q, k, v, dO, 1, bias, 4)
    assert np.abs(r["dq"]).max() == 0 and np.abs(r["dk"]).max() == 0
    np.testing.assert_allclose(r["dv"], dO, rtol=1e-15, atol=0)
    assert np.abs(r["dbias"]).max() == 0


def test_clip_only_masks_the_sign_path(oracle):
    """dq(clip) - dq(clip = 0) is the sign path: it vanishes exactly where
    |q| > clip and equals the unclipped sign path elsewhere."""
    rng = _rng(9)
    q, k, v = (rng.standard_normal((1, 2, 9, 8)).astype(np.float32) for _ in range(3))
    dO = rng.standard_normal((1, 2, 9, 8))
    base = oracle.attention_bwd(q, k, v, dO, ste_clip=0.0)["dq"]
    full = oracle.attention_bwd(q, k, v, dO)["dq"] - base
    half = oracle.attention_bwd(q, k, v, dO, ste_clip=0.5)["dq"] - base
    inside = np.abs(q) <= 0.5
    np.testing.assert_allclose(half[inside], full[inside], rtol=1e-12, atol=1e-15)
    assert np.abs(half[~inside]).max() < 1e-15
