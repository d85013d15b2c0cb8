"""GPU parity of the training-side backward (ba_attention_bwd, Key design 4 of
the BA notes: straight-through estimators) against the oracle's backward.

Tolerance, from the arithmetic: the GPU forms scores, P and the dot products
in fp32 (relative error ~1e-6 of each gradient's scale after summing at most a
few thousand terms), and takes D_i = dO_i . O_i from the GPU forward output,
which matches the oracle's to ~1e-6.  A u8 code of P~ sitting on a rounding
boundary can round the other way in fp32: that moves dv_j by at most
|dO_i| / (255 l_i) <= max|dO| / 255.  So per gradient tensor: max-abs error
<= 2e-3 max|reference| (plus max|dO| / 255 for dv), mean-abs error <= 2e-4
max|reference|, each plus 1e-5 for the fp32 rounding of dO.V^ - D where the
exact gradient vanishes (with one key, dS is zero in exact arithmetic).
"""
import numpy as np
import pytest

import oracle as O
from bit_qk_attention_ba_b200.workloads import BIAS_KIND, Workload, make_inputs

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import bit_qk_attention_ba_b200 as ba  # noqa: E402
from guard import Guarded  # noqa: E402

DEV = torch.device("cuda:0")


def _run(w, inp, dO, clip):
    tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    q, k, v = (torch.from_numpy(inp[n]).to(tdt).to(DEV) for n in ("q", "k", "v"))
    bias = None if inp["bias"] is None else torch.from_numpy(inp["bias"]).to(DEV)
    kind = BIAS_KIND[w.bias]
    bq, muq, bk, muk, vq, sv = ba.prepass_qkv(q, k, v)
    out = ba.attention_fwd(bq, muq, bk, muk, vq, sv, w.d, bias=bias, bias_kind=kind, ld=inp["ld"], grid=w.grid,
                           out_dtype=torch.float32)
    g = torch.from_numpy(dO.astype(np.float32)).to(DEV)
    guard = Guarded()
    shape = (w.B, w.H, w.N, w.d)
    grads = (guard.empty(shape, torch.float32, DEV), guard.empty(shape, torch.float32, DEV),
             guard.empty(shape, torch.float32, DEV),
             None if bias is None else guard.empty(tuple(bias.shape), torch.float32, DEV))
    dq, dk, dv, db = ba.attention_bwd(q, k, bq, muq, bk, muk, vq, sv, out, g, bias=bias, bias_kind=kind,
                                      ld=inp["ld"], grid=w.grid, ste_clip=clip, grads=grads)
    torch.cuda.synchronize()
    guard.check()
    assert ba.check_device_status() == 0
    to = lambda t: None if t is None else t.cpu().numpy().astype(np.float64)
    return dict(dq=to(dq), dk=to(dk), dv=to(dv), dbias=to(db))


def _oracle(w, inp, dO, clip):
    gh, gw = w.grid
    # the oracle reads the values the GPU saw: bf16-rounded inputs
    r = lambda a: torch.from_numpy(a).to(torch.bfloat16).float().numpy() if w.dtype == "bf16" else a
    return O.attention_bwd(r(inp["q"]), r(inp["k"]), r(inp["v"]), dO, BIAS_KIND[w.bias], inp["bias"], inp["ld"],
                           gh, gw, ste_clip=clip)


FLOOR = 1e-5          # fp32 rounding of dO.V^ - D where the exact gradient is 0 (unit-scale inputs)


def _check(got, want, dO, name, extra=0.0):
    scale = np.abs(want).max()
    err = np.abs(got - want)
    assert np.isfinite(got).all(), name
    assert err.max() <= 2e-3 * scale + extra + FLOOR, (name, err.max(), scale)
    assert err.mean() <= 2e-4 * scale + FLOOR, (name, err.mean(), scale)


SHAPES = [
    # name, B, H, N, d, dtype, bias, grid, clip
    ("dense_ragged", 2, 2, 77, 64, "bf16", "dense", (0, 0), float("inf")),
    ("none_d72_clip", 1, 2, 50, 72, "f32", "none", (0, 0), 1.0),
    ("relpos", 1, 2, 48, 32, "bf16", "relpos2d", (6, 8), float("inf")),
    ("relpos_cls", 2, 1, 37, 64, "f32", "relpos2d_cls", (4, 9), 1.5),
    ("d128", 1, 1, 40, 128, "bf16", "dense", (0, 0), float("inf")),
    ("n1", 2, 2, 1, 64, "f32", "dense", (0, 0), float("inf")),
    ("d1", 1, 1, 33, 1, "f32", "none", (0, 0), float("inf")),
]


@pytest.mark.parametrize("spec", SHAPES, ids=[s[0] for s in SHAPES])
def test_backward_matches_oracle(spec):
    name, B, H, N, d, dtype, bias, grid, clip = spec
    w = Workload(name, B, H, N, d, dtype=dtype, bias=bias, grid=grid, bias_std=0.3)
    inp = make_inputs(w)
    dO = np.random.default_rng(4).standard_normal((B, H, N, d))
    got = _run(w, inp, dO, clip)
    want = _oracle(w, inp, dO, clip)
    dmax = np.abs(dO).max()
    _check(got["dq"], want["dq"], dO, "dq")
    _check(got["dk"], want["dk"], dO, "dk")
    _check(got["dv"], want["dv"], dO, "dv", extra=dmax / 255.0)
    if bias != "none":
        wb = want["dbias"]
        gb = got["dbias"]
        if bias == "dense":
            assert not gb[:, :, N:].any()
            gb, wb = gb[:, :, :N], wb[:, :, :N]
        _check(gb, wb, dO, "dbias")
    if N == 1:      # P = 1 whatever the scores: no gradient reaches q or k beyond rounding
        assert np.abs(got["dq"]).max() <= FLOOR and np.abs(got["dk"]).max() <= FLOOR


def test_backward_deit_s_shape_with_outliers():
    """A DeiT-S-shaped head set with x8 outlier channels (peaked rows)."""
    w = Workload("bwd_s", 4, 6, 197, 64, outlier_frac=0.02)
    inp = make_inputs(w)
    dO = np.random.default_rng(8).standard_normal((w.B, w.H, w.N, w.d))
    got = _run(w, inp, dO, float("inf"))
    want = _oracle(w, inp, dO, float("inf"))
    _check(got["dq"], want["dq"], dO, "dq")
    _check(got["dk"], want["dk"], dO, "dk")
    _check(got["dv"], want["dv"], dO, "dv", extra=np.abs(dO).max() / 255.0)
    _check(got["dbias"][:, :, :w.N], want["dbias"][:, :, :w.N], dO, "dbias")
