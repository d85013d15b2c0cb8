"""GPU parity of the decode-shaped forward (ba_attention_decode) against the
oracle's decode forward: Nq query tokens against an Nk-token cache of packed
key bits, key scales and int8 value codes.  Outputs within max-abs 2e-2 and
mean-abs 2e-3, on the raw errors and on the errors divided by max(1, std of
the value channel), as for the square forward."""
import numpy as np
import pytest

import oracle as O

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import bit_qk_attention_ba_b200 as ba  # noqa: E402
from guard import Guarded  # noqa: E402
from bit_qk_attention_ba_b200 import _native as NAT  # noqa: E402

DEV = torch.device("cuda:0")
MAX_ABS, MEAN_ABS = 2e-2, 2e-3


def _inputs(B, H, Nq, Nk, d, dtype, bias, seed):
    rng = np.random.default_rng(seed)
    off = lambda: rng.standard_normal((H, d)).astype(np.float32) * np.float32(0.5)
    q = (rng.standard_normal((B, H, Nq, d)).astype(np.float32) + off()[None, :, None])
    k = (rng.standard_normal((B, H, Nk, d)).astype(np.float32) + off()[None, :, None])
    v = (rng.standard_normal((B, H, Nk, d)).astype(np.float32) + off()[None, :, None])
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    q, k, v = (torch.from_numpy(x).to(tdt) for x in (q, k, v))
    b = None
    if bias:
        ld = (Nk + 3) // 4 * 4
        b = np.zeros((H, Nq, ld), np.float32)
        b[:, :, :Nk] = rng.standard_normal((H, Nq, Nk)).astype(np.float32) * np.float32(0.3)
    return q, k, v, b


def _run(q, k, v, b, d):
    bq, muq = ba.pack_qk(q.to(DEV))
    bk, muk = ba.pack_qk(k.to(DEV))
    vq, sv = ba.quant_v(v.to(DEV))
    bt = None if b is None else torch.from_numpy(b).to(DEV)
    guard = Guarded()
    B, H, Nq = muq.shape
    out = ba.attention_decode(bq, muq, bk, muk, vq, sv, d, bias=bt,
                              out=guard.empty((B, H, Nq, d), torch.float32, DEV))
    torch.cuda.synchronize()
    guard.check()
    return out.cpu().numpy()


def _check(got, q, k, v, b):
    Nk = k.shape[2]
    ref = O.decode_forward(q.float().numpy(), k.float().numpy(), v.float().numpy(), b, 0 if b is None else b.shape[-1])
    raw = np.abs(got.astype(np.float64) - ref)
    assert np.isfinite(got).all()
    assert raw.max() <= MAX_ABS and raw.mean() <= MEAN_ABS, ("raw", raw.max(), raw.mean(), Nk)
    scale = np.maximum(1.0, v.float().numpy().astype(np.float64).std(axis=2, keepdims=True))
    err = raw / scale
    assert err.max() <= MAX_ABS and err.mean() <= MEAN_ABS, (err.max(), err.mean(), Nk)


SHAPES = [
    # B, H, Nq, Nk, d, dtype, dense bias
    (1, 2, 1, 1, 64, "bf16", False),
    (2, 3, 1, 300, 64, "bf16", True),
    (1, 2, 4, 5000, 64, "bf16", True),
    (1, 1, 16, 4097, 128, "f32", False),
    (2, 2, 3, 777, 72, "bf16", True),
    (1, 2, 7, 2049, 32, "f32", True),
    (1, 1, 2, 70001, 64, "bf16", False),
    (3, 1, 16, 33, 1, "f32", True),
    # one query row (the kernels' one-row instances) for every sign-word count
    (1, 2, 1, 4097, 128, "f32", True),
    (2, 2, 1, 777, 72, "bf16", False),
    (1, 3, 1, 20000, 32, "bf16", True),
    (2, 1, 1, 33, 1, "f32", False),
]


@pytest.mark.parametrize("shape", SHAPES, ids=["x".join(map(str, s[:5])) + s[5] + ("b" if s[6] else "") for s in SHAPES])
def test_decode_matches_oracle(shape):
    B, H, Nq, Nk, d, dtype, bias = shape
    q, k, v, b = _inputs(B, H, Nq, Nk, d, dtype, bias, seed=Nk + d)
    got = _run(q, k, v, b, d)
    _check(got, q, k, v, b)
    assert ba.check_device_status() == 0


def test_decode_dominant_bias_selects_cached_value():
    """A +100 bias entry per query row picks one cached key, also across
    split boundaries (Nk spans several splits)."""
    B, H, Nq, Nk, d = 1, 2, 5, 6000, 64
    q, k, v, b = _inputs(B, H, Nq, Nk, d, "bf16", True, seed=5)
    picks = [0, 2047, 2048, 4500, Nk - 1]
    b[:] = 0.0
    for i, j in enumerate(picks):
        b[:, i, j] = 100.0
    got = _run(q, k, v, b, d)
    vq, sv = O.quant_v(v.float().numpy().reshape(H, Nk, d))
    for i, j in enumerate(picks):
        np.testing.assert_allclose(got[0, :, i], vq[:, j].astype(np.float64) * sv, rtol=1e-5, atol=1e-6)


def test_decode_row_equals_square_forward_row():
    """Decoding the first Nq tokens of a square problem's queries against all
    of its keys gives the square forward's first Nq rows (the fused square
    kernel, through the same C ABI), within rounding of either path."""
    B, H, N, d, Nq = 2, 2, 300, 64, 4
    q, k, v, _ = _inputs(B, H, N, N, d, "bf16", False, seed=11)
    qd, kd, vd = (x.to(DEV) for x in (q, k, v))
    sq = ba.forward(qd, kd, vd, out_dtype=torch.float32).cpu().numpy()[:, :, :Nq]
    dec = _run(q[:, :, :Nq].contiguous(), k, v, None, d)
    np.testing.assert_allclose(dec, sq, rtol=0, atol=2e-3)
