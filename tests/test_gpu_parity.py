"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle.

Integer outputs (sign bits, int8 V codes, binary scores) must match bit for
bit.  Floating outputs: mu within fp32 summation error; the attention output
within max-abs 2e-2 and mean-abs 2e-3 of the oracle (exact row max, fp64),
asserted on the raw errors and again on the errors divided by max(1, std of
the value channel) -- the reading of "on unit-scale V" for the x8 outlier
channels of the DeiT-S workload, which the raw check already implies.  The
GPU also takes the exact row maximum (two sweeps over the keys) but computes in
fp32, so a code sitting on a rounding boundary can move by one unit; that is
what the tolerance covers.
"""
import numpy as np
import pytest

import oracle as O
from bit_qk_attention_ba_b200.workloads import BIAS_KIND, WORKLOADS, Workload, make_inputs

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import bit_qk_attention_ba_b200 as ba  # noqa: E402
from bit_qk_attention_ba_b200 import _native as NAT  # noqa: E402
from guard import Guarded  # noqa: E402

DEV = torch.device("cuda:0")
MAX_ABS, MEAN_ABS = 2e-2, 2e-3
TC_VARIANTS = [NAT.BA_QK_TC_I8, NAT.BA_QK_TC_F8]


def _gpu(x, dtype):
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t.to(DEV).to(torch.bfloat16 if dtype == "bf16" else torch.float32).contiguous()


def _bits(t):
    return t.cpu().numpy().view(np.uint32)


def _vq_natural(vq_t, N):
    """GPU layout [B,H,d,ldv] -> oracle layout [BH, N, d]."""
    a = vq_t.cpu().numpy()
    B, H, d, _ = a.shape
    return np.ascontiguousarray(a[..., :N].transpose(0, 1, 3, 2)).reshape(B * H, N, d)


def _assert_close(out_gpu, out_orc, v):
    """Raw errors within the stated bounds, and (implied by it, since the
    scale is at least 1) the errors divided by max(1, std of the value
    channel) as well."""
    raw = np.abs(out_gpu.astype(np.float64) - out_orc)
    assert np.isfinite(out_gpu).all()
    assert raw.max() <= MAX_ABS, "raw max-abs %.3g" % raw.max()
    assert raw.mean() <= MEAN_ABS, "raw mean-abs %.3g" % raw.mean()
    scale = np.maximum(1.0, v.astype(np.float64).std(axis=2, keepdims=True))
    err = raw / scale
    assert err.max() <= MAX_ABS, "max-abs %.3g" % err.max()
    assert err.mean() <= MEAN_ABS, "mean-abs %.3g" % err.mean()
    return err


def _bias_gpu(inp, w):
    return None if inp["bias"] is None else torch.from_numpy(inp["bias"]).to(DEV)


def _run_gpu(w, inp, variant=NAT.BA_QK_AUTO, out_dtype=torch.float32):
    """The benchmarked hot path: the fused pre-pass, then the attention call.
    Every output sits inside guard bytes, checked after the kernels ran."""
    q, k, v = (_gpu(inp[n], w.dtype) for n in ("q", "k", "v"))
    g = Guarded()
    B, H, N, d = w.B, w.H, w.N, w.d
    outs = (g.empty((B, H, N, ba.words(d)), torch.int32, DEV), g.empty((B, H, N), torch.float32, DEV),
            g.empty((B, H, N, ba.words(d)), torch.int32, DEV), g.empty((B, H, N), torch.float32, DEV),
            g.empty((B, H, d, ba.vq_ld(N)), torch.int8, DEV), g.empty((B, H, d), torch.float32, DEV))
    bq, muq, bk, muk, vq, sv = ba.prepass_qkv(q, k, v, outs)
    out = ba.attention_fwd(bq, muq, bk, muk, vq, sv, w.d, bias=_bias_gpu(inp, w),
                           bias_kind=BIAS_KIND[w.bias], ld=inp["ld"], grid=w.grid,
                           out=g.empty((B, H, N, d), out_dtype, DEV), variant=variant)
    torch.cuda.synchronize()
    g.check()
    return dict(bq=bq, muq=muq, bk=bk, muk=muk, vq=vq, sv=sv, out=out)


def _oracle_full(w, inp):
    gh, gw = w.grid
    return O.forward(inp["q"], inp["k"], inp["v"], BIAS_KIND[w.bias], inp["bias"], inp["ld"], gh, gw)


# ------------------------------------------------------------------ pre-passes

@pytest.mark.parametrize("name", list(WORKLOADS))
def test_pack_and_quant_full_size(name):
    w = WORKLOADS[name]
    inp = make_inputs(w)
    BH = w.B * w.H
    for key in ("q", "k"):
        x = _gpu(inp[key], w.dtype)
        bits, mu = ba.pack_qk(x)
        torch.cuda.synchronize()
        ob, om = O.pack(inp[key].reshape(BH, w.N, w.d))
        np.testing.assert_array_equal(_bits(bits).reshape(ob.shape), ob)
        rel = np.abs(mu.cpu().numpy().reshape(om.shape).astype(np.float64) - om) / np.maximum(om, 1e-30)
        assert rel.max() <= w.d * 2.0 ** -24 + 2.0 ** -23
        del x, bits, mu
    v = _gpu(inp["v"], w.dtype)
    vq, sv = ba.quant_v(v)
    torch.cuda.synchronize()
    ovq, osv = O.quant_v(inp["v"].reshape(BH, w.N, w.d))
    np.testing.assert_array_equal(sv.cpu().numpy().reshape(osv.shape), osv)
    np.testing.assert_array_equal(_vq_natural(vq, w.N), ovq)
    assert vq.shape[-1] == ba.vq_ld(w.N)
    assert not vq[..., w.N:].any()


def _check_prepass(w, inp):
    """prepass_qkv against the oracle (bits, codes and scales bit for bit, mu
    within fp32 summation error) and against the separate passes (all six
    outputs bit for bit: they run the same device routines)."""
    BH = w.B * w.H
    q, k, v = (_gpu(inp[n], w.dtype) for n in ("q", "k", "v"))
    fused = ba.prepass_qkv(q, k, v)
    sep = ba.pack_qk(q) + ba.pack_qk(k) + ba.quant_v(v)
    torch.cuda.synchronize()
    for a, b in zip(fused, sep):
        assert torch.equal(a, b)
    for key, bits, mu in (("q", fused[0], fused[1]), ("k", fused[2], fused[3])):
        ob, om = O.pack(inp[key].reshape(BH, w.N, w.d))
        np.testing.assert_array_equal(_bits(bits).reshape(ob.shape), ob)
        rel = np.abs(mu.cpu().numpy().reshape(om.shape).astype(np.float64) - om) / np.maximum(om, 1e-30)
        assert rel.max() <= w.d * 2.0 ** -24 + 2.0 ** -23
    ovq, osv = O.quant_v(inp["v"].reshape(BH, w.N, w.d))
    np.testing.assert_array_equal(fused[5].cpu().numpy().reshape(osv.shape), osv)
    np.testing.assert_array_equal(_vq_natural(fused[4], w.N), ovq)
    assert not fused[4][..., w.N:].any()


@pytest.mark.parametrize("name", list(WORKLOADS))
def test_prepass_fused_full_size(name):
    w = WORKLOADS[name]
    _check_prepass(w, make_inputs(w))


PREPASS_SHAPES = [
    # B, H, N, d, dtype: fused shapes (16-byte vectors per token in {2,4,8,9,12,16}) and fallbacks
    (2, 3, 1, 64, "bf16"), (2, 3, 77, 16, "bf16"), (1, 2, 300, 72, "bf16"), (1, 2, 129, 96, "bf16"),
    (1, 2, 200, 128, "bf16"), (2, 2, 197, 64, "f32"), (1, 2, 50, 36, "f32"), (1, 2, 65, 48, "f32"),
    (1, 1, 90, 8, "f32"), (1, 2, 100, 72, "f32"), (1, 2, 90, 33, "f32"), (1, 1, 1500, 64, "bf16"),
    (1, 2, 2000, 64, "bf16"),
    # 128-byte tokens (the TMA-fed kernel): one box, a unit of two boxes, a
    # one-token unit after it, the largest head whose V it takes whole (1024
    # code columns), one row past that (V absmax apart), and fp32 d = 32
    (3, 2, 577, 64, "bf16"), (1, 3, 128, 64, "bf16"), (1, 3, 256, 64, "bf16"), (1, 2, 257, 64, "bf16"),
    (2, 2, 1024, 64, "bf16"), (1, 2, 1025, 64, "bf16"), (2, 2, 197, 32, "f32"), (1, 1, 5, 32, "f32"),
    (1, 2, 3000, 32, "f32"),
    # 144-byte tokens (nine 16-byte chunks, no swizzle): whole-head V and V
    # absmax apart, bf16 d = 72 and fp32 d = 36
    (2, 2, 577, 72, "bf16"), (1, 3, 1025, 72, "bf16"), (2, 2, 197, 36, "f32"), (1, 1, 3000, 36, "f32"),
    # 256-byte tokens (two swizzled 128-byte rows each): bf16 d = 128 with V's
    # absmax apart, fp32 d = 64 over three units
    (1, 2, 1025, 128, "bf16"), (1, 1, 2000, 64, "f32"),
    # a one-token head for each token width (a 128-row box over one row)
    (1, 2, 1, 72, "bf16"), (1, 2, 1, 64, "f32"), (2, 1, 1, 128, "bf16"),
]


@pytest.mark.parametrize("shape", PREPASS_SHAPES, ids=["x".join(map(str, s)) for s in PREPASS_SHAPES])
def test_prepass_shapes(shape):
    B, H, N, d, dtype = shape
    w = Workload("pp", B, H, N, d, dtype=dtype)
    inp = make_inputs(w)
    inp["q"][0, 0, 0, :] = 0.0          # sign(0) and sign(-0) read as +1
    inp["k"][0, 0, 0, :] = -0.0
    _check_prepass(w, inp)
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    es = 2 if dtype == "bf16" else 4
    nv = d * es // 16 if (d * es) % 16 == 0 else 0
    fits = d * (ba.vq_ld(N) + 4) <= 100 * 1024      # the code tile of one (b, h) in shared memory
    if nv in (8, 9, 16):    # 128-, 144- and 256-byte tokens: one launch up to 1024 code columns, else three
        assert ba.prepass_launches(N, d, tdt) == (1 if ba.vq_ld(N) <= 1024 else 3)
    else:
        assert (ba.prepass_launches(N, d, tdt) == 1) == (nv in (2, 4, 12) and fits)


@pytest.mark.parametrize("N", [300, 5000])
def test_quant_codes_at_rounding_boundaries(N):
    """V values placed on and next to the code boundaries x / s = k + 1/2
    (ties included) for several channel scales s; the codes must match the
    oracle's IEEE fp32 division and round-half-even bit for bit.  N = 300 runs
    the single-pass quantiser, N = 5000 the tiled one."""
    rng = np.random.default_rng(7)
    d = 64
    absmax = np.array([127.0, 12.7, 38.1, 1.0, 0.3, 1e-3, 5e4, 3.0] * 8, np.float32)
    s = (absmax / np.float32(127.0)).astype(np.float32)
    k = rng.integers(-127, 127, size=(N, d)).astype(np.float32)
    delta = rng.choice(np.array([0.0, 1e-7, -1e-7, 1e-6, -1e-6, 1e-5, -1e-5, 1e-4, -1e-4, 3e-3], np.float32),
                       size=(N, d))
    v = ((k + np.float32(0.5) + delta) * s).astype(np.float32)
    v[0] = absmax                      # pin each channel's absmax
    v = np.clip(v, -absmax, absmax).astype(np.float32)
    vt = torch.from_numpy(v.reshape(1, 1, N, d)).to(DEV).contiguous()
    vq, sv = ba.quant_v(vt)
    torch.cuda.synchronize()
    ovq, osv = O.quant_v(v.reshape(1, N, d))
    np.testing.assert_array_equal(sv.cpu().numpy().reshape(osv.shape), osv)
    np.testing.assert_array_equal(_vq_natural(vq, N), ovq)


@pytest.mark.parametrize("d", [1, 31, 33, 72, 96, 128])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_pack_and_quant_odd_d(d, dtype):
    w = Workload("odd", 2, 3, 77, d, dtype=dtype)
    inp = make_inputs(w)
    inp["q"][0, 0, 0, :] = 0.0
    inp["q"][0, 0, 1, :] = -0.0
    bits, mu = ba.pack_qk(_gpu(inp["q"], dtype))
    vq, sv = ba.quant_v(_gpu(inp["v"], dtype))
    torch.cuda.synchronize()
    ob, om = O.pack(inp["q"].reshape(6, 77, d))
    np.testing.assert_array_equal(_bits(bits).reshape(ob.shape), ob)
    np.testing.assert_allclose(mu.cpu().numpy().reshape(om.shape), om, rtol=d * 2.0 ** -24 + 2.0 ** -23)
    ovq, osv = O.quant_v(inp["v"].reshape(6, 77, d))
    np.testing.assert_array_equal(_vq_natural(vq, 77), ovq)
    np.testing.assert_array_equal(sv.cpu().numpy().reshape(osv.shape), osv)


# ------------------------------------------------------------------ binary scores

@pytest.mark.parametrize("name", list(WORKLOADS))
def test_scores_debug_bit_exact(name):
    w = WORKLOADS[name]
    inp = make_inputs(w)
    bq, _ = ba.pack_qk(_gpu(inp["q"], w.dtype))
    bk, _ = ba.pack_qk(_gpu(inp["k"], w.dtype))
    ob, _ = O.pack(inp["q"].reshape(w.B * w.H, w.N, w.d))
    okb, _ = O.pack(inp["k"].reshape(w.B * w.H, w.N, w.d))
    Wd = ba.words(w.d)
    heads = sorted({0, (w.B * w.H) // 2, w.B * w.H - 1})
    rng = np.random.default_rng(1)
    for bh in heads:
        b, h = divmod(bh, w.H)
        z = ba.scores_debug(bq[b:b + 1, h:h + 1], bk[b:b + 1, h:h + 1], w.d)   # views: 4-byte aligned
        torch.cuda.synchronize()
        rows = np.arange(w.N) if w.N <= 1024 else np.sort(rng.choice(w.N, 48, replace=False))
        zo = O.scores_rows(ob[bh], okb[bh], w.d, rows)
        np.testing.assert_array_equal(z[0, 0].cpu().numpy()[rows], zo)
        del z
    assert Wd == (w.d + 31) // 32


# ------------------------------------------------------------------ attention

SMALL = [
    # name, B, H, N, d, dtype, bias, grid
    ("tiles_ragged", 2, 3, 300, 64, "bf16", "dense", (0, 0)),
    ("relpos", 1, 2, 300, 64, "bf16", "relpos2d", (15, 20)),
    ("relpos_128", 1, 2, 384, 64, "bf16", "relpos2d", (3, 128)),
    ("nobias_d72", 2, 2, 257, 72, "bf16", "none", (0, 0)),
    ("f32_d64", 1, 3, 197, 64, "f32", "dense", (0, 0)),
    ("n1", 2, 2, 1, 64, "bf16", "dense", (0, 0)),
    ("n2", 1, 1, 2, 64, "f32", "none", (0, 0)),
    ("n127", 1, 2, 127, 64, "bf16", "dense", (0, 0)),
    ("n129", 1, 2, 129, 72, "bf16", "dense", (0, 0)),
    ("d32", 1, 2, 200, 32, "bf16", "dense", (0, 0)),
    ("d96", 1, 2, 150, 96, "f32", "dense", (0, 0)),
    ("d128", 1, 1, 140, 128, "bf16", "none", (0, 0)),
    ("d33", 1, 2, 90, 33, "f32", "dense", (0, 0)),
    ("d1", 1, 1, 40, 1, "f32", "none", (0, 0)),
    # 2-D rel-pos over a patch grid plus a class token (token 0)
    ("relpos_cls", 1, 2, 13, 64, "bf16", "relpos2d_cls", (3, 4)),
    ("relpos_cls_tiles", 2, 3, 301, 64, "bf16", "relpos2d_cls", (15, 20)),
    ("relpos_cls_d72_f32", 1, 2, 145, 72, "f32", "relpos2d_cls", (12, 12)),
    # dense bias with B >= 2: the paired kernel (two batch elements per CTA)
    ("pair_odd_b", 3, 2, 200, 64, "bf16", "dense", (0, 0)),
    ("pair_d72", 2, 2, 130, 72, "bf16", "dense", (0, 0)),
    ("pair_d128", 2, 1, 100, 128, "f32", "dense", (0, 0)),
    ("pair_d32_n64", 4, 1, 64, 32, "bf16", "dense", (0, 0)),
]


def _small_workload(spec):
    name, B, H, N, d, dtype, bias, grid = spec
    return Workload(name, B, H, N, d, dtype=dtype, bias=bias, grid=grid, bias_std=0.3)


@pytest.mark.parametrize("spec", SMALL, ids=[s[0] for s in SMALL])
@pytest.mark.parametrize("variant", [NAT.BA_QK_AUTO, NAT.BA_QK_POPC, NAT.BA_QK_MMA_B1] + TC_VARIANTS)
def test_attention_small_cases(spec, variant):
    w = _small_workload(spec)
    inp = make_inputs(w)
    try:
        g = _run_gpu(w, inp, variant)
    except NAT.BAError as e:
        assert e.status == NAT.BA_ERR_UNSUPPORTED and variant in TC_VARIANTS
        pytest.skip("variant does not take this shape")
    ref = _oracle_full(w, inp)
    _assert_close(g["out"].cpu().numpy(), ref["out"], inp["v"])
    assert ba.check_device_status() == 0


def test_attention_bf16_output_matches_f32_output():
    w = _small_workload(SMALL[0])
    inp = make_inputs(w)
    a = _run_gpu(w, inp, out_dtype=torch.float32)["out"]
    b = _run_gpu(w, inp, out_dtype=torch.bfloat16)["out"]
    torch.testing.assert_close(b.float(), a.to(torch.bfloat16).float(), rtol=0, atol=0)


def test_dominant_bias_selects_value_on_gpu():
    """Special case on the GPU: a +100 bias entry per row picks one key."""
    w = Workload("dom", 1, 2, 260, 64, bias="dense")
    inp = make_inputs(w)
    b = np.zeros_like(inp["bias"])
    for i in range(w.N):
        b[:, i, (5 * i + 1) % w.N] = 100.0
    inp["bias"] = b
    g = _run_gpu(w, inp)
    ref = _oracle_full(w, inp)
    _assert_close(g["out"].cpu().numpy(), ref["out"], inp["v"])


@pytest.mark.parametrize("variant", [NAT.BA_QK_AUTO, NAT.BA_QK_POPC, NAT.BA_QK_MMA_B1] + TC_VARIANTS)
def test_relpos_cls_entries_decide_on_gpu(variant):
    """The three class entries made large (class -> patch +3, patch -> class
    -4, class -> class +9): the class row and column move far beyond the
    tolerance if any kernel reads the wrong entry."""
    w = Workload("cls_dom", 1, 2, 7 * 9 + 1, 64, bias="relpos2d_cls", grid=(7, 9), bias_std=0.3)
    inp = make_inputs(w)
    G = 13 * 17
    inp["bias"][:, G] = 3.0
    inp["bias"][:, G + 1] = -4.0
    inp["bias"][:, G + 2] = 9.0
    g = _run_gpu(w, inp, variant)
    ref = _oracle_full(w, inp)
    _assert_close(g["out"].cpu().numpy(), ref["out"], inp["v"])


@pytest.mark.parametrize("variant", [NAT.BA_QK_AUTO, NAT.BA_QK_MMA_B1])
@pytest.mark.parametrize("name", list(WORKLOADS))
def test_attention_full_size(name, variant):
    """Every workload at its full size, in the launch configuration the
    benchmark times (the default QK path, and the warp-MMA .b1 one).  Small
    heads are compared in full; for the large ones the oracle computes sampled
    rows one by one."""
    w = WORKLOADS[name]
    inp = make_inputs(w)
    g = _run_gpu(w, inp, variant)
    out = g["out"].cpu().numpy()
    del g
    torch.cuda.empty_cache()
    gh, gw = w.grid
    BH = w.B * w.H
    kind = BIAS_KIND[w.bias]
    if w.B * w.H * w.N * w.N <= 4e7:
        ref = _oracle_full(w, inp)
        _assert_close(out, ref["out"], inp["v"])
        return
    bq, muq = O.pack(inp["q"].reshape(BH, w.N, w.d))
    bk, muk = O.pack(inp["k"].reshape(BH, w.N, w.d))
    vq, sv = O.quant_v(inp["v"].reshape(BH, w.N, w.d))
    rng = np.random.default_rng(2)
    heads = sorted({0, BH // 3, BH - 1})
    n_rows = w.N if w.N <= 1024 else 40
    got, want, vs = [], [], []
    for bh in heads:
        rows = np.arange(w.N) if n_rows == w.N else np.sort(rng.choice(w.N, n_rows, replace=False))
        for r in rows:
            o, _, _, _ = O.attention_rows(bq, muq, bk, muk, vq, sv, kind, inp["bias"], inp["ld"], gh, gw,
                                          w.H, bh, int(r), int(r) + 1, w.d)
            want.append(o[0])
            got.append(out.reshape(BH, w.N, w.d)[bh, r])
        vs.append(np.broadcast_to(inp["v"].reshape(BH, w.N, w.d)[bh].std(axis=0), (len(rows), w.d)))
    raw = np.abs(np.array(got) - np.array(want))
    assert raw.max() <= MAX_ABS and raw.mean() <= MEAN_ABS, ("raw", raw.max(), raw.mean())
    scale = np.maximum(1.0, np.concatenate(vs))
    err = raw / scale
    assert err.max() <= MAX_ABS and err.mean() <= MEAN_ABS, (err.max(), err.mean())


def test_device_status_is_clean():
    assert ba.check_device_status() == 0


MISALIGNED_SHAPES = [(2, 2, 577, 64, "bf16"), (1, 2, 300, 72, "bf16"), (2, 2, 197, 32, "f32"), (1, 1, 1025, 64, "bf16")]


@pytest.mark.parametrize("shape", MISALIGNED_SHAPES, ids=["x".join(map(str, s)) for s in MISALIGNED_SHAPES])
def test_prepass_misaligned_inputs(shape):
    """q, k, v one element past a 16-byte boundary (element-aligned, as the
    ABI allows) cannot take the tensor-copy or fused paths; the passes they
    fall back to give the same bits, codes and scales, and mu within fp32
    summation error (the fallback adds |x| in another fixed order)."""
    B, H, N, d, dtype = shape
    w = Workload("pp", B, H, N, d, dtype=dtype)
    inp = make_inputs(w)
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32

    def misaligned(x):
        flat = torch.from_numpy(x).to(tdt).reshape(-1)
        buf = torch.zeros(flat.numel() + 1, dtype=tdt, device=DEV)
        view = buf[1:].view(x.shape)
        view.copy_(flat.view(x.shape).to(DEV))
        assert view.data_ptr() % 16 != 0
        return view

    aligned = [_gpu(inp[n], dtype) for n in ("q", "k", "v")]
    shifted = [misaligned(inp[n]) for n in ("q", "k", "v")]
    want = ba.prepass_qkv(*aligned)
    got = ba.prepass_qkv(*shifted)
    torch.cuda.synchronize()
    for idx in (0, 2, 4, 5):                       # bq, bk, vq, sv
        assert torch.equal(want[idx], got[idx])
    for idx in (1, 3):                             # muq, muk
        a, b = want[idx].double(), got[idx].double()
        assert ((a - b).abs() / a.abs().clamp_min(1e-30)).max().item() <= d * 2.0 ** -24 + 2.0 ** -23
    assert ba.check_device_status() == 0
