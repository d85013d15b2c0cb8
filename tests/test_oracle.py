"""Pins for the CPU oracle: checks against things other than the oracle itself.

Each test names the passage of the BA notes (paper-notes page "BinaryAttention:
One-Bit QK-Attention for Vision and Diffusion Transformers", CVPR 2026) it
pins, and what it is pinned to: a hand-worked example (tests/golden/), a
library routine, a closed form, an invariant, brute force, or the exact
full-precision attention within the provable quantisation error bound.
"""
import os

import numpy as np
import pytest

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
D_LIST = [1, 31, 32, 33, 64, 72, 96, 128]


def _rng(seed=0):
    return np.random.default_rng(seed)


def _read_golden(name):
    rows = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, rest = line.split(None, 1)
            rows[key] = [[float(t) for t in part.split()] for part in rest.split("|")]
    return rows


# ---------------------------------------------------------------- Key design 1

@pytest.mark.parametrize("d", D_LIST)
def test_bits_match_numpy_packbits(oracle, d):
    """KD1 sign bits, pinned to numpy.packbits (little bit order) of x >= 0."""
    x = _rng(d).standard_normal((5, 7, d)).astype(np.float32)
    x[0, 0, 0] = 0.0
    x[0, 1, 0] = -0.0          # reading: -0.0 counts as non-negative -> +1
    bits, _ = oracle.pack(x)
    W = (d + 31) // 32
    packed = np.packbits(x >= 0, axis=-1, bitorder="little")
    pad = np.zeros(x.shape[:-1] + (4 * W,), np.uint8)
    pad[..., : packed.shape[-1]] = packed
    expect = pad.view("<u4")
    assert bits.shape == x.shape[:-1] + (W,)
    np.testing.assert_array_equal(bits, expect)
    assert bits[0, 1, 0] & 1 == 1


@pytest.mark.parametrize("d", D_LIST)
def test_dot_forms_agree_with_bruteforce(oracle, d):
    """KD1 XNOR/popcount identity: s.t = d - 2 popc(xor) equals the +-1 dot
    product computed by brute force in Python, and the definition form."""
    rng = _rng(100 + d)
    for _ in range(20):
        q = rng.standard_normal(d).astype(np.float32)
        k = rng.standard_normal(d).astype(np.float32)
        brute = sum((1 if a >= 0 else -1) * (1 if b >= 0 else -1) for a, b in zip(q, k))
        bq, _ = oracle.pack(q[None])
        bk, _ = oracle.pack(k[None])
        assert oracle.dot_bits(bq[0], bk[0], d) == brute
        assert oracle.dot_pm1(q, k) == brute


def test_scores_match_sign_matmul(oracle):
    """KD1 score matrix pinned to a numpy matmul of the +-1 sign matrices."""
    rng = _rng(7)
    for d in (33, 64, 72):
        q = rng.standard_normal((3, 41, d)).astype(np.float32)
        k = rng.standard_normal((3, 41, d)).astype(np.float32)
        bq, _ = oracle.pack(q)
        bk, _ = oracle.pack(k)
        z = oracle.scores(bq, bk, d)
        sq = np.where(q >= 0, 1, -1).astype(np.int64)
        sk = np.where(k >= 0, 1, -1).astype(np.int64)
        np.testing.assert_array_equal(z, np.einsum("bic,bjc->bij", sq, sk))
        assert np.all(np.abs(z) <= d) and np.all((z - d) % 2 == 0)


def test_scores_rows_match_sign_matmul(oracle):
    """KD1 scores for a chosen block of query rows (the routine the full-size
    score checks use) pinned to a numpy matmul of the +-1 sign matrices, with
    rows out of order and repeated, and to the whole-matrix routine."""
    rng = _rng(17)
    for d in (1, 33, 64, 72, 128):
        N = 53
        q = rng.standard_normal((N, d)).astype(np.float32)
        k = rng.standard_normal((N, d)).astype(np.float32)
        q[3, 0] = 0.0
        k[5, -1] = -0.0
        bq, _ = oracle.pack(q)
        bk, _ = oracle.pack(k)
        rows = np.array([40, 0, 52, 7, 7, 19, 0], np.int32)
        z = oracle.scores_rows(bq, bk, d, rows)
        sq = np.where(q >= 0, 1, -1).astype(np.int64)
        sk = np.where(k >= 0, 1, -1).astype(np.int64)
        np.testing.assert_array_equal(z, (sq @ sk.T)[rows])
        np.testing.assert_array_equal(z, oracle.scores(bq[None], bk[None], d)[0][rows])
        assert z.shape == (len(rows), N) and z.dtype == np.int32


def test_scores_sign_flip_invariance(oracle):
    """Negating both Q and K (inputs without zeros) leaves every z unchanged."""
    rng = _rng(8)
    q = rng.standard_normal((2, 30, 64)).astype(np.float32)
    k = rng.standard_normal((2, 30, 64)).astype(np.float32)
    q[q == 0] = 1.0
    k[k == 0] = 1.0
    z1 = oracle.scores(oracle.pack(q)[0], oracle.pack(k)[0], 64)
    z2 = oracle.scores(oracle.pack(-q)[0], oracle.pack(-k)[0], 64)
    np.testing.assert_array_equal(z1, z2)


def test_mu_is_l2_optimal_scale(oracle):
    """KD1 scale: mu minimises ||x - mu sign(x)||^2 (closed form; checked with
    scipy's scalar minimiser, an independent routine)."""
    from scipy.optimize import minimize_scalar
    rng = _rng(9)
    x = (rng.standard_normal((12, 72)) * 1.7 + 0.3).astype(np.float32)
    _, mu = oracle.pack(x)
    s = np.where(x >= 0, 1.0, -1.0)
    for t in range(x.shape[0]):
        xt = x[t].astype(np.float64)
        f = lambda m: float(np.sum((xt - m * s[t]) ** 2))
        best = minimize_scalar(f, bounds=(0.0, 10.0), method="bounded",
                               options={"xatol": 1e-10}).x
        assert abs(mu[t] - best) < 1e-6
        assert f(mu[t]) <= f(mu[t] + 1e-3) and f(mu[t]) <= f(mu[t] - 1e-3)


# ---------------------------------------------------------------- Key design 3 (V)

def test_quant_v_against_numpy_and_roundtrip(oracle):
    """KD3 channel-wise int8 V: numpy fp32 division + rint (half-even) agree
    bit for bit; |sv*vq - v| <= sv/2; the absmax element maps to +-127; an
    all-zero channel has scale 0 and codes 0."""
    rng = _rng(10)
    v = (rng.standard_normal((3, 50, 72)) * 2.0).astype(np.float32)
    v[1, :, 5] = 0.0
    vq, sv = oracle.quant_v(v)
    a = np.abs(v).max(axis=1)
    sv_np = (a / np.float32(127.0)).astype(np.float32)
    np.testing.assert_array_equal(sv, sv_np)
    with np.errstate(invalid="ignore", divide="ignore"):
        r = np.where(sv_np[:, None, :] > 0, v / sv_np[:, None, :], np.float32(0))
    vq_np = np.clip(np.rint(r.astype(np.float32)), -127, 127).astype(np.int8)
    np.testing.assert_array_equal(vq, vq_np)
    err = np.abs(sv[:, None, :].astype(np.float64) * vq - v)
    assert np.all(err <= sv[:, None, :] * (0.5 + 1e-6) + 1e-30)
    idx = np.abs(v).argmax(axis=1)
    for bh in range(3):
        for c in range(72):
            if a[bh, c] > 0:
                assert abs(int(vq[bh, idx[bh, c], c])) == 127
    assert sv[1, 5] == 0 and np.all(vq[1, :, 5] == 0)


# ---------------------------------------------------------------- golden fixtures

def test_golden_tiny_forward(oracle):
    """The hand-worked d=4, N=2 example (tests/golden/tiny_d4_dense.txt)."""
    g = _read_golden("tiny_d4_dense.txt")
    q = np.array(g["q"], np.float32)[None, None]
    k = np.array(g["k"], np.float32)[None, None]
    v = np.array(g["v"], np.float32)[None, None]
    assert np.signbit(k[0, 0, 1, 0])            # the fixture's -0.0 survived parsing
    bias = np.array(g["bias"], np.float32)[None]
    res = oracle.forward(q, k, v, oracle.BIAS_DENSE, bias, ld=2)
    np.testing.assert_array_equal(res["bits_q"].ravel(), np.array(g["bits_q"]).ravel())
    np.testing.assert_array_equal(res["bits_k"].ravel(), np.array(g["bits_k"]).ravel())
    np.testing.assert_allclose(res["mu_q"].ravel(), np.array(g["mu_q"]).ravel(), rtol=0, atol=1e-15)
    np.testing.assert_allclose(res["mu_k"].ravel(), np.array(g["mu_k"]).ravel(), rtol=0, atol=1e-15)
    z = oracle.scores(res["bits_q"], res["bits_k"], 4)
    np.testing.assert_array_equal(z.ravel(), np.array(g["z"]).ravel())
    np.testing.assert_array_equal(res["sv"].ravel(), np.array(g["sv"]).ravel())
    out, pq, l, _ = oracle.attention_rows(res["bits_q"], res["mu_q"], res["bits_k"], res["mu_k"],
                                          res["vq"], res["sv"], oracle.BIAS_DENSE, bias, 2, 0, 0,
                                          1, 0, 0, 2, 4, want_pq=True)
    np.testing.assert_array_equal(pq, np.array(g["pq"]))
    np.testing.assert_allclose(l, np.array(g["l"]).ravel(), rtol=1e-15)
    np.testing.assert_allclose(out, np.array(g["out"]), rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(res["out"][0, 0], np.array(g["out"]), rtol=1e-13, atol=1e-13)


def test_golden_relpos_indexing(oracle):
    """KD2 2-D relative-position indexing, hand-worked on a 2x3 grid; with an
    integer-valued table T[k] = k every bias value is its own index."""
    gh, gw = 2, 3
    table = np.arange((2 * gh - 1) * (2 * gw - 1), dtype=np.float32)[None]
    with open(os.path.join(GOLDEN, "relpos_2x3.txt")) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                i, j, idx = (int(t) for t in line.split())
                assert oracle.bias_value(2, table, 0, 0, gh * gw, gh, gw, i, j) == idx


@pytest.mark.parametrize("gh,gw", [(3, 4), (5, 5), (1, 7), (4, 1)])
def test_relpos_structure(oracle, gh, gw):
    """Brute force over every pair: the index depends only on the offset
    (delta_row, delta_col); distinct offsets hit distinct entries and together
    cover the whole table; zero offset is the centre; +1 column offset is +1,
    +1 row offset is +(2 gw - 1) (row-major table)."""
    N = gh * gw
    table = np.arange((2 * gh - 1) * (2 * gw - 1), dtype=np.float32)[None]
    seen = {}
    for i in range(N):
        for j in range(N):
            dr, dc = i // gw - j // gw, i % gw - j % gw
            v = int(oracle.bias_value(2, table, 0, 0, N, gh, gw, i, j))
            assert seen.setdefault((dr, dc), v) == v
    assert len(set(seen.values())) == len(seen) == (2 * gh - 1) * (2 * gw - 1)
    assert seen[(0, 0)] == (gh - 1) * (2 * gw - 1) + (gw - 1)
    for (dr, dc), v in seen.items():
        if (dr, dc + 1) in seen:
            assert seen[(dr, dc + 1)] == v + 1
        if (dr + 1, dc) in seen:
            assert seen[(dr + 1, dc)] == v + 2 * gw - 1


def test_golden_relpos_cls_indexing(oracle):
    """2-D relative position with a class token, hand-worked on a 2x3 grid
    plus the class token; with T[k] = k every bias value is its own index."""
    gh, gw = 2, 3
    table = np.arange((2 * gh - 1) * (2 * gw - 1) + 3, dtype=np.float32)[None]
    n = 0
    with open(os.path.join(GOLDEN, "relpos_cls_2x3.txt")) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                i, j, idx = (int(t) for t in line.split())
                assert oracle.bias_value(3, table, 0, 0, gh * gw + 1, gh, gw, i, j) == idx
                n += 1
    assert n == 8


@pytest.mark.parametrize("gh,gw", [(3, 4), (2, 2), (1, 5), (4, 1)])
def test_relpos_cls_structure(oracle, gh, gw):
    """Brute force over every pair of a grid plus a class token: the class row
    and column are constant and take the three extra entries; the patch block
    is the plain rel-pos map of the grid (pinned above) shifted by one token;
    each head reads its own table."""
    G = (2 * gh - 1) * (2 * gw - 1)
    N = gh * gw + 1
    H = 2
    table = np.arange(H * (G + 3), dtype=np.float32).reshape(H, G + 3)
    plain = np.arange(G, dtype=np.float32)[None]
    for h in range(H):
        base = h * (G + 3)
        assert oracle.bias_value(3, table, 0, h, N, gh, gw, 0, 0) == base + G + 2
        for t in range(1, N):
            assert oracle.bias_value(3, table, 0, h, N, gh, gw, 0, t) == base + G
            assert oracle.bias_value(3, table, 0, h, N, gh, gw, t, 0) == base + G + 1
        for i in range(1, N):
            for j in range(1, N):
                want = base + oracle.bias_value(2, plain, 0, 0, N - 1, gh, gw, i - 1, j - 1)
                assert oracle.bias_value(3, table, 0, h, N, gh, gw, i, j) == want


def test_dense_bias_indexing(oracle):
    """Dense bias b[h][i][j] at row stride ld; shared over the batch."""
    H, N, ld = 2, 5, 8
    bias = np.arange(H * N * ld, dtype=np.float32).reshape(H, N, ld)
    for h in range(H):
        for i in range(N):
            for j in range(N):
                assert oracle.bias_value(1, bias, ld, h, N, 0, 0, i, j) == bias[h, i, j]


# ---------------------------------------------------------------- P quantisation

def _small_case(oracle, seed, B=2, H=2, N=37, d=64, bias_std=0.3, kind=1):
    rng = _rng(seed)
    q = (rng.standard_normal((B, H, N, d)) + 0.2).astype(np.float32)
    k = (rng.standard_normal((B, H, N, d)) - 0.1).astype(np.float32)
    v = rng.standard_normal((B, H, N, d)).astype(np.float32)
    bias = (rng.standard_normal((H, N, N)) * bias_std).astype(np.float32) if kind == 1 else None
    return q, k, v, bias


def test_p_rowsum_and_range(oracle):
    """KD3 u8 P with scale 1/255: 0 <= pq <= 255; the row's argmax has
    pq = 255; dequantised rows sum to 1 within N / (510 l) (each rounding error
    is at most 1/510 and l >= 1)."""
    q, k, v, bias = _small_case(oracle, 11)
    B, H, N, d = q.shape
    res = oracle.forward(q, k, v, 1, bias, ld=N)
    for bh in range(B * H):
        out, pq, l, m = oracle.attention_rows(res["bits_q"], res["mu_q"], res["bits_k"], res["mu_k"],
                                              res["vq"], res["sv"], 1, bias, N, 0, 0, H, bh, 0, N, d,
                                              want_pq=True)
        assert pq.max() <= 255 and np.all(l >= 1.0)
        sums = pq.sum(axis=1) / (255.0 * l)
        assert np.all(np.abs(sums - 1.0) <= N / (510.0 * l) + 1e-12)
        z = oracle.scores(res["bits_q"][bh:bh + 1], res["bits_k"][bh:bh + 1], d)[0]
        S = (res["mu_q"][bh][:, None] * res["mu_k"][bh][None, :] * z / np.sqrt(d)
             + bias[bh % H].astype(np.float64))
        assert np.all(pq[np.arange(N), S.argmax(axis=1)] == 255)


# ---------------------------------------------------------------- special cases

def _dequant(res):
    return res["sv"][:, None, :].astype(np.float64) * res["vq"]


def test_equal_scores_give_mean_of_dequantised_v(oracle):
    """All scores equal (identical K rows, no bias): every P~ = 1, pq = 255,
    so O = mean over keys of the dequantised V, exactly."""
    rng = _rng(12)
    B, H, N, d = 1, 2, 23, 64
    q = rng.standard_normal((B, H, N, d)).astype(np.float32)
    k = np.broadcast_to(rng.standard_normal((B, H, 1, d)), (B, H, N, d)).astype(np.float32)
    v = rng.standard_normal((B, H, N, d)).astype(np.float32)
    res = oracle.forward(q, k, v)
    expect = _dequant(res).mean(axis=1).reshape(B, H, 1, d)
    np.testing.assert_allclose(res["out"], np.broadcast_to(expect, res["out"].shape),
                               rtol=1e-12, atol=1e-14)


def test_single_key_returns_its_value(oracle):
    """N = 1: softmax over one key is 1, so O = sv * vq of that key."""
    rng = _rng(13)
    q = rng.standard_normal((2, 3, 1, 72)).astype(np.float32)
    k = rng.standard_normal((2, 3, 1, 72)).astype(np.float32)
    v = rng.standard_normal((2, 3, 1, 72)).astype(np.float32)
    res = oracle.forward(q, k, v)
    np.testing.assert_allclose(res["out"].reshape(6, 1, 72), _dequant(res), rtol=1e-14, atol=0)
    np.testing.assert_array_equal(np.abs(res["vq"]).max(axis=1), 127 * (np.abs(v).reshape(6, 72) > 0))


def test_dominant_bias_selects_one_key(oracle):
    """A +100 bias entry at (i, j*) makes every other P~ < e^-80 (pq = 0), so
    row i of O is the dequantised value of key j*."""
    q, k, v, _ = _small_case(oracle, 14, B=1, H=1, N=19)
    N = q.shape[2]
    bias = np.zeros((1, N, N), np.float32)
    target = {i: (7 * i + 3) % N for i in range(N)}
    for i, j in target.items():
        bias[0, i, j] = 100.0
    res = oracle.forward(q, k, v, 1, bias, ld=N)
    dv = _dequant(res)[0]
    for i, j in target.items():
        np.testing.assert_allclose(res["out"][0, 0, i], dv[j], rtol=1e-14, atol=0)


def test_key_permutation_invariance(oracle):
    """Permuting the keys together with their values and bias columns leaves
    O unchanged (softmax and the int PV sum are order-free)."""
    q, k, v, bias = _small_case(oracle, 15, B=1, H=2, N=29)
    perm = _rng(16).permutation(29)
    a = oracle.forward(q, k, v, 1, bias, ld=29)["out"]
    b = oracle.forward(q, k[:, :, perm], v[:, :, perm], 1,
                       np.ascontiguousarray(bias[:, :, perm]), ld=29)["out"]
    np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-14)


# ---------------------------------------------------------------- error bound

def _float_attention(q, k, v, bias, d_scale=None, use_bias=True, use_mu=True, transpose_bias=False):
    """Full-precision attention over the binarised scores (no P/V
    quantisation), from numpy primitives and scipy's softmax.  The keyword
    switches plant one plausible mistake each, for the sensitivity check."""
    from scipy.special import softmax
    B, H, N, d = q.shape
    sq, sk = np.where(q >= 0, 1.0, -1.0), np.where(k >= 0, 1.0, -1.0)
    z = np.einsum("bhic,bhjc->bhij", sq, sk)
    mq = np.abs(q.astype(np.float64)).mean(-1) if use_mu else np.ones((B, H, N))
    mk = np.abs(k.astype(np.float64)).mean(-1) if use_mu else np.ones((B, H, N))
    S = mq[..., :, None] * mk[..., None, :] * z / np.sqrt(d_scale or d)
    if use_bias:
        bb = bias[:, :, :N].astype(np.float64)
        S = S + (np.swapaxes(bb, 1, 2) if transpose_bias else bb)[None]
    P = softmax(S, axis=-1)
    return np.einsum("bhij,bhjc->bhic", P, v.astype(np.float64)), P


def test_within_quantisation_bound_of_float_attention(oracle):
    """The method's output differs from full-precision softmax attention over
    the same binarised scores only by the two 8-bit quantisations (KD3):
        |O - O_exact|_ic <= sum_j |vd_jc| / (510 l_i) + sv_c / 2
    (P rounding <= 1/510 per entry; V rounding <= sv/2).  Each planted mistake
    (no bias, no scales, sqrt of the padded width, transposed bias) must break
    the bound, which shows the check is sharp enough to catch it."""
    q, k, v, bias = _small_case(oracle, 17, B=2, H=2, N=24, d=40, bias_std=1.0)
    B, H, N, d = q.shape
    res = oracle.forward(q, k, v, 1, bias, ld=N)
    dv = _dequant(res).reshape(B, H, N, d)
    exact, _ = _float_attention(q, k, v, bias)
    l = np.zeros((B * H, N))
    for bh in range(B * H):
        _, _, l[bh], _ = oracle.attention_rows(res["bits_q"], res["mu_q"], res["bits_k"], res["mu_k"],
                                               res["vq"], res["sv"], 1, bias, N, 0, 0, H, bh, 0, N, d)
    l = l.reshape(B, H, N)
    bound = (np.abs(dv).sum(axis=2)[:, :, None, :] / (510.0 * l[..., None])
             + res["sv"].reshape(B, H, 1, d) / 2.0 + 1e-12)
    assert np.all(np.abs(res["out"] - exact) <= bound)
    for mistake in (dict(use_bias=False), dict(use_mu=False), dict(d_scale=64),
                    dict(transpose_bias=True)):
        wrong, _ = _float_attention(q, k, v, bias, **mistake)
        assert np.any(np.abs(res["out"] - wrong) > bound), mistake


def test_threaded_driver_matches_row_function(oracle):
    """The threaded whole-tensor driver gives the same rows as the row routine."""
    q, k, v, bias = _small_case(oracle, 18, B=2, H=3, N=45, d=33)
    B, H, N, d = q.shape
    res = oracle.forward(q, k, v, 1, bias, ld=N, nthreads=3)
    for bh in (0, 4):
        out, _, _, _ = oracle.attention_rows(res["bits_q"], res["mu_q"], res["bits_k"], res["mu_k"],
                                             res["vq"], res["sv"], 1, bias, N, 0, 0, H, bh, 10, 30, d)
        np.testing.assert_array_equal(out, res["out"].reshape(B * H, N, d)[bh, 10:30])


def test_relpos_forward_matches_dense_expansion(oracle):
    """A rel-pos table gives the same forward as the dense bias built from it
    through the (pinned) index map."""
    rng = _rng(19)
    gh, gw, H, d = 3, 4, 2, 32
    N = gh * gw
    q = rng.standard_normal((1, H, N, d)).astype(np.float32)
    k = rng.standard_normal((1, H, N, d)).astype(np.float32)
    v = rng.standard_normal((1, H, N, d)).astype(np.float32)
    table = (rng.standard_normal((H, (2 * gh - 1) * (2 * gw - 1))) * 0.5).astype(np.float32)
    dense = np.zeros((H, N, N), np.float32)
    for h in range(H):
        for i in range(N):
            for j in range(N):
                dr, dc = i // gw - j // gw, i % gw - j % gw
                dense[h, i, j] = table[h, (dr + gh - 1) * (2 * gw - 1) + dc + gw - 1]
    a = oracle.forward(q, k, v, 2, table, 0, gh, gw)["out"]
    b = oracle.forward(q, k, v, 1, dense, N)["out"]
    np.testing.assert_array_equal(a, b)


def test_relpos_cls_forward_matches_dense_expansion(oracle):
    """A rel-pos table with class-token entries gives the same forward as the
    dense bias built from it through the (pinned) index map, and a dominant
    class -> class entry makes the class query return the class value."""
    rng = _rng(23)
    gh, gw, H, d = 3, 3, 2, 32
    G = (2 * gh - 1) * (2 * gw - 1)
    N = gh * gw + 1
    q = rng.standard_normal((1, H, N, d)).astype(np.float32)
    k = rng.standard_normal((1, H, N, d)).astype(np.float32)
    v = rng.standard_normal((1, H, N, d)).astype(np.float32)
    table = (rng.standard_normal((H, G + 3)) * 0.5).astype(np.float32)
    dense = np.zeros((H, N, N), np.float32)
    for h in range(H):
        for i in range(N):
            for j in range(N):
                dense[h, i, j] = oracle.bias_value(3, table, 0, h, N, gh, gw, i, j)
    a = oracle.forward(q, k, v, 3, table, 0, gh, gw)["out"]
    b = oracle.forward(q, k, v, 1, dense, N)["out"]
    np.testing.assert_array_equal(a, b)
    table[:, G + 2] = 100.0
    res = oracle.forward(q, k, v, 3, table, 0, gh, gw)
    vq, sv = res["vq"].reshape(H, N, d), res["sv"].reshape(H, d)
    np.testing.assert_allclose(res["out"][0, :, 0], vq[:, 0].astype(np.float64) * sv, rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------- decode shape

def _decode_case(seed, B=2, H=3, Nq=4, Nk=53, d=64):
    rng = _rng(seed)
    q = (rng.standard_normal((B, H, Nq, d)) + 0.2).astype(np.float32)
    k = (rng.standard_normal((B, H, Nk, d)) - 0.1).astype(np.float32)
    v = rng.standard_normal((B, H, Nk, d)).astype(np.float32)
    return q, k, v


def test_decode_rows_match_square_forward(oracle):
    """Decode of Nq queries against Nk cached keys equals the first Nq rows of
    the (pinned) square forward over Nk tokens whose first Nq queries are
    those queries, with the dense bias embedded in the first Nq rows."""
    q, k, v = _decode_case(29)
    B, H, Nq, d = q.shape
    Nk = k.shape[2]
    rng = _rng(30)
    bias = (rng.standard_normal((H, Nq, Nk)) * 0.4).astype(np.float32)
    q_sq = rng.standard_normal((B, H, Nk, d)).astype(np.float32)
    q_sq[:, :, :Nq] = q
    bias_sq = np.zeros((H, Nk, Nk), np.float32)
    bias_sq[:, :Nq] = bias
    want = oracle.forward(q_sq, k, v, 1, bias_sq, Nk)["out"][:, :, :Nq]
    got = oracle.decode_forward(q, k, v, bias, Nk)
    np.testing.assert_array_equal(got, want)
    got_nb = oracle.decode_forward(q, k, v)
    want_nb = oracle.forward(q_sq, k, v)["out"][:, :, :Nq]
    np.testing.assert_array_equal(got_nb, want_nb)


def test_decode_special_cases(oracle):
    """One cached token returns its dequantised value; a dominant bias entry
    selects its key; identical keys and no bias give the mean of the
    dequantised values; permuting the cache leaves the output unchanged."""
    q, k, v = _decode_case(31, B=1, H=2, Nq=3, Nk=1)
    out = oracle.decode_forward(q, k, v)
    vq, sv = oracle.quant_v(v.reshape(2, 1, -1))
    deq0 = vq[:, 0].astype(np.float64) * sv.astype(np.float64)
    np.testing.assert_allclose(out.reshape(2, 3, -1), np.broadcast_to(deq0[:, None], (2, 3, 64)),
                               rtol=1e-13, atol=1e-13)

    q, k, v = _decode_case(32, B=1, H=2, Nq=3, Nk=40)
    bias = np.zeros((2, 3, 40), np.float32)
    picks = [7, 0, 39]
    for i, j in enumerate(picks):
        bias[:, i, j] = 100.0
    out = oracle.decode_forward(q, k, v, bias, 40)
    vq, sv = oracle.quant_v(v.reshape(2, 40, -1))
    for i, j in enumerate(picks):
        np.testing.assert_allclose(out[0, :, i], vq[:, j].astype(np.float64) * sv.astype(np.float64),
                                   rtol=1e-12, atol=1e-12)

    k_same = np.broadcast_to(k[:, :, :1], k.shape).copy()
    out = oracle.decode_forward(q, k_same, v)
    vq, sv = oracle.quant_v(v.reshape(2, 40, -1))
    mean = (vq.astype(np.float64) * sv[:, None].astype(np.float64)).mean(axis=1)
    np.testing.assert_allclose(out[0], np.broadcast_to(mean[:, None], (2, 3, 64)), rtol=1e-12, atol=1e-12)

    perm = _rng(33).permutation(40)
    a = oracle.decode_forward(q, k, v, bias, 40)
    b = oracle.decode_forward(q, k[:, :, perm], v[:, :, perm], bias[:, :, perm].copy(), 40)
    np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-12)
