"""CPU oracle for the BinaryAttention forward pass (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import this package.  The CUDA
product path never does, and the two share no code: this wrapper loads
``ba_oracle.c`` (plain C, fp64), compiled with gcc into ``libba_oracle.so``.

Source ("BA notes"): the paper-notes page "BinaryAttention: One-Bit
QK-Attention for Vision and Diffusion Transformers" (CVPR 2026), sections
Key design 1 (scaled binary Q/K), Key design 2 (bias enhancement), Key
design 3 (hybrid 8-bit quantisation of P and V) and, for the training-side
backward pass, Key design 4 (QAT with a straight-through estimator for sign).
Every numeric step lives in the C file; this module only marshals numpy
arrays.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ba_oracle.c")
_LIB = os.path.join(_HERE, "libba_oracle.so")
_lib = None

BIAS_NONE, BIAS_DENSE, BIAS_RELPOS2D, BIAS_RELPOS2D_CLS = 0, 1, 2, 3


def build(force: bool = False) -> str:
    """Compile ba_oracle.c with gcc (no fast-math, no FMA contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp.%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared",
                               "-ffp-contract=off", "-fno-fast-math", "-D_GNU_SOURCE",
                               "-o", tmp, _SRC, "-lm", "-lpthread"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is not None:
        return _lib
    lib = ctypes.CDLL(build())
    P = ctypes.c_void_p
    i32, i64 = ctypes.c_int, ctypes.c_int64
    lib.bao_words.argtypes = [i32]
    lib.bao_words.restype = i32
    lib.bao_pack.argtypes = [P, i64, i32, P, P]
    lib.bao_pack.restype = None
    lib.bao_dot_pm1.argtypes = [P, P, i32]
    lib.bao_dot_pm1.restype = ctypes.c_int32
    lib.bao_dot_bits.argtypes = [P, P, i32]
    lib.bao_dot_bits.restype = ctypes.c_int32
    lib.bao_scores.argtypes = [P, P, i64, i32, i32, P]
    lib.bao_scores.restype = None
    lib.bao_scores_rows.argtypes = [P, P, i32, i32, P, i32, P]
    lib.bao_scores_rows.restype = None
    lib.bao_bias_value.argtypes = [i32, P, i64, i32, i32, i32, i32, i32, i32]
    lib.bao_bias_value.restype = ctypes.c_double
    lib.bao_quant_v.argtypes = [P, i64, i32, i32, P, P]
    lib.bao_quant_v.restype = None
    lib.bao_attention_rows.argtypes = [P, P, P, P, P, P, i32, P, i64, i32, i32,
                                       i32, i32, i32, i64, i32, i32, P, P, P, P]
    lib.bao_attention_rows.restype = None
    lib.bao_attention_fwd.argtypes = [P, P, P, P, P, P, i32, P, i64, i32, i32,
                                      i32, i32, i32, i32, P, i32]
    lib.bao_attention_fwd.restype = i32
    lib.bao_attention_fwd_rows.argtypes = [P, P, P, P, P, P, i32, P, i64, i32, i32,
                                           i64, i32, i32, i32, i32, i32, P, i32]
    lib.bao_attention_fwd_rows.restype = i32
    lib.bao_attention_decode.argtypes = [P, P, P, P, P, P, i32, P, i64, i64, i32, i32, i32, i32, P]
    lib.bao_attention_decode.restype = None
    lib.bao_bwd_core.argtypes = [P, P, P, P, P, P, i32, i32, i32, P, P, P, P, P, P, P, P]
    lib.bao_bwd_core.restype = None
    lib.bao_attention_bwd.argtypes = [P, P, P, i32, P, i64, i32, i32, i32, i32, i32, i32, P,
                                      ctypes.c_double, i32, P, P, P, P, P]
    lib.bao_attention_bwd.restype = None
    _lib = lib
    return lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def words(d: int) -> int:
    return _load().bao_words(d)


def pack(x):
    """Sign bits [..., W] uint32 and per-token mean |x| [...] float64."""
    x = _c(x, np.float32)
    d = x.shape[-1]
    T = x.size // d
    W = words(d)
    bits = np.zeros(x.shape[:-1] + (W,), np.uint32)
    mu = np.zeros(x.shape[:-1], np.float64)
    _load().bao_pack(_ptr(x), T, d, _ptr(bits), _ptr(mu))
    return bits, mu


def dot_pm1(q, k) -> int:
    q, k = _c(q, np.float32), _c(k, np.float32)
    return int(_load().bao_dot_pm1(_ptr(q), _ptr(k), q.shape[-1]))


def dot_bits(a, b, d: int) -> int:
    a, b = _c(a, np.uint32), _c(b, np.uint32)
    return int(_load().bao_dot_bits(_ptr(a), _ptr(b), d))


def scores(bq, bk, d: int):
    """z [BH, N, N] int32 from bits [BH, N, W]."""
    bq, bk = _c(bq, np.uint32), _c(bk, np.uint32)
    BH, N = bq.shape[0], bq.shape[1]
    z = np.zeros((BH, N, N), np.int32)
    _load().bao_scores(_ptr(bq), _ptr(bk), BH, N, d, _ptr(z))
    return z


def scores_rows(bq_head, bk_head, d: int, rows):
    """z [len(rows), N] int32 for one head's bits [N, W] and chosen query rows."""
    bq, bk = _c(bq_head, np.uint32), _c(bk_head, np.uint32)
    r = _c(rows, np.int32)
    N = bk.shape[0]
    z = np.zeros((len(r), N), np.int32)
    _load().bao_scores_rows(_ptr(bq), _ptr(bk), N, d, _ptr(r), len(r), _ptr(z))
    return z


def bias_value(kind, bias, ld, h, N, gh, gw, i, j) -> float:
    b = None if bias is None else _c(bias, np.float32)
    return float(_load().bao_bias_value(kind, _ptr(b), ld, h, N, gh, gw, i, j))


def quant_v(v):
    """vq [BH, N, d] int8 and sv [BH, d] float32 from v [BH, N, d]."""
    v = _c(v, np.float32)
    BH, N, d = v.shape
    vq = np.zeros((BH, N, d), np.int8)
    sv = np.zeros((BH, d), np.float32)
    _load().bao_quant_v(_ptr(v), BH, N, d, _ptr(vq), _ptr(sv))
    return vq, sv


def attention_rows(bq, muq, bk, muk, vq, sv, bias_kind, bias, ld, gh, gw,
                   H, bh, row_lo, row_hi, d, want_pq=False):
    """Rows [row_lo, row_hi) of head bh; returns (out, pq, l, m)."""
    bq, bk = _c(bq, np.uint32), _c(bk, np.uint32)
    muq, muk = _c(muq, np.float64), _c(muk, np.float64)
    vq, sv = _c(vq, np.int8), _c(sv, np.float32)
    b = None if bias is None else _c(bias, np.float32)
    N = bq.shape[1]
    R = row_hi - row_lo
    out = np.zeros((R, d), np.float64)
    pq = np.zeros((R, N), np.uint8) if want_pq else None
    l = np.zeros(R, np.float64)
    m = np.zeros(R, np.float64)
    _load().bao_attention_rows(_ptr(bq), _ptr(muq), _ptr(bk), _ptr(muk), _ptr(vq), _ptr(sv),
                               bias_kind, _ptr(b), ld, gh, gw, H, N, d, bh, row_lo, row_hi,
                               _ptr(out), _ptr(pq), _ptr(l), _ptr(m))
    return out, pq, l, m


def attention_fwd(bq, muq, bk, muk, vq, sv, bias_kind, bias, ld, gh, gw, B, H, d, nthreads=0):
    """Full forward, out [BH, N, d] float64; returns (out, threads_used)."""
    bq, bk = _c(bq, np.uint32), _c(bk, np.uint32)
    muq, muk = _c(muq, np.float64), _c(muk, np.float64)
    vq, sv = _c(vq, np.int8), _c(sv, np.float32)
    b = None if bias is None else _c(bias, np.float32)
    N = bq.shape[1]
    out = np.zeros((B * H, N, d), np.float64)
    used = _load().bao_attention_fwd(_ptr(bq), _ptr(muq), _ptr(bk), _ptr(muk), _ptr(vq), _ptr(sv),
                                     bias_kind, _ptr(b), ld, gh, gw, B, H, N, d, _ptr(out), nthreads)
    return out, used


def attention_fwd_rows(bq, muq, bk, muk, vq, sv, bias_kind, bias, ld, gh, gw, n_heads, H, d,
                       row_lo, row_hi, nthreads=0):
    """Threaded rows [row_lo, row_hi) of heads [0, n_heads); out [n_heads, rows, d]."""
    bq, bk = _c(bq, np.uint32), _c(bk, np.uint32)
    muq, muk = _c(muq, np.float64), _c(muk, np.float64)
    vq, sv = _c(vq, np.int8), _c(sv, np.float32)
    b = None if bias is None else _c(bias, np.float32)
    N = bq.shape[1]
    out = np.zeros((n_heads, row_hi - row_lo, d), np.float64)
    used = _load().bao_attention_fwd_rows(_ptr(bq), _ptr(muq), _ptr(bk), _ptr(muk), _ptr(vq), _ptr(sv),
                                          bias_kind, _ptr(b), ld, gh, gw, n_heads, H, N, d, row_lo, row_hi,
                                          _ptr(out), nthreads)
    return out, used


def attention_decode(bq, muq, bk, muk, vq, sv, H, d, bias=None, ld=0):
    """Decode-shaped forward: bq [BH, Nq, W] / muq [BH, Nq] against the cached
    bk [BH, Nk, W], muk [BH, Nk], vq [BH, Nk, d], sv [BH, d]; optional dense
    bias [H, Nq, ld].  Returns out [BH, Nq, d] float64."""
    bq, bk = _c(bq, np.uint32), _c(bk, np.uint32)
    muq, muk = _c(muq, np.float64), _c(muk, np.float64)
    vq, sv = _c(vq, np.int8), _c(sv, np.float32)
    b = None if bias is None else _c(bias, np.float32)
    BH, Nq = bq.shape[0], bq.shape[1]
    Nk = bk.shape[1]
    out = np.zeros((BH, Nq, d), np.float64)
    _load().bao_attention_decode(_ptr(bq), _ptr(muq), _ptr(bk), _ptr(muk), _ptr(vq), _ptr(sv),
                                 1 if b is not None else 0, _ptr(b), int(ld), BH, H, Nq, Nk, d, _ptr(out))
    return out


def decode_forward(q, k, v, bias=None, ld=0):
    """Whole decode pipeline from raw q [B, H, Nq, d] and the cache's raw
    k, v [B, H, Nk, d]; returns out [B, H, Nq, d] float64."""
    B, H, Nq, d = q.shape
    Nk = k.shape[2]
    bq, muq = pack(np.asarray(q, np.float32).reshape(B * H, Nq, d))
    bk, muk = pack(np.asarray(k, np.float32).reshape(B * H, Nk, d))
    vq, sv = quant_v(np.asarray(v, np.float32).reshape(B * H, Nk, d))
    return attention_decode(bq, muq, bk, muk, vq, sv, H, d, bias, ld).reshape(B, H, Nq, d)


def forward(q, k, v, bias_kind=BIAS_NONE, bias=None, ld=0, gh=0, gw=0, nthreads=0):
    """Whole pipeline from raw q, k, v [B, H, N, d] (float32 values).

    Returns a dict with every intermediate the tests compare: bits_q, mu_q,
    bits_k, mu_k (shaped [BH, N, ...]), vq [BH, N, d], sv [BH, d] and
    out [B, H, N, d] float64.
    """
    B, H, N, d = q.shape
    bq, muq = pack(np.asarray(q, np.float32).reshape(B * H, N, d))
    bk, muk = pack(np.asarray(k, np.float32).reshape(B * H, N, d))
    vq, sv = quant_v(np.asarray(v, np.float32).reshape(B * H, N, d))
    out, used = attention_fwd(bq, muq, bk, muk, vq, sv, bias_kind, bias, ld, gh, gw, B, H, d, nthreads)
    return dict(bits_q=bq, mu_q=muq, bits_k=bk, mu_k=muk, vq=vq, sv=sv,
                out=out.reshape(B, H, N, d), threads=used)


def bwd_core(s, t, muq, muk, vh, bias, dO, quantise_p=False):
    """The differentiable core of one head (Key design 4 backward, see the C
    file): continuous s, t, vh [N, d], muq, muk [N], bias [N, N] or None,
    dO [N, d].  Returns dict O, ds, dt, dvh, dmuq, dmuk, dbias (float64)."""
    s, t, vh, dO = (_c(a, np.float64) for a in (s, t, vh, dO))
    muq, muk = _c(muq, np.float64), _c(muk, np.float64)
    b = None if bias is None else _c(bias, np.float64)
    N, d = s.shape
    out = {k: np.zeros((N, d)) for k in ("O", "ds", "dt", "dvh")}
    out["dmuq"], out["dmuk"] = np.zeros(N), np.zeros(N)
    out["dbias"] = np.zeros((N, N)) if b is not None else None
    _load().bao_bwd_core(_ptr(s), _ptr(t), _ptr(muq), _ptr(muk), _ptr(vh), _ptr(b), N, d, int(bool(quantise_p)),
                         _ptr(dO), _ptr(out["O"]), _ptr(out["ds"]), _ptr(out["dt"]), _ptr(out["dvh"]),
                         _ptr(out["dmuq"]), _ptr(out["dmuk"]), _ptr(out["dbias"]))
    return out


def attention_bwd(q, k, v, dO, bias_kind=BIAS_NONE, bias=None, ld=0, gh=0, gw=0, ste_clip=float("inf"),
                  quantise=True):
    """Backward with straight-through estimators from raw q, k, v [B, H, N, d]
    and dO [B, H, N, d].  Returns dict dq, dk, dv, O [B, H, N, d] and dbias
    (dense [H, N, ld], or the rel-pos table's shape [H, G (+3)], or None)."""
    B, H, N, d = q.shape
    q, k, v = (_c(a, np.float32) for a in (q, k, v))
    dO = _c(dO, np.float64)
    b = None if bias is None else _c(bias, np.float32)
    res = {n: np.zeros((B, H, N, d)) for n in ("dq", "dk", "dv", "O")}
    db = None
    if bias_kind == BIAS_DENSE:
        db = np.zeros((H, N, ld))
    elif bias_kind in (BIAS_RELPOS2D, BIAS_RELPOS2D_CLS):
        G = (2 * gh - 1) * (2 * gw - 1) + (3 if bias_kind == BIAS_RELPOS2D_CLS else 0)
        db = np.zeros((H, G))
    _load().bao_attention_bwd(_ptr(q), _ptr(k), _ptr(v), bias_kind, _ptr(b), int(ld), gh, gw, B, H, N, d,
                              _ptr(dO), float(ste_clip), int(bool(quantise)), _ptr(res["dq"]), _ptr(res["dk"]),
                              _ptr(res["dv"]), _ptr(res["O"]), _ptr(db))
    res["dbias"] = db
    return res
