"""B200-native BinaryAttention forward (sm_100a CUDA behind a C ABI).

Python surface over libba (include/ba.h).  Tensors are torch CUDA tensors;
the functions allocate outputs with torch (the library itself allocates
nothing) and queue work on torch's current stream.

Method: the paper-notes page "BinaryAttention: One-Bit QK-Attention for Vision
and Diffusion Transformers" (CVPR 2026): Key design 1 (sign Q/K with per-token
scales, XNOR/popcount scores), Key design 2 (additive bias), Key design 3 (u8
P with scale 1/255, channel-wise int8 V, integer PV).
"""
from __future__ import annotations

import ctypes

from . import _native as N

__all__ = ["pack_qk", "quant_v", "prepass_qkv", "attention_fwd", "attention_fwd_noalloc", "attention_workspace",
           "ForwardGraph",
           "workspace_bytes", "attention_bwd", "attention_decode", "scores_debug", "forward",
           "check_device_status", "words", "vq_ld"]


def _torch():
    import torch
    return torch


def _dt(t) -> int:
    torch = _torch()
    if t.dtype == torch.bfloat16:
        return N.BA_BF16
    if t.dtype == torch.float32:
        return N.BA_F32
    raise TypeError("expected float32 or bfloat16, got %s" % t.dtype)


def _stream(device) -> ctypes.c_void_p:
    torch = _torch()
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _call(device, fn, *args):
    """Call a libba entry point with `device` current: the library looks up
    its per-device state (status word, SM count, static scratch) on the
    current device, and rejects a stream that belongs to another one.  The
    device is switched only when another one is current (the switch costs a
    few microseconds of host time per call)."""
    torch = _torch()
    if device.index is None or torch.cuda.current_device() == device.index:
        N.call(fn, *args)
        return
    with torch.cuda.device(device):
        N.call(fn, *args)


def _same_device(*ts):
    devs = {t.device for t in ts if t is not None}
    if len(devs) > 1:
        raise ValueError("all tensors must be on one CUDA device, got %s" % sorted(map(str, devs)))


def _need_cuda(*ts):
    for t in ts:
        if t is not None and (not t.is_cuda or not t.is_contiguous()):
            raise ValueError("tensors must be contiguous CUDA tensors")


def words(d: int) -> int:
    return (d + 31) // 32


def vq_ld(n: int) -> int:
    return (n + 15) // 16 * 16


def pack_qk(x, bits=None, mu=None):
    """Sign bits [B,H,N,W] (int32 storage of the uint32 words) and mu [B,H,N]."""
    torch = _torch()
    _need_cuda(x)
    B, H, Nn, d = x.shape
    if bits is None:
        bits = torch.empty((B, H, Nn, words(d)), dtype=torch.int32, device=x.device)
    if mu is None:
        mu = torch.empty((B, H, Nn), dtype=torch.float32, device=x.device)
    _same_device(x, bits, mu)
    _call(x.device, "ba_pack_qk", _p(x), _dt(x), B, H, Nn, d, _p(bits), _p(mu), _stream(x.device))
    return bits, mu


def quant_v(v, vq=None, sv=None):
    """int8 codes [B,H,d,ldv] (channel-major) and scales sv [B,H,d]."""
    torch = _torch()
    _need_cuda(v)
    B, H, Nn, d = v.shape
    if vq is None:
        vq = torch.empty((B, H, d, vq_ld(Nn)), dtype=torch.int8, device=v.device)
    if sv is None:
        sv = torch.empty((B, H, d), dtype=torch.float32, device=v.device)
    _same_device(v, vq, sv)
    _call(v.device, "ba_quant_v", _p(v), _dt(v), B, H, Nn, d, _p(vq), _p(sv), _stream(v.device))
    return vq, sv


def prepass_qkv(q, k, v, outs=None):
    """Pack Q and K and quantise V in one call (ba_prepass_qkv): returns
    (bq, muq, bk, muk, vq, sv), the outputs of pack_qk(q), pack_qk(k) and
    quant_v(v).  `outs` reuses a previous call's tuple."""
    torch = _torch()
    _need_cuda(q, k, v)
    B, H, Nn, d = q.shape
    if k.shape != q.shape or v.shape != q.shape or k.dtype != q.dtype or v.dtype != q.dtype:
        raise ValueError("q, k, v must share shape and dtype")
    if outs is None:
        dev = q.device
        outs = (torch.empty((B, H, Nn, words(d)), dtype=torch.int32, device=dev),
                torch.empty((B, H, Nn), dtype=torch.float32, device=dev),
                torch.empty((B, H, Nn, words(d)), dtype=torch.int32, device=dev),
                torch.empty((B, H, Nn), dtype=torch.float32, device=dev),
                torch.empty((B, H, d, vq_ld(Nn)), dtype=torch.int8, device=dev),
                torch.empty((B, H, d), dtype=torch.float32, device=dev))
    bq, muq, bk, muk, vq, sv = outs
    _same_device(q, k, v, *outs)
    _call(q.device, "ba_prepass_qkv", _p(q), _p(k), _p(v), _dt(q), B, H, Nn, d, _p(bq), _p(muq), _p(bk),
          _p(muk), _p(vq), _p(sv), _stream(q.device))
    return outs


def prepass_launches(n, d, dtype):
    """Kernel launches prepass_qkv makes for this shape (1 when fused)."""
    torch = _torch()
    return int(N.lib().ba_prepass_launches(int(n), int(d), N.BA_BF16 if dtype == torch.bfloat16 else N.BA_F32))


def _bias_args(bias, bias_kind, ld, grid):
    if bias is None or bias_kind == N.BA_BIAS_NONE:
        return N.BA_BIAS_NONE, None, 0, 0, 0
    _need_cuda(bias)
    gh, gw = grid if grid else (0, 0)
    if bias_kind == N.BA_BIAS_DENSE and not ld:
        ld = bias.shape[-1]
    return bias_kind, _p(bias), int(ld or 0), int(gh), int(gw)


def workspace_bytes(B, H, n, d, bias_kind=N.BA_BIAS_NONE, grid=None) -> int:
    """Device scratch bytes the fused forward needs (ba_attention_workspace_bytes)."""
    rel = bias_kind in (N.BA_BIAS_RELPOS2D, N.BA_BIAS_RELPOS2D_CLS)
    gh, gw = grid if (grid and rel) else (0, 0)
    nb = N.lib().ba_attention_workspace_bytes(B, H, n, d, int(bias_kind), int(gh), int(gw))
    if nb < 0:
        raise ValueError("invalid sizes or bias arguments for the fused forward")
    return int(nb)


def attention_workspace(B, H, n, d, bias_kind=N.BA_BIAS_NONE, grid=None, device=None):
    """A workspace tensor for attention_fwd (None when none is needed)."""
    torch = _torch()
    nb = workspace_bytes(B, H, n, d, bias_kind, grid)
    if nb == 0:
        return None
    # 256-byte alignment: the caching allocator returns 512-byte aligned blocks.
    return torch.empty((nb,), dtype=torch.uint8, device=device)


def attention_fwd(bq, muq, bk, muk, vq, sv, d, bias=None, bias_kind=N.BA_BIAS_NONE, ld=0, grid=None,
                  out=None, out_dtype=None, variant=N.BA_QK_AUTO, workspace=None):
    """Fused forward; returns out [B,H,N,d] (float32 unless out_dtype given).
    `workspace` (a uint8 CUDA tensor of at least workspace_bytes(...) bytes) is
    allocated here when not given."""
    torch = _torch()
    _need_cuda(bq, muq, bk, muk, vq, sv)
    B, H, Nn = muq.shape
    if out is None:
        out = torch.empty((B, H, Nn, d), dtype=out_dtype or torch.float32, device=muq.device)
    kind, bp, ld, gh, gw = _bias_args(bias, bias_kind, ld, grid)
    if workspace is None:
        if int(variant) not in (N.BA_QK_POPC, N.BA_QK_MMA_B1):   # the warp-level kernels stage nothing
            workspace = attention_workspace(B, H, Nn, d, kind, (gh, gw), device=muq.device)
    else:
        _need_cuda(workspace)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _same_device(bq, muq, bk, muk, vq, sv, out, workspace, bias)
    _call(muq.device, "ba_attention_fwd_variant", _p(bq), _p(muq), _p(bk), _p(muk), _p(vq), _p(sv), kind, bp, ld,
          gh, gw, B, H, Nn, d, _p(workspace), ws_bytes, _p(out), _dt(out), int(variant), _stream(muq.device))
    return out


class ForwardGraph:
    """The forward hot path -- prepass_qkv(q, k, v) then attention_fwd -- for
    fixed tensors, recorded once as a CUDA graph (ba_fwd_graph_create).
    launch() queues one whole step on the current stream as a single graph
    launch and returns `out`.  The object keeps a reference to every tensor
    the graph reads or writes (q, k, v, the pre-pass outputs `pre`, `out`, the
    bias and the workspace), so their storage outlives the graph; refill q, k
    and v in place between steps.  `kernels` is the number of kernel
    launches one step replays."""

    def __init__(self, q, k, v, bias=None, bias_kind=N.BA_BIAS_NONE, ld=0, grid=None, out=None, out_dtype=None,
                 variant=N.BA_QK_AUTO, pre=None, workspace=None):
        torch = _torch()
        self._h = None
        _need_cuda(q, k, v)
        B, H, Nn, d = q.shape
        if k.shape != q.shape or v.shape != q.shape or k.dtype != q.dtype or v.dtype != q.dtype:
            raise ValueError("q, k, v must share shape and dtype")
        dev = q.device
        if pre is None:
            pre = (torch.empty((B, H, Nn, words(d)), dtype=torch.int32, device=dev),
                   torch.empty((B, H, Nn), dtype=torch.float32, device=dev),
                   torch.empty((B, H, Nn, words(d)), dtype=torch.int32, device=dev),
                   torch.empty((B, H, Nn), dtype=torch.float32, device=dev),
                   torch.empty((B, H, d, vq_ld(Nn)), dtype=torch.int8, device=dev),
                   torch.empty((B, H, d), dtype=torch.float32, device=dev))
        if out is None:
            out = torch.empty((B, H, Nn, d), dtype=out_dtype or torch.float32, device=dev)
        kind, bp, ld, gh, gw = _bias_args(bias, bias_kind, ld, grid)
        if workspace is None:
            if int(variant) not in (N.BA_QK_POPC, N.BA_QK_MMA_B1):
                workspace = attention_workspace(B, H, Nn, d, kind, (gh, gw), device=dev)
        else:
            _need_cuda(workspace)
        ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
        _same_device(q, k, v, *pre, out, workspace, bias)
        bq, muq, bk, muk, vq, sv = pre
        h = ctypes.c_void_p()
        _call(dev, "ba_fwd_graph_create", _p(q), _p(k), _p(v), _dt(q), B, H, Nn, d, _p(bq), _p(muq), _p(bk),
              _p(muk), _p(vq), _p(sv), kind, bp, ld, gh, gw, _p(workspace), ws_bytes, _p(out), _dt(out),
              int(variant), ctypes.byref(h))
        self._h = h
        self._keep = (q, k, v, bias, workspace)
        self.pre, self.out, self.device = pre, out, dev
        self.kernels = int(N.lib().ba_fwd_graph_kernels(h))

    def launch(self):
        if self._h is None:
            raise RuntimeError("ForwardGraph used after close()")
        _call(self.device, "ba_fwd_graph_launch", self._h, _stream(self.device))
        return self.out

    def close(self):
        if getattr(self, "_h", None) is not None:
            N.check("ba_fwd_graph_destroy", N.lib().ba_fwd_graph_destroy(self._h))
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def attention_fwd_noalloc(bq, muq, bk, muk, vq, sv, d, bias=None, bias_kind=N.BA_BIAS_NONE, ld=0, grid=None,
                          out=None, out_dtype=None):
    """attention_fwd with the library's own static scratch instead of a
    workspace (ba_attention_fwd_noalloc)."""
    torch = _torch()
    _need_cuda(bq, muq, bk, muk, vq, sv)
    B, H, Nn = muq.shape
    if out is None:
        out = torch.empty((B, H, Nn, d), dtype=out_dtype or torch.float32, device=muq.device)
    kind, bp, ld, gh, gw = _bias_args(bias, bias_kind, ld, grid)
    _same_device(bq, muq, bk, muk, vq, sv, out, bias)
    _call(muq.device, "ba_attention_fwd_noalloc", _p(bq), _p(muq), _p(bk), _p(muk), _p(vq), _p(sv), kind, bp, ld,
          gh, gw, B, H, Nn, d, _p(out), _dt(out), _stream(muq.device))
    return out


def attention_bwd(q, k, bq, muq, bk, muk, vq, sv, out, dout, bias=None, bias_kind=N.BA_BIAS_NONE, ld=0,
                  grid=None, ste_clip=float("inf"), want_dbias=True, workspace=None, grads=None):
    """Backward of the fused forward with straight-through estimators
    (ba_attention_bwd): q, k the raw inputs [B,H,N,d] (their |x| decides the
    clipped estimator), the pre-pass outputs, the forward output `out` and the
    upstream gradient `dout` (both fp32 [B,H,N,d]).  Returns (dq, dk, dv,
    dbias) in fp32; dbias is None without a bias or when not wanted.  `grads`
    may hold preallocated (dq, dk, dv, dbias) tensors."""
    torch = _torch()
    _need_cuda(q, k, bq, muq, bk, muk, vq, sv, out, dout)
    B, H, Nn, d = q.shape
    dev = q.device
    kind, bp, ld, gh, gw = _bias_args(bias, bias_kind, ld, grid)
    if grads is not None:
        dq, dk, dv, dbias = grads
        if kind == N.BA_BIAS_NONE or not want_dbias:
            dbias = None
    else:
        dq, dk, dv = (torch.empty((B, H, Nn, d), dtype=torch.float32, device=dev) for _ in range(3))
        dbias = None
        if want_dbias and kind != N.BA_BIAS_NONE:
            dbias = torch.empty_like(bias, dtype=torch.float32)
    if workspace is None:
        nb = int(N.lib().ba_attention_bwd_workspace_bytes(B, H, Nn))
        if nb < 0:
            raise ValueError("invalid sizes for the backward pass")
        workspace = torch.empty((nb,), dtype=torch.uint8, device=dev)
    _same_device(q, k, bq, muq, bk, muk, vq, sv, out, dout, bias, workspace)
    _call(dev, "ba_attention_bwd", _p(q), _p(k), _dt(q), _p(bq), _p(muq), _p(bk), _p(muk), _p(vq), _p(sv), kind,
          bp, ld, gh, gw, B, H, Nn, d, _p(out), _p(dout), float(ste_clip), _p(workspace),
          workspace.numel(), _p(dq), _p(dk), _p(dv), _p(dbias), _stream(dev))
    return dq, dk, dv, dbias


def scores_debug(bq, bk, d, z=None):
    """Integer binary scores z [B,H,N,N] int32."""
    torch = _torch()
    _need_cuda(bq, bk)
    B, H, Nn, _ = bq.shape
    if z is None:
        z = torch.empty((B, H, Nn, Nn), dtype=torch.int32, device=bq.device)
    _same_device(bq, bk, z)
    _call(bq.device, "ba_scores_debug", _p(bq), _p(bk), B, H, Nn, d, _p(z), _stream(bq.device))
    return z


def forward(q, k, v, bias=None, bias_kind=N.BA_BIAS_NONE, ld=0, grid=None, out_dtype=None,
            variant=N.BA_QK_AUTO, workspace=None):
    """The whole hot path: pack Q, pack K and quantise V (one fused pre-pass
    call), then the fused attention."""
    d = q.shape[-1]
    bq, muq, bk, muk, vq, sv = prepass_qkv(q, k, v)
    return attention_fwd(bq, muq, bk, muk, vq, sv, d, bias=bias, bias_kind=bias_kind, ld=ld, grid=grid,
                         out_dtype=out_dtype or q.dtype, variant=variant, workspace=workspace)


def attention_decode(bq, muq, bk, muk, vq, sv, d, bias=None, out=None, out_dtype=None, workspace=None):
    """Decode-shaped forward (ba_attention_decode): bq/muq [B,H,Nq,...] from
    pack_qk of the queries, bk/muk/vq/sv from pack_qk / quant_v of the cached
    keys and values; optional dense bias [H, Nq, ld] (ld >= Nk).  Returns out
    [B,H,Nq,d]; `workspace` (uint8 CUDA tensor) is allocated when not given."""
    torch = _torch()
    _need_cuda(bq, muq, bk, muk, vq, sv)
    B, H, Nq = muq.shape
    Nk = muk.shape[2]
    if out is None:
        out = torch.empty((B, H, Nq, d), dtype=out_dtype or torch.float32, device=muq.device)
    if workspace is None:
        workspace = decode_workspace(B, H, Nq, Nk, d, device=muq.device)
    bp, ld = None, 0
    if bias is not None:
        _need_cuda(bias)
        bp, ld = _p(bias), int(bias.shape[-1])
    _same_device(bq, muq, bk, muk, vq, sv, out, workspace, bias)
    _call(muq.device, "ba_attention_decode", _p(bq), _p(muq), Nq, _p(bk), _p(muk), _p(vq), _p(sv), Nk, bp, ld, B,
          H, d, _p(workspace), workspace.numel(), _p(out), _dt(out), _stream(muq.device))
    return out


def decode_workspace(B, H, nq, nk, d, device=None):
    """A workspace tensor for attention_decode."""
    torch = _torch()
    with torch.cuda.device(device if device is not None else torch.cuda.current_device()):
        nb = int(N.lib().ba_attention_decode_workspace_bytes(B, H, nq, nk, d))
    if nb < 0:
        raise ValueError("invalid decode sizes (1 <= Nq <= 16, d <= 128) or no CUDA device")
    return torch.empty((max(nb, 256),), dtype=torch.uint8, device=device)


def check_device_status(device=None) -> int:
    """Synchronise and return the device status word (0 = no kernel failure)."""
    torch = _torch()
    code = ctypes.c_int(0)
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    with torch.cuda.device(dev):
        st = N.lib().ba_check_device_status(_stream(dev), ctypes.byref(code))
    if st not in (N.BA_OK, N.BA_ERR_DEVICE_STATUS):
        N.check("ba_check_device_status", st)
    return code.value
