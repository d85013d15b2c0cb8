"""ba_fwd_graph_*: the forward hot path replayed from one CUDA graph.

A step of the graph must write, bit for bit, what the two eager calls it
records write (ba_prepass_qkv, then ba_attention_fwd_variant): the pre-pass
outputs and the attention output, on its first launch and again after q, k
and v are refilled in place, on the default stream and on a side stream; and
it must report the kernel launches it replays.  The eager calls themselves
are checked against the oracle in the parity tests.
"""
import ctypes

import pytest

from bit_qk_attention_ba_b200 import _native as NAT
from bit_qk_attention_ba_b200.workloads import BIAS_KIND, Workload, make_inputs

FAKE = ctypes.c_void_p(1 << 20)


@pytest.fixture(scope="module")
def lib():
    try:
        return NAT.load()
    except ImportError as e:
        pytest.skip(str(e))


def test_graph_entry_points_reject_null_handles(lib):
    """Host-only checks: no device is touched."""
    assert lib.ba_fwd_graph_kernels(None) == -1
    assert lib.ba_fwd_graph_destroy(None) == NAT.BA_OK
    assert lib.ba_fwd_graph_launch(None, None) == NAT.BA_ERR_INVALID_ARG
    assert lib.ba_fwd_graph_create(FAKE, FAKE, FAKE, NAT.BA_BF16, 1, 1, 8, 64, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
                                   0, None, 0, 0, 0, FAKE, 0, FAKE, NAT.BA_BF16, 0, None) == NAT.BA_ERR_INVALID_ARG


# (workload, QK variant, kernel launches of the attention call after the pre-pass)
CASES = [
    (Workload("g_deit_t", 1, 3, 197, 64, dtype="f32"), 0, 2),                       # key staging + 128-key kernel
    (Workload("g_pair", 2, 2, 197, 64, bias_std=0.3), 0, 2),                        # key staging + paired kernel
    (Workload("g_rp_fast", 1, 2, 256, 64, bias="relpos2d", grid=(2, 128), bias_std=0.3), 0, 3),  # + table rows
    (Workload("g_rp_cls", 1, 2, 65, 64, bias="relpos2d_cls", grid=(8, 8), bias_std=0.3), 0, 2),
    (Workload("g_long", 1, 2, 1500, 64, bias="none"), 0, 2),                        # three pre-pass launches
    (Workload("g_popc", 1, 2, 100, 48, dtype="f32", bias="none"), 1, 1),            # CUDA-core variant
    (Workload("g_b1", 1, 2, 130, 96, bias="dense", bias_std=0.3), 2, 1),            # mma.sync .b1 variant
]


def _cuda():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    return torch


@pytest.mark.gpu
@pytest.mark.parametrize("case", CASES, ids=lambda c: c[0].name)
def test_graph_step_equals_eager_calls(case):
    torch = _cuda()
    import bit_qk_attention_ba_b200 as ba
    w, variant, attn_launches = case
    dev = torch.device("cuda:0")
    tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    inp = make_inputs(w)
    q, k, v = (torch.from_numpy(inp[n]).to(tdt).to(dev) for n in ("q", "k", "v"))
    bias = None if inp["bias"] is None else torch.from_numpy(inp["bias"]).to(dev)
    kind, ld, grid = BIAS_KIND[w.bias], inp["ld"], w.grid
    g = ba.ForwardGraph(q, k, v, bias=bias, bias_kind=kind, ld=ld, grid=grid, out_dtype=tdt, variant=variant)
    assert g.kernels == ba.prepass_launches(w.N, w.d, tdt) + attn_launches
    side = torch.cuda.Stream(dev)
    for step in range(3):
        if step > 0:        # new inputs, same buffers
            nxt = make_inputs(w, seed=w.seed + 17 * step)
            for t, name in ((q, "q"), (k, "k"), (v, "v")):
                t.copy_(torch.from_numpy(nxt[name]).to(tdt))
        if step == 2:
            side.wait_stream(torch.cuda.current_stream(dev))
            with torch.cuda.stream(side):
                g.launch()
            torch.cuda.current_stream(dev).wait_stream(side)
        else:
            g.launch()
        out_g = g.out.clone()
        pre_g = [t.clone() for t in g.pre]
        pre_e = ba.prepass_qkv(q, k, v)
        out_e = ba.attention_fwd(*pre_e, w.d, bias=bias, bias_kind=kind, ld=ld, grid=grid, out_dtype=tdt,
                                 variant=variant)
        torch.cuda.synchronize(dev)
        for a, b in zip(pre_g, pre_e):
            assert torch.equal(a, b)
        assert torch.equal(out_g, out_e)
        assert ba.check_device_status(dev) == 0
    g.close()
    g.close()                # a second close is a no-op
    with pytest.raises(RuntimeError):
        g.launch()


@pytest.mark.gpu
def test_graph_create_rejects_invalid_arguments():
    torch = _cuda()
    import bit_qk_attention_ba_b200 as ba
    dev = torch.device("cuda:0")
    w = Workload("g_bad", 1, 2, 64, 64)
    inp = make_inputs(w)
    q, k, v = (torch.from_numpy(inp[n]).to(torch.bfloat16).to(dev) for n in ("q", "k", "v"))
    bias = torch.from_numpy(inp["bias"]).to(dev)
    with pytest.raises(NAT.BAError) as e:      # a dense-bias row stride below N
        ba.ForwardGraph(q, k, v, bias=bias, bias_kind=BIAS_KIND["dense"], ld=60)
    assert e.value.status == NAT.BA_ERR_INVALID_ARG
    with pytest.raises(NAT.BAError) as e:      # a workspace too small for the staged key side
        ba.ForwardGraph(q, k, v, workspace=torch.empty(256, dtype=torch.uint8, device=dev))
    assert e.value.status == NAT.BA_ERR_INVALID_ARG
    torch.cuda.synchronize(dev)
    assert ba.check_device_status(dev) == 0


@pytest.mark.gpu
@pytest.mark.parametrize("mode", ["relaxed", "global"])
def test_entry_points_record_into_a_callers_graph(mode):
    """The eager calls recorded by the caller's own stream capture (torch's
    CUDA graph) replay to the same results as running them directly."""
    torch = _cuda()
    import bit_qk_attention_ba_b200 as ba
    dev = torch.device("cuda:0")
    w = Workload("g_user", 2, 2, 197, 64, bias_std=0.3)
    inp = make_inputs(w)
    q, k, v = (torch.from_numpy(inp[n]).to(torch.bfloat16).to(dev) for n in ("q", "k", "v"))
    bias = torch.from_numpy(inp["bias"]).to(dev)
    kind, ld = BIAS_KIND[w.bias], inp["ld"]
    pre = ba.prepass_qkv(q, k, v)
    ws = ba.attention_workspace(w.B, w.H, w.N, w.d, kind, device=dev)
    out = torch.empty((w.B, w.H, w.N, w.d), dtype=torch.bfloat16, device=dev)
    ba.attention_fwd(*pre, w.d, bias=bias, bias_kind=kind, ld=ld, out=out, workspace=ws)   # attributes set once
    torch.cuda.synchronize(dev)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, capture_error_mode=mode):
        ba.prepass_qkv(q, k, v, pre)
        ba.attention_fwd(*pre, w.d, bias=bias, bias_kind=kind, ld=ld, out=out, workspace=ws)
    nxt = make_inputs(w, seed=5)
    for t, name in ((q, "q"), (k, "k"), (v, "v")):
        t.copy_(torch.from_numpy(nxt[name]).to(torch.bfloat16))
    graph.replay()
    got = out.clone()
    pre_e = ba.prepass_qkv(q, k, v)
    ref = ba.attention_fwd(*pre_e, w.d, bias=bias, bias_kind=kind, ld=ld, out_dtype=torch.bfloat16)
    torch.cuda.synchronize(dev)
    assert torch.equal(got, ref)
    assert ba.check_device_status(dev) == 0
    del graph
