"""The bounded waits of the tensor-core forward, made to run out on purpose.

ba_test_attention_fwd_starved runs the 128-key kernel with its loader
stopping before a chosen key step and a 2 ms give-up time on every barrier
wait.  Nothing is left in flight when the waits give up (every copy issued
before that step has been consumed), so this faults, traps and hangs nothing:
the MMA and softmax roles record their bits in the device status word, free
tensor memory and return.  The status word must report them, and the next
normal call must run clean and match the oracle.
"""
import ctypes
import time

import numpy as np
import pytest

import oracle as O
from bit_qk_attention_ba_b200.workloads import Workload, make_inputs

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import bit_qk_attention_ba_b200 as ba  # noqa: E402
from bit_qk_attention_ba_b200 import _native as NAT  # noqa: E402

DEV = torch.device("cuda:0")
PRODUCER, MMA, SOFTMAX = 1, 2, 4        # status bits of the kernel roles


@pytest.mark.parametrize("starve_step", [1, 5])     # pass A (maximum sweep) and pass B (P and PV)
def test_timeout_is_reported_and_the_next_call_is_clean(starve_step):
    w = Workload("starve", 1, 2, 512, 64, bias="none")      # 4 key steps per sweep, 8 in all
    inp = make_inputs(w)
    q, k, v = (torch.from_numpy(inp[n]).to(torch.bfloat16).to(DEV) for n in ("q", "k", "v"))
    bq, muq, bk, muk, vq, sv = ba.prepass_qkv(q, k, v)
    ws = ba.attention_workspace(w.B, w.H, w.N, w.d, device=DEV)
    out = torch.empty((w.B, w.H, w.N, w.d), dtype=torch.float32, device=DEV)
    assert ba.check_device_status() == 0
    lib = NAT.lib()
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    stream = ctypes.c_void_p(torch.cuda.current_stream(DEV).cuda_stream)
    t0 = time.perf_counter()
    st = lib.ba_test_attention_fwd_starved(p(bq), p(muq), p(bk), p(muk), p(vq), p(sv), w.B, w.H, w.N, w.d,
                                           p(ws), ws.numel(), p(out), NAT.BA_F32, starve_step, 2_000_000, stream)
    assert st == NAT.BA_OK
    code = ba.check_device_status()
    elapsed = time.perf_counter() - t0
    assert code & MMA and code & SOFTMAX, code
    assert not code & PRODUCER, code
    assert elapsed < 5.0                      # the waits gave up after ~2 ms, not the production 2 s
    assert ba.check_device_status() == 0      # reading the word cleared it
    # the context is usable: a normal call runs clean and is right
    good = ba.attention_fwd(bq, muq, bk, muk, vq, sv, w.d, workspace=ws)
    assert ba.check_device_status() == 0
    ref = O.forward(inp["q"], inp["k"], inp["v"])["out"]
    err = np.abs(good.cpu().numpy().astype(np.float64) - ref)
    assert err.max() <= 2e-2 and err.mean() <= 2e-3


def test_starved_entry_point_checks_its_arguments():
    lib = NAT.lib()
    f = ctypes.c_void_p(1 << 20)
    args = [f] * 6
    # negative step, too short a limit, too long a limit
    for step, ns in ((-1, 2_000_000), (1, 10), (1, 5_000_000_000)):
        assert lib.ba_test_attention_fwd_starved(*args, 1, 1, 256, 64, f, 1 << 30, f, 0, step, ns,
                                                 None) == NAT.BA_ERR_INVALID_ARG
