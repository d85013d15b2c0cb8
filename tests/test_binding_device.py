"""The Python binding calls libba with the tensors' device current (the
library keeps its per-device state on the current device): it switches the
device around the call when another one is current, and leaves it alone
when the tensors' device already is.  Checked with a fake torch and a fake
native call, no GPU."""
import contextlib
import types

import bit_qk_attention_ba_b200 as ba


class _Dev:
    def __init__(self, index):
        self.index = index


def _fake_torch(current, entered):
    @contextlib.contextmanager
    def device(dev):
        entered.append(dev.index)
        yield
    cuda = types.SimpleNamespace(current_device=lambda: current, device=device)
    return types.SimpleNamespace(cuda=cuda)


def test_call_switches_only_to_a_device_that_is_not_current(monkeypatch):
    calls, entered = [], []
    monkeypatch.setattr(ba.N, "call", lambda fn, *args: calls.append((fn, args)))
    monkeypatch.setattr(ba, "_torch", lambda: _fake_torch(0, entered))
    ba._call(_Dev(0), "ba_words", 1)            # already current: no switch
    assert entered == [] and calls == [("ba_words", (1,))]
    ba._call(_Dev(1), "ba_words", 2)            # another device: switched for the call
    assert entered == [1] and calls[-1] == ("ba_words", (2,))
    ba._call(_Dev(None), "ba_words", 3)         # "cuda" without an index means the current one
    assert entered == [1] and len(calls) == 3
