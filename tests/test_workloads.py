"""The seeded input generator: deterministic, right shapes and dtypes."""
import numpy as np

from bit_qk_attention_ba_b200.workloads import WORKLOADS, make_inputs


def test_table_matches_the_five_shapes():
    got = {k: (w.B, w.H, w.N, w.d) for k, w in WORKLOADS.items()}
    assert got == {"deit_t": (1, 3, 197, 64), "deit_s": (64, 6, 197, 64), "deit_b384": (32, 12, 577, 64),
                   "dit_xl2": (32, 16, 256, 72), "hires16k": (4, 12, 16384, 64),
                   "deit_b384_rpc": (32, 12, 577, 64)}
    w = WORKLOADS["deit_b384_rpc"]
    assert w.bias == "relpos2d_cls" and w.grid[0] * w.grid[1] + 1 == w.N
    assert make_inputs(w.scaled(B=1, H=2))["bias"].shape == (2, 47 * 47 + 3)
    assert WORKLOADS["hires16k"].bias == "relpos2d" and WORKLOADS["hires16k"].grid == (128, 128)
    assert WORKLOADS["deit_t"].dtype == "f32"


def test_deterministic_and_bf16_exact():
    w = WORKLOADS["deit_s"].scaled(B=2)
    a, b = make_inputs(w), make_inputs(w)
    for k in ("q", "k", "v", "bias"):
        np.testing.assert_array_equal(a[k], b[k])
    # bf16 values: the low 16 bits of every float32 are zero
    assert np.all((a["q"].view(np.uint32) & 0xFFFF) == 0)
    assert a["bias"].shape == (w.H, w.N, 200) and np.all(a["bias"][:, :, w.N:] == 0)


def test_outlier_channels_and_offsets():
    w = WORKLOADS["deit_s"].scaled(B=4)
    x = make_inputs(w)["v"]
    rms = np.sqrt((x.astype(np.float64) ** 2).mean(axis=(0, 2)))      # [H, d]
    assert np.sum(rms > 4.0) == round(0.02 * w.H * w.d)
    w2 = WORKLOADS["dit_xl2"].scaled(B=2)
    m = make_inputs(w2)["q"].mean(axis=(0, 2))
    assert np.all(np.abs(m) < 0.2)                                     # no channel offset for DiT


def test_relpos_table_shape():
    w = WORKLOADS["hires16k"].scaled(B=1, H=2, N=64, grid=(8, 8))
    inp = make_inputs(w)
    assert inp["bias"].shape == (2, 15 * 15)
