"""Host-side checks of the C ABI (no GPU needed, no compute calls).

The library must load, export every function include/*.h declares, and
reject invalid arguments before it touches the CUDA runtime.
"""
import ctypes
import glob
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from bit_qk_attention_ba_b200 import build as B
    B.build()
    from bit_qk_attention_ba_b200 import _native
    return _native.load()


def _declared():
    src = "".join(open(p).read() for p in sorted(glob.glob(os.path.join(ROOT, "include", "*.h"))))
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(ba_[a-z_0-9]+)\s*\(", src)))


def test_header_declares_the_entry_points():
    names = _declared()
    for n in ("ba_pack_qk", "ba_quant_v", "ba_attention_fwd", "ba_scores_debug"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    from bit_qk_attention_ba_b200 import _native
    for name in _declared():
        assert hasattr(lib, name), name
        assert name in _native.SIGNATURES, "binding lacks " + name


def test_pure_helpers(lib):
    assert lib.ba_words(1) == 1 and lib.ba_words(32) == 1 and lib.ba_words(33) == 2
    assert lib.ba_words(72) == 3 and lib.ba_words(128) == 4
    assert lib.ba_vq_ld(1) == 16 and lib.ba_vq_ld(577) == 592 and lib.ba_vq_ld(16384) == 16384
    assert lib.ba_status_string(0) == b"BA_OK"
    assert lib.ba_status_string(1) == b"BA_ERR_INVALID_ARG"
    assert lib.ba_status_string(4) == b"BA_ERR_DEVICE_STATUS"


def test_prepass_launch_count(lib):
    """One fused launch when a (b, h) block of V fits in shared memory and the
    token is 2, 4, 8, 9, 12 or 16 vectors of 16 bytes; else pack Q, pack K and
    one (one-block V) or three (tiled V) quantiser launches.  128-, 144- and
    256-byte tokens take one launch up to 1024 code columns, else three
    (V's absmax, then Q, K and the V codes, then V's scales)."""
    bf16, f32 = 1, 0
    assert lib.ba_prepass_launches(577, 64, bf16) == 1        # DeiT-B/384
    assert lib.ba_prepass_launches(197, 64, f32) == 1         # DeiT-T
    assert lib.ba_prepass_launches(256, 72, bf16) == 1        # DiT-XL/2 (9 vectors)
    assert lib.ba_prepass_launches(256, 72, f32) == 3         # 18 vectors: not fused, V in one block
    assert lib.ba_prepass_launches(16384, 64, bf16) == 3      # HiRes: V absmax, Q K V codes, V scales
    assert lib.ba_prepass_launches(1024, 64, bf16) == 1
    assert lib.ba_prepass_launches(1025, 64, bf16) == 3
    assert lib.ba_prepass_launches(1500, 32, f32) == 3
    assert lib.ba_prepass_launches(16384, 72, bf16) == 3      # 144-byte tokens
    assert lib.ba_prepass_launches(16384, 64, f32) == 3       # 256-byte tokens
    assert lib.ba_prepass_launches(16384, 48, f32) == 5       # 192-byte tokens: separate passes, V tiled
    assert lib.ba_prepass_launches(90, 33, f32) == 5          # d * 4 not a multiple of 16
    assert lib.ba_prepass_launches(0, 64, bf16) == -1
    assert lib.ba_prepass_launches(8, 129, bf16) == -1
    assert lib.ba_prepass_launches(8, 64, 7) == -1


FAKE = ctypes.c_void_p(1 << 20)          # aligned, never dereferenced (validation fails first)
MIS = ctypes.c_void_p((1 << 20) + 1)      # misaligned for every element type


@pytest.mark.parametrize("B,H,N,d", [(0, 1, 8, 64), (1, 0, 8, 64), (1, 1, 0, 64), (1, 1, 8, 0), (1, 1, 8, 129),
                                     (70000, 1, 8, 64)])
def test_bad_sizes_rejected(lib, B, H, N, d):
    assert lib.ba_pack_qk(FAKE, 1, B, H, N, d, FAKE, FAKE, None) == 1
    assert lib.ba_quant_v(FAKE, 1, B, H, N, d, FAKE, FAKE, None) == 1
    assert lib.ba_scores_debug(FAKE, FAKE, B, H, N, d, FAKE, None) == 1
    assert lib.ba_prepass_qkv(FAKE, FAKE, FAKE, 1, B, H, N, d, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None) == 1
    assert lib.ba_attention_fwd(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 0, None, 0, 0, 0,
                                B, H, N, d, None, 0, FAKE, 0, None) == 1


def test_null_and_misaligned_pointers_rejected(lib):
    assert lib.ba_pack_qk(None, 1, 1, 1, 8, 64, FAKE, FAKE, None) == 1
    assert lib.ba_pack_qk(MIS, 1, 1, 1, 8, 64, FAKE, FAKE, None) == 1
    assert lib.ba_quant_v(FAKE, 1, 1, 1, 8, 64, MIS, FAKE, None) == 1
    assert lib.ba_scores_debug(FAKE, None, 1, 1, 8, 64, FAKE, None) == 1
    pp = [FAKE] * 6
    assert lib.ba_prepass_qkv(FAKE, None, FAKE, 1, 1, 1, 8, 64, *pp, None) == 1
    assert lib.ba_prepass_qkv(FAKE, FAKE, MIS, 1, 1, 1, 8, 64, *pp, None) == 1
    assert lib.ba_prepass_qkv(FAKE, FAKE, FAKE, 1, 1, 1, 8, 64, FAKE, FAKE, FAKE, FAKE, MIS, FAKE, None) == 1
    assert lib.ba_prepass_qkv(FAKE, FAKE, FAKE, 5, 1, 1, 8, 64, *pp, None) == 1
    args = [FAKE] * 6
    assert lib.ba_attention_fwd(*args[:5], None, 0, None, 0, 0, 0, 1, 1, 8, 64, None, 0, FAKE, 0, None) == 1
    assert lib.ba_attention_fwd(*args, 0, None, 0, 0, 0, 1, 1, 8, 64, None, 0, MIS, 0, None) == 1


def test_bad_dtypes_and_bias_rejected(lib):
    assert lib.ba_pack_qk(FAKE, 7, 1, 1, 8, 64, FAKE, FAKE, None) == 1
    args = [FAKE] * 6
    # dense bias: ld < N, ld not a multiple of 4, null table
    assert lib.ba_attention_fwd(*args, 1, FAKE, 4, 0, 0, 1, 1, 8, 64, None, 0, FAKE, 0, None) == 1
    assert lib.ba_attention_fwd(*args, 1, FAKE, 9, 0, 0, 1, 1, 8, 64, None, 0, FAKE, 0, None) == 1
    assert lib.ba_attention_fwd(*args, 1, None, 8, 0, 0, 1, 1, 8, 64, None, 0, FAKE, 0, None) == 1
    # rel-pos: N must equal grid_h * grid_w (+ 1 with a class token)
    assert lib.ba_attention_fwd(*args, 2, FAKE, 0, 3, 3, 1, 1, 8, 64, None, 0, FAKE, 0, None) == 1
    assert lib.ba_attention_fwd(*args, 3, FAKE, 0, 3, 3, 1, 1, 9, 64, None, 0, FAKE, 0, None) == 1
    assert lib.ba_attention_fwd(*args, 3, None, 0, 3, 3, 1, 1, 10, 64, None, 0, FAKE, 0, None) == 1
    assert lib.ba_attention_workspace_bytes(1, 1, 9, 64, 3, 3, 3) == -1
    assert lib.ba_attention_workspace_bytes(1, 1, 10, 64, 3, 3, 3) > 0
    assert lib.ba_attention_workspace_bytes(1, 1, 10, 64, 4, 3, 3) == -1
    assert lib.ba_attention_fwd(*args, 5, FAKE, 0, 0, 0, 1, 1, 8, 64, None, 0, FAKE, 0, None) == 1
    # out dtype and unknown QK variant
    assert lib.ba_attention_fwd(*args, 0, None, 0, 0, 0, 1, 1, 8, 64, None, 0, FAKE, 9, None) == 1
    assert lib.ba_attention_fwd_variant(*args, 0, None, 0, 0, 0, 1, 1, 8, 64, None, 0, FAKE, 0, 5, None) == 1
    assert lib.ba_attention_fwd_variant(*args, 0, None, 0, 0, 0, 1, 1, 8, 64, None, 0, FAKE, 0, -1, None) == 1


def _staged(B, H, N, d, general_relpos=False, keys=128):
    """Staged key side: tiles of +-1 operand bytes for `keys` keys, then the
    key scales (and for the general rel-pos bias the key offsets).  A dense
    bias with B >= 2 runs the paired kernel, whose tiles hold 64 keys."""
    dpad = 32 * ((d + 31) // 32)
    tile = keys * dpad + keys * 4 + (keys * 4 if general_relpos else 0)
    return B * H * ((N + keys - 1) // keys) * tile


def test_decode_arguments_checked(lib):
    """ba_attention_decode rejects bad sizes, pointers and bias strides before
    touching the device."""
    p = [FAKE] * 2
    good = dict(Nq=1, Nk=64, B=1, H=1, d=64)
    def call(Nq=1, Nk=64, B=1, H=1, d=64, bq=FAKE, vq=FAKE, bias=None, ld=0, ws=FAKE, out_dt=0):
        return lib.ba_attention_decode(bq, FAKE, Nq, FAKE, FAKE, vq, FAKE, Nk, bias, ld, B, H, d,
                                       ws, 1 << 30, FAKE, out_dt, None)
    assert call(Nq=0) == 1 and call(Nq=17) == 1 and call(Nk=0) == 1 and call(d=129) == 1
    assert call(bq=None) == 1 and call(vq=MIS) == 1 and call(ws=None) == 1 and call(out_dt=5) == 1
    assert call(bias=FAKE, ld=32) == 1                     # ld < Nk
    assert lib.ba_attention_decode_workspace_bytes(1, 1, 17, 64, 64) == -1
    assert lib.ba_attention_decode_workspace_bytes(1, 1, 0, 64, 64) == -1


def test_workspace_size_query(lib):
    """Workspace = staged key tiles, and for a rel-pos grid width that is a
    multiple of 128 four shifted copies of every reversed table row."""
    ws = lib.ba_attention_workspace_bytes
    rps = 12 * (2 * 128 - 1) * 4 * (2 * 128) * 4
    kst = _staged(4, 12, 16384, 64)
    assert kst % 256 == 0
    assert ws(4, 12, 16384, 64, 2, 128, 128) == kst + rps
    assert ws(4, 12, 16384, 64, 0, 0, 0) == kst
    assert ws(32, 12, 577, 64, 1, 0, 0) == _staged(32, 12, 577, 64, keys=64)
    assert ws(1, 3, 197, 64, 1, 0, 0) == _staged(1, 3, 197, 64)              # B = 1: nothing to pair
    assert ws(2, 2, 300, 72, 2, 15, 20) == _staged(2, 2, 300, 72, general_relpos=True)
    assert ws(0, 1, 8, 64, 0, 0, 0) == -1
    assert ws(1, 1, 8, 64, 2, 3, 3) == -1
    assert ws(1, 1, 8, 64, 7, 0, 0) == -1


def test_workspace_checked_before_launch(lib):
    args = [FAKE] * 6
    need = lib.ba_attention_workspace_bytes(1, 1, 256, 64, 0, 0, 0)
    assert need > 0
    assert lib.ba_attention_fwd(*args, 0, None, 0, 0, 0, 1, 1, 256, 64, None, 0, FAKE, 0, None) == 1
    assert lib.ba_attention_fwd(*args, 0, None, 0, 0, 0, 1, 1, 256, 64, FAKE, need - 16, FAKE, 0, None) == 1
    assert lib.ba_attention_fwd(*args, 0, None, 0, 0, 0, 1, 1, 256, 64, MIS, need, FAKE, 0, None) == 1
    assert lib.ba_attention_fwd(*args, 0, None, 0, 0, 0, 1, 1, 256, 64, FAKE, -1, FAKE, 0, None) == 1


def test_product_path_has_no_oracle_or_fallback():
    """The package never imports the oracle and has no CPU compute path."""
    pkg = os.path.join(ROOT, "bit_qk_attention_ba_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(dirpath, f)).read()
                assert "import oracle" not in text and "from oracle" not in text, f
                assert "ba_oracle" not in text, f
