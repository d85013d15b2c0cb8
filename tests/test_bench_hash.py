"""The source hash that ties a committed ncu summary to the kernel it was
taken on (bench.source_hash): it covers the kernel file and the local headers
it includes, transitively; comments and whitespace do not count."""
import os
import sys

sys.path.insert(0, os.path.join(os.path.dirname(__file__), ".."))

import bench  # noqa: E402


def _write(d, name, text):
    with open(os.path.join(d, name), "w") as f:
        f.write(text)


def test_hash_follows_includes_only(tmp_path):
    d = str(tmp_path)
    _write(d, "k.cu", '#include "a.cuh"\n__global__ void k() {}\n')
    _write(d, "a.cuh", '#pragma once\n#include "b.cuh"\nint a();\n')
    _write(d, "b.cuh", "#pragma once\nint b();\n")
    _write(d, "other.cuh", "int other();\n")
    k = os.path.join(d, "k.cu")
    h0 = bench.source_hash(k)
    _write(d, "other.cuh", "int other(); int more();\n")          # not included: same hash
    assert bench.source_hash(k) == h0
    _write(d, "b.cuh", "#pragma once\n// a comment\nint  b();\n")  # comments and spacing: same hash
    assert bench.source_hash(k) == h0
    _write(d, "b.cuh", "#pragma once\nint b(int);\n")               # code of an included header: new hash
    assert bench.source_hash(k) != h0


def test_hash_of_the_kernels_is_stable_and_distinct():
    csrc = bench.CSRC
    h_tc = bench.source_hash(os.path.join(csrc, "ba_attn_tc.cu"))
    h_pre = bench.source_hash(os.path.join(csrc, "ba_prepass_tma.cu"))
    assert h_tc == bench.source_hash(os.path.join(csrc, "ba_attn_tc.cu"))
    assert h_tc != h_pre and len(h_tc) == 16
