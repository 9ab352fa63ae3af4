"""Host-only checks of libminf.so: it loads, exports every symbol that
include/minf.h declares, sizes workspaces and rejects bad arguments before
launching anything (no GPU needed)."""
import ctypes
import os
import re
import subprocess

import pytest

from dynamic_sparse_attention_minf_b200 import build as bld
from dynamic_sparse_attention_minf_b200 import minf

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    bld.build()
    return minf.lib()


def _declared():
    src = open(os.path.join(ROOT, "include", "minf.h")).read()
    return sorted(set(re.findall(r"^\w[\w\s\*]*?\b(minf_\w+)\s*\(", src, re.M)))


def test_header_declares_the_boundary():
    names = _declared()
    for n in ("minf_estimate_vs", "minf_estimate_bs", "minf_build_index", "minf_sparse_attn_vs",
              "minf_sparse_attn_bs", "minf_attn_ashape", "minf_dense_attn"):
        assert n in names


def test_exports_every_declared_symbol(L):
    out = subprocess.run(["nm", "-D", "--defined-only", minf.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\b(minf_\w+)\b", out))
    for n in _declared():
        assert n in exported, n
        assert hasattr(L, n)
    assert set(minf.EXPORTS) <= exported


def test_workspace_sizes(L):
    s = minf.Shape(1, 32, 8, 131072, 128, 0.0)
    for op in range(7):
        assert L.minf_workspace_size(op, ctypes.byref(s), 24, 1000, 6096, 100) >= 256
    vs = L.minf_workspace_size(minf.OP_ESTIMATE_VS, ctypes.byref(s), 24, 1000, 6096, 0)
    assert vs >= 24 * 131072 * 4 * 2          # both score vectors
    # Block-Sparse: the pooled means and score matrix; with a budget the
    # tensor-core path takes (k_b = 100), also the means' three bf16 parts
    base = 2 * 6 * 2048 * 128 * 4 + 6 * 2048 * 2048 * 4
    parts = 2 * 3 * 6 * 2048 * 128 * 2
    bs = L.minf_workspace_size(minf.OP_ESTIMATE_BS, ctypes.byref(s), 6, 0, 0, 100)
    assert bs >= base + parts
    for kb in (0, 200):
        bs0 = L.minf_workspace_size(minf.OP_ESTIMATE_BS, ctypes.byref(s), 6, 0, 0, kb)
        assert base <= bs0 < base + parts
    bad = minf.Shape(1, 32, 8, 1000, 128, 0.0)
    assert L.minf_workspace_size(0, ctypes.byref(bad), 24, 1, 1, 1) == 0
    assert L.minf_workspace_size(99, ctypes.byref(s), 24, 1, 1, 1) == 0
    assert L.minf_vs_wmap_words(131072) * 32 >= 131072 + 64


def test_argument_validation_without_launch(L):
    fake = ctypes.c_void_p(1 << 20)
    ok = minf.Shape(1, 2, 1, 1024, 128, 0.0)
    bad_n = minf.Shape(1, 2, 1, 1000, 128, 0.0)
    bad_d = minf.Shape(1, 2, 1, 1024, 96, 0.0)
    bad_g = minf.Shape(1, 3, 2, 1024, 128, 0.0)
    args = lambda s: (ctypes.byref(s), fake, fake, fake, None, 2, fake, None, fake, 256, None)
    assert L.minf_dense_attn(*args(bad_n)) == 1
    assert L.minf_dense_attn(*args(bad_g)) == 1
    assert L.minf_dense_attn(*args(bad_d)) == 2
    # workspace too small
    assert L.minf_dense_attn(ctypes.byref(ok), fake, fake, fake, None, 2, fake, None, fake, 8, None) == 4
    # null operand
    assert L.minf_dense_attn(ctypes.byref(ok), None, fake, fake, None, 2, fake, None, fake, 256, None) == 1
    # A-shape needs n_local >= 1 and a head list
    assert L.minf_attn_ashape(ctypes.byref(ok), fake, fake, fake, None, 2, 0, 8, fake, None, fake, 256, None) == 1
    assert L.minf_attn_ashape(ctypes.byref(ok), fake, fake, fake, fake, 2, 0, 0, fake, None, fake, 256, None) == 1
    # estimation: k out of range, last_q out of range, block != 64
    assert L.minf_estimate_vs(ctypes.byref(ok), fake, fake, fake, 2, 64, 0, 8, fake, fake, None, None,
                              fake, 1 << 30, None) == 1
    assert L.minf_estimate_vs(ctypes.byref(ok), fake, fake, fake, 2, 65, 8, 8, fake, fake, None, None,
                              fake, 1 << 30, None) == 1
    assert L.minf_estimate_bs(ctypes.byref(ok), fake, fake, fake, 2, 32, 4, fake, fake, None,
                              fake, 1 << 30, None) == 2
    assert L.minf_status_string(6) == b"device index out of range"
