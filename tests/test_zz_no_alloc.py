"""The allocation-free Vertical-Slash estimation entry point.

minf_estimate_vs_noalloc serves callers that cannot allocate device memory
when they run the estimation (a graph capture that forbids allocation, an
engine plugin with pre-planned memory), so they have no workspace to pass.
It must give exactly what minf_estimate_vs gives with a workspace, call
after call, although every call reuses the same built-in scratch array.
This file is collected last so that a failure here never hides the others.
"""
import ctypes

import numpy as np
import pytest
import torch

from dynamic_sparse_attention_minf_b200 import minf
from dynamic_sparse_attention_minf_b200 import workloads as wl

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    minf.lib()


def _call_noalloc(q, k, heads, k_v, k_s):
    """Through the C ABI directly (ctypes), with only inputs and outputs."""
    L = minf.lib()
    fn = L.minf_estimate_vs_noalloc
    vp, i = ctypes.c_void_p, ctypes.c_int
    fn.argtypes = [ctypes.POINTER(minf.Shape), vp, vp, vp, i, i, i, i, vp, vp, vp, vp, vp]
    fn.restype = ctypes.c_int
    shp = minf.shape_of(q, k)
    hd = torch.tensor(heads, dtype=torch.int32, device=q.device)
    nh = len(heads)
    v_idx = torch.full((1, nh, k_v), -7, dtype=torch.int32, device=q.device)
    s_idx = torch.full((1, nh, k_s), -7, dtype=torch.int32, device=q.device)
    vs = torch.full((1, nh, shp.N), -1.0, dtype=torch.float32, device=q.device)
    ss = torch.full((1, nh, shp.N), -1.0, dtype=torch.float32, device=q.device)
    code = fn(ctypes.byref(shp), ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()),
              ctypes.c_void_p(hd.data_ptr()), nh, 64, k_v, k_s, ctypes.c_void_p(v_idx.data_ptr()),
              ctypes.c_void_p(s_idx.data_ptr()), ctypes.c_void_p(vs.data_ptr()), ctypes.c_void_p(ss.data_ptr()),
              ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert code == 0, code
    torch.cuda.synchronize()
    return v_idx, s_idx, vs, ss


def _reference(q, k, heads, k_v, k_s):
    return minf.minf_estimate_vs(q, k, heads, k_v, k_s, return_scores=True)


def test_noalloc_matches_workspace_entry_point_twice_in_a_row():
    cases = [(wl.config(0), [0]),
             (wl.small(Hq=4, Hkv=2, N=2048, d=128, seed=31, k_v=64, k_s=128), [3, 0, 2])]
    for w, heads in cases:
        q, k, _ = wl.make_qkv(w, "cuda")
        ref = _reference(q, k, heads, w.k_v, w.k_s)
        for _ in range(2):                       # second call sees the first call's leftovers
            got = _call_noalloc(q, k, heads, w.k_v, w.k_s)
            assert torch.equal(got[0], ref[0]) and torch.equal(got[1], ref[1])
            np.testing.assert_allclose(got[2].cpu().numpy(), ref[2].cpu().numpy(), rtol=1e-4, atol=1e-7)
            np.testing.assert_allclose(got[3].cpu().numpy(), ref[3].cpu().numpy(), rtol=1e-4, atol=1e-7)


def test_noalloc_rejects_problems_beyond_its_scratch():
    L = minf.lib()
    fn = L.minf_estimate_vs_noalloc
    vp, i = ctypes.c_void_p, ctypes.c_int
    fn.argtypes = [ctypes.POINTER(minf.Shape), vp, vp, vp, i, i, i, i, vp, vp, vp, vp, vp]
    fn.restype = ctypes.c_int
    big = minf.Shape(1, 32, 8, 1048576, 128, 0.0)    # 32 heads x 1M tokens: far above 64 MiB
    fake = ctypes.c_void_p(1 << 20)
    assert fn(ctypes.byref(big), fake, fake, fake, 32, 64, 8, 8, fake, fake, None, None, None) == 4


def test_noalloc_reports_a_bad_head_through_its_status_getter():
    """A head id outside [0, Hq) is reported by the estimation kernels into
    the built-in scratch's status word; the getter returns it once and clears
    it, and a good call afterwards leaves it clear."""
    w = wl.small(Hq=4, Hkv=2, N=1024, d=128, seed=33, k_v=32, k_s=64)
    q, k, _ = wl.make_qkv(w, "cuda")
    assert minf.minf_noalloc_device_status() == 0
    minf.minf_estimate_vs_noalloc(q, k, [1, 99], w.k_v, w.k_s)
    assert minf.minf_noalloc_device_status() == 6   # MINF_ERR_DEVICE_BOUNDS
    assert minf.minf_noalloc_device_status() == 0
    got = minf.minf_estimate_vs_noalloc(q, k, [1, 2], w.k_v, w.k_s)
    ref = minf.minf_estimate_vs(q, k, [1, 2], w.k_v, w.k_s)
    assert minf.minf_noalloc_device_status() == 0
    assert torch.equal(got[0], ref[0]) and torch.equal(got[1], ref[1])


def test_noalloc_captures_in_a_graph_without_allocating():
    """The reason the entry point exists: captured into a CUDA graph under the
    global capture mode (where an allocating call would invalidate the
    capture) and replayed, it gives the workspace path's indices, and neither
    torch's allocator nor the device's free memory moves against it."""
    w = wl.small(Hq=4, Hkv=2, N=2048, d=128, seed=35, k_v=64, k_s=128)
    q, k, _ = wl.make_qkv(w, "cuda")
    heads = [0, 3]
    hd = torch.tensor(heads, dtype=torch.int32, device="cuda")
    ref = minf.minf_estimate_vs(q, k, heads, w.k_v, w.k_s)
    L = minf.lib()
    fn = L.minf_estimate_vs_noalloc
    vp, i = ctypes.c_void_p, ctypes.c_int
    fn.argtypes = [ctypes.POINTER(minf.Shape), vp, vp, vp, i, i, i, i, vp, vp, vp, vp, vp]
    fn.restype = ctypes.c_int
    shp = minf.shape_of(q, k)
    v_idx = torch.full((1, 2, w.k_v), -7, dtype=torch.int32, device="cuda")
    s_idx = torch.full((1, 2, w.k_s), -7, dtype=torch.int32, device="cuda")
    args = lambda st: (ctypes.byref(shp), vp(q.data_ptr()), vp(k.data_ptr()), vp(hd.data_ptr()), 2, 64,
                       w.k_v, w.k_s, vp(v_idx.data_ptr()), vp(s_idx.data_ptr()), None, None, vp(st))
    side = torch.cuda.Stream()
    with torch.cuda.stream(side):
        assert fn(*args(side.cuda_stream)) == 0      # warm-up outside the capture
    torch.cuda.synchronize()
    alloc0 = torch.cuda.memory_allocated()
    g = torch.cuda.CUDAGraph()
    codes = []
    # an allocating call inside the capture would invalidate it (global mode)
    with torch.cuda.graph(g, stream=side, capture_error_mode="global"):
        codes.append(fn(*args(side.cuda_stream)))
    assert codes == [0]
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()   # after the graph is instantiated
    for _ in range(2):
        v_idx.fill_(-7)
        s_idx.fill_(-7)
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(v_idx, ref[0]) and torch.equal(s_idx, ref[1])
    assert minf.minf_noalloc_device_status() == 0
    # nothing was allocated: neither torch's allocator nor the device grew
    assert torch.cuda.memory_allocated() <= alloc0
    free1, _ = torch.cuda.mem_get_info()
    assert free1 >= free0
    del g
