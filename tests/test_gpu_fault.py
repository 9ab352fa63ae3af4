"""Failure detection on the GPU without a GPU fault: device-side errors are
latched into the workspace status word and read by the host, and the context
stays usable afterwards."""
import numpy as np
import pytest
import torch

from dynamic_sparse_attention_minf_b200 import minf
from dynamic_sparse_attention_minf_b200 import workloads as wl

pytestmark = pytest.mark.gpu

TIMEOUT, BOUNDS = 5, 6


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    minf.lib()


def test_bounded_wait_reports_timeout_and_context_survives():
    w = wl.small(Hq=2, Hkv=2, N=512, d=128, seed=2)
    q, k, v = wl.make_qkv(w, "cuda")
    ws = minf.workspace(minf.OP_DENSE_ATTN, minf.shape_of(q, k), 2)
    ws[24:28].view(torch.int32).fill_(1)          # the first CTA withholds its key tiles
    minf.minf_dense_attn(q, k, v, ws=ws)            # launch succeeds; the kernel gives up after 2 s
    assert minf.minf_get_device_status(ws) == TIMEOUT
    # the status was cleared; with the hook off the same context computes correctly
    ws[24:28].view(torch.int32).fill_(0)
    o, lse = minf.minf_dense_attn(q, k, v, ws=ws)
    assert minf.minf_get_device_status(ws) == 0
    ref = torch.nn.functional.scaled_dot_product_attention(q.float(), k.float(), v.float(), is_causal=True)
    assert (o.float() - ref).abs().max().item() < 2e-2


def test_index_validation_reports_bounds():
    w = wl.small(Hq=1, Hkv=1, N=1024, d=64, seed=3)
    q, k, v = wl.make_qkv(w, "cuda")
    shp = minf.shape_of(q, k)
    v_idx = torch.tensor([[[3, 9, 40]]], dtype=torch.int32, device="cuda")
    s_idx = torch.tensor([[[0, 300, 200]]], dtype=torch.int32, device="cuda")   # not ascending
    ws = minf.workspace(minf.OP_BUILD_INDEX, shp, 1)
    minf.minf_build_index(shp, v_idx, s_idx, ws=ws)
    assert minf.minf_get_device_status(ws) == BOUNDS
    s_idx = torch.tensor([[[0, 200, 5000]]], dtype=torch.int32, device="cuda")  # beyond N
    minf.minf_build_index(shp, v_idx, s_idx, ws=ws)
    assert minf.minf_get_device_status(ws) == BOUNDS
    s_idx = torch.tensor([[[0, 200, 300]]], dtype=torch.int32, device="cuda")
    minf.minf_build_index(shp, v_idx, s_idx, ws=ws)
    assert minf.minf_get_device_status(ws) == 0
