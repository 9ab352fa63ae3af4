"""Host-side pieces of the bench: the launch count it reports, the source
digest that decides whether the recorded DRAM traffic still applies, and the
committed launch-list summary that the count must agree with."""
import os
import re
import types

import bench
from dynamic_sparse_attention_minf_b200 import layer
from dynamic_sparse_attention_minf_b200 import workloads as wl


def _plan(cid):
    w = wl.config(cid)
    present = lambda pat: (object() if w.heads_of(pat) else None)
    return types.SimpleNamespace(w=w, vs_heads=present(wl.PAT_VS), bs_heads=present(wl.PAT_BS),
                                 a_heads=present(wl.PAT_A))


def test_launches_per_step_matches_launch_list_profile():
    """The count the bench reports equals the kernels ncu listed per layer:
    the run holds layers with one attention launch for every head (the
    product path) and layers with one attention launch per pattern."""
    n = layer.launches_per_step(_plan(4))
    n_sep = layer.launches_per_step(_plan(4), fused=False)
    text = open(os.path.join(bench.ROOT, "profiles", "launches_llama3_8b_layer_n1m.md")).read()
    m = re.search(r"(\d+) launches of libminf kernels in all = (\d+) x (\d+) \+ (\d+) x (\d+)", text)
    total, lf, nf, ls, ns = (int(g) for g in m.groups())
    listed = sum(int(c) for c in re.findall(r"^\| `minf::[^|]*\| (\d+) \|", text, re.M))
    assert (nf, ns) == (n, n_sep) == (29, 31)
    assert listed == total == lf * nf + ls * ns
    attn = sum(int(c) for c in re.findall(r"^\| `minf::attn_kernel[^|]*\| (\d+) \|", text, re.M))
    assert attn == lf + 3 * ls


def test_launches_per_step_other_layers():
    # 512K, Vertical-Slash heads only: estimation 4 + two 9-launch top-k, index 3, attention 1
    assert layer.launches_per_step(_plan(3)) == 26
    # 128K mixed layer: the same kernels as the 1M layer (one attention launch for all heads)
    assert layer.launches_per_step(_plan(2)) == 29
    # one attention launch per pattern instead
    assert layer.launches_per_step(_plan(2), fused=False) == 31


def test_digest_ignores_comments_and_whitespace():
    a = "int f(int x) { return x + 1; }  // one\n/* two */"
    b = "int  f(int x)\n{\n  return x + 1;   /* another note */ }\n"
    assert bench._code_only(a) == bench._code_only(b)
    assert bench._code_only(a) != bench._code_only(a.replace("+ 1", "+ 2"))


def test_recorded_traffic_gated_by_digest(monkeypatch):
    t = bench._recorded_traffic()
    assert t is None or t > 0
    monkeypatch.setattr(bench, "kernel_sources_digest", lambda: "0" * 64)
    assert bench._recorded_traffic() is None


def test_attention_counters_read_from_a_workspace():
    """The bench's tile and kept-entry counters come from the status block of
    an attention workspace (bytes 8..23)."""
    import torch
    ws = torch.zeros(256, dtype=torch.uint8)
    ws[8:24].view(torch.int64)[:] = torch.tensor([12345, 678])
    assert bench._counters(ws) == (12345, 678)
