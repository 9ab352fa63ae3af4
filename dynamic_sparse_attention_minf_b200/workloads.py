"""Seeded synthetic inputs for the pre-fill sparse-attention path.

This module only *draws* inputs; it holds none of the method's arithmetic
(no scores, no selection, no masks, no attention).  Both the CUDA path and the
CPU oracle consume the tensors it returns, so that parity compares the two on
identical bf16 values.

The pages ("MInference 1.0", summary and abstract) name no dataset that can be
run here (their RULER / InfiniteBench / PG-19 / needle runs need model weights);
these generators stand in for the *shape* of that workload: LLaMA-3-8B attention
geometry (32 query heads, 8 KV heads, head dim 128), prompts of 4K to 1M tokens,
and the structure the three patterns are meant to exploit (attention sinks for
the vertical lines, a decaying local band for the slashes, block locality for
Block-Sparse).

Recipes (all i.i.d. N(0,1) in fp32 from ``torch.Generator(device).manual_seed``,
biases added in fp32, then one round-to-nearest-even cast to bf16):

* sink bias: 16 distinct key positions per KV head get ``+3 u`` (``u`` a seeded
  unit vector of that KV head); the last 64 query rows of every query head get
  ``+1.5 u`` of their KV head.
* local-band bias: ``beta * phi(i)`` added to Q_i and K_i on the last 2F dims,
  ``phi_{2f} = cos(w_f i)/sqrt(F)``, ``phi_{2f+1} = sin(w_f i)/sqrt(F)``,
  ``F = 8``, ``w_f = pi / (256 * 2^f)``, ``beta^2 = 2 sqrt(d)``: a RoPE-like
  logit bonus of about +2 at offset 0 that decays with the offset.
* block-locality bias: per head an orthonormal ``U`` (d x 8) and per 64-token
  block a code ``c_b ~ N(0, I_8)``; rows of block ``b`` get ``+2.0 U c_b`` in
  both Q and K.

GQA: query head ``h`` reads KV head ``h // (Hq // Hkv)``.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

PAT_VS, PAT_BS, PAT_A = 0, 1, 2
PATTERN_NAMES = {PAT_VS: "vertical_slash", PAT_BS: "block_sparse", PAT_A: "a_shape"}


@dataclass
class Workload:
    """One attention layer's worth of synthetic pre-fill inputs and settings."""
    name: str
    Hq: int
    Hkv: int
    N: int
    d: int
    seed: int
    bias: str                      # "sink", "block", "sink+band"
    patterns: list = field(default_factory=list)   # per query head: PAT_*
    last_q: int = 64
    k_v: int = 0
    k_s: int = 0
    k_b: int = 0
    block: int = 64
    n_sink: int = 0
    n_local: int = 0
    B: int = 1

    @property
    def group(self) -> int:
        return self.Hq // self.Hkv

    def heads_of(self, pat: int) -> list:
        return [h for h, p in enumerate(self.patterns) if p == pat]


def _mixed_table(Hq: int, seed: int) -> list:
    """Seeded head -> pattern table: 24 VS, 6 BS, 2 A-shape out of 32 heads."""
    g = torch.Generator(device="cpu").manual_seed(seed + 7)
    perm = torch.randperm(Hq, generator=g).tolist()
    n_vs = Hq * 24 // 32
    n_bs = Hq * 6 // 32
    pats = [PAT_VS] * Hq
    for h in perm[n_vs:n_vs + n_bs]:
        pats[h] = PAT_BS
    for h in perm[n_vs + n_bs:]:
        pats[h] = PAT_A
    return pats


def config(cid: int, N: int | None = None) -> Workload:
    """The five workloads (ids 0..4); ``N`` may be overridden for scaled-down runs."""
    if cid == 0:
        w = Workload("vs_h1_n4k_d64", 1, 1, 4096, 64, 1000, "sink",
                     [PAT_VS], k_v=128, k_s=256)
    elif cid == 1:
        w = Workload("bs_h8_n32k_d128", 8, 8, 32768, 128, 1001, "block",
                     [PAT_BS] * 8, k_b=64)
    elif cid == 2:
        w = Workload("llama3_8b_layer_n128k", 32, 8, 131072, 128, 1002, "sink+band",
                     _mixed_table(32, 1002), k_v=1000, k_s=6096, k_b=100,
                     n_sink=128, n_local=4096)
    elif cid == 3:
        w = Workload("llama3_8b_allvs_n512k", 32, 8, 524288, 128, 1003, "sink+band",
                     [PAT_VS] * 32, k_v=1000, k_s=6096)
    elif cid == 4:
        w = Workload("llama3_8b_layer_n1m", 32, 8, 1048576, 128, 1004, "sink+band",
                     _mixed_table(32, 1002), k_v=2000, k_s=12000, k_b=100,
                     n_sink=128, n_local=4096)
    else:
        raise ValueError(f"unknown workload id {cid}")
    if N is not None:
        w.N = N
    return w


def small(Hq=2, Hkv=1, N=1024, d=64, seed=7, bias="sink+band", patterns=None,
          **kw) -> Workload:
    """A free-form workload for parity tests at sizes the oracle finishes quickly."""
    return Workload(f"small_h{Hq}_{Hkv}_n{N}_d{d}", Hq, Hkv, N, d, seed, bias,
                    list(patterns) if patterns is not None else [PAT_VS] * Hq, **kw)


def _unit(gen, d, device):
    u = torch.randn(d, generator=gen, device=device, dtype=torch.float32)
    return u / u.norm()


@torch.no_grad()
def make_qkv(w: Workload, device="cpu"):
    """Draw Q [B,Hq,N,d], K, V [B,Hkv,N,d] in bf16 on ``device``.

    Generation runs head by head so that a 1M-token layer never holds more
    than one fp32 head at a time beyond the bf16 outputs.
    """
    dev = torch.device(device)
    gen = torch.Generator(device=dev).manual_seed(w.seed)
    B, Hq, Hkv, N, d = w.B, w.Hq, w.Hkv, w.N, w.d
    q = torch.empty(B, Hq, N, d, dtype=torch.bfloat16, device=dev)
    k = torch.empty(B, Hkv, N, d, dtype=torch.bfloat16, device=dev)
    v = torch.empty(B, Hkv, N, d, dtype=torch.bfloat16, device=dev)

    band = None
    if "band" in w.bias:
        F = 8
        beta = math.sqrt(2.0 * math.sqrt(d))
        pos = torch.arange(N, device=dev, dtype=torch.float64)
        cols = []
        for f in range(F):
            wf = math.pi / (256.0 * 2.0 ** f)
            cols.append(torch.cos(wf * pos) / math.sqrt(F))
            cols.append(torch.sin(wf * pos) / math.sqrt(F))
        band = (beta * torch.stack(cols, dim=1)).to(torch.float32)   # [N, 2F]

    sink_u = []
    for b in range(B):
        for hk in range(Hkv):
            kk = torch.randn(N, d, generator=gen, device=dev, dtype=torch.float32)
            u = _unit(gen, d, dev)
            sink_u.append(u)
            if "sink" in w.bias:
                pos = torch.randperm(N, generator=gen, device=dev)[:16]
                kk[pos] += 3.0 * u
            if band is not None:
                kk[:, d - band.shape[1]:] += band
            k[b, hk] = kk.to(torch.bfloat16)
            v[b, hk] = torch.randn(N, d, generator=gen, device=dev,
                                   dtype=torch.float32).to(torch.bfloat16)
        for h in range(Hq):
            qq = torch.randn(N, d, generator=gen, device=dev, dtype=torch.float32)
            if "sink" in w.bias:
                qq[N - 64:] += 1.5 * sink_u[b * Hkv + h // w.group]
            if band is not None:
                qq[:, d - band.shape[1]:] += band
            q[b, h] = qq.to(torch.bfloat16)

    if w.bias == "block":
        nb = N // w.block
        for b in range(B):
            for h in range(Hq):
                a = torch.randn(d, 8, generator=gen, device=dev, dtype=torch.float32)
                U, _ = torch.linalg.qr(a.cpu())
                U = U.to(dev)
                codes = torch.randn(nb, 8, generator=gen, device=dev, dtype=torch.float32)
                bias = (2.0 * codes @ U.T).repeat_interleave(w.block, dim=0)   # [N, d]
                q[b, h] = (q[b, h].float() + bias).to(torch.bfloat16)
                if h < Hkv:
                    k[b, h] = (k[b, h].float() + bias).to(torch.bfloat16)
    return q, k, v


def sample_rows(N: int, n_rows: int, seed: int, block: int = 64) -> torch.Tensor:
    """Stratified query-row sample for large-N checks (sorted, unique).

    An eighth of the rows cover the first block, a few block boundaries and the
    last 64 rows; the rest are uniform from a seeded generator.
    """
    if n_rows >= N:
        return torch.arange(N)
    g = torch.Generator(device="cpu").manual_seed(seed + 13)
    fixed = set(range(0, min(block, N), 8)) | set(range(N - 64, N, 4))
    nb = N // block
    for b in torch.randint(1, max(nb, 2), (8,), generator=g).tolist():
        fixed.update({b * block - 1, b * block})
    fixed = {r for r in fixed if 0 <= r < N}
    rest = torch.randperm(N, generator=g)[: n_rows * 2].tolist()
    out = list(sorted(fixed))[: n_rows // 8 + 1]
    seen = set(out)
    for r in rest:
        if len(out) >= n_rows:
            break
        if r not in seen:
            out.append(r)
            seen.add(r)
    return torch.tensor(sorted(out), dtype=torch.int64)
