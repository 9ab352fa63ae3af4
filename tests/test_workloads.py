"""Host-side checks of the seeded input generator (no method arithmetic)."""
import torch

from dynamic_sparse_attention_minf_b200 import workloads as wl


def test_configs_shapes_and_tables():
    for cid in range(5):
        w = wl.config(cid)
        assert w.Hq % w.Hkv == 0 and w.N % 64 == 0 and w.d in (64, 128)
        assert len(w.patterns) == w.Hq
    w2 = wl.config(2)
    assert [w2.patterns.count(p) for p in (wl.PAT_VS, wl.PAT_BS, wl.PAT_A)] == [24, 6, 2]
    assert wl.config(4).patterns == w2.patterns


def test_make_qkv_deterministic_and_biased():
    w = wl.small(Hq=4, Hkv=2, N=512, d=64, seed=3, bias="sink+band")
    q1, k1, v1 = wl.make_qkv(w)
    q2, k2, v2 = wl.make_qkv(w)
    assert q1.dtype == torch.bfloat16 and q1.shape == (1, 4, 512, 64) and k1.shape == (1, 2, 512, 64)
    assert torch.equal(q1, q2) and torch.equal(k1, k2) and torch.equal(v1, v2)
    # the band bias makes q_i . k_i larger on average than q_i . k_{i+300}
    qf, kf = q1[0, 0].float(), k1[0, 0].float()
    near = (qf[:-300, -16:] * kf[:-300, -16:]).sum(-1).mean()
    far = (qf[:-300, -16:] * kf[300:, -16:]).sum(-1).mean()
    assert near > far + 1.0


def test_block_bias_and_sample_rows():
    w = wl.small(Hq=2, Hkv=2, N=256, d=32, seed=5, bias="block", patterns=[wl.PAT_BS] * 2)
    q, k, _ = wl.make_qkv(w)
    assert torch.isfinite(q.float()).all() and torch.isfinite(k.float()).all()
    rows = wl.sample_rows(131072, 512, 1)
    assert rows.numel() == 512 and torch.all(rows[1:] > rows[:-1])
    assert rows.min() >= 0 and rows.max() < 131072 and (rows >= 131072 - 64).any()
