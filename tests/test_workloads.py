"""The seeded generators draw what the workload texts describe (CPU)."""

import numpy as np
import torch

import workloads as W


def test_stq_grid_structure_and_determinism():
    w = W.stq_grid_weights(32, 512, "cpu", 0, "t")
    w2 = W.stq_grid_weights(32, 512, "cpu", 0, "t")
    assert torch.equal(w, w2)
    g = w.view(32, 128, 4)
    assert torch.all((g == 0).sum(-1) == 1)            # exactly one zero per group
    d = w.view(32, 2, 256).abs().amax(-1)
    assert torch.all(d.half().float() == d)             # FP16-representable scale
    nz = w.view(32, 2, 256).abs()
    assert torch.all((nz == d.unsqueeze(-1)) | (nz == 0))
    assert not torch.equal(w, W.stq_grid_weights(32, 512, "cpu", 1, "t"))


def test_mxfp4_random_ranges():
    c, s = W.mxfp4_random(16, 256, "cpu", 0, "m")
    assert c.dtype == torch.uint8 and c.shape == (16, 128)
    assert s.shape == (16, 8) and int(s.min()) >= 118 and int(s.max()) <= 127


def test_zipf_routing_distinct_and_skewed():
    ids, w = W.zipf_routing(512, 256, 8, "cpu", 0, "z")
    assert ids.shape == (512, 8)
    for row in ids.tolist():
        assert len(set(row)) == 8
    assert torch.allclose(w.sum(1), torch.ones(512), atol=1e-6)
    counts = np.bincount(ids.view(-1).numpy(), minlength=256)
    assert counts.max() > 10 * np.median(counts[counts > 0]) / 2   # heavy head


def test_workload_table():
    assert W.WORKLOADS["stacked_decode"].formats == ("stq", "mx") * 4
    assert W.HIDDEN == 6144 and W.INTER == 2048 and W.EXPERTS == 256 and W.TOPK == 8


def test_bench_unit_bytes():
    """The bench's algorithmic bytes per matrix: STQ1_0 42 B per 256 weights, MXFP4 a half
    byte per weight + one scale per 32, MXFP8 a byte per weight + one scale per 32, BF16 2."""
    import bench

    n = 2048 * 6144
    assert bench.STQ_MAT == n // 256 * 42 == 2_064_384
    assert bench.MX_MAT == n // 2 + n // 32 == 6_684_672
    assert bench.MX8_MAT == n + n // 32 == 12_976_128
    assert bench.BF16_MAT == 2 * n == 25_165_824
