"""The seeded workload generator: determinism, slicing, statistics and the
configurations' shapes."""
import numpy as np
import torch

from latent_compressed_attention_mla_b200 import workloads as W


def test_generator_deterministic_and_sliceable():
    a = W.normal(3, 5, 1000)
    b = W.normal(3, 5, 1000)
    assert torch.equal(a, b)
    c = W.normal(3, 5, 300, start=700)
    assert torch.equal(a[700:], c)
    assert not torch.equal(a, W.normal(4, 5, 1000))
    assert not torch.equal(a, W.normal(3, 6, 1000))


def test_generator_statistics():
    x = W.normal(0, 1, 1 << 20).double()
    assert abs(x.mean().item()) < 5e-3
    assert abs(x.var().item() - 1.0) < 5e-3
    assert x.abs().max().item() <= 2 * np.sqrt(3) + 1e-6
    u = W.uniform(0, 2, 1 << 20).double()
    assert abs(u.mean().item() - 0.5) < 2e-3 and u.min() >= 0 and u.max() < 1


def test_configs():
    c = W.CONFIGS
    assert [x.seed for x in c] == [0, 1, 2, 3, 4]
    assert c[0].softmax_scale == 1 / np.sqrt(48) and c[1].softmax_scale == 1 / np.sqrt(192)
    assert int(np.sum(c[2].L)) == 1145364 and min(c[2].L) == 2286 and max(c[2].L) == 32542
    assert c[4].T == 2 and c[4].cache_dtype == "fp8"


def test_page_table_is_a_permutation():
    cfg = W.V3_RAGGED_B64
    pt = W.page_table(cfg)
    used = pt[pt >= 0]
    assert len(used) == cfg.num_pages and len(np.unique(used)) == cfg.num_pages
    for b in range(cfg.B):
        assert (pt[b] >= 0).sum() == cfg.pages_per_seq[b]


def test_history_rows_slices_agree():
    cfg = W.TINY_F32
    full = W.history_rows(cfg, 0, 0, 256)
    part = W.history_rows(cfg, 0, 100, 140)
    assert torch.equal(full["c"][100:140], part["c"]) and torch.equal(full["kr"][100:140], part["kr"])
    f8 = W.history_rows(W.V3_FP8_B128_T2, 3, 10, 20)
    assert f8["codes"].dtype == torch.uint8 and f8["scales"].shape == (10, 4)
