"""bench.py's host logic without a GPU: both arms describe the workload with the
same `config` dict, the device timeline is read back into per-kernel spans,
and the roofline arithmetic of a step reproduces hand-computed figures."""
import importlib.util
import os

import numpy as np
import pytest

from latent_compressed_attention_mla_b200 import binding as B
from latent_compressed_attention_mla_b200 import workloads as W

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_cpu_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


@pytest.mark.parametrize("cfg", W.CONFIGS, ids=lambda c: c.name)
def test_config_dict_names_only_the_workload(cfg):
    d = _bench().config_dict(cfg)
    assert d["workload"] == cfg.name and d["batch"] == cfg.B and d["n_q"] == cfg.T
    # launch details of one arm (split count, L2 handling, ranks) live outside `config`
    assert not {"l2", "splits", "parallelism", "path"} & set(d)


def test_default_workload_is_the_largest():
    bench = _bench()
    sizes = [int(c.seq_lens.sum()) * B.cache_page_bytes(B.dims_for(c)) // c.page_size for c in W.CONFIGS]
    assert W.CONFIGS[int(np.argmax(sizes))] is W.V3_FP8_B128_T2
    src = open(os.path.join(ROOT, "bench.py")).read()
    assert 'ap.add_argument("--config", type=int, default=4)' in src
    assert W.CONFIGS[4] is W.V3_FP8_B128_T2
    assert set(bench.EXTRA_CONFIGS) == {1, 2, 3}


def test_timeline_spans():
    nk = len(B.TRACE_KERNELS)
    v = np.zeros(2 * nk, dtype=np.int64)
    v[0::2] = -1  # kernels that did not run keep the initial begin
    k_att = B.TRACE_KERNELS.index("attend")
    v[2 * k_att], v[2 * k_att + 1] = 1_000_000, 1_250_000
    k_cmb = B.TRACE_KERNELS.index("combine")
    v[2 * k_cmb], v[2 * k_cmb + 1] = 1_260_000, 1_270_500
    assert B.timeline_spans_ns(v) == {"attend": 250_000, "combine": 10_500}


def test_step_summary_roofline_arithmetic():
    bench = _bench()
    cfg = W.V3_LONG_B8
    peaks = {"hbm_gbs": 6549.4, "bf16_tflops": 1639.1, "bf16_tflops_sustained": 1381.7}
    work = bench.kernel_work(cfg, 64 * 1152)
    att = work["attend"]
    # the attend kernel timed at exactly its core roofline -> fraction 1
    t_core = max(att["cache_bytes"] / 6549.4e9, att["flops"] / 1639.1e12)
    kms = {"append_project": 0.004, "absorb": 0.005, "attend": 1e3 * t_core, "combine": 0.006}
    s = bench.step_summary(cfg, work, kms, sum(kms.values()), peaks, 1639.1)
    assert s["attend"]["frac_of_core_roofline"] == pytest.approx(1.0)
    assert s["attend"]["latent_cache_TBps"] == pytest.approx(att["cache_bytes"] / t_core / 1e12)
    # 8 x 131073 keys x 1152 B: the long-context cache bytes
    assert att["cache_bytes"] == 8 * 131073 * 1152
    # 2176 flops per (query, head, key)
    assert att["flops"] == 2 * att["pairs"] * 128 * (576 + 512)
    assert 0 < s["full_step_frac"] <= 1.0
    rt = bench.roofline_times(work, peaks, 1639.1)
    assert s["full_step_roofline_us"] == pytest.approx(1e6 * sum(max(rt[k]) for k in kms))
