"""bench.py's host-side arithmetic on CPU: algorithmic bytes per launch, the
memory-bound kernels' rooflines, and the committed ncu summaries it reads
(each must carry the hash of the current kernel sources, or its traffic
figure is stale)."""
import os
import re

import pytest

import bench
from mixture_experts_layer_45_b200 import workloads as wl

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_ffn_bytes_match_the_stated_formula():
    w = wl.workload("switch-top1")                 # bf16, R = 3940 kept rows, 32 active experts
    R, Ea, es = 3940, 32, 2
    # W1 of the active experts + b1 + xp read + h write
    assert bench.algorithmic_bytes("ffn1", w, R, Ea, es) == 32 * 3072 * 768 * 2 + 32 * 3072 * 2 + R * 768 * 2 \
        + R * 3072 * 2 == 181450752
    # W2 + b2 + h read + direct output write + row gates
    assert bench.algorithmic_bytes("ffn2", w, R, Ea, es) == 32 * 768 * 3072 * 2 + 32 * 768 * 2 + R * 3072 * 2 \
        + R * 768 * 2 + R * 4


def test_memory_kernel_bytes():
    w = wl.workload("skewed-top2")                 # k = 2, no capacity: R = T * k
    T, d, k, R = 16384, 1024, 2, 32768
    assert bench.algorithmic_bytes("router", w, R, 64, 2) == T * d * 2 + 64 * d * 2 + T * k * 8 + 64 * 4
    assert bench.algorithmic_bytes("permute", w, R, 64, 2) == T * d * 2 + R * d * 2 + T * k * 12 + R * 8
    assert bench.algorithmic_bytes("combine", w, R, 64, 2) == R * d * 2 + T * d * 2 + T * k * 4
    # direct top-1 output: the dispatch also zeroes the dropped tokens' rows
    s = wl.workload("switch-top1")
    assert bench.algorithmic_bytes("permute", s, 3940, 32, 2) == 4096 * 768 * 2 + 3940 * 768 * 2 + 4096 * 12 \
        + 3940 * 8 + (4096 - 3940) * 768 * 2
    # shared experts add their rows to the combine
    sh = wl.workload("skewed-top2", shared=2)
    assert bench.algorithmic_bytes("combine", sh, R, 64, 2) == (R + 2 * T) * d * 2 + T * d * 2 + T * k * 4


def test_add_memory_rooflines():
    w = wl.workload("skewed-top2")
    R = 32768
    kernels = {"combine": {"launches": 10, "ms_per_launch": 0.02, "share": 0.1},
               "ffn1": {"launches": 10, "ms_per_launch": 0.3, "share": 0.9}}
    bench.add_memory_rooflines(kernels, w, R, 64, 2, hbm_gbs=6555.2)
    nbytes = bench.algorithmic_bytes("combine", w, R, 64, 2)
    assert kernels["combine"]["gbs"] == pytest.approx(nbytes / 20e-6 / 1e9)
    assert kernels["combine"]["frac_of_hbm"] == pytest.approx(kernels["combine"]["gbs"] / 6555.2)
    assert "gbs" not in kernels["ffn1"]


def test_committed_profiles_are_current():
    """Every profile summary with a traffic line names the current hash of
    its kernel's sources."""
    pdir = os.path.join(ROOT, "profiles")
    checked = 0
    for name in sorted(os.listdir(pdir)):
        text = open(os.path.join(pdir, name)).read()
        h = re.search(r"source_hash:\s*([0-9a-f]+)", text)
        if not h:
            continue
        kernel, tag = name[:-3].split("_", 1)
        assert h.group(1) == bench.kernel_source_hash(kernel, bench.tag_dtype(tag)), name
        assert re.search(r"dram_bytes_per_launch:\s*[0-9]+", text), name
        checked += 1
    assert checked >= 8


def test_traffic_is_read_for_the_bench_workload():
    w = wl.workload("large-top2")                  # the bench's default workload
    assert bench.committed_traffic("ffn1", bench.workload_tag(w)) == 1527696240.0
    assert bench.committed_traffic("ffn1", "no-such-workload") is None


def test_defaults_meet_the_run_contract():
    """No flags: one GPU, at least 3 warm-up steps, and the largest
    single-GPU workload (the large top-2 layer, tensor-bound FFN)."""
    a = bench.parse_args([])
    assert a.gpus == 1 and a.warmup >= 3 and a.steps >= 1 and a.impl == "ours" and not a.no_e2e
    w = bench.get_workload(a)
    assert (w.name, w.T, w.d, w.ff, w.E, w.k, w.dtype, w.cf) == ("large-top2", 8192, 4096, 14336, 8, 2, "bf16",
                                                                 None)
    assert bench.workload_tag(w) == "large-top2-bf16-cfnone"


def test_oracle_sample_is_bounded_by_flops():
    """The oracle's timed sample: a power of two, at most the cap, fewer
    tokens where each costs more (about 32 GFLOP of float64 per pass)."""
    big = wl.workload("large-top2")                 # 4*2*4096*14336 = 470 MFLOP per token
    assert bench.oracle_sample_tokens(big, 1024) == 64
    sw = wl.workload("switch-top1")                 # 9.4 MFLOP per token
    assert bench.oracle_sample_tokens(sw, 1024) == 1024 and bench.oracle_sample_tokens(sw, 512) == 512
    tiny = wl.workload("dense-top2-f32")
    assert bench.oracle_sample_tokens(tiny, 1024) == 1024
    for w in wl.all_workloads():
        n = bench.oracle_sample_tokens(w, 1024)
        assert 16 <= n <= 1024 and n & (n - 1) == 0
        assert n == 16 or n * 4 * w.k * w.d * w.ff <= bench.ORACLE_FLOPS_PER_PASS


def test_reference_arm_line(capsys, monkeypatch):
    """`--impl reference` times the oracle on the host cores and prints the
    contract's line; under a multi-rank launch only rank 0 does so."""
    import json
    monkeypatch.setenv("RANK", "0")
    assert bench.main(["--impl", "reference", "--workload", "switch-top1", "--steps", "1", "--warmup", "0"]) == 0
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["metric"] == bench.METRIC and line["unit"] == "tokens/s"
    assert line["value"] > 0 and line["higher_is_better"] is True and line["steps"] == 1
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["cpu_baseline"]["value"] == line["value"]
    assert line["e2e"] == {"value": line["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}
    assert line["config"]["workload"].startswith("switch-top1 T=4096")
    monkeypatch.setenv("RANK", "1")
    assert bench.main(["--impl", "reference", "--steps", "1", "--warmup", "0"]) == 0   # no draw, no output
    assert capsys.readouterr().out == ""
