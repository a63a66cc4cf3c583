"""Host-side logic of bench.py that needs no GPU: the roofline traffic record is used
only for the kernel source it was captured on, the workload table is consistent, and
the command line parses."""
import json
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from quantized_attention_fine_b200 import workloads as wl  # noqa: E402


def test_traffic_record_matches_the_current_kernel_source():
    """The committed record was captured on the attention kernel source in the tree."""
    rec = json.load(open(os.path.join(ROOT, "profiles", "attn_fwd_traffic.json")))["llm_prefill"]
    if rec["kernel_source_hash"] != bench.kernel_source_hash():
        pytest.skip("the traffic record is from another kernel source (bench.py reports traffic null)")
    assert bench.recorded_traffic("llm_prefill") == rec["dram_bytes_read"] + rec["dram_bytes_write"]
    assert bench.recorded_traffic("no_such_workload") is None


def test_traffic_record_ignored_for_another_source(monkeypatch):
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: "0" * 16)
    assert bench.recorded_traffic("llm_prefill") is None


def test_workloads_ops_and_names():
    assert wl.LLM_PREFILL.ops() == pytest.approx(4 * 32 * 32768 ** 2 * 128 / 2)
    assert wl.LLM_PREFILL_GQA.ops() == wl.LLM_PREFILL.ops()     # work is per query head
    assert wl.LLM_PREFILL_GQA.Hk == 8 and wl.LLM_PREFILL.Hk == 32
    for n in wl.SWEEP_N:
        for d in (64, 128):
            for c in ("causal", "full"):
                w = wl.by_name("sweep_n%d_d%d_%s" % (n, d, c))
                assert (w.N_q, w.d, w.causal) == (n, d, c == "causal")
    seeds = [w.seed for w in wl.WORKLOADS.values()]
    assert len(set(seeds)) == len(seeds)
    with pytest.raises(KeyError):
        wl.by_name("sweep_n123_d128_full")


def test_command_line(monkeypatch):
    monkeypatch.setattr(sys, "argv", ["bench.py", "--gpus", "2", "--steps", "5", "--warmup", "3", "--pv", "fp16",
                                      "--graph", "--workload", "image_dit"])
    a = bench.parse_args()
    assert (a.gpus, a.steps, a.warmup, a.pv, a.graph, a.workload) == (2, 5, 3, "fp16", True, "image_dit")
    monkeypatch.setattr(sys, "argv", ["bench.py"])
    a = bench.parse_args()
    assert (a.gpus, a.pv, a.graph, a.impl, a.workload) == (1, "fp8", False, "ours", "llm_prefill")
    assert a.warmup >= 3
