"""Host-side arithmetic of bench.py that needs no GPU: the algorithmic bytes the
roofline divides by, and the DRAM traffic read back from the committed ncu
summaries."""
import pytest

import bench
from block_diffusion_attention_prefix_b200 import workloads as W


@pytest.mark.parametrize("name,recompute,reuse", [
    # prefix K+V 2*8*32768*128*2 = 134,217,728 B; Q, block K/V, cache rows and output on top
    ("dlm8b_b4", 134_366_208, 148_480),
    ("dlm8b_b16", 134_811_648, 593_920),
    ("long_100k", 409_748_480, 148_480),
])
def test_step_bytes(name, recompute, reuse):
    assert bench.step_bytes(W.get(name)) == (recompute, reuse)


def test_reuse_bytes_match_the_stated_per_step_figures():
    # about 145 KB (B = 4) and 578 KB (B = 16) per reuse step at the dLM-8B shapes
    assert bench.step_bytes(W.get("dlm8b_b4"))[1] / 1024 == pytest.approx(145, rel=0.01)
    assert bench.step_bytes(W.get("dlm8b_b16"))[1] / 1024 == pytest.approx(578, rel=0.01)


@pytest.mark.parametrize("name", ["tiny_f32", "dlm8b_b4", "dlm8b_b16", "video"])
def test_step_bytes_scale_with_the_batch(name):
    w = W.get(name)
    one = bench.step_bytes(w, batch=1)
    seven = bench.step_bytes(w, batch=7)
    assert seven == (7 * one[0], 7 * one[1])
    assert bench.step_bytes(w) == (w.batch * one[0], w.batch * one[1])


@pytest.mark.parametrize("name", ["dlm8b_b4", "dlm8b_b16", "long_100k"])
def test_committed_traffic_is_near_the_algorithmic_bytes(name):
    t = bench.ncu_traffic(name)
    if t is None:  # the kernel's sources changed since the capture
        pytest.skip("profile taken on other sources")
    alg = bench.step_bytes(W.get(name))[0]
    assert 1.0 <= t / alg < 1.05


def test_cpu_baseline_reports_all_cores_and_one_thread():
    r = bench.cpu_baseline(W.get("tiny_f32"), 0, budget_s=0.3, one_thread_budget_s=0.3)
    assert r["kind"] == "oracle" and r["unit"] == "steps/s" and r["value"] > 0 and r["cores"] >= 1
    assert "KV-head" in r["sample"]
    one = r["one_thread"]
    assert one is not None and one["cores"] == 1 and one["value"] > 0


def test_tensor_roofline_uses_the_burst_peak():
    r = bench.tensor_roofline(706.0)
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
    assert r["peak"] > 0 and r["frac"] == pytest.approx(706.0 / r["peak"])
    assert r["frac_of_sustained"] >= r["frac"]        # the sustained figure is the lower one
    assert "burst" in r["peak_source"]
