"""The benchmark's byte and FLOP accounting (the denominators of every roofline figure it
prints) against values worked out by hand from the layer shapes."""
import importlib.util
import os

import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
_spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(ROOT, "bench.py"))
bench = importlib.util.module_from_spec(_spec)
_spec.loader.exec_module(bench)

W = synth.WORKLOADS


def test_int4_expert_bytes():
    # H=6144, I=2048: gate+up codes 2 * 2048 * 3072, row scales 2 * 2048 * 4; down codes
    # 6144 * 1024, row scales 6144 * 4 -- 18,915,328 bytes per expert (about 19 MB)
    b = bench.expert_bytes(W["decode1"])
    assert b == {"gate_up": 12_599_296, "down": 6_316_032}
    assert sum(b.values()) == 18_915_328


def test_nvfp4_expert_bytes():
    # H=2048, I=512: codes 3 * 512 * 1024, E4M3 block scales 3 * 512 * 128, three fp32
    # tensor scales -- 1,769,484 bytes per expert
    b = bench.expert_bytes(W["nvfp4_1"])
    assert sum(b.values()) == 1_769_484


def test_decode1_layer_bytes():
    # 8 routed + 1 shared expert, fp32 router matrix and bias, fp16 x in and y out
    ab = bench.algorithmic_bytes(W["decode1"], 8)
    assert ab["weights"] == 9 * 18_915_328
    assert ab["router"] == 256 * 6144 * 4 + 256 * 4 + 6144 * 2
    assert ab["total"] == 9 * 18_915_328 + 256 * 6144 * 4 + 256 * 4 + 2 * 6144 * 2 == 176_555_008
    assert ab["gate_up"] == 9 * 12_599_296 + 6144 * 2


def test_prefill512_flops():
    # 2 FLOP per weight per token for each of the 3 matrices (2 * 3 * I * H per pair),
    # 4096 routed pairs + 512 shared, plus the router's 2 * T * E * H
    assert bench.flops(W["prefill512"]) == 349_502_963_712
    # with adaptive top-p only the kept pairs count
    assert bench.flops(W["prefill512"], assignments=2048) == 6 * 2048 * 6144 * (2048 + 512) + 2 * 512 * 256 * 6144


def test_region_count_covers_the_minimum_time():
    assert bench.region_count(1.08, 0.5) == 463          # 20 decode steps of 54 us
    assert bench.region_count(46.0, 0.5) == 11
    assert bench.region_count(900.0, 0.5) == 3           # never fewer than three
    assert bench.region_count(0.0, 0.5) >= 3


def test_config_entry_figures():
    w = W["decode8"]
    ab = bench.algorithmic_bytes(w, 45)
    r = {"w": w, "ab": ab, "ms_step": 0.2, "U": 45.0, "tflops": 1.0, "region_ms": [4.0] * 7,
         "kernels_ms": {"layer": 0.19}, "roofline": {"peak": 6538.3}, "clocks": {},
         "e2e": {"value": 30000.0}, "peaks": {}}
    e = bench.config_entry(1, r, 20)
    assert e["tokens_per_s"] == 8 / 0.2e-3
    assert e["quantized_weight_gbs"] == ab["weights"] / 0.2e-3 / 1e9
    assert e["frac_quantized_of_8tbs"] == e["quantized_weight_gbs"] / 8000.0
    assert e["timed_regions"] == 7 and e["e2e_tokens_per_s"] == 30000.0
    assert "tflops_frac_of_dense_fp16_peak" not in e
    rp = dict(r, w=W["prefill512"], ab=bench.algorithmic_bytes(W["prefill512"], 228), ms_step=2.3,
              tflops=150.0, peaks={"bf16_tflops": 1500.0})
    assert bench.config_entry(1, rp, 20)["tflops_frac_of_dense_fp16_peak"] == 0.1


def test_config_steps_are_capped_by_each_workloads_defaults():
    # the headline's K and W as given; the other workloads of the line at most their own
    assert bench.config_steps("prefill512", 40000, 400) == (bench.DEFAULTS["prefill512"][0], 20)
    assert bench.config_steps("decode8", 20, 5) == (20, 5)
    assert bench.config_steps("int8_8", 20, 1) == (20, 3)          # at least 3 warm-up steps
    assert bench.config_steps("not_a_workload", 7, 4) == (7, 4)
    for name in bench.EXTRA_CONFIGS:
        assert name in bench.DEFAULTS
