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
