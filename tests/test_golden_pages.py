"""Pins against values the pages print (tests/golden/pages_printed_values.json, cited there)."""
import json
import math
import os

from fp8_fp4_moe_b200 import inputs as I

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "pages_printed_values.json")


def _golden():
    with open(GOLDEN) as f:
        return json.load(f)


def test_fine_grained_combination_count_matches_the_printed_order_of_magnitude():
    g = _golden()["fine_grained_combinations"]
    exact = math.comb(g["n"], g["k"])
    assert abs(exact - g["approx_value"]) / g["approx_value"] < 0.05     # "about 400 trillion"


def test_deepseek_v3_workloads_use_the_printed_shape():
    g = _golden()["deepseek_v3_shape"]
    for name in ("dsv3_t1", "dsv3_t512", "dsv3_t8192_zipf", "dsv3_t32768"):
        w = I.WORKLOADS[name]
        assert (w.E, w.shared, w.k, w.H) == (g["routed_experts"], g["shared_experts"], g["active"], g["d_model"]), name
