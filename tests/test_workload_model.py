"""Pins of the FLOP / byte model against the pages' worked example."""
import os

from moe_expert_grouped_softmax_b200 import workload as W

GOLD = os.path.join(os.path.dirname(__file__), "golden",
                    "lora_in_moe_worked_example.txt")


def _golden():
    vals = {}
    for line in open(GOLD):
        line = line.split("#")[0].strip()
        if line:
            key, val = (x.strip() for x in line.split("="))
            vals[key] = int(val)
    return vals


def test_lora_param_count_matches_page():
    g = _golden()
    p = W.lora_params_per_projection(g["m"], g["n"], g["r"])
    assert p == g["lora_params_per_projection_per_expert"]
    assert round(100 * p / (g["m"] * g["n"])) == g["lora_fraction_of_mn_percent_approx"]


def test_memory_crossover_matches_page():
    g = _golden()
    # split LoRA is better while E m n > k s n, i.e. s < E m / k
    assert g["E"] * g["m"] // g["k"] == g["memory_crossover_tokens"]


def test_split_flops_formula():
    # per-projection formula 2k(smn + smr + srn) with s tokens per expert slot
    s, m, n, r, k = 100, 64, 48, 8, 4
    assert W.split_lora_proj_flops(k * s, m, n, r) == 2 * k * (s*m*n + s*m*r + s*r*n)
    assert W.merged_lora_flops(16, k * s, m, n, r) == 16 * (2*m*n*r + m*n) + 2*k*s*m*n


def test_block_flops_gpt_oss():
    f = W.block_flops(8192, 2880, 2880, 32, 4, 16)
    # base GEMMs: fwd 6HI per row, bwd (dX only) 6HI per row
    assert f["base_gemm"] == 12 * 32768 * 2880 * 2880
    assert abs(f["total"] / 1e12 - 3.307) < 0.01
