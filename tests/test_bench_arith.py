"""The benchmark's speed-of-light arithmetic against the numbers the pages print."""
import json
import os

import bench
import synthetic as syn

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "sol_arithmetic.json")


def test_mpk_a100_bound():
    g = json.load(open(GOLDEN))["mpk_a100"]
    rate = bench.sol_tokens_per_s(g["weight_bytes"], g["hbm_bytes_per_s"])
    assert abs(1000.0 / rate - g["bound_ms"]) < 1e-9
    # MPK at 80% of the bound, vLLM/SGLang at 69%
    assert round(100 * g["bound_ms"] / g["mpk_ms_per_token"]) == 80
    assert round(100 * g["bound_ms"] / g["vllm_ms_per_token"]) == 69


def test_cohere_h100_bound_and_fractions():
    g = json.load(open(GOLDEN))["cohere_h100"]
    sol = bench.sol_tokens_per_s(g["weight_bytes"] + g["kv_bytes"], g["hbm_bytes_per_s"])
    assert abs(sol - g["sol_tokens_per_s_approx"]) < 5
    assert round(100 * g["megakernel_tokens_per_s"] / sol) == g["megakernel_percent_of_sol"]
    assert round(100 * g["vllm_tokens_per_s"] / sol) == g["vllm_percent_of_sol"]
    assert round(g["megakernel_tokens_per_s"] / g["vllm_tokens_per_s"], 2) == g["speedup_vs_vllm"]


def test_kv_bytes_per_step_8b():
    # (p+1) x 32 layers x (K,V) x 8 heads x 128 x 2 B = (p+1) x 128 KiB
    assert bench.kv_read_bytes(syn.LLAMA8B, [0]) == 128 * 1024
    assert bench.kv_read_bytes(syn.LLAMA8B, [38, 40]) == 40 * 128 * 1024
