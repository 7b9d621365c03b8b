"""bench.py host helpers on CPU: the algorithmic FLOP and byte counts the
roofline fractions divide by, the oracle sample sizing, and the reference
arm's JSON line on the toy layer."""
import json

import numpy as np

import bench
import moe_inputs as mi


def test_algorithmic_counts_v3_prefill():
    s = mi.SHAPES["v3_prefill_bf16"]
    counts = np.full(s.n_routed, s.T * s.top_k // s.n_routed)  # every expert touched
    A = bench.algorithmic(s, counts)
    assert A["U"] == 256
    # FLOPs = T (k + n_s) 6 d d_ff: three d x d_ff matrices per selected or shared expert, 2 FLOPs per MAC
    assert A["flops"] == 4096 * 9 * 6 * 7168 * 2048
    # touched expert weights (3 matrices of d x d_ff per expert, bf16) + router + x in + y out
    assert A["layer_bytes"] == 257 * 3 * 7168 * 2048 * 2 + 256 * 7168 * 2 + 2 * 4096 * 7168 * 2
    assert abs(257 * 3 * 7168 * 2048 * 2 / 1e9 - 22.64) < 0.01  # the 22.6 GB of weights the bench states
    # SwiGLU GEMM, algorithmic: W1, W3 of touched experts + shared, x read once
    assert A["swiglu_alg"] == 257 * 2 * 7168 * 2048 * 2 + 4096 * 7168 * 2
    # and with the implementation's token-row reads and h writes
    R = 4096 * 8
    assert A["swiglu_impl"] == 257 * 2 * 7168 * 2048 * 2 + (R + 4096) * 7168 * 2 + (R + 4096) * 2048 * 2


def test_untouched_experts_do_not_count():
    s = mi.SHAPES["v3_decode_bf16"]
    counts = np.zeros(s.n_routed, dtype=np.int64)
    counts[:57] = 1
    A = bench.algorithmic(s, counts)
    assert A["U"] == 57
    assert A["layer_bytes"] == 58 * 3 * 7168 * 2048 * 2 + 256 * 7168 * 2 + 2 * 128 * 7168 * 2


def test_sample_token_cap_bounds():
    s = mi.SHAPES["v3_prefill_bf16"]
    n = bench.sample_token_cap(s, 4)
    assert 1 <= n <= 4
    assert bench.sample_token_cap(s, 1) == 1


def test_reference_arm_line_on_the_toy_layer(capsys):
    assert bench.main(["--impl", "reference", "--config", "gshard_tiny_f32", "--steps", "3", "--warmup", "3"]) == 0
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["metric"] == bench.METRIC
    assert line["value"] > 0 and line["unit"] == "tokens/s" and line["higher_is_better"] is True
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["value"] == line["value"]
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
