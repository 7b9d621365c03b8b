"""bench.py host helpers on CPU: the algorithmic FLOP and byte counts the
roofline fractions divide by, the oracle sample sizing, the reference arm's
JSON line on the toy layer, the timed loops' event wait and the clock
summary."""
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


def test_wait_event_polls_until_the_event_completes():
    class FakeEvent:
        def __init__(self, n):
            self.left = n

        def query(self):
            self.left -= 1
            return self.left < 0

    ev = FakeEvent(3)
    bench.wait_event(ev, poll_s=0.0)
    assert ev.left == -1  # queried until it reported completion, and no further


def test_clock_summary_counts_throttle_reasons():
    c = bench.ClockSampler(None)
    assert c.summary()["reasons"] == ["unsampled"]
    c.max_mhz = 1965.0
    c.samples = [(1965.0, 0), (1500.0, 0x4), (1400.0, 0x4 | 0x40)]
    s = c.summary()
    assert s["sm_mhz"] == 1500.0 and s["sm_min_mhz"] == 1400.0 and s["samples"] == 3
    assert s["reasons"] == ["hw_thermal_slowdown", "sw_power_cap"]
    assert s["reason_samples"] == {"sw_power_cap": 2, "hw_thermal_slowdown": 1}
