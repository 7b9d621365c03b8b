"""The seeded input generator (test infrastructure) against its published
definition: SplitMix64 reference outputs, the Irwin-Hall transform and the
two rounding steps, and host/device bit identity."""
import json
import math
import os
import struct

import numpy as np
import pytest

import moe_inputs as mi

M64 = (1 << 64) - 1
GOLDEN = 0x9E3779B97F4A7C15


def splitmix64_out(z):
    z = (z + GOLDEN) & M64
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & M64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & M64
    return z ^ (z >> 31)


def f32_bits(v):
    return struct.unpack("<I", struct.pack("<f", v))[0]


def bf16_of(v):
    u = f32_bits(v)
    u = (u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFFFFFF
    return u >> 16


def test_splitmix64_reference_outputs():
    g = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "splitmix64_vectors.json")))
    got = [splitmix64_out((g["seed"] + i * GOLDEN) & M64) for i in range(5)]
    assert got == g["outputs"]


def test_host_hash_matches_definition():
    seed, tid, off = 3, 7, 123456789
    h = mi.host_hash(seed, tid, off, 16)
    for i in range(16):
        c = (seed << 56) | (tid << 48) | (off + i)
        assert int(h[i]) == splitmix64_out(c)


@pytest.mark.parametrize("bf16", [True, False])
def test_host_normal_matches_definition(bf16):
    seed, tid, off, n = 2, 3, 10**9, 64
    factor = (1.0 / math.sqrt(5120)) / mi.IRWIN_HALL4_SD
    out = mi.host_normal(seed, tid, off, n, factor, bf16)
    for i in range(n):
        h = splitmix64_out((seed << 56) | (tid << 48) | (off + i))
        s = (h & 0xFFFF) + ((h >> 16) & 0xFFFF) + ((h >> 32) & 0xFFFF) + (h >> 48)
        v = float(s - 131070) * factor
        f = struct.unpack("<f", struct.pack("<f", v))[0]
        if bf16:
            assert int(out[i]) == bf16_of(f)
        else:
            assert float(out[i]) == f


def test_host_uniform_matches_definition():
    out = mi.host_uniform(4, 2, 0, 32, -0.1, 0.1, False)
    for i in range(32):
        h = splitmix64_out((4 << 56) | (2 << 48) | i)
        u = float(h >> 11) * 2.0 ** -53
        v = -0.1 + (0.1 - -0.1) * u
        assert float(out[i]) == struct.unpack("<f", struct.pack("<f", v))[0]


def test_distribution_moments_and_shapes():
    s = mi.SHAPES["v3_prefill_bf16"]
    w = mi.bf16_to_f32(mi.host_tensor(s, "W1", 0, 1 << 20)).astype(np.float64)
    assert abs(w.mean()) < 1e-3 / math.sqrt(s.d) * 10
    assert abs(w.std() * math.sqrt(s.d) - 1.0) < 5e-3
    x = mi.bf16_to_f32(mi.host_tensor(s, "x", 0, 1 << 20)).astype(np.float64)
    assert abs(x.std() - 1.0) < 5e-3 and abs(x).max() <= math.sqrt(12) * 1.01
    assert mi.dims_of(s, "W1") == (256, 2048, 7168) and mi.dims_of(s, "Ws2") == (7168, 2048)


def test_decode_shape_zipf_offsets():
    s = mi.SHAPES["v3_decode_bf16"]
    o = mi.zipf_offsets(s)
    ranks = np.rint(np.exp(-o / 1.2)).astype(int)
    assert sorted(ranks.tolist()) == list(range(1, 257))
    x = mi.host_rows(s, "x", [0, 5])
    assert (mi.bf16_to_f32(x[:, 0]) == 1.0).all()
    w = mi.host_rows(s, "W_r", [0, 1, 2])
    np.testing.assert_allclose(mi.bf16_to_f32(w[:, 0]), o[:3], rtol=2 ** -8)


def test_slices_are_order_independent():
    s = mi.SHAPES["v2_layer_bf16"]
    whole = mi.host_tensor(s, "W2", 1000, 5000)
    a = mi.host_tensor(s, "W2", 1000, 2000)
    b = mi.host_tensor(s, "W2", 3000, 3000)
    assert (np.concatenate([a, b]) == whole).all()


@pytest.mark.gpu
def test_device_generator_matches_host():
    import torch
    from moe_inputs import build, device
    build.build_device()
    for name in ("gshard_tiny_f32", "v3_decode_bf16"):
        s = mi.SHAPES[name]
        for nm in ("x", "W_r", "W2", "b"):
            if nm == "b" and not s.bias:
                continue
            t = device.device_tensor(s, nm)
            torch.cuda.synchronize()
            n = min(t.numel(), 1 << 20)
            dev = t.reshape(-1)[:n].cpu()
            dev = dev.view(torch.int16).numpy().view(np.uint16) if t.dtype == torch.bfloat16 else dev.numpy()
            host = mi.host_tensor(s, nm, 0, n)
            assert (dev == host).all(), (name, nm)


def _e4m3_nearest(x):
    """Nearest finite E4M3 code to x by brute force over the code table, ties
    to the even code (the one whose mantissa LSB is 0), saturating at 448."""
    vals = []
    for c in range(0x7F):
        e, m = c >> 3, c & 7
        vals.append(m * 2.0 ** -9 if e == 0 else (1 + m / 8) * 2.0 ** (e - 7))
    vals = np.array(vals)
    a = min(abs(x), 448.0)
    d = np.abs(vals - a)
    best = np.flatnonzero(d == d.min())
    c = int(best[0]) if len(best) == 1 else int([b for b in best if b % 2 == 0][0])
    return c | (0x80 if x < 0 else 0)


def test_fp8_generator_matches_definition():
    # codes: nearest e4m3 to v * 2^-e_b with the block exponent from the
    # scale tensor's hash; scales: e_b + 127
    s = mi.SHAPES["v3_prefill_fp8"]
    nm = "W1"
    rows, cols = mi.mat_dims(s, nm)
    e0 = mi.fp8_e0(s, nm)
    idx = np.concatenate([np.arange(0, 300), np.arange(5 * cols + 100, 5 * cols + 400),
                          np.arange(200 * cols + 7000, 200 * cols + 7168)])
    codes = np.concatenate([mi.host_fp8(s, nm, int(i), 1) for i in idx])
    factor = mi.factor_of(s, nm)
    for i, code in zip(idx.tolist(), codes.tolist()):
        h = mi.host_hash(s.seed, mi.TID[nm], i, 1)[0]
        sm = int(h & 0xFFFF) + int((h >> 16) & 0xFFFF) + int((h >> 32) & 0xFFFF) + int(h >> 48)
        v = float(sm - 131070) * factor
        r, c = divmod(i, cols)
        blk = (r // 128) * (cols // 128) + c // 128
        eb = e0 + int(mi.host_hash(s.seed, mi.TID_SCALE[nm], blk, 1)[0] & 3)
        assert code == _e4m3_nearest(math.ldexp(v, -eb)), (i, hex(code))
        assert int(mi.host_fp8_scales(s, nm, blk, 1)[0]) == eb + 127
    # the largest value the generator makes still fits: codes never saturate
    assert 131070 * factor <= 448 * 2.0 ** e0


def test_fp8_expert_slices_are_the_stacked_matrix():
    s = mi.SHAPES["v3_decode_fp8"]
    (q1, s1), _, (q2, s2) = mi.host_expert_fp8(s, 3)
    F, d = s.d_ff, s.d
    assert q1.shape == (F, d) and s1.shape == (F // 128, d // 128)
    assert np.array_equal(q1[:2].reshape(-1), mi.host_fp8(s, "W1", 3 * F * d, 2 * d))
    assert np.array_equal(s2.reshape(-1)[:5], mi.host_fp8_scales(s, "W2", 3 * (d // 128) * (F // 128), 5))


@pytest.mark.gpu
def test_device_fp8_generator_matches_host():
    import torch
    from moe_inputs import build, device
    build.build_device()
    s = mi.SHAPES["v3_decode_fp8"]
    for nm in ("W1", "W2", "Ws2"):
        q, sc = device.device_fp8(s, nm)
        torch.cuda.synchronize()
        n = min(q.numel(), 1 << 21)
        assert np.array_equal(q.reshape(-1)[:n].cpu().numpy(), mi.host_fp8(s, nm, 0, n)), nm
        assert np.array_equal(sc.reshape(-1).cpu().numpy(), mi.host_fp8_scales(s, nm)), nm
