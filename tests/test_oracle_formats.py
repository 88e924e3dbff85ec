"""Pins for the oracle's number formats (bf16 and FP8 E4M3) against library casts
and hand-derived values; none of these re-types the oracle's own formula."""
import json
import os
import struct

import numpy as np
import pytest
import torch
from hypothesis import given, settings, strategies as st

from oracle import bf16_round, e4m3_encode, e4m3_decode, fp8_quantise_block, to_f32

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def test_bf16_matches_torch_cast_on_fp32_inputs():
    rng = np.random.default_rng(1)
    with np.errstate(over="ignore"):                                 # some become inf on purpose
        x = np.concatenate([
            rng.standard_normal(200000).astype(np.float32),
            (rng.standard_normal(20000) * 1e-39).astype(np.float32),     # bf16 subnormal range
            (rng.standard_normal(2000) * 3e38).astype(np.float32),       # near and past overflow
            np.array([0.0, -0.0, 1.0, -1.0], np.float32),
        ])
    ref = torch.tensor(x).to(torch.bfloat16).to(torch.float64).numpy()
    got = bf16_round(x.astype(np.float64))
    assert np.array_equal(np.isinf(ref), np.isinf(got))
    fin = np.isfinite(ref)
    assert np.array_equal(ref[fin], got[fin])


def test_bf16_single_rounding_golden():
    d = json.load(open(os.path.join(GOLD, "bf16_single_rounding.json")))
    for c in d["cases"]:
        x = struct.unpack("<d", int(c["x_hex"], 16).to_bytes(8, "little"))[0]
        want = float("inf") if c["bf16_value"] == "inf" else float(c["bf16_value"])
        got = float(bf16_round(np.array([x]))[0])
        assert got == want, (c["x_hex"], got, want, c["why"])


def test_e4m3_hand_codes():
    d = json.load(open(os.path.join(GOLD, "e4m3_hand_codes.json")))
    xs = np.array([c["x"] for c in d["cases"]])
    want = np.array([c["code"] for c in d["cases"]], np.uint8)
    got = e4m3_encode(xs)
    for x, w, g, c in zip(xs, want, got, d["cases"]):
        assert w == g, (x, hex(w), hex(g), c["why"])


def test_e4m3_all_codes_round_trip():
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], np.uint8)
    vals = e4m3_decode(codes)
    back = e4m3_encode(vals)
    # +0 and -0 both decode to zero; everything else must come back bit for bit
    nz = vals != 0
    assert np.array_equal(back[nz], codes[nz])
    assert e4m3_decode(np.array([0x7E]))[0] == 448.0
    assert e4m3_decode(np.array([0x01]))[0] == 2.0 ** -9
    assert np.isnan(e4m3_decode(np.array([0x7F]))[0])


def test_e4m3_matches_torch_cast_in_range():
    rng = np.random.default_rng(2)
    x = np.concatenate([
        rng.uniform(-448, 448, 100000),
        rng.standard_normal(100000),
        rng.standard_normal(50000) * 0.01,
    ]).astype(np.float32).astype(np.float64)
    ref = torch.tensor(x, dtype=torch.float32).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = e4m3_encode(x)
    # torch maps -0.0 results to 0x80 as we do; compare all codes bit for bit
    assert np.array_equal(ref, got)


def test_fp8_block_absmax_and_zero_block():
    rng = np.random.default_rng(3)
    x = to_f32(rng.standard_normal((16, 64)))
    i = np.unravel_index(np.argmax(np.abs(x)), x.shape)
    codes, scale, deq = fp8_quantise_block(x)
    assert scale == float(np.float32(np.abs(x).max() / 448.0))
    assert codes[i] in (0x7E, 0xFE)
    # values e4m3 * scale round-trip exactly
    codes2, scale2, deq2 = fp8_quantise_block(deq)
    assert np.array_equal(codes2, codes)
    z = np.zeros((16, 64))
    c0, s0, d0 = fp8_quantise_block(z)
    assert s0 == 0.0 and not c0.any() and not d0.any()


def test_fp8_block_error_bound():
    rng = np.random.default_rng(4)
    x = to_f32(rng.standard_normal((16, 64)) * 3.0)
    _, scale, deq = fp8_quantise_block(x)
    # E4M3 relative step is 2^-3 for normals: rounding error <= half a step, plus the
    # subnormal floor of half of 2^-9 * scale
    bound = np.maximum(np.abs(x) * 2.0 ** -4, 2.0 ** -10 * scale) * (1 + 1e-6)
    assert np.all(np.abs(deq - x) <= bound)


@settings(max_examples=30, deadline=None, derandomize=True)
@given(rows=st.integers(1, 16), cols=st.integers(1, 128), log2_mag=st.integers(-40, 40),
       outlier=st.floats(1.0, 1e4), seed=st.integers(0, 10 ** 6))
def test_fp8_block_matches_torch_float8_swept(rows, cols, log2_mag, outlier, seed):
    """Per-block absmax E4M3 quantisation against torch's float8 cast with an fp32 scale,
    over block shapes, magnitudes from 2^-40 to 2^40 (bf16 cache inputs) and outliers."""
    import brute
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((rows, cols)) * 2.0 ** log2_mag
    x.flat[rng.integers(x.size)] *= outlier
    x = bf16_round(x)
    _, _, deq = fp8_quantise_block(x)
    np.testing.assert_array_equal(deq, brute.fp8_dequant_torch(x))


# ---- dimension-adaptive FP8 ("XStreamVGGT" abstract; K per channel, V per token)

def test_dimension_adaptive_reduces_to_per_block_quantisation():
    from oracle import fp8_quantise_block, fp8_quantise_channels, fp8_quantise_tokens
    rng = np.random.default_rng(21)
    x = rng.standard_normal((16, 64)) * np.exp(rng.standard_normal(64))[None, :]
    x[:, 3] *= 1000.0                               # an outlier channel
    ck, sk, dk = fp8_quantise_channels(x)
    cv, sv, dv = fp8_quantise_tokens(x)
    for d in range(64):
        c, s_, q = fp8_quantise_block(x[:, d])
        assert np.array_equal(ck[:, d], c) and sk[d] == s_ and np.array_equal(dk[:, d], q)
    for i in range(16):
        c, s_, q = fp8_quantise_block(x[i])
        assert np.array_equal(cv[i], c) and sv[i] == s_ and np.array_equal(dv[i], q)


def test_dimension_adaptive_matches_torch_float8_per_channel_and_token():
    import brute
    from oracle import fp8_quantise_channels, fp8_quantise_tokens
    from oracle import bf16_round
    rng = np.random.default_rng(22)
    x = bf16_round(rng.standard_normal((16, 32)) * np.exp(2 * rng.standard_normal(32))[None, :])   # cache inputs
    _, _, dk = fp8_quantise_channels(x)
    _, _, dv = fp8_quantise_tokens(x)
    for d in range(32):
        np.testing.assert_array_equal(dk[:, d], brute.fp8_dequant_torch(x[:, d]))
    for i in range(16):
        np.testing.assert_array_equal(dv[i], brute.fp8_dequant_torch(x[i]))


def test_outlier_channel_costs_other_channels_nothing():
    """Per-block scales let one outlier channel flush its block's small values; per-channel
    scales keep every other channel at E4M3's relative precision (2^-4)."""
    from oracle import fp8_quantise_block, fp8_quantise_channels
    from oracle import bf16_round
    rng = np.random.default_rng(23)
    x = bf16_round(rng.uniform(0.5, 1.0, (16, 8)))
    x[:, 0] = 2.0 ** 20                             # the page's amax lives in channel 0
    _, _, blk = fp8_quantise_block(x)
    _, _, ch = fp8_quantise_channels(x)
    rel_ch = np.abs(ch[:, 1:] - x[:, 1:]) / x[:, 1:]
    assert rel_ch.max() <= 2.0 ** -4
    assert (blk[:, 1:] == 0).all()                  # x / (2^20 / 448) < 2^-10: below E4M3's subnormals
