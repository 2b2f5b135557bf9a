"""Pins for the seeded input generator (storage encodings, determinism)."""
import numpy as np

import synth


def test_bf16_known_encodings_and_ties():
    x = np.array([1.0, -2.0, 0.0, 3.140625, 1.0 + 2.0**-8, 1.0 + 3 * 2.0**-8, 65504.0], np.float32)
    bits = synth.to_bf16_bits(x)
    # 1.0 = 0x3F80, -2 = 0xC000; 1+2^-8 is a tie -> even (0x3F80); 1+3*2^-8 tie -> 0x3F82
    assert list(bits[:6]) == [0x3F80, 0xC000, 0x0000, 0x4049, 0x3F80, 0x3F82]
    back = synth.bf16_bits_to_f64(bits)
    assert back[0] == 1.0 and back[3] == 3.140625
    # every bf16 value is an fp32 value with 16 zero low bits
    y = synth.normal_f32(5, 1, (1000,))
    b = synth.bf16_bits_to_f64(synth.to_bf16_bits(y))
    assert np.max(np.abs(b - y) / np.abs(y)) <= 2.0**-8


def test_e4m3_known_encodings():
    bits, descale, deq = synth.quantize_e4m3(np.array([448.0, -448.0, 1.0, 2.0**-9], np.float32))
    # amax = 448 -> scale 1; 448 = 0x7E, -448 = 0xFE, 1.0 = 0x38, 2^-9 = min subnormal 0x01
    assert list(bits) == [0x7E, 0xFE, 0x38, 0x01]
    assert descale == 1.0
    np.testing.assert_array_equal(deq, [448.0, -448.0, 1.0, 2.0**-9])


def test_e4m3_amax_scaling():
    x = synth.normal_f32(3, 2, (4096,))
    bits, descale, deq = synth.quantize_e4m3(x)
    assert np.max(np.abs(deq)) <= np.max(np.abs(x)) * (1 + 2.0**-3)
    assert abs(np.max(np.abs(deq)) - np.max(np.abs(x))) <= np.max(np.abs(x)) * 2.0**-4
    rel = np.abs(deq - x) / np.maximum(np.abs(x), 1e-3)
    assert np.median(rel) < 2.0**-4


def test_streams_are_deterministic_and_independent():
    a = synth.normal_f32(1234, 1, (4, 5))
    b = synth.normal_f32(1234, 1, (4, 5))
    c = synth.normal_f32(1234, 2, (4, 5))
    np.testing.assert_array_equal(a, b)
    assert not np.array_equal(a, c)
    z = synth.normal_f32(7, 3, (200000,))
    assert abs(z.mean()) < 0.01 and abs(z.std() - 1) < 0.01


def test_attention_inputs_layout():
    inp = synth.attention_inputs(2, 3, 5, 8, seed=9, q_mult=8.0)
    assert inp["q_bits"].shape == (2, 3, 5, 8) and inp["q_bits"].dtype == np.uint16
    base = synth.attention_inputs(2, 3, 5, 8, seed=9)
    np.testing.assert_array_equal(inp["q"], 8.0 * base["q"])    # power of two: exact
    np.testing.assert_array_equal(inp["k"], base["k"])
    f8 = synth.attention_inputs(1, 2, 7, 16, seed=4, storage="e4m3")
    assert f8["q_bits"].dtype == np.uint8 and "do" not in f8
