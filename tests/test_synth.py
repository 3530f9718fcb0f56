"""Pins for the shared input generator (SplitMix64 + Box-Muller), CPU only."""
import numpy as np
import pytest

import synth


def test_splitmix64_published_sequence():
    # SplitMix64 seeded with state 0 (Steele, Lea and Flood 2014; the widely reproduced reference
    # sequence): the first two outputs.
    assert synth.raw(0, 0) == 0xE220A8397B1DCDAF
    assert synth.raw(0, 1) == 0x6E789E6AA1B965F4


def test_slices_are_consistent():
    a = synth.normal_bf16(7, 3, 0, 0, 10001, 0.02)
    for start in (0, 1, 2, 999, 5000):
        b = synth.normal_bf16(7, 3, 0, start, 37, 0.02, threads=1)
        assert np.array_equal(a[start:start + 37], b)


def test_threads_do_not_change_values():
    a = synth.normal_f32(1, 2, 0, 123, 300001, 1.0, threads=1)
    b = synth.normal_f32(1, 2, 0, 123, 300001, 1.0, threads=7)
    assert np.array_equal(a, b)


def test_streams_and_attempts_differ():
    a = synth.normal_bf16(0, 1, 0, 0, 1000, 1.0)
    b = synth.normal_bf16(0, 1, 1, 0, 1000, 1.0)
    c = synth.normal_bf16(0, 2, 0, 0, 1000, 1.0)
    d = synth.normal_bf16(1, 1, 0, 0, 1000, 1.0)
    for o in (b, c, d):
        assert np.mean(a == o) < 0.05


def test_normal_moments():
    z = synth.normal_f32(0, 9, 0, 0, 2_000_000, 1.0).astype(np.float64)
    assert abs(z.mean()) < 5e-3
    assert abs(z.std() - 1.0) < 5e-3
    assert abs(np.mean(z ** 4) - 3.0) < 0.05  # kurtosis of a normal
    assert abs(np.mean(np.abs(z) < 1.0) - 0.6827) < 2e-3


def test_bf16_rounding_matches_fp32_rounding_path():
    # The generator rounds std*z (double) once to bf16.  Except in the rare case where rounding to
    # fp32 first creates a tie, that equals rounding the fp32 value to bf16.
    std = 0.02
    bits = synth.normal_bf16(3, 4, 0, 0, 200000, std)
    f32 = synth.normal_f32(3, 4, 0, 0, 200000, std)
    via = synth.f32_to_bf16_bits(f32)
    assert np.mean(bits == via) > 0.9999


def test_workloads_shapes():
    wl = synth.WORKLOADS["tiny"]
    x = synth.gen_x(wl)
    assert x.shape == (64, 256) and x.dtype == np.uint16
    w1 = synth.gen_expert(wl, "w1", 3)
    w2 = synth.gen_expert(wl, "w2", 3)
    assert w1.shape == (512, 256) and w2.shape == (256, 512)
    all_w1 = synth.gen_experts(wl, "w1")
    assert np.array_equal(all_w1[3], w1)
    # per-row attempts redraw only that row
    att = np.zeros(wl.T, dtype=np.int64)
    att[5] = 2
    x2 = synth.gen_x(wl, attempts=att)
    assert np.array_equal(np.delete(x2, 5, 0), np.delete(x, 5, 0))
    assert not np.array_equal(x2[5], x[5])
    assert synth.gen_bias(synth.WORKLOADS["skewed"])[[3, 11]].tolist() == [2.0, 2.0]


def test_mlp_workloads_draw_their_own_weights():
    wl = synth.MLP_WORKLOADS["mlp_tiny"]
    assert wl.E == 1 and wl.K == 1 and wl.layer == "mlp"
    w1 = synth.gen_experts(wl, "w1")
    assert w1.shape == (1, 512, 256)
    # same shape as the tiny MoE layer's expert 0, but another stream
    assert not np.array_equal(w1[0], synth.gen_expert(synth.WORKLOADS["tiny"], "w1", 0))
    assert set(synth.ALL_WORKLOADS) == set(synth.WORKLOADS) | set(synth.MLP_WORKLOADS)
