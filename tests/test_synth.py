"""Input generator: determinism, slice independence and the recipe's distributions."""
import math

import numpy as np
import pytest

import synth


def test_splitmix64_reference_values():
    # SplitMix64 started from state 0 (Steele, Lea & Flood 2014; the same sequence is the
    # seeding generator of xoshiro/xoroshiro): first outputs are published constants.
    want = [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F]
    got = [int(v) for v in synth.draws(0, 0, 3)]
    assert got == want


def test_slices_are_pure_functions_of_index():
    key = synth.stream_key(7, synth.K_X, 3, 5)
    full = synth.normals(key, 0, 1000)
    assert np.array_equal(full[317:700], synth.normals(key, 317, 383))
    b = synth.random_bytes(key, 0, 999)
    assert np.array_equal(b[13:501], synth.random_bytes(key, 13, 488))


def test_own_ln_cos_close_to_libm():
    u = synth.uniforms(synth.stream_key(1, 9), 0, 200000)
    assert np.max(np.abs(synth.ln_series(u) - np.log(u)) / np.abs(np.log(u))) < 1e-15
    assert np.max(np.abs(synth.cos_turns(u) - np.cos(2 * np.pi * u))) < 1e-15


def test_normal_moments():
    z = synth.normals(synth.stream_key(0, synth.K_X, 0, 0), 0, 400000)
    assert abs(z.mean()) < 0.01 and abs(z.std() - 1) < 0.01
    assert abs(np.mean(z ** 4) - 3) < 0.05


def test_recipe_distributions():
    w = synth.WORKLOADS["decode_t1_l48_h2048_e256_k8_i512_int4"]
    wr = synth.router_weights(w, 0)
    assert abs(wr.std() * math.sqrt(w.H) - 1) < 0.01
    ex = synth.expert_tensors(w, 0, 3)
    s = synth.f16_bits_to_f64(ex["scale"][0])
    assert s.min() >= 1e-3 and abs((s - 1e-3).mean() - math.sqrt(0.02) * math.sqrt(2 / math.pi)) < 0.005
    z = synth.f16_bits_to_f64(ex["zero"][0])
    assert z.min() >= 0 and z.max() <= 15 and abs(z.mean() - 7.5) < 0.1
    q = synth.unpack_codes(ex["codes"][0][:64], 4, w.H)
    assert q.min() == 0 and q.max() == 15 and abs(q.mean() - 7.5) < 0.1


def test_mixed_bits_and_zipf():
    w = synth.WORKLOADS["decode_t16_l24_h2048_e256_k8_i768_mixed468_zipf1.1"]
    b = synth.expert_bits(w, 5)
    assert (b == 8).sum() == 26 and (b == 6).sum() == 77 and (b == 4).sum() == 153
    assert not np.array_equal(b, synth.expert_bits(w, 6))
    bias = synth.router_bias(w, 5)
    assert np.isclose(np.sort(bias)[::-1], -1.1 * np.log(np.arange(1, 257))).all()
    ex = synth.expert_tensors(w, 5, int(np.argmax(b == 6)))
    assert ex["bits"] == 6 and ex["codes"][2].shape == (w.H, w.I * 6 // 8)
