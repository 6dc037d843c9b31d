"""The seeded input generator: determinism, counter access, distributions, workload shape."""
import math

import numpy as np
import pytest

import synth


def test_splitmix64_reference_values():
    # SplitMix64 started from state 0: the published first outputs of the generator
    # (state += 0x9E3779B97F4A7C15, then the mix function).
    L = synth.lib()
    assert L.synth_draw(0, 0) == 0xE220A8397B1DCDAF
    assert L.synth_draw(0, 1) == 0x6E789E6AA1B965F4
    assert L.synth_draw(0, 2) == 0x06C45D188009454F


def test_counter_access_matches_sequential():
    key = synth.lib().synth_key(7, 3, synth.T_GATE_Q)
    full = synth._bytes(key, 1000)
    for start, n in ((0, 1), (5, 17), (8, 8), (993, 7), (100, 500)):
        assert np.array_equal(synth._bytes(key, n, start=start), full[start:start + n])
    sc = synth._scales(key, 300)
    assert np.array_equal(synth._scales(key, 50, start=250), sc[250:])


def test_determinism_and_stream_separation():
    w = synth.WORKLOADS["tiny_b1"]
    a, b = synth.layer_weights(w, 0), synth.layer_weights(w, 0)
    c = synth.layer_weights(w, 1)
    for k in synth.WEIGHT_NAMES:
        assert np.array_equal(a[k], b[k])
    assert not np.array_equal(a["gate_q"], c["gate_q"])
    assert not np.array_equal(a["gate_q"], a["up_q"])


def test_distributions():
    w = synth.WORKLOADS["tiny_b1"]
    W = synth.layer_weights(w, 0)
    codes = np.concatenate([(W["gate_q"] & 15).ravel(), (W["gate_q"] >> 4).ravel()])
    hist = np.bincount(codes, minlength=16) / codes.size
    assert np.all(np.abs(hist - 1 / 16) < 0.004)
    s = W["gate_s"].ravel()
    assert s.min() == 121 and s.max() == 125
    assert np.all(np.abs(np.bincount(s, minlength=126)[121:] / s.size - 0.2) < 0.01)
    for name, fan_in in (("router", 512), ("w_down_lat", 512), ("w_up_lat", 256)):
        v = synth.bf16_to_f32(W[name]).astype(np.float64)
        assert abs(v.mean()) < 0.01 / math.sqrt(fan_in) * 10
        assert abs(v.std() * math.sqrt(fan_in) - 1) < 0.01
    x = synth.bf16_to_f32(synth.tokens(synth.WORKLOADS["full_b16"])).astype(np.float64)
    assert abs(x.mean()) < 0.01 and abs(x.std() - 1) < 0.01


def test_bf16_rounding_is_rne_of_float():
    rng = np.random.default_rng(0)
    vals = rng.standard_normal(2000) * 3
    got = np.array([synth.lib().synth_bf16_from_double(float(v)) for v in vals], dtype=np.uint16)
    assert np.array_equal(got, synth.f32_to_bf16(vals.astype(np.float32)))
    # ties to even: 1 + 2^-8 sits halfway between bf16 1.0 and 1 + 2^-7
    assert synth.lib().synth_bf16_from_double(1 + 2 ** -8) == 0x3F80
    assert synth.lib().synth_bf16_from_double(1 + 3 * 2 ** -8) == 0x3F82


def test_perturbed_second_token():
    w = synth.WORKLOADS["full_b2"]
    x = synth.bf16_to_f32(synth.tokens(w)).astype(np.float64)
    d = x[1] - x[0]
    assert 0.09 < d.std() < 0.11


def test_hot_set_shape():
    w = synth.WORKLOADS["full_b64_skewed"]
    hs = synth.hot_set(w, 0)
    assert len(hs) == 32 and len(set(hs.tolist())) == 32 and hs.min() >= 0 and hs.max() < 896
    assert not np.array_equal(hs, synth.hot_set(w, 1))
    R0 = synth.router_weights(w, 0, beta=0.0)
    R1 = synth.router_weights(w, 0)
    cold = np.setdiff1d(np.arange(896), hs)
    assert np.array_equal(R0[cold], R1[cold]) and not np.array_equal(R0[hs], R1[hs])


@pytest.mark.slow
def test_skewed_workload_hot_share_near_half():
    import oracle
    w = synth.WORKLOADS["full_b64_skewed"]
    x = synth.tokens(w)
    shares = []
    for layer in range(w.layers):
        _, idx, _ = oracle.route(synth.router_weights(w, layer), x, w.dims.top_k)
        shares.append(np.isin(idx, synth.hot_set(w, layer)).mean())
    assert 0.45 <= float(np.mean(shares)) <= 0.55
