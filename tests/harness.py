"""Helpers shared by the GPU tests: upload seeded weights, run the layer, compare with the oracle."""
from __future__ import annotations

import dataclasses

import numpy as np

import synth

TOL_REL_L2 = 5e-3       # relative L2 error bound of every float output
TOL_MAX_REL = 1e-2      # max |err| <= TOL_MAX_REL * max |ref|


def to_device(arr: np.ndarray, device="cuda"):
    import torch
    if arr.dtype == np.uint16:
        return torch.from_numpy(arr.view(np.int16)).to(device)
    return torch.from_numpy(arr).to(device)


def upload_weights(W: dict, device="cuda") -> dict:
    return {k: to_device(np.ascontiguousarray(v), device) for k, v in W.items()}


def layer_dims(d: synth.Dims):
    from moe_decode_layer_moedec_b200 import LayerDims
    return LayerDims(d.hidden, d.latent, d.n_experts, d.top_k, d.expert_inter, d.shared_inter, 1)


def bf16_tensor_to_f32(t) -> np.ndarray:
    return synth.bf16_to_f32(t.cpu().numpy().view(np.uint16))


def rel_errors(got: np.ndarray, ref: np.ndarray):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    err = got - ref
    rel_l2 = float(np.linalg.norm(err) / max(np.linalg.norm(ref), 1e-300))
    max_rel = float(np.abs(err).max() / max(np.abs(ref).max(), 1e-300))
    return rel_l2, max_rel


# (config, tap) -> worst (relative L2, max|err|/max|ref|) seen by assert_close in this session;
# printed at the end of the run (tests/conftest.py), and written as JSON to $MOEDEC_PARITY_REPORT
MARGINS: dict = {}
_CONFIG = ["-"]


def set_config(name: str):
    """Label under which the following assert_close calls record their errors."""
    _CONFIG[0] = name


def assert_close(got, ref, name: str):
    rel_l2, max_rel = rel_errors(got, ref)
    key = (_CONFIG[0], name.split("[")[0])
    old = MARGINS.get(key, (0.0, 0.0))
    MARGINS[key] = (max(old[0], rel_l2), max(old[1], max_rel))
    assert rel_l2 <= TOL_REL_L2 and max_rel <= TOL_MAX_REL, \
        f"{name}: relative L2 {rel_l2:.3e} (bound {TOL_REL_L2}), max|err|/max|ref| {max_rel:.3e} (bound {TOL_MAX_REL})"
    return rel_l2, max_rel


def assert_logits_match(got: np.ndarray, ref: np.ndarray, name: str = "logits"):
    """fp32 logits from fp64 sums: identical except where the exact sum sits within fp64
    rounding of an fp32 rounding boundary (then they differ by one ulp)."""
    got = np.asarray(got, dtype=np.float32)
    ref = np.asarray(ref, dtype=np.float32)
    diff = got != ref
    if diff.any():
        ulps = np.abs(got.view(np.int32).astype(np.int64) - ref.view(np.int32).astype(np.int64))
        assert ulps[diff].max() <= 1, f"{name}: logits differ by more than one ulp"
        assert diff.sum() <= max(1, 1e-4 * diff.size), f"{name}: {int(diff.sum())} logits differ"


def oracle_scores(logits: np.ndarray) -> np.ndarray:
    """The oracle's fp32 score of every logit (same shape)."""
    import oracle
    flat = np.ascontiguousarray(logits, dtype=np.float32).ravel()
    return np.array([oracle.score(float(v)) for v in flat], dtype=np.float32).reshape(logits.shape)


def run_layer(layer, x_np: np.ndarray):
    """One step through the C ABI; returns (out fp32, idx, w, taps dict) as numpy."""
    import torch
    x = to_device(x_np)
    out = layer.step(x)
    B = x_np.shape[0]
    idx, w = layer.routing(B)
    taps = layer.taps(B)
    taps["scores"] = layer.scores(B)
    torch.cuda.synchronize()
    return (bf16_tensor_to_f32(out), idx.cpu().numpy(), w.cpu().numpy(),
            {k: v.cpu().numpy() for k, v in taps.items()})


def oracle_layer_of_shard(wd: synth.Dims, W: dict, shard):
    """The oracle's dims, weights and n_shared for one shard: the shard's arrays (from
    ep.shard_weights) in a full-size layer whose other experts have zero codes."""
    from moe_decode_layer_moedec_b200 import LayerDims
    from moe_decode_layer_moedec_b200 import ep
    d = LayerDims(wd.hidden, wd.latent, wd.n_experts, wd.top_k, wd.expert_inter, wd.shared_inter, 1)
    sd, SW = ep.shard_weights(d, W, shard)
    O = {n: W[n] for n in ("router", "w_down_lat", "w_up_lat")}
    e0, e1 = shard.expert_begin, shard.expert_begin + shard.expert_count
    for n in ("gate_q", "up_q", "down_q"):
        a = np.zeros_like(W[n])
        a[e0:e1] = SW[n]
        O[n] = a
    for n in ("gate_s", "up_s", "down_s"):
        a = np.full_like(W[n], 127)
        a[e0:e1] = SW[n]
        O[n] = a
    if sd.n_shared:
        for n in ("sh_gate_q", "sh_gate_s", "sh_up_q", "sh_up_s", "sh_down_q", "sh_down_s"):
            O[n] = np.ascontiguousarray(SW[n])
        od = dataclasses.replace(wd, shared_inter=shard.shared_count)
    else:  # no slice: the oracle is told there is no shared expert (its arrays are not read)
        od = dataclasses.replace(wd, shared_inter=128)
        H = wd.hidden
        for n, shape in (("sh_gate_q", (128, H // 2)), ("sh_gate_s", (128, H // 32)), ("sh_up_q", (128, H // 2)),
                         ("sh_up_s", (128, H // 32)), ("sh_down_q", (H, 64)), ("sh_down_s", (H, 4))):
            O[n] = np.zeros(shape, dtype=np.uint8)
    return od, O, sd.n_shared
