"""The allocation-free router-logits entry point, checked against the oracle and the step.

Some callers cannot call cudaMalloc: code that runs while its stream is being captured into a
CUDA graph under a no-allocation policy, processes whose device memory is all handed to another
allocator, and runtimes with a fixed memory plan.  moedec_router_logits_noalloc serves them from
a static device array inside the library.  Its logits must equal the oracle's fp32 rounding of
the exact sums (up to a rare one-ulp difference where the exact sum sits on an fp32 rounding
boundary), and be bitwise equal to the logits of a step that runs the same router body (the
multi-kernel schedule), on two calls in a row (the array keeps the last call's contents).

This file runs last (pytest collects it last by name) and must pass both alone in a fresh
process and after the other GPU tests.
"""
import dataclasses

import numpy as np
import pytest

import oracle
import synth
from tests.harness import assert_logits_match, layer_dims, to_device, upload_weights

pytestmark = pytest.mark.gpu


def _multi_kernel_logits(w, W_dev, x_dev, B):
    import torch
    from moe_decode_layer_moedec_b200 import FLAG_MULTI_KERNEL, MoeDecodeLayer
    layer = MoeDecodeLayer(layer_dims(w.dims), W_dev, max_batch=B, flags=FLAG_MULTI_KERNEL)
    layer.step(x_dev)
    lg = layer.taps(B)["logits"]
    torch.cuda.synchronize()
    out = lg.cpu().numpy()
    layer.close()
    return out


def _twice(R_dev, x_dev, B, E):
    import torch
    from moe_decode_layer_moedec_b200 import router_logits_noalloc
    outs = []
    for _ in range(2):
        out = torch.full((B, E), float("nan"), device="cuda")
        router_logits_noalloc(R_dev, x_dev, logits=out)
        torch.cuda.synchronize()
        got = out.cpu().numpy()
        assert np.isfinite(got).all()
        outs.append(got)
    return outs


@pytest.mark.parametrize("name,B", [("tiny_b1", 1), ("tiny_b1", 64), ("full_b16", 16)])
def test_noalloc_logits_match_oracle_and_step_twice_in_a_row(name, B):
    import torch
    w = synth.WORKLOADS[name]
    W = synth.layer_weights(w, 0)
    W_dev = upload_weights(W)
    x = synth.tokens(w, step=7, batch=B)
    x_dev = to_device(x)
    ref = oracle.router_logits(W["router"], x)
    step = _multi_kernel_logits(w, W_dev, x_dev, B)
    for got in _twice(W_dev["router"], x_dev, B, w.dims.n_experts):
        assert_logits_match(got, ref, "noalloc logits vs oracle")
        assert np.array_equal(got, step), "noalloc logits differ from the step's router body"
    del W_dev
    torch.cuda.empty_cache()


@pytest.mark.parametrize("hidden,B", [(384, 8), (640, 3), (768, 9), (1280, 1)])
def test_noalloc_k_ranges_below_512(hidden, B):
    # hidden not a multiple of 512: K ranges of 128 (384, 640) or 256 (768, 1280) per split,
    # fewer than eight 32-element chunks per split
    d = dataclasses.replace(synth.TINY, hidden=hidden)
    w = synth.Workload(f"h{hidden}", d, B, 2000 + hidden)
    R = synth.router_weights(w, 0)
    x = synth.tokens(w, batch=B)
    ref = oracle.router_logits(R, x)
    for got in _twice(to_device(R), to_device(x), B, d.n_experts):
        assert_logits_match(got, ref, f"noalloc logits H={hidden}")


def test_noalloc_rejects_sizes_beyond_its_scratch_and_bad_arguments():
    import torch
    from moe_decode_layer_moedec_b200 import MoedecError, router_logits_noalloc
    w = synth.WORKLOADS["full_b16"]
    R = to_device(synth.router_weights(w, 0))
    x = to_device(synth.tokens(w, batch=21))   # 14 splits x 21 x 896 x 8 B > 2 MiB
    with pytest.raises(MoedecError, match="UNSUPPORTED"):
        router_logits_noalloc(R, x)
    out = router_logits_noalloc(R, x[:20])      # the largest batch that fits
    torch.cuda.synchronize()
    assert out.shape == (20, 896) and torch.isfinite(out).all()
    with pytest.raises(ValueError):
        router_logits_noalloc(R.t(), x[:2])     # not contiguous
    with pytest.raises(ValueError):
        router_logits_noalloc(R, x[:2], logits=torch.empty((2, 895), device="cuda"))
    with pytest.raises(ValueError):
        router_logits_noalloc(R, x[:2].float())
