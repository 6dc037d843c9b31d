"""The allocation-free router-logits entry point against the step's own logits.

Some callers cannot call cudaMalloc (a stream being captured under a no-allocation policy, a
device whose memory another allocator owns, a fixed memory plan).  moedec_router_logits_noalloc
serves them from a static device array.  This file runs last (pytest collects it last by name)
and must pass both alone in a fresh process and after the other GPU tests.
"""
import numpy as np
import pytest

import synth
from tests.harness import assert_logits_match, layer_dims, to_device, upload_weights

pytestmark = pytest.mark.gpu


def _step_logits(w, W_dev, x_dev, B):
    import torch
    from moe_decode_layer_moedec_b200 import MoeDecodeLayer
    layer = MoeDecodeLayer(layer_dims(w.dims), W_dev, max_batch=B)
    layer.step(x_dev)
    lg = layer.taps(B)["logits"]
    torch.cuda.synchronize()
    out = lg.cpu().numpy()
    layer.close()
    return out


@pytest.mark.parametrize("name,B", [("tiny_b1", 1), ("tiny_b1", 64), ("full_b16", 16)])
def test_noalloc_logits_match_the_step_twice_in_a_row(name, B):
    import torch
    from moe_decode_layer_moedec_b200 import router_logits_noalloc
    w = synth.WORKLOADS[name]
    W = synth.layer_weights(w, 0)
    W_dev = upload_weights(W)
    x = synth.tokens(w, step=7, batch=B)
    x_dev = to_device(x)
    ref = _step_logits(w, W_dev, x_dev, B)
    for _ in range(2):
        out = torch.full((B, w.dims.n_experts), float("nan"), device="cuda")
        router_logits_noalloc(W_dev["router"], x_dev, logits=out)
        torch.cuda.synchronize()
        got = out.cpu().numpy()
        assert np.isfinite(got).all()
        assert_logits_match(got, ref, "noalloc logits")
    del W_dev
    torch.cuda.empty_cache()


def test_noalloc_rejects_sizes_beyond_its_scratch():
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
