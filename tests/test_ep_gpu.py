"""GPU parity of the expert-parallel step: every rank's shard of a layer on one device.

The ranks are emulated in rank order on one stream: each rank's partial step, then each rank's
publish, then each rank's combine (`ep.EmulatedExpertParallel`).  No kernel waits for one that
has not run: every combine finds its flags already set.  Checked against the oracle:
  - each rank's routing bit-exactly (every rank routes over all experts);
  - each rank's fp32 partial output against the oracle's output for that shard (its arrays in a
    full-size layer whose other experts have zero codes), at the float tolerance;
  - the combined bf16 output against the oracle's output for the whole layer, at the float
    tolerance, and bit-identical on every rank.
Cases: worlds 1-4 and 8, batches 1-65 (small-batch and split-K steps, a shard with no selection at
all), the three step schedules, epochs that reuse the partial buffers, a combine whose flags never
come (bounded wait, reported as MOEDEC_ERR_TIMEOUT), and the full-size layer at 16 tokens over 8
ranks.
"""
import numpy as np
import pytest

import oracle
import synth
from tests.harness import (assert_close, bf16_tensor_to_f32, layer_dims, oracle_layer_of_shard, set_config, to_device,
                           upload_weights)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def tiny():
    import torch
    assert torch.cuda.is_available()
    w = synth.WORKLOADS["tiny_b1"]
    W = synth.layer_weights(w, 0)
    return w, W, upload_weights(W)


def _flags(schedule: str) -> int:
    from moe_decode_layer_moedec_b200 import FLAG_MULTI_KERNEL, FLAG_NO_TMA_RING
    return {"fused": 0, "multi": FLAG_MULTI_KERNEL, "noring": FLAG_NO_TMA_RING}[schedule]


def _check_group(w, W, grp, x_np, label, shard_partials=True, tokens=None):
    import torch
    x = to_device(x_np)
    outs, parts = grp.step(x)
    B = x_np.shape[0]
    routes = [layer.routing(B) for layer in grp.layers]
    torch.cuda.synchronize()
    tok = range(B) if tokens is None else tokens
    full = oracle.step(w.dims, W, x_np, tokens=tok)
    set_config(label)
    ref_bits = outs[0].cpu().numpy().view(np.uint16)
    for r, o in enumerate(outs):
        assert np.array_equal(o.cpu().numpy().view(np.uint16), ref_bits), f"{label}: rank {r} output differs"
    got = bf16_tensor_to_f32(outs[0])[tok.start:tok.stop]
    assert_close(got, full["out"], f"{label} out")
    for r, (idx, wts) in enumerate(routes):
        assert np.array_equal(idx.cpu().numpy()[tok.start:tok.stop], full["idx"]), f"{label}: rank {r} routing"
        assert np.array_equal(wts.cpu().numpy()[tok.start:tok.stop], full["w"]), f"{label}: rank {r} weights"
    if shard_partials:
        for r, s in enumerate(grp.shards):
            od, O, ns = oracle_layer_of_shard(w.dims, W, s)
            ref = oracle.step(od, O, x_np, tokens=tok, n_shared=ns)["out"]
            assert_close(parts[r].cpu().numpy()[tok.start:tok.stop], ref, f"{label} partial[{r}]")
    total = sum(p.double().cpu().numpy()[tok.start:tok.stop] for p in parts)
    assert_close(total, full["out"], f"{label} sum of partials")
    return outs


@pytest.mark.parametrize("schedule", ["fused", "multi", "noring"])
@pytest.mark.parametrize("world", [1, 2, 3, 4])
@pytest.mark.parametrize("B", [1, 3, 9, 65])
def test_ep_tiny_parity(tiny, world, B, schedule):
    from moe_decode_layer_moedec_b200 import ep
    w, W, W_dev = tiny
    grp = ep.EmulatedExpertParallel(layer_dims(w.dims), W_dev, world, max_batch=B, flags=_flags(schedule))
    try:
        _check_group(w, W, grp, synth.tokens(w, step=3, batch=B), f"ep tiny G{world} B{B} {schedule}")
    finally:
        grp.close()


def test_ep_shard_with_no_selection(tiny):
    # 16 ranks of 4 experts: at one token (top-4) most shards have no selected expert and, but for
    # the last two, no shared slice either; their partial outputs are exactly zero
    from moe_decode_layer_moedec_b200 import ep
    w, W, W_dev = tiny
    grp = ep.EmulatedExpertParallel(layer_dims(w.dims), W_dev, 16, max_batch=1)
    try:
        x = synth.tokens(w, step=1, batch=1)
        _check_group(w, W, grp, x, "ep tiny G16 B1")
        idx = oracle.step(w.dims, W, x)["idx"][0]
        _, parts = grp.step(to_device(x))
        idle = [r for r, s in enumerate(grp.shards)
                if s.shared_count == 0 and not any(s.expert_begin <= e < s.expert_begin + s.expert_count for e in idx)]
        assert idle
        for r in idle:
            assert not parts[r].cpu().numpy().any(), r
    finally:
        grp.close()


def test_ep_epochs_reuse_the_partial_buffers(tiny):
    from moe_decode_layer_moedec_b200 import ep
    w, W, W_dev = tiny
    grp = ep.EmulatedExpertParallel(layer_dims(w.dims), W_dev, 3, max_batch=65)
    try:
        for step, B in enumerate([3, 9, 1, 65, 2]):
            _check_group(w, W, grp, synth.tokens(w, step=10 + step, batch=B), f"ep tiny G3 epoch{step + 1} B{B}",
                         shard_partials=False)
        assert grp.clock.epoch == 5
    finally:
        grp.close()


def test_ep_combine_times_out_without_flags(tiny):
    # rank 1 never publishes: rank 0's combine waits (bounded, 1 s), leaves its output unwritten,
    # and the next synchronising call of rank 0's handle reports MOEDEC_ERR_TIMEOUT; afterwards a
    # full step works (epochs only grow, so the late flags of the stalled epoch do no harm)
    import torch
    from moe_decode_layer_moedec_b200 import MoedecError, ep
    w, W, W_dev = tiny
    grp = ep.EmulatedExpertParallel(layer_dims(w.dims), W_dev, 2, max_batch=4)
    try:
        B = 4
        x = to_device(synth.tokens(w, step=2, batch=B))
        epoch, parity = grp.clock.next()
        for r, layer in enumerate(grp.layers):
            layer.step_partial(x, grp.parts[r, parity])
        grp.layers[0].ep_publish([grp.flag_ptr(q, 0) for q in range(2)], epoch)
        out = torch.full((B, w.dims.hidden), 0x40E0, dtype=torch.int16, device="cuda")  # bf16 7.0
        grp.layers[0].ep_combine([grp.parts[g, parity].data_ptr() for g in range(2)], grp.flag_ptr(0, 0), epoch, B,
                                 out)
        with pytest.raises(MoedecError, match="TIMEOUT"):
            grp.layers[0].routing(B)
        assert bool((out == 0x40E0).all())
        _check_group(w, W, grp, synth.tokens(w, step=4, batch=B), "ep tiny G2 after a combine timeout",
                     shard_partials=False)
    finally:
        grp.close()


def test_step_partial_of_a_whole_layer_takes_the_small_batch_kernel():
    # the streaming schedule writes bf16 only: a partial step of a handle created with
    # MOEDEC_FLAG_STREAM runs the small-batch kernel instead (one launch, not four).  The mid-size
    # layer: every dimension a multiple of 512, so its full steps do take the streaming schedule
    from moe_decode_layer_moedec_b200 import FLAG_STREAM, MoeDecodeLayer
    w = synth.WORKLOADS["mid_b2"]
    W = synth.layer_weights(w, 0)
    W_dev = upload_weights(W)
    layer = MoeDecodeLayer(layer_dims(w.dims), W_dev, max_batch=2, flags=FLAG_STREAM)
    launches = lambda: sum(layer.launch_counts().values())
    try:
        for B in (1, 2):
            x_np = synth.tokens(w, step=7, batch=B)
            before = launches()
            part = layer.step_partial(to_device(x_np))
            assert launches() - before == 1
            set_config(f"partial mid B{B} stream flag")
            assert_close(part.cpu().numpy(), oracle.step(w.dims, W, x_np)["out"], f"partial mid B{B}")
            before = launches()
            layer.step(to_device(x_np))
            assert launches() - before == layer.kernels_per_step(B) == 4
    finally:
        layer.close()


def test_ipc_export_names_the_allocation_and_the_offset():
    import torch
    from moe_decode_layer_moedec_b200 import IPC_HANDLE_BYTES, ipc_export
    buf = torch.empty(1 << 22, dtype=torch.uint8, device="cuda")
    h0, o0 = ipc_export(buf.data_ptr())
    h1, o1 = ipc_export(buf[8192:].data_ptr())
    assert len(h0) == IPC_HANDLE_BYTES and h0 == h1 and o1 - o0 == 8192


def test_ep_full_b16_over_8_ranks():
    # the full-size layer at 16 tokens, split over 8 ranks (112 experts and 256 shared columns
    # each), TMA-ring split-K step on every rank: all tokens' routing, 4 tokens' outputs
    import torch
    from moe_decode_layer_moedec_b200 import ep
    w = synth.WORKLOADS["full_b16"]
    W = synth.layer_weights(w, 0)
    W_dev = upload_weights(W)
    grp = ep.EmulatedExpertParallel(layer_dims(w.dims), W_dev, 8, max_batch=16)
    try:
        assert all(layer.tma_ring() for layer in grp.layers)
        x = synth.tokens(w, batch=16)
        xd = to_device(x)
        outs, parts = grp.step(xd)
        _, idx_ref, w_ref = oracle.route(W["router"], x, w.dims.top_k)
        for layer in grp.layers:
            idx, wts = layer.routing(16)
            assert np.array_equal(idx.cpu().numpy(), idx_ref) and np.array_equal(wts.cpu().numpy(), w_ref)
        _check_group(w, W, grp, x, "ep full_b16 G8", shard_partials=False, tokens=range(0, 4))
    finally:
        grp.close()
        del W_dev
        torch.cuda.empty_cache()
