"""GPU parity: the CUDA step through the C ABI against the CPU oracle, element by element.

Routing indices must match bit-exactly; every float output (out, and the h / ylat / sh / up
taps, checked separately because the shared expert dominates the magnitude of out) must meet
relative L2 <= 5e-3 and max|err| <= 1e-2 * max|ref|.  Sizes: the tiny layer at several batches
(ragged n-tiles, every token checked) and the full-size layer in the launch configuration the
bench times (all tokens' routing, sampled tokens' outputs).
"""
import numpy as np
import pytest

import oracle
import synth
from tests.harness import (assert_close, assert_logits_match, bf16_tensor_to_f32, layer_dims, oracle_scores, rel_errors,
                           run_layer, set_config, to_device, upload_weights)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def torch_cuda():
    import torch
    assert torch.cuda.is_available()
    return torch


SCHEDULES = ["fused", "multi", "stream"]


def _make_layer(w, W_dev, max_batch, flags=None, schedule="fused"):
    # schedules: "fused" (the default), "multi" (eight stream-ordered kernels), "stream" (the
    # streaming small-batch kernel at 1-2 tokens), "noring" (fused, with the split-K step's
    # routed experts on register-fed loads instead of the per-warp TMA rings)
    from moe_decode_layer_moedec_b200 import (FLAG_MULTI_KERNEL, FLAG_NO_TMA_RING, FLAG_STREAM, FLAG_TAPS,
                                              MoeDecodeLayer)
    f = FLAG_TAPS if flags is None else flags
    if schedule == "multi":
        f |= FLAG_MULTI_KERNEL
    if schedule == "stream":
        f |= FLAG_STREAM
    if schedule == "noring":
        f |= FLAG_NO_TMA_RING
    return MoeDecodeLayer(layer_dims(w.dims), W_dev, max_batch=max_batch, flags=f)


_ORACLE_CACHE: dict = {}


def _oracle_rows(w, W, x, toks, layer_idx=0):
    """oracle.step rows of the tokens `toks` of x, cached per token (the oracle does not depend on
    the schedule); one oracle call over all tokens when most of them are asked for."""
    key = (w.name, w.dims, layer_idx, x.shape, hash(x.tobytes()), hash(W["router"].tobytes()))
    if _ORACLE_CACHE.get("key") != key:
        _ORACLE_CACHE.clear()
        _ORACLE_CACHE["key"] = key
    toks = list(toks)
    missing = [t for t in toks if t not in _ORACLE_CACHE]
    if len(missing) > x.shape[0] // 2:
        r = oracle.step(w.dims, W, x)
        for t in range(x.shape[0]):
            _ORACLE_CACHE[t] = {k: v[t] for k, v in r.items()}
    else:
        for t in missing:
            r = oracle.step(w.dims, W, x, tokens=range(t, t + 1))
            _ORACLE_CACHE[t] = {k: v[0] for k, v in r.items()}
    return {t: _ORACLE_CACHE[t] for t in toks}


def _check_step(w, W, x, layer, tokens=None, check_all_routing=True, label=None, layer_idx=0):
    out, idx, wts, taps = run_layer(layer, x)
    B = x.shape[0]
    set_config(label or f"{w.name} B{B}")
    if check_all_routing:
        lg, ridx, rw = oracle.route(W["router"], x, w.dims.top_k)
        assert np.array_equal(idx, ridx), "routing indices differ from the oracle"
        np.testing.assert_allclose(wts, rw, rtol=2e-6, atol=0)
        assert_logits_match(taps["logits"], lg)
        # every score the top-k ranked by: CUDA exp(double) against libm exp on the same logits
        assert np.array_equal(taps["scores"].view(np.uint32), oracle_scores(taps["logits"]).view(np.uint32)), \
            "fp32 scores differ from the oracle's"
    toks = range(B) if tokens is None else tokens
    rows = _oracle_rows(w, W, x, toks, layer_idx)
    for t in toks:
        r = rows[t]
        assert np.array_equal(idx[t], r["idx"])
        assert_close(taps["h"][t], r["h"], f"h[{t}]")
        assert_close(taps["ylat"][t], r["ylat"], f"ylat[{t}]")
        assert_close(taps["sh"][t], r["sh"], f"sh[{t}]")
        assert_close(taps["up"][t], r["out"] - r["sh"], f"up[{t}]")
        assert_close(out[t], r["out"], f"out[{t}]")
    return out, idx


# ---- mid-size layer (every dimension a multiple of 512: the streaming schedule runs on it) -----

@pytest.fixture(scope="module")
def mid(torch_cuda):
    w = synth.WORKLOADS["mid_b2"]
    W = synth.layer_weights(w, 0)
    return w, W, upload_weights(W)


@pytest.mark.parametrize("B", [1, 2])
@pytest.mark.parametrize("schedule", SCHEDULES)
def test_mid_parity(mid, B, schedule):
    w, W, W_dev = mid
    x = synth.tokens(w, batch=B)
    layer = _make_layer(w, W_dev, max_batch=B, schedule=schedule)
    _check_step(w, W, x, layer, label=f"mid B{B} {schedule}")
    if schedule == "stream":
        assert layer.kernels_per_step(B) == 4  # the streaming kernel ran (4 launches per step)


@pytest.mark.parametrize("B", [5, 13, 64])
@pytest.mark.parametrize("schedule", ["fused", "noring"])
def test_mid_split_k_parity(mid, B, schedule):
    # L = I = 512: two 128-byte lines per row, so the ring phases run four row groups of two
    # warps that add their K halves in shared memory
    w, W, W_dev = mid
    x = synth.tokens(w, step=B, batch=B)
    layer = _make_layer(w, W_dev, max_batch=B, schedule=schedule)
    assert layer.tma_ring() == (schedule == "fused")
    _check_step(w, W, x, layer, label=f"mid B{B} {schedule}")


@pytest.mark.parametrize("schedule", ["fused", "stream"])
def test_mid_back_to_back_and_graph(mid, torch_cuda, schedule):
    # consecutive steps of different tokens, eager and replayed from a CUDA graph, agree with a
    # fresh handle's single step (the control block is clean between steps)
    torch = torch_cuda
    w, W, W_dev = mid
    layer = _make_layer(w, W_dev, max_batch=2, schedule=schedule)
    xs = [to_device(synth.tokens(w, step=s, batch=2)) for s in range(3)]
    ref = [run_layer(_make_layer(w, W_dev, max_batch=2, schedule=schedule), synth.tokens(w, step=s, batch=2))[0]
           for s in range(3)]
    outs = [torch.empty_like(x) for x in xs]
    stream = torch.cuda.Stream()
    with torch.cuda.stream(stream):
        for x, o in zip(xs, outs):
            layer.step(x, out=o, stream=stream)
    torch.cuda.synchronize()
    for o, r in zip(outs, ref):
        _assert_replays(bf16_tensor_to_f32(o), r, exact=schedule == "stream")
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream, capture_error_mode="thread_local"):
        for x, o in zip(xs, outs):
            layer.step(x, out=o, stream=stream)
    for o in outs:
        o.zero_()
    g.replay()
    torch.cuda.synchronize()
    for o, r in zip(outs, ref):
        _assert_replays(bf16_tensor_to_f32(o), r, exact=schedule == "stream")
    del g


def _assert_replays(out, ref, exact):
    # The streaming and multi-kernel schedules add split-K partials and the k slots in a fixed
    # order: a replay is bitwise equal (exact).  The fused schedules add the expert rows into
    # ylat with fp32 reductions (the order of a token's k slots is not fixed), so ylat may differ
    # in its last bits and an output element by at most one bf16 unit in the last place.
    if exact:
        assert np.array_equal(out, ref)
        return
    ulp = np.exp2(np.floor(np.log2(np.maximum(np.abs(ref), 1e-30))) - 7)
    assert np.all(np.abs(out - ref) <= ulp), np.max(np.abs(out - ref) / ulp)


# ---- tiny layer -------------------------------------------------------------------------------

@pytest.fixture(scope="module")
def tiny(torch_cuda):
    w = synth.WORKLOADS["tiny_b1"]
    W = synth.layer_weights(w, 0)
    return w, W, upload_weights(W)


@pytest.mark.parametrize("schedule", SCHEDULES)
@pytest.mark.parametrize("B", [1, 2, 3, 5, 8, 9, 17, 33, 64, 65, 128, 200, 256, 512])
def test_tiny_parity(tiny, B, schedule):
    # above 64 tokens: several 64-bit token-mask words per expert, token groups in the dense parts
    # (the speculative-decoding shapes: batch x (drafts + 1) tokens)
    w, W, W_dev = tiny
    layer = _make_layer(w, W_dev, max_batch=max(64, B), schedule=schedule)
    x = synth.tokens(w, step=B, batch=B)
    _check_step(w, W, x, layer, label=f"tiny B{B} {schedule}")


@pytest.mark.parametrize("B", [1, 2, 3, 5, 9, 17, 64, 65, 200, 512])
def test_tiny_parity_register_path(tiny, B):
    # the fused steps' routed experts on register-fed loads (MOEDEC_FLAG_NO_TMA_RING)
    w, W, W_dev = tiny
    layer = _make_layer(w, W_dev, max_batch=max(64, B), schedule="noring")
    assert not layer.tma_ring()
    x = synth.tokens(w, step=B, batch=B)
    _check_step(w, W, x, layer, label=f"tiny B{B} noring")


@pytest.mark.parametrize("schedule", SCHEDULES)
def test_tiny_launch_variant_counts(tiny, schedule):
    w, W, W_dev = tiny
    layer = _make_layer(w, W_dev, max_batch=16, schedule=schedule)
    run_layer(layer, synth.tokens(w, batch=1))
    run_layer(layer, synth.tokens(w, batch=2))
    c = layer.launch_counts()
    assert c["small"] == 2 * layer.kernels_per_step(1) and c["splitk"] == 0
    run_layer(layer, synth.tokens(w, batch=16))
    assert layer.launch_counts()["splitk"] == layer.kernels_per_step(16)


@pytest.mark.parametrize("schedule", SCHEDULES)
def test_tiny_deterministic(tiny, schedule):
    w, W, W_dev = tiny
    layer = _make_layer(w, W_dev, max_batch=8, schedule=schedule)
    x = synth.tokens(w, batch=8)
    a = run_layer(layer, x)
    b = run_layer(layer, x)
    assert np.array_equal(a[1], b[1])
    # At 8 tokens only the multi-kernel schedule adds the k slots in a fixed order; the fused
    # split-K kernel (also taken by "stream" above 2 tokens) adds them into ylat with fp32
    # reductions: ylat and what follows from it agree to rounding, the rest bitwise.
    exact = schedule == "multi"
    _assert_replays(a[0], b[0], exact)
    for k in a[3]:
        if not exact and k in ("ylat", "up"):
            r, _ = rel_errors(a[3][k], b[3][k])
            assert r < 1e-5, (k, r)
        else:
            assert np.array_equal(a[3][k], b[3][k]), k


@pytest.mark.parametrize("schedule", SCHEDULES)
def test_tiny_back_to_back_steps_see_their_own_tokens(tiny, torch_cuda, schedule):
    # Several steps queued on one stream with different tokens, then one graph replay of two
    # steps: every output must match its own token batch (no stale activations).
    torch = torch_cuda
    w, W, W_dev = tiny
    layer = _make_layer(w, W_dev, max_batch=4, flags=0, schedule=schedule)
    xs = [synth.tokens(w, step=100 + i, batch=4) for i in range(3)]
    xd = [to_device(x) for x in xs]
    outs = [layer.step(x) for x in xd]
    torch.cuda.synchronize()
    for x, o in zip(xs, outs):
        ref = oracle.step(w.dims, W, x)
        got = synth.bf16_to_f32(o.cpu().numpy().view(np.uint16))
        assert_close(got, ref["out"], "queued out")
    g = torch.cuda.CUDAGraph()
    o1 = torch.empty_like(xd[0])
    o2 = torch.empty_like(xd[0])
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        layer.step(xd[0], out=o1)
        layer.step(xd[1], out=o2)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    with torch.cuda.graph(g):
        layer.step(xd[1], out=o1)
        layer.step(xd[2], out=o2)
    o1.zero_()
    o2.zero_()
    g.replay()
    torch.cuda.synchronize()
    for x, o in ((xs[1], o1), (xs[2], o2)):
        ref = oracle.step(w.dims, W, x)
        assert_close(synth.bf16_to_f32(o.cpu().numpy().view(np.uint16)), ref["out"], "graph out")
    del g


def test_batch_zero_and_limits(tiny, torch_cuda):
    from moe_decode_layer_moedec_b200 import MoedecError, lib
    torch = torch_cuda
    w, W, W_dev = tiny
    layer = _make_layer(w, W_dev, max_batch=4)
    x = to_device(synth.tokens(w, batch=8))
    out = torch.empty_like(x)
    s = torch.cuda.current_stream().cuda_stream
    assert lib.moedec_step(layer._h, x.data_ptr(), 0, out.data_ptr(), s) == 0
    assert lib.moedec_step(layer._h, x.data_ptr(), 5, out.data_ptr(), s) == -2      # > max_batch
    assert lib.moedec_step(layer._h, x.data_ptr() + 2, 1, out.data_ptr(), s) == -1  # misaligned
    assert lib.moedec_step(layer._h, x.data_ptr(), 2, x.data_ptr() + 16, s) == -1   # overlapping
    assert lib.moedec_step(None, x.data_ptr(), 1, out.data_ptr(), s) == -1
    with pytest.raises(MoedecError):
        layer.routing(3)  # not the last step's batch


@pytest.mark.parametrize("schedule", ["fused", "stream"])
def test_fused_wait_timeout_is_reported_and_context_stays_usable(tiny, schedule):
    # MOEDEC_FLAG_TEST_STALL: the router never publishes its logits, so the top-k item's bounded
    # wait runs out (20 ms); every CTA leaves and the step reports MOEDEC_ERR_TIMEOUT.
    from moe_decode_layer_moedec_b200 import FLAG_TEST_STALL, MoedecError
    w, W, W_dev = tiny
    stalled = _make_layer(w, W_dev, max_batch=2, flags=FLAG_TEST_STALL, schedule=schedule)
    x = to_device(synth.tokens(w, batch=2))
    stalled.step(x)
    with pytest.raises(MoedecError, match="TIMEOUT"):
        stalled.routing(2)
    stalled.step(x)  # the control block was cleared on the way out: it stalls again, no hang
    with pytest.raises(MoedecError, match="TIMEOUT"):
        stalled.routing(2)
    stalled.close()
    layer = _make_layer(w, W_dev, max_batch=2, schedule=schedule)
    _check_step(w, W, synth.tokens(w, batch=2), layer)


@pytest.mark.parametrize("B", [2, 9, 65])
def test_ring_wait_timeout_is_reported_and_context_stays_usable(tiny, B):
    # MOEDEC_FLAG_TEST_STALL_EXPERTS: the TMA-ring gate/up phase never counts its units, so the
    # expert down phase's bounded wait for them runs out (20 ms); every CTA drains its ring and
    # leaves, and the step reports MOEDEC_ERR_TIMEOUT (B = 2: small-batch step, 9 and 65: split-K)
    from moe_decode_layer_moedec_b200 import FLAG_TEST_STALL_EXPERTS, MoedecError
    w, W, W_dev = tiny
    stalled = _make_layer(w, W_dev, max_batch=B, flags=FLAG_TEST_STALL_EXPERTS)
    assert stalled.tma_ring()
    x = to_device(synth.tokens(w, batch=B))
    for _ in range(2):  # the control block was cleared on the way out: it stalls again, no hang
        stalled.step(x)
        with pytest.raises(MoedecError, match="TIMEOUT"):
            stalled.routing(B)
    stalled.close()
    layer = _make_layer(w, W_dev, max_batch=B)
    _check_step(w, W, synth.tokens(w, batch=B), layer, label=f"tiny B{B} after a ring timeout")


@pytest.mark.parametrize("batch,schedule", [(2, "stream"), (3, "fused"), (9, "fused")])
def test_fused_and_multi_agree(tiny, batch, schedule):
    # batch 2 runs the streaming kernel, batch 3 the small-batch fused kernel, batch 9 the split-K one
    w, W, W_dev = tiny
    x = synth.tokens(w, step=5, batch=batch)
    a = run_layer(_make_layer(w, W_dev, max_batch=16, schedule=schedule), x)
    b = run_layer(_make_layer(w, W_dev, max_batch=16, schedule="multi"), x)
    assert np.array_equal(a[1], b[1])
    for k in ("h", "ylat", "sh", "up"):
        r, m = rel_errors(a[3][k], b[3][k])
        assert r < 1e-5, (k, r)


def test_create_rejects_bad_config(tiny):
    from moe_decode_layer_moedec_b200 import MoedecError, MoeDecodeLayer
    w, W, W_dev = tiny
    d = layer_dims(w.dims)
    with pytest.raises(MoedecError, match="UNSUPPORTED"):
        MoeDecodeLayer(d, W_dev, max_batch=513)
    import dataclasses as dc
    with pytest.raises(MoedecError, match="UNSUPPORTED"):   # 512 tokens x top-32 > 8192 selections
        MoeDecodeLayer(dc.replace(d, top_k=32), W_dev, max_batch=512)
    bad = dict(W_dev)
    bad["gate_s"] = W_dev["gate_s"].clone()
    bad["gate_s"][3, 7, 1] = 150   # scale 2^23: outside the exact fp16 range
    with pytest.raises(MoedecError, match="UNSUPPORTED"):
        MoeDecodeLayer(d, bad, max_batch=1)
    import dataclasses
    with pytest.raises(MoedecError, match="UNSUPPORTED"):
        MoeDecodeLayer(dataclasses.replace(d, hidden=500), W_dev, max_batch=1)


def test_tiny_tied_router_rows(tiny, torch_cuda):
    # duplicated router rows give equal logits: the lower expert index must win
    w, W, W_dev = tiny
    x = synth.tokens(w, batch=4)
    lg, idx, _ = oracle.route(W["router"], x, w.dims.top_k)
    W2 = {k: v.copy() for k, v in W.items()}
    top = int(idx[0, 0])
    other = (top + 1) % w.dims.n_experts
    W2["router"][other] = W["router"][top]
    W2_dev = dict(W_dev)
    W2_dev["router"] = to_device(W2["router"])
    layer = _make_layer(w, W2_dev, max_batch=4)
    out, gidx, _, _ = run_layer(layer, x)
    _, ridx, _ = oracle.route(W2["router"], x, w.dims.top_k)
    assert np.array_equal(gidx, ridx)
    assert min(top, other) == ridx[0, 0]


# ---- full-size layer ----------------------------------------------------------------------------

@pytest.fixture(scope="module")
def full_layers(torch_cuda):
    cache = {}

    def get(name, layer_idx=0):
        key = (name, layer_idx)
        if key not in cache:
            cache.clear()  # one full layer (3 GB) resident at a time
            torch_cuda.cuda.empty_cache()
            w = synth.WORKLOADS[name]
            W = synth.layer_weights(w, layer_idx)
            cache[key] = (w, W, upload_weights(W))
        return cache[key]
    return get


@pytest.mark.parametrize("schedule", SCHEDULES)
@pytest.mark.parametrize("name", ["full_b1", "full_b2"])
def test_full_small_batches_all_tokens(full_layers, name, schedule):
    w, W, W_dev = full_layers(name)
    layer = _make_layer(w, W_dev, max_batch=w.batch, schedule=schedule)
    x = synth.tokens(w)
    out, idx = _check_step(w, W, x, layer, label=f"{name} L0 {schedule}")
    if name == "full_b2":
        assert 0 < len(set(idx[0]) & set(idx[1])) < w.dims.top_k


# Above two tokens the streaming schedule is the split-K kernel too, so B >= 16 runs the fused
# split-K kernel and the multi-kernel schedule; layer 15 and 31 as well as 0 (distinct weights).
LARGE_CASES = [(l, s) for l in (0, 15, 31) for s in ("fused", "multi")] + [(0, "noring")]


@pytest.mark.parametrize("layer_idx,schedule", LARGE_CASES)
def test_full_b16_all_tokens(full_layers, layer_idx, schedule):
    w, W, W_dev = full_layers("full_b16", layer_idx)
    layer = _make_layer(w, W_dev, max_batch=w.batch, schedule=schedule)
    assert layer.tma_ring() == (schedule != "noring")
    x = synth.tokens(w)
    _check_step(w, W, x, layer, label=f"full_b16 L{layer_idx} {schedule}", layer_idx=layer_idx)


@pytest.mark.parametrize("layer_idx,schedule", LARGE_CASES)
def test_full_b64_skewed_all_tokens(full_layers, layer_idx, schedule):
    w, W, W_dev = full_layers("full_b64_skewed", layer_idx)
    layer = _make_layer(w, W_dev, max_batch=w.batch, schedule=schedule)
    x = synth.tokens(w)
    _, idx = _check_step(w, W, x, layer, label=f"full_b64_skewed L{layer_idx} {schedule}", layer_idx=layer_idx)
    # the skew is there: about half of all selections go to the 32 hot experts
    share = np.isin(idx, synth.hot_set(w, layer_idx)).mean()
    assert 0.3 < share < 0.7, share


@pytest.mark.parametrize("schedule", ["fused", "multi"])
def test_full_b256_routing_all_outputs_sampled(full_layers, schedule):
    # speculative-decoding batch: every token's routing, logits and scores; 32 tokens' outputs
    w, W, W_dev = full_layers("full_b256")
    layer = _make_layer(w, W_dev, max_batch=w.batch, schedule=schedule)
    x = synth.tokens(w)
    _check_step(w, W, x, layer, tokens=range(0, 256, 8), label=f"full_b256 L0 {schedule}")


# ---- one expert with many tokens: every token group and operand path of the expert items ------

def _tiny_skewed(B, hot, beta, seed):
    return synth.Workload(f"tiny_hot{hot}_b{B}", synth.TINY, B, seed, hot_experts=hot, hot_beta=beta)


@pytest.mark.parametrize("schedule", ["fused", "multi", "noring"])
def test_tiny_hot_experts_token_groups(torch_cuda, schedule):
    # 8 hot experts of 64 at B = 64 (k = 4, beta = 4): experts take 1..4, 5..8, 9..16 and 17..32
    # tokens, so an expert item runs one or two 16-token groups on either operand path
    w = _tiny_skewed(64, 8, 4.0, 3100)
    W = synth.layer_weights(w, 0)
    x = synth.tokens(w)
    _, ridx, _ = oracle.route(W["router"], x, w.dims.top_k)
    c = np.bincount(ridx.ravel(), minlength=w.dims.n_experts)
    for lo, hi in ((1, 4), (5, 8), (9, 16), (17, 32)):
        assert ((c >= lo) & (c <= hi)).any(), (lo, hi, c)
    layer = _make_layer(w, upload_weights(W), max_batch=64, schedule=schedule)
    _check_step(w, W, x, layer, label=f"tiny hot8 B64 {schedule}")


@pytest.mark.parametrize("B", [17, 64])
@pytest.mark.parametrize("schedule", ["fused", "multi", "noring"])
def test_tiny_identical_tokens_one_expert_takes_every_token(tiny, B, schedule):
    # B copies of one token: each of its k experts receives all B tokens (the largest bucket: up
    # to four 16-token groups of one expert item)
    w, W, W_dev = tiny
    x = np.repeat(synth.tokens(w, step=11, batch=1), B, axis=0)
    layer = _make_layer(w, W_dev, max_batch=64, schedule=schedule)
    out, idx = _check_step(w, W, x, layer, label=f"tiny identical B{B} {schedule}")
    assert (idx == idx[0]).all()


# ---- cross-layer prefetch hint ------------------------------------------------------------------

@pytest.mark.parametrize("B", [1, 3, 9])
def test_next_layer_hint_leaves_results_unchanged(tiny, torch_cuda, B):
    # two layers of distinct weights hinting each other (the small-batch kernel at B <= 4, the
    # split-K kernel above); every step still matches the oracle, and a mismatched handle is refused
    from moe_decode_layer_moedec_b200 import MoedecError
    w, W0, W0_dev = tiny
    W1 = synth.layer_weights(w, 1)
    W1_dev = upload_weights(W1)
    l0 = _make_layer(w, W0_dev, max_batch=16)
    l1 = _make_layer(w, W1_dev, max_batch=16)
    l0.set_next(l1)
    l1.set_next(l0)
    for s in range(2):
        x = synth.tokens(w, step=40 + s, batch=B)
        _check_step(w, W0, x, l0, label=f"tiny B{B} hinted")
        _check_step(w, W1, x, l1, label=f"tiny B{B} hinted")
    mid = synth.WORKLOADS["mid_b2"]
    other = _make_layer(mid, upload_weights(synth.layer_weights(mid, 0)), max_batch=2)
    with pytest.raises(MoedecError, match="INVALID_ARG"):
        l0.set_next(other)
    l0.set_next(None)
    _check_step(w, W0, synth.tokens(w, step=50, batch=B), l0, label=f"tiny B{B}")
