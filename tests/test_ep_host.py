"""Expert parallelism on the CPU: the partition, the shard weights, and the exchange's host logic.

A shard's step is the layer's step with the other shards' experts and the rest of the shared
expert taken out, and the layer's output is the sum of the shards' outputs before rounding.  These
tests pin the host side of that against the oracle.  Each shard's weights come from
`ep.shard_weights`.  They are put back into a full-size layer whose other experts have zero
codes (an E2M1 code 0 is +0, so those experts add exactly nothing).  The oracle's outputs of the
shards, summed, must equal its output for the whole layer (fp64, so up to rounding), and every
shard must route the same.  The world-size-2 tests run the same over two gloo processes, with the
partition agreed through `ep.exchange`, and map each other's exchange buffers from exported
handles (a fake IPC opener stands in for the GPU: the addresses, the offsets, one opening per
allocation, and the flag slot each rank publishes into).
"""
import dataclasses
import datetime
import os
import socket

import numpy as np
import pytest

import oracle
import synth
from moe_decode_layer_moedec_b200 import EP_MAX_WORLD, LayerDims, MoedecError, lib
from moe_decode_layer_moedec_b200 import ep
from tests.harness import oracle_layer_of_shard


def _dims(d: synth.Dims) -> LayerDims:
    return LayerDims(d.hidden, d.latent, d.n_experts, d.top_k, d.expert_inter, d.shared_inter, 1)


@pytest.mark.parametrize("E,Is,world", [(64, 256, 1), (64, 256, 2), (64, 256, 3), (64, 256, 4), (64, 256, 16),
                                        (896, 2048, 8), (896, 2048, 5), (896, 2048, 16), (7, 128, 7), (130, 384, 4)])
def test_partition_covers_every_expert_and_the_shared_expert_once(E, Is, world):
    d = LayerDims(512, 256, E, 4, 256, Is, 1)
    shards = ep.partition(d, world)
    assert [s.rank for s in shards] == list(range(world)) and all(s.world == world for s in shards)
    e = 0
    for s in shards:  # contiguous, in rank order, covering [0, E)
        assert s.expert_begin == e and s.expert_count >= 1
        e += s.expert_count
    assert e == E
    counts = [s.expert_count for s in shards]
    assert max(counts) - min(counts) <= 1 and counts == sorted(counts, reverse=True)
    c = 0
    for s in shards:
        assert s.shared_begin == c and s.shared_count % ep.SHARED_UNIT == 0
        c += s.shared_count
    assert c == Is
    units = [s.shared_count // ep.SHARED_UNIT for s in shards]
    assert max(units) - min(units) <= 1 and units == sorted(units)


def test_partition_rejects_bad_worlds():
    d = LayerDims(512, 256, 8, 2, 256, 256, 1)
    for world in (0, 9, EP_MAX_WORLD + 1):
        with pytest.raises(ValueError):
            ep.partition(d, world)
    with pytest.raises(ValueError):
        ep.partition(dataclasses.replace(d, shared_inter=200), 2)
    # no shared expert: nobody gets a slice
    assert all(s.shared_count == 0 for s in ep.partition(dataclasses.replace(d, n_shared=0), 3))


def test_shard_weights_are_views_and_the_shared_down_columns():
    w = synth.WORKLOADS["tiny_b1"]
    W = synth.layer_weights(w, 0)
    d = _dims(w.dims)
    s = ep.partition(d, 2)[1]
    sd, SW = ep.shard_weights(d, W, s)
    assert sd.shared_inter == s.shared_count and sd.n_shared == 1 and sd.n_experts == d.n_experts
    e0, e1 = s.expert_begin, s.expert_begin + s.expert_count
    for n in ("gate_q", "gate_s", "up_q", "up_s", "down_q", "down_s"):
        assert np.shares_memory(SW[n], W[n]) and SW[n].shape[0] == s.expert_count
        assert np.array_equal(SW[n], W[n][e0:e1])
    s0, s1 = s.shared_begin, s.shared_begin + s.shared_count
    assert np.array_equal(SW["sh_gate_q"], W["sh_gate_q"][s0:s1])
    assert SW["sh_down_q"].flags["C_CONTIGUOUS"] and SW["sh_down_q"].shape == (d.hidden, s.shared_count // 2)
    assert np.array_equal(SW["sh_down_q"], W["sh_down_q"][:, s0 // 2:s1 // 2])
    assert np.array_equal(SW["sh_down_s"], W["sh_down_s"][:, s0 // 32:s1 // 32])
    none = ep.shard_weights(d, W, ep.Shard(0, 4, 0, 16, 0, 0))
    assert none[0].n_shared == 0 and none[1]["sh_down_q"] is None


@pytest.mark.parametrize("world", [2, 3])
def test_shard_outputs_sum_to_the_layer_output(world):
    w = synth.WORKLOADS["tiny_b1"]
    W = synth.layer_weights(w, 0)
    x = synth.tokens(w, 0, batch=5)
    full = oracle.step(w.dims, W, x)
    total = np.zeros_like(full["out"])
    for s in ep.partition(_dims(w.dims), world):
        od, O, ns = oracle_layer_of_shard(w.dims, W, s)
        r = oracle.step(od, O, x, n_shared=ns)
        assert np.array_equal(r["idx"], full["idx"]) and np.array_equal(r["w"], full["w"])
        total += r["out"]
    scale = np.abs(full["out"]).max()
    assert np.abs(total - full["out"]).max() <= 1e-12 * scale
    # a partition that dropped one shard would not add up
    s0 = ep.partition(_dims(w.dims), world)[0]
    od, O, ns = oracle_layer_of_shard(w.dims, W, s0)
    assert np.abs(total - oracle.step(od, O, x, n_shared=ns)["out"] - full["out"]).max() > 1e-6 * scale


def test_epochs_alternate_the_partial_buffers():
    c = ep.EpochCounter()
    assert [c.next() for _ in range(5)] == [(1, 1), (2, 0), (3, 1), (4, 0), (5, 1)]


def test_shard_arguments_are_checked_without_gpu():
    import ctypes
    from moe_decode_layer_moedec_b200 import ABI_VERSION, FLAG_STREAM, _Config, _Weights
    h = ctypes.c_void_p()
    w = _Weights()
    for begin, count in ((-1, 4), (0, 0), (60, 8), (64, 1)):
        cfg = _Config(ABI_VERSION, 512, 256, 64, 4, 256, 256, 1, 4, 0)
        assert lib.moedec_create_shard(ctypes.byref(cfg), ctypes.byref(w), begin, count, ctypes.byref(h)) == -1
    cfg = _Config(ABI_VERSION, 512, 256, 64, 4, 256, 256, 1, 4, FLAG_STREAM)
    assert lib.moedec_create_shard(ctypes.byref(cfg), ctypes.byref(w), 0, 32, ctypes.byref(h)) == -2
    assert lib.moedec_ep_publish(None, None, 1, 1, None) == -1
    assert lib.moedec_ep_combine(None, None, None, 1, 1, 1, None, None) == -1
    assert lib.moedec_ipc_export(None, None, None) == -1
    assert lib.moedec_ipc_open(None, None) == -1
    assert lib.moedec_ipc_close(None) == -1
    with pytest.raises(ValueError):
        from moe_decode_layer_moedec_b200 import ipc_open
        ipc_open(b"short")
    assert MoedecError


# ---- two gloo ranks ---------------------------------------------------------------------------

def _free_port() -> int:
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, q) -> None:
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank), OMP_NUM_THREADS="2")
    import torch
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        w = synth.WORKLOADS["tiny_b1"]
        W = synth.layer_weights(w, 0)
        x = synth.tokens(w, 0, batch=3)
        shards = ep.partition(_dims(w.dims), world)
        mine = shards[rank]
        agreed = ep.exchange(mine)  # every rank must hold the same table
        od, O, ns = oracle_layer_of_shard(w.dims, W, mine)
        r = oracle.step(od, O, x, n_shared=ns)
        parts = ep.exchange(r["out"])  # the partial outputs, in rank order
        total = np.zeros_like(parts[0])
        for p in parts:
            total += p
        t = torch.from_numpy(r["out"].copy())
        dist.all_reduce(t)
        q.put((rank, agreed == shards, total, t.numpy(), r["idx"]))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_reassemble_the_layer_output():
    import torch.multiprocessing as mp
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(300)
    for p in procs:
        if p.is_alive():
            p.kill()
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    got = sorted((q.get(timeout=10) for _ in range(world)), key=lambda g: g[0])
    w = synth.WORKLOADS["tiny_b1"]
    full = oracle.step(w.dims, synth.layer_weights(w, 0), synth.tokens(w, 0, batch=3))
    scale = np.abs(full["out"]).max()
    for rank, agreed, total, reduced, idx in got:
        assert agreed, rank
        assert np.array_equal(idx, full["idx"])
        assert np.abs(total - full["out"]).max() <= 1e-12 * scale
        assert np.abs(reduced - full["out"]).max() <= 1e-12 * scale
    assert np.array_equal(got[0][2], got[1][2])  # the same rank-order sum on both ranks


def _fake_handle(kind: str, rank: int) -> bytes:
    return (kind.encode() + bytes([rank])).ljust(64, b"\0")


def _fake_base(handle: bytes) -> int:
    return 0x1000_0000 * (handle[1] + 1) + (0x100_0000 if handle[:1] == b"F" else 0)


def _rank_main_peers(rank: int, world: int, port: int, q) -> None:
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        # rank 0: both buffers in one allocation (one handle, two offsets); rank 1: two allocations
        parts = (_fake_handle("P", rank), 256 * (rank + 1))
        flags = (_fake_handle("P", rank), 4096) if rank == 0 else (_fake_handle("F", rank), 64)
        handles = ep.exchange((parts, flags))
        opened_calls = []

        def fake_open(h):
            opened_calls.append(h)
            return _fake_base(h)
        local = (0xAAAA_0000 + rank, 0xBBBB_0000 + rank)
        pp, pf, opened = ep.peer_addresses(rank, handles, local, fake_open)
        q.put((rank, pp, pf, opened, opened_calls, ep.publish_slots(rank, pf)))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_map_each_others_exchange_buffers():
    import torch.multiprocessing as mp
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main_peers, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
    for p in procs:
        if p.is_alive():
            p.kill()
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    got = {g[0]: g[1:] for g in (q.get(timeout=10) for _ in range(world))}
    # rank 0 sees rank 1's two allocations, each opened once, at base + offset
    pp, pf, opened, calls, slots = got[0]
    assert pp[0] == 0xAAAA_0000 and pf[0] == 0xBBBB_0000
    assert pp[1] == _fake_base(_fake_handle("P", 1)) + 512 and pf[1] == _fake_base(_fake_handle("F", 1)) + 64
    assert calls == [_fake_handle("P", 1), _fake_handle("F", 1)] and len(opened) == 2
    assert slots == [pf[0], pf[1]]
    # rank 1 sees rank 0's single allocation opened once, with the two offsets
    pp, pf, opened, calls, slots = got[1]
    assert pp[1] == 0xAAAA_0001 and pf[1] == 0xBBBB_0001
    base = _fake_base(_fake_handle("P", 0))
    assert pp[0] == base + 256 and pf[0] == base + 4096
    assert calls == [_fake_handle("P", 0)] and opened == [base]
    assert slots == [pf[0] + 4, pf[1] + 4]
