"""Expert parallelism for the decode layer step: the partition, the shard weights, and the step.

A layer is split over G ranks (one GPU each).  Rank r holds a contiguous range of the routed
experts and a slice of the shared expert's inner width, in multiples of 128.  Router, top-k and
the latent projections run on every rank, so every rank computes the same routing.  Each rank's
step gives an fp32 partial output, and the layer's output is the bf16 rounding of their sum.  This
is exact up to fp32 rounding order: W_up ylat is linear in the experts' terms, and
SD(silu(SG x) * (SU x)) is a sum over the shared expert's inner index.

The pages run the MoE tensor-parallel on the GPUs of one NVLink domain, with partial results in
buffers every GPU can reach and one fused reduction ("快是可以生成的，可信只能证明（vLLM 重写
Kimi K3 解码路径…）", section 他们换掉了什么).  Here the exchange is the library's publish and
combine kernels over peer memory: `ExpertParallelLayer` for one process per GPU, and
`EmulatedExpertParallel` to run every rank's shard on one device in rank order.  The emulated ranks
never wait on each other: each kernel finds the flags it needs already set by earlier launches on
the same stream.

Everything here is argument marshalling and bookkeeping; the arithmetic runs in libmoedec.so.
"""
from __future__ import annotations

from dataclasses import dataclass, replace

from . import EP_MAX_WORLD, LayerDims, MoeDecodeLayer

SHARED_UNIT = 128  # the shared expert's inner width is split in multiples of this


@dataclass(frozen=True)
class Shard:
    rank: int
    world: int
    expert_begin: int
    expert_count: int
    shared_begin: int   # first inner index of the shared expert's slice
    shared_count: int   # width of the slice (a multiple of SHARED_UNIT; 0: no shared slice)


def partition(dims: LayerDims, world: int) -> list[Shard]:
    """Shards of a layer over `world` ranks.

    The experts are split into contiguous ranges whose sizes differ by at most one; the lower
    ranks take the extra experts.  The shared expert is split into SHARED_UNIT-wide slices by the
    same rule, except that the higher ranks take the extra units, so that a rank with more
    experts does not also get more of the shared expert.
    """
    if not 1 <= world <= EP_MAX_WORLD:
        raise ValueError(f"world must be 1..{EP_MAX_WORLD}")
    E = dims.n_experts
    if world > E:
        raise ValueError("more ranks than experts")
    base, extra = divmod(E, world)
    units = dims.shared_inter // SHARED_UNIT if dims.n_shared else 0
    if dims.n_shared and dims.shared_inter % SHARED_UNIT:
        raise ValueError(f"shared_inter must be a multiple of {SHARED_UNIT}")
    ubase, uextra = divmod(units, world)
    shards, e0, s0 = [], 0, 0
    for r in range(world):
        ne = base + (1 if r < extra else 0)
        nu = ubase + (1 if r >= world - uextra else 0)
        shards.append(Shard(r, world, e0, ne, s0, nu * SHARED_UNIT))
        e0 += ne
        s0 += nu * SHARED_UNIT
    return shards


def _contiguous(a):
    if hasattr(a, "contiguous"):
        return a.contiguous()
    import numpy as np
    return np.ascontiguousarray(a)


def shard_weights(dims: LayerDims, weights: dict, shard: Shard) -> tuple[LayerDims, dict]:
    """The dims and weights of one shard, from the whole layer's (torch tensors or numpy arrays).

    The router and the latent projections are the layer's own arrays.  The expert arrays and the
    rows of SG and SU are views of the layer's arrays.  The columns of SD are copied into dense
    arrays of their own.  Shapes follow the library's layouts: expert arrays [E][...], shared
    gate/up [I_s][...], shared down [H][I_s/2] and [H][I_s/32].
    """
    e0, e1 = shard.expert_begin, shard.expert_begin + shard.expert_count
    W = {n: weights[n] for n in ("router", "w_down_lat", "w_up_lat")}
    for n in ("gate_q", "gate_s", "up_q", "up_s", "down_q", "down_s"):
        W[n] = weights[n][e0:e1]
    if shard.shared_count:
        s0, s1 = shard.shared_begin, shard.shared_begin + shard.shared_count
        for n in ("sh_gate_q", "sh_gate_s", "sh_up_q", "sh_up_s"):
            W[n] = weights[n][s0:s1]
        W["sh_down_q"] = _contiguous(weights["sh_down_q"][:, s0 // 2:s1 // 2])
        W["sh_down_s"] = _contiguous(weights["sh_down_s"][:, s0 // 32:s1 // 32])
        sd = replace(dims, shared_inter=shard.shared_count, n_shared=1)
    else:
        for n in ("sh_gate_q", "sh_gate_s", "sh_up_q", "sh_up_s", "sh_down_q", "sh_down_s"):
            W[n] = None
        sd = replace(dims, shared_inter=SHARED_UNIT, n_shared=0)
    return sd, W


def make_shard_layer(dims: LayerDims, weights: dict, shard: Shard, max_batch: int, flags: int = 0) -> MoeDecodeLayer:
    """A shard handle on the current device, from the whole layer's device tensors."""
    sd, W = shard_weights(dims, weights, shard)
    layer = MoeDecodeLayer(sd, W, max_batch=max_batch, flags=flags,
                           expert_range=(shard.expert_begin, shard.expert_count))
    layer.shard = shard
    return layer


class EpochCounter:
    """Step epochs (1, 2, ...) and the partial buffer each uses (epoch parity)."""

    def __init__(self):
        self.epoch = 0

    def next(self) -> tuple[int, int]:
        self.epoch += 1
        return self.epoch, self.epoch % 2


class EmulatedExpertParallel:
    """Every rank's shard of one layer on the current device, stepped in rank order.

    A step runs each rank's partial step, then each rank's publish, then each rank's combine.  All
    of them go on one stream, so every combine finds its flags already set.  Every rank's output
    is kept, and they must be bit-identical.
    """

    def __init__(self, dims: LayerDims, weights: dict, world: int, max_batch: int, flags: int = 0):
        import torch
        self.dims, self.world, self.max_batch = dims, world, max_batch
        self.shards = partition(dims, world)
        self.layers = [make_shard_layer(dims, weights, s, max_batch, flags) for s in self.shards]
        H = dims.hidden
        self.parts = torch.empty((world, 2, max_batch, H), dtype=torch.float32, device="cuda")
        self.flags = torch.zeros((world, world), dtype=torch.int32, device="cuda")
        self.clock = EpochCounter()

    def flag_ptr(self, owner: int, slot: int) -> int:
        """Device address of flag word `slot` (the publishing rank) in rank `owner`'s flag array."""
        return self.flags.data_ptr() + 4 * (owner * self.world + slot)

    def step(self, x, stream=None):
        """Returns (outs, parts): each rank's output [B, H] (bf16 values in x's dtype: torch.bfloat16
        or 16-bit integer bit patterns) and fp32 partial [B, H]."""
        import torch
        B = x.shape[0]
        epoch, parity = self.clock.next()
        for r, layer in enumerate(self.layers):
            layer.step_partial(x, self.parts[r, parity], stream)
        for r, layer in enumerate(self.layers):
            layer.ep_publish([self.flag_ptr(q, r) for q in range(self.world)], epoch, stream)
        outs = []
        for r, layer in enumerate(self.layers):
            out = torch.empty((B, self.dims.hidden), dtype=x.dtype, device=x.device)
            layer.ep_combine([self.parts[g, parity].data_ptr() for g in range(self.world)], self.flag_ptr(r, 0),
                             epoch, B, out, stream)
            outs.append(out)
        return outs, [self.parts[r, parity, :B] for r in range(self.world)]

    def close(self):
        for layer in self.layers:
            layer.close()


def peer_addresses(rank: int, handles: list, local: tuple, open_fn):
    """This process's addresses of every rank's partial buffers and flag array.

    handles[g] = ((parts_handle, parts_offset), (flags_handle, flags_offset)) as rank g exported
    them; local = (parts_ptr, flags_ptr) of this rank; open_fn maps an exported handle to the base
    address of its allocation here.  A handle is opened once even when both buffers of a rank lie
    in one allocation.  Returns (parts[g], flags[g], opened bases to close later)."""
    parts, flags, opened = [], [], []
    for g, ((hp, op), (hf, of)) in enumerate(handles):
        if g == rank:
            parts.append(local[0])
            flags.append(local[1])
            continue
        bp = open_fn(hp)
        opened.append(bp)
        if hf == hp:
            bf = bp
        else:
            bf = open_fn(hf)
            opened.append(bf)
        parts.append(bp + op)
        flags.append(bf + of)
    return parts, flags, opened


def publish_slots(rank: int, peer_flags: list) -> list:
    """The flag word that rank `rank` release-stores into, in every rank's flag array (u32 words)."""
    return [f + 4 * rank for f in peer_flags]


def exchange(obj, group=None) -> list:
    """Every rank's `obj`, in rank order (one all_gather_object over the process group)."""
    import torch.distributed as dist
    out = [None] * dist.get_world_size(group)
    dist.all_gather_object(out, obj, group=group)
    return out


class ExpertParallelLayer:
    """This rank's shard of an expert-parallel layer, one process per GPU of one node.

    The flag array int32 [world] and the two partial buffers fp32 [2][max_batch][H] are allocated
    here and mapped into every other rank with CUDA IPC once, at construction (a collective over
    the default process group).  `step` then needs no collective of the process group: the
    exchange is the publish and combine kernels over peer memory.
    """

    def __init__(self, dims: LayerDims, weights: dict, max_batch: int, flags: int = 0, group=None):
        import torch
        import torch.distributed as dist
        from . import ipc_export, ipc_open
        self.dims, self.max_batch = dims, max_batch
        self.rank, self.world = dist.get_rank(group), dist.get_world_size(group)
        self.shard = partition(dims, self.world)[self.rank]
        self.layer = make_shard_layer(dims, weights, self.shard, max_batch, flags)
        H = dims.hidden
        self.parts = torch.empty((2, max_batch, H), dtype=torch.float32, device="cuda")
        self.flags = torch.zeros((self.world,), dtype=torch.int32, device="cuda")
        torch.cuda.synchronize()
        handles = exchange((ipc_export(self.parts.data_ptr()), ipc_export(self.flags.data_ptr())), group)
        self.peer_parts, self.peer_flags, self._opened = peer_addresses(
            self.rank, handles, (self.parts.data_ptr(), self.flags.data_ptr()), ipc_open)
        self.clock = EpochCounter()
        self._part_bytes = max_batch * H * 4

    def step(self, x, out=None, stream=None):
        import torch
        B = x.shape[0]
        if out is None:
            out = torch.empty((B, self.dims.hidden), dtype=x.dtype, device=x.device)
        epoch, parity = self.clock.next()
        self.layer.step_partial(x, self.parts[parity], stream)
        self.layer.ep_publish(publish_slots(self.rank, self.peer_flags), epoch, stream)
        self.layer.ep_combine([p + parity * self._part_bytes for p in self.peer_parts], self.flags.data_ptr(),
                              epoch, B, out, stream)
        return out

    def close(self):
        from . import ipc_close
        import torch
        torch.cuda.synchronize()
        for p in self._opened:
            ipc_close(p)
        self._opened = []
        self.layer.close()
