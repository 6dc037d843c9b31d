"""Python binding of libmoedec.so, the B200 (sm_100a) sparse latent-MoE decode layer step.

Argument marshalling only: every step of the layer runs in the library's CUDA kernels.  PyTorch
is used for device memory and streams.  There is no CPU path: if the shared library is missing
or cannot be loaded, importing this package raises.

    layer = MoeDecodeLayer(dims, weights, max_batch=64)   # weights: dict of CUDA tensors
    out = layer.step(x)                                   # x: bf16 [B, H] on the same device
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoedec.so")

ABI_VERSION = 1
FLAG_TAPS = 1
FLAG_SKIP_SCALE_CHECK = 2
FLAG_TEST_STALL = 4
FLAG_MULTI_KERNEL = 8
FLAG_TRACE = 16
FLAG_STREAM = 32
FLAG_NO_TMA_RING = 64
FLAG_TEST_STALL_EXPERTS = 128
TRACE_STAMPS = 16
EP_MAX_WORLD = 16
IPC_HANDLE_BYTES = 64
STATUS = {0: "MOEDEC_OK", -1: "MOEDEC_ERR_INVALID_ARG", -2: "MOEDEC_ERR_UNSUPPORTED", -3: "MOEDEC_ERR_CUDA",
          -4: "MOEDEC_ERR_OOM", -5: "MOEDEC_ERR_TIMEOUT", -6: "MOEDEC_ERR_DEVICE"}
WEIGHT_NAMES = ("router", "w_down_lat", "w_up_lat", "gate_q", "gate_s", "up_q", "up_s", "down_q", "down_s",
                "sh_gate_q", "sh_gate_s", "sh_up_q", "sh_up_s", "sh_down_q", "sh_down_s")


class MoedecError(RuntimeError):
    def __init__(self, call: str, status: int, detail: str = ""):
        self.status = status
        msg = f"{call} failed: {STATUS.get(status, status)}"
        if detail:
            msg += f" ({detail})"
        super().__init__(msg)


class _Config(ctypes.Structure):
    _fields_ = [("abi_version", ctypes.c_int32), ("hidden", ctypes.c_int32), ("latent", ctypes.c_int32),
                ("n_experts", ctypes.c_int32), ("top_k", ctypes.c_int32), ("expert_inter", ctypes.c_int32),
                ("shared_inter", ctypes.c_int32), ("n_shared", ctypes.c_int32), ("max_batch", ctypes.c_int32),
                ("flags", ctypes.c_uint32)]


class _Weights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in WEIGHT_NAMES]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing; build it with `python -m moe_decode_layer_moedec_b200.build` "
                          "(nvcc, sm_100a)")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i32 = ctypes.c_void_p, ctypes.c_int
    lib.moedec_create.argtypes = [ctypes.POINTER(_Config), ctypes.POINTER(_Weights), ctypes.POINTER(vp)]
    lib.moedec_create.restype = i32
    lib.moedec_step.argtypes = [vp, vp, i32, vp, vp]
    lib.moedec_step.restype = i32
    lib.moedec_destroy.argtypes = [vp]
    lib.moedec_destroy.restype = i32
    lib.moedec_get_routing.argtypes = [vp, vp, vp, i32, vp]
    lib.moedec_get_routing.restype = i32
    lib.moedec_get_taps.argtypes = [vp, vp, vp, vp, vp, vp, i32, vp]
    lib.moedec_get_taps.restype = i32
    lib.moedec_set_next.argtypes = [vp, vp]
    lib.moedec_set_next.restype = i32
    lib.moedec_tma_ring.argtypes = [vp]
    lib.moedec_tma_ring.restype = i32
    lib.moedec_get_scores.argtypes = [vp, vp, i32, vp]
    lib.moedec_get_scores.restype = i32
    lib.moedec_get_launch_counts.argtypes = [vp, ctypes.POINTER(ctypes.c_uint64), ctypes.POINTER(i32)]
    lib.moedec_get_launch_counts.restype = i32
    lib.moedec_profile_enable.argtypes = [vp, i32]
    lib.moedec_profile_enable.restype = i32
    lib.moedec_profile_read.argtypes = [vp, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_uint64),
                                        ctypes.POINTER(ctypes.c_char_p), ctypes.POINTER(i32)]
    lib.moedec_profile_read.restype = i32
    lib.moedec_router_logits_noalloc.argtypes = [vp, vp, i32, i32, i32, vp, vp]
    lib.moedec_router_logits_noalloc.restype = i32
    lib.moedec_get_trace.argtypes = [vp, ctypes.POINTER(ctypes.c_uint64), ctypes.POINTER(i32), vp]
    lib.moedec_get_trace.restype = i32
    lib.moedec_kernels_per_step.argtypes = [vp, i32]
    lib.moedec_kernels_per_step.restype = i32
    lib.moedec_last_cuda_error.argtypes = [vp]
    lib.moedec_last_cuda_error.restype = ctypes.c_char_p
    lib.moedec_create_shard.argtypes = [ctypes.POINTER(_Config), ctypes.POINTER(_Weights), i32, i32, ctypes.POINTER(vp)]
    lib.moedec_create_shard.restype = i32
    lib.moedec_step_partial.argtypes = [vp, vp, i32, vp, vp]
    lib.moedec_step_partial.restype = i32
    lib.moedec_ep_publish.argtypes = [vp, ctypes.POINTER(vp), i32, ctypes.c_uint32, vp]
    lib.moedec_ep_publish.restype = i32
    lib.moedec_ep_combine.argtypes = [vp, ctypes.POINTER(vp), vp, i32, ctypes.c_uint32, i32, vp, vp]
    lib.moedec_ep_combine.restype = i32
    lib.moedec_ipc_export.argtypes = [vp, vp, ctypes.POINTER(ctypes.c_uint64)]
    lib.moedec_ipc_export.restype = i32
    lib.moedec_ipc_open.argtypes = [vp, ctypes.POINTER(vp)]
    lib.moedec_ipc_open.restype = i32
    lib.moedec_ipc_close.argtypes = [vp]
    lib.moedec_ipc_close.restype = i32
    lib.moedec_status_string.argtypes = [i32]
    lib.moedec_status_string.restype = ctypes.c_char_p
    return lib


lib = _load()


@dataclass(frozen=True)
class LayerDims:
    hidden: int
    latent: int
    n_experts: int
    top_k: int
    expert_inter: int
    shared_inter: int
    n_shared: int = 1


def _stream_ptr(stream) -> int:
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream)


def _ptr(t) -> int:
    return 0 if t is None else int(t.data_ptr())


class MoeDecodeLayer:
    """One MoE layer's decode step on the current CUDA device (a moedec handle).

    `weights` maps the names in WEIGHT_NAMES to contiguous CUDA tensors: bf16 matrices as
    torch.bfloat16 or torch.uint16/int16 bit patterns, MXFP4 codes and E8M0 scales as uint8.
    The tensors are borrowed: keep them alive and unchanged while the layer exists.

    With `expert_range=(begin, count)` the handle is one shard of an expert-parallel layer
    (moedec_create_shard): `dims.n_experts` is the layer's total, the expert arrays hold experts
    begin .. begin+count-1 only, and `dims.shared_inter` / the sh_* arrays are this shard's slice
    of the shared expert.  Such a shard gives its fp32 partial output with `step_partial`.
    """

    def __init__(self, dims: LayerDims, weights: dict, max_batch: int, flags: int = 0, expert_range=None):
        self.dims = dims
        self.max_batch = max_batch
        self.flags = flags
        self.expert_range = None if expert_range is None else (int(expert_range[0]), int(expert_range[1]))
        self._weights = {n: weights.get(n) for n in WEIGHT_NAMES}  # keep the tensors alive
        for n, t in self._weights.items():
            if t is not None and not t.is_contiguous():
                raise ValueError(f"weight {n} must be contiguous")
        cfg = _Config(ABI_VERSION, dims.hidden, dims.latent, dims.n_experts, dims.top_k, dims.expert_inter,
                      dims.shared_inter, dims.n_shared, max_batch, flags)
        w = _Weights(*[_ptr(self._weights[n]) for n in WEIGHT_NAMES])
        h = ctypes.c_void_p()
        if self.expert_range is None:
            rc = lib.moedec_create(ctypes.byref(cfg), ctypes.byref(w), ctypes.byref(h))
        else:
            rc = lib.moedec_create_shard(ctypes.byref(cfg), ctypes.byref(w), self.expert_range[0],
                                         self.expert_range[1], ctypes.byref(h))
        if rc != 0:
            raise MoedecError("moedec_create" if self.expert_range is None else "moedec_create_shard", rc)
        self._h = h

    def _check(self, call: str, rc: int):
        if rc != 0:
            detail = lib.moedec_last_cuda_error(self._h).decode() if self._h else ""
            raise MoedecError(call, rc, detail)

    def step(self, x, out=None, stream=None):
        """out[b] = layer(x[b]) for x bf16 [B, H] on the device; asynchronous on `stream`."""
        import torch
        B = x.shape[0]
        if out is None:
            out = torch.empty((B, self.dims.hidden), dtype=x.dtype, device=x.device)
        assert x.is_contiguous() and out.is_contiguous()
        self._check("moedec_step", lib.moedec_step(self._h, _ptr(x), B, _ptr(out), _stream_ptr(stream)))
        return out

    def step_partial(self, x, partial=None, stream=None):
        """partial[b] = W_up ylat[b] + sh[b] in fp32, before rounding (this handle's experts and
        shared slice only when it is a shard); asynchronous on `stream`."""
        import torch
        B = x.shape[0]
        if partial is None:
            partial = torch.empty((B, self.dims.hidden), dtype=torch.float32, device=x.device)
        assert x.is_contiguous() and partial.is_contiguous() and partial.dtype == torch.float32
        assert partial.numel() >= B * self.dims.hidden
        self._check("moedec_step_partial",
                    lib.moedec_step_partial(self._h, _ptr(x), B, _ptr(partial), _stream_ptr(stream)))
        return partial

    def ep_publish(self, slot_ptrs, epoch: int, stream=None):
        """Release-store `epoch` into each device address of `slot_ptrs` (this rank's flag word in
        every rank's flag array) after the work already on `stream`."""
        arr = (ctypes.c_void_p * len(slot_ptrs))(*[int(p) for p in slot_ptrs])
        self._check("moedec_ep_publish",
                    lib.moedec_ep_publish(self._h, arr, len(slot_ptrs), epoch & 0xffffffff, _stream_ptr(stream)))

    def ep_combine(self, part_ptrs, flags_ptr: int, epoch: int, batch: int, out, stream=None):
        """out = bf16(sum of the ranks' fp32 partials, rank order) once every flag word at
        `flags_ptr` (one per rank; 0 for no wait) has reached `epoch`."""
        arr = (ctypes.c_void_p * len(part_ptrs))(*[int(p) for p in part_ptrs])
        self._check("moedec_ep_combine",
                    lib.moedec_ep_combine(self._h, arr, int(flags_ptr) or None, len(part_ptrs), epoch & 0xffffffff,
                                          batch, _ptr(out), _stream_ptr(stream)))
        return out

    def step_ptr(self, x_ptr: int, batch: int, out_ptr: int, stream_ptr: int):
        self._check("moedec_step", lib.moedec_step(self._h, x_ptr, batch, out_ptr, stream_ptr))

    def routing(self, batch: int, stream=None):
        """(idx int32 [B, k], w fp32 [B, k]) of the last step, in rank order."""
        import torch
        dev = torch.device("cuda", torch.cuda.current_device())
        idx = torch.empty((batch, self.dims.top_k), dtype=torch.int32, device=dev)
        w = torch.empty((batch, self.dims.top_k), dtype=torch.float32, device=dev)
        self._check("moedec_get_routing", lib.moedec_get_routing(self._h, _ptr(idx), _ptr(w), batch, _stream_ptr(stream)))
        return idx, w

    def taps(self, batch: int, stream=None) -> dict:
        """fp32 intermediates of the last step: logits [B,E], h/ylat [B,L], sh (and up with FLAG_TAPS) [B,H]."""
        import torch
        d = self.dims
        dev = torch.device("cuda", torch.cuda.current_device())
        f = lambda *s: torch.empty(s, dtype=torch.float32, device=dev)
        r = dict(logits=f(batch, d.n_experts), h=f(batch, d.latent), ylat=f(batch, d.latent), sh=f(batch, d.hidden))
        if self.flags & FLAG_TAPS:
            r["up"] = f(batch, d.hidden)
        self._check("moedec_get_taps", lib.moedec_get_taps(self._h, _ptr(r["logits"]), _ptr(r["h"]), _ptr(r["ylat"]),
                                                           _ptr(r["sh"]), _ptr(r.get("up")), batch, _stream_ptr(stream)))
        return r

    def set_next(self, nxt: "MoeDecodeLayer | None"):
        """Prefetch hint: steps of this layer pull `nxt`'s router rows into L2 (None clears it)."""
        self._next = nxt  # keep the next layer's handle (and its router tensor) alive
        self._check("moedec_set_next", lib.moedec_set_next(self._h, nxt._h if nxt is not None else None))

    def tma_ring(self) -> bool:
        """True when steps of 2 or more tokens stream the routed experts through per-warp TMA rings."""
        r = lib.moedec_tma_ring(self._h)
        if r < 0:
            self._check("moedec_tma_ring", r)
        return r == 1

    def scores(self, batch: int, stream=None):
        """fp32 router scores [B, E] of the last step, from the same device function the top-k uses."""
        import torch
        dev = torch.device("cuda", torch.cuda.current_device())
        s = torch.empty((batch, self.dims.n_experts), dtype=torch.float32, device=dev)
        self._check("moedec_get_scores", lib.moedec_get_scores(self._h, _ptr(s), batch, _stream_ptr(stream)))
        return s

    def launch_counts(self):
        arr = (ctypes.c_uint64 * 2)()
        n = ctypes.c_int(2)
        self._check("moedec_get_launch_counts", lib.moedec_get_launch_counts(self._h, arr, ctypes.byref(n)))
        return {"small": int(arr[0]), "splitk": int(arr[1])}

    def profile(self, enable: bool = True):
        """Bracket every kernel of later steps with CUDA events on its own stream (resets the sums)."""
        self._check("moedec_profile_enable", lib.moedec_profile_enable(self._h, 1 if enable else 0))

    def profile_read(self) -> dict:
        """{kernel name: (total ms, launches)} since profile(True); synchronises."""
        cap = 16
        ms = (ctypes.c_double * cap)()
        cnt = (ctypes.c_uint64 * cap)()
        names = (ctypes.c_char_p * cap)()
        n = ctypes.c_int(cap)
        self._check("moedec_profile_read", lib.moedec_profile_read(self._h, ms, cnt, names, ctypes.byref(n)))
        return {names[i].decode(): (float(ms[i]), int(cnt[i])) for i in range(n.value)}

    def trace(self, stream=None):
        """Per-CTA phase timestamps (ns) of the last fused step: list of rows (FLAG_TRACE only)."""
        cap = 16 * 256  # 16 rows per SM
        buf = (ctypes.c_uint64 * (cap * TRACE_STAMPS))()
        n = ctypes.c_int(cap)
        self._check("moedec_get_trace", lib.moedec_get_trace(self._h, buf, ctypes.byref(n), _stream_ptr(stream)))
        return [[int(buf[r * TRACE_STAMPS + i]) for i in range(TRACE_STAMPS)] for r in range(n.value)]

    def kernels_per_step(self, batch: int) -> int:
        return int(lib.moedec_kernels_per_step(self._h, batch))

    def close(self):
        """Destroy the handle and drop the references to the weight tensors and the hinted layer."""
        if getattr(self, "_h", None):
            lib.moedec_destroy(self._h)
            self._h = None
        self._weights = None
        self._next = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def router_logits_noalloc(router, x, logits=None, stream=None):
    """fp32 router logits [B, E] without any device allocation by the library (see include/moedec.h).

    For callers that cannot call cudaMalloc; `logits` may be passed in pre-allocated.  router
    [E, H] and x [B, H] are contiguous 16-bit (bf16 bit patterns) tensors on the current device;
    logits, if given, is a contiguous fp32 [B, E] tensor there."""
    import torch
    dev = torch.device("cuda", torch.cuda.current_device())
    for name, t in (("router", router), ("x", x)):
        if t.dim() != 2 or t.element_size() != 2 or not t.is_contiguous() or t.device != dev:
            raise ValueError(f"{name} must be a contiguous 2-D 16-bit tensor on {dev}")
    E, H = router.shape
    B = x.shape[0]
    if x.shape[1] != H:
        raise ValueError(f"x has width {x.shape[1]}, the router {H}")
    if logits is None:
        logits = torch.empty((B, E), dtype=torch.float32, device=dev)
    elif (logits.dtype != torch.float32 or tuple(logits.shape) != (B, E) or not logits.is_contiguous()
          or logits.device != dev):
        raise ValueError(f"logits must be a contiguous float32 [{B}, {E}] tensor on {dev}")
    rc = lib.moedec_router_logits_noalloc(_ptr(router), _ptr(x), E, H, B, _ptr(logits), _stream_ptr(stream))
    if rc != 0:
        raise MoedecError("moedec_router_logits_noalloc", rc)
    return logits


def ipc_export(ptr: int) -> tuple[bytes, int]:
    """CUDA IPC handle (IPC_HANDLE_BYTES bytes) of the device allocation that contains `ptr`, and
    the offset of `ptr` inside it."""
    buf = ctypes.create_string_buffer(IPC_HANDLE_BYTES)
    off = ctypes.c_uint64()
    rc = lib.moedec_ipc_export(int(ptr), buf, ctypes.byref(off))
    if rc != 0:
        raise MoedecError("moedec_ipc_export", rc)
    return buf.raw, int(off.value)


def ipc_open(handle: bytes) -> int:
    """Map an allocation exported by another process; returns its base address here (add the
    exporter's offset)."""
    if len(handle) != IPC_HANDLE_BYTES:
        raise ValueError("IPC handle must be %d bytes" % IPC_HANDLE_BYTES)
    buf = ctypes.create_string_buffer(handle, IPC_HANDLE_BYTES)
    p = ctypes.c_void_p()
    rc = lib.moedec_ipc_open(buf, ctypes.byref(p))
    if rc != 0:
        raise MoedecError("moedec_ipc_open", rc)
    return int(p.value)


def ipc_close(ptr: int) -> None:
    rc = lib.moedec_ipc_close(int(ptr))
    if rc != 0:
        raise MoedecError("moedec_ipc_close", rc)
