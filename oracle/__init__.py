"""CPU oracle of the sparse latent-MoE decode layer step (ctypes wrapper of ``oracle.c``).

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU
baseline may import this package.  The product path (``moe_decode_layer_moedec_b200``) never
imports it, and this package never imports the product path; both take inputs from ``synth``.

Every function here is a thin marshalling layer: the arithmetic lives in ``oracle.c``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SO = os.path.join(_HERE, "liboracle.so")
_SRC = os.path.join(_HERE, "oracle.c")


def build(force: bool = False) -> str:
    """Compile liboracle.so next to its source (gcc, OpenMP row loops)."""
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", _SRC, "-o", _SO, "-lm"])
    return _SO


class _Dims(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in
                ("hidden", "latent", "n_experts", "top_k", "expert_inter", "shared_inter", "n_shared")]


_WNAMES = ("router", "w_down_lat", "w_up_lat", "gate_q", "gate_s", "up_q", "up_s", "down_q", "down_s",
           "sh_gate_q", "sh_gate_s", "sh_up_q", "sh_up_s", "sh_down_q", "sh_down_s")


class _Weights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in _WNAMES]


_lib = None


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_SO)
        vp, i32, dbl = ctypes.c_void_p, ctypes.c_int, ctypes.c_double
        L.oracle_bf16.argtypes = [ctypes.c_uint16]
        L.oracle_bf16.restype = dbl
        L.oracle_e2m1.argtypes = [ctypes.c_uint]
        L.oracle_e2m1.restype = dbl
        L.oracle_e8m0.argtypes = [ctypes.c_uint]
        L.oracle_e8m0.restype = dbl
        L.oracle_mxfp4_element.argtypes = [vp, vp, i32, i32, i32]
        L.oracle_mxfp4_element.restype = dbl
        L.oracle_bf16_matvec.argtypes = [vp, i32, i32, vp, vp]
        L.oracle_mxfp4_matvec.argtypes = [vp, vp, i32, i32, vp, vp]
        L.oracle_silu.argtypes = [dbl]
        L.oracle_silu.restype = dbl
        L.oracle_router_logits.argtypes = [vp, vp, i32, i32, i32, vp]
        L.oracle_score.argtypes = [ctypes.c_float]
        L.oracle_score.restype = ctypes.c_float
        L.oracle_topk.argtypes = [vp, i32, i32, vp, vp]
        L.oracle_route.argtypes = [vp, vp, i32, i32, i32, i32, vp, vp, vp]
        L.oracle_expert.argtypes = [ctypes.POINTER(_Dims), ctypes.POINTER(_Weights), i32, vp, vp]
        L.oracle_shared_expert.argtypes = [ctypes.POINTER(_Dims), ctypes.POINTER(_Weights), vp, vp]
        L.oracle_step_tokens.argtypes = [ctypes.POINTER(_Dims), ctypes.POINTER(_Weights), vp, i32, i32, i32,
                                         vp, vp, vp, vp, vp, vp, vp]
        L.oracle_step_tokens.restype = i32
        L.oracle_threads.restype = i32
        _lib = L
    return _lib


def _p(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"], "arrays passed to the oracle must be C-contiguous"
    return a.ctypes.data


def threads() -> int:
    return lib().oracle_threads()


def bf16(bits: int) -> float:
    return lib().oracle_bf16(bits)


def e2m1(code: int) -> float:
    return lib().oracle_e2m1(code)


def e8m0(s: int) -> float:
    return lib().oracle_e8m0(s)


def mxfp4_element(q: np.ndarray, s: np.ndarray, n: int, k: int) -> float:
    K = q.shape[-1] * 2
    return lib().oracle_mxfp4_element(_p(q), _p(s), K, n, k)


def mxfp4_matvec(q: np.ndarray, s: np.ndarray, v: np.ndarray) -> np.ndarray:
    N, K = q.shape[0], q.shape[1] * 2
    assert s.shape == (N, K // 32) and v.shape == (K,)
    v = np.ascontiguousarray(v, dtype=np.float64)
    out = np.empty(N, dtype=np.float64)
    lib().oracle_mxfp4_matvec(_p(q), _p(s), N, K, _p(v), _p(out))
    return out


def bf16_matvec(W: np.ndarray, v: np.ndarray) -> np.ndarray:
    N, K = W.shape
    v = np.ascontiguousarray(v, dtype=np.float64)
    out = np.empty(N, dtype=np.float64)
    lib().oracle_bf16_matvec(_p(W), N, K, _p(v), _p(out))
    return out


def silu(z: float) -> float:
    return lib().oracle_silu(z)


def score(logit: float) -> float:
    return lib().oracle_score(logit)


def topk(scores: np.ndarray, k: int):
    scores = np.ascontiguousarray(scores, dtype=np.float32)
    E = scores.shape[0]
    idx = np.empty(k, dtype=np.int32)
    w = np.empty(k, dtype=np.float32)
    lib().oracle_topk(_p(scores), E, k, _p(idx), _p(w))
    return idx, w


def route(router: np.ndarray, x: np.ndarray, k: int):
    """logits [B,E] fp32, idx [B,k] int32, w [B,k] fp32."""
    E, H = router.shape
    x = np.ascontiguousarray(x)
    B = x.shape[0]
    logits = np.empty((B, E), dtype=np.float32)
    idx = np.empty((B, k), dtype=np.int32)
    w = np.empty((B, k), dtype=np.float32)
    lib().oracle_route(_p(router), _p(x), B, E, H, k, _p(logits), _p(idx), _p(w))
    return logits, idx, w


def router_logits(router: np.ndarray, x: np.ndarray) -> np.ndarray:
    E, H = router.shape
    B = x.shape[0]
    logits = np.empty((B, E), dtype=np.float32)
    lib().oracle_router_logits(_p(router), _p(np.ascontiguousarray(x)), B, E, H, _p(logits))
    return logits


def make_dims(d, n_shared: int = 1) -> _Dims:
    return _Dims(d.hidden, d.latent, d.n_experts, d.top_k, d.expert_inter, d.shared_inter, n_shared)


def _weights(W: dict) -> _Weights:
    for n in _WNAMES:
        assert W[n].flags["C_CONTIGUOUS"], n
    return _Weights(*[_p(W[n]) for n in _WNAMES])


def expert(d, W: dict, e: int, h: np.ndarray) -> np.ndarray:
    dims, ws = make_dims(d), _weights(W)
    h = np.ascontiguousarray(h, dtype=np.float64)
    y = np.empty(d.latent, dtype=np.float64)
    lib().oracle_expert(ctypes.byref(dims), ctypes.byref(ws), e, _p(h), _p(y))
    return y


def shared_expert(d, W: dict, x: np.ndarray, n_shared: int = 1) -> np.ndarray:
    dims, ws = make_dims(d, n_shared), _weights(W)
    x = np.ascontiguousarray(x, dtype=np.float64)
    sh = np.empty(d.hidden, dtype=np.float64)
    lib().oracle_shared_expert(ctypes.byref(dims), ctypes.byref(ws), _p(x), _p(sh))
    return sh


def step(d, W: dict, x: np.ndarray, tokens: range | None = None, dense_masked: bool = False,
         n_shared: int = 1) -> dict:
    """One layer step for x [B,H] (bf16 bits); `tokens` is a contiguous range of rows to evaluate.

    Returns out/sh [nb,H] (double), h/ylat [nb,L] (double), logits [nb,E] fp32, idx/w [nb,k].
    """
    x = np.ascontiguousarray(x)
    B = x.shape[0]
    if tokens is None:
        tokens = range(B)
    assert tokens.step == 1 and 0 <= tokens.start <= tokens.stop <= B
    nb = len(tokens)
    H, L, E, k = d.hidden, d.latent, d.n_experts, d.top_k
    r = dict(out=np.empty((nb, H)), sh=np.empty((nb, H)), h=np.empty((nb, L)), ylat=np.empty((nb, L)),
             logits=np.empty((nb, E), dtype=np.float32), idx=np.empty((nb, k), dtype=np.int32),
             w=np.empty((nb, k), dtype=np.float32))
    dims, ws = make_dims(d, n_shared), _weights(W)
    rc = lib().oracle_step_tokens(ctypes.byref(dims), ctypes.byref(ws), _p(x), tokens.start, nb,
                                  1 if dense_masked else 0, _p(r["out"]), _p(r["h"]), _p(r["ylat"]), _p(r["sh"]),
                                  _p(r["logits"]), _p(r["idx"]), _p(r["w"]))
    if rc != 0:
        raise ValueError("oracle_step_tokens rejected the dimensions")
    return r
