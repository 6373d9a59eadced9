"""Seeded synthetic workloads for the indirect expert matmul (MoE MUL_MAT_ID).

This module holds the input recipe and nothing of the operator's arithmetic:
it builds Q8_0 expert weights, activations and routing ids from a
counter-based generator (``gen.c``), so the CPU oracle and the GPU library
consume byte-identical inputs while sharing no method code.

Shapes follow the workloads the pages discuss: the DeepSeek-Lite and
DeepSeek-V3/R1 expert layers of "CUDA: better MoE implementation" (ik_llama.cpp
PR #283, sections 2 and 3.1), the shared-expert decode step of llama.cpp
b11370 ("CUDA: fuse shared experts into MMVQ"), and a skewed-popularity stress
case.  No model weights or datasets are involved.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass, field

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gen.c")
_LIB = os.path.join(_HERE, "_gen.so")

# Tensor ids of the counter-based streams (one stream per tensor).
T_W = 1            # mul_mat_id weights
T_WG, T_WU, T_WD = 2, 3, 4          # routed expert gate / up / down
T_SG, T_SU, T_SD = 5, 6, 7          # shared expert gate / up / down
T_X = 100          # activations, one row per token
T_X_SLOT = 102     # activations, one row per (token, slot)
T_ROUTE = 200      # routing keys (uses T_ROUTE and T_ROUTE + 1)
T_RW = 300         # router weights of the routed slots
LAYER_STRIDE = 1000  # decode layers l use tensor ids + l * LAYER_STRIDE

D_LO, D_HI = 0.001, 0.01   # Q8_0 scale range


def build(force: bool = False) -> str:
    """Compile gen.c into _gen.so (gcc, OpenMP) if missing or stale."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def _L():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        i64, u64, dbl, vp, i32 = ctypes.c_int64, ctypes.c_uint64, ctypes.c_double, ctypes.c_void_p, ctypes.c_int
        _lib.wl_fill_q8_0.argtypes = [vp, i64, i64, i64, u64, u64, dbl, dbl]
        _lib.wl_fill_mxfp4.argtypes = [vp, i64, i64, i64, u64, u64, i32, i32]
        for f in (_lib.wl_fill_normal_f32, _lib.wl_fill_normal_bf16, _lib.wl_fill_normal_f16):
            f.argtypes = [vp, i64, i64, u64, u64]
        _lib.wl_fill_uniform_f32.argtypes = [vp, i64, i64, dbl, dbl, u64, u64]
        _lib.wl_route_topk_normal.argtypes = [vp, i64, i64, i32, i32, dbl, u64, u64]
        _lib.wl_route_uniform.argtypes = [vp, i64, i64, i32, i32, u64, u64]
        _lib.wl_route_zipf.argtypes = [vp, i64, i64, i32, i32, dbl, i32, u64, u64]
    return _lib


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return ctypes.c_void_p(a.ctypes.data)


# --------------------------------------------------------------------------
# generators
# --------------------------------------------------------------------------
def q8_0_weights(n_experts: int, n_out: int, n_in: int, seed: int, tensor: int,
                 out: np.ndarray | None = None) -> np.ndarray:
    """Stacked Q8_0 weights, uint8 array [n_experts][n_out][n_in/32][34]."""
    if n_in % 32:
        raise ValueError("n_in must be a multiple of 32 for Q8_0")
    shape = (n_experts, n_out, n_in // 32, 34)
    if out is None:
        out = np.empty(shape, dtype=np.uint8)
    assert out.shape == shape and out.dtype == np.uint8
    _L().wl_fill_q8_0(_ptr(out), 0, n_experts * n_out, n_in, seed, tensor, D_LO, D_HI)
    return out


def q8_0_weights_experts(e0: int, n_e: int, n_out: int, n_in: int, seed: int, tensor: int) -> np.ndarray:
    """Experts e0 .. e0+n_e-1 of a stacked Q8_0 matrix, byte-identical to the
    same slice of q8_0_weights(...) (the generator is counter-based)."""
    if n_in % 32:
        raise ValueError("n_in must be a multiple of 32 for Q8_0")
    out = np.empty((n_e, n_out, n_in // 32, 34), dtype=np.uint8)
    _L().wl_fill_q8_0(_ptr(out), e0 * n_out, n_e * n_out, n_in, seed, tensor, D_LO, D_HI)
    return out


# MXFP4 scale bytes: 2^(X - 127) for X in [X_LO, X_HI], i.e. block scales 2^-9 .. 2^-3,
# so the weights (element values up to 6 times the scale) span about 0.001 .. 0.75
X_LO, X_HI = 118, 124


def mxfp4_weights(n_experts: int, n_out: int, n_in: int, seed: int, tensor: int, e0: int = 0) -> np.ndarray:
    """Stacked MXFP4 weights, uint8 array [n_experts][n_out][n_in/32][17]: per
    block the scale byte, then 16 bytes of 4-bit codes (random bytes only).
    Experts are numbered from e0 (counter-based: a slice equals the same
    experts of a larger matrix)."""
    if n_in % 32:
        raise ValueError("n_in must be a multiple of 32 for MXFP4")
    out = np.empty((n_experts, n_out, n_in // 32, 17), dtype=np.uint8)
    _L().wl_fill_mxfp4(_ptr(out), e0 * n_out, n_experts * n_out, n_in, seed, tensor, X_LO, X_HI)
    return out


def activations(n_rows: int, n_in: int, dtype: str, seed: int, tensor: int, row0: int = 0) -> np.ndarray:
    """N(0,1) activations [n_rows][n_in]; rows numbered globally from row0.

    dtype "f32" -> float32; "bf16" / "f16" -> uint16 bit patterns."""
    n = n_rows * n_in
    if dtype == "f32":
        out = np.empty((n_rows, n_in), dtype=np.float32)
        _L().wl_fill_normal_f32(_ptr(out), row0 * n_in, n, seed, tensor)
    elif dtype == "bf16":
        out = np.empty((n_rows, n_in), dtype=np.uint16)
        _L().wl_fill_normal_bf16(_ptr(out), row0 * n_in, n, seed, tensor)
    elif dtype == "f16":
        out = np.empty((n_rows, n_in), dtype=np.uint16)
        _L().wl_fill_normal_f16(_ptr(out), row0 * n_in, n, seed, tensor)
    else:
        raise ValueError(dtype)
    return out


def uniform_f32(n: int, lo: float, hi: float, seed: int, tensor: int, i0: int = 0) -> np.ndarray:
    """U[lo, hi) float32 samples i0 .. i0+n-1 of a tensor."""
    out = np.empty(n, dtype=np.float32)
    if n:
        _L().wl_fill_uniform_f32(_ptr(out), i0, n, lo, hi, seed, tensor)
    return out


def router_weights(n_tokens: int, k: int, seed: int, tensor: int = T_RW, t0: int = 0) -> np.ndarray:
    """Router weights float32 [n_tokens][k]: U[0.05, 1) per slot, scaled in fp64 so
    that each token's weights sum to one (the shape a softmax over the chosen
    experts gives), then rounded to float32."""
    u = uniform_f32(n_tokens * k, 0.05, 1.0, seed, tensor, i0=t0 * k).astype(np.float64).reshape(n_tokens, k)
    if n_tokens == 0:
        return u.astype(np.float32)
    return (u / u.sum(axis=1, keepdims=True)).astype(np.float32)


def routing(kind: str, n_tokens: int, n_experts: int, k: int, seed: int, tensor: int = T_ROUTE,
            t0: int = 0, bias_sigma: float = 0.0, zipf_s: float = 1.2, n_zero: int = 0) -> np.ndarray:
    """Routing ids int32 [n_tokens][k], distinct experts per token."""
    if not (1 <= k <= n_experts):
        raise ValueError("need 1 <= k <= n_experts")
    ids = np.empty((n_tokens, k), dtype=np.int32)
    if n_tokens == 0:
        return ids
    if kind == "topk_normal":
        _L().wl_route_topk_normal(_ptr(ids), t0, n_tokens, n_experts, k, bias_sigma, seed, tensor)
    elif kind == "uniform":
        _L().wl_route_uniform(_ptr(ids), t0, n_tokens, n_experts, k, seed, tensor)
    elif kind == "zipf":
        if n_experts - n_zero < k:
            raise ValueError("too few experts with nonzero popularity")
        _L().wl_route_zipf(_ptr(ids), t0, n_tokens, n_experts, k, zipf_s, n_zero, seed, tensor)
    else:
        raise ValueError(kind)
    return ids


# --------------------------------------------------------------------------
# the five workloads
# --------------------------------------------------------------------------
@dataclass(frozen=True)
class Workload:
    name: str
    op: str                 # "mul_mat_id" or "ffn"
    n_experts: int
    k: int
    n_in: int               # n_embd for ffn
    n_out: int              # expert ffn width for ffn
    n_tokens: tuple         # token counts exercised
    x_dtype: str            # "f32" or "bf16"
    routing: str            # "topk_normal", "uniform" or "zipf"
    modes: tuple = ("broadcast",)
    bias_sigma: float = 0.0
    zipf_s: float = 1.2
    n_zero: int = 0
    n_ff_shared: int = 0    # 0 = no shared expert
    seed: int = 0
    notes: str = ""

    def ids(self, n_tokens: int, t0: int = 0, layer: int = 0) -> np.ndarray:
        return routing(self.routing, n_tokens, self.n_experts, self.k, self.seed,
                       T_ROUTE + layer * LAYER_STRIDE, t0=t0, bias_sigma=self.bias_sigma,
                       zipf_s=self.zipf_s, n_zero=self.n_zero)

    def x(self, n_tokens: int, t0: int = 0, mode: str = "broadcast", layer: int = 0) -> np.ndarray:
        if mode == "broadcast":
            return activations(n_tokens, self.n_in, self.x_dtype, self.seed, T_X + layer * LAYER_STRIDE, row0=t0)
        return activations(n_tokens * self.k, self.n_in, self.x_dtype, self.seed,
                           T_X_SLOT + layer * LAYER_STRIDE, row0=t0 * self.k)


WORKLOADS = {
    "tiny": Workload("tiny", "mul_mat_id", 8, 2, 256, 512, (64,), "f32", "topk_normal",
                     notes="top-2 of N(0,1) logits; fp32 activations; broadcast"),
    "lite": Workload("lite", "ffn", 64, 6, 2048, 1408, (512,), "bf16", "uniform",
                     notes="DeepSeek-Lite-shaped expert FFN, uniform routing"),
    "v3": Workload("v3", "ffn", 256, 8, 7168, 2048, (4096,), "bf16", "topk_normal", bias_sigma=0.5,
                   notes="DeepSeek-V3-shaped layer, top-8 of N(0,1) logits + per-expert N(0,0.5) bias"),
    "decode": Workload("decode", "ffn", 256, 8, 2048, 512, (1, 4, 8), "bf16", "uniform", n_ff_shared=512,
                       notes="decode step with one always-on shared expert"),
    "skew": Workload("skew", "mul_mat_id", 128, 4, 2880, 2880, (8192,), "bf16", "zipf",
                     modes=("broadcast", "per_slot"), zipf_s=1.2, n_zero=8,
                     notes="Zipf(1.2) expert popularity; the 8 lowest-ranked experts get none"),
}
