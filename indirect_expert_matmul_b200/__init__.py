"""B200-native MoE indirect matrix multiplication (GGML_OP_MUL_MAT_ID).

Thin ctypes binding of ``libmoe_b200.so`` (C ABI in ``include/moe.h``).
Every function here only marshals arguments: it takes torch CUDA tensors for
device memory and the current torch stream, and calls the library.  All
arithmetic runs in the library's sm_100a kernels; there is no CPU or PyTorch
fallback, and importing fails loudly if the library has not been built.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe_b200.so")

OK, ERR_INVALID, ERR_RANGE, ERR_BAD_ID, ERR_CUDA, ERR_TIMEOUT, ERR_UNSUPPORTED = 0, -1, -2, -3, -4, -5, -6
BROADCAST, PER_SLOT = 0, 1
BF16, F16, F32 = 0, 1, 2
Q8_0, MXFP4 = 0, 1
_WTYPE = {"q8_0": Q8_0, "mxfp4": MXFP4, Q8_0: Q8_0, MXFP4: MXFP4}

# every symbol declared in include/moe.h
ABI_SYMBOLS = (
    "moe_status_string", "moe_workspace_size", "moe_workspace_init", "moe_get_status",
    "moe_weights_prepared_size", "moe_weights_prepare", "moe_row_ids", "moe_mul_mat_id", "moe_ffn",
    "moe_ffn_decode_noalloc", "moe_route", "moe_combine", "moe_set_gemv_threshold", "moe_get_gemv_threshold",
    "moe_set_path", "moe_profile_enable", "moe_profile_read", "moe_weights_prepared_size_w", "moe_weights_prepare_w",
    "moe_mul_mat_id_w", "moe_ffn_w", "moe_testing_stall",
)

_lib = None
_vp, _i32, _i64, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t


def _L() -> ctypes.CDLL:
    """The loaded library; raises ImportError when it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing; build it with `python -m indirect_expert_matmul_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    L.moe_status_string.argtypes = [_i32]
    L.moe_status_string.restype = ctypes.c_char_p
    L.moe_workspace_size.argtypes = [_i64, _i32, _i32, _i32, _i32, _i32, _i32]
    L.moe_workspace_size.restype = _sz
    L.moe_workspace_init.argtypes = [_vp, _vp]
    L.moe_get_status.argtypes = [_vp, _vp]
    L.moe_weights_prepared_size.argtypes = [_i32, _i32, _i32]
    L.moe_weights_prepared_size.restype = _sz
    L.moe_weights_prepare.argtypes = [_vp, _i32, _i32, _i32, _vp, _vp]
    L.moe_weights_prepared_size_w.argtypes = [_i32, _i32, _i32, _i32]
    L.moe_weights_prepared_size_w.restype = _sz
    L.moe_weights_prepare_w.argtypes = [_i32, _vp, _i32, _i32, _i32, _vp, _vp]
    L.moe_mul_mat_id_w.argtypes = [_i32, _vp, _i32, _i32, _i32, _vp, _i32, _vp, _i64, _i32, _i32, _vp, _vp, _vp]
    L.moe_ffn_w.argtypes = [_i32, _vp, _vp, _vp, _i32, _i32, _i32, _vp, _vp, _vp, _i32, _vp, _i32, _vp, _i64, _i32,
                            _vp, _vp, _vp, _vp]
    L.moe_row_ids.argtypes = [_vp, _i64, _i32, _i32, _i32, _vp, _vp, _vp, _vp, _vp]
    L.moe_mul_mat_id.argtypes = [_vp, _i32, _i32, _i32, _vp, _i32, _vp, _i64, _i32, _i32, _vp, _vp, _vp]
    L.moe_ffn.argtypes = [_vp, _vp, _vp, _i32, _i32, _i32, _vp, _vp, _vp, _i32, _vp, _i32, _vp, _i64, _i32,
                          _vp, _vp, _vp, _vp]
    L.moe_ffn_decode_noalloc.argtypes = [_vp, _vp, _vp, _i32, _i32, _i32, _vp, _vp, _vp, _i32, _vp, _i32, _vp, _i64,
                                         _i32, _vp, _vp, _vp, _vp]
    L.moe_route.argtypes = [_vp, _vp, _i64, _i32, _i32, _i32, _vp, _vp, _vp]
    L.moe_combine.argtypes = [_vp, _vp, _vp, _i64, _i32, _i64, _vp, _vp]
    L.moe_set_gemv_threshold.argtypes = [_i32]
    L.moe_set_gemv_threshold.restype = None
    L.moe_get_gemv_threshold.argtypes = []
    L.moe_set_path.argtypes = [_i32]
    L.moe_set_path.restype = None
    L.moe_testing_stall.argtypes = [_i32, _i32, _i32]
    L.moe_testing_stall.restype = None
    L.moe_profile_enable.argtypes = [_i32]
    L.moe_profile_enable.restype = None
    L.moe_profile_read.argtypes = [ctypes.POINTER(ctypes.c_char_p), ctypes.POINTER(_i32),
                                   ctypes.POINTER(ctypes.c_double), _i32]
    _lib = L
    return L


class MoeError(RuntimeError):
    def __init__(self, code: int, what: str = ""):
        self.code = code
        super().__init__(f"{what}: {status_string(code)} ({code})")


def status_string(code: int) -> str:
    return _L().moe_status_string(code).decode()


def lib() -> ctypes.CDLL:
    return _L()


def _chk(rc: int, what: str):
    if rc != OK:
        raise MoeError(rc, what)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device=None):
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


_XTYPE = {torch.bfloat16: BF16, torch.float16: F16, torch.float32: F32}
_MODE = {"broadcast": BROADCAST, "per_slot": PER_SLOT, BROADCAST: BROADCAST, PER_SLOT: PER_SLOT}


def _gpu(t, name):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")


def _cuda(t, name, dtype=None, device=None):
    """A CUDA tensor, contiguous, of `dtype` (if given) and on `device` (if
    given: the device whose stream the call launches on - a tensor elsewhere
    would reach the kernels as another GPU's or an unmapped address)."""
    _gpu(t, name)
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}; the call runs on {device}")
    return t


def _need(t, name, dtype, numel, device=None):
    """A caller-supplied input, output or workspace: CUDA, contiguous, of
    `dtype`, on `device`, and at least `numel` elements (the library reads or
    writes that many)."""
    _cuda(t, name, dtype, device)
    if t.numel() < numel:
        raise ValueError(f"{name} holds {t.numel()} elements; the call writes {numel}")
    return t


# ----------------------------------------------------------------- memory
def workspace_size(n_tokens, k, n_experts, n_in, n_hidden=0, n_hidden_shared=0, x_dtype=torch.bfloat16) -> int:
    return _L().moe_workspace_size(n_tokens, k, n_experts, n_in, n_hidden, n_hidden_shared, _XTYPE[x_dtype])


def workspace(n_tokens, k, n_experts, n_in, n_hidden=0, n_hidden_shared=0, x_dtype=torch.bfloat16, device="cuda"):
    """A zero-status workspace tensor (uint8) for calls of these sizes."""
    n = workspace_size(n_tokens, k, n_experts, n_in, n_hidden, n_hidden_shared, x_dtype)
    ws = torch.empty(max(n, 256), dtype=torch.uint8, device=device)
    _chk(_L().moe_workspace_init(_ptr(ws), _stream(ws.device)), "moe_workspace_init")
    return ws


def get_status(ws) -> int:
    """Synchronise the current stream, return and clear the device status."""
    return _L().moe_get_status(_ptr(ws), _stream(ws.device))


# ---------------------------------------------------------------- weights
def weights_prepared_size(n_experts, n_out, n_in, wtype="q8_0") -> int:
    return _L().moe_weights_prepared_size_w(_WTYPE[wtype], n_experts, n_out, n_in)


_BLOCK_BYTES = {Q8_0: 34, MXFP4: 17}


def weights_prepare(blocks, n_experts, n_out, n_in, out=None, wtype="q8_0"):
    """Repack Q8_0 blocks (uint8 [E][n_out][n_in/32][34]) or MXFP4 blocks
    (uint8 [E][n_out][n_in/32][17]), on the GPU, into the form the kernels read."""
    w = _WTYPE[wtype]
    _need(blocks, "blocks", torch.uint8, n_experts * n_out * (n_in // 32) * _BLOCK_BYTES[w])
    n = weights_prepared_size(n_experts, n_out, n_in, w)
    if out is None:
        out = torch.empty(n, dtype=torch.uint8, device=blocks.device)
    _need(out, "out", torch.uint8, n, blocks.device)
    _chk(_L().moe_weights_prepare_w(w, _ptr(blocks), n_experts, n_out, n_in, _ptr(out), _stream(blocks.device)),
         "moe_weights_prepare")
    return out


# ----------------------------------------------------------------- row ids
def row_ids(ids, n_experts, mode="broadcast", ws=None):
    """(ids_src1, ids_dst, expert_bounds) int32 tensors of the stable counting sort."""
    _cuda(ids, "ids", torch.int32)
    T, k = ids.shape
    S = T * k
    dev = ids.device
    src1 = torch.empty(max(S, 1), dtype=torch.int32, device=dev)
    dst = torch.empty(max(S, 1), dtype=torch.int32, device=dev)
    bounds = torch.empty(n_experts + 1, dtype=torch.int32, device=dev)
    if ws is None:
        ws = workspace(T, k, n_experts, 0, device=dev)
    _need(ws, "ws", torch.uint8, workspace_size(T, k, n_experts, 0), dev)
    _chk(_L().moe_row_ids(_ptr(ids), T, k, n_experts, _MODE[mode], _ptr(src1), _ptr(dst), _ptr(bounds), _ptr(ws),
                          _stream(dev)), "moe_row_ids")
    return src1[:S], dst[:S], bounds


# --------------------------------------------------------------- operators
def mul_mat_id(W, n_experts, n_out, n_in, x, ids, mode="broadcast", ws=None, out=None, wtype="q8_0"):
    """dst float32 [T][k][n_out] = W[ids[t][s]] . x[t or (t, s)].

    W: prepared weights of type `wtype` ("q8_0" or "mxfp4").  Without `ws` the
    call makes its own workspace, synchronises and raises MoeError on a
    device-side error; with `ws` the caller reads get_status."""
    w = _WTYPE[wtype]
    _cuda(x, "x")
    dev = x.device
    _cuda(ids, "ids", torch.int32, dev)
    T, k = ids.shape
    _need(W, "W", torch.uint8, weights_prepared_size(n_experts, n_out, n_in, w), dev)
    _need(x, "x", x.dtype, (T if _MODE[mode] == BROADCAST else T * k) * n_in)
    own_ws = ws is None
    if own_ws:
        ws = workspace(T, k, n_experts, n_in, x_dtype=x.dtype, device=dev)
    _need(ws, "ws", torch.uint8, workspace_size(T, k, n_experts, n_in, x_dtype=x.dtype), dev)
    if out is None:
        out = torch.empty((T, k, n_out), dtype=torch.float32, device=dev)
    _need(out, "out", torch.float32, T * k * n_out, dev)
    _chk(_L().moe_mul_mat_id_w(w, _ptr(W), n_experts, n_out, n_in, _ptr(x), _XTYPE[x.dtype], _ptr(ids), T, k,
                               _MODE[mode], _ptr(out), _ptr(ws), _stream(x.device)), "moe_mul_mat_id")
    if own_ws:
        _chk(get_status(ws), "moe_mul_mat_id (device status)")
    return out


def _check_ffn_inputs(Wg, Wu, Wd, Sg, Su, Sd, n_experts, n_embd, n_ff, n_ff_sh, x, T, w=Q8_0):
    dev = x.device
    _need(Wg, "Wg", torch.uint8, weights_prepared_size(n_experts, n_ff, n_embd, w), dev)
    _need(Wu, "Wu", torch.uint8, weights_prepared_size(n_experts, n_ff, n_embd, w), dev)
    _need(Wd, "Wd", torch.uint8, weights_prepared_size(n_experts, n_embd, n_ff, w), dev)
    if n_ff_sh:
        _need(Sg, "Sg", torch.uint8, weights_prepared_size(1, n_ff_sh, n_embd, w), dev)
        _need(Su, "Su", torch.uint8, weights_prepared_size(1, n_ff_sh, n_embd, w), dev)
        _need(Sd, "Sd", torch.uint8, weights_prepared_size(1, n_embd, n_ff_sh, w), dev)
    _need(x, "x", x.dtype, T * n_embd)


def ffn(Wg, Wu, Wd, n_experts, n_embd, n_ff, x, ids, shared=None, ws=None, out=None, out_shared=None, wtype="q8_0"):
    """Routed SwiGLU expert FFN (+ optional shared expert (Sg, Su, Sd, n_ff_shared)),
    every matrix prepared as `wtype` ("q8_0" or "mxfp4").

    Returns (dst [T][k][n_embd], dst_shared [T][n_embd] or None), float32."""
    w = _WTYPE[wtype]
    _cuda(x, "x")
    dev = x.device
    _cuda(ids, "ids", torch.int32, dev)
    T, k = ids.shape
    Sg = Su = Sd = None
    n_ff_sh = 0
    if shared is not None:
        Sg, Su, Sd, n_ff_sh = shared
    _check_ffn_inputs(Wg, Wu, Wd, Sg, Su, Sd, n_experts, n_embd, n_ff, n_ff_sh, x, T, w)
    own_ws = ws is None
    if own_ws:
        ws = workspace(T, k, n_experts, n_embd, n_ff, n_ff_sh, x.dtype, device=dev)
    _need(ws, "ws", torch.uint8, workspace_size(T, k, n_experts, n_embd, n_ff, n_ff_sh, x.dtype), dev)
    if out is None:
        out = torch.empty((T, k, n_embd), dtype=torch.float32, device=dev)
    _need(out, "out", torch.float32, T * k * n_embd, dev)
    if shared is not None and out_shared is None:
        out_shared = torch.empty((T, n_embd), dtype=torch.float32, device=dev)
    if shared is not None:
        _need(out_shared, "out_shared", torch.float32, T * n_embd, dev)
    _chk(_L().moe_ffn_w(w, _ptr(Wg), _ptr(Wu), _ptr(Wd), n_experts, n_embd, n_ff, _ptr(Sg), _ptr(Su), _ptr(Sd),
                        n_ff_sh, _ptr(x), _XTYPE[x.dtype], _ptr(ids), T, k, _ptr(out), _ptr(out_shared), _ptr(ws),
                        _stream(x.device)), "moe_ffn")
    if own_ws:
        _chk(get_status(ws), "moe_ffn (device status)")
    return out, out_shared


def ffn_decode_noalloc(Wg, Wu, Wd, n_experts, n_embd, n_ff, x, ids, shared=None, out=None, out_shared=None,
                       status=None):
    """moe_ffn for decode sizes (n_tokens*k <= 64, n_ff and n_ff_shared <= 2048)
    through the entry point that takes no workspace.  `status`: optional int32
    CUDA tensor of one element that receives the device status."""
    _cuda(x, "x")
    dev = x.device
    _cuda(ids, "ids", torch.int32, dev)
    T, k = ids.shape
    Sg = Su = Sd = None
    n_ff_sh = 0
    if shared is not None:
        Sg, Su, Sd, n_ff_sh = shared
    _check_ffn_inputs(Wg, Wu, Wd, Sg, Su, Sd, n_experts, n_embd, n_ff, n_ff_sh, x, T)
    if out is None:
        out = torch.empty((T, k, n_embd), dtype=torch.float32, device=dev)
    _need(out, "out", torch.float32, T * k * n_embd, dev)
    if shared is not None and out_shared is None:
        out_shared = torch.empty((T, n_embd), dtype=torch.float32, device=dev)
    if shared is not None:
        _need(out_shared, "out_shared", torch.float32, T * n_embd, dev)
    if status is not None:
        _need(status, "status", torch.int32, 1, dev)
    _chk(_L().moe_ffn_decode_noalloc(_ptr(Wg), _ptr(Wu), _ptr(Wd), n_experts, n_embd, n_ff, _ptr(Sg), _ptr(Su),
                                     _ptr(Sd), n_ff_sh, _ptr(x), _XTYPE[x.dtype], _ptr(ids), T, k, _ptr(out),
                                     _ptr(out_shared), _ptr(status), _stream(x.device)), "moe_ffn_decode_noalloc")
    return out, out_shared


def route(logits, k, bias=None, normalize=True, ids=None, weights=None):
    """Router through moe_route: the k largest logit + bias per token (ties to
    the lower expert) and their softmax weights.  logits: float32 CUDA [T][E];
    bias: float32 [E] or None.  Returns (ids int32 [T][k], weights float32 [T][k])."""
    _cuda(logits, "logits", torch.float32)
    dev = logits.device
    T, E = logits.shape
    if bias is not None:
        _need(bias, "bias", torch.float32, E, dev)
    if ids is None:
        ids = torch.empty((T, k), dtype=torch.int32, device=dev)
    if weights is None:
        weights = torch.empty((T, k), dtype=torch.float32, device=dev)
    _need(ids, "ids", torch.int32, T * k, dev)
    _need(weights, "weights", torch.float32, T * k, dev)
    _chk(_L().moe_route(_ptr(logits), _ptr(bias), T, E, k, 1 if normalize else 0, _ptr(ids), _ptr(weights),
                        _stream(logits.device)), "moe_route")
    return ids, weights


def combine(dst, weights, shared=None, out=None):
    """y[t] = sum_s weights[t][s] * dst[t][s] (+ shared[t]) through moe_combine.
    dst: float32 CUDA [T][k][n] (or [T*k][n] with weights [T][k]); weights:
    float32 [T][k]; shared: float32 [T][n] or None; out: float32 [T][n] or None."""
    _cuda(dst, "dst", torch.float32)
    dev = dst.device
    _cuda(weights, "weights", torch.float32, dev)
    T, k = weights.shape
    n = dst.shape[-1]
    if dst.numel() != T * k * n:
        raise ValueError("dst must hold n_tokens*k rows of n")
    if shared is not None:
        _need(shared, "shared", torch.float32, T * n, dev)
    if out is None:
        out = torch.empty((T, n), dtype=torch.float32, device=dev)
    _need(out, "out", torch.float32, T * n, dev)
    _chk(_L().moe_combine(_ptr(dst), _ptr(weights), _ptr(shared), T, k, n, _ptr(out), _stream(dst.device)),
         "moe_combine")
    return out


# ------------------------------------------------------------------ tuning
def set_gemv_threshold(n: int):
    _L().moe_set_gemv_threshold(n)


def get_gemv_threshold() -> int:
    return _L().moe_get_gemv_threshold()


def set_path(path: int):
    """0 = by threshold, 1 = mat-vec kernel, 2 = grouped tensor-core GEMM."""
    _L().moe_set_path(path)


# --------------------------------------------------------------- profiling
def profile_enable(on: bool = True):
    """Record CUDA events between the library's kernels (see moe_profile_enable)."""
    _L().moe_profile_enable(1 if on else 0)


def profile_read(max_stages: int = 32) -> dict:
    """{stage name: (launches, total device ms)} of the calls recorded so far."""
    names = (ctypes.c_char_p * max_stages)()
    launches = (_i32 * max_stages)()
    ms = (ctypes.c_double * max_stages)()
    n = _L().moe_profile_read(names, launches, ms, max_stages)
    if n < 0:
        raise MoeError(n, "moe_profile_read")
    return {names[i].decode(): (launches[i], ms[i]) for i in range(n)}
