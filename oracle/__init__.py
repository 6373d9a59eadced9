"""CPU oracle for the indirect expert matmul - TEST INFRASTRUCTURE ONLY.

Only the test suite, ``__graft_entry__.smoke()`` and the benchmark's CPU
baseline leg may import this package.  The library never does.  It wraps
``moe_oracle.c`` (plain C, fp64, no code shared with the GPU library) with
numpy-in / numpy-out helpers.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB = os.path.join(_HERE, "_oracle.so")

BROADCAST, PER_SLOT = 0, 1
DTYPES = {"bf16": 0, "f16": 1, "f32": 2}
OK, ERR_INVALID, ERR_RANGE, ERR_BAD_ID = 0, -1, -2, -3


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (-O2, OpenMP; no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fno-fast-math", "-shared", "-fPIC",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def _L():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        vp, i64, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
        _lib.oracle_check_args.argtypes = [i64, i32, i32]
        _lib.oracle_row_ids.argtypes = [vp, i64, i32, i32, i32, vp, vp, vp]
        for f in (_lib.oracle_mul_mat_id_brute, _lib.oracle_mul_mat_id_grouped):
            f.argtypes = [vp, i32, i32, i32, vp, i32, vp, i64, i32, i32, vp, vp, i32]
        _lib.oracle_mul_mat_id_rows.argtypes = [vp, i32, i32, i32, vp, i32, vp, i64, i32, i32, vp, i64, vp, vp, i32]
        _lib.oracle_ffn_rows.argtypes = [vp, vp, vp, i32, i32, i32, vp, i32, vp, i64, i32, vp, i64, vp, vp, i32]
        _lib.oracle_shared_rows.argtypes = [vp, vp, vp, i32, i32, vp, i32, vp, i64, vp, vp, i32]
        _lib.oracle_ffn_hidden.argtypes = [vp, vp, i32, i32, i32, vp, i32, vp, i64, i32, vp, i64, vp, vp, vp, i32]
        _lib.oracle_dequant.argtypes = [vp, i32, i32, i32, vp, i32]
        _lib.oracle_dequant.restype = None
        _lib.oracle_combine.argtypes = [vp, vp, vp, i64, i32, i64, vp, vp]
        _lib.oracle_combine.restype = None
        _lib.oracle_route.argtypes = [vp, vp, i64, i32, i32, i32, vp, vp]
        _lib.oracle_num_threads.argtypes = []
        _lib.oracle_set_num_threads.argtypes = [i32]
        _lib.oracle_set_num_threads.restype = None
    return _lib


def _p(a):
    if a is None:
        return None
    assert isinstance(a, np.ndarray) and a.flags["C_CONTIGUOUS"], "need a C-contiguous numpy array"
    return ctypes.c_void_p(a.ctypes.data)


def _mode(mode):
    return {"broadcast": BROADCAST, "per_slot": PER_SLOT}.get(mode, mode)


# weight types, told apart by the block size of the stacked array's last axis
Q8_0, MXFP4 = 0, 1
_BLOCK_BYTES = {34: Q8_0, 17: MXFP4}


def wtype(W: np.ndarray) -> int:
    """Q8_0 (34-byte blocks) or MXFP4 (17-byte blocks) of a stacked weight
    array [E][n_out][n_in/32][block bytes]."""
    try:
        return _BLOCK_BYTES[W.shape[-1]]
    except KeyError:
        raise ValueError(f"unknown weight block size {W.shape[-1]}") from None


class OracleError(RuntimeError):
    def __init__(self, code):
        super().__init__(f"oracle error {code}")
        self.code = code


def _chk(rc):
    if rc != OK:
        raise OracleError(rc)


def check_args(n_tokens, k, n_experts) -> int:
    return _L().oracle_check_args(n_tokens, k, n_experts)


def row_ids(ids: np.ndarray, n_experts: int, mode="broadcast"):
    """(ids_src1, ids_dst, expert_bounds) of the stable counting sort."""
    ids = np.ascontiguousarray(ids, dtype=np.int32)
    T, k = ids.shape
    S = T * k
    src1 = np.zeros(max(S, 1), np.int32)
    dst = np.zeros(max(S, 1), np.int32)
    bounds = np.zeros(n_experts + 1, np.int32)
    _chk(_L().oracle_row_ids(_p(ids), T, k, n_experts, _mode(mode), _p(src1), _p(dst), _p(bounds)))
    return src1[:S], dst[:S], bounds


def dequant(W: np.ndarray, e: int) -> np.ndarray:
    """fp64 weights of expert e, [n_out][n_in], from Q8_0 or MXFP4 blocks."""
    E, n_out, nb, _ = W.shape
    out = np.empty((n_out, nb * 32), np.float64)
    _L().oracle_dequant(_p(W), n_out, nb * 32, e, _p(out), wtype(W))
    return out


def mul_mat_id(W, x, x_type, ids, mode="broadcast", grouped=False):
    """dst [T][k][n_out] (fp64) and its per-element tolerance."""
    E, n_out, nb, _ = W.shape
    ids = np.ascontiguousarray(ids, dtype=np.int32)
    T, k = ids.shape
    dst = np.zeros((T, k, n_out), np.float64)
    tol = np.zeros((T, k, n_out), np.float64)
    f = _L().oracle_mul_mat_id_grouped if grouped else _L().oracle_mul_mat_id_brute
    _chk(f(_p(W), E, n_out, nb * 32, _p(x), DTYPES[x_type], _p(ids), T, k, _mode(mode), _p(dst), _p(tol), wtype(W)))
    return dst, tol


def mul_mat_id_rows(W, x, x_type, ids, slots, mode="broadcast"):
    """Rows of dst for flat slots t*k+s only: ([n][n_out], tol)."""
    E, n_out, nb, _ = W.shape
    ids = np.ascontiguousarray(ids, dtype=np.int32)
    T, k = ids.shape
    slots = np.ascontiguousarray(slots, dtype=np.int64)
    out = np.zeros((len(slots), n_out), np.float64)
    tol = np.zeros_like(out)
    _chk(_L().oracle_mul_mat_id_rows(_p(W), E, n_out, nb * 32, _p(x), DTYPES[x_type], _p(ids), T, k,
                                     _mode(mode), _p(slots), len(slots), _p(out), _p(tol), wtype(W)))
    return out, tol


def _same_wtype(*Ws):
    t = {wtype(W) for W in Ws}
    if len(t) != 1:
        raise ValueError("the FFN's matrices must share one weight type")
    return t.pop()


def ffn(Wg, Wu, Wd, x, x_type, ids, slots=None):
    """Routed expert FFN rows ([n][n_embd] fp64, tol) for flat slots (all when None)."""
    E, n_ff, nb, _ = Wg.shape
    n_embd = nb * 32
    ids = np.ascontiguousarray(ids, dtype=np.int32)
    T, k = ids.shape
    if slots is None:
        n = T * k
        sp = None
    else:
        slots = np.ascontiguousarray(slots, dtype=np.int64)
        n = len(slots)
        sp = _p(slots)
    y = np.zeros((n, n_embd), np.float64)
    tol = np.zeros_like(y)
    _chk(_L().oracle_ffn_rows(_p(Wg), _p(Wu), _p(Wd), E, n_embd, n_ff, _p(x), DTYPES[x_type], _p(ids), T, k,
                              sp, n, _p(y), _p(tol), _same_wtype(Wg, Wu, Wd)))
    return y, tol


def shared_ffn(Sg, Su, Sd, x, x_type, tokens=None):
    """Shared-expert FFN rows for the listed tokens (all when None)."""
    _, n_ff, nb, _ = Sg.shape
    n_embd = nb * 32
    T = x.shape[0]
    tokens = np.arange(T, dtype=np.int64) if tokens is None else np.ascontiguousarray(tokens, dtype=np.int64)
    y = np.zeros((len(tokens), n_embd), np.float64)
    tol = np.zeros_like(y)
    _chk(_L().oracle_shared_rows(_p(Sg), _p(Su), _p(Sd), n_embd, n_ff, _p(x), DTYPES[x_type], _p(tokens),
                                 len(tokens), _p(y), _p(tol), _same_wtype(Sg, Su, Sd)))
    return y, tol


def ffn_hidden(Wg, Wu, x, x_type, ids, slots):
    """(h, g, u) fp64 [n][n_ff] for flat slots."""
    E, n_ff, nb, _ = Wg.shape
    ids = np.ascontiguousarray(ids, dtype=np.int32)
    T, k = ids.shape
    slots = np.ascontiguousarray(slots, dtype=np.int64)
    h = np.zeros((len(slots), n_ff), np.float64)
    g = np.zeros_like(h)
    u = np.zeros_like(h)
    _chk(_L().oracle_ffn_hidden(_p(Wg), _p(Wu), E, nb * 32, n_ff, _p(x), DTYPES[x_type], _p(ids), T, k,
                                _p(slots), len(slots), _p(h), _p(g), _p(u), _same_wtype(Wg, Wu)))
    return h, g, u


def combine(dst, r, dst_shared=None):
    """Weighted combine y[t] = sum_s r[t][s]*dst[t][s] (+ dst_shared[t]), fp64,
    ascending s (moe_oracle.c: oracle_combine).  dst float32 [T][k][n] (or
    [T*k][n]), r float32 [T][k], dst_shared float32 [T][n] or None.  Returns
    (y, mag): y float64 [T][n] and mag = sum of the terms' magnitudes."""
    r = np.ascontiguousarray(r, dtype=np.float32)
    T, k = r.shape
    dst = np.ascontiguousarray(dst, dtype=np.float32)
    n = dst.shape[-1]
    dst = dst.reshape(T, k, n)
    sh = None if dst_shared is None else np.ascontiguousarray(dst_shared, dtype=np.float32).reshape(T, n)
    y = np.empty((T, n), dtype=np.float64)
    mag = np.empty((T, n), dtype=np.float64)
    _L().oracle_combine(_p(dst), _p(r), _p(sh), T, k, n, _p(y), _p(mag))
    return y, mag


def combine_tolerance(mag, k, shared):
    """Bound on |float32 evaluation - exact| for the combine as the library
    evaluates it: k fused multiply-adds in ascending s, then one add of the
    shared term, each rounding once (relative 2^-24 of the running magnitude,
    at most mag): (k + 1 + shared) * 2^-24 * mag, plus the smallest normal float
    for sums that vanish."""
    return (k + 1 + (1 if shared else 0)) * 2.0 ** -24 * mag + 1.2e-38


def route(logits, k, bias=None, normalize=True):
    """Router (moe_oracle.c: oracle_route).  logits float32 [T][E], bias float32
    [E] or None.  Returns (ids int32 [T][k], w float64 [T][k], tol float64
    [T][k]): the k largest float32 keys logit + bias in descending order (ties to
    the lower index), their softmax probabilities (renormalised over the k when
    `normalize`), and the bound a float32 evaluation of the weights meets."""
    logits = np.ascontiguousarray(logits, dtype=np.float32)
    T, E = logits.shape
    b = None if bias is None else np.ascontiguousarray(bias, dtype=np.float32).reshape(E)
    ids = np.empty((T, k), dtype=np.int32)
    w = np.empty((T, k), dtype=np.float64)
    st = _L().oracle_route(_p(logits), _p(b), T, E, k, 1 if normalize else 0, _p(ids), _p(w))
    if st != 0:
        raise ValueError("need 1 <= k <= n_experts")
    return ids, w, route_tolerance(w, logits, E, k, normalize)


def route_tolerance(w, logits, E, k, normalize):
    """Relative bound for float32 softmax weights: the exponent's argument
    l - max rounds once (2^-24 of |l - max|, at most the row's logit span), the
    exponential is within a few units in the last place, the sum of E terms
    and of the k chosen ones round once per addition, and the divisions once
    each: (span + 4 + E + k + 4) * 2^-24, applied to |w|."""
    span = (logits.max(axis=1) - logits.min(axis=1)).astype(np.float64)[:, None]
    rel = (span + 8.0 + E + (k if normalize else 0)) * 2.0 ** -24
    return rel * np.abs(w) + 1e-30


def num_threads() -> int:
    """OpenMP threads the oracle's parallel loops use."""
    return int(_L().oracle_num_threads())


def set_num_threads(n: int) -> None:
    """Set the oracle's OpenMP thread count (e.g. to all host cores when a
    launcher capped OMP_NUM_THREADS)."""
    _L().oracle_set_num_threads(int(n))
