"""Small hand-built inputs shared by the CPU pin tests and the GPU parity tests."""
import json
import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def pack_q8_0(d: np.ndarray, q: np.ndarray) -> np.ndarray:
    """Q8_0 block bytes [..., n_in/32, 34] from scales d [..., n_in/32] and int8 q [..., n_in]."""
    d = np.asarray(d, dtype=np.float16)
    q = np.asarray(q, dtype=np.int8)
    nb = q.shape[-1] // 32
    assert d.shape[-1] == nb
    out = np.empty(q.shape[:-1] + (nb, 34), np.uint8)
    out[..., 0:2] = d.reshape(d.shape + (1,)).view(np.uint8).reshape(d.shape + (2,))
    out[..., 2:] = q.reshape(q.shape[:-1] + (nb, 32)).view(np.uint8)
    return out


def unpack_q8_0(W: np.ndarray) -> np.ndarray:
    """fp64 weights from Q8_0 blocks by numpy (independent of the oracle's decoder)."""
    d = np.ascontiguousarray(W[..., 0:2]).view(np.float16)[..., 0].astype(np.float64)
    q = np.ascontiguousarray(W[..., 2:]).view(np.int8).astype(np.float64)
    w = d[..., None] * q
    return w.reshape(W.shape[:-2] + (W.shape[-2] * 32,))


def hand_example():
    """The 2-expert hand-worked case of tests/golden/hand_example_2experts.json."""
    with open(os.path.join(GOLDEN, "hand_example_2experts.json")) as f:
        g = json.load(f)
    j = np.arange(32)
    alt = np.where(j % 2 == 0, 1, -1)
    q = np.zeros((2, 2, 32), np.int8)
    d = np.zeros((2, 2, 1), np.float64)
    q[0, 0] = 1; d[0, 0] = 0.5
    q[0, 1] = j - 16; d[0, 1] = 1.0
    q[1, 0] = alt; d[1, 0] = 0.25
    q[1, 1] = (j < 4).astype(np.int8); d[1, 1] = 2.0
    W = pack_q8_0(d, q)
    xb = np.stack([np.ones(32), j.astype(np.float64), alt.astype(np.float64)]).astype(np.float32)
    xs = np.stack([xb[(t + s) % 3] for t in range(3) for s in range(2)]).astype(np.float32)
    ids = np.array(g["ids"], np.int32)
    return g, W, xb, xs, ids


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """bfloat16 bit patterns (round to nearest even) of float32 values."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = u + 0x7FFF + ((u >> 16) & 1)
    return (u >> 16).astype(np.uint16)


def bf16_bits_to_f64(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, np.uint32) << 16).view(np.float32).astype(np.float64)
