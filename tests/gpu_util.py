"""Helpers for the GPU parity tests: move seeded inputs to the device and
compare the library's outputs with the oracle element by element."""
import numpy as np
import torch

import indirect_expert_matmul_b200 as moe


def to_dev_x(x: np.ndarray, dtype: str) -> torch.Tensor:
    if dtype == "f32":
        return torch.from_numpy(np.ascontiguousarray(x)).cuda()
    t = torch.from_numpy(np.ascontiguousarray(x).view(np.int16))
    return t.view(torch.bfloat16 if dtype == "bf16" else torch.float16).cuda()


def prep(W: np.ndarray) -> torch.Tensor:
    """Upload Q8_0 blocks [E][n_out][n_in/32][34] and repack them on the GPU."""
    E, n_out, nb, _ = W.shape
    raw = torch.from_numpy(np.ascontiguousarray(W)).cuda()
    out = moe.weights_prepare(raw, E, n_out, nb * 32)
    del raw
    return out


def check_close(gpu: torch.Tensor, ref: np.ndarray, tol: np.ndarray, what: str = ""):
    g = gpu.detach().cpu().numpy().astype(np.float64)
    assert g.shape == ref.shape, (g.shape, ref.shape)
    err = np.abs(g - ref)
    bad = ~(err <= tol)  # NaN counts as bad
    if bad.any():
        idx = np.argwhere(bad)[:5]
        msg = ", ".join(f"{tuple(i)}: gpu={g[tuple(i)]!r} ref={ref[tuple(i)]!r} tol={tol[tuple(i)]!r}" for i in idx)
        raise AssertionError(f"{what}: {bad.sum()} of {bad.size} elements outside tolerance; first: {msg}")
    return float((err / tol).max()) if err.size else 0.0


def sample_slots(ids: np.ndarray, n_experts: int, per_expert: int = 2, seed: int = 0) -> np.ndarray:
    """Flat slots t*k+s: `per_expert` per non-empty expert (first and last in
    sorted order plus random ones) - every expert's tiles are visited."""
    flat = ids.reshape(-1)
    rng = np.random.default_rng(seed)
    out = []
    for e in range(n_experts):
        where = np.nonzero(flat == e)[0]
        if len(where) == 0:
            continue
        pick = {int(where[0]), int(where[-1])}
        if len(where) > 2 and per_expert > 2:
            pick.update(int(v) for v in rng.choice(where[1:-1], size=min(per_expert - 2, len(where) - 2),
                                                   replace=False))
        out.extend(sorted(pick)[:max(per_expert, 2)])
    return np.array(sorted(set(out)), np.int64)


class paths:
    """Context manager forcing the library's mat-vec (1) or GEMM (2) path."""

    def __init__(self, path: int):
        self.path = path

    def __enter__(self):
        moe.set_path(self.path)

    def __exit__(self, *a):
        moe.set_path(0)
