"""mul_mat_id and the expert FFN on the GPU against the oracle, at sizes the
oracle finishes in seconds: every element within
|gpu - oracle| <= 2e-3 * sum|w*x| + 1e-5 (propagated through SwiGLU for the FFN).
Both library paths are exercised: the weight-streaming mat-vec kernel and the
tensor-core grouped GEMM.
"""
import numpy as np
import pytest
import torch

import indirect_expert_matmul_b200 as moe
import oracle
import workloads
from tests.fixtures import hand_example
from tests.gpu_util import check_close, paths, prep, to_dev_x

pytestmark = pytest.mark.gpu

PATHS = [pytest.param(1, id="gemv"), pytest.param(2, id="gemm")]  # mat-vec, grouped GEMM


@pytest.mark.parametrize("path", PATHS)
@pytest.mark.parametrize("mode", ["broadcast", "per_slot"])
def test_hand_example_exact(path, mode):
    g, W, xb, xs, ids = hand_example()
    Wp = prep(W)
    x = xb if mode == "broadcast" else xs
    with paths(path):
        dst = moe.mul_mat_id(Wp, 2, 2, 32, to_dev_x(x, "f32"), torch.from_numpy(ids).cuda(), mode)
    want = np.array(g["dst_broadcast" if mode == "broadcast" else "dst_per_slot"], np.float64)
    assert np.array_equal(dst.cpu().numpy().astype(np.float64), want)


@pytest.mark.parametrize("path", PATHS)
def test_tiny_config(path):
    wl = workloads.WORKLOADS["tiny"]
    W = workloads.q8_0_weights(wl.n_experts, wl.n_out, wl.n_in, wl.seed, workloads.T_W)
    T = wl.n_tokens[0]
    x, ids = wl.x(T), wl.ids(T)
    ref, tol = oracle.mul_mat_id(W, x, "f32", ids)
    with paths(path):
        dst = moe.mul_mat_id(prep(W), wl.n_experts, wl.n_out, wl.n_in, to_dev_x(x, "f32"),
                             torch.from_numpy(ids).cuda())
    check_close(dst, ref, tol, f"tiny path {path}")


@pytest.mark.parametrize("path", PATHS)
@pytest.mark.parametrize("mode", ["broadcast", "per_slot"])
@pytest.mark.parametrize("x_type", ["bf16", "f16"])
def test_ragged_shapes(path, mode, x_type):
    """n_out with a 64-row tail tile, n_in with a 32-column tail, odd token counts,
    an expert count above the token count (empty experts)."""
    rng_seed = 3
    E, k, T, n_in, n_out = 40, 3, 37, 160, 208
    W = workloads.q8_0_weights(E, n_out, n_in, rng_seed, 11)
    ids = workloads.routing("uniform", T, E, k, rng_seed)
    rows = T if mode == "broadcast" else T * k
    x = workloads.activations(rows, n_in, x_type, rng_seed, 12)
    ref, tol = oracle.mul_mat_id(W, x, x_type, ids, mode)
    with paths(path):
        dst = moe.mul_mat_id(prep(W), E, n_out, n_in, to_dev_x(x, x_type), torch.from_numpy(ids).cuda(), mode)
    check_close(dst, ref, tol, f"ragged path {path} {mode} {x_type}")


@pytest.mark.parametrize("path", PATHS)
@pytest.mark.parametrize("E,k,T", [(300, 4, 40), (16384, 6, 24), (1024, 1023, 2)])
def test_expert_and_slot_count_limits(path, E, k, T):
    """Beyond 256 experts the GEMM reads its schedule tables from global memory
    (300 experts); the largest expert count (16384) runs the row-id pass with
    one counting chunk; the largest k (1023: 2046 slots, past the mat-vec
    kernel's slot limit, so both settings run the GEMM).  Small matrices keep
    the oracle fast."""
    n_in, n_out = 64, 48
    W = workloads.q8_0_weights(E, n_out, n_in, 17, 13)
    ids = workloads.routing("uniform", T, E, k, 17)
    x = workloads.activations(T, n_in, "bf16", 17, 14)
    ref, tol = oracle.mul_mat_id(W, x, "bf16", ids)
    with paths(path):
        dst = moe.mul_mat_id(prep(W), E, n_out, n_in, to_dev_x(x, "bf16"), torch.from_numpy(ids).cuda())
    check_close(dst, ref, tol, f"limits path {path} E={E} k={k} T={T}")


@pytest.mark.parametrize("path", PATHS)
@pytest.mark.parametrize("mode", ["broadcast", "per_slot"])
def test_skew_shape_small_batch(path, mode):
    """The skewed-load expert shape (2880 x 2880, 128 experts, top-4 Zipf) on
    300 tokens: heavy experts span several column tiles, some get none."""
    wl = workloads.WORKLOADS["skew"]
    T = 250  # 1000 slots: within the mat-vec path's limit of 1024
    W = workloads.q8_0_weights(wl.n_experts, wl.n_out, wl.n_in, wl.seed, workloads.T_W)
    ids = wl.ids(T)
    x = wl.x(T, mode=mode)
    slots = np.arange(T * wl.k)[::7]
    ref, tol = oracle.mul_mat_id_rows(W, x, "bf16", ids, slots, mode)
    with paths(path):
        dst = moe.mul_mat_id(prep(W), wl.n_experts, wl.n_out, wl.n_in, to_dev_x(x, "bf16"),
                             torch.from_numpy(ids).cuda(), mode)
    check_close(dst.reshape(T * wl.k, wl.n_out)[torch.from_numpy(slots).cuda()], ref, tol, f"skew path {path}")


def _ffn_inputs(wl, T, with_shared):
    Wg = workloads.q8_0_weights(wl.n_experts, wl.n_out, wl.n_in, wl.seed, workloads.T_WG)
    Wu = workloads.q8_0_weights(wl.n_experts, wl.n_out, wl.n_in, wl.seed, workloads.T_WU)
    Wd = workloads.q8_0_weights(wl.n_experts, wl.n_in, wl.n_out, wl.seed, workloads.T_WD)
    sh = None
    if with_shared:
        sh = (workloads.q8_0_weights(1, wl.n_ff_shared, wl.n_in, wl.seed, workloads.T_SG),
              workloads.q8_0_weights(1, wl.n_ff_shared, wl.n_in, wl.seed, workloads.T_SU),
              workloads.q8_0_weights(1, wl.n_in, wl.n_ff_shared, wl.seed, workloads.T_SD))
    return Wg, Wu, Wd, sh, wl.x(T), wl.ids(T)


@pytest.mark.parametrize("path", PATHS)
def test_lite_ffn(path):
    """The whole Lite-shaped output (every slot, every element) against the oracle."""
    wl = workloads.WORKLOADS["lite"]
    T = wl.n_tokens[0] if path == 2 else 160  # the mat-vec path takes up to 1024 slots
    Wg, Wu, Wd, _, x, ids = _ffn_inputs(wl, T, False)
    ref, tol = oracle.ffn(Wg, Wu, Wd, x, "bf16", ids)
    with paths(path):
        dst, _ = moe.ffn(prep(Wg), prep(Wu), prep(Wd), wl.n_experts, wl.n_in, wl.n_out, to_dev_x(x, "bf16"),
                         torch.from_numpy(ids).cuda())
    check_close(dst.reshape(T * wl.k, wl.n_in), ref, tol, f"lite path {path}")


@pytest.mark.parametrize("path", [pytest.param(0, id="auto-gemv"), pytest.param(2, id="gemm")])
@pytest.mark.parametrize("T", [1, 4, 8])
def test_decode_ffn_with_shared_expert(path, T):
    wl = workloads.WORKLOADS["decode"]
    Wg, Wu, Wd, sh, x, ids = _ffn_inputs(wl, T, True)
    ref, tol = oracle.ffn(Wg, Wu, Wd, x, "bf16", ids)
    ref_sh, tol_sh = oracle.shared_ffn(*sh, x, "bf16")
    with paths(path):
        dst, dsh = moe.ffn(prep(Wg), prep(Wu), prep(Wd), wl.n_experts, wl.n_in, wl.n_out, to_dev_x(x, "bf16"),
                           torch.from_numpy(ids).cuda(), shared=(prep(sh[0]), prep(sh[1]), prep(sh[2]), wl.n_ff_shared))
    check_close(dst.reshape(T * wl.k, wl.n_in), ref, tol, f"decode T={T} routed")
    check_close(dsh, ref_sh, tol_sh, f"decode T={T} shared")


@pytest.mark.parametrize("n_out", [1024, 1000, 384])
@pytest.mark.parametrize("mode", ["broadcast", "per_slot"])
def test_matvec_row_tile_pairs(n_out, mode):
    """The mat-vec path with many distinct experts over several row tiles: a
    single-matrix launch takes items of two full 128-row tiles (one tensor copy
    for both, every k-step of a row group in one warp) when the padded n_out is
    a multiple of 256 - 1024, and 1000 with the last pair ragged - and 128-row
    items otherwise (384, three tiles)."""
    E, k, T, n_in = 64, 8, 8, 256
    W = workloads.q8_0_weights(E, n_out, n_in, 23, 5)
    ids = workloads.routing("uniform", T, E, k, 23)
    rows = T if mode == "broadcast" else T * k
    x = workloads.activations(rows, n_in, "bf16", 23, 6)
    ref, tol = oracle.mul_mat_id(W, x, "bf16", ids, mode)
    with paths(1):
        dst = moe.mul_mat_id(prep(W), E, n_out, n_in, to_dev_x(x, "bf16"), torch.from_numpy(ids).cuda(), mode)
    check_close(dst, ref, tol, f"mat-vec row tile pairs n_out={n_out} {mode}")


@pytest.mark.parametrize("path", PATHS)
def test_f32_activations_ffn(path):
    """fp32 x goes through fp16 operands for gate/up; bf16 h for down."""
    E, k, T, n_embd, n_ff = 6, 2, 19, 128, 96
    Wg = workloads.q8_0_weights(E, n_ff, n_embd, 9, 1)
    Wu = workloads.q8_0_weights(E, n_ff, n_embd, 9, 2)
    Wd = workloads.q8_0_weights(E, n_embd, n_ff, 9, 3)
    x = workloads.activations(T, n_embd, "f32", 9, 4)
    ids = workloads.routing("uniform", T, E, k, 9)
    ref, tol = oracle.ffn(Wg, Wu, Wd, x, "f32", ids)
    with paths(path):
        dst, _ = moe.ffn(prep(Wg), prep(Wu), prep(Wd), E, n_embd, n_ff, to_dev_x(x, "f32"),
                         torch.from_numpy(ids).cuda())
    check_close(dst.reshape(T * k, n_embd), ref, tol, f"f32 ffn path {path}")


@pytest.mark.parametrize("x_type", ["bf16", "f32"])
def test_gemm_rows_far_from_unit_scale(x_type):
    """The GEMM path stores activations as fp16 after scaling each row by a power
    of two; rows near 2^20 (beyond the fp16 range unscaled), rows near 2^-20 and
    an all-zero row still agree with the oracle element by element."""
    E, k, T, n_in, n_out = 6, 2, 40, 256, 192
    W = workloads.q8_0_weights(E, n_out, n_in, 11, 1)
    x = workloads.activations(T, n_in, x_type, 11, 2)
    f = x.astype(np.uint32).__lshift__(16).view(np.float32) if x_type == "bf16" else x.copy()
    for t in range(T):
        f[t] *= {1: 2.0 ** 20, 2: 2.0 ** -20}.get(t % 4, 1.0) if t != 3 else 0.0
    x = (f.view(np.uint32) >> 16).astype(np.uint16) if x_type == "bf16" else f.astype(np.float32)
    ids = workloads.routing("uniform", T, E, k, 11)
    ref, tol = oracle.mul_mat_id(W, x, x_type, ids)
    with paths(2):
        dst = moe.mul_mat_id(prep(W), E, n_out, n_in, to_dev_x(x, x_type), torch.from_numpy(ids).cuda())
    check_close(dst, ref, tol, f"scaled rows {x_type}")
    assert np.all(ref[3] == 0) and float(dst[3].abs().max()) == 0.0


def test_gemm_is_repeatable():
    wl = workloads.WORKLOADS["tiny"]
    W = workloads.q8_0_weights(wl.n_experts, wl.n_out, wl.n_in, wl.seed, workloads.T_W)
    T = 64
    x, ids = to_dev_x(wl.x(T), "f32"), torch.from_numpy(wl.ids(T)).cuda()
    Wp = prep(W)
    outs = []
    with paths(2):
        for _ in range(10):
            outs.append(moe.mul_mat_id(Wp, wl.n_experts, wl.n_out, wl.n_in, x, ids).cpu())
    for o in outs[1:]:
        assert torch.equal(o.view(torch.int32), outs[0].view(torch.int32))


def test_empty_batch():
    Wp = prep(workloads.q8_0_weights(4, 32, 64, 0, 1))
    x = torch.zeros((0, 64), dtype=torch.bfloat16, device="cuda")
    ids = torch.zeros((0, 2), dtype=torch.int32, device="cuda")
    dst = moe.mul_mat_id(Wp, 4, 32, 64, x, ids)
    assert dst.shape == (0, 2, 32)


def test_bad_id_reports_status():
    Wp = prep(workloads.q8_0_weights(4, 32, 64, 0, 1))
    x = torch.ones((3, 64), dtype=torch.bfloat16, device="cuda")
    ids = torch.tensor([[0, 1], [2, 4], [3, 0]], dtype=torch.int32, device="cuda")
    ws = moe.workspace(3, 2, 4, 64)
    for path in (1, 2):
        with paths(path):
            moe.mul_mat_id(Wp, 4, 32, 64, x, ids, ws=ws)
        assert moe.get_status(ws) == moe.ERR_BAD_ID


def test_host_argument_errors():
    Wp = prep(workloads.q8_0_weights(4, 32, 64, 0, 1))
    x = torch.ones((3, 64), dtype=torch.bfloat16, device="cuda")
    ids = torch.zeros((3, 2), dtype=torch.int32, device="cuda")
    with pytest.raises(moe.MoeError) as e:
        moe.mul_mat_id(Wp, 4, 32, 48, x[:, :48].contiguous(), ids)   # n_in % 32 != 0
    assert e.value.code == moe.ERR_INVALID
    with pytest.raises(moe.MoeError) as e:
        moe.mul_mat_id(Wp, 1, 32, 64, x, ids)                         # k > E
    assert e.value.code == moe.ERR_RANGE
