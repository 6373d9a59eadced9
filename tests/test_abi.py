"""The C-ABI library loads and exports every symbol include/moe.h declares; its
host-side logic (sizes, argument checks) works without a GPU."""
import ctypes
import os
import re

import pytest

import indirect_expert_matmul_b200 as moe

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    src = ""
    for f in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if f.endswith(".h"):
            src += open(os.path.join(ROOT, "include", f)).read()
    return sorted(set(re.findall(r"MOE_API\s+[\w\s\*]*?\b(moe_\w+)\s*\(", src)))


def test_library_exports_every_declared_symbol():
    syms = declared_symbols()
    assert len(syms) >= 14
    lib = moe.lib()
    missing = [s for s in syms if not hasattr(lib, s)]
    assert not missing, missing
    assert set(syms) == set(moe.ABI_SYMBOLS)


def test_status_strings():
    for code, name in [(0, "MOE_OK"), (-1, "MOE_ERR_INVALID"), (-2, "MOE_ERR_RANGE"), (-3, "MOE_ERR_BAD_ID"),
                       (-4, "MOE_ERR_CUDA"), (-5, "MOE_ERR_TIMEOUT"), (-6, "MOE_ERR_UNSUPPORTED")]:
        assert moe.status_string(code) == name


def test_prepared_size_is_q8_0_size():
    for E, n_out, n_in in [(256, 2048, 7168), (256, 7168, 2048), (128, 2880, 2880), (64, 1408, 2048), (8, 512, 256)]:
        assert moe.weights_prepared_size(E, n_out, n_in) == E * n_out * n_in // 32 * 34
    # padding: n_out to 16, n_in to 64
    assert moe.weights_prepared_size(1, 17, 32) == 32 * 1 * 68
    assert moe.weights_prepared_size(0, 16, 64) == 0


def test_workspace_size_covers_tables_and_hidden():
    T, k, E, n_in, n_ff = 4096, 8, 256, 7168, 2048
    s = moe.workspace_size(T, k, E, n_in, n_ff, 0)
    assert s >= 2 * T * k * 4 + T * k * n_ff * 2 + 3 * (E + 1) * 4
    assert s % 256 == 0
    assert moe.workspace_size(T, k, E, n_in, 0, 0, __import__("torch").float32) >= T * k * n_in * 2


def test_host_argument_checks_without_gpu():
    lib = moe.lib()
    nul = None
    # k > n_experts
    assert lib.moe_row_ids(nul, 4, 3, 2, 0, nul, nul, nul, nul, nul) == moe.ERR_RANGE
    # n_tokens >= 2^22
    assert lib.moe_row_ids(nul, 1 << 22, 1, 2, 0, nul, nul, nul, nul, nul) == moe.ERR_RANGE
    # k >= 2^10
    assert lib.moe_mul_mat_id(nul, 2000, 8, 64, nul, 0, nul, 1, 1024, 0, nul, nul, nul) == moe.ERR_RANGE
    # n_in not a multiple of 32
    assert lib.moe_mul_mat_id(nul, 4, 8, 48, nul, 0, nul, 1, 1, 0, nul, nul, nul) == moe.ERR_INVALID
    # bad mode / dtype
    assert lib.moe_mul_mat_id(nul, 4, 8, 64, nul, 0, nul, 1, 1, 7, nul, nul, nul) == moe.ERR_INVALID
    assert lib.moe_mul_mat_id(nul, 4, 8, 64, nul, 9, nul, 1, 1, 0, nul, nul, nul) == moe.ERR_INVALID
    # null workspace
    assert lib.moe_mul_mat_id(nul, 4, 8, 64, nul, 0, nul, 1, 1, 0, nul, nul, nul) == moe.ERR_INVALID
    # n_experts above the supported maximum
    assert lib.moe_row_ids(nul, 1, 1, 20000, 0, nul, nul, nul, nul, nul) == moe.ERR_RANGE
    # ffn: shared width not a multiple of 32
    assert lib.moe_ffn(nul, nul, nul, 4, 64, 64, nul, nul, nul, 40, nul, 0, nul, 1, 1, nul, nul, nul,
                       nul) == moe.ERR_INVALID
    # the no-workspace entry point: n_tokens far past 2^22 is refused before n_tokens*k is formed
    # (2^61 + 1 times 8 would wrap to 8, under its 64-slot limit)
    for T in ((1 << 61) + 1, 1 << 22):
        assert lib.moe_ffn_decode_noalloc(nul, nul, nul, 256, 2048, 512, nul, nul, nul, 0, nul, 0, nul, T, 8, nul,
                                          nul, nul, nul) == moe.ERR_RANGE
    assert lib.moe_ffn_decode_noalloc(nul, nul, nul, 2048, 2048, 512, nul, nul, nul, 0, nul, 0, nul, 1, 1024, nul,
                                      nul, nul, nul) == moe.ERR_RANGE


def test_router_and_combine_argument_checks_without_gpu():
    lib = moe.lib()
    nul = None
    # router: k outside [1, n_experts], no logits, more than 1024 experts, too many tokens
    assert lib.moe_route(nul, nul, 4, 8, 0, 1, nul, nul, nul) == moe.ERR_INVALID
    assert lib.moe_route(nul, nul, 4, 8, 9, 1, nul, nul, nul) == moe.ERR_INVALID
    assert lib.moe_route(nul, nul, 4, 8, 2, 1, nul, nul, nul) == moe.ERR_INVALID
    assert lib.moe_route(nul, nul, 4, 1025, 2, 1, nul, nul, nul) == moe.ERR_RANGE
    assert lib.moe_route(nul, nul, 1 << 22, 8, 2, 1, nul, nul, nul) == moe.ERR_RANGE
    assert lib.moe_route(nul, nul, 0, 8, 2, 1, nul, nul, nul) == moe.OK  # nothing to do
    # combine: k < 1, n < 1, null pointers, misaligned, k >= 2^10, too many tokens
    assert lib.moe_combine(nul, nul, nul, 4, 0, 8, nul, nul) == moe.ERR_INVALID
    assert lib.moe_combine(nul, nul, nul, 4, 2, 0, nul, nul) == moe.ERR_INVALID
    assert lib.moe_combine(nul, nul, nul, 4, 2, 8, nul, nul) == moe.ERR_INVALID
    assert lib.moe_combine(4098, 4096, nul, 4, 2, 8, 4096, nul) == moe.ERR_INVALID
    assert lib.moe_combine(nul, nul, nul, 4, 1024, 8, nul, nul) == moe.ERR_RANGE
    assert lib.moe_combine(nul, nul, nul, 1 << 22, 2, 8, nul, nul) == moe.ERR_RANGE
    assert lib.moe_combine(nul, nul, nul, 0, 2, 8, nul, nul) == moe.OK


def test_gemv_threshold_setting():
    old = moe.get_gemv_threshold()
    try:
        moe.set_gemv_threshold(3)
        assert moe.get_gemv_threshold() == 3
    finally:
        moe.set_gemv_threshold(old)


def test_caller_buffers_are_checked_before_any_launch(monkeypatch):
    # outputs and workspaces handed in by the caller must hold what the call writes
    import torch
    monkeypatch.setattr(moe, "_gpu", lambda t, name: None)  # no GPU here: accept host tensors as device ones
    moe._need(torch.empty(10), "out", torch.float32, 10)
    with pytest.raises(ValueError, match="holds 9 elements"):
        moe._need(torch.empty(9), "out", torch.float32, 10)


def test_tensors_on_another_device_are_refused(monkeypatch):
    # every tensor of a call must sit on the device whose stream the call uses;
    # "meta" stands in for a second GPU (no GPU here)
    import torch
    monkeypatch.setattr(moe, "_gpu", lambda t, name: None)
    here, other = torch.device("cpu"), torch.device("meta")
    moe._need(torch.empty(4), "out", torch.float32, 4, here)
    with pytest.raises(ValueError, match="is on meta"):
        moe._need(torch.empty(4, device=other), "out", torch.float32, 4, here)
    # through the operators, before the library is called
    called = []
    real = moe.lib()

    class SizesOnly:  # the library's size queries run; any other entry point is recorded
        def __getattr__(self, name):
            if "_size" in name or name == "moe_status_string":
                return getattr(real, name)
            return lambda *a: called.append(name) or 0

    monkeypatch.setattr(moe, "_L", lambda: SizesOnly())
    x = torch.zeros((2, 64), dtype=torch.bfloat16)
    ids = torch.zeros((2, 1), dtype=torch.int32)
    W = torch.empty(moe_prepared_bytes(4, 32, 64), dtype=torch.uint8, device=other)
    with pytest.raises(ValueError, match="W is on meta"):
        moe.mul_mat_id(W, 4, 32, 64, x, ids, ws=torch.empty(1, dtype=torch.uint8))
    with pytest.raises(ValueError, match="ids is on meta"):
        moe.mul_mat_id(W, 4, 32, 64, x, ids.to(other), ws=torch.empty(1, dtype=torch.uint8))
    with pytest.raises(ValueError, match="Wg is on meta"):
        moe.ffn(W, W, W, 4, 64, 32, x, ids, ws=torch.empty(1, dtype=torch.uint8))
    with pytest.raises(ValueError, match="weights is on meta"):
        moe.combine(torch.zeros((2, 1, 8)), torch.zeros((2, 1), device=other))
    with pytest.raises(ValueError, match="bias is on meta"):
        moe.route(torch.zeros((2, 8)), 2, bias=torch.zeros(8, device=other))
    assert not called


def moe_prepared_bytes(E, n_out, n_in):
    return E * ((n_out + 15) // 16 * 16) * ((n_in + 63) // 64) * 68


def test_unknown_weight_type_is_refused():
    lib = moe.lib()
    with pytest.raises(KeyError):
        moe.weights_prepared_size(1, 16, 32, "q4_k")
    assert lib.moe_weights_prepared_size_w(7, 1, 16, 32) == 0
    assert lib.moe_weights_prepare_w(7, 16, 1, 16, 32, 16, None) == moe.ERR_INVALID
    assert lib.moe_mul_mat_id_w(7, None, 4, 8, 64, None, 0, None, 1, 1, 0, None, None, None) == moe.ERR_INVALID
    assert lib.moe_ffn_w(7, None, None, None, 4, 64, 64, None, None, None, 0, None, 0, None, 1, 1, None, None, None,
                         None) == moe.ERR_INVALID
    # MXFP4 sizes: 17 bytes per 32 weights
    assert moe.weights_prepared_size(256, 2048, 7168, "mxfp4") == 256 * 2048 * 7168 // 32 * 17
    assert moe.weights_prepared_size(1, 17, 32, "mxfp4") == 32 * 1 * 34
