"""The C-ABI library loads and exports every function its public header
declares (no GPU needed: nothing here launches a kernel), and the host-side
argument checks answer without touching the device."""
import ctypes
import os
import re

import pytest

from nvfp4_post_weight_b200 import binding as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "nvfp4pw.h")


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", " ", src, flags=re.S)
    src = re.sub(r"//[^\n]*", " ", src)
    names = re.findall(r"\b([A-Za-z_][A-Za-z0-9_]*)\s*\([^;{}]*\)\s*;", src)
    return sorted({n for n in names if n.startswith("nvfp4_")})


def test_header_declares_the_path():
    names = declared_functions()
    for n in ("nvfp4_hessian_accumulate", "nvfp4_gptq_prepare",
              "nvfp4_gptq_schur_replay_quantize", "nvfp4_dequant", "nvfp4_layer_error"):
        assert n in names


def test_library_exports_every_declared_function():
    lib = ctypes.CDLL(B._LIB_PATH)
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing


def test_debug_library_exports_the_same_calls_and_says_so():
    """libnvfp4pw_debug.so (NVFP4_DEBUG: kernel index checks) is the same ABI;
    nvfp4_debug_build tells the two apart."""
    dbg = ctypes.CDLL(B._LIB_DEBUG_PATH)
    missing = [n for n in declared_functions() if not hasattr(dbg, n)]
    assert not missing, missing
    assert B.debug_lib().nvfp4_debug_build() == 1
    assert B.lib().nvfp4_debug_build() == 0
    assert B.lib().nvfp4_status_string(9) == b"index left its array (debug build check)"


def test_binding_covers_every_declared_function():
    lib = B.lib()
    for n in declared_functions():
        assert getattr(lib, n).restype is not None or n in (
            "nvfp4_default_params",), n


def test_host_side_checks_need_no_device():
    L = B.lib()
    null = None
    # d_in not a multiple of 16 -> NVFP4_ERR_SHAPE before any device work
    assert L.nvfp4_gptq_schur_replay_quantize(
        ctypes.c_void_p(256), 0, 4, 20, ctypes.c_void_p(256), null, null,
        ctypes.c_void_p(256), ctypes.c_void_p(256), ctypes.c_void_p(256), null,
        ctypes.c_void_p(256), 1 << 20, null) == 2
    # negative sizes -> NVFP4_ERR_INVALID_ARG
    assert L.nvfp4_dequant(null, null, null, -1, 16, null, 0, null) == 1
    # a workspace that is too small -> NVFP4_ERR_WORKSPACE
    assert L.nvfp4_gptq_prepare(ctypes.c_void_p(256), 32, 0.01, ctypes.c_void_p(256), null,
                                null, ctypes.c_void_p(256), 16, null) == 3
    # host-streamed Hessian: bad chunk size, missing workspace, shape
    assert L.nvfp4_hessian_accumulate_host(ctypes.c_void_p(256), ctypes.c_void_p(256), 0, 100,
                                           256, 0, 0, ctypes.c_void_p(256), 1 << 30, null) == 1
    assert L.nvfp4_hessian_accumulate_host(ctypes.c_void_p(256), ctypes.c_void_p(256), 0, 100,
                                           256, 0, 64, null, 0, null) == 3
    assert L.nvfp4_hessian_accumulate_host(ctypes.c_void_p(256), ctypes.c_void_p(256), 0, 100,
                                           250, 0, 64, ctypes.c_void_p(256), 1 << 30, null) == 2
    assert B.nvfp4_hessian_host_workspace_size(256, 1024) == 2 * 1024 * 256 * 2
    assert L.nvfp4_hessian_host_workspace_size(256, 0, 0) == 0
    # an unknown block-scale rule -> NVFP4_ERR_UNSUPPORTED
    bad = B.solve_params(3)
    assert L.nvfp4_gptq_schur_replay_quantize(
        ctypes.c_void_p(256), 0, 4, 32, ctypes.c_void_p(256), ctypes.byref(bad), null,
        ctypes.c_void_p(256), ctypes.c_void_p(256), ctypes.c_void_p(256), null,
        ctypes.c_void_p(256), 1 << 20, null) == 8
    assert B.solve_params("block_mse").scale_rule == 2 and B.default_params().scale_rule == 0
    # the allocation-free quantize refuses layers beyond its fixed scratch
    assert L.nvfp4_gptq_schur_replay_quantize_noalloc(
        ctypes.c_void_p(256), 0, 4096, 4096, ctypes.c_void_p(256), null, null,
        ctypes.c_void_p(256), ctypes.c_void_p(256), ctypes.c_void_p(256), null, null,
        null) == 3
    # batched forms: count < 0 or missing arrays are rejected on the host
    assert L.nvfp4_hessian_accumulate_batched(-1, null, null, 0, null, null, 0, null) == 1
    assert L.nvfp4_gptq_prepare_batched(2, null, null, 0.01, null, null, null, null, 0,
                                        null) == 1
    assert L.nvfp4_dequant_batched(0, null, null, null, null, null, null, 0, null) == 0
    # a batched workspace that is too small -> NVFP4_ERR_WORKSPACE (nothing queued)
    H = (ctypes.c_void_p * 2)(256, 512)
    d = (ctypes.c_int64 * 2)(32, 32)
    assert L.nvfp4_gptq_prepare_batched(2, H, d, 0.01, H, null, null, ctypes.c_void_p(256), 16,
                                        null) == 3
    # a problem with a bad shape decides the status before anything is queued
    d_bad = (ctypes.c_int64 * 2)(32, 20)
    assert L.nvfp4_gptq_prepare_batched(2, H, d_bad, 0.01, H, null, null, ctypes.c_void_p(256),
                                        1 << 30, null) == 2
    # an unsupported precision -> NVFP4_ERR_UNSUPPORTED
    p = B.default_params()
    assert p.precision == 0
    p.precision = 1
    assert L.nvfp4_gptq_schur_replay_quantize(
        ctypes.c_void_p(256), 0, 4, 32, ctypes.c_void_p(256), ctypes.byref(p), null,
        ctypes.c_void_p(256), ctypes.c_void_p(256), ctypes.c_void_p(256), null,
        ctypes.c_void_p(256), 1 << 20, null) == 8
    assert L.nvfp4_status_string(5) == b"damped Hessian is not positive definite"
    assert L.nvfp4_prepare_workspace_size(-1) == 0


@pytest.mark.parametrize("d_out,d_in", [(0, 0), (1, 16), (4096, 4096)])
def test_workspace_sizes_grow_with_the_layer(d_out, d_in):
    q = B.nvfp4_quantize_workspace_size(d_out, d_in)
    assert q >= 8 * d_out * d_in
    assert B.nvfp4_prepare_workspace_size(d_in) >= 4 * d_in * d_in


def test_batched_workspace_covers_the_problems():
    """One workspace for a batched call: at least every problem's own scratch
    arrays, at most the single-call workspaces plus the status header."""
    ds = [4096, 1536, 4096, 4096, 1536]
    b = B.nvfp4_prepare_batched_workspace_size(ds)
    singles = sum(B.nvfp4_prepare_workspace_size(d) for d in ds)
    assert sum(3 * 8 * d * d for d in ds) <= b <= singles + 256 * (len(ds) + 1)
    shapes = [(1536, 4096), (1536, 4096), (4096, 1536)] * 3
    q = B.nvfp4_quantize_batched_workspace_size(shapes)
    qs = sum(B.nvfp4_quantize_workspace_size(*s) for s in shapes)
    assert sum(8 * o * i for o, i in shapes) <= q <= qs + 256 * (len(shapes) + 1)
    assert B.nvfp4_prepare_batched_workspace_size([]) > 0   # the status header


def test_binding_rejects_bad_buffers_on_the_host():
    """Tensor arguments are checked before the library is called: a buffer of
    the wrong kind is NVFP4_ERR_INVALID_ARG, not a device access."""
    import torch
    codes = torch.zeros((4, 16), dtype=torch.uint8)
    scales = torch.zeros((4, 2), dtype=torch.uint8)
    sg = torch.zeros(1)
    out = torch.zeros((4, 32))
    with pytest.raises(B.Nvfp4Error) as e:
        B.nvfp4_dequant(codes, scales, sg, out)     # host tensors
    assert e.value.code == 1 and "CUDA" in str(e.value)
    with pytest.raises(B.Nvfp4Error) as e:
        B._need("call", torch.zeros((4, 8), dtype=torch.uint8), "codes", (4, 16), torch.uint8,
                device=False)
    assert e.value.code == 1 and "shape" in str(e.value)
    with pytest.raises(B.Nvfp4Error):
        B._need("call", torch.zeros((4, 16)).t(), "W", device=False)   # not contiguous
    with pytest.raises(B.Nvfp4Error):
        B._need("call", torch.zeros(3), "ws", dtype=torch.uint8, device=False)
    with pytest.raises(B.Nvfp4Error):
        B._need("call", torch.zeros(8, dtype=torch.uint8), "ws", numel_min=16, device=False)
