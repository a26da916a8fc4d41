"""ctypes binding of libnvfp4pw.so: the C-ABI calls under the same names.

Argument marshalling only -- every step of the solve runs in the library's CUDA
kernels.  torch provides device memory and streams.  If the library is not
built, importing the calls raises: there is no CPU fallback.
"""
from __future__ import annotations

import ctypes
import os

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libnvfp4pw.so")
# the same library built with NVFP4_DEBUG (kernel index checks, see
# nvfp4_debug_build in the header); NVFP4PW_DEBUG=1 makes lib() load it
_LIB_DEBUG_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)),
                               "libnvfp4pw_debug.so")

NVFP4_BF16 = 0
NVFP4_F32 = 1

_STATUS = {
    0: "ok", 1: "invalid argument", 2: "unsupported shape", 3: "workspace",
    4: "non-finite input", 5: "not positive definite", 6: "timeout", 7: "CUDA error",
    8: "unsupported parameter", 9: "index left its array (debug build)",
}


class Nvfp4Error(RuntimeError):
    def __init__(self, call, code, detail=None):
        self.code = int(code)
        msg = f"{call}: status {code} ({_STATUS.get(int(code), 'unknown')})"
        super().__init__(msg if detail is None else f"{msg}: {detail}")


class SolveParams(ctypes.Structure):
    _fields_ = [("n_candidates", ctypes.c_int), ("cand_lo", ctypes.c_int),
                ("lazy_batch", ctypes.c_int), ("scale_rule", ctypes.c_int),
                ("precision", ctypes.c_int)]


_lib = None


def lib():
    """The loaded library (the debug build when NVFP4PW_DEBUG=1); raises if it
    has not been built."""
    global _lib
    if _lib is None:
        _lib = _load(_LIB_DEBUG_PATH if os.environ.get("NVFP4PW_DEBUG") == "1" else _LIB_PATH)
    return _lib


_debug_lib = None


def debug_lib():
    """The debug build, loaded beside the release one (its calls take the
    same arguments); raises if it has not been built."""
    global _debug_lib
    if _debug_lib is None:
        _debug_lib = _load(_LIB_DEBUG_PATH)
    return _debug_lib


def _load(path):
    if not os.path.exists(path):
        raise RuntimeError(
            f"{path} is missing: build it with `python -m nvfp4_post_weight_b200.build`")
    L = ctypes.CDLL(path)
    vp, i64, sz, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_size_t, ctypes.c_int
    f32 = ctypes.c_float
    sig = {
        "nvfp4_status_string": ([i32], ctypes.c_char_p),
        "nvfp4_workspace_status": ([vp, vp], i32),
        "nvfp4_default_params": ([ctypes.POINTER(SolveParams)], None),
        "nvfp4_hessian_accumulate": ([vp, vp, i32, i64, i64, i32, vp], i32),
        "nvfp4_hessian_status": ([vp], i32),
        "nvfp4_hessian_host_workspace_size": ([i64, i64, i32], sz),
        "nvfp4_hessian_accumulate_host": ([vp, vp, i32, i64, i64, i32, i64, vp, sz, vp],
                                          i32),
        "nvfp4_prepare_workspace_size": ([i64], sz),
        "nvfp4_hessian_f64_workspace_size": ([i64, i64], sz),
        "nvfp4_hessian_accumulate_f64": ([vp, vp, i32, i64, i64, i32, vp, sz, vp], i32),
        "nvfp4_gptq_prepare_f64": ([vp, i64, f32, vp, vp, vp, vp, sz, vp], i32),
        "nvfp4_gptq_prepare": ([vp, i64, f32, vp, vp, vp, vp, sz, vp], i32),
        "nvfp4_quantize_workspace_size": ([i64, i64, ctypes.POINTER(SolveParams)], sz),
        "nvfp4_gptq_schur_replay_quantize": (
            [vp, i32, i64, i64, vp, ctypes.POINTER(SolveParams), vp, vp, vp, vp, vp, vp, sz,
             vp], i32),
        "nvfp4_gptq_schur_replay_quantize_noalloc": (
            [vp, i32, i64, i64, vp, ctypes.POINTER(SolveParams), vp, vp, vp, vp, vp, vp,
             vp], i32),
        "nvfp4_dequant": ([vp, vp, vp, i64, i64, vp, i32, vp], i32),
        "nvfp4_weight_amax": ([vp, i32, i64, i64, vp, vp, vp], i32),
        "nvfp4_export_scales_size": ([i64, i64], sz),
        "nvfp4_export_scales": ([vp, i64, i64, vp, vp], i32),
        "nvfp4_gptq_schur_replay_quantize_rows": (
            [vp, i32, i64, i64, vp, ctypes.POINTER(SolveParams), vp, vp, vp, vp, vp, vp, vp,
             sz, vp], i32),
        "nvfp4_hessian_accumulate_batched": ([i32, vp, vp, i32, vp, vp, i32, vp], i32),
        "nvfp4_prepare_batched_workspace_size": ([i32, vp], sz),
        "nvfp4_quantize_batched_workspace_size": ([i32, vp, vp, ctypes.POINTER(SolveParams)],
                                                  sz),
        "nvfp4_batched_workspace_status": ([vp, i32, vp, vp], i32),
        "nvfp4_gptq_prepare_batched": ([i32, vp, vp, f32, vp, vp, vp, vp, sz, vp], i32),
        "nvfp4_gptq_schur_replay_quantize_batched": (
            [i32, vp, i32, vp, vp, vp, ctypes.POINTER(SolveParams), vp, vp, vp, vp, vp, vp,
             sz, vp], i32),
        "nvfp4_dequant_batched": ([i32, vp, vp, vp, vp, vp, vp, i32, vp], i32),
        "nvfp4_layer_error_batched_workspace_size": ([i32, vp, vp], sz),
        "nvfp4_layer_error_batched": ([i32, vp, i32, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp],
                                      i32),
        "nvfp4_gemm_nt_f32": ([i64, i64, i64, f32, vp, i64, vp, i64, f32, vp, i64, i32, vp,
                               vp], i32),
        "nvfp4_layer_error_workspace_size": ([i64, i64], sz),
        "nvfp4_layer_error": ([vp, i32, vp, vp, vp, vp, i64, i64, vp, vp, sz, vp], i32),
        "nvfp4_launch_count": ([], ctypes.c_longlong),
        "nvfp4_debug_build": ([], i32),
        "nvfp4_set_wait_limit_ns": ([ctypes.c_ulonglong], i32),
        "nvfp4_profile_begin": ([], i32),
        "nvfp4_profile_end": ([vp, vp, i32], i32),
        "nvfp4_profile_work": ([vp, i32], i32),
    }
    for name, (args, res) in sig.items():
        fn = getattr(L, name)
        fn.argtypes = args
        fn.restype = res
    return L


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check(call, code):
    if code != 0:
        raise Nvfp4Error(call, code)


NVFP4_ERR_INVALID_ARG = 1


def _need(call, t, name, shape=None, dtype=None, numel_min=None, device=True):
    """Host-side check of one tensor argument before the library is called:
    present, contiguous, on a CUDA device (or the host, device=False), of the
    given dtype and shape (or at least numel_min elements).  A mismatch would
    otherwise become an out-of-bounds device access, so it raises
    Nvfp4Error(call, NVFP4_ERR_INVALID_ARG)."""
    def bad(why):
        raise Nvfp4Error(call, NVFP4_ERR_INVALID_ARG, f"{name}: {why}")
    if t is None:
        bad("missing")
    if not isinstance(t, torch.Tensor):
        bad(f"not a tensor ({type(t).__name__})")
    if device and not t.is_cuda:
        bad("not a CUDA tensor")
    if not device and t.is_cuda:
        bad("must be a host tensor")
    if not t.is_contiguous():
        bad("not contiguous")
    if dtype is not None:
        dts = dtype if isinstance(dtype, tuple) else (dtype,)
        if t.dtype not in dts:
            bad(f"dtype {t.dtype}, expected {' or '.join(str(d) for d in dts)}")
    if shape is not None and tuple(t.shape) != tuple(int(v) for v in shape):
        bad(f"shape {tuple(t.shape)}, expected {tuple(int(v) for v in shape)}")
    if numel_min is not None and t.numel() < numel_min:
        bad(f"{t.numel()} elements, expected at least {numel_min}")
    return t


def _opt_need(call, t, name, **kw):
    return None if t is None else _need(call, t, name, **kw)


def _matrix(call, t, name, dtype=None, device=True):
    _need(call, t, name, dtype=dtype, device=device)
    if t.dim() != 2:
        raise Nvfp4Error(call, NVFP4_ERR_INVALID_ARG, f"{name}: expected a matrix")
    return t.shape


_IO_DTYPES = (torch.bfloat16, torch.float32)
_U8, _F32, _F64, _I32 = torch.uint8, torch.float32, torch.float64, torch.int32


def _check_solve_outputs(call, d_out, d_in, codes, scales, global_scale, err_out):
    _need(call, codes, "codes", (d_out, d_in // 2), _U8)
    _need(call, scales, "scales", (d_out, d_in // 16), _U8)
    _need(call, global_scale, "global_scale", (1,), _F32)
    _opt_need(call, err_out, "err_out", shape=(1,), dtype=_F64)


def _ws_bytes(call, ws, need):
    """Workspace tensor: a contiguous uint8 CUDA tensor of at least `need`
    bytes (the library also checks its size and alignment)."""
    _need(call, ws, "workspace", dtype=_U8, numel_min=need)
    return ws.numel()


def _dtype_code(t):
    if t.dtype == torch.bfloat16:
        return NVFP4_BF16
    if t.dtype == torch.float32:
        return NVFP4_F32
    raise TypeError(f"unsupported dtype {t.dtype}")


def workspace(nbytes: int, device) -> torch.Tensor:
    """A 256-byte aligned device byte buffer of at least nbytes."""
    buf = torch.empty(int(nbytes) + 256, dtype=torch.uint8, device=device)
    off = (-buf.data_ptr()) % 256
    return buf[off:off + int(nbytes)]


def default_params() -> SolveParams:
    p = SolveParams()
    lib().nvfp4_default_params(ctypes.byref(p))
    return p


# nvfp4_scale_rule values
SCALE_RULES = {"schur_replay": 0, "amax": 1, "block_mse": 2}


def solve_params(scale_rule="schur_replay") -> SolveParams:
    """The default parameters with the given block-scale rule (a name of
    SCALE_RULES or its integer value)."""
    p = default_params()
    p.scale_rule = SCALE_RULES.get(scale_rule, scale_rule)
    return p


def nvfp4_workspace_status(ws, stream=None) -> int:
    return int(lib().nvfp4_workspace_status(_ptr(ws), _stream(stream)))


def nvfp4_hessian_host_workspace_size(d, chunk_tok, dtype=torch.bfloat16) -> int:
    code = NVFP4_BF16 if dtype == torch.bfloat16 else NVFP4_F32
    return int(lib().nvfp4_hessian_host_workspace_size(int(d), int(chunk_tok), code))


def nvfp4_hessian_accumulate_host(H, X_host, chunk_tok, ws, beta=0, stream=None):
    """H (device) (+)= X_host^T X_host with X_host a CPU tensor (pinned for
    overlap), streamed in chunks of chunk_tok tokens through ws."""
    call = "nvfp4_hessian_accumulate_host"
    n_tok, d = _matrix(call, X_host, "X_host", _IO_DTYPES, device=False)
    _need(call, H, "H", (d, d), _F32)
    nws = _ws_bytes(call, ws, nvfp4_hessian_host_workspace_size(d, chunk_tok, X_host.dtype))
    _check(call, lib().nvfp4_hessian_accumulate_host(
        _ptr(H), ctypes.c_void_p(X_host.data_ptr()), _dtype_code(X_host), n_tok, d, int(beta),
        int(chunk_tok), _ptr(ws), nws, _stream(stream)))


def nvfp4_hessian_accumulate(H, X, beta=0, stream=None):
    call = "nvfp4_hessian_accumulate"
    n_tok, d = _matrix(call, X, "X", _IO_DTYPES)
    _need(call, H, "H", (d, d), _F32)
    _check(call, lib().nvfp4_hessian_accumulate(
        _ptr(H), _ptr(X), _dtype_code(X), n_tok, d, int(beta), _stream(stream)))


def nvfp4_hessian_f64_workspace_size(n_tok, d) -> int:
    return int(lib().nvfp4_hessian_f64_workspace_size(int(n_tok), int(d)))


def nvfp4_hessian_accumulate_f64(H, X, ws, beta=0, stream=None):
    """H (fp64, d x d) (+)= X^T X to fp64 accuracy (int8-slice tensor cores)."""
    call = "nvfp4_hessian_accumulate_f64"
    n_tok, d = _matrix(call, X, "X", _IO_DTYPES)
    _need(call, H, "H", (d, d), _F64)
    nws = _ws_bytes(call, ws, nvfp4_hessian_f64_workspace_size(n_tok, d))
    _check(call, lib().nvfp4_hessian_accumulate_f64(
        _ptr(H), _ptr(X), _dtype_code(X), n_tok, d, int(beta), _ptr(ws), nws, _stream(stream)))


def nvfp4_gptq_prepare_f64(H, damp, U, dead=None, lambda_out=None, ws=None, stream=None):
    """nvfp4_gptq_prepare from an fp64 H."""
    call = "nvfp4_gptq_prepare_f64"
    d, _ = _matrix(call, H, "H", _F64)
    _need(call, H, "H", (d, d))
    _need(call, U, "U", (d, d), _F32)
    _opt_need(call, dead, "dead", shape=(d,), dtype=_U8)
    _opt_need(call, lambda_out, "lambda_out", shape=(1,), dtype=_F32)
    nws = _ws_bytes(call, ws, nvfp4_prepare_workspace_size(d))
    _check(call, lib().nvfp4_gptq_prepare_f64(
        _ptr(H), d, float(damp), _ptr(U), _ptr(dead), _ptr(lambda_out), _ptr(ws), nws,
        _stream(stream)))


def nvfp4_hessian_status(stream=None) -> int:
    return int(lib().nvfp4_hessian_status(_stream(stream)))


def nvfp4_prepare_workspace_size(d) -> int:
    return int(lib().nvfp4_prepare_workspace_size(int(d)))


def nvfp4_gptq_prepare(H, damp, U, dead=None, lambda_out=None, ws=None, stream=None):
    call = "nvfp4_gptq_prepare"
    d, d2 = _matrix(call, H, "H", _F32)
    _need(call, H, "H", (d, d))
    _need(call, U, "U", (d, d), _F32)
    _opt_need(call, dead, "dead", shape=(d,), dtype=_U8)
    _opt_need(call, lambda_out, "lambda_out", shape=(1,), dtype=_F32)
    nws = _ws_bytes(call, ws, nvfp4_prepare_workspace_size(d))
    _check(call, lib().nvfp4_gptq_prepare(
        _ptr(H), d, float(damp), _ptr(U), _ptr(dead), _ptr(lambda_out), _ptr(ws), nws,
        _stream(stream)))


def nvfp4_quantize_workspace_size(d_out, d_in, params=None) -> int:
    p = params if params is not None else default_params()
    return int(lib().nvfp4_quantize_workspace_size(int(d_out), int(d_in), ctypes.byref(p)))


def nvfp4_gptq_schur_replay_quantize(W, U, codes, scales, global_scale, err_out=None,
                                     dead=None, ws=None, params=None, stream=None):
    call = "nvfp4_gptq_schur_replay_quantize"
    d_out, d_in = _matrix(call, W, "W", _IO_DTYPES)
    _need(call, U, "U", (d_in, d_in), _F32)
    _opt_need(call, dead, "dead", shape=(d_in,), dtype=_U8)
    _check_solve_outputs(call, d_out, d_in, codes, scales, global_scale, err_out)
    p = params if params is not None else default_params()
    nws = _ws_bytes(call, ws, nvfp4_quantize_workspace_size(d_out, d_in, p))
    _check(call, lib().nvfp4_gptq_schur_replay_quantize(
        _ptr(W), _dtype_code(W), d_out, d_in, _ptr(U), ctypes.byref(p), _ptr(dead),
        _ptr(codes), _ptr(scales), _ptr(global_scale), _ptr(err_out), _ptr(ws), nws,
        _stream(stream)))


def nvfp4_export_scales_size(d_out, d_in) -> int:
    return int(lib().nvfp4_export_scales_size(int(d_out), int(d_in)))


def nvfp4_export_scales(scales, out, stream=None):
    """scales: (d_out, d_in/16) uint8 device tensor -> out (flat uint8 device
    tensor of nvfp4_export_scales_size bytes) in the 128 x 4 tiled layout."""
    call = "nvfp4_export_scales"
    d_out, nb = _matrix(call, scales, "scales", _U8)
    _need(call, out, "out", dtype=_U8, numel_min=nvfp4_export_scales_size(d_out, nb * 16))
    _check(call, lib().nvfp4_export_scales(
        _ptr(scales), d_out, nb * 16, _ptr(out), _stream(stream)))


def nvfp4_weight_amax(W, amax_out, dead=None, stream=None):
    call = "nvfp4_weight_amax"
    d_out, d_in = _matrix(call, W, "W", _IO_DTYPES)
    _need(call, amax_out, "amax_out", (1,), _F32)
    _opt_need(call, dead, "dead", shape=(d_in,), dtype=_U8)
    _check(call, lib().nvfp4_weight_amax(
        _ptr(W), _dtype_code(W), d_out, d_in, _ptr(dead), _ptr(amax_out), _stream(stream)))


def nvfp4_gptq_schur_replay_quantize_rows(W, U, amax, codes, scales, global_scale, err_out=None,
                                          dead=None, ws=None, params=None, stream=None):
    call = "nvfp4_gptq_schur_replay_quantize_rows"
    d_out, d_in = _matrix(call, W, "W", _IO_DTYPES)
    _need(call, U, "U", (d_in, d_in), _F32)
    _need(call, amax, "amax", (1,), _F32)
    _opt_need(call, dead, "dead", shape=(d_in,), dtype=_U8)
    _check_solve_outputs(call, d_out, d_in, codes, scales, global_scale, err_out)
    p = params if params is not None else default_params()
    nws = _ws_bytes(call, ws, nvfp4_quantize_workspace_size(d_out, d_in, p))
    _check(call, lib().nvfp4_gptq_schur_replay_quantize_rows(
        _ptr(W), _dtype_code(W), d_out, d_in, _ptr(U), ctypes.byref(p), _ptr(dead), _ptr(amax),
        _ptr(codes), _ptr(scales), _ptr(global_scale), _ptr(err_out), _ptr(ws), nws,
        _stream(stream)))


def nvfp4_gptq_schur_replay_quantize_noalloc(W, U, codes, scales, global_scale, err_out=None,
                                             status_out=None, dead=None, params=None,
                                             stream=None):
    """The quantize call without a workspace: the library's fixed device
    scratch array is used instead, for callers that cannot allocate."""
    call = "nvfp4_gptq_schur_replay_quantize_noalloc"
    d_out, d_in = _matrix(call, W, "W", _IO_DTYPES)
    _need(call, U, "U", (d_in, d_in), _F32)
    _opt_need(call, dead, "dead", shape=(d_in,), dtype=_U8)
    _opt_need(call, status_out, "status_out", shape=(1,), dtype=_I32)
    _check_solve_outputs(call, d_out, d_in, codes, scales, global_scale, err_out)
    p = params if params is not None else default_params()
    _check(call,
           lib().nvfp4_gptq_schur_replay_quantize_noalloc(
               _ptr(W), _dtype_code(W), d_out, d_in, _ptr(U), ctypes.byref(p), _ptr(dead),
               _ptr(codes), _ptr(scales), _ptr(global_scale), _ptr(err_out), _ptr(status_out),
               _stream(stream)))


def nvfp4_dequant(codes, scales, global_scale, out, stream=None):
    call = "nvfp4_dequant"
    d_out, d_in = _matrix(call, out, "out", _IO_DTYPES)
    _need(call, codes, "codes", (d_out, d_in // 2), _U8)
    _need(call, scales, "scales", (d_out, d_in // 16), _U8)
    _need(call, global_scale, "global_scale", (1,), _F32)
    _check(call, lib().nvfp4_dequant(
        _ptr(codes), _ptr(scales), _ptr(global_scale), d_out, d_in, _ptr(out),
        _dtype_code(out), _stream(stream)))


def nvfp4_layer_error_workspace_size(d_out, d_in) -> int:
    return int(lib().nvfp4_layer_error_workspace_size(int(d_out), int(d_in)))


def nvfp4_layer_error(W, codes, scales, global_scale, H, err_out, ws, stream=None):
    call = "nvfp4_layer_error"
    d_out, d_in = _matrix(call, W, "W", _IO_DTYPES)
    _need(call, codes, "codes", (d_out, d_in // 2), _U8)
    _need(call, scales, "scales", (d_out, d_in // 16), _U8)
    _need(call, global_scale, "global_scale", (1,), _F32)
    _need(call, H, "H", (d_in, d_in), _F32)
    _need(call, err_out, "err_out", (1,), _F64)
    nws = _ws_bytes(call, ws, nvfp4_layer_error_workspace_size(d_out, d_in))
    _check(call, lib().nvfp4_layer_error(
        _ptr(W), _dtype_code(W), _ptr(codes), _ptr(scales), _ptr(global_scale), _ptr(H),
        d_out, d_in, _ptr(err_out), _ptr(ws), nws, _stream(stream)))


def nvfp4_gemm_nt_f32(P, Q, C, alpha=1.0, beta=0.0, lower=False, status=None, stream=None):
    """C = beta C + alpha P Q^T (3xTF32 on the tensor cores); P, Q, C fp32
    matrices with unit column stride (row strides are passed as leading
    dimensions)."""
    call = "nvfp4_gemm_nt_f32"
    for name, t in (("P", P), ("Q", Q), ("C", C)):
        if not isinstance(t, torch.Tensor) or not t.is_cuda or t.dtype != _F32 or \
                t.dim() != 2 or t.stride(1) != 1:
            raise Nvfp4Error(call, NVFP4_ERR_INVALID_ARG,
                             f"{name}: expected a CUDA fp32 matrix with unit column stride")
    M, K = P.shape
    N = Q.shape[0]
    if Q.shape[1] != K or tuple(C.shape) != (M, N):
        raise Nvfp4Error(call, NVFP4_ERR_INVALID_ARG,
                         f"shapes P {tuple(P.shape)}, Q {tuple(Q.shape)}, C {tuple(C.shape)}")
    if status is not None:
        _need(call, status, "status", (1,), _I32)
    if status is None:
        status = torch.zeros(1, dtype=torch.int32, device=P.device)
    _check("nvfp4_gemm_nt_f32", lib().nvfp4_gemm_nt_f32(
        M, N, K, float(alpha), _ptr(P), P.stride(0), _ptr(Q), Q.stride(0), float(beta), _ptr(C),
        C.stride(0), int(bool(lower)), _ptr(status), _stream(stream)))
    return status


# ---------------------------------------------------------------------------
# batched forms: lists of per-problem tensors -> host arrays of pointers/sizes
# ---------------------------------------------------------------------------
def _ptrs(ts):
    """Host array of device pointers (NULL for None entries), kept alive by
    the caller holding the returned object."""
    arr = (ctypes.c_void_p * len(ts))(*[None if t is None else t.data_ptr() for t in ts])
    return arr


def _i64s(vals):
    return (ctypes.c_int64 * len(vals))(*[int(v) for v in vals])


def _opt(ts):
    return None if ts is None else _ptrs(ts)


def _each(call, n, lists):
    for name, ts in lists.items():
        if ts is not None and len(ts) != n:
            raise Nvfp4Error(call, NVFP4_ERR_INVALID_ARG, f"{name}: {len(ts)} entries, not {n}")


def nvfp4_hessian_accumulate_batched(Hs, Xs, beta=0, stream=None):
    call = "nvfp4_hessian_accumulate_batched"
    n = len(Hs)
    _each(call, n, {"X": Xs})
    if len({x.dtype for x in Xs}) > 1:
        raise Nvfp4Error(call, NVFP4_ERR_INVALID_ARG, "all X must share one dtype")
    for i in range(n):
        _, d = _matrix(call, Xs[i], f"X[{i}]", _IO_DTYPES)
        _need(call, Hs[i], f"H[{i}]", (d, d), _F32)
    _check(call, lib().nvfp4_hessian_accumulate_batched(
        n, _ptrs(Hs), _ptrs(Xs), _dtype_code(Xs[0]) if n else 0,
        _i64s([x.shape[0] for x in Xs]), _i64s([x.shape[1] for x in Xs]), int(beta),
        _stream(stream)))


def nvfp4_prepare_batched_workspace_size(ds) -> int:
    return int(lib().nvfp4_prepare_batched_workspace_size(len(ds), _i64s(ds)))


def nvfp4_quantize_batched_workspace_size(shapes, params=None) -> int:
    """shapes: [(d_out, d_in)] of the problems."""
    p = params if params is not None else default_params()
    return int(lib().nvfp4_quantize_batched_workspace_size(
        len(shapes), _i64s([s[0] for s in shapes]), _i64s([s[1] for s in shapes]),
        ctypes.byref(p)))


def nvfp4_batched_workspace_status(ws, count, stream=None):
    """(first non-OK status of any problem, [status of each problem])."""
    st = (ctypes.c_int * max(count, 1))()
    r = int(lib().nvfp4_batched_workspace_status(_ptr(ws), int(count), st, _stream(stream)))
    return r, [int(st[i]) for i in range(count)]


def nvfp4_gptq_prepare_batched(Hs, damp, Us, deads=None, lambdas=None, ws=None, stream=None):
    """All factors in one call; ws: one workspace of
    nvfp4_prepare_batched_workspace_size bytes for the whole call."""
    call = "nvfp4_gptq_prepare_batched"
    n = len(Hs)
    _each(call, n, {"U": Us, "dead": deads, "lambda_out": lambdas})
    ds = []
    for i in range(n):
        d, _ = _matrix(call, Hs[i], f"H[{i}]", _F32)
        _need(call, Hs[i], f"H[{i}]", (d, d))
        _need(call, Us[i], f"U[{i}]", (d, d), _F32)
        if deads is not None:
            _opt_need(call, deads[i], f"dead[{i}]", shape=(d,), dtype=_U8)
        if lambdas is not None:
            _opt_need(call, lambdas[i], f"lambda_out[{i}]", shape=(1,), dtype=_F32)
        ds.append(d)
    nws = _ws_bytes(call, ws, nvfp4_prepare_batched_workspace_size(ds)) if n else 0
    _check(call, lib().nvfp4_gptq_prepare_batched(
        n, _ptrs(Hs), _i64s(ds), float(damp), _ptrs(Us), _opt(deads), _opt(lambdas), _ptr(ws),
        nws, _stream(stream)))


def nvfp4_gptq_schur_replay_quantize_batched(Ws, Us, codes, scales, global_scales,
                                             errs=None, deads=None, ws=None, params=None,
                                             stream=None):
    """All weight matrices in one call; ws: one workspace of
    nvfp4_quantize_batched_workspace_size bytes for the whole call."""
    call = "nvfp4_gptq_schur_replay_quantize_batched"
    n = len(Ws)
    _each(call, n, {"U": Us, "codes": codes, "scales": scales, "global_scale": global_scales,
                    "err_out": errs, "dead": deads})
    if len({w.dtype for w in Ws}) > 1:
        raise Nvfp4Error(call, NVFP4_ERR_INVALID_ARG, "all W must share one dtype")
    p = params if params is not None else default_params()
    shapes = []
    for i in range(n):
        d_out, d_in = _matrix(call, Ws[i], f"W[{i}]", _IO_DTYPES)
        _need(call, Us[i], f"U[{i}]", (d_in, d_in), _F32)
        if deads is not None:
            _opt_need(call, deads[i], f"dead[{i}]", shape=(d_in,), dtype=_U8)
        _check_solve_outputs(call, d_out, d_in, codes[i], scales[i], global_scales[i],
                             None if errs is None else errs[i])
        shapes.append((d_out, d_in))
    nws = _ws_bytes(call, ws, nvfp4_quantize_batched_workspace_size(shapes, p)) if n else 0
    _check(call,
           lib().nvfp4_gptq_schur_replay_quantize_batched(
               n, _ptrs(Ws), _dtype_code(Ws[0]) if n else 0, _i64s([s[0] for s in shapes]),
               _i64s([s[1] for s in shapes]), _ptrs(Us), ctypes.byref(p), _opt(deads),
               _ptrs(codes), _ptrs(scales), _ptrs(global_scales), _opt(errs), _ptr(ws), nws,
               _stream(stream)))


def nvfp4_dequant_batched(codes, scales, global_scales, outs, stream=None):
    call = "nvfp4_dequant_batched"
    n = len(outs)
    _each(call, n, {"codes": codes, "scales": scales, "global_scale": global_scales})
    if len({o.dtype for o in outs}) > 1:
        raise Nvfp4Error(call, NVFP4_ERR_INVALID_ARG, "all outputs must share one dtype")
    for i in range(n):
        d_out, d_in = _matrix(call, outs[i], f"out[{i}]", _IO_DTYPES)
        _need(call, codes[i], f"codes[{i}]", (d_out, d_in // 2), _U8)
        _need(call, scales[i], f"scales[{i}]", (d_out, d_in // 16), _U8)
        _need(call, global_scales[i], f"global_scale[{i}]", (1,), _F32)
    _check(call, lib().nvfp4_dequant_batched(
        n, _ptrs(codes), _ptrs(scales), _ptrs(global_scales), _i64s([o.shape[0] for o in outs]),
        _i64s([o.shape[1] for o in outs]), _ptrs(outs), _dtype_code(outs[0]) if n else 0,
        _stream(stream)))


def nvfp4_set_wait_limit_ns(ns: int) -> None:
    """Pipeline-wait limit of the library's tensor-core kernels on the
    current device (0: the default 4 s); for testing the timeout path."""
    _check("nvfp4_set_wait_limit_ns", lib().nvfp4_set_wait_limit_ns(int(ns)))


def nvfp4_layer_error_batched_workspace_size(shapes) -> int:
    """shapes: [(d_out, d_in)] of the problems."""
    return int(lib().nvfp4_layer_error_batched_workspace_size(
        len(shapes), _i64s([s[0] for s in shapes]), _i64s([s[1] for s in shapes])))


def nvfp4_layer_error_batched(Ws, codes, scales, global_scales, Hs, errs, ws, stream=None):
    """Every problem's tr((W - Q) H (W - Q)^T) in one call (one workspace)."""
    call = "nvfp4_layer_error_batched"
    n = len(Ws)
    _each(call, n, {"codes": codes, "scales": scales, "global_scale": global_scales, "H": Hs,
                    "err_out": errs})
    if len({w.dtype for w in Ws}) > 1:
        raise Nvfp4Error(call, NVFP4_ERR_INVALID_ARG, "all W must share one dtype")
    shapes = []
    for i in range(n):
        d_out, d_in = _matrix(call, Ws[i], f"W[{i}]", _IO_DTYPES)
        _need(call, codes[i], f"codes[{i}]", (d_out, d_in // 2), _U8)
        _need(call, scales[i], f"scales[{i}]", (d_out, d_in // 16), _U8)
        _need(call, global_scales[i], f"global_scale[{i}]", (1,), _F32)
        _need(call, Hs[i], f"H[{i}]", (d_in, d_in), _F32)
        _need(call, errs[i], f"err_out[{i}]", (1,), _F64)
        shapes.append((d_out, d_in))
    nws = _ws_bytes(call, ws, nvfp4_layer_error_batched_workspace_size(shapes)) if n else 0
    _check(call, lib().nvfp4_layer_error_batched(
        n, _ptrs(Ws), _dtype_code(Ws[0]) if n else 0, _ptrs(codes), _ptrs(scales),
        _ptrs(global_scales), _ptrs(Hs), _i64s([s[0] for s in shapes]),
        _i64s([s[1] for s in shapes]), _ptrs(errs), _ptr(ws), nws, _stream(stream)))
