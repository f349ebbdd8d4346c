"""ctypes binding of libswimba.so (include/swimba.h): argument marshalling only.

Every function named ``swimba_*`` here calls the C function of the same name with device pointers
taken from torch tensors (``tensor.data_ptr()``) and the current torch CUDA stream unless one is
given. Every step of the layer runs in the library's CUDA kernels; there is no Python or CPU
compute path. Importing this module fails loudly when the library has not been built.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libswimba.so")
if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python -m parameter_space_moe_swimba_b200.build` "
        "(nvcc, sm_100a)"
    )
_lib = ctypes.CDLL(LIB_PATH)

import torch  # noqa: E402  (after the library check so a missing build is reported first)

SWIMBA_F32 = 0
SWIMBA_BF16 = 1
(SWIMBA_OP_ROUTE, SWIMBA_OP_PROJ, SWIMBA_OP_SCAN, SWIMBA_OP_STEP, SWIMBA_OP_LAYER, SWIMBA_OP_SUMMARY,
 SWIMBA_OP_SEPARATE, SWIMBA_OP_SCAN_BWD, SWIMBA_OP_PROJ_BWD, SWIMBA_OP_ROUTE_BWD) = range(10)

STATUS = {
    0: "SWIMBA_OK",
    1: "SWIMBA_ERR_INVALID_ARG",
    2: "SWIMBA_ERR_UNSUPPORTED",
    3: "SWIMBA_ERR_ALIGN",
    4: "SWIMBA_ERR_WORKSPACE",
    5: "SWIMBA_ERR_CUDA",
    6: "SWIMBA_ERR_TIMEOUT",
}

# Every symbol include/swimba.h declares.
EXPORTED = [
    "swimba_workspace_size",
    "swimba_route",
    "swimba_mixed_proj",
    "swimba_scan_fwd",
    "swimba_scan_fwd_zoh",
    "swimba_scan_fwd_noalloc",
    "swimba_scan_fwd_noalloc_status",
    "swimba_scan_fwd_noalloc_status_block",
    "swimba_scan_summary",
    "swimba_scan_chain",
    "swimba_scan_bwd",
    "swimba_proj_bwd",
    "swimba_route_bwd",
    "swimba_ssd_scan",
    "swimba_separate_proj",
    "swimba_separate_scan",
    "swimba_step",
    "swimba_get_device_status",
    "swimba_check_wait_timeout",
    "swimba_status_string",
    "swimba_kernel_launches",
    "swimba_last_error_string",
    "swimba_conv1d_fwd",
    "swimba_conv1d_step",
    "swimba_block_gemm",
    "swimba_block_workspace_size",
    "swimba_block_fwd",
    "swimba_block_step",
]


class swimba_dims(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int64),
        ("seqlen", ctypes.c_int64),
        ("d_inner", ctypes.c_int32),
        ("d_state", ctypes.c_int32),
        ("dt_rank", ctypes.c_int32),
        ("n_experts", ctypes.c_int32),
        ("top_k", ctypes.c_int32),
        ("io_dtype", ctypes.c_int32),
        ("w_dtype", ctypes.c_int32),
    ]


class swimba_ssd_dims(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int64),
        ("seqlen", ctypes.c_int64),
        ("n_heads", ctypes.c_int32),
        ("head_dim", ctypes.c_int32),
        ("d_state", ctypes.c_int32),
        ("top_k", ctypes.c_int32),
    ]


class swimba_weights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("W_r", "W_x", "W_dt", "b_dt", "A", "D_skip")]


class swimba_block_dims(ctypes.Structure):
    _fields_ = [("layer", swimba_dims), ("d_model", ctypes.c_int32), ("d_conv", ctypes.c_int32)]


class swimba_block_weights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("W_in", "conv_w", "conv_b", "W_out")] + [("layer", swimba_weights)]


_P = ctypes.c_void_p
_lib.swimba_workspace_size.argtypes = [ctypes.POINTER(swimba_dims), ctypes.c_int]
_lib.swimba_workspace_size.restype = ctypes.c_size_t
_lib.swimba_route.argtypes = [ctypes.POINTER(swimba_dims), _P, _P, _P, _P, _P]
_lib.swimba_route.restype = ctypes.c_int
_lib.swimba_mixed_proj.argtypes = [ctypes.POINTER(swimba_dims), _P, _P, _P, ctypes.POINTER(swimba_weights), _P, _P,
                                   _P, _P, ctypes.c_size_t, _P]
_lib.swimba_mixed_proj.restype = ctypes.c_int
_lib.swimba_scan_fwd.argtypes = [ctypes.POINTER(swimba_dims), _P, _P, _P, _P, _P, _P, _P,
                                 ctypes.POINTER(swimba_weights), _P, _P, _P, _P, _P, ctypes.c_size_t, _P]
_lib.swimba_scan_fwd.restype = ctypes.c_int
_lib.swimba_scan_fwd_zoh.argtypes = _lib.swimba_scan_fwd.argtypes
_lib.swimba_scan_fwd_zoh.restype = ctypes.c_int
_lib.swimba_scan_fwd_noalloc.argtypes = [ctypes.POINTER(swimba_dims), _P, _P, _P, _P, _P, _P, _P,
                                         ctypes.POINTER(swimba_weights), _P, _P, _P, _P, _P]
_lib.swimba_scan_fwd_noalloc.restype = ctypes.c_int
_lib.swimba_scan_fwd_noalloc_status.argtypes = [_P]
_lib.swimba_scan_fwd_noalloc_status.restype = ctypes.c_int
_lib.swimba_scan_fwd_noalloc_status_block.argtypes = []
_lib.swimba_scan_fwd_noalloc_status_block.restype = ctypes.c_void_p
_lib.swimba_scan_summary.argtypes = [ctypes.POINTER(swimba_dims), _P, _P, _P, _P, _P, ctypes.POINTER(swimba_weights),
                                     _P, _P, _P, ctypes.c_size_t, _P]
_lib.swimba_scan_summary.restype = ctypes.c_int
_lib.swimba_scan_chain.argtypes = [ctypes.POINTER(swimba_dims), ctypes.c_int32, _P, _P, _P, _P, _P]
_lib.swimba_scan_chain.restype = ctypes.c_int
_lib.swimba_scan_bwd.argtypes = [ctypes.POINTER(swimba_dims)] + [_P] * 7 + [ctypes.POINTER(swimba_weights)] + \
    [_P] * 11 + [_P, ctypes.c_size_t, _P]
_lib.swimba_scan_bwd.restype = ctypes.c_int
_lib.swimba_proj_bwd.argtypes = [ctypes.POINTER(swimba_dims), _P, _P, _P, ctypes.POINTER(swimba_weights)] + \
    [_P] * 5 + [ctypes.c_int32] + [_P] * 5 + [ctypes.c_size_t, _P]
_lib.swimba_proj_bwd.restype = ctypes.c_int
_lib.swimba_route_bwd.argtypes = [ctypes.POINTER(swimba_dims)] + [_P] * 7 + [ctypes.c_int32, _P, _P, ctypes.c_size_t, _P]
_lib.swimba_route_bwd.restype = ctypes.c_int
_lib.swimba_ssd_scan.argtypes = [ctypes.POINTER(swimba_ssd_dims)] + [_P] * 10 + [_P, ctypes.c_size_t, _P]
_lib.swimba_ssd_scan.restype = ctypes.c_int
_lib.swimba_separate_proj.argtypes = [ctypes.POINTER(swimba_dims), _P, _P, _P, ctypes.POINTER(swimba_weights), _P,
                                      _P, _P, _P]
_lib.swimba_separate_proj.restype = ctypes.c_int
_lib.swimba_separate_scan.argtypes = [ctypes.POINTER(swimba_dims), _P, _P, _P, _P, _P, _P, _P,
                                      ctypes.POINTER(swimba_weights), _P, _P, _P, _P, _P, ctypes.c_size_t, _P]
_lib.swimba_separate_scan.restype = ctypes.c_int
_lib.swimba_step.argtypes = [ctypes.POINTER(swimba_dims), _P, _P, _P, _P, _P, _P, _P,
                             ctypes.POINTER(swimba_weights), _P, _P, _P]
_lib.swimba_step.restype = ctypes.c_int
_lib.swimba_get_device_status.argtypes = [_P, _P]
_lib.swimba_get_device_status.restype = ctypes.c_int
_lib.swimba_check_wait_timeout.argtypes = [_P, ctypes.c_size_t, ctypes.c_uint64, _P]
_lib.swimba_check_wait_timeout.restype = ctypes.c_int
_lib.swimba_status_string.argtypes = [ctypes.c_int]
_lib.swimba_status_string.restype = ctypes.c_char_p
_lib.swimba_last_error_string.argtypes = []
_lib.swimba_last_error_string.restype = ctypes.c_char_p
_lib.swimba_kernel_launches.argtypes = []
_lib.swimba_kernel_launches.restype = ctypes.c_uint64
_lib.swimba_conv1d_fwd.argtypes = [ctypes.POINTER(swimba_dims), ctypes.c_int32, _P, _P, _P, _P, _P, _P, _P]
_lib.swimba_conv1d_fwd.restype = ctypes.c_int
_lib.swimba_conv1d_step.argtypes = [ctypes.POINTER(swimba_dims), ctypes.c_int32, _P, _P, _P, _P, _P, _P]
_lib.swimba_conv1d_step.restype = ctypes.c_int
_I = ctypes.c_int32
_lib.swimba_block_gemm.argtypes = [_I, _I, _I, _I, _P, _I, _P, _I, _P, _I, _P, _I, _I, _P, _I, _P, ctypes.c_size_t, _P]
_lib.swimba_block_gemm.restype = ctypes.c_int
_lib.swimba_block_workspace_size.argtypes = [ctypes.POINTER(swimba_block_dims)]
_lib.swimba_block_workspace_size.restype = ctypes.c_size_t
_lib.swimba_block_fwd.argtypes = [ctypes.POINTER(swimba_block_dims), _P, ctypes.POINTER(swimba_block_weights), _P, _P,
                                  _P, _P, _P, _P, ctypes.c_size_t, _P]
_lib.swimba_block_fwd.restype = ctypes.c_int
_lib.swimba_block_step.argtypes = [ctypes.POINTER(swimba_block_dims), _P, ctypes.POINTER(swimba_block_weights), _P,
                                   _P, _P, _P, ctypes.c_size_t, _P]
_lib.swimba_block_step.restype = ctypes.c_int


class SwimbaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        detail = f"; {swimba_last_error_string()}" if status == 5 else ""
        super().__init__(f"{where}: {STATUS.get(status, status)} ({swimba_status_string(status)}{detail})")


def _ptr(t) -> int | None:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def check(status: int, where: str = "swimba") -> None:
    if status != 0:
        raise SwimbaError(status, where)


# ------------------------------------------------------------------------------------------------
# the C functions, same names
# ------------------------------------------------------------------------------------------------

def swimba_status_string(status: int) -> str:
    return _lib.swimba_status_string(int(status)).decode()


def swimba_last_error_string() -> str:
    return _lib.swimba_last_error_string().decode()


def swimba_kernel_launches() -> int:
    return int(_lib.swimba_kernel_launches())


def swimba_workspace_size(dims: swimba_dims, op: int) -> int:
    return int(_lib.swimba_workspace_size(ctypes.byref(dims), op))


def swimba_route(dims, x, W_r, idx, gates, stream=None) -> int:
    return _lib.swimba_route(ctypes.byref(dims), _ptr(x), _ptr(W_r), _ptr(idx), _ptr(gates), _stream(stream))


def swimba_mixed_proj(dims, x, idx, gates, weights, delta, B_mix, C_mix, ws, ws_bytes, stream=None) -> int:
    return _lib.swimba_mixed_proj(ctypes.byref(dims), _ptr(x), _ptr(idx), _ptr(gates), ctypes.byref(weights),
                                  _ptr(delta), _ptr(B_mix), _ptr(C_mix), _ptr(ws), int(ws_bytes), _stream(stream))


def swimba_scan_fwd(dims, x, z, delta, B_mix, C_mix, idx, gates, weights, h0, out, h_final, y_pre, ws, ws_bytes,
                    stream=None) -> int:
    return _lib.swimba_scan_fwd(ctypes.byref(dims), _ptr(x), _ptr(z), _ptr(delta), _ptr(B_mix), _ptr(C_mix),
                                _ptr(idx), _ptr(gates), ctypes.byref(weights), _ptr(h0), _ptr(out), _ptr(h_final),
                                _ptr(y_pre), _ptr(ws), int(ws_bytes), _stream(stream))


def swimba_scan_fwd_zoh(dims, x, z, delta, B_mix, C_mix, idx, gates, weights, h0, out, h_final, y_pre, ws, ws_bytes,
                        stream=None) -> int:
    return _lib.swimba_scan_fwd_zoh(ctypes.byref(dims), _ptr(x), _ptr(z), _ptr(delta), _ptr(B_mix), _ptr(C_mix),
                                    _ptr(idx), _ptr(gates), ctypes.byref(weights), _ptr(h0), _ptr(out),
                                    _ptr(h_final), _ptr(y_pre), _ptr(ws), int(ws_bytes), _stream(stream))


def swimba_scan_fwd_noalloc(dims, x, z, delta, B_mix, C_mix, idx, gates, weights, h0, out, h_final, y_pre,
                            stream=None) -> int:
    return _lib.swimba_scan_fwd_noalloc(ctypes.byref(dims), _ptr(x), _ptr(z), _ptr(delta), _ptr(B_mix), _ptr(C_mix),
                                        _ptr(idx), _ptr(gates), ctypes.byref(weights), _ptr(h0), _ptr(out),
                                        _ptr(h_final), _ptr(y_pre), _stream(stream))


def swimba_scan_fwd_noalloc_status(stream=None) -> int:
    return _lib.swimba_scan_fwd_noalloc_status(_stream(stream))


def swimba_scan_fwd_noalloc_status_block() -> int | None:
    return _lib.swimba_scan_fwd_noalloc_status_block()


def swimba_scan_summary(dims, x, delta, B_mix, idx, gates, weights, h_zero, log_decay, ws, ws_bytes,
                        stream=None) -> int:
    return _lib.swimba_scan_summary(ctypes.byref(dims), _ptr(x), _ptr(delta), _ptr(B_mix), _ptr(idx), _ptr(gates),
                                    ctypes.byref(weights), _ptr(h_zero), _ptr(log_decay), _ptr(ws), int(ws_bytes),
                                    _stream(stream))


def swimba_scan_chain(dims, parts, h_zero, log_decay, h0, h_start, stream=None) -> int:
    return _lib.swimba_scan_chain(ctypes.byref(dims), int(parts), _ptr(h_zero), _ptr(log_decay), _ptr(h0),
                                  _ptr(h_start), _stream(stream))


def swimba_scan_bwd(dims, x, z, delta, B_mix, C_mix, idx, gates, weights, h0, g_out, dx, dz, ddelta, dB, dC, dgates,
                    dA, dD, dh0, ws, ws_bytes, stream=None) -> int:
    return _lib.swimba_scan_bwd(ctypes.byref(dims), _ptr(x), _ptr(z), _ptr(delta), _ptr(B_mix), _ptr(C_mix), _ptr(idx),
                                _ptr(gates), ctypes.byref(weights), _ptr(h0), _ptr(g_out), _ptr(dx), _ptr(dz),
                                _ptr(ddelta), _ptr(dB), _ptr(dC), _ptr(dgates), _ptr(dA), _ptr(dD), _ptr(dh0), _ptr(ws),
                                int(ws_bytes), _stream(stream))


def swimba_proj_bwd(dims, x, idx, gates, weights, delta, g_delta, g_B, g_C, dx, dx_accumulate, dgates, dW_x, dW_dt,
                    db_dt, ws, ws_bytes, stream=None) -> int:
    return _lib.swimba_proj_bwd(ctypes.byref(dims), _ptr(x), _ptr(idx), _ptr(gates), ctypes.byref(weights), _ptr(delta),
                                _ptr(g_delta), _ptr(g_B), _ptr(g_C), _ptr(dx), int(dx_accumulate), _ptr(dgates),
                                _ptr(dW_x), _ptr(dW_dt), _ptr(db_dt), _ptr(ws), int(ws_bytes), _stream(stream))


def swimba_route_bwd(dims, x, W_r, idx, gates, g_gates_a, g_gates_b, dx, dx_accumulate, dW_r, ws, ws_bytes,
                     stream=None) -> int:
    return _lib.swimba_route_bwd(ctypes.byref(dims), _ptr(x), _ptr(W_r), _ptr(idx), _ptr(gates), _ptr(g_gates_a),
                                 _ptr(g_gates_b), _ptr(dx), int(dx_accumulate), _ptr(dW_r), _ptr(ws), int(ws_bytes),
                                 _stream(stream))


def swimba_ssd_scan(dims, X, B_j, C_mix, gates, delta, A, D_skip, S0, y, S_final, ws, ws_bytes, stream=None) -> int:
    return _lib.swimba_ssd_scan(ctypes.byref(dims), _ptr(X), _ptr(B_j), _ptr(C_mix), _ptr(gates), _ptr(delta), _ptr(A),
                                _ptr(D_skip), _ptr(S0), _ptr(y), _ptr(S_final), _ptr(ws), int(ws_bytes),
                                _stream(stream))


def swimba_separate_proj(dims, x, idx, gates, weights, delta_j, B_j, C_j, stream=None) -> int:
    return _lib.swimba_separate_proj(ctypes.byref(dims), _ptr(x), _ptr(idx), _ptr(gates), ctypes.byref(weights),
                                     _ptr(delta_j), _ptr(B_j), _ptr(C_j), _stream(stream))


def swimba_separate_scan(dims, x, z, delta_j, B_j, C_j, idx, gates, weights, h0, out, h_final, y_pre, ws, ws_bytes,
                         stream=None) -> int:
    return _lib.swimba_separate_scan(ctypes.byref(dims), _ptr(x), _ptr(z), _ptr(delta_j), _ptr(B_j), _ptr(C_j),
                                     _ptr(idx), _ptr(gates), ctypes.byref(weights), _ptr(h0), _ptr(out),
                                     _ptr(h_final), _ptr(y_pre), _ptr(ws), int(ws_bytes), _stream(stream))


def swimba_step(dims, x, z, delta, B_mix, C_mix, idx, gates, weights, h, out, stream=None) -> int:
    return _lib.swimba_step(ctypes.byref(dims), _ptr(x), _ptr(z), _ptr(delta), _ptr(B_mix), _ptr(C_mix), _ptr(idx),
                            _ptr(gates), ctypes.byref(weights), _ptr(h), _ptr(out), _stream(stream))


def swimba_get_device_status(ws, stream=None) -> int:
    return _lib.swimba_get_device_status(_ptr(ws), _stream(stream))


def swimba_check_wait_timeout(ws, ws_bytes, limit_ns, stream=None) -> int:
    return _lib.swimba_check_wait_timeout(_ptr(ws), ws_bytes, limit_ns, _stream(stream))


def swimba_conv1d_fwd(dims, d_conv, x_pre, conv_w, conv_b, conv_state_in, x, conv_state_out, stream=None) -> int:
    return _lib.swimba_conv1d_fwd(ctypes.byref(dims), int(d_conv), _ptr(x_pre), _ptr(conv_w), _ptr(conv_b),
                                  _ptr(conv_state_in), _ptr(x), _ptr(conv_state_out), _stream(stream))


def swimba_conv1d_step(dims, d_conv, x_pre, conv_w, conv_b, conv_state, x, stream=None) -> int:
    return _lib.swimba_conv1d_step(ctypes.byref(dims), int(d_conv), _ptr(x_pre), _ptr(conv_w), _ptr(conv_b),
                                   _ptr(conv_state), _ptr(x), _stream(stream))


def swimba_block_workspace_size(bdims: swimba_block_dims) -> int:
    return int(_lib.swimba_block_workspace_size(ctypes.byref(bdims)))


def swimba_block_gemm(dtype, M, N, K, A, lda, B, ldb, C0, ldc0, C1, ldc1, split, R, ldr, ws, ws_bytes,
                      stream=None) -> int:
    return _lib.swimba_block_gemm(int(dtype), int(M), int(N), int(K), _ptr(A), int(lda), _ptr(B), int(ldb), _ptr(C0),
                                  int(ldc0), _ptr(C1), int(ldc1), int(split), _ptr(R), int(ldr), _ptr(ws),
                                  int(ws_bytes), _stream(stream))


def swimba_block_fwd(bdims, u, bweights, h0, conv_state_in, out, h_final, conv_state_out, ws, ws_bytes,
                     stream=None) -> int:
    return _lib.swimba_block_fwd(ctypes.byref(bdims), _ptr(u), ctypes.byref(bweights), _ptr(h0), _ptr(conv_state_in),
                                 _ptr(out), _ptr(h_final), _ptr(conv_state_out), _ptr(ws), int(ws_bytes),
                                 _stream(stream))


def swimba_block_step(bdims, u, bweights, h, conv_state, out, ws, ws_bytes, stream=None) -> int:
    return _lib.swimba_block_step(ctypes.byref(bdims), _ptr(u), ctypes.byref(bweights), _ptr(h), _ptr(conv_state),
                                  _ptr(out), _ptr(ws), int(ws_bytes), _stream(stream))


# ------------------------------------------------------------------------------------------------
# marshalling helpers: shapes, host arrays -> device tensors, buffers of one layer call
# ------------------------------------------------------------------------------------------------

def dtype_code(name: str) -> int:
    return {"f32": SWIMBA_F32, "bf16": SWIMBA_BF16}[name]


_dtype_code = dtype_code


def make_dims(cfg, seqlen=None, batch=None, n_experts=None, top_k=None) -> swimba_dims:
    return swimba_dims(
        batch=cfg.batch if batch is None else batch,
        seqlen=cfg.seqlen if seqlen is None else seqlen,
        d_inner=cfg.d_inner,
        d_state=cfg.d_state,
        dt_rank=cfg.dt_rank,
        n_experts=cfg.n_experts if n_experts is None else n_experts,
        top_k=cfg.top_k if top_k is None else top_k,
        io_dtype=_dtype_code(cfg.io_dtype),
        w_dtype=_dtype_code(cfg.w_dtype),
    )


def to_device(stored: np.ndarray, dtype: str, device="cuda", pin=False) -> torch.Tensor:
    """A stored array (uint16 bf16 bits or float32) as a torch tensor of the matching dtype."""
    if dtype == "bf16":
        t = torch.from_numpy(np.ascontiguousarray(stored).view(np.int16)).view(torch.bfloat16)
    else:
        t = torch.from_numpy(np.ascontiguousarray(stored))
    if device == "cpu":
        return t.pin_memory() if pin else t
    return t.to(device, non_blocking=False)


@dataclass
class DeviceWeights:
    W_r: torch.Tensor
    W_x: torch.Tensor
    W_dt: torch.Tensor
    b_dt: torch.Tensor
    A: torch.Tensor
    D_skip: torch.Tensor

    def struct(self) -> swimba_weights:
        return swimba_weights(*(t.data_ptr() for t in (self.W_r, self.W_x, self.W_dt, self.b_dt, self.A, self.D_skip)))


def upload_weights(w, device="cuda") -> DeviceWeights:
    """``w`` is a ``synth.LayerWeights`` (or anything with the same fields)."""
    return DeviceWeights(
        W_r=to_device(w.W_r, "f32", device),
        W_x=to_device(w.W_x, w.w_dtype, device),
        W_dt=to_device(w.W_dt, w.w_dtype, device),
        b_dt=to_device(w.b_dt, "f32", device),
        A=to_device(w.A, "f32", device),
        D_skip=to_device(w.D_skip, "f32", device),
    )


def new_workspace(dims: swimba_dims, op: int = SWIMBA_OP_LAYER, device="cuda") -> torch.Tensor:
    n = swimba_workspace_size(dims, op)
    if n == 0:
        raise SwimbaError(1, "swimba_workspace_size")
    return torch.zeros(n, dtype=torch.uint8, device=device)


class LayerBuffers:
    """The intermediate and output buffers of one layer call for ``dims`` (allocated by torch)."""

    def __init__(self, dims: swimba_dims, io_torch_dtype, device="cuda", with_y=False):
        B, L, D, N, k = dims.batch, dims.seqlen, dims.d_inner, dims.d_state, dims.top_k
        f32 = dict(dtype=torch.float32, device=device)
        self.idx = torch.empty((B, L, k), dtype=torch.int32, device=device)
        self.gates = torch.empty((B, L, k), **f32)
        self.delta = torch.empty((B, L, D), **f32)
        self.B_mix = torch.empty((B, L, N), **f32)
        self.C_mix = torch.empty((B, L, N), **f32)
        self.out = torch.empty((B, L, D), dtype=io_torch_dtype, device=device)
        self.h_final = torch.empty((B, D, N), **f32)
        self.y = torch.empty((B, L, D), **f32) if with_y else None
        self.ws = new_workspace(dims, SWIMBA_OP_LAYER, device)


def layer_forward(dims, x, z, weights: swimba_weights, buf: LayerBuffers, h0=None, stream=None) -> LayerBuffers:
    """route -> mixed_proj -> scan_fwd on one stream (three library calls)."""
    check(swimba_route(dims, x, ctypes.c_void_p(weights.W_r).value, buf.idx, buf.gates, stream), "swimba_route")
    ws_bytes = buf.ws.numel()
    check(swimba_mixed_proj(dims, x, buf.idx, buf.gates, weights, buf.delta, buf.B_mix, buf.C_mix, buf.ws, ws_bytes,
                            stream), "swimba_mixed_proj")
    check(swimba_scan_fwd(dims, x, z, buf.delta, buf.B_mix, buf.C_mix, buf.idx, buf.gates, weights, h0, buf.out,
                          buf.h_final, buf.y, buf.ws, ws_bytes, stream), "swimba_scan_fwd")
    return buf


def decode_step(dims, x, z, weights: swimba_weights, buf: LayerBuffers, h, stream=None) -> LayerBuffers:
    """route -> mixed_proj -> step (seqlen 1), updating the cached state ``h`` in place."""
    check(swimba_route(dims, x, ctypes.c_void_p(weights.W_r).value, buf.idx, buf.gates, stream), "swimba_route")
    ws_bytes = buf.ws.numel()
    check(swimba_mixed_proj(dims, x, buf.idx, buf.gates, weights, buf.delta, buf.B_mix, buf.C_mix, buf.ws, ws_bytes,
                            stream), "swimba_mixed_proj")
    check(swimba_step(dims, x, z, buf.delta, buf.B_mix, buf.C_mix, buf.idx, buf.gates, weights, h, buf.out, stream),
          "swimba_step")
    return buf
