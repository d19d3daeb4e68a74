"""Python binding of libbq: linear layers on packed binary-g128 / ternary-g128 weights for
NVIDIA B200 (sm_100a).

This module only marshals arguments: it passes device pointers of torch tensors and the
current CUDA stream to the C ABI declared in ``include/bq.h``. Every step of the
computation runs in libbq's CUDA kernels. If the compiled library is missing the import
fails loudly; there is no fallback.

Build the library with ``python -m ternary_g128_weight_bq_b200.build``.
"""

from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libbq.so")

BINARY_G128 = 0
TERNARY_G128 = 1
TERNARY_B3_G128 = 2      # ternary codes in base-3 bytes (26 per group of 128): 1.75 bits/weight

_DTYPE = {torch.float16: 0, torch.bfloat16: 1, torch.float32: 2}

STATUS = {
    0: "BQ_OK", 1: "BQ_ERR_INVALID_ARG", 2: "BQ_ERR_SHAPE", 3: "BQ_ERR_ALIGNMENT",
    4: "BQ_ERR_DTYPE", 5: "BQ_ERR_INVALID_CODE", 6: "BQ_ERR_CUDA", 7: "BQ_ERR_TIMEOUT",
    8: "BQ_ERR_UNSUPPORTED", 9: "BQ_ERR_WORKSPACE",
}


class BQError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS.get(status, status)}: {message}")
        self.status = status
        self.status_name = STATUS.get(status, str(status))


class _Weight(ctypes.Structure):
    _fields_ = [("fmt", ctypes.c_int), ("N", ctypes.c_int64), ("K", ctypes.c_int64),
                ("words", ctypes.c_void_p), ("scales", ctypes.c_void_p)]


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded libbq (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"libbq.so not found at {LIB_PATH}; build it with "
                              "`python -m ternary_g128_weight_bq_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P, I64, I = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
        W = ctypes.POINTER(_Weight)
        sig = {
            "bq_version": ([], ctypes.c_char_p),
            "bq_status_string": ([I], ctypes.c_char_p),
            "bq_last_error": ([], ctypes.c_char_p),
            "bq_kernel_launches": ([], ctypes.c_ulonglong),
            "bq_packed_words": ([I, I64, I64], ctypes.c_size_t),
            "bq_packed_bytes": ([I, I64, I64], ctypes.c_size_t),
            "bq_pack_binary_g128": ([P, P, I64, I64, P, P, P], I),
            "bq_pack_ternary_g128": ([P, P, I64, I64, P, P, P], I),
            "bq_pack_ternary_b3_g128": ([P, P, I64, I64, P, P, P], I),
            "bq_quantize_g128": ([P, I, I64, I64, I, P, P, P], I),
            "bq_unpack_g128": ([W, P, P, P], I),
            "bq_gemv": ([P, I, I64, W, P, I, P, ctypes.c_size_t, P], I),
            "bq_gemv_workspace_bytes": ([I64, W], ctypes.c_size_t),
            "bq_gemv_noalloc": ([P, I, I64, W, P, I, P], I),
            "bq_gemv_topk": ([P, I, I64, W, I, P, P, P, ctypes.c_float, ctypes.c_float, P, P, ctypes.c_size_t, P], I),
            "bq_gemv_topk_workspace_bytes": ([I64, W, I], ctypes.c_size_t),
            "bq_mlp_swiglu": ([P, I, I64, W, W, W, P, I, P, ctypes.c_size_t, P], I),
            "bq_mlp_swiglu_workspace_bytes": ([I64, W, W, W], ctypes.c_size_t),
            "bq_gemm_prefill": ([P, I, I64, W, P, I, P, ctypes.c_size_t, P], I),
            "bq_gemm_prefill_workspace_bytes": ([I64, W], ctypes.c_size_t),
            "bq_embed_gather": ([P, I64, W, P, I, P], I),
            "bq_get_device_error": ([P], I),
            "bq_debug_set_wait_limit_ns": ([ctypes.c_uint64], None),
            "bq_debug_fail_next_launches": ([I], None),
        }
        for name, (args, res) in sig.items():
            f = getattr(L, name)
            f.argtypes = args
            f.restype = res
        _lib = L
    return _lib


def _check(status: int):
    if status != 0:
        raise BQError(status, lib().bq_last_error().decode())


def _stream(device=None) -> int:
    return torch.cuda.current_stream(device).cuda_stream


def _dev(t: torch.Tensor, name: str):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _same_device(name: str, t: torch.Tensor, ref: torch.Tensor):
    if t.device != ref.device:
        raise ValueError(f"{name} is on {t.device}, expected {ref.device}")


def _out(out, shape, dtype, x: torch.Tensor, w) -> torch.Tensor:
    """The caller's output tensor, checked (shape, dtype, device), or a new one."""
    if out is None:
        return torch.empty(shape, dtype=dtype, device=x.device)
    _dev(out, "out")
    if tuple(out.shape) != tuple(shape):
        raise ValueError(f"out must have shape {tuple(shape)}, got {tuple(out.shape)}")
    if out.dtype not in _DTYPE:
        raise ValueError(f"out dtype {out.dtype} is not supported")
    _same_device("out", out, x)
    return out


def _operands(x: torch.Tensor, w) -> None:
    _dev(x, "x")
    if x.dim() != 2 or x.shape[1] != w.K:
        raise ValueError(f"x must be [M, {w.K}]")
    if x.dtype not in _DTYPE:
        raise ValueError(f"x dtype {x.dtype} is not supported")
    _same_device("weight words", w.words, x)
    _same_device("weight scales", w.scales, x)


@dataclass
class BQWeight:
    """A packed weight matrix held in device memory.

    words: int32 [N, K/32] (binary) or [N, K/16] (ternary), the uint32 bit patterns, or
        uint8 [N, 26 K/128] (ternary in base-3 bytes).
    scales: float16 [N, K/128].
    """
    fmt: int
    N: int
    K: int
    words: torch.Tensor
    scales: torch.Tensor

    def __post_init__(self):
        _dev(self.words, "words")
        _dev(self.scales, "scales")
        shape, dtype = _packed_shape(self.fmt, self.N, self.K)
        if tuple(self.words.shape) != shape or self.words.dtype != dtype:
            raise ValueError(f"words must be {dtype} {list(shape)}")
        if tuple(self.scales.shape) != (self.N, self.K // 128) or self.scales.dtype != torch.float16:
            raise ValueError(f"scales must be float16 [{self.N}, {self.K // 128}]")
        self._c = _Weight(self.fmt, self.N, self.K, self.words.data_ptr(), self.scales.data_ptr())

    @property
    def c(self):
        return ctypes.byref(self._c)

    @property
    def nbytes(self) -> int:
        return self.words.numel() * self.words.element_size() + self.scales.numel() * 2


def _packed_shape(fmt: int, N: int, K: int):
    """Shape and dtype of the packed-weight tensor of a format."""
    if fmt == TERNARY_B3_G128:
        return (N, 26 * (K // 128)), torch.uint8
    if fmt in (BINARY_G128, TERNARY_G128):
        return (N, K // (32 if fmt == BINARY_G128 else 16)), torch.int32
    raise ValueError(f"unknown format {fmt}")


def version() -> str:
    return lib().bq_version().decode()


def kernel_launches() -> int:
    """Kernel launches enqueued through libbq so far in this process."""
    return int(lib().bq_kernel_launches())


def packed_words(fmt: int, N: int, K: int) -> int:
    return int(lib().bq_packed_words(fmt, N, K))


def packed_bytes(fmt: int, N: int, K: int) -> int:
    return int(lib().bq_packed_bytes(fmt, N, K))


def _pack(fn, fmt, q, s):
    _dev(q, "q")
    _dev(s, "s")
    if q.dtype != torch.int8 or q.dim() != 2:
        raise ValueError("q must be int8 [N, K]")
    N, K = q.shape
    if s.dtype != torch.float16:
        raise ValueError("s must be float16 [N, K/128]")
    shape, dtype = _packed_shape(fmt, N, max(K, 128))
    words = torch.empty(shape, dtype=dtype, device=q.device)
    s_out = torch.empty((N, max(K // 128, 1)), dtype=torch.float16, device=q.device)
    _check(fn(q.data_ptr(), s.data_ptr(), N, K, words.data_ptr(), s_out.data_ptr(),
              _stream(q.device)))
    return BQWeight(fmt, N, K, words, s_out)


def pack_binary_g128(q: torch.Tensor, s: torch.Tensor) -> BQWeight:
    """Pack int8 q in {-1, +1} [N, K] and fp16 scales [N, K/128] (synchronous; validates q)."""
    return _pack(lib().bq_pack_binary_g128, BINARY_G128, q, s)


def pack_ternary_g128(q: torch.Tensor, s: torch.Tensor) -> BQWeight:
    """Pack int8 q in {-1, 0, +1} [N, K] and fp16 scales (synchronous; validates q)."""
    return _pack(lib().bq_pack_ternary_g128, TERNARY_G128, q, s)


def pack_ternary_b3_g128(q: torch.Tensor, s: torch.Tensor) -> BQWeight:
    """Pack int8 q in {-1, 0, +1} [N, K] into base-3 bytes (26 per group of 128) and fp16
    scales (synchronous; validates q)."""
    return _pack(lib().bq_pack_ternary_b3_g128, TERNARY_B3_G128, q, s)


def quantize_g128(w: torch.Tensor, fmt: int) -> BQWeight:
    """Dense weights [N, K] (fp32, bf16 or fp16) to a packed matrix of format fmt: the
    least-squares fit of every group of 128 (asynchronous on the current stream)."""
    _dev(w, "w")
    if w.dim() != 2 or w.dtype not in _DTYPE:
        raise ValueError("w must be a 2-D fp32, bf16 or fp16 tensor")
    N, K = w.shape
    shape, dtype = _packed_shape(fmt, N, max(K, 128))
    packed = torch.empty(shape, dtype=dtype, device=w.device)
    scales = torch.empty((N, max(K // 128, 1)), dtype=torch.float16, device=w.device)
    with torch.cuda.device(w.device):
        _check(lib().bq_quantize_g128(w.data_ptr(), _DTYPE[w.dtype], N, K, fmt, packed.data_ptr(),
                                      scales.data_ptr(), _stream(w.device)))
    return BQWeight(fmt, N, K, packed, scales)


def unpack_g128(w: BQWeight):
    """(q int8 [N, K], scales fp16 [N, K/128]) of a packed matrix (synchronous)."""
    q = torch.empty((w.N, w.K), dtype=torch.int8, device=w.words.device)
    s = torch.empty_like(w.scales)
    _check(lib().bq_unpack_g128(w.c, q.data_ptr(), s.data_ptr(), _stream(q.device)))
    return q, s


def gemv_workspace_bytes(M: int, w: BQWeight) -> int:
    return int(lib().bq_gemv_workspace_bytes(M, w.c))


def gemv(x: torch.Tensor, w: BQWeight, out_dtype=torch.float32, out: torch.Tensor = None,
         workspace: torch.Tensor = None) -> torch.Tensor:
    """Decode GEMV: y[M, N] = x[M, K] @ W^T for M <= 8 (fp32 accumulation)."""
    _operands(x, w)
    M = x.shape[0]
    out = _out(out, (M, w.N), out_dtype, x, w)
    need = gemv_workspace_bytes(M, w)
    if workspace is not None:
        _dev(workspace, "workspace")
        _same_device("workspace", workspace, x)
    if need and (workspace is None or workspace.numel() * workspace.element_size() < need):
        workspace = torch.empty(need, dtype=torch.uint8, device=x.device)
    ws_ptr = workspace.data_ptr() if workspace is not None else None
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    with torch.cuda.device(x.device):
        _check(lib().bq_gemv(x.data_ptr(), _DTYPE[x.dtype], M, w.c, out.data_ptr(), _DTYPE[out.dtype],
                             ws_ptr, ws_bytes, _stream(x.device)))
    return out


def gemv_noalloc(x: torch.Tensor, w: BQWeight, out_dtype=torch.float32,
                 out: torch.Tensor = None) -> torch.Tensor:
    """gemv with the library's fixed scratch array instead of a workspace (no device
    allocation inside the call; calls on one device must not overlap)."""
    _operands(x, w)
    M = x.shape[0]
    out = _out(out, (M, w.N), out_dtype, x, w)
    with torch.cuda.device(x.device):
        _check(lib().bq_gemv_noalloc(x.data_ptr(), _DTYPE[x.dtype], M, w.c, out.data_ptr(),
                                     _DTYPE[out.dtype], _stream(x.device)))
    return out


def gemv_topk_workspace_bytes(M: int, w: BQWeight, k: int) -> int:
    return int(lib().bq_gemv_topk_workspace_bytes(M, w.c, k))


def gemv_topk(x: torch.Tensor, w: BQWeight, k: int = 20, u: torch.Tensor = None, temperature: float = 0.7,
              top_p: float = 0.95, workspace: torch.Tensor = None, out=None):
    """The k largest outputs of x @ W^T per token row, without writing the outputs:
    (vals fp32 [M, k] descending, idx int32 [M, k]). With u (fp32 [M] uniform numbers in [0, 1))
    also the token drawn from them with temperature and top-p: (vals, idx, tokens int32 [M]).
    out: optional (vals, idx[, tokens]) tensors to fill."""
    _operands(x, w)
    M = x.shape[0]
    if out is None:
        vals = torch.empty((M, k), dtype=torch.float32, device=x.device)
        idx = torch.empty((M, k), dtype=torch.int32, device=x.device)
        tokens = torch.empty((M,), dtype=torch.int32, device=x.device) if u is not None else None
    else:
        vals, idx = out[0], out[1]
        tokens = out[2] if u is not None else None
    for name, t, dt, shape in (("vals", vals, torch.float32, (M, k)), ("idx", idx, torch.int32, (M, k))):
        _dev(t, name)
        _same_device(name, t, x)
        if t.dtype != dt or tuple(t.shape) != shape:
            raise ValueError(f"{name} must be {dt} {list(shape)}")
    if u is not None:
        _dev(u, "u")
        _same_device("u", u, x)
        if u.dtype != torch.float32 or tuple(u.shape) != (M,):
            raise ValueError(f"u must be float32 [{M}]")
        _dev(tokens, "tokens")
        if tokens.dtype != torch.int32 or tuple(tokens.shape) != (M,):
            raise ValueError(f"tokens must be int32 [{M}]")
    need = gemv_topk_workspace_bytes(M, w, k)
    if workspace is None or workspace.numel() * workspace.element_size() < need:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=x.device)
    else:
        _dev(workspace, "workspace")
        _same_device("workspace", workspace, x)
    with torch.cuda.device(x.device):
        _check(lib().bq_gemv_topk(x.data_ptr(), _DTYPE[x.dtype], M, w.c, k, vals.data_ptr(), idx.data_ptr(),
                                  u.data_ptr() if u is not None else None, temperature, top_p,
                                  tokens.data_ptr() if tokens is not None else None, workspace.data_ptr(),
                                  workspace.numel() * workspace.element_size(), _stream(x.device)))
    return (vals, idx) if u is None else (vals, idx, tokens)


def mlp_swiglu_workspace_bytes(M: int, gate: BQWeight, up: BQWeight, down: BQWeight) -> int:
    return int(lib().bq_mlp_swiglu_workspace_bytes(M, gate.c, up.c, down.c))


def mlp_swiglu(x: torch.Tensor, gate: BQWeight, up: BQWeight, down: BQWeight, out_dtype=torch.float32,
               out: torch.Tensor = None, workspace: torch.Tensor = None) -> torch.Tensor:
    """y = (silu(x @ Wg^T) * (x @ Wu^T)) @ Wd^T for M <= 8 token rows (the gate/up GEMV writes the
    SwiGLU activations, the down GEMV reads them)."""
    _operands(x, gate)
    for name, w in (("up", up), ("down", down)):
        _same_device(f"{name} words", w.words, x)
    M = x.shape[0]
    out = _out(out, (M, down.N), out_dtype, x, down)
    need = mlp_swiglu_workspace_bytes(M, gate, up, down)
    if workspace is None or workspace.numel() * workspace.element_size() < need:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=x.device)
    with torch.cuda.device(x.device):
        _check(lib().bq_mlp_swiglu(x.data_ptr(), _DTYPE[x.dtype], M, gate.c, up.c, down.c, out.data_ptr(),
                                   _DTYPE[out.dtype], workspace.data_ptr(),
                                   workspace.numel() * workspace.element_size(), _stream(x.device)))
    return out


def prefill_workspace_bytes(M: int, w: BQWeight) -> int:
    return int(lib().bq_gemm_prefill_workspace_bytes(M, w.c))


def gemm_prefill(x: torch.Tensor, w: BQWeight, out_dtype=torch.float32,
                 out: torch.Tensor = None, workspace: torch.Tensor = None) -> torch.Tensor:
    """Prefill GEMM: Y[M, N] = X[M, K] @ W^T on the tensor cores (fp32 accumulation)."""
    _operands(x, w)
    M = x.shape[0]
    out = _out(out, (M, w.N), out_dtype, x, w)
    need = prefill_workspace_bytes(M, w)
    if workspace is not None:
        _dev(workspace, "workspace")
        _same_device("workspace", workspace, x)
    if need and (workspace is None or workspace.numel() * workspace.element_size() < need):
        workspace = torch.empty(need, dtype=torch.uint8, device=x.device)
    ws_ptr = workspace.data_ptr() if workspace is not None else None
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    with torch.cuda.device(x.device):
        _check(lib().bq_gemm_prefill(x.data_ptr(), _DTYPE[x.dtype], M, w.c, out.data_ptr(),
                                     _DTYPE[out.dtype], ws_ptr, ws_bytes, _stream(x.device)))
    return out


def embed_gather(ids: torch.Tensor, w: BQWeight, out_dtype=torch.bfloat16,
                 out: torch.Tensor = None) -> torch.Tensor:
    """Embedding lookup: out[t, :] = dequantised row ids[t] of w."""
    _dev(ids, "ids")
    if ids.dtype != torch.int32 or ids.dim() != 1:
        raise ValueError("ids must be int32 [T]")
    T = ids.shape[0]
    _same_device("weight words", w.words, ids)
    _same_device("weight scales", w.scales, ids)
    out = _out(out, (T, w.K), out_dtype, ids, w)
    with torch.cuda.device(ids.device):
        _check(lib().bq_embed_gather(ids.data_ptr(), T, w.c, out.data_ptr(), _DTYPE[out.dtype],
                                     _stream(ids.device)))
    return out


def get_device_error():
    """Synchronise the current stream and raise BQError if a device-side condition was
    recorded (an out-of-range embedding id, a bounded wait that gave up)."""
    _check(lib().bq_get_device_error(_stream()))


def debug_set_wait_limit_ns(ns: int):
    """Test hook: the kernels' pipeline waits give up after `ns` ns (0: the built-in 2 s); a
    wait that gives up is reported by get_device_error() as BQ_ERR_TIMEOUT."""
    lib().bq_debug_set_wait_limit_ns(int(ns))


def debug_fail_next_launches(count: int):
    """Test hook: the next `count` compute calls fail with BQ_ERR_CUDA before launching."""
    lib().bq_debug_fail_next_launches(int(count))
