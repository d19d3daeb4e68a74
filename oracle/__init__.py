"""CPU oracle for packed binary/ternary g128 linear layers -- TEST INFRASTRUCTURE ONLY.

Only the test suite, the smoke check and the benchmark's CPU-baseline leg may import
this package. The product (``ternary_g128_weight_bq_b200``) never imports it.

The arithmetic lives in plain C (``bq_oracle.c``, fp64); this module compiles it with
gcc into ``liboracle.so`` and wraps it with ctypes. Arrays go in and out as numpy
arrays; no function here does any of the method's arithmetic itself.
"""

from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "bq_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

BINARY = 0
TERNARY = 1
TERNARY_B3 = 2
X_F16 = 0
X_BF16 = 1
OK = 0
ERR_SHAPE = 1
ERR_CODE = 2

_default = None


def build(force: bool = False, src: str = _SRC, out: str = _LIB) -> str:
    """Compile the oracle C source into a shared library (plain -O2, no fast-math,
    no FMA contraction)."""
    deps = [src, os.path.join(_HERE, "bq_oracle.h")]
    stale = not os.path.exists(out) or os.path.getmtime(out) < max(os.path.getmtime(d) for d in deps)
    if force or stale:
        tmp = out + ".tmp%d" % os.getpid()
        subprocess.run(["gcc", "-std=c11", "-O2", "-fno-fast-math", "-ffp-contract=off",
                        "-shared", "-fPIC", "-Wall", "-I", _HERE, "-o", tmp, src, "-lm"],
                       check=True)
        os.replace(tmp, out)
    return out


def _c(a, dtype):
    a = np.ascontiguousarray(a)
    if a.dtype != dtype:
        raise TypeError(f"expected {np.dtype(dtype)}, got {a.dtype}")
    return a


def _p(a):
    return a.ctypes.data_as(ctypes.c_void_p)


def _bits16(a) -> np.ndarray:
    """fp16/bf16 data as raw uint16 bits (accepts numpy float16/uint16 or torch tensors)."""
    if hasattr(a, "detach"):  # torch tensor: reinterpret the 16-bit payload
        import torch
        t = a.detach().cpu().contiguous()
        if t.dtype in (torch.float16, torch.bfloat16):
            t = t.view(torch.int16)
        return t.numpy().view(np.uint16)
    a = np.ascontiguousarray(a)
    if a.dtype in (np.float16, np.uint16, np.int16):
        return a.view(np.uint16)
    raise TypeError(f"expected 16-bit data, got {a.dtype}")


def _u32(a) -> np.ndarray:
    if hasattr(a, "detach"):
        a = a.detach().cpu().contiguous().numpy()
    a = np.ascontiguousarray(a)
    if a.dtype not in (np.uint32, np.int32):
        raise TypeError(f"expected 32-bit words, got {a.dtype}")
    return a.view(np.uint32)


def _weights(fmt: int, a) -> np.ndarray:
    """Packed weights as the oracle reads them: uint32 words, or bytes for base-3."""
    if fmt != TERNARY_B3:
        return _u32(a)
    if hasattr(a, "detach"):
        a = a.detach().cpu().contiguous().numpy()
    a = np.ascontiguousarray(a)
    if a.dtype not in (np.uint8, np.int8):
        raise TypeError(f"expected bytes, got {a.dtype}")
    return a.view(np.uint8)


def _i8(a) -> np.ndarray:
    if hasattr(a, "detach"):
        a = a.detach().cpu().contiguous().numpy()
    return _c(a, np.int8)


class Oracle:
    """ctypes wrapper around one compiled copy of the oracle."""

    def __init__(self, path: str = None):
        if path is None:
            path = build()
        L = ctypes.CDLL(path)
        P = ctypes.c_void_p
        I64 = ctypes.c_int64
        L.bqo_f16_to_f64.argtypes = [ctypes.c_uint16]
        L.bqo_f16_to_f64.restype = ctypes.c_double
        L.bqo_bf16_to_f64.argtypes = [ctypes.c_uint16]
        L.bqo_bf16_to_f64.restype = ctypes.c_double
        L.bqo_f64_to_bf16.argtypes = [ctypes.c_double]
        L.bqo_f64_to_bf16.restype = ctypes.c_uint16
        L.bqo_f64_to_bf16_array.argtypes = [P, I64, P]
        L.bqo_f64_to_bf16_array.restype = None
        L.bqo_f64_to_f16.argtypes = [ctypes.c_double]
        L.bqo_f64_to_f16.restype = ctypes.c_uint16
        L.bqo_words_per_row.argtypes = [ctypes.c_int, I64]
        L.bqo_words_per_row.restype = I64
        L.bqo_row_bytes.argtypes = [ctypes.c_int, I64]
        L.bqo_row_bytes.restype = I64
        for f in (L.bqo_pack_binary_g128, L.bqo_pack_ternary_g128, L.bqo_pack_ternary_b3):
            f.argtypes = [P, P, I64, I64, P, P]
            f.restype = ctypes.c_int
        for f in (L.bqo_unpack_binary_g128, L.bqo_unpack_ternary_g128, L.bqo_unpack_ternary_b3):
            f.argtypes = [P, I64, I64, P]
            f.restype = I64
        L.bqo_weight.argtypes = [ctypes.c_int, P, P, I64, I64, I64]
        L.bqo_weight.restype = ctypes.c_double
        L.bqo_dequant.argtypes = [ctypes.c_int, P, P, I64, I64, P]
        L.bqo_dequant.restype = ctypes.c_int
        L.bqo_gemv_rows.argtypes = [ctypes.c_int, P, ctypes.c_int, I64, I64, P, P, I64, P, I64, P, P]
        L.bqo_gemv_rows.restype = ctypes.c_int
        L.bqo_embed.argtypes = [ctypes.c_int, P, I64, P, P, I64, I64, P]
        L.bqo_embed.restype = I64
        L.bqo_mlp_swiglu.argtypes = [ctypes.c_int, P, ctypes.c_int, I64, I64, P, P, P, P, I64, ctypes.c_int,
                                     P, P, I64, P, P, P]
        L.bqo_mlp_swiglu.restype = ctypes.c_int
        L.bqo_quantize_g128.argtypes = [ctypes.c_int, P, I64, I64, P, P]
        L.bqo_quantize_g128.restype = ctypes.c_int
        L.bqo_topk.argtypes = [P, I64, I64, ctypes.c_int, P, P]
        L.bqo_topk.restype = ctypes.c_int
        L.bqo_sample_topk.argtypes = [P, P, ctypes.c_int, ctypes.c_double, ctypes.c_double, ctypes.c_double]
        L.bqo_sample_topk.restype = I64
        L.bqo_mlx_affine_dequant.argtypes = [ctypes.c_uint16, ctypes.c_int]
        L.bqo_mlx_affine_dequant.restype = ctypes.c_uint16
        self.L = L
        self.path = path

    def words_per_row(self, fmt: int, K: int) -> int:
        return int(self.L.bqo_words_per_row(fmt, K))

    def row_bytes(self, fmt: int, K: int) -> int:
        return int(self.L.bqo_row_bytes(fmt, K))

    def pack(self, fmt: int, q, s):
        """(q int8[N,K], s fp16[N,K/128]) -> (status, packed, s_out uint16); packed is
        uint32[N, W] for the binary and 2-bit formats and uint8[N, 26 K/128] for base-3."""
        q = _i8(q)
        s = _bits16(s)
        N, K = q.shape
        RB = self.row_bytes(fmt, K)
        if RB < 0:
            return ERR_SHAPE, None, None
        if fmt == TERNARY_B3:
            words = np.zeros((N, RB), dtype=np.uint8)
        else:
            words = np.zeros((N, RB // 4), dtype=np.uint32)
        s_out = np.zeros((N, K // 128), dtype=np.uint16)
        f = {BINARY: self.L.bqo_pack_binary_g128, TERNARY: self.L.bqo_pack_ternary_g128,
             TERNARY_B3: self.L.bqo_pack_ternary_b3}[fmt]
        st = f(_p(q), _p(s), N, K, _p(words), _p(s_out))
        return st, words, s_out

    def unpack(self, fmt: int, words, K: int):
        """packed[N, ...] -> (q int8[N, K], number of invalid codes or bytes)."""
        w = _weights(fmt, words)
        N = w.shape[0]
        q = np.zeros((N, K), dtype=np.int8)
        f = {BINARY: self.L.bqo_unpack_binary_g128, TERNARY: self.L.bqo_unpack_ternary_g128,
             TERNARY_B3: self.L.bqo_unpack_ternary_b3}[fmt]
        bad = f(_p(w), N, K, _p(q))
        return q, int(bad)

    def dequant(self, fmt: int, words, scales, K: int) -> np.ndarray:
        w = _weights(fmt, words)
        s = _bits16(scales)
        N = w.shape[0]
        out = np.zeros((N, K), dtype=np.float64)
        st = self.L.bqo_dequant(fmt, _p(w), _p(s), N, K, _p(out))
        if st != OK:
            raise ValueError(f"dequant status {st}")
        return out

    def gemv(self, fmt: int, x, xt: int, words, scales, K: int, rows=None):
        """y[M, R] and bound[M, R] in fp64 for the selected rows (all rows by default)."""
        xb = _bits16(x)
        M = xb.shape[0]
        w = _weights(fmt, words)
        s = _bits16(scales)
        N = w.shape[0]
        r = (np.arange(N, dtype=np.int64) if rows is None
             else np.ascontiguousarray(rows, dtype=np.int64))
        y = np.zeros((M, len(r)), dtype=np.float64)
        b = np.zeros((M, len(r)), dtype=np.float64)
        st = self.L.bqo_gemv_rows(fmt, _p(xb), xt, M, K, _p(w), _p(s), N, _p(r), len(r),
                                  _p(y), _p(b))
        if st != OK:
            raise ValueError(f"gemv status {st}")
        return y, b

    def embed(self, fmt: int, ids, words, scales, K: int):
        """(out fp64[T, K], number of out-of-range ids)."""
        i = np.ascontiguousarray(ids.numpy() if hasattr(ids, "numpy") else ids, dtype=np.int32)
        w = _weights(fmt, words)
        s = _bits16(scales)
        out = np.zeros((len(i), K), dtype=np.float64)
        bad = self.L.bqo_embed(fmt, _p(i), len(i), _p(w), _p(s), w.shape[0], K, _p(out))
        return out, int(bad)

    def mlp_swiglu(self, x, xt: int, fmt_gu: int, gate, up, fmt_d: int, down):
        """(a [M, F], y [M, N], bound [M, N]) in fp64 for gate/up/down = (packed, scales) pairs,
        gate and up [F, K], down [N, F]."""
        xb = _bits16(x)
        M, K = xb.shape
        wg, sg = _weights(fmt_gu, gate[0]), _bits16(gate[1])
        wu, su = _weights(fmt_gu, up[0]), _bits16(up[1])
        wd, sd = _weights(fmt_d, down[0]), _bits16(down[1])
        F, N = wg.shape[0], wd.shape[0]
        a = np.zeros((M, F), dtype=np.float64)
        y = np.zeros((M, N), dtype=np.float64)
        b = np.zeros((M, N), dtype=np.float64)
        st = self.L.bqo_mlp_swiglu(fmt_gu, _p(xb), xt, M, K, _p(wg), _p(sg), _p(wu), _p(su), F, fmt_d,
                                   _p(wd), _p(sd), N, _p(a), _p(y), _p(b))
        if st != OK:
            raise ValueError(f"mlp status {st}")
        return a, y, b

    def quantize(self, fmt: int, w):
        """Dense fp32 w [N, K] -> (q int8 [N, K], s fp16 bits uint16 [N, K/128]): the
        least-squares binary or ternary fit of every group of 128."""
        if hasattr(w, "detach"):
            w = w.detach().cpu().float().numpy()
        w = np.ascontiguousarray(w, dtype=np.float32)
        N, K = w.shape
        q = np.zeros((N, K), dtype=np.int8)
        s = np.zeros((N, K // 128), dtype=np.uint16)
        st = self.L.bqo_quantize_g128(fmt, _p(w), N, K, _p(q), _p(s))
        if st != OK:
            raise ValueError(f"quantize status {st}")
        return q, s

    def topk(self, y, k: int):
        """(idx int64[M, k], vals fp64[M, k]): the k largest of each row of y (fp64 [M, N]),
        descending, equal values in ascending index order."""
        y = np.ascontiguousarray(y, dtype=np.float64)
        M, N = y.shape
        idx = np.zeros((M, k), dtype=np.int64)
        vals = np.zeros((M, k), dtype=np.float64)
        st = self.L.bqo_topk(_p(y), M, N, k, _p(idx), _p(vals))
        if st != OK:
            raise ValueError(f"topk status {st}")
        return idx, vals

    def sample_topk(self, vals, idx, T: float, top_p: float, u: float) -> int:
        """Token drawn from one row of top-k candidates (vals descending) with temperature T,
        top-p and the uniform number u."""
        v = np.ascontiguousarray(vals, dtype=np.float64)
        i = np.ascontiguousarray(idx, dtype=np.int64)
        return int(self.L.bqo_sample_topk(_p(v), _p(i), len(v), T, top_p, u))

    def to_bf16_bits(self, v) -> np.ndarray:
        """Round fp64 values to bfloat16 (ties to even); returns uint16 bits."""
        v = np.ascontiguousarray(v, dtype=np.float64)
        out = np.zeros(v.shape, dtype=np.uint16)
        self.L.bqo_f64_to_bf16_array(_p(v), v.size, _p(out))
        return out

    def to_f16_bits(self, v) -> np.ndarray:
        v = np.ascontiguousarray(v, dtype=np.float64)
        return np.array([self.L.bqo_f64_to_f16(float(a)) for a in v.ravel()],
                        dtype=np.uint16).reshape(v.shape)

    def f16_value(self, bits: int) -> float:
        return float(self.L.bqo_f16_to_f64(bits))

    def bf16_value(self, bits: int) -> float:
        return float(self.L.bqo_bf16_to_f64(bits))

    def mlx_affine_dequant(self, s_bits: int, q01: int) -> int:
        return int(self.L.bqo_mlx_affine_dequant(s_bits, q01))


def default() -> Oracle:
    """The oracle compiled from this directory's source (built on first use)."""
    global _default
    if _default is None:
        _default = Oracle()
    return _default
