"""The C-ABI library builds, loads and exports every symbol include/bq.h declares; host-side
validation rejects bad arguments before any CUDA call (runs without a GPU)."""

import ctypes
import os
import re
import subprocess
import sys

import pytest

import ternary_g128_weight_bq_b200 as bq
from ternary_g128_weight_bq_b200 import build as bqbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def libbq():
    bqbuild.build()
    return bq.lib()


def declared_functions():
    text = open(os.path.join(ROOT, "include", "bq.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(bq_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for must in ("bq_pack_binary_g128", "bq_pack_ternary_g128", "bq_unpack_g128", "bq_gemv",
                 "bq_gemm_prefill", "bq_embed_gather", "bq_get_device_error"):
        assert must in names


def test_every_declared_symbol_is_exported(libbq):
    out = subprocess.run(["nm", "-D", "--defined-only", bq.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    missing = [n for n in declared_functions() if n not in exported]
    assert not missing, f"declared but not exported: {missing}"
    for n in declared_functions():
        assert getattr(libbq, n) is not None


def test_header_compiles_as_plain_c(tmp_path):
    src = tmp_path / "use.c"
    src.write_text('#include "bq.h"\nint main(void){ return (int)bq_packed_words(BQ_BINARY_G128, 1, 128); }\n')
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-c", "-I", os.path.join(ROOT, "include"),
                    "-I", "/usr/local/cuda/include", str(src), "-o", str(tmp_path / "use.o")],
                   check=True)


def test_sizes_and_strings(libbq):
    assert libbq.bq_packed_words(0, 3, 256) == 3 * 8
    assert libbq.bq_packed_words(1, 3, 256) == 3 * 16
    assert libbq.bq_packed_words(0, 3, 100) == 0
    assert libbq.bq_packed_words(7, 3, 128) == 0
    assert libbq.bq_status_string(5) == b"BQ_ERR_INVALID_CODE"
    assert b"sm_100a" in libbq.bq_version()


def _weight(fmt=0, N=4, K=256, words=16, scales=16):
    return bq._Weight(fmt, N, K, words, scales)


def test_validation_before_any_cuda_call(libbq):
    """Every one of these fails in host validation, before the library touches CUDA."""
    W = ctypes.byref
    # NULL weight view / NULL pointers
    assert libbq.bq_gemv(16, 1, 1, None, 16, 2, None, 0, None) == 1
    assert libbq.bq_gemv(16, 1, 1, W(_weight(words=0)), 16, 2, None, 0, None) == 1
    # K not a multiple of 128, N < 1
    assert libbq.bq_gemv(16, 1, 1, W(_weight(K=100)), 16, 2, None, 0, None) == 2
    assert libbq.bq_gemv(16, 1, 1, W(_weight(N=0)), 16, 2, None, 0, None) == 2
    # unknown format
    assert libbq.bq_gemv(16, 1, 1, W(_weight(fmt=3)), 16, 2, None, 0, None) == 1
    # misaligned words / x
    assert libbq.bq_gemv(16, 1, 1, W(_weight(words=20)), 16, 2, None, 0, None) == 3
    assert libbq.bq_gemv(18, 1, 1, W(_weight()), 16, 2, None, 0, None) == 3
    # dtypes (fp32 x is accepted by the GEMV, not by the prefill)
    assert libbq.bq_gemv(16, 5, 1, W(_weight()), 16, 2, None, 0, None) == 4
    assert libbq.bq_gemm_prefill(16, 2, 1, W(_weight()), 16, 2, None, 0, None) == 4
    assert libbq.bq_gemv(16, 1, 1, W(_weight()), 16, 9, None, 0, None) == 4
    # M range
    assert libbq.bq_gemv(16, 1, 0, W(_weight()), 16, 2, None, 0, None) == 2
    assert libbq.bq_gemv(16, 1, 9, W(_weight()), 16, 2, None, 0, None) == 2
    assert libbq.bq_gemm_prefill(16, 1, 0, W(_weight()), 16, 2, None, 0, None) == 2
    # pack: NULLs, shapes, alignment
    assert libbq.bq_pack_binary_g128(None, 16, 1, 128, 16, 16, None) == 1
    assert libbq.bq_pack_ternary_g128(16, 16, 1, 96, 16, 16, None) == 2
    assert libbq.bq_pack_binary_g128(17, 16, 1, 128, 16, 16, None) == 3
    # embed: dtype and NULL ids
    assert libbq.bq_embed_gather(None, 4, W(_weight()), 16, 1, None) == 1
    assert libbq.bq_embed_gather(16, 4, W(_weight()), 16, 7, None) == 4
    assert libbq.bq_embed_gather(16, 4, W(_weight()), 24, 1, None) == 3
    assert libbq.bq_embed_gather(16, -1, W(_weight()), 16, 1, None) == 2
    msg = libbq.bq_last_error()
    assert b"T=-1" in msg


def test_size_queries_reject_out_of_range_views(libbq):
    """The size queries apply the calls' limits (format, 1 <= N <= 2^31, 128 <= K <= 2^24, K a
    multiple of 128) and return 0 outside them, instead of planning for the shape (a view of
    N = 2^50, K = 2^40 once reached the planner and divided by zero)."""
    W = ctypes.byref
    huge = _weight(N=1 << 50, K=1 << 40)
    for w in (huge, _weight(fmt=3), _weight(N=(1 << 31) + 1), _weight(K=(1 << 24) + 128), _weight(K=100)):
        assert libbq.bq_gemv_workspace_bytes(1, W(w)) == 0
        assert libbq.bq_gemv_topk_workspace_bytes(1, W(w), 20) == 0
        assert libbq.bq_mlp_swiglu_workspace_bytes(1, W(w), W(w), W(w)) == 0
        assert libbq.bq_gemm_prefill_workspace_bytes(512, W(w)) == 0
        assert libbq.bq_packed_words(w.fmt, w.N, w.K) == 0
    ok = _weight(N=20480, K=5120)
    assert libbq.bq_gemv_workspace_bytes(1, W(ok)) > 0
    assert libbq.bq_gemm_prefill_workspace_bytes(1 << 25, W(ok)) == 0
    assert libbq.bq_packed_words(0, 1 << 31, 1 << 24) == (1 << 31) * (1 << 19)


def _symbol_size(name: str) -> int:
    out = subprocess.run(["nm", "-S", "-C", bq.LIB_PATH], capture_output=True, text=True,
                         check=True).stdout
    for line in out.splitlines():
        parts = line.split()
        if len(parts) >= 4 and parts[-1] == name:
            return int(parts[1], 16)
    raise AssertionError(f"{name} not found")


def test_noalloc_array_covers_every_supported_shape(libbq):
    """bq_gemv_noalloc serves a shape from the library's fixed array only when the workspace
    bq_gemv would need fits in it. That array must hold every shape the GEMV kernels take on a
    148-SM B200 (without a GPU the library plans for 148 SMs): every M, all three formats, K up
    to 64K, N up to 2^22. The array's size is read from the library's symbol table."""
    cap = _symbol_size("bq::g_gemv_scratch")
    assert 64 << 10 <= cap <= 4 << 20
    worst = 0
    for fmt in (bq.BINARY_G128, bq.TERNARY_G128, bq.TERNARY_B3_G128):
        for M in range(1, 9):
            for K in (128, 1024, 2048, 4096, 5120, 6144, 8192, 16384, 20480, 65536):
                for N in (1, 129, 5120, 20480, 248320, 1 << 22):
                    w = bq._Weight(fmt, N, K, 16, 16)
                    need = int(libbq.bq_gemv_workspace_bytes(M, ctypes.byref(w)))
                    worst = max(worst, need)
                    assert need <= cap, (fmt, M, K, N, need, cap)
    assert worst > 0


def _gemv_call(libbq):
    """bq_gemv with valid-looking arguments (aligned fake pointers): validation passes."""
    w = bq._Weight(bq.BINARY_G128, 256, 1024, 1 << 20, 1 << 21)
    return libbq.bq_gemv(1 << 22, 1, 1, ctypes.byref(w), 1 << 23, 2, 1 << 24, 1 << 20, None)


def test_injected_launch_failure(libbq):
    """bq_debug_fail_next_launches(n): the next n calls that pass validation return
    BQ_ERR_CUDA with the injected-failure message and launch nothing; invalid arguments are
    still reported as such first."""
    libbq.bq_debug_fail_next_launches(2)
    try:
        w = bq._Weight(bq.BINARY_G128, 256, 1000, 1 << 20, 1 << 21)          # K not a multiple of 128
        assert libbq.bq_gemv(1 << 22, 1, 1, ctypes.byref(w), 1 << 23, 2, None, 0, None) == 2
        for _ in range(2):
            assert _gemv_call(libbq) == 6
            assert b"injected launch failure" in libbq.bq_last_error()
        st = _gemv_call(libbq)                                                # back to the real path
        assert b"injected" not in libbq.bq_last_error()
        if not torch_cuda_available():
            assert st == 6                                                    # no device here
    finally:
        libbq.bq_debug_fail_next_launches(0)


def torch_cuda_available():
    import torch
    return torch.cuda.is_available()


def test_fault_injection_from_environment(tmp_path):
    """BQ_FAULT=launch:2 makes the first two compute calls of a fresh process fail as injected."""
    code = (
        "import ctypes, sys\n"
        f"sys.path.insert(0, {ROOT!r})\n"
        "import ternary_g128_weight_bq_b200 as bq\n"
        "L = bq.lib()\n"
        "w = bq._Weight(0, 256, 1024, 1 << 20, 1 << 21)\n"
        "out = []\n"
        "for _ in range(3):\n"
        "    L.bq_gemv(1 << 22, 1, 1, ctypes.byref(w), 1 << 23, 2, 1 << 24, 1 << 20, None)\n"
        "    out.append(b'injected' in L.bq_last_error())\n"
        "print(out)\n")
    env = dict(os.environ, BQ_FAULT="launch:2")
    p = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, env=env, timeout=120)
    assert p.returncode == 0, p.stderr
    assert p.stdout.strip().splitlines()[-1] == "[True, True, False]"


def test_new_calls_validate_before_any_cuda_call(libbq):
    """The base-3 pack, the quantiser, the top-k GEMV and the SwiGLU MLP reject bad arguments in
    host validation; sizes of the base-3 storage; the workspace queries of the new calls."""
    W = ctypes.byref
    V = ctypes.c_void_p
    # sizes: 26 bytes per group of 128; words rounded up
    assert libbq.bq_packed_bytes(2, 3, 256) == 3 * 52
    assert libbq.bq_packed_words(2, 3, 128) == (3 * 26 + 3) // 4
    assert libbq.bq_packed_bytes(0, 3, 256) == 3 * 32 and libbq.bq_packed_bytes(1, 3, 256) == 3 * 64
    assert libbq.bq_packed_bytes(2, 3, 100) == 0
    # base-3 pack
    assert libbq.bq_pack_ternary_b3_g128(None, 16, 1, 128, 16, 16, None) == 1
    assert libbq.bq_pack_ternary_b3_g128(16, 16, 1, 96, 16, 16, None) == 2
    assert libbq.bq_pack_ternary_b3_g128(17, 16, 1, 128, 16, 16, None) == 3
    # quantiser: NULL, format, dtype, shape, alignment
    assert libbq.bq_quantize_g128(None, 2, 4, 256, 0, 16, 16, None) == 1
    assert libbq.bq_quantize_g128(16, 2, 4, 256, 7, 16, 16, None) == 1
    assert libbq.bq_quantize_g128(16, 9, 4, 256, 0, 16, 16, None) == 4
    assert libbq.bq_quantize_g128(16, 2, 4, 200, 0, 16, 16, None) == 2
    assert libbq.bq_quantize_g128(16, 2, 4, 256, 0, 24, 16, None) == 3
    # top-k: k range, NULL outputs, sampling arguments, shape the tensor-core path cannot take,
    # workspace
    w = bq._Weight(0, 256, 1024, 1 << 20, 1 << 21)
    big = 1 << 30
    args = lambda k=20, vals=1 << 22, u=None, T=0.7, p=0.95, tok=None, ws=1 << 24, wsb=big, K_w=w: (
        1 << 23, 1, 1, W(K_w), k, vals, 1 << 25, u, T, p, tok, ws, wsb, None)
    for f in (libbq.bq_gemv_topk,):
        f.argtypes = [V, ctypes.c_int, ctypes.c_int64, ctypes.POINTER(bq._Weight), ctypes.c_int, V, V, V,
                      ctypes.c_float, ctypes.c_float, V, V, ctypes.c_size_t, V]
    assert libbq.bq_gemv_topk(*args(k=0)) == 2 and libbq.bq_gemv_topk(*args(k=33)) == 2
    assert libbq.bq_gemv_topk(*args(vals=None)) == 1
    assert libbq.bq_gemv_topk(*args(u=1 << 26)) == 1                          # u without tokens
    assert libbq.bq_gemv_topk(*args(u=1 << 26, tok=1 << 27, T=0.0)) == 1
    assert libbq.bq_gemv_topk(*args(u=1 << 26, tok=1 << 27, p=1.5)) == 1
    w640 = bq._Weight(0, 256, 640, 1 << 20, 1 << 21)
    assert libbq.bq_gemv_topk(*args(K_w=w640)) == 2
    assert libbq.bq_gemv_topk(*args(ws=1 << 24, wsb=16)) == 9
    assert libbq.bq_gemv_topk_workspace_bytes(1, W(w), 20) > 0
    assert libbq.bq_gemv_topk_workspace_bytes(1, W(w640), 20) == 0
    lm = bq._Weight(0, 248320, 5120, 1 << 20, 1 << 21)
    assert libbq.bq_gemv_topk_workspace_bytes(8, W(lm), 20) > 148 * 8 * 20 * 8
    # SwiGLU MLP: shapes must chain, M range
    g = bq._Weight(0, 512, 1024, 1 << 20, 1 << 21)
    u2 = bq._Weight(0, 528, 1024, 1 << 20, 1 << 21)
    d = bq._Weight(0, 256, 512, 1 << 20, 1 << 21)
    dbad = bq._Weight(0, 256, 640, 1 << 20, 1 << 21)
    assert libbq.bq_mlp_swiglu(1 << 23, 1, 1, W(g), W(u2), W(d), 1 << 22, 2, 1 << 24, big, None) == 2
    assert libbq.bq_mlp_swiglu(1 << 23, 1, 1, W(g), W(g), W(dbad), 1 << 22, 2, 1 << 24, big, None) == 2
    assert libbq.bq_mlp_swiglu(1 << 23, 1, 9, W(g), W(g), W(d), 1 << 22, 2, 1 << 24, big, None) == 2
    assert libbq.bq_mlp_swiglu(1 << 23, 1, 1, W(g), W(g), W(d), 1 << 22, 2, 1 << 24, 16, None) == 9
    assert libbq.bq_mlp_swiglu_workspace_bytes(1, W(g), W(g), W(d)) > 0
    assert libbq.bq_mlp_swiglu_workspace_bytes(1, W(g), W(u2), W(d)) == 0
    # injected failures reach the new calls after validation, with nothing launched
    libbq.bq_debug_fail_next_launches(4)
    try:
        assert libbq.bq_gemv_topk(*args()) == 6 and b"injected" in libbq.bq_last_error()
        assert libbq.bq_mlp_swiglu(1 << 23, 1, 1, W(g), W(g), W(d), 1 << 22, 2, 1 << 24, big, None) == 6
        assert b"injected" in libbq.bq_last_error()
        assert libbq.bq_quantize_g128(16, 2, 4, 256, 2, 32, 48, None) == 6
        assert b"injected" in libbq.bq_last_error()
        assert libbq.bq_pack_ternary_b3_g128(16, 32, 1, 128, 48, 64, None) == 6
        assert b"injected" in libbq.bq_last_error()
    finally:
        libbq.bq_debug_fail_next_launches(0)
