"""CPU oracle for the weight-only quantized matmul (test infrastructure only).

Only the test-suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product library never does; it
shares no code with this oracle (see ``qmm_oracle.c`` for the definitions and
the pages each one follows).

This module compiles ``qmm_oracle.c`` with gcc (``-O2 -ffp-contract=off``)
into ``liboracle.so`` next to it and wraps it with ctypes, taking and
returning numpy arrays.  Large calls are split over output rows and run on a
thread pool: ctypes drops the GIL during the foreign call, so the C code runs
in parallel while each thread stays plain single-threaded C.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from concurrent.futures import ThreadPoolExecutor

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "qmm_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

F32, F16, BF16 = 0, 1, 2
_NP_STORAGE = {F32: np.float32, F16: np.uint16, BF16: np.uint16}
ORC_OK, ORC_ERR_ARG, ORC_ERR_ID = 0, 1, 7

_lock = threading.Lock()
_lib = None


CFLAGS = ["-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared"]


def compile_oracle(src: str, out: str) -> str:
    """gcc `src` into the shared library `out` with the oracle's flags."""
    subprocess.run(["gcc", *CFLAGS, "-o", out, src, "-lm"], check=True)
    return out


def build_oracle(force: bool = False) -> str:
    """Compile the oracle shared library (idempotent); returns its path."""
    with _lock:
        fresh = os.path.exists(_LIB) and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC)
        if force or not fresh:
            tmp = _LIB + f".tmp{os.getpid()}"
            compile_oracle(_SRC, tmp)
            os.replace(tmp, _LIB)
    return _LIB


class _Stack(ctypes.Structure):
    _fields_ = [("packed", ctypes.c_void_p), ("scales", ctypes.c_void_p),
                ("biases", ctypes.c_void_p), ("s_dtype", ctypes.c_int),
                ("num_experts", ctypes.c_int64), ("n_rows", ctypes.c_int64),
                ("n_cols", ctypes.c_int64), ("gs", ctypes.c_int), ("bits", ctypes.c_int)]


def bind(path: str) -> ctypes.CDLL:
    """Load a compiled oracle library and declare its C signatures."""
    L = ctypes.CDLL(path)
    vp, i64, c_int = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
    L.orc_bf16_to_f32.argtypes = [ctypes.c_uint16]
    L.orc_bf16_to_f32.restype = ctypes.c_float
    L.orc_f16_to_f32.argtypes = [ctypes.c_uint16]
    L.orc_f16_to_f32.restype = ctypes.c_float
    L.orc_f32_to_bf16.argtypes = [ctypes.c_float]
    L.orc_f32_to_bf16.restype = ctypes.c_uint16
    L.orc_f32_to_f16.argtypes = [ctypes.c_float]
    L.orc_f32_to_f16.restype = ctypes.c_uint16
    L.orc_words_per_row.argtypes = [i64, c_int]
    L.orc_words_per_row.restype = i64
    L.orc_pack_row.argtypes = [vp, i64, c_int, vp]
    L.orc_pack_row.restype = None
    L.orc_fp4_e2m1.argtypes = [ctypes.c_uint32]
    L.orc_fp4_e2m1.restype = ctypes.c_float
    L.orc_e8m0.argtypes = [ctypes.c_uint32]
    L.orc_e8m0.restype = ctypes.c_float
    L.orc_fp8_e4m3.argtypes = [ctypes.c_uint32]
    L.orc_fp8_e4m3.restype = ctypes.c_float
    L.orc_dequantize_mx.argtypes = [vp, vp, c_int, i64, i64, vp, c_int, i64, i64]
    L.orc_dequantize_mx.restype = c_int
    L.orc_matmul_mx.argtypes = [vp, c_int, i64, i64, vp, vp, c_int, i64, vp, i64, i64]
    L.orc_matmul_mx.restype = c_int
    L.orc_quantize_dynamic_int8.argtypes = [vp, c_int, i64, vp, vp]
    L.orc_quantize_dynamic_int8.restype = c_int
    L.orc_dequantize_dynamic_int8.argtypes = [vp, i64, vp, vp, c_int]
    L.orc_dequantize_dynamic_int8.restype = c_int
    L.orc_matmul_dynamic_int8.argtypes = [vp, c_int, i64, i64, vp, vp, i64, vp, i64, i64]
    L.orc_matmul_dynamic_int8.restype = c_int
    L.orc_code_integral.argtypes = [vp, c_int, i64]
    L.orc_code_integral.restype = ctypes.c_uint32
    L.orc_code_u64.argtypes = [vp, i64, c_int, i64]
    L.orc_code_u64.restype = ctypes.c_uint32
    L.orc_quantize.argtypes = [vp, c_int, i64, i64, c_int, c_int, c_int, vp, vp, vp, i64, i64]
    L.orc_dequantize.argtypes = [vp, vp, vp, c_int, i64, i64, c_int, c_int, vp, c_int, i64, i64]
    L.orc_matmul.argtypes = [vp, c_int, i64, i64, vp, vp, vp, c_int, i64, c_int, c_int, c_int,
                             vp, i64, i64]
    L.orc_matmul_element.argtypes = [vp, c_int, i64, i64, vp, vp, vp, c_int, i64, c_int,
                                     c_int, c_int, i64, i64]
    L.orc_matmul_element.restype = ctypes.c_double
    sp = ctypes.POINTER(_Stack)
    L.orc_moe_gemv_id.argtypes = [vp, c_int, vp, i64, i64, sp, vp, i64, i64]
    L.orc_moe_gemv_id_batched.argtypes = [vp, c_int, vp, i64, i64, i64, i64, sp, vp, i64, i64]
    L.orc_moe_gate_up_silu.argtypes = [vp, c_int, vp, i64, sp, sp, vp, i64, i64]
    L.orc_moe_gate_up_silu_batched.argtypes = [vp, c_int, vp, i64, i64, i64, i64, sp, sp, vp,
                                               i64, i64]
    return L


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        _lib = bind(build_oracle())
    return _lib


def _ptr(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data


def _threads(n_threads):
    if n_threads is None:
        try:
            n_threads = len(os.sched_getaffinity(0))
        except AttributeError:
            n_threads = os.cpu_count() or 1
    return max(1, int(n_threads))


def _split(lo, hi, parts):
    n = hi - lo
    if n <= 0:
        return []
    parts = max(1, min(parts, n))
    step = (n + parts - 1) // parts
    return [(a, min(a + step, hi)) for a in range(lo, hi, step)]


def _run(fn, lo, hi, n_threads):
    chunks = _split(lo, hi, _threads(n_threads) * 2)
    if len(chunks) <= 1:
        rcs = [fn(a, b) for a, b in chunks]
    else:
        with ThreadPoolExecutor(max_workers=_threads(n_threads)) as ex:
            rcs = list(ex.map(lambda ab: fn(*ab), chunks))
    return max(rcs) if rcs else ORC_OK


def dtype_code(storage: str) -> int:
    return {"f32": F32, "f16": F16, "bf16": BF16}[storage]


# ---------------------------------------------------------------- conversions
def bf16_to_f32(h: int) -> float:
    return float(lib().orc_bf16_to_f32(int(h)))


def f16_to_f32(h: int) -> float:
    return float(lib().orc_f16_to_f32(int(h)))


def f32_to_bf16(v: float) -> int:
    return int(lib().orc_f32_to_bf16(float(v)))


def f32_to_f16(v: float) -> int:
    return int(lib().orc_f32_to_f16(float(v)))


def words_per_row(cols: int, bits: int) -> int:
    return int(lib().orc_words_per_row(cols, bits))


# ---------------------------------------------------------------- packing
def pack_row(codes: np.ndarray, bits: int) -> np.ndarray:
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    words = np.zeros(words_per_row(codes.size, bits), dtype=np.uint32)
    lib().orc_pack_row(_ptr(codes), codes.size, bits, _ptr(words))
    return words


def code_integral(row: np.ndarray, bits: int, i: int) -> int:
    row = np.ascontiguousarray(row, dtype=np.uint32)
    return int(lib().orc_code_integral(_ptr(row), bits, i))


def code_u64(row: np.ndarray, bits: int, i: int) -> int:
    row = np.ascontiguousarray(row, dtype=np.uint32)
    return int(lib().orc_code_u64(_ptr(row), row.size, bits, i))


# ---------------------------------------------------------------- quantize / dequantize
def quantize(w: np.ndarray, w_dtype: int, group_size: int, bits: int, s_dtype: int,
             n_threads=None):
    """w: [rows, cols] array in its storage form (float32, or uint16 bits for f16/bf16).
    Returns (packed u32 [rows, cols*bits/32], scales, biases [rows, cols/gs]) in storage form."""
    w = np.ascontiguousarray(w)
    rows, cols = w.shape
    packed = np.zeros((rows, cols * bits // 32), dtype=np.uint32)
    G = cols // group_size
    scales = np.zeros((rows, G), dtype=_NP_STORAGE[s_dtype])
    biases = np.zeros((rows, G), dtype=_NP_STORAGE[s_dtype])
    L = lib()

    def fn(a, b):
        return L.orc_quantize(_ptr(w), w_dtype, rows, cols, group_size, bits, s_dtype,
                              _ptr(packed), _ptr(scales), _ptr(biases), a, b)
    rc = _run(fn, 0, rows, n_threads)
    if rc != ORC_OK:
        raise ValueError(f"oracle quantize rejected the arguments (rc={rc})")
    return packed, scales, biases


def dequantize(packed, scales, biases, s_dtype: int, cols: int, group_size: int, bits: int,
               out_dtype: int, n_threads=None) -> np.ndarray:
    packed = np.ascontiguousarray(packed, dtype=np.uint32)
    rows = packed.shape[0]
    out = np.zeros((rows, cols), dtype=_NP_STORAGE[out_dtype])
    L = lib()

    def fn(a, b):
        return L.orc_dequantize(_ptr(packed), _ptr(scales), _ptr(biases), s_dtype, rows, cols,
                                group_size, bits, _ptr(out), out_dtype, a, b)
    rc = _run(fn, 0, rows, n_threads)
    if rc != ORC_OK:
        raise ValueError(f"oracle dequantize rejected the arguments (rc={rc})")
    return out


# ---------------------------------------------------------------- matmul
def matmul(x, x_dtype: int, packed, scales, biases, s_dtype: int, N: int, group_size: int,
           bits: int, transpose: bool = True, n_threads=None) -> np.ndarray:
    """fp64 y[M, N] = x . dequant(W)^T (transpose) or x . dequant(W)."""
    x = np.ascontiguousarray(x)
    M, K = x.shape
    y = np.zeros((M, N), dtype=np.float64)
    L = lib()
    packed = np.ascontiguousarray(packed, dtype=np.uint32)

    def fn(a, b):
        return L.orc_matmul(_ptr(x), x_dtype, M, K, _ptr(packed), _ptr(scales), _ptr(biases),
                            s_dtype, N, group_size, bits, int(bool(transpose)), _ptr(y), a, b)
    rc = _run(fn, 0, N, n_threads)
    if rc != ORC_OK:
        raise ValueError(f"oracle matmul rejected the arguments (rc={rc})")
    return y


def widen_f64(x, x_dtype: int) -> np.ndarray:
    """Storage-form activations (float32, or the uint16 bit patterns of f16 /
    bf16) as float64: exact widening, element by element by definition
    (bf16 = the high half of an fp32; f16 = IEEE binary16)."""
    x = np.ascontiguousarray(x)
    if x_dtype == BF16:
        return (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    if x_dtype == F16:
        return x.view(np.float16).astype(np.float64)
    return x.astype(np.float64)


def matmul_dense(x, x_dtype: int, packed, scales, biases, s_dtype: int, N: int, group_size: int,
                 bits: int, n_threads=None) -> np.ndarray:
    """fp64 y[M, N] = x . dequant(W)^T for whole-output checks of large
    calls: the weights are dequantized by this oracle (fmaf, bit-exact) and
    widened to fp64, then the product is one library fp64 matrix multiply
    (numpy).  Same definition as matmul(); only the summation order differs,
    so the two agree within K * 2^-53 * sum |x| |w| per element."""
    x = np.ascontiguousarray(x)
    M, K = x.shape
    w = dequantize(packed, scales, biases, s_dtype, K, group_size, bits, F32, n_threads)
    return widen_f64(x, x_dtype) @ w.astype(np.float64).T


def matmul_elements(x, x_dtype: int, packed, scales, biases, s_dtype: int, N: int,
                    group_size: int, bits: int, coords, transpose: bool = True,
                    n_threads=None) -> np.ndarray:
    """fp64 y[m, n] for each (m, n) in coords (sampled checks at full size)."""
    x = np.ascontiguousarray(x)
    M, K = x.shape
    packed = np.ascontiguousarray(packed, dtype=np.uint32)
    coords = list(coords)
    out = np.zeros(len(coords), dtype=np.float64)
    L = lib()

    def fn(a, b):
        for i in range(a, b):
            m, n = coords[i]
            out[i] = L.orc_matmul_element(_ptr(x), x_dtype, M, K, _ptr(packed), _ptr(scales),
                                          _ptr(biases), s_dtype, N, group_size, bits,
                                          int(bool(transpose)), int(m), int(n))
        return ORC_OK
    _run(fn, 0, len(coords), n_threads)
    return out


# ---------------------------------------------------------------- MoE
class Stack:
    """Host-side expert stack: packed [E*n_rows, n_cols*bits/32] u32, scales and
    biases [E*n_rows, n_cols/gs] in storage form."""

    def __init__(self, packed, scales, biases, s_dtype, num_experts, n_rows, n_cols, group_size,
                 bits):
        self.packed = np.ascontiguousarray(packed, dtype=np.uint32)
        self.scales = np.ascontiguousarray(scales)
        self.biases = np.ascontiguousarray(biases)
        self.c = _Stack(self.packed.ctypes.data, self.scales.ctypes.data,
                        self.biases.ctypes.data, s_dtype, num_experts, n_rows, n_cols,
                        group_size, bits)
        self.n_rows = n_rows
        self.n_cols = n_cols


def moe_gemv_id(a, a_dtype, ids, n_selected, src1_stride, st: Stack, n_threads=None):
    a = np.ascontiguousarray(a)
    ids = np.ascontiguousarray(ids, dtype=np.int32)
    out = np.zeros((n_selected, st.n_rows), dtype=np.float64)
    L = lib()

    def fn(lo, hi):
        return L.orc_moe_gemv_id(_ptr(a), a_dtype, _ptr(ids), n_selected, src1_stride,
                                 ctypes.byref(st.c), _ptr(out), lo, hi)
    rc = _run(fn, 0, n_selected, n_threads)
    return out, rc


def moe_gemv_id_batched(a, a_dtype, ids, m, top_k, outer, inner, st: Stack, n_threads=None):
    a = np.ascontiguousarray(a)
    ids = np.ascontiguousarray(ids, dtype=np.int32)
    out = np.zeros((m * top_k, st.n_rows), dtype=np.float64)
    L = lib()

    def fn(lo, hi):
        return L.orc_moe_gemv_id_batched(_ptr(a), a_dtype, _ptr(ids), m, top_k, outer, inner,
                                         ctypes.byref(st.c), _ptr(out), lo, hi)
    rc = _run(fn, 0, m * top_k, n_threads)
    return out, rc


def moe_gate_up_silu(a, a_dtype, ids, n_selected, gate: Stack, up: Stack, n_threads=None):
    a = np.ascontiguousarray(a)
    ids = np.ascontiguousarray(ids, dtype=np.int32)
    out = np.zeros((n_selected, gate.n_rows), dtype=np.float64)
    L = lib()

    def fn(lo, hi):
        return L.orc_moe_gate_up_silu(_ptr(a), a_dtype, _ptr(ids), n_selected,
                                      ctypes.byref(gate.c), ctypes.byref(up.c), _ptr(out), lo, hi)
    rc = _run(fn, 0, n_selected, n_threads)
    return out, rc


def moe_gate_up_silu_batched(a, a_dtype, ids, m, top_k, outer, inner, gate: Stack, up: Stack,
                             n_threads=None):
    a = np.ascontiguousarray(a)
    ids = np.ascontiguousarray(ids, dtype=np.int32)
    out = np.zeros((m * top_k, gate.n_rows), dtype=np.float64)
    L = lib()

    def fn(lo, hi):
        return L.orc_moe_gate_up_silu_batched(_ptr(a), a_dtype, _ptr(ids), m, top_k, outer,
                                              inner, ctypes.byref(gate.c), ctypes.byref(up.c),
                                              _ptr(out), lo, hi)
    rc = _run(fn, 0, m * top_k, n_threads)
    return out, rc


def moe_batched_dense(a, a_dtype, ids, m, top_k, outer, inner, st: Stack, n_threads=None):
    """fp64 out[p] = a[(p/top_k)*outer + (p%top_k)*inner : ... + n_cols] .
    dequant(W[ids[p]])^T for whole-output checks of large MoE calls: each
    expert used is dequantized by this oracle (fmaf, bit-exact), its pairs'
    rows are gathered, and the product is one library fp64 matrix multiply
    per expert (numpy).  Same definition as moe_gemv_id_batched (summation
    order aside); a pair with an id outside [0, E) gets a zero row and
    rc = ORC_ERR_ID."""
    a = widen_f64(np.ascontiguousarray(a).reshape(-1), a_dtype)
    ids = np.ascontiguousarray(ids, dtype=np.int32).reshape(-1)
    P = m * top_k
    out = np.zeros((P, st.n_rows), dtype=np.float64)
    rc = ORC_OK
    K = st.n_cols
    n_experts = st.c.num_experts
    for e in np.unique(ids[:P]):
        sel = np.nonzero(ids[:P] == e)[0]
        if e < 0 or e >= n_experts:
            rc = ORC_ERR_ID
            continue
        r0, r1 = int(e) * st.n_rows, (int(e) + 1) * st.n_rows
        w = dequantize(st.packed[r0:r1], st.scales[r0:r1], st.biases[r0:r1], st.c.s_dtype, K,
                       st.c.gs, st.c.bits, F32, n_threads).astype(np.float64)
        offs = (sel // top_k) * outer + (sel % top_k) * inner
        rows = a[offs[:, None] + np.arange(K)[None, :]]
        out[sel] = rows @ w.T
    return out, rc


# ---------------------------------------------------------------- microscaled modes
MODE_AFFINE, MODE_MXFP4, MODE_MXFP8, MODE_NVFP4 = 0, 1, 2, 3
MX_PARAMS = {MODE_MXFP4: (4, 32), MODE_MXFP8: (8, 32), MODE_NVFP4: (4, 16)}  # (bits, group size)


def fp4_e2m1(code: int) -> float:
    return float(lib().orc_fp4_e2m1(int(code)))


def e8m0(s: int) -> float:
    return float(lib().orc_e8m0(int(s)))


def fp8_e4m3(b: int) -> float:
    return float(lib().orc_fp8_e4m3(int(b)))


def dequantize_mx(packed, scales, mode: int, cols: int, out_dtype: int, n_threads=None) -> np.ndarray:
    """w_hat = lane(q) * scale(s) of a microscaled matrix: packed [rows,
    cols*bits/32] u32, scales [rows, cols/gs] u8 (no biases)."""
    packed = np.ascontiguousarray(packed, dtype=np.uint32)
    scales = np.ascontiguousarray(scales, dtype=np.uint8)
    rows = packed.shape[0]
    out = np.zeros((rows, cols), dtype=_NP_STORAGE[out_dtype])
    L = lib()

    def fn(a, b):
        return L.orc_dequantize_mx(_ptr(packed), _ptr(scales), mode, rows, cols, _ptr(out), out_dtype,
                                   a, b)
    rc = _run(fn, 0, rows, n_threads)
    if rc != ORC_OK:
        raise ValueError(f"oracle dequantize_mx rejected the arguments (rc={rc})")
    return out


def matmul_mx(x, x_dtype: int, packed, scales, mode: int, N: int, n_threads=None) -> np.ndarray:
    """fp64 y[M, N] = x . dequant_mx(W)^T (W is [N, K] quantized along K)."""
    x = np.ascontiguousarray(x)
    M, K = x.shape
    packed = np.ascontiguousarray(packed, dtype=np.uint32)
    scales = np.ascontiguousarray(scales, dtype=np.uint8)
    y = np.zeros((M, N), dtype=np.float64)
    L = lib()

    def fn(a, b):
        return L.orc_matmul_mx(_ptr(x), x_dtype, M, K, _ptr(packed), _ptr(scales), mode, N, _ptr(y), a, b)
    rc = _run(fn, 0, N, n_threads)
    if rc != ORC_OK:
        raise ValueError(f"oracle matmul_mx rejected the arguments (rc={rc})")
    return y


# ---------------------------------------------------------------- per-tensor dynamic int8
def quantize_dynamic_int8(w, w_dtype: int):
    """whole-tensor min/max int8: (q int8 same shape, params float32[4] =
    {input_min, input_max, output_min, output_max})"""
    w = np.ascontiguousarray(w)
    q = np.zeros(w.shape, dtype=np.int8)
    params = np.zeros(4, dtype=np.float32)
    rc = lib().orc_quantize_dynamic_int8(_ptr(w), w_dtype, w.size, _ptr(q), _ptr(params))
    if rc != ORC_OK:
        raise ValueError(f"oracle quantize_dynamic_int8 rejected the arguments (rc={rc})")
    return q, params


def dequantize_dynamic_int8(q, params, out_dtype: int) -> np.ndarray:
    q = np.ascontiguousarray(q, dtype=np.int8)
    params = np.ascontiguousarray(params, dtype=np.float32)
    out = np.zeros(q.shape, dtype=_NP_STORAGE[out_dtype])
    rc = lib().orc_dequantize_dynamic_int8(_ptr(q), q.size, _ptr(params), _ptr(out), out_dtype)
    if rc != ORC_OK:
        raise ValueError(f"oracle dequantize_dynamic_int8 rejected the arguments (rc={rc})")
    return out


def matmul_dynamic_int8(x, x_dtype: int, q, params, n_threads=None) -> np.ndarray:
    """fp64 y[M, N] = x . w_hat^T for an int8 [N, K] weight"""
    x = np.ascontiguousarray(x)
    M, K = x.shape
    q = np.ascontiguousarray(q, dtype=np.int8)
    N = q.shape[0]
    params = np.ascontiguousarray(params, dtype=np.float32)
    y = np.zeros((M, N), dtype=np.float64)
    L = lib()

    def fn(a, b):
        return L.orc_matmul_dynamic_int8(_ptr(x), x_dtype, M, K, _ptr(q), _ptr(params), N, _ptr(y), a, b)
    rc = _run(fn, 0, N, n_threads)
    if rc != ORC_OK:
        raise ValueError(f"oracle matmul_dynamic_int8 rejected the arguments (rc={rc})")
    return y
