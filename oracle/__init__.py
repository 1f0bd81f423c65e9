"""CPU oracle for group-wise INT4 quantization and the W4A16 decode product.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
package.  The product library never loads it and shares no code with it.

The arithmetic lives in ``q4_oracle.c`` (plain single-threaded C11, IEEE fp32
for the quantizer as the pages state it, fp64 for the products); this module
only compiles it with gcc on first use and marshals numpy arrays.

Functions with no independent pin beyond their definition are listed in the
header of ``q4_oracle.c``; every function here is pinned by
``tests/test_oracle_pins.py``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import tempfile

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "q4_oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD, "libq4oracle.so")
CFLAGS = ["-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off", "-fno-fast-math",
          "-fvisibility=hidden", "-Wall", "-Wextra"]

_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle shared library (idempotent); returns its path."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    os.makedirs(_BUILD, exist_ok=True)
    fd, tmp = tempfile.mkstemp(suffix=".so", dir=_BUILD)
    os.close(fd)
    subprocess.run(["gcc", *CFLAGS, _SRC, "-o", tmp, "-lm"], check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is not None:
        return _lib
    lib = ctypes.CDLL(build())
    P = ctypes.c_void_p
    I64 = ctypes.c_int64
    I32 = ctypes.c_int32
    lib.oracle_f16_to_f32.argtypes = [ctypes.c_uint16]
    lib.oracle_f16_to_f32.restype = ctypes.c_float
    lib.oracle_f32_to_f16.argtypes = [ctypes.c_float]
    lib.oracle_f32_to_f16.restype = ctypes.c_uint16
    lib.oracle_bf16_to_f32.argtypes = [ctypes.c_uint16]
    lib.oracle_bf16_to_f32.restype = ctypes.c_float
    lib.oracle_f32_to_bf16.argtypes = [ctypes.c_float]
    lib.oracle_f32_to_bf16.restype = ctypes.c_uint16
    for name in ("oracle_f16_to_f32_n", "oracle_f32_to_f16_n", "oracle_bf16_to_f32_n",
                 "oracle_f32_to_bf16_n"):
        getattr(lib, name).argtypes = [P, P, I64]
        getattr(lib, name).restype = None
    lib.oracle_quantize_value.argtypes = [ctypes.c_float, ctypes.c_float, I32, I32, I32]
    lib.oracle_quantize_value.restype = I32
    lib.oracle_quantize_pack.argtypes = [P, I64, I64, I32, I32, P, P, P]
    lib.oracle_quantize_pack.restype = ctypes.c_int
    lib.oracle_code_at.argtypes = [P, I64, I64, I64, I32]
    lib.oracle_code_at.restype = I32
    lib.oracle_dequant_f32.argtypes = [P, P, P, I64, I64, I32, I32, P]
    lib.oracle_dequant_f32.restype = ctypes.c_int
    lib.oracle_gemv_rows_f64.argtypes = [P, P, P, I64, I64, I32, I32, P, I64, P, I64, P]
    lib.oracle_gemv_rows_f64.restype = ctypes.c_int
    lib.oracle_gemv_f64.argtypes = [P, P, P, I64, I64, I32, I32, P, I64, P]
    lib.oracle_gemv_f64.restype = ctypes.c_int
    lib.oracle_dense_rows_f64.argtypes = [P, I64, I64, P, I64, P, I64, P]
    lib.oracle_dense_rows_f64.restype = ctypes.c_int
    lib.oracle_quantize_pack_perm.argtypes = [P, I64, I64, I32, I32, P, P, P, P]
    lib.oracle_quantize_pack_perm.restype = ctypes.c_int
    lib.oracle_clip_search_group.argtypes = [P, I32, I32, P, P]
    lib.oracle_clip_search_group.restype = I32
    lib.oracle_quantize_pack_clip.argtypes = [P, I64, I64, I32, I32, P, P, P]
    lib.oracle_q8_quantize_per_channel.argtypes = [P, I64, I64, P, P]
    lib.oracle_q8_dequant_f32.argtypes = [P, P, I64, I64, P]
    lib.oracle_q8_gemv_rows_f64.argtypes = [P, P, I64, I64, P, I64, P, I64, P]
    lib.oracle_kv_quantize_int8.argtypes = [P, I64, I64, I32, P, P]
    lib.oracle_kv_dequant_int8.argtypes = [P, P, I64, I64, I32, P]
    lib.oracle_e2m1_to_f32.argtypes = [ctypes.c_uint8]
    lib.oracle_e2m1_to_f32.restype = ctypes.c_float
    lib.oracle_f32_to_e2m1.argtypes = [ctypes.c_float]
    lib.oracle_f32_to_e2m1.restype = ctypes.c_uint8
    lib.oracle_e4m3_to_f32.argtypes = [ctypes.c_uint8]
    lib.oracle_e4m3_to_f32.restype = ctypes.c_float
    lib.oracle_f32_to_e4m3_sat.argtypes = [ctypes.c_float]
    lib.oracle_f32_to_e4m3_sat.restype = ctypes.c_uint8
    lib.oracle_mxfp4_quantize.argtypes = [P, I64, I64, P, P]
    lib.oracle_mxfp4_dequant.argtypes = [P, P, I64, I64, P]
    lib.oracle_nvfp4_quantize.argtypes = [P, I64, I64, P, P, P]
    lib.oracle_nvfp4_dequant.argtypes = [P, P, ctypes.c_float, I64, I64, P]
    lib.oracle_fp4_gemm_f64.argtypes = [P, P, ctypes.c_float, P, P, ctypes.c_float, I32, I64, I64,
                                        I64, P]
    lib.oracle_quantize_pack_clip.restype = ctypes.c_int
    _lib = lib
    return lib


def _ptr(a: np.ndarray | None):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


# ----------------------------------------------------------------- codecs

def f16_to_f32(h: int) -> float:
    return _load().oracle_f16_to_f32(int(h))


def f32_to_f16(f: float) -> int:
    return _load().oracle_f32_to_f16(float(f))


def bf16_to_f32(b: int) -> float:
    return _load().oracle_bf16_to_f32(int(b))


def f32_to_bf16(f: float) -> int:
    return _load().oracle_f32_to_bf16(float(f))


def _codec_n(fn: str, a: np.ndarray, in_dtype, out_dtype) -> np.ndarray:
    src = np.ascontiguousarray(a, dtype=in_dtype)
    dst = np.empty(src.shape, dtype=out_dtype)
    getattr(_load(), fn)(_ptr(src), _ptr(dst), src.size)
    return dst


def f16_bits_to_f32_array(h: np.ndarray) -> np.ndarray:
    """Element-wise oracle fp16 decode of a uint16 array."""
    return _codec_n("oracle_f16_to_f32_n", h, np.uint16, np.float32)


def f32_to_f16_bits_array(f: np.ndarray) -> np.ndarray:
    """Element-wise oracle fp32 -> fp16 (round to nearest even) encode."""
    return _codec_n("oracle_f32_to_f16_n", f, np.float32, np.uint16)


def bf16_bits_to_f32_array(b: np.ndarray) -> np.ndarray:
    return _codec_n("oracle_bf16_to_f32_n", b, np.uint16, np.float32)


def f32_to_bf16_bits_array(f: np.ndarray) -> np.ndarray:
    return _codec_n("oracle_f32_to_bf16_n", f, np.float32, np.uint16)


def quantize_value(w: float, s: float, z: int, qmin: int, qmax: int) -> int:
    """clamp(rne(w / s) + z, qmin, qmax) with an fp32 scale s."""
    return _load().oracle_quantize_value(float(w), float(s), int(z), int(qmin), int(qmax))


# -------------------------------------------------------------- quantizer

def quantize_pack(W: np.ndarray, group_size: int, symmetric: bool):
    """W: [out, in] float32 (exact values of fp16/bf16 weights).

    Returns (qweight uint8 [out, in/2], scales uint16 fp16-bits [out, in/g],
    zeros uint16 fp16-bits [out, in/g] or None)."""
    W = np.ascontiguousarray(W, dtype=np.float32)
    out, inn = W.shape
    G = inn // group_size
    q = np.zeros((out, inn // 2), dtype=np.uint8)
    s = np.zeros((out, G), dtype=np.uint16)
    z = None if symmetric else np.zeros((out, G), dtype=np.uint16)
    rc = _load().oracle_quantize_pack(_ptr(W), out, inn, int(group_size), int(bool(symmetric)),
                                      _ptr(q), _ptr(s), _ptr(z))
    if rc != 0:
        raise ValueError("oracle_quantize_pack rejected its arguments")
    return q, s, z


def quantize_pack_perm(W: np.ndarray, group_size: int, symmetric: bool, perm: np.ndarray):
    """Act-order quantization: columns taken in the order perm (groups over
    that order, codes and scales stored in it).  Same outputs as quantize_pack."""
    W = np.ascontiguousarray(W, dtype=np.float32)
    perm = np.ascontiguousarray(perm, dtype=np.int32)
    out, inn = W.shape
    G = inn // group_size
    q = np.zeros((out, inn // 2), dtype=np.uint8)
    s = np.zeros((out, G), dtype=np.uint16)
    z = None if symmetric else np.zeros((out, G), dtype=np.uint16)
    rc = _load().oracle_quantize_pack_perm(_ptr(W), out, inn, int(group_size), int(bool(symmetric)),
                                           _ptr(perm), _ptr(q), _ptr(s), _ptr(z))
    if rc != 0:
        raise ValueError("oracle_quantize_pack_perm rejected its arguments")
    return q, s, z


def g_idx(perm: np.ndarray, group_size: int) -> np.ndarray:
    """Group of each original column: g_idx[perm[j]] = j // group_size."""
    perm = np.asarray(perm, dtype=np.int64)
    gi = np.empty(perm.size, dtype=np.int32)
    gi[perm] = np.arange(perm.size) // group_size
    return gi


def quantize_pack_clip(W: np.ndarray, group_size: int, n_alpha: int):
    """Symmetric INT4 with the per-group range search (see
    oracle_clip_search_group).  Returns (qweight uint8 [out, in/2], scales
    uint16 fp16-bits [out, in/g], alpha index int32 [out, in/g])."""
    W = np.ascontiguousarray(W, dtype=np.float32)
    out, inn = W.shape
    G = inn // group_size
    q = np.zeros((out, inn // 2), dtype=np.uint8)
    s = np.zeros((out, G), dtype=np.uint16)
    idx = np.zeros((out, G), dtype=np.int32)
    rc = _load().oracle_quantize_pack_clip(_ptr(W), out, inn, int(group_size), int(n_alpha),
                                           _ptr(q), _ptr(s), _ptr(idx))
    if rc != 0:
        raise ValueError("oracle_quantize_pack_clip rejected its arguments")
    return q, s, idx


def clip_errors(w: np.ndarray, n_alpha: int):
    """One group: (chosen index, fp64 errors E_j [n], fp16 scale bits [n])."""
    w = np.ascontiguousarray(w, dtype=np.float32).ravel()
    err = np.zeros(n_alpha, dtype=np.float64)
    s16 = np.zeros(n_alpha, dtype=np.uint16)
    best = _load().oracle_clip_search_group(_ptr(w), int(w.size), int(n_alpha), _ptr(err), _ptr(s16))
    return int(best), err, s16


def code_at(qweight: np.ndarray, inn: int, r: int, k: int, symmetric: bool) -> int:
    return _load().oracle_code_at(_ptr(np.ascontiguousarray(qweight)), inn, r, k, int(symmetric))


def dequant(qweight, scales, zeros, out: int, inn: int, group_size: int, symmetric: bool):
    """Returns W_hat [out, in] float32 = s * (q - z) (exact in fp32)."""
    qweight = np.ascontiguousarray(qweight, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint16)
    zeros = None if zeros is None else np.ascontiguousarray(zeros, dtype=np.uint16)
    W_hat = np.empty((out, inn), dtype=np.float32)
    rc = _load().oracle_dequant_f32(_ptr(qweight), _ptr(scales), _ptr(zeros), out, inn,
                                    int(group_size), int(bool(symmetric)), _ptr(W_hat))
    if rc != 0:
        raise ValueError("oracle_dequant_f32 rejected its arguments")
    return W_hat


def gemv(qweight, scales, zeros, out: int, inn: int, group_size: int, symmetric: bool,
         x: np.ndarray, rows=None) -> np.ndarray:
    """y [B, len(rows)] fp64 = x . W_hat^T over the given rows (all if None).

    x: [B, in] float (exact values of the bf16/fp16 activations)."""
    qweight = np.ascontiguousarray(qweight, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint16)
    zeros = None if zeros is None else np.ascontiguousarray(zeros, dtype=np.uint16)
    x = np.ascontiguousarray(np.atleast_2d(x), dtype=np.float64)
    B = x.shape[0]
    if rows is None:
        rows = np.arange(out, dtype=np.int64)
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    y = np.empty((B, rows.shape[0]), dtype=np.float64)
    rc = _load().oracle_gemv_rows_f64(_ptr(qweight), _ptr(scales), _ptr(zeros), out, inn,
                                      int(group_size), int(bool(symmetric)), _ptr(x), B,
                                      _ptr(rows), rows.shape[0], _ptr(y))
    if rc != 0:
        raise ValueError("oracle_gemv_rows_f64 rejected its arguments")
    return y


def dense(W: np.ndarray, x: np.ndarray, rows=None) -> np.ndarray:
    """y [B, len(rows)] fp64 = x . W^T for float32 W (exact bf16 values)."""
    W = np.ascontiguousarray(W, dtype=np.float32)
    out, inn = W.shape
    x = np.ascontiguousarray(np.atleast_2d(x), dtype=np.float64)
    B = x.shape[0]
    if rows is None:
        rows = np.arange(out, dtype=np.int64)
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    y = np.empty((B, rows.shape[0]), dtype=np.float64)
    rc = _load().oracle_dense_rows_f64(_ptr(W), out, inn, _ptr(x), B, _ptr(rows),
                                       rows.shape[0], _ptr(y))
    if rc != 0:
        raise ValueError("oracle_dense_rows_f64 rejected its arguments")
    return y


# ------------------------------------------------ per-channel INT8 weights

def q8_quantize_per_channel(W: np.ndarray):
    """W: [out, in] float32.  Returns (q int8 [out, in], scales float32 [out])."""
    W = np.ascontiguousarray(W, dtype=np.float32)
    out, inn = W.shape
    q = np.zeros((out, inn), dtype=np.int8)
    s = np.zeros(out, dtype=np.float32)
    if _load().oracle_q8_quantize_per_channel(_ptr(W), out, inn, _ptr(q), _ptr(s)) != 0:
        raise ValueError("oracle_q8_quantize_per_channel rejected its arguments")
    return q, s


def q8_dequant(q: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """W_hat [out, in] float32 = q * s (one fp32 multiplication)."""
    q = np.ascontiguousarray(q, dtype=np.int8)
    scales = np.ascontiguousarray(scales, dtype=np.float32)
    out, inn = q.shape
    W_hat = np.empty((out, inn), dtype=np.float32)
    if _load().oracle_q8_dequant_f32(_ptr(q), _ptr(scales), out, inn, _ptr(W_hat)) != 0:
        raise ValueError("oracle_q8_dequant_f32 rejected its arguments")
    return W_hat


def q8_gemv(q: np.ndarray, scales: np.ndarray, x: np.ndarray, rows=None) -> np.ndarray:
    """y [B, len(rows)] fp64 = s[r] * sum_k q[r, k] x[b, k] over the given rows."""
    q = np.ascontiguousarray(q, dtype=np.int8)
    scales = np.ascontiguousarray(scales, dtype=np.float32)
    out, inn = q.shape
    x = np.ascontiguousarray(np.atleast_2d(x), dtype=np.float64)
    B = x.shape[0]
    if rows is None:
        rows = np.arange(out, dtype=np.int64)
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    y = np.empty((B, rows.shape[0]), dtype=np.float64)
    if _load().oracle_q8_gemv_rows_f64(_ptr(q), _ptr(scales), out, inn, _ptr(x), B, _ptr(rows),
                                       rows.shape[0], _ptr(y)) != 0:
        raise ValueError("oracle_q8_gemv_rows_f64 rejected its arguments")
    return y


# ------------------------------------------------------------- KV cache

def kv_quantize_int8(kv: np.ndarray, is_bf16: bool):
    """kv: [..., head_dim] float32 (exact values of an fp16 / bf16 cache).

    Returns (codes int8 [..., head_dim], scales uint16 bits of the cache
    type [...]), one scale per row of head_dim values."""
    kv = np.ascontiguousarray(kv, dtype=np.float32)
    d = kv.shape[-1]
    rows = kv.size // d
    codes = np.zeros(kv.shape, dtype=np.int8)
    scales = np.zeros(kv.shape[:-1], dtype=np.uint16)
    if _load().oracle_kv_quantize_int8(_ptr(kv), rows, d, int(bool(is_bf16)), _ptr(codes),
                                       _ptr(scales)) != 0:
        raise ValueError("oracle_kv_quantize_int8 rejected its arguments")
    return codes, scales


def kv_dequant_int8(codes: np.ndarray, scales: np.ndarray, is_bf16: bool) -> np.ndarray:
    """uint16 bits of the cache type, q * s rounded once."""
    codes = np.ascontiguousarray(codes, dtype=np.int8)
    scales = np.ascontiguousarray(scales, dtype=np.uint16)
    d = codes.shape[-1]
    out = np.zeros(codes.shape, dtype=np.uint16)
    if _load().oracle_kv_dequant_int8(_ptr(codes), _ptr(scales), codes.size // d, d,
                                      int(bool(is_bf16)), _ptr(out)) != 0:
        raise ValueError("oracle_kv_dequant_int8 rejected its arguments")
    return out


def kv_quantize_int4(kv: np.ndarray, group_size: int):
    """INT4 group quantization of a KV cache along head_dim ("压缩算法"
    section 7.4.1.2, quantize_kv_cache_int4): the symmetric group quantizer
    (s = amax / 7, codes in [-8, 7], two codes per byte) on the rows of
    head_dim values.  Returns (packed uint8 [..., head_dim/2], scales uint16
    fp16 bits [..., head_dim/group_size])."""
    kv = np.ascontiguousarray(kv, dtype=np.float32)
    d = kv.shape[-1]
    q, s, _ = quantize_pack(kv.reshape(-1, d), group_size, True)
    lead = kv.shape[:-1]
    return q.reshape(*lead, d // 2), s.reshape(*lead, d // group_size)


# ------------------------------------------------------ FP4 microscaling

def e2m1_to_f32(c: int) -> float:
    return _load().oracle_e2m1_to_f32(int(c))


def f32_to_e2m1(v: float) -> int:
    return _load().oracle_f32_to_e2m1(float(v))


def e4m3_to_f32(c: int) -> float:
    return _load().oracle_e4m3_to_f32(int(c))


def f32_to_e4m3_sat(v: float) -> int:
    return _load().oracle_f32_to_e4m3_sat(float(v))


def mxfp4_quantize(W: np.ndarray):
    """W [out, in] float32 -> (packed uint8 [out, in/2], E8M0 scale bytes [out, in/32])."""
    W = np.ascontiguousarray(W, dtype=np.float32)
    out, inn = W.shape
    q = np.zeros((out, inn // 2), dtype=np.uint8)
    s = np.zeros((out, inn // 32), dtype=np.uint8)
    if _load().oracle_mxfp4_quantize(_ptr(W), out, inn, _ptr(q), _ptr(s)) != 0:
        raise ValueError("oracle_mxfp4_quantize rejected its arguments")
    return q, s


def mxfp4_dequant(q: np.ndarray, s: np.ndarray) -> np.ndarray:
    q = np.ascontiguousarray(q, dtype=np.uint8)
    s = np.ascontiguousarray(s, dtype=np.uint8)
    out, inn = q.shape[0], q.shape[1] * 2
    W_hat = np.empty((out, inn), dtype=np.float32)
    if _load().oracle_mxfp4_dequant(_ptr(q), _ptr(s), out, inn, _ptr(W_hat)) != 0:
        raise ValueError("oracle_mxfp4_dequant rejected its arguments")
    return W_hat


def nvfp4_quantize(W: np.ndarray):
    """W [out, in] float32 -> (packed uint8 [out, in/2], E4M3 scale bytes
    [out, in/16], fp32 tensor scale)."""
    W = np.ascontiguousarray(W, dtype=np.float32)
    out, inn = W.shape
    q = np.zeros((out, inn // 2), dtype=np.uint8)
    s = np.zeros((out, inn // 16), dtype=np.uint8)
    st = np.zeros(1, dtype=np.float32)
    if _load().oracle_nvfp4_quantize(_ptr(W), out, inn, _ptr(q), _ptr(s), _ptr(st)) != 0:
        raise ValueError("oracle_nvfp4_quantize rejected its arguments")
    return q, s, float(st[0])


def nvfp4_dequant(q: np.ndarray, s: np.ndarray, tensor_scale: float) -> np.ndarray:
    q = np.ascontiguousarray(q, dtype=np.uint8)
    s = np.ascontiguousarray(s, dtype=np.uint8)
    out, inn = q.shape[0], q.shape[1] * 2
    W_hat = np.empty((out, inn), dtype=np.float32)
    if _load().oracle_nvfp4_dequant(_ptr(q), _ptr(s), float(tensor_scale), out, inn,
                                    _ptr(W_hat)) != 0:
        raise ValueError("oracle_nvfp4_dequant rejected its arguments")
    return W_hat


def fp4_gemm(fmt: str, wq, ws, w_st, xq, xs, x_st) -> np.ndarray:
    """W4A4 product y [B, out] fp64 of two FP4 operands of the same format
    (packed codes and scale bytes as mxfp4_quantize / nvfp4_quantize return
    them; w_st, x_st the NVFP4 tensor scales, ignored for MXFP4)."""
    wq = np.ascontiguousarray(wq, dtype=np.uint8)
    ws = np.ascontiguousarray(ws, dtype=np.uint8)
    xq = np.ascontiguousarray(np.atleast_2d(xq), dtype=np.uint8)
    xs = np.ascontiguousarray(np.atleast_2d(xs), dtype=np.uint8)
    out, inn, B = wq.shape[0], wq.shape[1] * 2, xq.shape[0]
    y = np.empty((B, out), dtype=np.float64)
    f = 0 if fmt == "mxfp4" else 1
    if _load().oracle_fp4_gemm_f64(_ptr(wq), _ptr(ws), float(w_st or 1.0), _ptr(xq), _ptr(xs),
                                   float(x_st or 1.0), f, out, inn, B, _ptr(y)) != 0:
        raise ValueError("oracle_fp4_gemm_f64 rejected its arguments")
    return y
