"""Python binding of the q4 C ABI (include/q4.h) for NVIDIA B200.

Argument marshalling only: every step of the quantize / dequantize / decode
product path runs in the CUDA kernels of ``libq4.so``.  PyTorch provides the
device memory (outputs are allocated here when not given) and the stream
(``torch.cuda.current_stream()`` unless one is passed).  There is no CPU path:
if ``libq4.so`` cannot be loaded every call raises ``Q4LibraryError``.

Names follow the C ABI: ``q4_quantize_pack``, ``q4_dequant``, ``q4_gemv``,
``q4_gemm_skinny``, ``bf16_gemv_ref_bw``, ``q4_sync_status``, the per-channel
INT8 weight calls ``q8_quantize_per_channel``, ``q8_dequant``, ``q8_gemv`` and
the KV-cache calls ``kv_quantize_int8``, ``kv_dequant_int8``,
``kv_quantize_int4``, ``kv_dequant_int4``.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libq4.so")

Q4_OK = 0
Q4_ERR_INVALID_ARG = 1
Q4_ERR_SHAPE = 2
Q4_ERR_ALIGNMENT = 3
Q4_ERR_UNSUPPORTED = 4
Q4_ERR_CUDA = 5
Q4_ERR_TIMEOUT = 6
Q4_ERR_WORKSPACE = 7

Q4_F16, Q4_BF16, Q4_F32 = 0, 1, 2
_DT = {torch.float16: Q4_F16, torch.bfloat16: Q4_BF16, torch.float32: Q4_F32}

# every symbol include/q4.h declares
ABI_SYMBOLS = (
    "q4_quantize_pack", "q4_dequant", "q4_gemv", "q4_gemm_skinny", "bf16_gemv_ref_bw",
    "q4_sync_status", "q4_status_string", "q4_version", "q4_selftest_wait_timeout",
    "q4_workspace_bytes", "q4_gemv_noalloc", "q4_quantize_pack_clip", "q4_quantize_pack_perm",
    "q4_permute_activations", "q8_quantize_per_channel", "q8_dequant", "q8_workspace_bytes",
    "q8_gemv", "kv_quantize_int8", "kv_dequant_int8", "kv_quantize_int4", "kv_dequant_int4",
    "mxfp4_quantize", "mxfp4_dequant", "nvfp4_quantize", "nvfp4_dequant", "q4_gemv_grouped",
    "fp4_gemm_workspace_bytes", "fp4_gemm", "bf16_ref_workspace_bytes",
)


class Q4LibraryError(RuntimeError):
    """libq4.so is missing or failed to load (there is no fallback)."""


class Q4Error(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)}")


class _CWeight(ctypes.Structure):
    _fields_ = [
        ("qweight", ctypes.c_void_p),
        ("scales", ctypes.c_void_p),
        ("zeros", ctypes.c_void_p),
        ("out", ctypes.c_int64),
        ("in_", ctypes.c_int64),
        ("group_size", ctypes.c_int32),
        ("bits", ctypes.c_int32),
        ("symmetric", ctypes.c_int32),
    ]


_lib = None


def load_library(path: str = LIB_PATH):
    """Load libq4.so (once) and declare the C signatures."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise Q4LibraryError(
            f"{path} not found: build it with `python -m post_weight_quantization_group_b200.build`")
    try:
        lib = ctypes.CDLL(path)
    except OSError as e:  # pragma: no cover - environment dependent
        raise Q4LibraryError(f"cannot load {path}: {e}") from e
    P, I64, I32, S = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_int
    W = ctypes.POINTER(_CWeight)
    lib.q4_quantize_pack.argtypes = [P, S, I64, I64, I32, I32, I32, P, P, P, P]
    lib.q4_dequant.argtypes = [W, P, S, P]
    lib.q4_quantize_pack_clip.argtypes = [P, S, I64, I64, I32, I32, P, P, P]
    lib.q4_quantize_pack_perm.argtypes = [P, S, I64, I64, I32, I32, I32, P, P, P, P, P]
    lib.q4_permute_activations.argtypes = [P, S, I64, I64, P, P, P]
    lib.q4_gemv.argtypes = [W, P, S, I64, P, S, P, ctypes.c_size_t, P]
    lib.q4_gemm_skinny.argtypes = [W, P, S, I64, P, S, P, ctypes.c_size_t, P]
    lib.q4_gemv_noalloc.argtypes = [W, P, S, I64, P, S, P]
    lib.q4_gemv_grouped.argtypes = [W, I32, P, S, I64, ctypes.POINTER(P), S, P, ctypes.c_size_t, P]
    lib.q4_workspace_bytes.argtypes = [I64, I64, I64, I32]
    lib.q4_workspace_bytes.restype = ctypes.c_size_t
    lib.bf16_gemv_ref_bw.argtypes = [P, I64, I64, P, I64, P, P, ctypes.c_size_t, P]
    lib.bf16_ref_workspace_bytes.argtypes = [I64, I64, I64]
    lib.bf16_ref_workspace_bytes.restype = ctypes.c_size_t
    lib.q4_sync_status.argtypes = [P]
    lib.q4_selftest_wait_timeout.argtypes = [I64, P]
    lib.q8_quantize_per_channel.argtypes = [P, S, I64, I64, P, P, P]
    lib.q8_dequant.argtypes = [P, P, I64, I64, P, S, P]
    lib.q8_workspace_bytes.argtypes = [I64, I64, I64]
    lib.q8_workspace_bytes.restype = ctypes.c_size_t
    lib.q8_gemv.argtypes = [P, P, I64, I64, P, S, I64, P, S, P, ctypes.c_size_t, P]
    lib.kv_quantize_int8.argtypes = [P, S, I64, I64, P, P, P]
    lib.kv_dequant_int8.argtypes = [P, P, S, I64, I64, P, P]
    lib.kv_quantize_int4.argtypes = [P, S, I64, I64, I32, P, P, P]
    lib.kv_dequant_int4.argtypes = [P, P, I64, I64, I32, P, S, P]
    lib.mxfp4_quantize.argtypes = [P, S, I64, I64, P, P, P]
    lib.mxfp4_dequant.argtypes = [P, P, I64, I64, P, S, P]
    lib.nvfp4_quantize.argtypes = [P, S, I64, I64, P, P, P, P]
    lib.nvfp4_dequant.argtypes = [P, P, P, I64, I64, P, S, P]
    lib.fp4_gemm_workspace_bytes.argtypes = [I32, I64, I64, I64]
    lib.fp4_gemm_workspace_bytes.restype = ctypes.c_size_t
    lib.fp4_gemm.argtypes = [I32, P, P, P, I64, I64, P, P, P, I64, P, S, P, ctypes.c_size_t, P]
    for f in ("q4_quantize_pack", "q4_quantize_pack_clip", "q4_quantize_pack_perm",
              "q4_permute_activations", "q4_dequant", "q4_gemv",
              "q4_gemm_skinny", "q4_gemv_noalloc",
              "bf16_gemv_ref_bw", "q4_sync_status", "q4_selftest_wait_timeout",
              "q8_quantize_per_channel", "q8_dequant", "q8_gemv", "kv_quantize_int8",
              "kv_dequant_int8", "kv_quantize_int4", "kv_dequant_int4", "mxfp4_quantize",
              "mxfp4_dequant", "nvfp4_quantize", "nvfp4_dequant", "fp4_gemm"):
        getattr(lib, f).restype = S
    lib.q4_status_string.argtypes = [S]
    lib.q4_status_string.restype = ctypes.c_char_p
    lib.q4_version.argtypes = []
    lib.q4_version.restype = ctypes.c_char_p
    _lib = lib
    return lib


def status_string(status: int) -> str:
    return load_library().q4_status_string(int(status)).decode()


def version() -> str:
    return load_library().q4_version().decode()


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _ptr(t: torch.Tensor | None) -> int | None:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("q4 takes device tensors only")
    if not t.is_contiguous():
        raise ValueError("q4 takes contiguous tensors only")
    return t.data_ptr()


def _check(status: int, what: str):
    if status != Q4_OK:
        raise Q4Error(status, what)


@dataclass
class Q4Weight:
    """A packed INT4 weight: codes [out, in/2] uint8, fp16 scales [out, in/g],
    fp16 zero points [out, in/g] (None if symmetric)."""
    qweight: torch.Tensor
    scales: torch.Tensor
    zeros: torch.Tensor | None
    out: int
    in_features: int
    group_size: int
    symmetric: bool
    bits: int = 4
    perm: torch.Tensor | None = None  # act order: stored column j is original column perm[j]

    def c_struct(self) -> _CWeight:
        return _CWeight(_ptr(self.qweight), _ptr(self.scales), _ptr(self.zeros), self.out,
                        self.in_features, self.group_size, self.bits, int(self.symmetric))

    @property
    def nbytes(self) -> int:
        n = self.qweight.numel() + self.scales.numel() * 2
        return n + (self.zeros.numel() * 2 if self.zeros is not None else 0)


def q4_quantize_pack(W: torch.Tensor, group_size: int = 128, symmetric: bool = True,
                     bits: int = 4, qweight: torch.Tensor | None = None,
                     scales: torch.Tensor | None = None, zeros: torch.Tensor | None = None,
                     stream=None) -> Q4Weight:
    lib = load_library()
    if W.dim() != 2 or W.dtype not in (torch.float16, torch.bfloat16):
        raise ValueError("W must be a 2-D fp16 or bf16 tensor")
    out, inn = W.shape
    G = inn // group_size if group_size > 0 else 0
    dev = W.device
    if qweight is None:
        qweight = torch.empty(out, inn // 2, dtype=torch.uint8, device=dev)
    if scales is None:
        scales = torch.empty(out, G, dtype=torch.float16, device=dev)
    if zeros is None and not symmetric:
        zeros = torch.empty(out, G, dtype=torch.float16, device=dev)
    st = lib.q4_quantize_pack(_ptr(W), _DT[W.dtype], out, inn, group_size, bits,
                              int(symmetric), _ptr(qweight), _ptr(scales), _ptr(zeros),
                              _stream(stream))
    _check(st, "q4_quantize_pack")
    return Q4Weight(qweight, scales, zeros, out, inn, group_size, bool(symmetric), bits)


def q4_quantize_pack_clip(W: torch.Tensor, group_size: int = 128, n_alpha: int = 21,
                          qweight: torch.Tensor | None = None,
                          scales: torch.Tensor | None = None, stream=None) -> Q4Weight:
    """Symmetric INT4 quantization with the per-group range search over
    n_alpha ranges from max|w| down to 0.8 max|w| (q4.h, q4_quantize_pack_clip)."""
    lib = load_library()
    if W.dim() != 2 or W.dtype not in (torch.float16, torch.bfloat16):
        raise ValueError("W must be a 2-D fp16 or bf16 tensor")
    out, inn = W.shape
    G = inn // group_size if group_size > 0 else 0
    dev = W.device
    if qweight is None:
        qweight = torch.empty(out, inn // 2, dtype=torch.uint8, device=dev)
    if scales is None:
        scales = torch.empty(out, G, dtype=torch.float16, device=dev)
    st = lib.q4_quantize_pack_clip(_ptr(W), _DT[W.dtype], out, inn, group_size, n_alpha,
                                   _ptr(qweight), _ptr(scales), _stream(stream))
    _check(st, "q4_quantize_pack_clip")
    return Q4Weight(qweight, scales, None, out, inn, group_size, True, 4)


def q4_quantize_pack_perm(W: torch.Tensor, perm: torch.Tensor, group_size: int = 128,
                          symmetric: bool = True, stream=None) -> Q4Weight:
    """Act-order quantization: columns taken in the order perm (int32 [in] on
    the device); the result carries perm for q4_gemm_act_order."""
    lib = load_library()
    if W.dim() != 2 or W.dtype not in (torch.float16, torch.bfloat16):
        raise ValueError("W must be a 2-D fp16 or bf16 tensor")
    if perm.dtype != torch.int32 or perm.dim() != 1 or perm.numel() != W.shape[1]:
        raise ValueError("perm must be int32 [in]")
    out, inn = W.shape
    G = inn // group_size if group_size > 0 else 0
    dev = W.device
    qweight = torch.empty(out, inn // 2, dtype=torch.uint8, device=dev)
    scales = torch.empty(out, G, dtype=torch.float16, device=dev)
    zeros = None if symmetric else torch.empty(out, G, dtype=torch.float16, device=dev)
    st = lib.q4_quantize_pack_perm(_ptr(W), _DT[W.dtype], out, inn, group_size, 4, int(symmetric),
                                   _ptr(perm), _ptr(qweight), _ptr(scales), _ptr(zeros),
                                   _stream(stream))
    _check(st, "q4_quantize_pack_perm")
    return Q4Weight(qweight, scales, zeros, out, inn, group_size, bool(symmetric), 4, perm)


def q4_permute_activations(x: torch.Tensor, perm: torch.Tensor, x_perm: torch.Tensor | None = None,
                           stream=None) -> torch.Tensor:
    """x_perm[b, j] = x[b, perm[j]] (the act-order gather)."""
    lib = load_library()
    if x.dim() != 2:
        raise ValueError("x must be [rows, in]")
    if x_perm is None:
        x_perm = torch.empty_like(x)
    st = lib.q4_permute_activations(_ptr(x), _DT[x.dtype], x.shape[0], x.shape[1], _ptr(perm),
                                    _ptr(x_perm), _stream(stream))
    _check(st, "q4_permute_activations")
    return x_perm


def q4_gemm_act_order(w: Q4Weight, x: torch.Tensor, y: torch.Tensor | None = None, y_dtype=None,
                      x_perm: torch.Tensor | None = None, workspace: torch.Tensor | None = None,
                      stream=None) -> torch.Tensor:
    """y = x W_hat^T for an act-order weight: the gather, then the product."""
    if w.perm is None:
        raise ValueError("w has no column order (quantize it with q4_quantize_pack_perm)")
    xp = q4_permute_activations(x, w.perm, x_perm, stream)
    return q4_gemm_skinny(w, xp, y, y_dtype, workspace, stream)


def q4_dequant(w: Q4Weight, out_dtype=torch.float32, W_hat: torch.Tensor | None = None,
               stream=None) -> torch.Tensor:
    lib = load_library()
    if W_hat is None:
        W_hat = torch.empty(w.out, w.in_features, dtype=out_dtype, device=w.qweight.device)
    cw = w.c_struct()
    st = lib.q4_dequant(ctypes.byref(cw), _ptr(W_hat), _DT[W_hat.dtype], _stream(stream))
    _check(st, "q4_dequant")
    return W_hat


_workspaces: dict = {}


def workspace_for(w: Q4Weight, B: int, device) -> torch.Tensor:
    """A zero-filled device workspace large enough for q4_gemv / q4_gemm_skinny
    on ``w`` with batch ``B``.  One buffer per device is kept and grown on
    demand; every completed call leaves it zero-filled.  Calls that may
    overlap on the GPU (different streams) must pass their own buffers."""
    need = int(load_library().q4_workspace_bytes(w.out, w.in_features, B, w.group_size))
    return _shared_workspace(need, device)


def _shared_workspace(need: int, device) -> torch.Tensor:
    """The per-device zero-filled workspace, grown to at least ``need`` bytes
    (q4 and q8 products share its layout)."""
    dev = torch.device(device)
    key = dev.index if dev.index is not None else torch.cuda.current_device()
    buf = _workspaces.get(key)
    if buf is None or buf.numel() < need:
        buf = torch.zeros(max(need, 1 << 20), dtype=torch.uint8, device=dev)
        _workspaces[key] = buf
    return buf


def _product(fn_name: str, w: Q4Weight, x: torch.Tensor, y, y_dtype, workspace, stream):
    lib = load_library()
    if x.dim() != 2:
        raise ValueError("x must be [B, in]")
    B = x.shape[0]
    if y is None:
        y = torch.empty(B, w.out, dtype=y_dtype or x.dtype, device=x.device)
    if workspace is None:
        workspace = workspace_for(w, B, x.device)
    cw = w.c_struct()
    st = getattr(lib, fn_name)(ctypes.byref(cw), _ptr(x), _DT[x.dtype], B, _ptr(y),
                               _DT[y.dtype], _ptr(workspace), workspace.numel() * workspace.element_size(),
                               _stream(stream))
    _check(st, fn_name)
    return y


def q4_gemv(w: Q4Weight, x: torch.Tensor, y: torch.Tensor | None = None, y_dtype=None,
            workspace: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """y = x W_hat^T for B <= 8 (x [B, in] bf16/fp16; y [B, out] x.dtype or fp32)."""
    return _product("q4_gemv", w, x, y, y_dtype, workspace, stream)


def q4_gemm_skinny(w: Q4Weight, x: torch.Tensor, y: torch.Tensor | None = None, y_dtype=None,
                   workspace: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """y = x W_hat^T for B <= 128."""
    return _product("q4_gemm_skinny", w, x, y, y_dtype, workspace, stream)


Q4_GROUP_MAX = 4


def q4_gemv_grouped(ws, x: torch.Tensor, ys=None, y_dtype=None,
                    workspace: torch.Tensor | None = None, stream=None):
    """[y_i = x W_hat_i^T for W_i in ws] in one call (weights sharing ``in``,
    group size and symmetry; at most Q4_GROUP_MAX); B <= 8 is one launch."""
    lib = load_library()
    if x.dim() != 2:
        raise ValueError("x must be [B, in]")
    ws = list(ws)
    B = x.shape[0]
    if ys is None:
        ys = [torch.empty(B, w.out, dtype=y_dtype or x.dtype, device=x.device) for w in ws]
    ys = list(ys)
    if len(ys) != len(ws):
        raise ValueError("one output per weight")
    if workspace is None:
        workspace = workspace_for(ws[0], B, x.device)
    arr = (_CWeight * len(ws))(*[w.c_struct() for w in ws])
    yp = (ctypes.c_void_p * len(ys))(*[_ptr(y) for y in ys])
    st = lib.q4_gemv_grouped(arr, len(ws), _ptr(x), _DT[x.dtype], B, yp, _DT[ys[0].dtype],
                             _ptr(workspace), workspace.numel() * workspace.element_size(),
                             _stream(stream))
    _check(st, "q4_gemv_grouped")
    return ys


def q4_gemv_noalloc(w: Q4Weight, x: torch.Tensor, y: torch.Tensor | None = None, y_dtype=None,
                    stream=None) -> torch.Tensor:
    """q4_gemv with the library's static device scratch instead of a
    workspace (B <= 8).  The C call allocates nothing; pass ``y`` to keep
    this binding from allocating the output.  Calls that may overlap on the
    GPU race on the one scratch per device."""
    lib = load_library()
    if x.dim() != 2:
        raise ValueError("x must be [B, in]")
    B = x.shape[0]
    if y is None:
        y = torch.empty(B, w.out, dtype=y_dtype or x.dtype, device=x.device)
    cw = w.c_struct()
    st = lib.q4_gemv_noalloc(ctypes.byref(cw), _ptr(x), _DT[x.dtype], B, _ptr(y), _DT[y.dtype],
                             _stream(stream))
    _check(st, "q4_gemv_noalloc")
    return y


def bf16_gemv_ref_bw(W: torch.Tensor, x: torch.Tensor, y: torch.Tensor | None = None,
                     workspace: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """y = x W^T for bf16 W [out, in], x [B, in], 1 <= B <= 128, on the
    tcgen05 tensor cores (the C entry point bf16_gemv_ref_bw)."""
    lib = load_library()
    out, inn = W.shape
    B = x.shape[0]
    if y is None:
        y = torch.empty(B, out, dtype=torch.bfloat16, device=x.device)
    if workspace is None:
        workspace = _shared_workspace(int(lib.bf16_ref_workspace_bytes(out, inn, B)), x.device)
    st = lib.bf16_gemv_ref_bw(_ptr(W), out, inn, _ptr(x), B, _ptr(y), _ptr(workspace),
                              workspace.numel() * workspace.element_size(), _stream(stream))
    _check(st, "bf16_gemv_ref_bw")
    return y


def q4_sync_status(stream=None) -> int:
    """Synchronize ``stream`` and return (and clear) the device status."""
    return load_library().q4_sync_status(_stream(stream))


def q4_selftest_wait_timeout(limit_ns: int, stream=None) -> int:
    """Launch a kernel whose bounded wait can never be satisfied; returns the
    launch status (the timeout is then reported by q4_sync_status)."""
    return load_library().q4_selftest_wait_timeout(int(limit_ns), _stream(stream))


# ------------------------------------------------ per-channel INT8 weights

@dataclass
class Q8Weight:
    """Per-output-channel INT8 weight: codes [out, in] int8, fp32 scales [out]."""
    qweight: torch.Tensor
    scales: torch.Tensor
    out: int
    in_features: int

    @property
    def nbytes(self) -> int:
        return self.qweight.numel() + self.scales.numel() * 4


def q8_quantize_per_channel(W: torch.Tensor, qweight: torch.Tensor | None = None,
                            scales: torch.Tensor | None = None, stream=None) -> Q8Weight:
    """s[r] = max(amax_r, 1e-6) / 127, q = clamp(rne(W / s), -127, 127)."""
    lib = load_library()
    if W.dim() != 2 or W.dtype not in (torch.float16, torch.bfloat16):
        raise ValueError("W must be a 2-D fp16 or bf16 tensor")
    out, inn = W.shape
    if qweight is None:
        qweight = torch.empty(out, inn, dtype=torch.int8, device=W.device)
    if scales is None:
        scales = torch.empty(out, dtype=torch.float32, device=W.device)
    st = lib.q8_quantize_per_channel(_ptr(W), _DT[W.dtype], out, inn, _ptr(qweight), _ptr(scales),
                                     _stream(stream))
    _check(st, "q8_quantize_per_channel")
    return Q8Weight(qweight, scales, out, inn)


def q8_dequant(w: Q8Weight, out_dtype=torch.float32, W_hat: torch.Tensor | None = None,
               stream=None) -> torch.Tensor:
    lib = load_library()
    if W_hat is None:
        W_hat = torch.empty(w.out, w.in_features, dtype=out_dtype, device=w.qweight.device)
    st = lib.q8_dequant(_ptr(w.qweight), _ptr(w.scales), w.out, w.in_features, _ptr(W_hat),
                        _DT[W_hat.dtype], _stream(stream))
    _check(st, "q8_dequant")
    return W_hat


def q8_workspace_for(w: Q8Weight, B: int, device) -> torch.Tensor:
    """The per-device zero-filled workspace (shared with q4_gemv) grown for
    q8_gemv on ``w`` with batch ``B``."""
    return _shared_workspace(int(load_library().q8_workspace_bytes(w.out, w.in_features, B)), device)


def q8_gemv(w: Q8Weight, x: torch.Tensor, y: torch.Tensor | None = None, y_dtype=None,
            workspace: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """y = x (q * s)^T for B <= 8 (x [B, in] bf16/fp16; y [B, out] x.dtype or fp32)."""
    lib = load_library()
    if x.dim() != 2:
        raise ValueError("x must be [B, in]")
    B = x.shape[0]
    if y is None:
        y = torch.empty(B, w.out, dtype=y_dtype or x.dtype, device=x.device)
    if workspace is None:
        workspace = q8_workspace_for(w, B, x.device)
    st = lib.q8_gemv(_ptr(w.qweight), _ptr(w.scales), w.out, w.in_features, _ptr(x), _DT[x.dtype],
                     B, _ptr(y), _DT[y.dtype], _ptr(workspace),
                     workspace.numel() * workspace.element_size(), _stream(stream))
    _check(st, "q8_gemv")
    return y


# ------------------------------------------------------------- KV cache

def _kv_rows(kv: torch.Tensor):
    if kv.dim() < 1 or kv.dtype not in (torch.float16, torch.bfloat16):
        raise ValueError("kv must be an fp16 or bf16 tensor [..., head_dim]")
    d = kv.shape[-1]
    return kv.numel() // d if d else 0, d


def kv_quantize_int8(kv: torch.Tensor, codes: torch.Tensor | None = None,
                     scales: torch.Tensor | None = None, stream=None):
    """INT8 along head_dim, one scale per row in the cache's dtype.
    Returns (codes int8 kv.shape, scales kv.shape[:-1])."""
    lib = load_library()
    rows, d = _kv_rows(kv)
    if codes is None:
        codes = torch.empty(kv.shape, dtype=torch.int8, device=kv.device)
    if scales is None:
        scales = torch.empty(kv.shape[:-1], dtype=kv.dtype, device=kv.device)
    st = lib.kv_quantize_int8(_ptr(kv), _DT[kv.dtype], rows, d, _ptr(codes), _ptr(scales),
                              _stream(stream))
    _check(st, "kv_quantize_int8")
    return codes, scales


def kv_dequant_int8(codes: torch.Tensor, scales: torch.Tensor, out: torch.Tensor | None = None,
                    stream=None) -> torch.Tensor:
    """cache_type(q * s), in the dtype of ``scales``."""
    lib = load_library()
    d = codes.shape[-1]
    rows = codes.numel() // d if d else 0
    if out is None:
        out = torch.empty(codes.shape, dtype=scales.dtype, device=codes.device)
    st = lib.kv_dequant_int8(_ptr(codes), _ptr(scales), _DT[scales.dtype], rows, d, _ptr(out),
                             _stream(stream))
    _check(st, "kv_dequant_int8")
    return out


def kv_quantize_int4(kv: torch.Tensor, group_size: int = 128, packed: torch.Tensor | None = None,
                     scales: torch.Tensor | None = None, stream=None):
    """INT4 groups of group_size along head_dim (fp16 scales, codes in
    [-8, 7], two per byte).  Returns (packed uint8 [..., d/2], scales fp16
    [..., d/group_size])."""
    lib = load_library()
    rows, d = _kv_rows(kv)
    lead = tuple(kv.shape[:-1])
    if packed is None:
        packed = torch.empty(lead + (d // 2,), dtype=torch.uint8, device=kv.device)
    if scales is None:
        G = d // group_size if group_size > 0 else 0
        scales = torch.empty(lead + (G,), dtype=torch.float16, device=kv.device)
    st = lib.kv_quantize_int4(_ptr(kv), _DT[kv.dtype], rows, d, group_size, _ptr(packed),
                              _ptr(scales), _stream(stream))
    _check(st, "kv_quantize_int4")
    return packed, scales


def kv_dequant_int4(packed: torch.Tensor, scales: torch.Tensor, group_size: int = 128,
                    out_dtype=torch.float16, out: torch.Tensor | None = None,
                    stream=None) -> torch.Tensor:
    lib = load_library()
    d = packed.shape[-1] * 2
    rows = packed.numel() * 2 // d if d else 0
    if out is None:
        out = torch.empty(tuple(packed.shape[:-1]) + (d,), dtype=out_dtype, device=packed.device)
    st = lib.kv_dequant_int4(_ptr(packed), _ptr(scales), rows, d, group_size, _ptr(out),
                             _DT[out.dtype], _stream(stream))
    _check(st, "kv_dequant_int4")
    return out


# ------------------------------------------------------ FP4 microscaling

@dataclass
class FP4Weight:
    """MXFP4 (block 32, E8M0 scales) or NVFP4 (block 16, E4M3 scales and an
    fp32 tensor scale) codes [out, in/2] uint8 with scale bytes [out, in/block]."""
    packed: torch.Tensor
    scales: torch.Tensor
    out: int
    in_features: int
    fmt: str                                  # "mxfp4" or "nvfp4"
    tensor_scale: torch.Tensor | None = None  # fp32 [1] on the device (NVFP4)

    @property
    def nbytes(self) -> int:
        return self.packed.numel() + self.scales.numel() + (4 if self.tensor_scale is not None else 0)


def mxfp4_quantize(W: torch.Tensor, stream=None) -> FP4Weight:
    lib = load_library()
    if W.dim() != 2 or W.dtype not in (torch.float16, torch.bfloat16):
        raise ValueError("W must be a 2-D fp16 or bf16 tensor")
    out, inn = W.shape
    packed = torch.empty(out, inn // 2, dtype=torch.uint8, device=W.device)
    scales = torch.empty(out, inn // 32, dtype=torch.uint8, device=W.device)
    _check(lib.mxfp4_quantize(_ptr(W), _DT[W.dtype], out, inn, _ptr(packed), _ptr(scales),
                              _stream(stream)), "mxfp4_quantize")
    return FP4Weight(packed, scales, out, inn, "mxfp4")


def nvfp4_quantize(W: torch.Tensor, stream=None) -> FP4Weight:
    lib = load_library()
    if W.dim() != 2 or W.dtype not in (torch.float16, torch.bfloat16):
        raise ValueError("W must be a 2-D fp16 or bf16 tensor")
    out, inn = W.shape
    packed = torch.empty(out, inn // 2, dtype=torch.uint8, device=W.device)
    scales = torch.empty(out, inn // 16, dtype=torch.uint8, device=W.device)
    ts = torch.empty(1, dtype=torch.float32, device=W.device)
    _check(lib.nvfp4_quantize(_ptr(W), _DT[W.dtype], out, inn, _ptr(packed), _ptr(scales),
                              _ptr(ts), _stream(stream)), "nvfp4_quantize")
    return FP4Weight(packed, scales, out, inn, "nvfp4", ts)


def fp4_dequant(w: FP4Weight, out_dtype=torch.float32, W_hat: torch.Tensor | None = None,
                stream=None) -> torch.Tensor:
    lib = load_library()
    if W_hat is None:
        W_hat = torch.empty(w.out, w.in_features, dtype=out_dtype, device=w.packed.device)
    if w.fmt == "mxfp4":
        st = lib.mxfp4_dequant(_ptr(w.packed), _ptr(w.scales), w.out, w.in_features, _ptr(W_hat),
                               _DT[W_hat.dtype], _stream(stream))
    else:
        st = lib.nvfp4_dequant(_ptr(w.packed), _ptr(w.scales), _ptr(w.tensor_scale), w.out,
                               w.in_features, _ptr(W_hat), _DT[W_hat.dtype], _stream(stream))
    _check(st, f"{w.fmt}_dequant")
    return W_hat


FP4_FORMATS = {"mxfp4": 0, "nvfp4": 1}  # Q4_FP4_MXFP4, Q4_FP4_NVFP4


def fp4_quantize(W: torch.Tensor, fmt: str, stream=None) -> FP4Weight:
    """mxfp4_quantize or nvfp4_quantize by name; activations [B, in] are
    quantized the same way as weights [out, in]."""
    if fmt == "mxfp4":
        return mxfp4_quantize(W, stream)
    if fmt == "nvfp4":
        return nvfp4_quantize(W, stream)
    raise ValueError(f"unknown FP4 format {fmt!r}")


def fp4_workspace_for(w: FP4Weight, B: int, device) -> torch.Tensor:
    need = int(load_library().fp4_gemm_workspace_bytes(FP4_FORMATS[w.fmt], w.out, w.in_features, B))
    return _shared_workspace(need, device)


def fp4_gemm(w: FP4Weight, x: FP4Weight, y: torch.Tensor | None = None,
             y_dtype=torch.bfloat16, workspace: torch.Tensor | None = None,
             stream=None) -> torch.Tensor:
    """W4A4 product y [B, out] of FP4 weights ``w`` [out, in] and FP4
    activations ``x`` [B, in] of the same format, on the block-scaled tensor
    cores (the C entry point fp4_gemm)."""
    lib = load_library()
    if w.fmt != x.fmt or w.in_features != x.in_features:
        raise ValueError("w and x must share the FP4 format and `in`")
    B = x.out
    dev = w.packed.device
    if y is None:
        y = torch.empty(B, w.out, dtype=y_dtype, device=dev)
    if workspace is None:
        workspace = fp4_workspace_for(w, B, dev)
    st = lib.fp4_gemm(FP4_FORMATS[w.fmt], _ptr(w.packed), _ptr(w.scales), _ptr(w.tensor_scale),
                      w.out, w.in_features, _ptr(x.packed), _ptr(x.scales), _ptr(x.tensor_scale),
                      B, _ptr(y), _DT[y.dtype], _ptr(workspace),
                      workspace.numel() * workspace.element_size(), _stream(stream))
    _check(st, "fp4_gemm")
    return y
