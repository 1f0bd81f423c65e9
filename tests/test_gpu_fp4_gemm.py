"""fp4_gemm: the W4A4 product of two FP4 microscaling operands on the
block-scaled tensor cores ("post-training-quantization-gptq-awq-and-rotation"
(arganzheng.life), sections 九.1-九.2), against the fp64 oracle -- the exact
product of the dequantized operands.

Product tests feed both sides the same seeded operand bytes (every E2M1 code,
the whole range of scale bytes) and compare sampled rows at full Llama-3-70B
sizes and every row on ragged small shapes; the end-to-end test quantizes
weights and activations on the GPU with the library's quantizers and on the
CPU with the oracle's, then compares the two products.  The host test checks
argument validation without a GPU.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import post_weight_quantization_group_b200 as q4
from post_weight_quantization_group_b200 import workloads as wl

TOL = 4e-3
A16 = 0x10000  # fake 16-byte-aligned device address: validation fails first
F32 = lambda v: float(np.float32(v))  # noqa: E731


def test_fp4_gemm_host_validation():
    from post_weight_quantization_group_b200 import build
    build.build()
    lib = q4.load_library()

    def call(fmt=1, out=256, inn=1024, B=4, wq=A16, ws=A16, wts=A16, xq=A16, xs=A16, xts=A16,
             y=A16, ydt=q4.Q4_BF16, work=A16):
        return lib.fp4_gemm(fmt, wq, ws, wts, out, inn, xq, xs, xts, B, y, ydt, work, 1 << 24,
                            None)

    assert call(fmt=2) == q4.Q4_ERR_INVALID_ARG
    assert call(ydt=7) == q4.Q4_ERR_INVALID_ARG
    assert call(inn=1024 + 128) == q4.Q4_ERR_SHAPE           # NVFP4: in % 256
    assert call(fmt=0, inn=1024 + 256) == q4.Q4_ERR_SHAPE    # MXFP4: in % 512
    assert call(B=0) == q4.Q4_ERR_SHAPE
    assert call(out=-1) == q4.Q4_ERR_SHAPE
    assert call(out=0) == q4.Q4_OK
    assert call(xq=None) == q4.Q4_ERR_INVALID_ARG
    assert call(wts=None) == q4.Q4_ERR_INVALID_ARG           # NVFP4 needs both tensor scales
    assert call(ws=A16 + 4) == q4.Q4_ERR_ALIGNMENT
    assert call(xs=A16 + 8) == q4.Q4_ERR_ALIGNMENT
    assert call(y=A16 + 1) == q4.Q4_ERR_ALIGNMENT
    assert call(work=None) == q4.Q4_ERR_WORKSPACE
    assert lib.fp4_gemm_workspace_bytes(2, 256, 1024, 4) == 0
    assert lib.fp4_gemm_workspace_bytes(1, 256, 1024, 0) == 0
    assert lib.fp4_gemm_workspace_bytes(0, 256, 1024, 4) > 0


def _within(y, y_ref, what):
    y = np.asarray(y, dtype=np.float64)
    rms = float(np.sqrt(np.mean(y_ref ** 2)))
    bound = TOL * (np.abs(y_ref) + rms)
    err = np.abs(y - y_ref)
    assert np.all(err <= bound), f"{what}: worst err/bound {float(np.max(err / bound)):.3f}"
    return float(np.max(err / bound))


def _sample(out, n, seed):
    if out <= n:
        return np.arange(out, dtype=np.int64)
    rng = np.random.default_rng(seed)
    return np.unique(np.concatenate([[0, out - 1], rng.choice(out, n - 2, replace=False)])).astype(np.int64)


def _tensor_scales(fmt):
    if fmt == "nvfp4":
        return F32(wl.FP4_W_TENSOR_SCALE), F32(wl.FP4_X_TENSOR_SCALE)
    return None, None


def _gpu_operand(packed, scales, rows, inn, fmt, ts):
    dev = torch.device("cuda:0")
    t = None if ts is None else torch.tensor([ts], dtype=torch.float32, device=dev)
    return q4.FP4Weight(packed.to(dev), scales.to(dev), rows, inn, fmt, t)


def _product_case(fmt, out, inn, B, seed, nrows, ydtype=torch.float32):
    wp, ws = wl.fp4_operand(out, inn, fmt, seed)
    xp, xs = wl.fp4_operand(B, inn, fmt, seed + 1)
    wts, xts = _tensor_scales(fmt)
    W = _gpu_operand(wp, ws, out, inn, fmt, wts)
    X = _gpu_operand(xp, xs, B, inn, fmt, xts)
    y = q4.fp4_gemm(W, X, y_dtype=ydtype)
    torch.cuda.synchronize()
    assert q4.q4_sync_status() == q4.Q4_OK
    rows = _sample(out, nrows, seed)
    y_ref = oracle.fp4_gemm(fmt, wp.numpy()[rows], ws.numpy()[rows], wts, xp.numpy(), xs.numpy(),
                            xts)
    _within(y.float().cpu().numpy()[:, rows], y_ref, f"{fmt} {out}x{inn} B={B}")
    return W, X, y


@pytest.mark.gpu
@pytest.mark.parametrize("fmt", ["nvfp4", "mxfp4"])
@pytest.mark.parametrize("name", ["q_proj", "gate_proj", "down_proj"])
@pytest.mark.parametrize("B", [16, 32, 64, 128])
def test_fp4_gemm_llama3_70b(fmt, name, B):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    out, inn = wl.LLAMA3_70B[name]
    _product_case(fmt, out, inn, B, seed=7 * B + len(name), nrows=24 if B == 128 else 48)


@pytest.mark.gpu
@pytest.mark.parametrize("fmt,inn", [("nvfp4", 1792), ("mxfp4", 1536), ("nvfp4", 256),
                                     ("mxfp4", 512)])
@pytest.mark.parametrize("B", [1, 5, 17, 130])
def test_fp4_gemm_ragged(fmt, inn, B):
    """300 rows: a partial row tile; NVFP4 in = 1792 ends in half a chunk; one
    chunk of K; B = 1 (the narrowest MMA), 17 (a partial 32-wide tile), 130
    (two launches of 128 and 2 activation rows); every row checked."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    _product_case(fmt, 300, inn, B, seed=100 + B, nrows=300)


@pytest.mark.gpu
@pytest.mark.parametrize("ydtype", [torch.bfloat16, torch.float16])
def test_fp4_gemm_output_dtypes(ydtype):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    W, X, y16 = _product_case("nvfp4", 1000, 2048, 24, seed=300, nrows=1000, ydtype=ydtype)
    y32 = q4.fp4_gemm(W, X, y_dtype=torch.float32)
    assert torch.equal(y16, y32.to(ydtype))


@pytest.mark.gpu
@pytest.mark.parametrize("fmt", ["nvfp4", "mxfp4"])
def test_fp4_gemm_deterministic_split_tiles(fmt):
    """70B down_proj: every row tile is split between CTAs (56 chunks of K
    over 148 CTAs); repeated calls agree bit for bit."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    out, inn = wl.LLAMA3_70B["down_proj"]
    W, X, y = _product_case(fmt, out, inn, 16, seed=400, nrows=32)
    for _ in range(3):
        assert torch.equal(q4.fp4_gemm(W, X, y_dtype=torch.float32), y)


@pytest.mark.gpu
@pytest.mark.parametrize("fmt,inn,B", [("nvfp4", 4096, 64), ("mxfp4", 2560, 100),
                                       ("nvfp4", 1536, 33)])
def test_fp4_gemm_cluster_fixup(fmt, inn, B):
    """B > 32 on 300 rows: the CTAs of a row tile form a cluster (8 chunks of
    K -> 8 CTAs of one chunk each, 5 -> 5, 3 -> 3) and add their partials
    through distributed shared memory; every row checked, repeated calls
    bit-identical."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    W, X, y = _product_case(fmt, 300, inn, B, seed=600 + B, nrows=300)
    for _ in range(2):
        assert torch.equal(q4.fp4_gemm(W, X, y_dtype=torch.float32), y)


@pytest.mark.gpu
@pytest.mark.parametrize("fmt", ["nvfp4", "mxfp4"])
def test_fp4_gemm_cluster_deterministic_70b(fmt):
    """70B down_proj at B = 128: 64 row tiles x 2 CTAs in clusters of two;
    repeated calls agree bit for bit."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    out, inn = wl.LLAMA3_70B["down_proj"]
    W, X, y = _product_case(fmt, out, inn, 128, seed=700, nrows=16)
    for _ in range(2):
        assert torch.equal(q4.fp4_gemm(W, X, y_dtype=torch.float32), y)


@pytest.mark.gpu
@pytest.mark.parametrize("fmt", ["nvfp4", "mxfp4"])
def test_fp4_gemm_end_to_end_quantized(fmt):
    """Weights N(0, 0.02^2) and activations with outlier channels, each
    quantized on the GPU by the library and on the CPU by the oracle; the
    W4A4 products agree within the tolerance."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    dev = torch.device("cuda:0")
    out, inn, B = 1024, 4096, 32
    Wd = wl.normal_weight(out, inn, 500, device=dev)
    xd = wl.activations(B, inn, 501, dtype=torch.bfloat16, n_outliers=4, outlier_seed=502,
                        device=dev)
    y = q4.fp4_gemm(q4.fp4_quantize(Wd, fmt), q4.fp4_quantize(xd, fmt), y_dtype=torch.float32)
    torch.cuda.synchronize()
    assert q4.q4_sync_status() == q4.Q4_OK
    Wc = Wd.float().cpu().numpy()
    xc = xd.float().cpu().numpy()
    if fmt == "nvfp4":
        wq, ws, wts = oracle.nvfp4_quantize(Wc)
        xq, xs, xts = oracle.nvfp4_quantize(xc)
    else:
        (wq, ws), wts = oracle.mxfp4_quantize(Wc), None
        (xq, xs), xts = oracle.mxfp4_quantize(xc), None
    y_ref = oracle.fp4_gemm(fmt, wq, ws, wts, xq, xs, xts)
    _within(y.cpu().numpy(), y_ref, f"{fmt} end to end")
