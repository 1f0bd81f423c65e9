"""q4_gemv_grouped: several products that share their activations in one call.

The GPU tests check every product of a group against the fp64 oracle (the
oracle quantizes each W itself) and against the single-product entry point,
at the group shapes a decoder layer runs back to back (q/k/v, gate/up) and on
ragged shapes; the host test checks argument validation without a GPU.
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


def _cw(**kw):
    d = dict(qweight=A16, scales=A16, zeros=None, out=64, in_=256, group_size=128, bits=4,
             symmetric=1)
    d.update(kw)
    return q4._CWeight(**d)


def test_grouped_host_validation():
    from post_weight_quantization_group_b200 import build
    build.build()
    lib = q4.load_library()
    ys = (ctypes.c_void_p * 5)(*([A16] * 5))

    def call(ws, n=None, B=1, x=A16):
        arr = (q4._CWeight * len(ws))(*ws)
        return lib.q4_gemv_grouped(arr, len(ws) if n is None else n, x, q4.Q4_BF16, B, ys,
                                   q4.Q4_BF16, A16, 1 << 20, None)

    assert call([_cw()], n=0) == q4.Q4_ERR_INVALID_ARG
    assert call([_cw()] * 5) == q4.Q4_ERR_INVALID_ARG
    assert call([_cw(), _cw(in_=512)]) == q4.Q4_ERR_SHAPE
    assert call([_cw(), _cw(group_size=64)]) == q4.Q4_ERR_SHAPE
    assert call([_cw(), _cw(symmetric=0, zeros=A16)]) == q4.Q4_ERR_SHAPE
    assert call([_cw(), _cw()], B=0) == q4.Q4_ERR_SHAPE
    assert call([_cw(), _cw()], x=None) == q4.Q4_ERR_INVALID_ARG
    assert call([_cw(out=0), _cw(out=0)]) == q4.Q4_OK


def _within(y, y_ref, what):
    y = np.asarray(y, dtype=np.float64)
    rms = float(np.sqrt(np.mean(y_ref ** 2)))
    bound = TOL * (np.abs(y_ref) + rms)
    err = np.abs(y - y_ref)
    assert np.all(err <= bound), f"{what}: worst err/bound {float(np.max(err / bound)):.3f}"


def _sample(out, n, seed):
    if out <= n:
        return np.arange(out, dtype=np.int64)
    rng = np.random.default_rng(seed)
    return np.unique(np.concatenate([[0, out - 1], rng.choice(out, n - 2, replace=False)])).astype(np.int64)


def _group_case(shapes, inn, g, sym, B, xdtype, ydtype=None, seed=0, nrows=160):
    dev = torch.device("cuda:0")
    Ws = [wl.normal_weight(o, inn, seed + i, device=dev) for i, o in enumerate(shapes)]
    ws = [q4.q4_quantize_pack(W, g, sym) for W in Ws]
    x = wl.activations(B, inn, seed + 50, dtype=xdtype, n_outliers=4, outlier_seed=seed + 60,
                       device=dev)
    ys = q4.q4_gemv_grouped(ws, x, y_dtype=ydtype)
    torch.cuda.synchronize()
    assert q4.q4_sync_status() == q4.Q4_OK
    xd = x.float().cpu().numpy().astype(np.float64)
    for i, (W, w, y) in enumerate(zip(Ws, ws, ys)):
        rows = _sample(W.shape[0], nrows, seed + i)
        q_ref, s_ref, z_ref = oracle.quantize_pack(W[torch.as_tensor(rows, device=dev)].float().cpu().numpy(), g, sym)
        y_ref = oracle.gemv(q_ref, s_ref, z_ref, len(rows), inn, g, sym, xd)
        _within(y.float().cpu().numpy()[:, rows], y_ref, f"product {i} ({W.shape[0]}x{inn}) vs oracle")
        # and the single-product entry point on the same weight
        y1 = q4.q4_gemm_skinny(w, x, y_dtype=ydtype)
        torch.cuda.synchronize()
        _within(y.float().cpu().numpy(), y1.double().cpu().numpy(), f"product {i} vs single call")
    return ws, x, ys


@pytest.mark.gpu
@pytest.mark.parametrize("B", [1, 4])
def test_grouped_llama3_8b_qkv_and_gate_up(B):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    s = wl.LLAMA3_8B
    _group_case([s["q_proj"][0], s["k_proj"][0], s["v_proj"][0]], 4096, 128, True, B, torch.bfloat16)
    _group_case([s["gate_proj"][0], s["up_proj"][0]], 4096, 128, True, B, torch.bfloat16, seed=10)


@pytest.mark.gpu
@pytest.mark.parametrize("sym", [True, False])
@pytest.mark.parametrize("g,inn", [(32, 1120), (64, 1216), (128, 1408)])
def test_grouped_ragged(sym, g, inn):
    """300, 1000 and 64 rows: partial row tiles at the seams between products;
    `in` ends in a partial chunk; fp16 activations, fp32 outputs."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    _group_case([300, 1000, 64], inn, g, sym, 5, torch.float16, ydtype=torch.float32, seed=20,
                nrows=1000)


@pytest.mark.gpu
def test_grouped_four_products_deterministic():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    ws, x, ys = _group_case([4096, 1024, 1024, 4096], 4096, 128, True, 2, torch.bfloat16,
                            ydtype=torch.float32, seed=30)
    again = q4.q4_gemv_grouped(ws, x, y_dtype=torch.float32)
    for a, b in zip(ys, again):
        assert torch.equal(a, b)


@pytest.mark.gpu
def test_grouped_skinny_batch():
    """B > 8 runs the tensor-core kernel once per product."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    _group_case([1024, 512], 2048, 128, False, 16, torch.bfloat16, seed=40)
