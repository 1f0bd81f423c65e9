"""Every output row of each product kernel on a Llama-3-70B shape against the
fp64 oracle (the other parity tests sample rows at these sizes): the
small-batch INT4 kernel, the tcgen05 INT4 kernel, the grouped INT4 launch, the
W8A16 kernel, the W4A4 FP4 product and the bf16 reference.  Each side
quantizes W itself (the oracle on the CPU), so every row tile, every stream-K
split and every fix-up of the launch is compared.
"""
import numpy as np
import pytest
import torch

import oracle
import post_weight_quantization_group_b200 as q4
from post_weight_quantization_group_b200 import workloads as wl

TOL = 4e-3


def _within(y, y_ref, what):
    y = np.asarray(y, dtype=np.float64)
    rms = float(np.sqrt(np.mean(y_ref ** 2)))
    bound = TOL * (np.abs(y_ref) + rms)
    err = np.abs(y - y_ref)
    assert np.all(err <= bound), f"{what}: worst err/bound {float(np.max(err / bound)):.3f}"


def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _int4_case(name, B, g, sym, api):
    out, inn = wl.LLAMA3_70B[name]
    W = wl.normal_weight(out, inn, 700 + B, device="cuda")
    x = wl.activations(B, inn, 701, n_outliers=4, outlier_seed=702, device="cuda")
    w = q4.q4_quantize_pack(W, g, sym)
    y = getattr(q4, api)(w, x, y_dtype=torch.float32)
    torch.cuda.synchronize()
    assert q4.q4_sync_status() == q4.Q4_OK
    q, s, z = oracle.quantize_pack(W.float().cpu().numpy(), g, sym)
    y_ref = oracle.gemv(q, s, z, out, inn, g, sym, x.float().cpu().numpy().astype(np.float64))
    _within(y.cpu().numpy(), y_ref, f"{api} {name} B={B} g{g} sym={sym}")


@pytest.mark.gpu
@pytest.mark.parametrize("name,B,g,sym", [("down_proj", 1, 128, True), ("q_proj", 8, 64, False)])
def test_full_rows_small_batch_int4(name, B, g, sym):
    _need_gpu()
    _int4_case(name, B, g, sym, "q4_gemv")


@pytest.mark.gpu
def test_full_rows_tcgen05_int4():
    _need_gpu()
    _int4_case("q_proj", 9, 128, True, "q4_gemm_skinny")


@pytest.mark.gpu
def test_full_rows_grouped_int4():
    """q, k and v of a 70B layer (8192 + 1024 + 1024 rows) in one launch."""
    _need_gpu()
    names = ("q_proj", "k_proj", "v_proj")
    Ws = [wl.normal_weight(wl.LLAMA3_70B[n][0], 8192, 710 + i, device="cuda")
          for i, n in enumerate(names)]
    x = wl.activations(2, 8192, 713, device="cuda")
    ws = [q4.q4_quantize_pack(W, 128, True) for W in Ws]
    ys = q4.q4_gemv_grouped(ws, x, y_dtype=torch.float32)
    torch.cuda.synchronize()
    assert q4.q4_sync_status() == q4.Q4_OK
    xd = x.float().cpu().numpy().astype(np.float64)
    for n, W, y in zip(names, Ws, ys):
        q, s, z = oracle.quantize_pack(W.float().cpu().numpy(), 128, True)
        y_ref = oracle.gemv(q, s, z, W.shape[0], 8192, 128, True, xd)
        _within(y.cpu().numpy(), y_ref, f"grouped {n}")


@pytest.mark.gpu
def test_full_rows_w8a16():
    _need_gpu()
    out, inn = wl.LLAMA3_70B["down_proj"]
    W = wl.normal_weight(out, inn, 720, device="cuda").to(torch.bfloat16)
    x = wl.activations(1, inn, 721, device="cuda")
    w = q4.q8_quantize_per_channel(W)
    y = q4.q8_gemv(w, x, y_dtype=torch.float32)
    torch.cuda.synchronize()
    assert q4.q4_sync_status() == q4.Q4_OK
    qr, sr = oracle.q8_quantize_per_channel(W.float().cpu().numpy())
    y_ref = oracle.q8_gemv(qr, sr, x.float().cpu().numpy().astype(np.float64))
    _within(y.cpu().numpy(), y_ref, "q8_gemv down_proj")


@pytest.mark.gpu
@pytest.mark.parametrize("fmt", ["nvfp4", "mxfp4"])
def test_full_rows_fp4(fmt):
    """8192 x 8192 at B = 2: every row tile, split tile and fix-up."""
    _need_gpu()
    out, inn = wl.LLAMA3_70B["q_proj"]
    wp, wsc = wl.fp4_operand(out, inn, fmt, 730)
    xp, xsc = wl.fp4_operand(2, inn, fmt, 731)
    nv = fmt == "nvfp4"
    wts = float(np.float32(wl.FP4_W_TENSOR_SCALE)) if nv else None
    xts = float(np.float32(wl.FP4_X_TENSOR_SCALE)) if nv else None
    dev = torch.device("cuda:0")
    t = lambda v: None if v is None else torch.tensor([v], dtype=torch.float32, device=dev)  # noqa: E731
    Wg = q4.FP4Weight(wp.to(dev), wsc.to(dev), out, inn, fmt, t(wts))
    Xg = q4.FP4Weight(xp.to(dev), xsc.to(dev), 2, inn, fmt, t(xts))
    y = q4.fp4_gemm(Wg, Xg, y_dtype=torch.float32)
    torch.cuda.synchronize()
    assert q4.q4_sync_status() == q4.Q4_OK
    y_ref = oracle.fp4_gemm(fmt, wp.numpy(), wsc.numpy(), wts, xp.numpy(), xsc.numpy(), xts)
    _within(y.cpu().numpy(), y_ref, f"fp4_gemm {fmt}")


@pytest.mark.gpu
@pytest.mark.parametrize("B", [1, 32])
def test_full_rows_bf16_reference(B):
    _need_gpu()
    out, inn = wl.LLAMA3_70B["down_proj"]
    W = wl.normal_weight(out, inn, 740, device="cuda").to(torch.bfloat16)
    x = wl.activations(B, inn, 741, device="cuda")
    y = q4.bf16_gemv_ref_bw(W, x)
    torch.cuda.synchronize()
    assert q4.q4_sync_status() == q4.Q4_OK
    y_ref = oracle.dense(W.float().cpu().numpy(), x.float().cpu().numpy().astype(np.float64))
    _within(y.float().cpu().numpy(), y_ref, f"bf16_gemv_ref_bw B={B}")
