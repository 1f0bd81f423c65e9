"""Parity of the FP4 microscaling quantizers (MXFP4, NVFP4) and their
dequantizations with the CPU oracle, through the C ABI: codes, scale bytes,
the tensor scale and every dequantised value bit-identical.  The oracle
quantizes the same seeded weights itself."""
import numpy as np
import pytest
import torch

import oracle
import post_weight_quantization_group_b200 as q4
from post_weight_quantization_group_b200 import workloads as wl

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from post_weight_quantization_group_b200 import build
    build.build()
    q4.load_library()


def _f32(t):
    return t.detach().cpu().float().numpy()


def _np16(t):
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def _sync_ok():
    torch.cuda.synchronize()
    assert q4.q4_sync_status() == q4.Q4_OK


def _weight(kind, out, inn, seed, dtype):
    if kind == "normal":
        W = wl.normal_weight(out, inn, seed, device="cuda")
    elif kind == "t3":
        W = wl.student_t_weight(out, inn, seed, device="cuda")
    else:
        W = wl.uniform_weight(out, inn, seed, device="cuda")
    return W.to(dtype)


def _check(W, fmt):
    if fmt == "mxfp4":
        w = q4.mxfp4_quantize(W)
        _sync_ok()
        q_ref, s_ref = oracle.mxfp4_quantize(_f32(W))
        deq_ref = oracle.mxfp4_dequant(q_ref, s_ref)
    else:
        w = q4.nvfp4_quantize(W)
        _sync_ok()
        q_ref, s_ref, st_ref = oracle.nvfp4_quantize(_f32(W))
        assert np.float32(w.tensor_scale.item()).view(np.uint32) == np.float32(st_ref).view(np.uint32)
        deq_ref = oracle.nvfp4_dequant(q_ref, s_ref, st_ref)
    assert np.array_equal(w.packed.cpu().numpy(), q_ref)
    assert np.array_equal(w.scales.cpu().numpy(), s_ref)
    return w, deq_ref


SHAPES = [(1, 32), (37, 288), (300, 4096), (129, 1056)]


@pytest.mark.parametrize("fmt", ["mxfp4", "nvfp4"])
@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("kind", ["normal", "t3", "uniform"])
@pytest.mark.parametrize("wdtype", [torch.float16, torch.bfloat16])
def test_fp4_quantize_bit_exact(fmt, shape, kind, wdtype):
    _check(_weight(kind, *shape, seed=5, dtype=wdtype), fmt)


@pytest.mark.parametrize("fmt", ["mxfp4", "nvfp4"])
def test_fp4_special_blocks(fmt):
    W = torch.zeros(6, 128, dtype=torch.float16, device="cuda")
    # amax 4 -> MXFP4 scale 1: exact E2M1 midpoints 0.25 .. 5 and their negatives
    ties = torch.tensor([4.0, 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, -0.25, -0.75, -2.5, -3.5, 0.1, -0.1,
                         -0.0, 5.0, 3.0], dtype=torch.float16, device="cuda")
    W[0, :16] = ties
    W[0, 16:32] = ties * 0.5
    W[1, 32:64] = 0.0                                   # zero blocks
    W[2] = wl.normal_weight(1, 128, 3, device="cuda")[0].to(torch.float16)
    W[2, 7] = 60000.0                                   # a huge outlier
    W[3] = W[2] * 1e-4                                  # tiny values (fp16 subnormals)
    W[4, :] = -1.0
    W[5, ::3] = 7.75                                    # clips at 6 under MXFP4's floor rule
    w, deq_ref = _check(W, fmt)
    got = q4.fp4_dequant(w, torch.float32)
    _sync_ok()
    assert np.array_equal(got.cpu().numpy().view(np.uint32), deq_ref.view(np.uint32))


@pytest.mark.parametrize("fmt", ["mxfp4", "nvfp4"])
@pytest.mark.parametrize("odt", [torch.float32, torch.bfloat16, torch.float16])
def test_fp4_dequant_bit_exact(fmt, odt):
    W = _weight("t3", 77, 1024, 6, torch.bfloat16)
    w, deq_ref = _check(W, fmt)
    got = q4.fp4_dequant(w, odt)
    _sync_ok()
    if odt == torch.float32:
        assert np.array_equal(got.cpu().numpy().view(np.uint32), deq_ref.view(np.uint32))
    elif odt == torch.bfloat16:
        assert np.array_equal(_np16(got), oracle.f32_to_bf16_bits_array(deq_ref))
    else:
        assert np.array_equal(_np16(got), oracle.f32_to_f16_bits_array(deq_ref))


@pytest.mark.parametrize("fmt", ["mxfp4", "nvfp4"])
def test_fp4_full_size_layer(fmt):
    """Llama-3-8B gate_proj 14336 x 4096, N(0, 0.02^2) fp16: every code, scale
    and the tensor scale (NVFP4's depends on the whole matrix)."""
    out, inn = wl.LLAMA3_8B["gate_proj"]
    W = wl.normal_weight(out, inn, 14, device="cuda")
    _check(W, fmt)


def test_fp4_accuracy_ordering():
    """NVFP4's finer blocks and scales give a smaller weight error than
    MXFP4 on Gaussian weights (arganzheng.life section 九.1)."""
    W = wl.normal_weight(512, 4096, 7, device="cuda")
    e_mx = (q4.fp4_dequant(q4.mxfp4_quantize(W)) - W.float()).pow(2).mean().item()
    e_nv = (q4.fp4_dequant(q4.nvfp4_quantize(W)) - W.float()).pow(2).mean().item()
    _sync_ok()
    assert e_nv < e_mx
