"""Parity of the per-channel INT8 weight path (quantizer, dequantization,
W8A16 product) and of the INT8 / INT4 KV-cache quantizers with the CPU
oracle, through the C ABI.

Codes and scales bit-identical; dequantised values bit-identical; products
within |y - y_ref| <= 4e-3 * (|y_ref| + rms(y_ref)) of the fp64 oracle.  The
oracle quantizes the inputs itself: no expected value comes from the GPU.
"""
import numpy as np
import pytest
import torch

import oracle
import post_weight_quantization_group_b200 as q4
from post_weight_quantization_group_b200 import workloads as wl

pytestmark = pytest.mark.gpu

TOL = 4e-3


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from post_weight_quantization_group_b200 import build
    build.build()
    q4.load_library()


def _np16(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def _f32(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().float().numpy()


def _assert_within(y, y_ref, what=""):
    y = np.asarray(y, dtype=np.float64)
    rms = float(np.sqrt(np.mean(y_ref ** 2)))
    bound = TOL * (np.abs(y_ref) + rms)
    err = np.abs(y - y_ref)
    worst = float(np.max(err / bound)) if err.size else 0.0
    assert np.all(err <= bound), f"{what}: worst err/bound = {worst:.3f}"


def _sample_rows(out, n, seed=0):
    if out <= n:
        return np.arange(out, dtype=np.int64)
    rng = np.random.default_rng(seed)
    rows = rng.choice(out, size=n - 2, replace=False)
    return np.unique(np.concatenate([[0, out - 1], rows])).astype(np.int64)


def _weight(kind, out, inn, seed, dtype=torch.bfloat16):
    if kind == "normal":
        W = wl.normal_weight(out, inn, seed, device="cuda")
    elif kind == "t3":
        W = wl.student_t_weight(out, inn, seed, device="cuda")
    else:
        W = wl.uniform_weight(out, inn, seed, device="cuda")
    return W.to(dtype)


def _sync_ok():
    torch.cuda.synchronize()
    assert q4.q4_sync_status() == q4.Q4_OK


# ------------------------------------------------------ INT8 weights

def _q8_check(W, rows=None):
    w = q4.q8_quantize_per_channel(W)
    _sync_ok()
    rt = None if rows is None else torch.as_tensor(rows, device=W.device)
    Wr = W if rows is None else W[rt]
    q_ref, s_ref = oracle.q8_quantize_per_channel(_f32(Wr))
    pick = (lambda t: t) if rows is None else (lambda t: t[rt])
    assert np.array_equal(pick(w.qweight).cpu().numpy(), q_ref)
    assert np.array_equal(pick(w.scales).cpu().numpy().view(np.uint32), s_ref.view(np.uint32))
    return w, q_ref, s_ref


@pytest.mark.parametrize("shape", [(1, 16), (37, 272), (300, 4096), (129, 1040)])
@pytest.mark.parametrize("kind", ["normal", "t3"])
@pytest.mark.parametrize("wdtype", [torch.float16, torch.bfloat16])
def test_q8_quantize_bit_exact(shape, kind, wdtype):
    _q8_check(_weight(kind, *shape, seed=3, dtype=wdtype))


def test_q8_quantize_special_rows():
    W = torch.zeros(6, 256, dtype=torch.float16, device="cuda")
    W[1, 5] = 1e-7                                    # below the eps floor
    W[2] = torch.arange(256, device="cuda").to(torch.float16) * 0.5 - 63.5  # amax 64: ties
    W[3, :] = 127.0                                   # scale exactly 1
    W[3, 1::2] = -2.5
    W[4] = wl.normal_weight(1, 256, 5, device="cuda")[0].to(torch.float16)
    W[4, 17] = 60000.0                                # one huge outlier in the row
    W[5] = -W[4]
    _q8_check(W)


@pytest.mark.parametrize("odt", [torch.float32, torch.bfloat16, torch.float16])
def test_q8_dequant_bit_exact(odt):
    W = _weight("t3", 77, 528, 4)
    w, q_ref, s_ref = _q8_check(W)
    got = q4.q8_dequant(w, odt)
    _sync_ok()
    ref = oracle.q8_dequant(q_ref, s_ref)
    if odt == torch.float32:
        assert np.array_equal(got.cpu().numpy().view(np.uint32), ref.view(np.uint32))
    elif odt == torch.bfloat16:
        assert np.array_equal(_np16(got), oracle.f32_to_bf16_bits_array(ref))
    else:
        assert np.array_equal(_np16(got), oracle.f32_to_f16_bits_array(ref))


def _q8_gemv_case(out, inn, B, xdtype, ydtype=None, kind="normal", seed=1, rows=None,
                  n_outliers=0):
    W = _weight(kind, out, inn, seed, dtype=xdtype)
    x = wl.activations(B, inn, seed + 100, dtype=xdtype, n_outliers=n_outliers,
                       outlier_seed=seed + 200, device="cuda")
    w = q4.q8_quantize_per_channel(W)
    y = q4.q8_gemv(w, x, y_dtype=ydtype)
    _sync_ok()
    rows = np.arange(out) if rows is None else rows
    q_ref, s_ref = oracle.q8_quantize_per_channel(_f32(W[torch.as_tensor(rows, device="cuda")]))
    y_ref = oracle.q8_gemv(q_ref, s_ref, x.float().cpu().numpy().astype(np.float64))
    _assert_within(y.float().cpu().numpy()[:, rows], y_ref, f"q8 {out}x{inn} B{B} {xdtype}")
    return y, w, x


@pytest.mark.parametrize("xdtype", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("inn", [16, 80, 128, 1040, 1104, 1152])
@pytest.mark.parametrize("B", [1, 2, 3, 5, 8])
def test_q8_gemv_ragged_tiles(xdtype, inn, B):
    # 300 rows: two full 128-row tiles and a ragged third; `in` ends inside
    # the first (16, 1040) or second (80, 1104) 64-code half of a chunk, or
    # on a chunk boundary (128, 1152)
    _q8_gemv_case(300, inn, B, xdtype)


@pytest.mark.parametrize("ydtype", [torch.float32, None])
@pytest.mark.parametrize("shape", [(256, 8192), (4096, 4096), (96, 28672), (8, 16)])
def test_q8_gemv_stream_k(ydtype, shape):
    _q8_gemv_case(*shape, 4, torch.bfloat16, ydtype=ydtype)


@pytest.mark.parametrize("name", ["q_proj", "k_proj", "gate_proj", "down_proj"])
@pytest.mark.parametrize("B", [1, 8])
def test_q8_gemv_llama3_70b(name, B):
    out, inn = wl.LLAMA3_70B[name]
    _q8_gemv_case(out, inn, B, torch.bfloat16, kind="t3", seed=30, rows=_sample_rows(out, 128),
                  n_outliers=4)


def test_q8_gemv_special_inputs():
    out, inn = 130, 512
    W = _weight("normal", out, inn, 2)
    w = q4.q8_quantize_per_channel(W)
    What = q4.q8_dequant(w, torch.float32)
    # one-hot x returns a column of W_hat exactly: s * q is one fp32 product
    for k in (0, 255, 511):
        x = torch.zeros(1, inn, dtype=torch.bfloat16, device="cuda")
        x[0, k] = 1
        y = q4.q8_gemv(w, x, y_dtype=torch.float32)
        assert torch.equal(y[0], What[:, k])
    x = wl.activations(2, inn, 3, device="cuda")
    y1 = q4.q8_gemv(w, x, y_dtype=torch.float32)
    y2 = q4.q8_gemv(w, (x.float() * 8).to(torch.bfloat16), y_dtype=torch.float32)
    assert torch.equal(y2, y1 * 8)
    assert not q4.q8_gemv(w, torch.zeros(4, inn, dtype=torch.bfloat16, device="cuda")).any()
    _sync_ok()


def test_q8_gemv_deterministic_and_batch_rows():
    W = _weight("normal", 700, 2048, 9)
    x = wl.activations(3, 2048, 10, device="cuda")
    w = q4.q8_quantize_per_channel(W)
    y32 = q4.q8_gemv(w, x, y_dtype=torch.float32)
    assert torch.equal(q4.q8_gemv(w, x).float(), y32.to(torch.bfloat16).float())
    assert torch.equal(q4.q8_gemv(w, x, y_dtype=torch.float32), y32)
    for b in range(3):
        assert torch.equal(q4.q8_gemv(w, x[b:b + 1].contiguous(), y_dtype=torch.float32)[0], y32[b])
    _sync_ok()


def test_q8_and_q4_share_one_workspace():
    W = _weight("normal", 1000, 4096, 12)
    x = wl.activations(5, 4096, 13, device="cuda")
    w8 = q4.q8_quantize_per_channel(W)
    w4 = q4.q4_quantize_pack(W, 128, True)
    need = max(int(q4.load_library().q8_workspace_bytes(1000, 4096, 5)),
               int(q4.load_library().q4_workspace_bytes(1000, 4096, 5, 128)))
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    a8 = q4.q8_gemv(w8, x, y_dtype=torch.float32, workspace=ws)
    a4 = q4.q4_gemv(w4, x, y_dtype=torch.float32, workspace=ws)
    b8 = q4.q8_gemv(w8, x, y_dtype=torch.float32, workspace=ws)
    b4 = q4.q4_gemv(w4, x, y_dtype=torch.float32, workspace=ws)
    _sync_ok()
    assert torch.equal(a8, b8) and torch.equal(a4, b4)
    assert not ws[:65536 * 4].any()      # every counter is zero again


def test_q8_empty_and_bad_shapes():
    w = q4.q8_quantize_per_channel(_weight("normal", 64, 256, 1))
    w0 = q4.Q8Weight(w.qweight[:0], w.scales[:0], 0, 256)
    assert q4.q8_gemv(w0, wl.activations(1, 256, 1, device="cuda")).shape == (1, 0)
    with pytest.raises(q4.Q4Error) as e:
        q4.q8_gemv(w, wl.activations(9, 256, 1, device="cuda"))
    assert e.value.status == q4.Q4_ERR_SHAPE
    _sync_ok()


# ------------------------------------------------------- INT8 KV cache

KV_SHAPES = [(1, 8, 1, 128), (2, 8, 333, 128), (1, 4, 17, 64), (1, 2, 5, 256), (1, 1, 3, 512),
             (1, 2, 7, 8), (1, 2, 7, 80), (3, 1, 1, 96)]


@pytest.mark.parametrize("shape", KV_SHAPES)
@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
def test_kv8_bit_exact(shape, dtype):
    kv = wl.kv_cache(*shape, seed=7, dtype=dtype, device="cuda")
    if shape[2] > 2:
        kv[0, 0, 2] = 0                 # an all-zero token
    codes, scales = q4.kv_quantize_int8(kv)
    deq = q4.kv_dequant_int8(codes, scales)
    _sync_ok()
    is_bf16 = dtype == torch.bfloat16
    c_ref, s_ref = oracle.kv_quantize_int8(_f32(kv), is_bf16)
    assert np.array_equal(codes.cpu().numpy(), c_ref)
    assert np.array_equal(_np16(scales), s_ref)
    assert np.array_equal(_np16(deq), oracle.kv_dequant_int8(c_ref, s_ref, is_bf16))


def test_kv8_llama3_70b_layer_cache_32k():
    """One layer's K cache of Llama-3-70B at 32768 tokens: [1, 8, 32768, 128] bf16."""
    kv = wl.kv_cache(1, wl.LLAMA3_70B_KV_HEADS, 32768, wl.LLAMA3_70B_HEAD_DIM, seed=8,
                     dtype=torch.bfloat16, device="cuda")
    codes, scales = q4.kv_quantize_int8(kv)
    deq = q4.kv_dequant_int8(codes, scales)
    _sync_ok()
    c_ref, s_ref = oracle.kv_quantize_int8(_f32(kv), True)
    assert np.array_equal(codes.cpu().numpy(), c_ref)
    assert np.array_equal(_np16(scales), s_ref)
    assert np.array_equal(_np16(deq), oracle.kv_dequant_int8(c_ref, s_ref, True))


# ------------------------------------------------------- INT4 KV cache

@pytest.mark.parametrize("shape,g", [((2, 8, 65, 128), 128), ((2, 8, 65, 128), 64),
                                     ((1, 4, 9, 128), 32), ((1, 2, 3, 64), 64), ((1, 2, 5, 96), 32)])
@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
def test_kv4_bit_exact(shape, g, dtype):
    kv = wl.kv_cache(*shape, seed=9, dtype=dtype, device="cuda")
    kv[0, 0, 1, :g] = 0                 # an all-zero group
    packed, scales = q4.kv_quantize_int4(kv, g)
    deq = q4.kv_dequant_int4(packed, scales, g, torch.float32)
    _sync_ok()
    p_ref, s_ref = oracle.kv_quantize_int4(_f32(kv), g)
    assert np.array_equal(packed.cpu().numpy(), p_ref)
    assert np.array_equal(_np16(scales), s_ref)
    d = shape[-1]
    ref = oracle.dequant(p_ref.reshape(-1, d // 2), s_ref.reshape(-1, d // g), None,
                         p_ref.size * 2 // d, d, g, True)
    assert np.array_equal(deq.reshape(-1, d).cpu().numpy().view(np.uint32), ref.view(np.uint32))
