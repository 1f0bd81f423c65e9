"""Parity of the CUDA path (through the C ABI) with the CPU oracle.

Codes, scales and zero points must be bit-identical; dequantised weights
bit-identical; products within |y - y_ref| <= 4e-3 * (|y_ref| + rms(y_ref))
of the fp64 oracle.  The oracle always quantizes W itself: no expected value
comes from the GPU.  Full-size layers are checked on sampled rows.
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


def _assert_within(y: np.ndarray, y_ref: np.ndarray, what=""):
    y = np.asarray(y, dtype=np.float64)
    rms = float(np.sqrt(np.mean(y_ref ** 2)))
    bound = TOL * (np.abs(y_ref) + rms)
    err = np.abs(y - y_ref)
    worst = float(np.max(err / bound)) if err.size else 0.0
    assert np.all(err <= bound), f"{what}: worst err/bound = {worst:.3f}"
    return worst


def _sample_rows(out, n, seed=0):
    if out <= n:
        return np.arange(out, dtype=np.int64)
    rng = np.random.default_rng(seed)
    rows = rng.choice(out, size=n - 2, replace=False)
    return np.unique(np.concatenate([[0, out - 1], rows])).astype(np.int64)


def _weight(kind, out, inn, seed, device="cuda"):
    if kind == "normal":
        return wl.normal_weight(out, inn, seed, device=device)
    if kind == "t3":
        return wl.student_t_weight(out, inn, seed, device=device)
    if kind == "uniform":
        return wl.uniform_weight(out, inn, seed, device=device)
    raise ValueError(kind)


def _quant_check(W, g, sym, rows=None):
    """GPU quantize of W (device), oracle quantize of the selected rows."""
    w = q4.q4_quantize_pack(W, g, sym)
    torch.cuda.synchronize()
    assert q4.q4_sync_status() == q4.Q4_OK
    rows_t = None if rows is None else torch.as_tensor(rows, device=W.device)
    Wr = W if rows is None else W[rows_t]
    q_ref, s_ref, z_ref = oracle.quantize_pack(_f32(Wr), g, sym)
    pick = (lambda t: t) if rows is None else (lambda t: t[rows_t])
    assert np.array_equal(pick(w.qweight).cpu().numpy(), q_ref)
    assert np.array_equal(_np16(pick(w.scales)), s_ref)
    if not sym:
        assert np.array_equal(_np16(pick(w.zeros)), z_ref)
    return w, (q_ref, s_ref, z_ref)


# --------------------------------------------------------------- quantize

@pytest.mark.parametrize("out,inn,g", [
    (512, 1024, 128),     # single linear, group 128
    (4, 8, 4),            # the tiny 4x8 group-4 case
    (37, 96, 32), (37, 96, 96), (50, 1216, 64), (33, 4096, 4096), (16, 520, 8), (9, 2560, 256),
])
@pytest.mark.parametrize("sym", [True, False])
@pytest.mark.parametrize("wdtype", [torch.float16, torch.bfloat16])
def test_quantize_pack_bit_exact(out, inn, g, sym, wdtype):
    W = wl.normal_weight(out, inn, 0, device="cuda").to(wdtype)
    _quant_check(W, g, sym)


@pytest.mark.parametrize("sym", [True, False])
def test_quantize_pack_edge_groups(sym):
    W = wl.student_t_weight(24, 512, 3, device="cuda")
    W[0, :128] = 0                        # all-zero group
    W[1, :64] = 0.25                      # constant group
    W[2, 64:128] = W[2, 64:128].abs()     # all-positive group
    W[3, :32] = -W[3, :32].abs()          # all-negative group
    W[4, :32] = 6e-8                      # subnormal fp16 values
    W[5, 32:64] = 60000.0                 # near the fp16 maximum
    W[6, :] = torch.linspace(-1, 1, 512, device="cuda").half()  # many exact ties
    for g in (32, 64, 128):
        _quant_check(W, g, sym)


@pytest.mark.parametrize("shape,kind,g,sym", [
    ((14336, 4096), "normal", 128, True),      # Llama-3-8B gate_proj
    ((4096, 14336), "normal", 128, True),      # Llama-3-8B down_proj
    ((28672, 8192), "t3", 32, True),           # Llama-3-70B gate_proj, heavy tail
    ((8192, 28672), "t3", 128, True),          # Llama-3-70B down_proj, heavy tail
    ((28672, 8192), "normal", 64, False),      # 70B stack: asymmetric group 64
])
def test_quantize_pack_full_size_sampled(shape, kind, g, sym):
    W = _weight(kind, *shape, seed=20)
    _quant_check(W, g, sym, rows=_sample_rows(shape[0], 96))


# ---------------------------------------------------------------- dequant

@pytest.mark.parametrize("sym", [True, False])
@pytest.mark.parametrize("g", [4, 32, 64, 128])
def test_dequant_bit_exact(sym, g):
    out, inn = 40, 1024
    W = wl.normal_weight(out, inn, 5, device="cuda")
    w, (q_ref, s_ref, z_ref) = _quant_check(W, g, sym)
    ref = oracle.dequant(q_ref, s_ref, z_ref, out, inn, g, sym)
    got = q4.q4_dequant(w, torch.float32)
    torch.cuda.synchronize()
    assert np.array_equal(_f32(got).view(np.uint32), ref.view(np.uint32))
    got16 = q4.q4_dequant(w, torch.float16)
    assert np.array_equal(_np16(got16), oracle.f32_to_f16_bits_array(ref))
    gotb = q4.q4_dequant(w, torch.bfloat16)
    assert np.array_equal(_np16(gotb), oracle.f32_to_bf16_bits_array(ref))


# ------------------------------------------------------------------- GEMV

def _gemv_case(out, inn, g, sym, B, xdtype, ydtype=None, kind="normal", seed=1,
               rows=None, n_outliers=0, api="q4_gemv"):
    W = _weight(kind, out, inn, seed)
    x = wl.activations(B, inn, seed + 100, dtype=xdtype, n_outliers=n_outliers,
                       outlier_seed=seed + 200, device="cuda")
    w = q4.q4_quantize_pack(W, g, sym)
    y = getattr(q4, api)(w, x, y_dtype=ydtype)
    torch.cuda.synchronize()
    assert q4.q4_sync_status() == q4.Q4_OK
    rows = np.arange(out) if rows is None else rows
    Wr = W[torch.as_tensor(rows, device="cuda")]
    q_ref, s_ref, z_ref = oracle.quantize_pack(_f32(Wr), g, sym)
    y_ref = oracle.gemv(q_ref, s_ref, z_ref, len(rows), inn, g, sym,
                        x.float().cpu().numpy().astype(np.float64))
    got = y.float().cpu().numpy()[:, rows]
    _assert_within(got, y_ref, f"{out}x{inn} g{g} sym{sym} B{B} {xdtype}")
    return y, w, x


@pytest.mark.parametrize("xdtype", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("sym", [True, False])
@pytest.mark.parametrize("g,inn", [(32, 1120), (64, 1216), (128, 1408)])
@pytest.mark.parametrize("B", [1, 2, 3, 5, 8])
def test_gemv_ragged_tiles(xdtype, sym, g, inn, B):
    # 300 rows = two full 128-row tiles and a ragged third; `in` ends in a
    # partial 256-code chunk
    _gemv_case(300, inn, g, sym, B, xdtype)


def test_gemv_single_linear_fp16():
    """512 x 1024, N(0, 0.02^2) fp16 weights, symmetric group 128, x fp16 [1, 1024]."""
    y, _, _ = _gemv_case(512, 1024, 128, True, 1, torch.float16)
    assert y.dtype == torch.float16


@pytest.mark.parametrize("ydtype", [torch.float32, None])
@pytest.mark.parametrize("shape", [(256, 8192), (4096, 4096), (96, 28672)])
def test_gemv_cluster_split_k(ydtype, shape):
    _gemv_case(*shape, 128, True, 4, torch.bfloat16, ydtype=ydtype)


def test_gemv_output_dtypes_consistent():
    W = wl.normal_weight(700, 2048, 9, device="cuda")
    x = wl.activations(3, 2048, 10, device="cuda")
    w = q4.q4_quantize_pack(W, 128, True)
    y32 = q4.q4_gemv(w, x, y_dtype=torch.float32)
    yb = q4.q4_gemv(w, x)
    assert torch.equal(y32.to(torch.bfloat16), yb)
    # deterministic: the split-K reduction has a fixed order
    assert torch.equal(q4.q4_gemv(w, x, y_dtype=torch.float32), y32)
    # row b of a batched call equals the B = 1 call on that row
    for b in range(3):
        y1 = q4.q4_gemv(w, x[b:b + 1].contiguous(), y_dtype=torch.float32)
        assert torch.equal(y1[0], y32[b])


@pytest.mark.parametrize("name", list(wl.LLAMA3_8B))
def test_gemv_llama3_8b_layer(name):
    out, inn = wl.LLAMA3_8B[name]
    seed = wl.llama3_8b_layer_seeds(0)[name]
    _gemv_case(out, inn, 128, True, 1, torch.bfloat16, seed=seed, rows=_sample_rows(out, 192))


@pytest.mark.parametrize("name", ["q_proj", "gate_proj", "up_proj", "down_proj"])
@pytest.mark.parametrize("g", [32, 128])
@pytest.mark.parametrize("B", [1, 4])
def test_gemv_llama3_70b_heavy_tail(name, g, B):
    out, inn = wl.LLAMA3_70B[name]
    _gemv_case(out, inn, g, True, B, torch.bfloat16, kind="t3", seed=20,
               rows=_sample_rows(out, 128), n_outliers=4)


@pytest.mark.parametrize("layer", [0, 39, 79])
@pytest.mark.parametrize("idx,name", list(enumerate(wl.LLAMA3_70B)))
@pytest.mark.parametrize("B", [1, 8])
def test_gemv_llama3_70b_stack_asym_g64(layer, idx, name, B):
    """The Llama-3-70B decode stack's weights (asymmetric group 64) of the
    first, middle and last layer, generated from the stack's seeds."""
    out, inn = wl.LLAMA3_70B[name]
    _gemv_case(out, inn, 64, False, B, torch.bfloat16, seed=wl.llama3_70b_stack_seed(layer, idx),
               rows=_sample_rows(out, 96, seed=layer))


def test_gemv_special_inputs():
    out, inn = 130, 512
    W = wl.normal_weight(out, inn, 2, device="cuda")
    w = q4.q4_quantize_pack(W, 64, False)
    What = q4.q4_dequant(w, torch.float32)
    # one-hot x returns a column of W_hat exactly (fp32 output)
    for k in (0, 255, 511):
        x = torch.zeros(1, inn, dtype=torch.bfloat16, device="cuda")
        x[0, k] = 1
        y = q4.q4_gemv(w, x, y_dtype=torch.float32)
        assert torch.equal(y[0], What[:, k])
    # scaling x by 2^p scales y by exactly 2^p
    x = wl.activations(2, inn, 3, device="cuda")
    y1 = q4.q4_gemv(w, x, y_dtype=torch.float32)
    y2 = q4.q4_gemv(w, (x.float() * 8).to(torch.bfloat16), y_dtype=torch.float32)
    assert torch.equal(y2, y1 * 8)
    # all-zero x gives zero
    y0 = q4.q4_gemv(w, torch.zeros(4, inn, dtype=torch.bfloat16, device="cuda"))
    assert not y0.any()


def test_gemv_empty_and_bad_alignment():
    w = q4.q4_quantize_pack(wl.normal_weight(64, 256, 1, device="cuda"), 128, True)
    x = wl.activations(1, 257, 1, device="cuda")
    with pytest.raises(q4.Q4Error) as e:
        q4.q4_gemv(w, x[:, 1:])  # contiguous view starting 2 bytes in
    assert e.value.status in (q4.Q4_ERR_ALIGNMENT, q4.Q4_ERR_SHAPE)
    x2 = wl.activations(1, 256, 1, device="cuda")
    w0 = q4.Q4Weight(w.qweight[:0], w.scales[:0], None, 0, 256, 128, True)
    y0 = q4.q4_gemv(w0, x2)
    assert y0.shape == (1, 0)


# ------------------------------------------------------ bf16 reference GEMV

@pytest.mark.parametrize("shape", [(300, 1024), (4096, 4096), (8192, 28672), (14336, 4096),
                                   (200, 1088)])
@pytest.mark.parametrize("B", [1, 4, 8, 9, 16, 33, 64, 128])
def test_bf16_reference(shape, B):
    """Row tiles split between CTAs (8192 x 28672), whole tiles (14336 x
    4096), a ragged row tile and a K tail inside a chunk (200 x 1088), every
    activation tile width."""
    out, inn = shape
    W = wl.normal_weight(out, inn, 30, device="cuda").to(torch.bfloat16)
    x = wl.activations(B, inn, 31, device="cuda")
    y = q4.bf16_gemv_ref_bw(W, x)
    torch.cuda.synchronize()
    assert q4.q4_sync_status() == q4.Q4_OK
    assert torch.equal(q4.bf16_gemv_ref_bw(W, x), y)  # deterministic
    rows = _sample_rows(out, 128)
    Wr = _f32(W[torch.as_tensor(rows, device="cuda")])
    y_ref = oracle.dense(Wr, x.float().cpu().numpy().astype(np.float64))
    _assert_within(y.float().cpu().numpy()[:, rows], y_ref, f"bf16 {shape} B{B}")


# ---------------------------------------------- failure path (no GPU fault)

def test_bounded_wait_reports_timeout_and_context_survives():
    assert q4.q4_sync_status() == q4.Q4_OK
    assert q4.q4_selftest_wait_timeout(2_000_000) == q4.Q4_OK   # 2 ms
    assert q4.q4_sync_status() == q4.Q4_ERR_TIMEOUT
    assert q4.q4_sync_status() == q4.Q4_OK                      # cleared
    _gemv_case(256, 1024, 128, True, 2, torch.bfloat16)          # still usable


WS_COUNTER_BYTES = 65536 * 4  # the workspace starts with one counter per row tile


def test_workspace_contract():
    """Every completed call leaves the workspace's counters (its first
    WS_COUNTER_BYTES, one per 128-row tile) at zero; a short workspace is
    rejected; results do not depend on the buffer's previous contents."""
    W = wl.normal_weight(3000, 4096, 12, device="cuda")
    w = q4.q4_quantize_pack(W, 128, True)
    x = wl.activations(3, 4096, 13, device="cuda")
    need = q4.load_library().q4_workspace_bytes(w.out, w.in_features, 3, 128)
    assert need > 0
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    y1 = q4.q4_gemv(w, x, y_dtype=torch.float32, workspace=ws)
    torch.cuda.synchronize()
    assert not ws[:WS_COUNTER_BYTES].any()
    y2 = q4.q4_gemv(w, x, y_dtype=torch.float32, workspace=ws)
    assert not ws[:WS_COUNTER_BYTES].any()
    assert torch.equal(y1, y2)
    with pytest.raises(q4.Q4Error) as e:
        q4.q4_gemv(w, x, workspace=ws[: need - 256])
    assert e.value.status == q4.Q4_ERR_WORKSPACE


def test_workspace_shared_across_shapes():
    """One buffer serves calls of different shapes in any order: a call with
    few row tiles leaves partial sums where a larger call keeps counters only
    if the layout depended on the shape."""
    big = (28672, 8192)
    need = q4.load_library().q4_workspace_bytes(big[0], big[1], 4, 128)
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    for (out, inn) in [(300, 4096), (4096, 4096), big, (1000, 8192), big]:
        W = wl.normal_weight(out, inn, out, device="cuda")
        w = q4.q4_quantize_pack(W, 128, True)
        x = wl.activations(4, inn, 7, device="cuda")
        y = q4.q4_gemv(w, x, y_dtype=torch.float32, workspace=ws)
        ref = x.float() @ q4.q4_dequant(w, torch.float32).T
        rms = ref.pow(2).mean().sqrt()
        assert torch.all((y - ref).abs() <= 4e-3 * (ref.abs() + rms)), (out, inn)


def test_workspace_shared_across_batches():
    """One buffer, sized for the largest call, serves the small-batch and the
    tensor-core kernels in any order."""
    shapes = [(300, 4096, 4), (4096, 4096, 40), (8192, 8192, 2), (1000, 8192, 128), (4096, 4096, 8)]
    lib = q4.load_library()
    need = max(lib.q4_workspace_bytes(o, i, b, 128) for o, i, b in shapes)
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    for (out, inn, B) in shapes:
        W = wl.normal_weight(out, inn, out + B, device="cuda")
        w = q4.q4_quantize_pack(W, 128, True)
        x = wl.activations(B, inn, 7, device="cuda")
        y = q4.q4_gemm_skinny(w, x, y_dtype=torch.float32, workspace=ws)
        ref = x.float() @ q4.q4_dequant(w, torch.float32).T
        rms = ref.pow(2).mean().sqrt()
        assert torch.all((y - ref).abs() <= 4e-3 * (ref.abs() + rms)), (out, inn, B)
        torch.cuda.synchronize()
        assert not ws[:WS_COUNTER_BYTES].any()


# ------------------------------------------------- skinny GEMM, 9 <= B <= 128

@pytest.mark.parametrize("xdtype", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("sym", [True, False])
@pytest.mark.parametrize("g,inn", [(32, 1120), (64, 1216), (128, 1408)])
@pytest.mark.parametrize("B", [9, 16, 24, 40, 100, 128])
def test_skinny_ragged_tiles(xdtype, sym, g, inn, B):
    # 300 rows = two full 128-row tiles and a ragged third; `in` ends in a
    # partial 256-code chunk; B pads to the 16/32/64/128-wide MMA tiles
    _gemv_case(300, inn, g, sym, B, xdtype, api="q4_gemm_skinny")


@pytest.mark.parametrize("ydtype", [torch.float32, None])
@pytest.mark.parametrize("shape,B", [((4096, 4096), 16), ((256, 8192), 32), ((96, 28672), 64),
                                     ((1024, 4096), 128)])
def test_skinny_split_k(ydtype, shape, B):
    # few row tiles and long K: every tile is split across CTAs
    _gemv_case(*shape, 128, True, B, torch.bfloat16, ydtype=ydtype, api="q4_gemm_skinny")


@pytest.mark.parametrize("name", ["q_proj", "gate_proj", "down_proj"])
@pytest.mark.parametrize("g", [32, 128])
@pytest.mark.parametrize("B", [16, 64, 128])
def test_skinny_llama3_70b_heavy_tail(name, g, B):
    """70B shapes, Student-t(3) weights, 4 outlier activation channels (x20),
    sampled rows against the oracle."""
    out, inn = wl.LLAMA3_70B[name]
    _gemv_case(out, inn, g, True, B, torch.bfloat16, kind="t3", seed=20,
               rows=_sample_rows(out, 96, seed=B), n_outliers=4, api="q4_gemm_skinny")


def test_skinny_consistency():
    """fp32 and bf16 outputs agree, repeated calls are bit-identical, and the
    rows of a batched call agree with the same rows run as a batch of 16."""
    W = wl.normal_weight(700, 2048, 9, device="cuda")
    x = wl.activations(48, 2048, 10, device="cuda")
    w = q4.q4_quantize_pack(W, 64, False)
    y32 = q4.q4_gemm_skinny(w, x, y_dtype=torch.float32)
    yb = q4.q4_gemm_skinny(w, x)
    assert torch.equal(y32.to(torch.bfloat16), yb)
    assert torch.equal(q4.q4_gemm_skinny(w, x, y_dtype=torch.float32), y32)
    y16 = q4.q4_gemm_skinny(w, x[16:32].contiguous(), y_dtype=torch.float32)
    ref = x.float() @ q4.q4_dequant(w, torch.float32).T
    rms = ref.pow(2).mean().sqrt()
    assert torch.all((y16 - y32[16:32]).abs() <= 4e-3 * (ref[16:32].abs() + rms))


# ------------------------------------------- range (clipping) search quantizer

def _codes(qweight: np.ndarray, inn: int) -> np.ndarray:
    """Signed codes [out, in] of a symmetric packed matrix."""
    lo = (qweight & 0xF).astype(np.int32)
    hi = (qweight >> 4).astype(np.int32)
    c = np.stack([lo, hi], axis=-1).reshape(qweight.shape[0], inn)
    return np.where(c >= 8, c - 16, c)


def _clip_check(W, g, n, rows=None):
    """GPU range search against the oracle: each group's scale is one of the
    oracle's minimum-error candidates (ties within the 1e-12 margin may go
    either way) and its codes are bit-exact at that scale."""
    w = q4.q4_quantize_pack_clip(W, g, n)
    torch.cuda.synchronize()
    assert q4.q4_sync_status() == q4.Q4_OK
    rows = np.arange(W.shape[0]) if rows is None else rows
    rows_t = torch.as_tensor(rows, device=W.device)
    Wr = _f32(W[rows_t])
    out, inn = Wr.shape
    G = inn // g
    gq = w.qweight[rows_t].cpu().numpy()
    gs = _np16(w.scales[rows_t])
    q_ref, s_ref, idx = oracle.quantize_pack_clip(Wr, g, n)
    same = gs == s_ref
    # groups where the GPU chose the oracle's scale: codes bit-exact there
    codes_gpu = _codes(gq, inn).reshape(out, G, g)
    codes_ref = _codes(q_ref, inn).reshape(out, G, g)
    assert np.array_equal(codes_gpu[same], codes_ref[same])
    # any other group must be a tie the margin allows, with consistent codes
    for r, j in zip(*np.nonzero(~same)):
        wg = Wr[r, j * g:(j + 1) * g]
        best, err, s16 = oracle.clip_errors(wg, n)
        cand = np.nonzero(s16 == gs[r, j])[0]
        assert cand.size and err[cand].min() <= err[best] * (1 + 1e-9), (r, j)
        sf = np.float32(np.uint16(gs[r, j]).view(np.float16))
        exp = np.clip(np.rint(wg / sf), -7, 7) if sf != 0 else np.zeros(g)
        assert np.array_equal(codes_gpu[r, j], exp.astype(np.int32)), (r, j)
    return w, float(np.mean(same))


@pytest.mark.parametrize("wdtype", [torch.float16, torch.bfloat16])
@pytest.mark.parametrize("kind", ["normal", "t3", "uniform"])
@pytest.mark.parametrize("g", [8, 32, 64, 128, 256])
def test_quantize_clip_parity(wdtype, kind, g):
    W = _weight(kind, 96, 1024, 51).to(wdtype)
    _, agree = _clip_check(W, g, 21)
    assert agree > 0.99


def test_quantize_clip_single_candidate_is_rtn():
    W = wl.student_t_weight(300, 2048, 52, device="cuda")
    a = q4.q4_quantize_pack_clip(W, 128, 1)
    b = q4.q4_quantize_pack(W, 128, True)
    assert torch.equal(a.qweight, b.qweight) and torch.equal(a.scales, b.scales)


@pytest.mark.parametrize("n", [2, 9, 64])
def test_quantize_clip_grid_sizes(n):
    _clip_check(wl.normal_weight(64, 2048, 53 + n, device="cuda"), 128, n)


def test_quantize_clip_full_size_sampled_and_lower_error():
    """70B gate_proj, Student-t(3): sampled rows against the oracle; over the
    whole matrix the range search lowers the weight error against RTN."""
    out, inn = wl.LLAMA3_70B["gate_proj"]
    W = wl.student_t_weight(out, inn, 54, device="cuda")
    w, _ = _clip_check(W, 128, 21, rows=_sample_rows(out, 64, seed=54))
    r = q4.q4_quantize_pack(W, 128, True)
    Wf = W.float()
    mse_clip = (q4.q4_dequant(w) - Wf).pow(2).mean().item()
    mse_rtn = (q4.q4_dequant(r) - Wf).pow(2).mean().item()
    assert mse_clip < 0.9 * mse_rtn


def test_quantize_clip_feeds_the_product():
    W = wl.student_t_weight(700, 2048, 55, device="cuda")
    w = q4.q4_quantize_pack_clip(W, 64, 21)
    x = wl.activations(3, 2048, 56, device="cuda")
    y = q4.q4_gemv(w, x, y_dtype=torch.float32)
    q_np = w.qweight.cpu().numpy()
    s_np = _np16(w.scales)
    y_ref = oracle.gemv(q_np, s_np, None, 700, 2048, 64, True, x.float().cpu().numpy().astype(np.float64))
    _assert_within(y.cpu().numpy(), y_ref, "clip-quantized product")


# ------------------------------------------------------------ act order

def _variance_order(inn, seed):
    """Columns by decreasing variance of synthetic activations with outlier
    channels (desc_act orders by the Hessian diagonal, the input variance)."""
    x = wl.activations(256, inn, seed, n_outliers=8, outlier_seed=seed + 1).float()
    return torch.argsort(x.var(dim=0), descending=True).to(torch.int32)


@pytest.mark.parametrize("order", ["random", "variance"])
@pytest.mark.parametrize("sym", [True, False])
@pytest.mark.parametrize("wdtype", [torch.float16, torch.bfloat16])
@pytest.mark.parametrize("g", [32, 128, 96])
def test_act_order_quantize_bit_exact(order, sym, wdtype, g):
    inn = 1152  # multiple of 32, 96 and 128... and of 8
    inn = 1536 if g == 128 else inn
    W = wl.student_t_weight(200, inn, 71, device="cuda").to(wdtype)
    if order == "random":
        perm = torch.randperm(inn, generator=torch.Generator().manual_seed(72)).to(torch.int32)
    else:
        perm = _variance_order(inn, 73)
    w = q4.q4_quantize_pack_perm(W, perm.cuda(), g, sym)
    torch.cuda.synchronize()
    assert q4.q4_sync_status() == q4.Q4_OK
    q_ref, s_ref, z_ref = oracle.quantize_pack_perm(_f32(W), g, sym, perm.numpy())
    assert np.array_equal(w.qweight.cpu().numpy(), q_ref)
    assert np.array_equal(_np16(w.scales), s_ref)
    if not sym:
        assert np.array_equal(_np16(w.zeros), z_ref)


def test_act_order_identity_and_gather():
    W = wl.normal_weight(128, 1024, 74, device="cuda")
    ident = torch.arange(1024, dtype=torch.int32, device="cuda")
    a = q4.q4_quantize_pack_perm(W, ident, 128, True)
    b = q4.q4_quantize_pack(W, 128, True)
    assert torch.equal(a.qweight, b.qweight) and torch.equal(a.scales, b.scales)
    x = wl.activations(5, 1024, 75, device="cuda")
    perm = torch.randperm(1024, generator=torch.Generator().manual_seed(76)).to(torch.int32).cuda()
    assert torch.equal(q4.q4_permute_activations(x, perm), x[:, perm.long()])


@pytest.mark.parametrize("B", [1, 5, 16, 40])
def test_act_order_product(B):
    out, inn, g = 700, 2048, 128
    W = wl.student_t_weight(out, inn, 77, device="cuda")
    perm = _variance_order(inn, 78)
    w = q4.q4_quantize_pack_perm(W, perm.cuda(), g, True)
    x = wl.activations(B, inn, 79, n_outliers=8, outlier_seed=74, device="cuda")
    y = q4.q4_gemm_act_order(w, x, y_dtype=torch.float32)
    torch.cuda.synchronize()
    assert q4.q4_sync_status() == q4.Q4_OK
    q_ref, s_ref, _ = oracle.quantize_pack_perm(_f32(W), g, True, perm.numpy())
    xn = x.float().cpu().numpy().astype(np.float64)
    y_ref = oracle.gemv(q_ref, s_ref, None, out, inn, g, True, xn[:, perm.numpy()])
    _assert_within(y.cpu().numpy(), y_ref, f"act-order B{B}")


def test_act_order_bad_index_is_reported():
    W = wl.normal_weight(64, 256, 80, device="cuda")
    perm = torch.arange(256, dtype=torch.int32, device="cuda")
    perm[17] = 9999
    q4.q4_quantize_pack_perm(W, perm, 128, True)
    assert q4.q4_sync_status() == q4.Q4_ERR_INVALID_ARG
    assert q4.q4_sync_status() == q4.Q4_OK
    _gemv_case(256, 1024, 128, True, 2, torch.bfloat16)  # still usable


@pytest.mark.parametrize("shape", [(6144, 4096), (28672, 4096)])
def test_gemv_fused_qkv_and_gate_up_shapes(shape):
    """The Llama-3-8B q/k/v and gate/up matrices stored row-concatenated."""
    _gemv_case(*shape, 128, True, 1, torch.bfloat16, seed=40, rows=_sample_rows(shape[0], 160))


@pytest.mark.gpu
def test_skinny_fp16_activation_range_reported():
    """B > 64 takes its activations in fp16: a finite bf16 activation beyond
    fp16's range is reported (Q4_ERR_INVALID_ARG), and the next call with
    in-range activations is clean and correct."""
    W = wl.normal_weight(256, 1024, 50, device="cuda")
    w = q4.q4_quantize_pack(W, 128, True)
    x = wl.activations(80, 1024, 51, device="cuda")
    x_big = x.clone()
    x_big[3, 17] = 1.0e5
    q4.q4_gemm_skinny(w, x_big)
    assert q4.q4_sync_status() == q4.Q4_ERR_INVALID_ARG
    y = q4.q4_gemm_skinny(w, x, y_dtype=torch.float32)
    assert q4.q4_sync_status() == q4.Q4_OK
    q_ref, s_ref, z_ref = oracle.quantize_pack(_f32(W), 128, True)
    y_ref = oracle.gemv(q_ref, s_ref, z_ref, 256, 1024, 128, True,
                        x.float().cpu().numpy().astype(np.float64))
    _assert_within(y.cpu().numpy(), y_ref, "skinny B=80 after a range error")
