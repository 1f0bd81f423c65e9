"""q4_gemv_noalloc: q4_gemv with the library's static device scratch.

The file is named to be collected last, so that its GPU test also runs after
every other test in the same process; it must pass alone in a fresh process
too.  The GPU test compares two calls in a row against q4_gemv (the
workspace entry point, itself checked against the oracle elsewhere) and
checks that calls after the first allocate no device memory.
"""
import ctypes

import pytest
import torch

import post_weight_quantization_group_b200 as q4
from post_weight_quantization_group_b200 import workloads as wl

TOL = 4e-3

# Fake device addresses for the host-validation test: each call there fails
# validation (or returns for an empty weight) before any CUDA call.
A16 = 0x10000


def _cw(**kw):
    d = dict(qweight=A16, scales=A16, zeros=None, out=64, in_=256, group_size=128, bits=4,
             symmetric=1)
    d.update(kw)
    return q4._CWeight(**d)


def test_noalloc_host_validation():
    from post_weight_quantization_group_b200 import build
    build.build()
    lib = q4.load_library()
    f = lib.q4_gemv_noalloc

    def call(w=None, x=A16, xdt=q4.Q4_BF16, B=1, y=A16, ydt=q4.Q4_BF16):
        w = w if w is not None else _cw()
        return f(ctypes.byref(w), x, xdt, B, y, ydt, None)

    assert call(B=0) == q4.Q4_ERR_SHAPE
    assert call(B=9) == q4.Q4_ERR_SHAPE
    assert call(w=_cw(group_size=256)) == q4.Q4_ERR_UNSUPPORTED
    assert call(xdt=q4.Q4_F32) == q4.Q4_ERR_UNSUPPORTED
    assert call(x=None) == q4.Q4_ERR_INVALID_ARG
    assert call(w=_cw(symmetric=0)) == q4.Q4_ERR_INVALID_ARG
    assert call(x=A16 + 2) == q4.Q4_ERR_ALIGNMENT
    assert call(w=_cw(out=0)) == q4.Q4_OK


def _within(y, y_ref, what):
    y = y.double().cpu()
    y_ref = y_ref.double().cpu()
    rms = float(torch.sqrt(torch.mean(y_ref ** 2)))
    bound = TOL * (y_ref.abs() + rms)
    err = (y - y_ref).abs()
    assert bool(torch.all(err <= bound)), f"{what}: worst err/bound {float((err / bound).max()):.3f}"


# (out, in, group, symmetric, B, x dtype, y dtype): stream-K partial tiles on
# 4096-row and ragged shapes, both zero-point modes, B = 1 and 8
CASES = [
    (4096, 4096, 128, True, 1, torch.bfloat16, torch.bfloat16),
    (14336, 4096, 128, True, 8, torch.bfloat16, torch.float32),
    (1000, 1408, 64, False, 5, torch.float16, torch.float16),
    (4096, 14336, 32, False, 1, torch.bfloat16, torch.bfloat16),
]


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_two_calls_in_a_row():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from post_weight_quantization_group_b200 import build
    build.build()
    q4.load_library()
    dev = torch.device("cuda:0")
    torch.cuda.set_device(dev)
    setup_done = False
    for i, (out, inn, g, sym, B, xdt, ydt) in enumerate(CASES):
        W = wl.normal_weight(out, inn, 300 + i, device=dev)
        w = q4.q4_quantize_pack(W, g, sym)
        x = wl.activations(B, inn, 400 + i, dtype=xdt, device=dev)
        y_ref = q4.q4_gemv(w, x, y_dtype=ydt)
        ys = [torch.full((B, out), float("nan"), dtype=ydt, device=dev) for _ in range(2)]
        torch.cuda.synchronize()
        free_before = torch.cuda.mem_get_info(dev)[0]
        for y in ys:  # two calls in a row, same stream
            q4.q4_gemv_noalloc(w, x, y=y)
        torch.cuda.synchronize()
        free_after = torch.cuda.mem_get_info(dev)[0]
        assert q4.q4_sync_status() == q4.Q4_OK
        if setup_done:
            assert free_after == free_before, "q4_gemv_noalloc allocated device memory"
        setup_done = True
        for k, y in enumerate(ys):
            _within(y, y_ref, f"case {i} call {k}")
            # the same kernel, plan and fix-up order as q4_gemv: bit for bit
            assert torch.equal(y, y_ref), f"case {i} call {k}: differs from q4_gemv"



@pytest.mark.gpu
def test_noalloc_rezeroes_scratch_after_reported_timeout():
    """After q4_sync_status reports Q4_ERR_TIMEOUT (a bounded wait that ran
    out may leave stream-K counters set), the next call zero-fills the static
    scratch before launching: two calls after a provoked timeout still match
    q4_gemv bit for bit and allocate nothing.  The timeout comes from the
    library's self-test kernel, a bounded wait on a barrier nothing arrives
    on, which ends by itself after 2 ms."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from post_weight_quantization_group_b200 import build
    build.build()
    q4.load_library()
    dev = torch.device("cuda:0")
    torch.cuda.set_device(dev)
    out, inn, g, B = 4096, 4096, 128, 1
    w = q4.q4_quantize_pack(wl.normal_weight(out, inn, 500, device=dev), g, True)
    x = wl.activations(B, inn, 501, device=dev)
    y_ref = q4.q4_gemv(w, x)
    y0 = torch.empty(B, out, dtype=torch.bfloat16, device=dev)
    q4.q4_gemv_noalloc(w, x, y=y0)  # set up (or reuse) the scratch
    assert q4.q4_sync_status() == q4.Q4_OK
    assert torch.equal(y0, y_ref)
    assert q4.q4_selftest_wait_timeout(2_000_000) == q4.Q4_OK
    assert q4.q4_sync_status() == q4.Q4_ERR_TIMEOUT
    ys = [torch.full((B, out), float("nan"), dtype=torch.bfloat16, device=dev) for _ in range(2)]
    torch.cuda.synchronize()
    free_before = torch.cuda.mem_get_info(dev)[0]
    for y in ys:
        q4.q4_gemv_noalloc(w, x, y=y)
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info(dev)[0] == free_before, "q4_gemv_noalloc allocated device memory"
    assert q4.q4_sync_status() == q4.Q4_OK
    for k, y in enumerate(ys):
        assert torch.equal(y, y_ref), f"call {k} after the timeout differs from q4_gemv"
