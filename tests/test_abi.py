"""The C-ABI library: it loads, exports every symbol include/*.h declares, and
rejects bad arguments on the host (before any CUDA call).  CPU only: no call
here launches work or touches device memory."""
import ctypes
import glob
import os
import re

import pytest

import post_weight_quantization_group_b200 as q4
from post_weight_quantization_group_b200 import build as q4build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    q4build.build()
    return q4.load_library()


def _declared_symbols():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        for m in re.finditer(r"^Q4_API\s+[\w\s\*]+?\b(\w+)\s*\(", text, flags=re.M):
            names.add(m.group(1))
    return names


def test_header_declares_the_abi():
    names = _declared_symbols()
    assert {"q4_quantize_pack", "q4_quantize_pack_clip", "q4_dequant", "q4_gemv",
            "q4_gemm_skinny", "bf16_gemv_ref_bw", "q4_sync_status", "q4_status_string"} <= names
    assert names == set(q4.ABI_SYMBOLS)


def test_library_exports_every_declared_symbol(lib):
    for name in _declared_symbols():
        assert hasattr(lib, name), name
        assert ctypes.cast(getattr(lib, name), ctypes.c_void_p).value


def test_library_exports_nothing_else():
    import subprocess
    out = subprocess.run(["nm", "-D", "--defined-only", q4.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = {l.split()[-1] for l in out.splitlines() if " T " in l}
    assert exported == _declared_symbols()


def test_status_strings_and_version(lib):
    assert q4.status_string(q4.Q4_OK) == "Q4_OK"
    assert q4.status_string(q4.Q4_ERR_TIMEOUT) == "Q4_ERR_TIMEOUT"
    assert "sm_100a" in q4.version()


# Fake device addresses: only ever compared, never dereferenced, because each
# call below fails validation before reaching CUDA.
A16 = 0x10000
A2 = 0x10002


def _w(**kw):
    d = dict(qweight=A16, scales=A16, zeros=None, out=64, in_=256, group_size=128, bits=4,
             symmetric=1)
    d.update(kw)
    return q4._CWeight(**d)


def test_quantize_pack_validation(lib):
    f = lib.q4_quantize_pack
    ok = dict(W=A16, dt=q4.Q4_F16, out=8, inn=256, g=128, bits=4, sym=1, q=A16, s=A16, z=None)

    def call(**kw):
        a = dict(ok)
        a.update(kw)
        return f(a["W"], a["dt"], a["out"], a["inn"], a["g"], a["bits"], a["sym"], a["q"],
                 a["s"], a["z"], None)

    assert call(bits=3) == q4.Q4_ERR_UNSUPPORTED
    assert call(dt=q4.Q4_F32) == q4.Q4_ERR_UNSUPPORTED
    assert call(dt=7) == q4.Q4_ERR_INVALID_ARG
    assert call(g=96) == q4.Q4_ERR_SHAPE            # does not divide 256
    assert call(g=3, inn=255) == q4.Q4_ERR_SHAPE    # odd group
    assert call(inn=260, g=130) == q4.Q4_ERR_SHAPE  # in not a multiple of 8
    assert call(out=-1) == q4.Q4_ERR_SHAPE
    assert call(W=None) == q4.Q4_ERR_INVALID_ARG
    assert call(q=None) == q4.Q4_ERR_INVALID_ARG
    assert call(z=A16) == q4.Q4_ERR_INVALID_ARG     # zeros given for symmetric
    assert call(sym=0) == q4.Q4_ERR_INVALID_ARG     # zeros missing for asymmetric
    assert call(sym=2) == q4.Q4_ERR_INVALID_ARG
    assert call(W=A2) == q4.Q4_ERR_ALIGNMENT
    assert call(s=A16 + 1) == q4.Q4_ERR_ALIGNMENT
    assert call(out=0) == q4.Q4_OK                  # empty: nothing to do, nothing launched


def test_product_validation(lib):
    for fn, bmax in ((lib.q4_gemv, 8), (lib.q4_gemm_skinny, 128)):
        def call(w=None, x=A16, xdt=q4.Q4_BF16, B=1, y=A16, ydt=q4.Q4_BF16, ws=None, wsb=0):
            w = w if w is not None else _w()
            return fn(ctypes.byref(w), x, xdt, B, y, ydt, ws, wsb, None)

        assert call(B=0) == q4.Q4_ERR_SHAPE
        assert call(B=bmax + 1) == q4.Q4_ERR_SHAPE
        assert call(w=_w(bits=8)) == q4.Q4_ERR_UNSUPPORTED
        assert call(w=_w(group_size=256)) == q4.Q4_ERR_UNSUPPORTED
        assert call(w=_w(group_size=96)) == q4.Q4_ERR_SHAPE
        assert call(xdt=q4.Q4_F32) == q4.Q4_ERR_UNSUPPORTED
        assert call(xdt=q4.Q4_BF16, ydt=q4.Q4_F16) == q4.Q4_ERR_UNSUPPORTED
        assert call(xdt=9) == q4.Q4_ERR_INVALID_ARG
        assert call(x=None) == q4.Q4_ERR_INVALID_ARG
        assert call(y=None) == q4.Q4_ERR_INVALID_ARG
        assert call(w=_w(qweight=None)) == q4.Q4_ERR_INVALID_ARG
        assert call(w=_w(symmetric=0)) == q4.Q4_ERR_INVALID_ARG   # no zeros
        assert call(w=_w(zeros=A16)) == q4.Q4_ERR_INVALID_ARG     # zeros with symmetric
        assert call(x=A2) == q4.Q4_ERR_ALIGNMENT
        assert call(y=A2) == q4.Q4_ERR_ALIGNMENT
        assert call(w=_w(qweight=A2)) == q4.Q4_ERR_ALIGNMENT
        assert call(w=_w(scales=A16 + 1)) == q4.Q4_ERR_ALIGNMENT
        assert call(w=_w(out=0)) == q4.Q4_OK
        assert call() == q4.Q4_ERR_WORKSPACE            # no workspace given


def test_bf16_reference_and_dequant_validation(lib):
    def f(W=A16, out=64, inn=128, x=A16, B=1, y=A16, ws=A16):
        return lib.bf16_gemv_ref_bw(W, out, inn, x, B, y, ws, 1 << 24, None)

    assert f(inn=100) == q4.Q4_ERR_SHAPE      # in not multiple of 64
    assert f(B=0) == q4.Q4_ERR_SHAPE
    assert f(B=129) == q4.Q4_ERR_SHAPE
    assert f(W=None) == q4.Q4_ERR_INVALID_ARG
    assert f(W=A2) == q4.Q4_ERR_ALIGNMENT
    assert f(y=A16 + 2) == q4.Q4_ERR_ALIGNMENT
    assert f(ws=None) == q4.Q4_ERR_WORKSPACE
    assert f(out=0) == q4.Q4_OK
    assert lib.bf16_ref_workspace_bytes(64, 128, 0) == 0
    assert lib.bf16_ref_workspace_bytes(64, 128, 129) == 0
    assert lib.bf16_ref_workspace_bytes(64, 128, 128) > 0
    d = lib.q4_dequant
    assert d(ctypes.byref(_w()), None, q4.Q4_F32, None) == q4.Q4_ERR_INVALID_ARG
    assert d(ctypes.byref(_w()), A16, 5, None) == q4.Q4_ERR_INVALID_ARG
    assert d(ctypes.byref(_w()), A2, q4.Q4_F32, None) == q4.Q4_ERR_ALIGNMENT
    assert d(None, A16, q4.Q4_F32, None) == q4.Q4_ERR_INVALID_ARG
    assert d(ctypes.byref(_w(bits=2)), A16, q4.Q4_F32, None) == q4.Q4_ERR_UNSUPPORTED


def test_workspace_query(lib):
    assert lib.q4_workspace_bytes(0, 256, 1, 128) == 0
    assert lib.q4_workspace_bytes(64, 0, 1, 128) == 0
    assert lib.q4_workspace_bytes(64, 256, 0, 128) == 0
    assert lib.q4_workspace_bytes(64, 256, 129, 128) == 0


def test_selftest_validation(lib):
    assert lib.q4_selftest_wait_timeout(0, None) == q4.Q4_ERR_INVALID_ARG
    assert lib.q4_selftest_wait_timeout(2_000_000_000, None) == q4.Q4_ERR_INVALID_ARG


def test_product_path_has_no_cpu_fallback(tmp_path, monkeypatch):
    """Without the library the binding raises instead of computing anything."""
    import importlib
    import post_weight_quantization_group_b200 as mod
    saved = mod._lib
    try:
        mod._lib = None
        with pytest.raises(mod.Q4LibraryError):
            mod.load_library(str(tmp_path / "missing.so"))
    finally:
        mod._lib = saved
    src = open(os.path.join(ROOT, "post_weight_quantization_group_b200", "__init__.py")).read()
    assert "import oracle" not in src and "from oracle" not in src


def test_quantize_pack_clip_validation(lib):
    f = lib.q4_quantize_pack_clip
    ok = dict(W=A16, dt=q4.Q4_F16, out=8, inn=256, g=128, n=21, q=A16, s=A16)

    def call(**kw):
        a = dict(ok)
        a.update(kw)
        return f(a["W"], a["dt"], a["out"], a["inn"], a["g"], a["n"], a["q"], a["s"], None)

    assert call(n=0) == q4.Q4_ERR_INVALID_ARG
    assert call(n=65) == q4.Q4_ERR_INVALID_ARG
    assert call(dt=q4.Q4_F32) == q4.Q4_ERR_UNSUPPORTED
    assert call(dt=7) == q4.Q4_ERR_INVALID_ARG
    assert call(g=96) == q4.Q4_ERR_SHAPE            # does not divide 256
    assert call(g=4, inn=256) == q4.Q4_ERR_UNSUPPORTED
    assert call(inn=260, g=130) == q4.Q4_ERR_SHAPE  # in not a multiple of 8
    assert call(out=-1) == q4.Q4_ERR_SHAPE
    assert call(W=None) == q4.Q4_ERR_INVALID_ARG
    assert call(s=None) == q4.Q4_ERR_INVALID_ARG
    assert call(W=A2) == q4.Q4_ERR_ALIGNMENT
    assert call(q=A2) == q4.Q4_ERR_ALIGNMENT
    assert call(out=0) == q4.Q4_OK                  # empty: nothing launched


def test_act_order_validation(lib):
    f = lib.q4_quantize_pack_perm
    ok = dict(W=A16, dt=q4.Q4_F16, out=8, inn=256, g=128, bits=4, sym=1, perm=A16, q=A16, s=A16, z=None)

    def call(**kw):
        a = dict(ok)
        a.update(kw)
        return f(a["W"], a["dt"], a["out"], a["inn"], a["g"], a["bits"], a["sym"], a["perm"],
                 a["q"], a["s"], a["z"], None)

    assert call(perm=None) == q4.Q4_ERR_INVALID_ARG
    assert call(perm=A2) == q4.Q4_ERR_ALIGNMENT
    assert call(bits=8) == q4.Q4_ERR_UNSUPPORTED
    assert call(g=96) == q4.Q4_ERR_SHAPE
    assert call(sym=0) == q4.Q4_ERR_INVALID_ARG      # zeros missing
    assert call(out=0) == q4.Q4_OK
    p = lib.q4_permute_activations
    assert p(A16, q4.Q4_BF16, 2, 100, A16, A16, None) == q4.Q4_ERR_SHAPE
    assert p(A16, q4.Q4_F32, 2, 128, A16, A16, None) == q4.Q4_ERR_UNSUPPORTED
    assert p(None, q4.Q4_BF16, 2, 128, A16, A16, None) == q4.Q4_ERR_INVALID_ARG
    assert p(A16, q4.Q4_BF16, 2, 128, A16, A2, None) == q4.Q4_ERR_ALIGNMENT
    assert p(A16, q4.Q4_BF16, 0, 128, A16, A16, None) == q4.Q4_OK


def test_q8_weight_validation(lib):
    qz = lib.q8_quantize_per_channel
    assert qz(A16, q4.Q4_F32, 8, 256, A16, A16, None) == q4.Q4_ERR_UNSUPPORTED
    assert qz(A16, 7, 8, 256, A16, A16, None) == q4.Q4_ERR_INVALID_ARG
    assert qz(A16, q4.Q4_BF16, 8, 200, A16, A16, None) == q4.Q4_ERR_SHAPE   # in % 16
    assert qz(A16, q4.Q4_BF16, -1, 256, A16, A16, None) == q4.Q4_ERR_SHAPE
    assert qz(A16, q4.Q4_BF16, 0, 256, A16, A16, None) == q4.Q4_OK
    assert qz(None, q4.Q4_BF16, 8, 256, A16, A16, None) == q4.Q4_ERR_INVALID_ARG
    assert qz(A16, q4.Q4_BF16, 8, 256, A2, A16, None) == q4.Q4_ERR_ALIGNMENT
    assert qz(A16, q4.Q4_BF16, 8, 256, A16, A2, None) == q4.Q4_ERR_ALIGNMENT
    dq = lib.q8_dequant
    assert dq(A16, A16, 8, 256, A16, 9, None) == q4.Q4_ERR_INVALID_ARG
    assert dq(A16, A16, 8, 24, A16, q4.Q4_F32, None) == q4.Q4_ERR_SHAPE
    assert dq(A16, A16, 0, 256, A16, q4.Q4_F32, None) == q4.Q4_OK
    assert dq(A16, A16, 8, 256, A2, q4.Q4_F32, None) == q4.Q4_ERR_ALIGNMENT
    g = lib.q8_gemv
    ok = dict(q=A16, s=A16, out=64, inn=256, x=A16, xdt=q4.Q4_BF16, B=1, y=A16, ydt=q4.Q4_BF16,
              ws=None, wsb=0)

    def call(**kw):
        a = dict(ok)
        a.update(kw)
        return g(a["q"], a["s"], a["out"], a["inn"], a["x"], a["xdt"], a["B"], a["y"], a["ydt"],
                 a["ws"], a["wsb"], None)

    assert call() == q4.Q4_ERR_WORKSPACE
    assert call(xdt=q4.Q4_F32) == q4.Q4_ERR_UNSUPPORTED
    assert call(ydt=q4.Q4_F16) == q4.Q4_ERR_UNSUPPORTED   # bf16 x, fp16 y
    assert call(B=0) == q4.Q4_ERR_SHAPE and call(B=9) == q4.Q4_ERR_SHAPE
    assert call(inn=120) == q4.Q4_ERR_SHAPE
    assert call(out=0) == q4.Q4_OK
    assert call(x=None) == q4.Q4_ERR_INVALID_ARG
    assert call(x=A2) == q4.Q4_ERR_ALIGNMENT and call(s=A2) == q4.Q4_ERR_ALIGNMENT
    assert lib.q8_workspace_bytes(64, 256, 9) == 0 and lib.q8_workspace_bytes(0, 256, 1) == 0


def test_kv_cache_validation(lib):
    k8 = lib.kv_quantize_int8
    assert k8(A16, q4.Q4_F32, 4, 128, A16, A16, None) == q4.Q4_ERR_UNSUPPORTED
    assert k8(A16, q4.Q4_F16, 4, 100, A16, A16, None) == q4.Q4_ERR_SHAPE    # head_dim % 8
    assert k8(A16, q4.Q4_F16, 4, 520, A16, A16, None) == q4.Q4_ERR_SHAPE    # > 512
    assert k8(A16, q4.Q4_F16, 0, 128, A16, A16, None) == q4.Q4_OK
    assert k8(A16, q4.Q4_F16, 4, 128, None, A16, None) == q4.Q4_ERR_INVALID_ARG
    assert k8(A2, q4.Q4_F16, 4, 128, A16, A16, None) == q4.Q4_ERR_ALIGNMENT
    d8 = lib.kv_dequant_int8
    assert d8(A16, A16, q4.Q4_BF16, 4, 128, A2, None) == q4.Q4_ERR_ALIGNMENT
    assert d8(A16, A16, q4.Q4_BF16, 4, 4, A16, None) == q4.Q4_ERR_SHAPE
    assert d8(A16, A16, q4.Q4_BF16, 0, 128, A16, None) == q4.Q4_OK
    k4 = lib.kv_quantize_int4
    assert k4(A16, q4.Q4_BF16, 4, 128, 96, A16, A16, None) == q4.Q4_ERR_SHAPE   # 96 does not divide
    assert k4(A16, q4.Q4_BF16, 4, 128, 127, A16, A16, None) == q4.Q4_ERR_SHAPE  # odd group
    assert k4(A16, q4.Q4_BF16, 0, 128, 128, A16, A16, None) == q4.Q4_OK
    assert k4(A16, q4.Q4_BF16, 4, 128, 128, A2, A16, None) == q4.Q4_ERR_ALIGNMENT
    d4 = lib.kv_dequant_int4
    assert d4(A16, A16, 4, 128, 128, None, q4.Q4_F16, None) == q4.Q4_ERR_INVALID_ARG
    assert d4(A16, A16, 4, 128, 96, A16, q4.Q4_F16, None) == q4.Q4_ERR_SHAPE
    assert d4(A16, A16, 0, 128, 128, A16, q4.Q4_F16, None) == q4.Q4_OK


def test_fp4_validation(lib):
    mq = lib.mxfp4_quantize
    assert mq(A16, q4.Q4_F32, 4, 64, A16, A16, None) == q4.Q4_ERR_UNSUPPORTED
    assert mq(A16, q4.Q4_BF16, 4, 48, A16, A16, None) == q4.Q4_ERR_SHAPE      # in % 32
    assert mq(A16, q4.Q4_BF16, 0, 64, A16, A16, None) == q4.Q4_OK
    assert mq(A2, q4.Q4_BF16, 4, 64, A16, A16, None) == q4.Q4_ERR_ALIGNMENT
    assert mq(A16, q4.Q4_BF16, 4, 64, None, A16, None) == q4.Q4_ERR_INVALID_ARG
    nq = lib.nvfp4_quantize
    assert nq(A16, q4.Q4_BF16, 4, 40, A16, A16, A16, None) == q4.Q4_ERR_SHAPE  # in % 16
    assert nq(A16, q4.Q4_BF16, 4, 64, A16, A16, None, None) == q4.Q4_ERR_INVALID_ARG
    assert nq(A16, q4.Q4_BF16, 4, 64, A16, A16, A2, None) == q4.Q4_ERR_ALIGNMENT
    assert nq(A16, q4.Q4_BF16, 0, 64, A16, A16, A16, None) == q4.Q4_OK
    md = lib.mxfp4_dequant
    assert md(A16, A16, 4, 64, A16, 9, None) == q4.Q4_ERR_INVALID_ARG
    assert md(A16, A16, 4, 48, A16, q4.Q4_F32, None) == q4.Q4_ERR_SHAPE
    assert md(A16, A16, 4, 64, A2, q4.Q4_F32, None) == q4.Q4_ERR_ALIGNMENT
    nd = lib.nvfp4_dequant
    assert nd(A16, A16, None, 4, 64, A16, q4.Q4_F32, None) == q4.Q4_ERR_INVALID_ARG
    assert nd(A16, A16, A16, 0, 64, A16, q4.Q4_F32, None) == q4.Q4_OK


def test_c_consumer_compiles_links_and_runs(lib, tmp_path):
    """A plain C99 program built against include/q4.h and linked with
    libq4.so runs its host-side checks (no GPU needed)."""
    import subprocess
    exe = tmp_path / "abi_from_c"
    libdir = os.path.dirname(q4.LIB_PATH)
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
                    os.path.join(ROOT, "tests", "c", "abi_from_c.c"), "-L", libdir, "-l:libq4.so",
                    f"-Wl,-rpath,{libdir}", "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True)
    assert out.returncode == 0, out.stderr
    assert "c abi ok" in out.stdout
