"""The B <= 8 product's cluster fix-up, on the edge cases of its partition.

When a product's row tiles times a cluster size S fit the grid, the library
launches row_tiles x S CTAs in clusters of S; the CTAs of a cluster split one
row tile's chunks of K and add their partials through distributed shared
memory.  These shapes are small enough that the device holds every cluster,
so the cluster path is the one that runs; each is checked on every row
against the fp64 oracle:
  * one chunk per CTA (in = 256 S), S = 8, 5 and 3;
  * S not dividing the chunk count, and `in` ending in a partial chunk;
  * ragged row tiles (out not a multiple of 128), every batch size 1..8;
  * a group of products whose ragged tiles meet inside a cluster's reach;
  * two calls give bit-identical results (rank-order reduction).
"""
import numpy as np
import pytest
import torch

import oracle
import post_weight_quantization_group_b200 as q4
from post_weight_quantization_group_b200 import workloads as wl

TOL = 4e-3


def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _within(y, y_ref, what):
    y = np.asarray(y, dtype=np.float64)
    rms = float(np.sqrt(np.mean(y_ref ** 2)))
    bound = TOL * (np.abs(y_ref) + rms)
    err = np.abs(y - y_ref)
    assert np.all(err <= bound), f"{what}: worst err/bound {float(np.max(err / bound)):.3f}"


def _case(out, inn, g, sym, B, xdtype=torch.bfloat16, ydtype=torch.float32, seed=0):
    dev = torch.device("cuda:0")
    W = wl.normal_weight(out, inn, seed, device=dev)
    w = q4.q4_quantize_pack(W, g, sym)
    x = wl.activations(B, inn, seed + 1, dtype=xdtype, n_outliers=2, outlier_seed=seed + 2,
                       device=dev)
    y = q4.q4_gemv(w, x, y_dtype=ydtype)
    torch.cuda.synchronize()
    assert q4.q4_sync_status() == q4.Q4_OK
    q_ref, s_ref, z_ref = oracle.quantize_pack(W.float().cpu().numpy(), g, sym)
    y_ref = oracle.gemv(q_ref, s_ref, z_ref, out, inn, g, sym,
                        x.float().cpu().numpy().astype(np.float64))
    _within(y.float().cpu().numpy(), y_ref, f"{out}x{inn} g{g} sym{sym} B{B}")
    return w, x, y


@pytest.mark.gpu
@pytest.mark.parametrize("out,inn", [(256, 2048), (300, 1280), (130, 768)])
@pytest.mark.parametrize("sym,g", [(True, 128), (False, 32)])
def test_one_chunk_per_cta(out, inn, sym, g):
    """in = 256 S with S = 8, 5, 3: every CTA holds exactly one chunk."""
    _need_gpu()
    _case(out, inn, g, sym, 1, seed=3)


@pytest.mark.gpu
@pytest.mark.parametrize("B", [1, 2, 3, 4, 5, 6, 7, 8])
def test_uneven_split_ragged_tiles(B):
    """1000 rows (7 full tiles and one of 104), in = 3968: 16 chunks, the
    last one half full, over clusters of 8 (two chunks per CTA)."""
    _need_gpu()
    _case(1000, 3968, 64, False, B, xdtype=torch.float16, ydtype=torch.float16, seed=10 + B)


@pytest.mark.gpu
@pytest.mark.parametrize("inn", [2816, 4352])
def test_chunks_not_a_multiple_of_the_cluster(inn):
    """11 and 17 chunks over clusters of 8: ranks hold 1 or 2 (2 or 3) chunks."""
    _need_gpu()
    _case(640, inn, 128, True, 2, seed=20)


@pytest.mark.gpu
def test_grouped_ragged_products_in_clusters():
    _need_gpu()
    dev = torch.device("cuda:0")
    outs, inn, g = [300, 100, 50], 1536, 64
    Ws = [wl.normal_weight(o, inn, 30 + i, device=dev) for i, o in enumerate(outs)]
    ws = [q4.q4_quantize_pack(W, g, True) for W in Ws]
    x = wl.activations(3, inn, 33, device=dev)
    ys = q4.q4_gemv_grouped(ws, x, y_dtype=torch.float32)
    torch.cuda.synchronize()
    assert q4.q4_sync_status() == q4.Q4_OK
    xd = x.float().cpu().numpy().astype(np.float64)
    for i, (W, y) in enumerate(zip(Ws, ys)):
        q_ref, s_ref, z_ref = oracle.quantize_pack(W.float().cpu().numpy(), g, True)
        y_ref = oracle.gemv(q_ref, s_ref, z_ref, outs[i], inn, g, True, xd)
        _within(y.float().cpu().numpy(), y_ref, f"product {i} ({outs[i]}x{inn})")


@pytest.mark.gpu
@pytest.mark.parametrize("out,inn", [(4096, 4096), (4096, 14336), (1024, 4096)])
def test_cluster_shapes_deterministic(out, inn):
    """The 8B o/down/k shapes (cluster fix-up): repeated calls are bit-identical."""
    _need_gpu()
    dev = torch.device("cuda:0")
    w = q4.q4_quantize_pack(wl.normal_weight(out, inn, 40, device=dev), 128, True)
    x = wl.activations(1, inn, 41, device=dev)
    y0 = q4.q4_gemv(w, x, y_dtype=torch.float32)
    for _ in range(3):
        assert torch.equal(q4.q4_gemv(w, x, y_dtype=torch.float32), y0)
    assert q4.q4_sync_status() == q4.Q4_OK
