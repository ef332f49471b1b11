"""GPU parity of the small-batch tensor-core GEMM (qnt_gemm with 3 <= M <= 128
on the 4-bit formats, one pass over the weights) against the CPU oracle.

The shapes are chosen to reach every part of the kernel's pipeline: two
128-row tiles of which the second is ragged (its row-group count is not a
multiple of 16, so part of its codes box lies past the end of the buffer and
reads as zeros), 18 stages of K (more than the deepest shared-memory ring, so
every ring slot and every tensor-memory A slot is reused), every group size
(1, 2 or 4 groups per stage), M on both sides of each multiple of 16 and of the
switch from four accumulators to two (M = 64 / 65), and both activation
types.  Tolerance: 4e-3 * sum_k |dq x| per element, as for every GEMV."""
import numpy as np
import pytest
import torch

from dequant_gemv_rtn_b200 import synth
from oracle import oracle as orc
from tests import gpu_helpers as H

pytestmark = pytest.mark.gpu

FOUR = [orc.INT4, orc.FP4, orc.AFPQ, orc.RAZER]


def _packed(fmt, N, K, g, seed):
    ref = orc.quantize(fmt, synth.llama_like(N, K, seed=seed), g)
    pc, pm = orc.pack(ref)
    return ref, torch.from_numpy(pc).cuda(), torch.from_numpy(pm).cuda()


@pytest.mark.parametrize("fmt", FOUR)
@pytest.mark.parametrize("g", [32, 64, 128])
@pytest.mark.parametrize("M,xdt", [(3, 1), (8, 0), (9, 0), (16, 1), (17, 0), (64, 1), (65, 0), (128, 1)])
def test_gemm_tc_parity(fmt, g, M, xdt):
    N, K = 200, 2304
    ref, pc, pm = _packed(fmt, N, K, g, seed=31 * M + g + fmt)
    Xb = H.to_x_bits(synth.activations(M, K, seed=M + 3 * xdt), xdt)
    yref, aref = orc.gemm(ref, Xb, xdt)
    y = H.run_gemm(fmt, N, K, g, pc, pm, Xb, xdt)
    H.assert_within_tol(y, yref, aref, f"gemm_tc fmt={fmt} g{g} M={M} xdt={xdt}", xdt)


@pytest.mark.parametrize("fmt", [orc.INT4, orc.RAZER])
@pytest.mark.parametrize("N,K,M", [(8, 128, 9), (1, 256, 33), (136, 128, 128), (2056, 384, 20)])
def test_gemm_tc_edges(fmt, N, K, M):
    """One stage of K; a single row (one row group, the rest of the tile past
    the end); a tile plus one row group; 17 tiles with a ragged last one."""
    ref, pc, pm = _packed(fmt, N, K, 128, seed=N + K + M)
    for xdt in (0, 1):
        Xb = H.to_x_bits(synth.activations(M, K, seed=N + xdt), xdt)
        yref, aref = orc.gemm(ref, Xb, xdt)
        y = H.run_gemm(fmt, N, K, 128, pc, pm, Xb, xdt)
        H.assert_within_tol(y, yref, aref, f"gemm_tc edge fmt={fmt} {N}x{K} M={M} xdt={xdt}", xdt)


def test_gemm_tc_rows_are_independent():
    """Each activation row's outputs depend on that row only: a batch whose
    rows are copies of one vector gives that vector's outputs in every row,
    bit for bit (the same MMA columns of the same tiles, the same sums)."""
    N, K, M = 384, 1024, 48
    ref, pc, pm = _packed(orc.INT4, N, K, 128, seed=5)
    x = H.to_x_bits(synth.activations(1, K, seed=6), 1)
    Y = H.run_gemm(orc.INT4, N, K, 128, pc, pm, np.repeat(x, M, axis=0), 1)
    assert np.array_equal(Y, np.repeat(Y[:1], M, axis=0))
    yref, aref = orc.gemm(ref, x, 1)
    H.assert_within_tol(Y[:1], yref, aref, "repeated rows", 1)
