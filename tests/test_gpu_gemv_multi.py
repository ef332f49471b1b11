"""GPU parity of qnt_gemm with 2 to 8 activation vectors on the batch-1 tensor-core
kernel (the 4-bit formats, group 128, K a multiple of 1024: the vectors share
every mma.sync, each in its own B column pair; eight vectors use two B operands
per decoded word) against the CPU oracle.

Shapes: one 128-row tile's worth of row groups on 25 CTAs with a ragged count of
rows (200); 1000 rows at K = 4096 (four runs of K per row); 513 row groups, more
than there are SMs, so CTAs hold 3 or 4 row groups.  M = 3 and M = 5 leave
vector slots empty (images of zeros that nothing reads back).  The cases the
launcher does not take (group 32 or 64, K not a multiple of 1024) go to the other
kernels and are checked here too, so every M in 2..4 is covered whatever the
dispatch.  Tolerance: 4e-3 * sum_k |dq x| per element, as for every GEMV."""
import numpy as np
import pytest

from dequant_gemv_rtn_b200 import synth
from oracle import oracle as orc
from tests import gpu_helpers as H

pytestmark = pytest.mark.gpu

import torch  # noqa: E402


def _packed(fmt, N, K, g, seed):
    ref = orc.quantize(fmt, synth.llama_like(N, K, seed=seed), g)
    pc, pm = orc.pack(ref)
    return ref, torch.from_numpy(pc).cuda(), torch.from_numpy(pm).cuda()


@pytest.mark.parametrize("fmt", [orc.INT4, orc.FP4, orc.AFPQ, orc.RAZER])
@pytest.mark.parametrize("N,K", [(200, 2048), (1000, 4096), (4104, 1024)])
@pytest.mark.parametrize("M", [2, 3, 4, 5, 8])
def test_gemv_multi_parity(fmt, N, K, M):
    ref, pc, pm = _packed(fmt, N, K, 128, seed=7 * N + K + M + fmt)
    for xdt in (0, 1):
        Xb = H.to_x_bits(synth.activations(M, K, seed=N + M + xdt), xdt)
        yref, aref = orc.gemm(ref, Xb, xdt)
        y = H.run_gemm(fmt, N, K, 128, pc, pm, Xb, xdt)
        H.assert_within_tol(y, yref, aref, f"gemv multi fmt={fmt} {N}x{K} M={M} xdt={xdt}", xdt)


@pytest.mark.parametrize("fmt,g,K", [(orc.AFPQ, 64, 2048), (orc.INT4, 64, 2048), (orc.RAZER, 128, 2304),
                                     (orc.FP4, 32, 1024), (orc.INT4, 32, 3072)])
@pytest.mark.parametrize("M", [2, 4, 8])
def test_gemv_multi_cases_taken_elsewhere(fmt, g, K, M):
    N = 264
    ref, pc, pm = _packed(fmt, N, K, g, seed=K + g + M)
    Xb = H.to_x_bits(synth.activations(M, K, seed=M), 0)
    yref, aref = orc.gemm(ref, Xb, 0)
    y = H.run_gemm(fmt, N, K, g, pc, pm, Xb, 0)
    H.assert_within_tol(y, yref, aref, f"M={M} fmt={fmt} g{g} K={K}", 0)


@pytest.mark.parametrize("M", [2, 4, 8])
def test_gemv_multi_vectors_are_independent(M):
    """Each vector meets only its own B column pair, so a batch of copies of
    one vector gives that vector's outputs in every row, bit for bit, and a
    vector's outputs do not change when the other vectors do."""
    N, K = 520, 3072
    ref, pc, pm = _packed(orc.INT4, N, K, 128, seed=11)
    x = H.to_x_bits(synth.activations(1, K, seed=12), 1)
    Y = H.run_gemm(orc.INT4, N, K, 128, pc, pm, np.repeat(x, M, axis=0), 1)
    assert np.array_equal(Y, np.repeat(Y[:1], M, axis=0))
    other = H.to_x_bits(synth.activations(M, K, seed=13), 1)
    other[0] = x[0]
    Y2 = H.run_gemm(orc.INT4, N, K, 128, pc, pm, other, 1)
    assert np.array_equal(Y2[0], Y[0])
    yref, aref = orc.gemm(ref, other, 1)
    H.assert_within_tol(Y2, yref, aref, "mixed vectors", 1)
