"""Parity at the full benchmark sizes, through the C ABI, in the launch
configuration the benchmark times.

Weights are drawn on the GPU by the seeded generator (too large to draw on the
host in seconds), quantized by the library, and compared on sampled rows: the
sampled rows of W are copied to the host, quantized by the oracle (codes and
metadata must match bit-exactly) and the oracle's binary64 GEMV/GEMM on those
rows checks the library's outputs element by element.

Shapes: the Llama-7B decode GEMVs (INT4 g128, batch 1), the FP4 / AFPQ / RaZeR
K=4096 N=14336 case (batch 1, 2, 4 and 8), the Llama-70B small-batch GEMMs (INT4
g128, bf16 activations, M = 1..4 and 8..128) and the selective-precision stack (INT8
per-channel down_proj, FP16 lm_head; batch 1 and 16)."""
import numpy as np
import pytest
import torch

from dequant_gemv_rtn_b200 import synth
from oracle import oracle as orc
from tests import gpu_helpers as H

pytestmark = pytest.mark.gpu


def _sample_rows(N, n=40, seed=0):
    rng = np.random.default_rng(seed)
    rows = set(range(4)) | set(range(N - 4, N)) | set(rng.integers(0, N, size=n).tolist())
    return np.array(sorted(rows))


def _check(fmt, N, K, g, Ms, xdt, seed):
    Q = H.q()
    W = synth.llama_like_device(N, K, seed=seed)
    codes, meta, st = H.gpu_quantize(fmt, W, g)
    assert int(st.item()) == 0
    rows = _sample_rows(N, seed=seed)
    Wr = W[torch.from_numpy(rows).cuda()].cpu().numpy()
    del W
    gg = g if fmt in (orc.INT4, orc.FP4, orc.AFPQ, orc.RAZER) else K
    ref = orc.quantize(fmt, Wr, g)
    got = H.unpack_rows(fmt, N, K, gg, codes, meta, rows)
    H.assert_quant_equal(got, ref, f"fmt={fmt} {N}x{K} sampled rows")
    for M in Ms:
        Xb = H.to_x_bits(synth.activations(M, K, seed=seed + M), xdt)
        Y = H.run_gemm(fmt, N, K, gg, codes, meta, Xb, xdt, use_gemv=(M == 1))
        yref, aref = orc.gemm(ref, Xb, xdt)
        H.assert_within_tol(Y[:, rows], yref, aref, f"fmt={fmt} {N}x{K} M={M}", xdt)
        assert np.all(np.isfinite(Y))
    torch.cuda.empty_cache()


@pytest.mark.parametrize("N,K", [(4096, 4096), (11008, 4096), (12288, 4096), (4096, 11008)])
def test_llama7b_decode_int4_g128(N, K):
    _check(orc.INT4, N, K, 128, [1], 0, seed=N + K)


@pytest.mark.parametrize("fmt", [orc.FP4, orc.AFPQ, orc.RAZER])
def test_fp4_family_k4096_n14336(fmt):
    _check(fmt, 14336, 4096, 128, [1, 2, 4, 8], 0, seed=31 + fmt)


@pytest.mark.parametrize("N,K", [(10240, 8192), (28672, 8192), (8192, 28672)])
def test_llama70b_small_batch_int4(N, K):
    # M = 2..4 take the batch-1 kernel with the vectors sharing its MMAs (at
    # K = 8192, N = 28672 with one ring slot per warp), or the tcgen05 GEMM
    # where four activation images do not fit (K = 28672, M = 3, 4)
    _check(orc.INT4, N, K, 128, [1, 2, 3, 4, 8, 16, 32, 64, 128], 1, seed=N ^ K)


def test_selective_precision_stack_modules():
    """The per-module table picks INT8 per-channel for down_proj in layers 0, 1,
    30, 31, FP16 for lm_head, INT4 g128 elsewhere; each picked format runs at
    its Llama-2-7B shape at batch 1 and 16."""
    Q = H.q()
    t = Q.qnt_table_create(Q.QNT_INT4_ASYM, 128)
    for layer in (0, 1, 30, 31):
        t.set(f"layers.{layer}.mlp.down_proj", Q.QNT_INT8_PERCHAN, 0)
    t.set("lm_head", Q.QNT_FP16, 0)
    cases = [("layers.0.mlp.down_proj", 4096, 11008), ("layers.5.mlp.down_proj", 4096, 11008),
             ("layers.31.self_attn.q_proj", 4096, 4096), ("lm_head", 32000, 4096)]
    want = {"layers.0.mlp.down_proj": Q.QNT_INT8_PERCHAN, "layers.5.mlp.down_proj": Q.QNT_INT4_ASYM,
            "layers.31.self_attn.q_proj": Q.QNT_INT4_ASYM, "lm_head": Q.QNT_FP16}
    for i, (name, N, K) in enumerate(cases):
        fmt, g = t.lookup(name)
        assert fmt == want[name]
        _check(fmt, N, K, g if g else K, [1, 16], 0, seed=500 + i)
    t.close()
