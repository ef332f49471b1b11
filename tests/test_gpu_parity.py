"""GPU parity: libqnt (through the C ABI) against the CPU oracle on the same
seeded inputs.  Codes and metadata bit-exact; GEMV / GEMM outputs within
4e-3 * sum_k |dq x| per element.  The GEMV inputs are packed by the oracle, so
no input of a GEMV check comes from the library's own quantizer."""
import numpy as np
import pytest
import torch

from dequant_gemv_rtn_b200 import synth
from oracle import oracle as orc
from tests import gpu_helpers as H

pytestmark = pytest.mark.gpu

FOUR = [orc.INT4, orc.FP4, orc.AFPQ, orc.RAZER]
ALL = FOUR + [orc.INT8, orc.FP16]


def _w(N, K, seed, kind="llama"):
    return synth.outlier_normal(N, K, seed=seed) if kind == "outlier" else synth.llama_like(N, K, seed=seed)


# ------------------------------------------------------------------ quantize, bit-exact
@pytest.mark.parametrize("fmt", ALL)
@pytest.mark.parametrize("N,K,g", [(256, 512, 32), (37, 384, 64), (300, 4224, 128), (5, 128, 32), (1, 256, 128)])
def test_quantize_bit_exact(fmt, N, K, g):
    W = _w(N, K, seed=N + K + fmt, kind="outlier" if g == 32 else "llama")
    codes, meta, st = H.gpu_quantize(fmt, torch.from_numpy(W).cuda(), g)
    assert int(st.item()) == 0
    got = H.unpack_rows(fmt, N, K, g if fmt in FOUR else K, codes, meta)
    ref = orc.quantize(fmt, W, g)
    assert ref.status == 0
    H.assert_quant_equal(got, ref, f"fmt={fmt} {N}x{K} g{g}")


def test_cfg1_tiny_int4_quantize_and_gemv():
    """Tiny INT4 case: W [256, 512] ~ N(0, 0.02^2) with 1% x10 outliers, g = 32,
    x fp16 [1, 512] ~ N(0, 1), seed 0."""
    N, K, g = 256, 512, 32
    W = synth.outlier_normal(N, K, seed=0)
    X = synth.activations(1, K, seed=0)
    codes, meta, st = H.gpu_quantize(orc.INT4, torch.from_numpy(W).cuda(), g)
    ref = orc.quantize(orc.INT4, W, g)
    H.assert_quant_equal(H.unpack_rows(orc.INT4, N, K, g, codes, meta), ref, "cfg1")
    Xb = H.to_x_bits(X, 0)
    yref, aref = orc.gemm(ref, Xb, 0)
    # GEMV on the oracle's packing (independent of the library quantizer) and on the library's
    pc, pm = orc.pack(ref)
    y1 = H.run_gemm(orc.INT4, N, K, g, torch.from_numpy(pc).cuda(), torch.from_numpy(pm).cuda(), Xb, 0, use_gemv=True)
    H.assert_within_tol(y1, yref, aref, "cfg1 gemv (oracle packing)")
    y2 = H.run_gemm(orc.INT4, N, K, g, codes, meta, Xb, 0, use_gemv=True)
    assert np.array_equal(y1, y2)


def test_quantize_edge_groups():
    """Constant, all-zero, one-sided and on-grid groups; a row of exact ties."""
    K, g = 256, 128
    rows = [np.zeros(K), np.full(K, 0.3), -np.abs(synth.llama_like(1, K, seed=3)[0]) - 1e-3,
            np.abs(synth.llama_like(1, K, seed=4)[0]) + 1e-3,
            np.tile(np.array([6, 5, 4.5, 3.5, 2.5, 1.75, 1.25, 0.75, 0.25, 0, -0.25, -0.75, -5, -6, 8, -8]), K // 16) / 64,
            np.tile(np.array([0, 15, 7.5, 3.5, 0.5, 14.5]) / 32.0, K // 6 + 1)[:K] - 0.2]
    W = np.stack(rows).astype(np.float32)
    for fmt in ALL:
        codes, meta, st = H.gpu_quantize(fmt, torch.from_numpy(W).cuda(), g)
        gg = g if fmt in FOUR else K
        got = H.unpack_rows(fmt, W.shape[0], K, gg, codes, meta)
        H.assert_quant_equal(got, orc.quantize(fmt, W, g), f"edge fmt={fmt}")


@pytest.mark.parametrize("fmt", [orc.INT4, orc.INT8])
def test_quantize_ties_and_near_ties(fmt):
    """Integer codes round the quotient w / S to nearest, ties to even.  Groups
    whose scale is exact (S = 1, 1/16) or not (S = fp16(0.1), from a range of
    1.5) hold weights on half-integer quotients and one binary32 ulp to either
    side of them, so that every rounding of the quotient is decided exactly at
    or next to a tie; codes and metadata must equal the oracle's bit for bit."""
    K, g = 256, 128
    rows = []
    for span in (15.0, 15.0 / 16, 1.5):
        if fmt == orc.INT4:   # min 0, max span: S = fp16(span / 15), z = 0
            S = float(np.float16(span / 15))
            ties = [(k + 0.5) * S for k in range(15)]
        else:                 # max |w| = 127 S
            S = float(np.float16(span / 15))
            ties = [(k + 0.5) * S for k in range(-127, 127)]
        t = np.array(ties, dtype=np.float32)
        vals = np.concatenate([t, np.nextafter(t, np.float32(np.inf)), np.nextafter(t, np.float32(-np.inf))])
        row = np.resize(vals, K).astype(np.float32)
        for c in range(0, K, g):   # every group spans the whole range
            if fmt == orc.INT4:
                row[c], row[c + 1] = 0.0, np.float32(span)
            else:
                row[c], row[c + 1] = np.float32(127 * S), np.float32(-127 * S)
        rows.append(row)
    W = np.stack(rows).astype(np.float32)
    codes, meta, st = H.gpu_quantize(fmt, torch.from_numpy(W).cuda(), g)
    assert int(st.item()) == 0
    gg = g if fmt in FOUR else K
    ref = orc.quantize(fmt, W, g)
    H.assert_quant_equal(H.unpack_rows(fmt, W.shape[0], K, gg, codes, meta), ref, f"ties fmt={fmt}")


@pytest.mark.parametrize("fmt", ALL)
def test_quantize_status_codes(fmt):
    K = 256
    W = synth.llama_like(4, K, seed=1)
    W[2, 77] = np.nan
    _, _, st = H.gpu_quantize(fmt, torch.from_numpy(W).cuda(), 128)
    assert int(st.item()) == orc.NONFINITE == orc.quantize(fmt, W, 128).status
    W = synth.llama_like(4, K, seed=1)
    W[1, 3] = 1e9       # scale (or FP16 code) overflows fp16
    _, _, st = H.gpu_quantize(fmt, torch.from_numpy(W).cuda(), 128)
    assert int(st.item()) == orc.RANGE == orc.quantize(fmt, W, 128).status


# ------------------------------------------------------------------ GEMV / GEMM on oracle-packed codes
def _oracle_packed(fmt, N, K, g, seed):
    W = _w(N, K, seed)
    ref = orc.quantize(fmt, W, g)
    pc, pm = orc.pack(ref)
    return ref, torch.from_numpy(pc).cuda(), torch.from_numpy(pm).cuda()


@pytest.mark.parametrize("fmt", ALL)
@pytest.mark.parametrize("N,K,g", [(300, 4224, 128), (37, 384, 64), (64, 512, 32), (1, 128, 128), (149, 8448, 128)])
@pytest.mark.parametrize("xdt", [0, 1])
def test_gemv_parity(fmt, N, K, g, xdt):
    ref, pc, pm = _oracle_packed(fmt, N, K, g, seed=N * 7 + fmt)
    Xb = H.to_x_bits(synth.activations(1, K, seed=fmt + xdt), xdt)
    yref, aref = orc.gemm(ref, Xb, xdt)
    y = H.run_gemm(fmt, N, K, g if fmt in FOUR else K, pc, pm, Xb, xdt, use_gemv=True)
    H.assert_within_tol(y, yref, aref, f"gemv fmt={fmt} {N}x{K} g{g} xdt={xdt}", xdt)


@pytest.mark.parametrize("fmt", ALL)
@pytest.mark.parametrize("M", [2, 3, 4, 8, 16, 33])
def test_gemm_parity(fmt, M):
    N, K, g = 160, 1024, 128
    ref, pc, pm = _oracle_packed(fmt, N, K, g, seed=M + fmt)
    xdt = M % 2
    Xb = H.to_x_bits(synth.activations(M, K, seed=M), xdt)
    yref, aref = orc.gemm(ref, Xb, xdt)
    y = H.run_gemm(fmt, N, K, g if fmt in FOUR else K, pc, pm, Xb, xdt)
    H.assert_within_tol(y, yref, aref, f"gemm fmt={fmt} M={M}", xdt)


@pytest.mark.parametrize("fmt", [orc.INT4, orc.RAZER, orc.FP16])
def test_gemv_extreme_activations(fmt):
    """Activation magnitudes far outside N(0,1): fp16 near its max, bf16 beyond
    the fp16 range and tiny bf16 values; zero rows give exactly zero."""
    N, K, g = 64, 1024, 128
    W = synth.llama_like(N, K, seed=5)
    W[7] = 0.0
    ref = orc.quantize(fmt, W, g)
    pc, pm = orc.pack(ref)
    pc, pm = torch.from_numpy(pc).cuda(), torch.from_numpy(pm).cuda()
    base = synth.activations(1, K, seed=9)
    for xdt, scale in [(0, 3000.0), (1, 1e6), (1, 1e-30), (0, 1e-6)]:
        Xb = H.to_x_bits(base * scale, xdt)
        yref, aref = orc.gemm(ref, Xb, xdt)
        y = H.run_gemm(fmt, N, K, g if fmt != orc.FP16 else K, pc, pm, Xb, xdt, use_gemv=True)
        H.assert_within_tol(y, yref, aref, f"extreme fmt={fmt} xdt={xdt} scale={scale}", xdt)
        assert y[0, 7] == 0.0


def test_gemv_one_hot_returns_dequantized_column():
    N, K, g = 96, 512, 64
    ref, pc, pm = _oracle_packed(orc.INT4, N, K, g, seed=2)
    D = orc.dequant(ref)
    for k in (0, 63, 64, 300, 511):
        x = np.zeros((1, K), np.float32)
        x[0, k] = 1.0
        y = H.run_gemm(orc.INT4, N, K, g, pc, pm, H.to_x_bits(x, 0), 0, use_gemv=True)
        assert np.array_equal(y[0], D[:, k].astype(np.float16).astype(np.float64))


def test_gemm_rows_equal_gemv():
    N, K, g = 128, 2048, 128
    ref, pc, pm = _oracle_packed(orc.FP4, N, K, g, seed=4)
    Xb = H.to_x_bits(synth.activations(4, K, seed=4), 0)
    Y = H.run_gemm(orc.FP4, N, K, g, pc, pm, Xb, 0)
    yref, aref = orc.gemm(ref, Xb, 0)
    H.assert_within_tol(Y, yref, aref, "batched")
    for m in range(4):
        y = H.run_gemm(orc.FP4, N, K, g, pc, pm, Xb[m:m + 1], 0, use_gemv=True)
        H.assert_within_tol(y[0], yref[m], aref[m], f"row {m}")


@pytest.mark.parametrize("fmt,M", [(orc.INT8, 1), (orc.FP16, 1), (orc.INT8, 3), (orc.INT4, 1), (orc.INT4, 2),
                                   (orc.INT4, 16), (orc.RAZER, 2), (orc.FP4, 4), (orc.AFPQ, 2)])
def test_largest_k_every_path(fmt, M):
    """K = QNT_MAX_GEMV_K on every kernel a call can take (the batch-1 kernel
    with one vector and with two sharing its MMAs, the CUDA-core kernel, the
    tcgen05 GEMM, which takes four vectors here since four images do not fit
    next to a ring): the activations fit in shared memory next to each
    kernel's weight ring."""
    Q = H.q()
    N, K, g = 72, Q.QNT_MAX_GEMV_K, 128
    ref, pc, pm = _oracle_packed(fmt, N, K, g, seed=K + fmt + M)
    xdt = M % 2
    Xb = H.to_x_bits(synth.activations(M, K, seed=M + 11), xdt)
    yref, aref = orc.gemm(ref, Xb, xdt)
    y = H.run_gemm(fmt, N, K, g if fmt in FOUR else K, pc, pm, Xb, xdt, use_gemv=(M == 1))
    H.assert_within_tol(y, yref, aref, f"largest K fmt={fmt} M={M}", xdt)
