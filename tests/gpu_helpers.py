"""Shared helpers for the GPU parity tests (test infrastructure, not collected).

The GPU side is always driven through the C ABI (dequant_gemv_rtn_b200.qnt);
expected values always come from the CPU oracle on the same seeded inputs.
"""
from __future__ import annotations

import numpy as np
import torch

from oracle import oracle as orc

TOL = 4e-3   # |y - y_ref| <= TOL * sum_k |dq x| per output element


def q():
    from dequant_gemv_rtn_b200 import build
    build.build()
    from dequant_gemv_rtn_b200 import qnt
    return qnt


def dev_bytes(n: int) -> torch.Tensor:
    return torch.zeros(max(int(n), 16), dtype=torch.uint8, device="cuda")


def gpu_quantize(fmt: int, W: torch.Tensor, g: int):
    """Quantize a device fp32 matrix; returns (codes, meta, status) device tensors."""
    Q = q()
    N, K = W.shape
    d = Q.desc(fmt, N, K, g)
    codes = dev_bytes(Q.qnt_codes_bytes(d))
    meta = dev_bytes(Q.qnt_meta_bytes(d))
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    Q.qnt_quantize(d, W, codes, meta, st)
    torch.cuda.synchronize()
    return codes, meta, st


def unpack_rows(fmt, N, K, g, codes: torch.Tensor, meta: torch.Tensor, rows=None) -> orc.Quant:
    """Unpack the GPU's packed buffers with the oracle's own unpacker."""
    pc = codes.cpu().numpy()[: orc.codes_bytes(fmt, N, K)]
    pm = meta.cpu().numpy()[: max(1, orc.meta_bytes(fmt, N, K, g))]
    u = orc.unpack(fmt, N, K, g, pc, pm)
    return u if rows is None else u.rows(rows)


def assert_quant_equal(a: orc.Quant, b: orc.Quant, ctx=""):
    assert np.array_equal(a.codes, b.codes), f"codes differ {ctx}: {np.argwhere(a.codes != b.codes)[:5]}"
    assert np.array_equal(a.s1, b.s1), f"scales differ {ctx}: {np.argwhere(a.s1 != b.s1)[:5]}"
    if a.fmt == orc.AFPQ:
        assert np.array_equal(a.s2, b.s2), f"s- differ {ctx}"
    if a.fmt in (orc.INT4, orc.RAZER):
        assert np.array_equal(a.z, b.z), f"zero/selector differ {ctx}: {np.argwhere(a.z != b.z)[:5]}"


def to_x_bits(X: np.ndarray, xdt: int) -> np.ndarray:
    return orc.f2bf(X) if xdt else orc.f2h(X)


def x_tensor(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(bits.astype(np.uint16).view(np.int16)).cuda()


def y_to_f64(Y: torch.Tensor, xdt: int) -> np.ndarray:
    bits = Y.cpu().view(torch.int16).numpy().view(np.uint16)
    if xdt:
        return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return bits.view(np.float16).astype(np.float64)


def run_gemm(fmt, N, K, g, codes, meta, Xbits: np.ndarray, xdt: int, use_gemv=False) -> np.ndarray:
    Q = q()
    M = Xbits.shape[0]
    d = Q.desc(fmt, N, K, g)
    X = x_tensor(Xbits)
    Y = torch.full((M, N), -1, dtype=torch.int16, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    if use_gemv:
        assert M == 1
        Q.qnt_gemv(d, codes, meta, X, Y, xdt, st)
    else:
        Q.qnt_gemm(d, codes, meta, X, Y, M, xdt, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0, f"device status {int(st.item())}"
    return y_to_f64(Y, xdt)


def assert_within_tol(y, yref, aref, ctx="", xdt=0):
    """|y - y_ref| <= 4e-3 * sum|dq x|, plus half the output type's subnormal
    spacing: below the smallest normal of fp16 (2^-14) the output grid itself is
    coarser than the relative bound, so the best attainable error there is
    half a spacing (2^-25 for fp16, 2^-134 for bf16)."""
    err = np.abs(y - yref)
    bound = TOL * aref + (2.0 ** -134 if xdt else 2.0 ** -25)
    bad = ~(err <= bound)
    assert not bad.any(), (f"{ctx}: {bad.sum()} of {bad.size} outside tolerance; worst ratio "
                           f"{np.max(err / np.maximum(bound, 1e-300)):.3g}; first {np.argwhere(bad)[:3]}")
