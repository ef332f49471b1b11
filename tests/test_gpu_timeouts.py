"""Bounded waits that expire, on the GPU, without a fault.

Every wait in the kernels has a time limit, after which the kernel reports
QNT_ERR_TIMEOUT through d_status, stops issuing work, lets every copy it issued
land and returns, so the context stays usable.  To make a wait expire, these
tests load the test build of the library (libqnt_test.so: the same sources with
fault injection compiled in; the product library has none):
  * a sequence in which CTA 0 never reports step 0 complete (a completion flag
    that nothing sets): with a 50 ms limit, every CTA's wait for step 0 gives up;
  * a tcgen05 GEMM in which one decode warp of CTA 0 never reports its first
    stage decoded: the MMA issuers' wait gives up, and the kernel must still
    free its tensor memory (the next GEMM allocates all of it).
In both, the call must return and report QNT_ERR_TIMEOUT, and the next ordinary
call on the same stream must be correct.
"""
import ctypes
import time

import numpy as np
import pytest
import torch

from dequant_gemv_rtn_b200 import synth
from oracle import oracle as orc
from tests import gpu_helpers as H

pytestmark = pytest.mark.gpu


def _test_lib(Q):
    from dequant_gemv_rtn_b200 import build
    lib = ctypes.CDLL(build.build(test=True))
    f = lib.qnt_test_gemv_seq_fault
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.POINTER(Q.qnt_seq_step), ctypes.c_int, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p,
                  ctypes.c_void_p, ctypes.c_int, ctypes.c_ulonglong]
    return f


def test_sequence_dependency_wait_expires_and_next_call_is_correct():
    Q = H.q()
    fault_call = _test_lib(Q)
    fmt, g, xdt = orc.INT4, 128, 0
    shapes = [(1024, 512), (768, 1024), (512, 768)]          # x of step i+1 = start of y of step i
    mats = []
    for i, (N, K) in enumerate(shapes):
        ref = orc.quantize(fmt, synth.llama_like(N, K, seed=60 + i), g)
        pc, pm = orc.pack(ref)
        mats.append((ref, torch.from_numpy(pc).cuda(), torch.from_numpy(pm).cuda()))
    x0 = H.x_tensor(H.to_x_bits(synth.activations(1, shapes[0][1], seed=6), xdt))
    ys = [torch.zeros(N, dtype=torch.int16, device="cuda") for N, _ in shapes]
    xs = [x0] + [ys[i][:shapes[i + 1][1]] for i in range(len(shapes) - 1)]
    steps = Q.seq_steps([(Q.desc(fmt, N, K, g), pc, pm, x, y, 1 if i else 0)
                         for i, ((ref, pc, pm), x, y, (N, K)) in enumerate(zip(mats, xs, ys, shapes))])
    work = H.dev_bytes(Q.qnt_gemv_seq_work_bytes(len(shapes)))
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    torch.cuda.synchronize()

    t0 = time.time()
    rc = fault_call(steps, len(shapes), xdt, work.data_ptr(), st.data_ptr(), stream, 1, 50_000_000)
    assert rc == Q.QNT_OK
    torch.cuda.synchronize()
    dt = time.time() - t0
    assert int(st.item()) == Q.QNT_ERR_TIMEOUT
    assert 0.05 <= dt < 10.0, dt

    # the same stream, the product library, fresh status: a correct result
    st.zero_()
    for y in ys:
        y.fill_(0x7E00)
    Q.qnt_gemv_seq(steps, xdt, work, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    for i, ((ref, _, _), x, y) in enumerate(zip(mats, xs, ys)):
        xb = x.cpu().view(torch.int16).numpy().view(np.uint16)[None, :]
        yref, aref = orc.gemm(ref, xb, xdt)
        H.assert_within_tol(H.y_to_f64(y[None, :], xdt), yref, aref, f"after the timeout, step {i}", xdt)

    # and the test build itself with no fault injected
    st.zero_()
    assert fault_call(steps, len(shapes), xdt, work.data_ptr(), st.data_ptr(), stream, 0, 2_000_000_000) == 0
    torch.cuda.synchronize()
    assert int(st.item()) == 0


def test_gemm_tc_wait_expires_frees_tensor_memory_and_next_call_is_correct():
    """The tcgen05 GEMM: in CTA 0 one decode warp never reports stage 0
    decoded, so the MMA issuers' wait for it expires (50 ms limit).  The call
    returns and reports QNT_ERR_TIMEOUT; the kernel has freed its tensor memory
    and let its copies land, so the next GEMMs on the same stream (which
    allocate all of it on their SMs) run and are correct: the product library,
    then the test build with no fault."""
    Q = H.q()
    from dequant_gemv_rtn_b200 import build
    lib = ctypes.CDLL(build.build(test=True))
    f = lib.qnt_test_gemm_fault
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.POINTER(Q.qnt_desc), ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                  ctypes.c_int, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_ulonglong]
    fmt, g, xdt, N, K, M = orc.INT4, 128, 1, 512, 2304, 16
    ref = orc.quantize(fmt, synth.llama_like(N, K, seed=81), g)
    pc, pm = orc.pack(ref)
    pc, pm = torch.from_numpy(pc).cuda(), torch.from_numpy(pm).cuda()
    Xb = H.to_x_bits(synth.activations(M, K, seed=82), xdt)
    X = H.x_tensor(Xb)
    Y = torch.full((M, N), -1, dtype=torch.int16, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    d = Q.desc(fmt, N, K, g)
    stream = torch.cuda.current_stream().cuda_stream
    torch.cuda.synchronize()

    t0 = time.time()
    rc = f(ctypes.byref(d), pc.data_ptr(), pm.data_ptr(), X.data_ptr(), Y.data_ptr(), M, xdt, st.data_ptr(), stream,
           1, 50_000_000)
    assert rc == Q.QNT_OK
    torch.cuda.synchronize()
    dt = time.time() - t0
    assert int(st.item()) == Q.QNT_ERR_TIMEOUT
    assert 0.05 <= dt < 10.0, dt

    yref, aref = orc.gemm(ref, Xb, xdt)
    st.zero_()
    Y.fill_(-1)
    Q.qnt_gemm(d, pc, pm, X, Y, M, xdt, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    H.assert_within_tol(H.y_to_f64(Y, xdt), yref, aref, "product GEMM after the timeout", xdt)

    st.zero_()
    Y.fill_(-1)
    assert f(ctypes.byref(d), pc.data_ptr(), pm.data_ptr(), X.data_ptr(), Y.data_ptr(), M, xdt, st.data_ptr(), stream,
             0, 2_000_000_000) == 0
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    H.assert_within_tol(H.y_to_f64(Y, xdt), yref, aref, "test build, no fault", xdt)
