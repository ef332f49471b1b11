"""qnt_gemv_seq_noalloc: the sequence entry point for callers that cannot
allocate device memory (for example a host framework whose device memory is
all handed out by its own pool, or a plug-in that may not call the CUDA
allocator), so cannot pass a workspace.  Its completion counters live in a
small array the library keeps in device memory.

The test runs a chain of dependent GEMVs through both entry points of the C ABI
and checks that the allocation-free one gives the outputs of the ordinary one
(within the 4e-3 * sum |dq x| tolerance of the other tests, against the CPU
oracle's sum of magnitudes), on two calls in a row: the second call starts
from counters the first one left behind.  This file is collected last so that a
run that stops at the first failure has run every other test before it; it
also passes on its own in a fresh process (its first call looks up the
array's address).
"""
import numpy as np
import pytest
import torch

from dequant_gemv_rtn_b200 import synth
from oracle import oracle as orc
from tests import gpu_helpers as H

pytestmark = pytest.mark.gpu

NAN16 = 0x7E00
# x of each step after the first is the start of the previous step's y
CHAIN = [(1536, 1024), (1032, 1536), (4224, 1024), (640, 4224), (2048, 640)]


def _setup(fmt, g, xdt, seed):
    mats = []
    for i, (N, K) in enumerate(CHAIN):
        ref = orc.quantize(fmt, synth.llama_like(N, K, seed=seed + i), g)
        pc, pm = orc.pack(ref)
        mats.append((ref, torch.from_numpy(pc).cuda(), torch.from_numpy(pm).cuda()))
    x0 = H.x_tensor(H.to_x_bits(synth.activations(1, CHAIN[0][1], seed=seed), xdt))
    return mats, x0


def _run(Q, fmt, g, xdt, mats, x0, use_noalloc, work=None):
    ys = [torch.full((N,), NAN16, dtype=torch.int16, device="cuda") for N, _ in CHAIN]
    xs = [x0] + [ys[i][:CHAIN[i + 1][1]] for i in range(len(CHAIN) - 1)]
    items = [(Q.desc(fmt, N, K, g), pc, pm, x, y, 1 if i else 0)
             for i, ((ref, pc, pm), x, y, (N, K)) in enumerate(zip(mats, xs, ys, CHAIN))]
    steps = Q.seq_steps(items)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    if use_noalloc:
        Q.qnt_gemv_seq_noalloc(steps, xdt, st)
    else:
        Q.qnt_gemv_seq(steps, xdt, work, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    return xs, ys


@pytest.mark.parametrize("fmt,g,xdt", [(orc.INT4, 128, 0), (orc.RAZER, 64, 1)])
def test_noalloc_matches_workspace_entry_point_twice(fmt, g, xdt):
    Q = H.q()
    mats, x0 = _setup(fmt, g, xdt, seed=700 + fmt + g)
    work = H.dev_bytes(Q.qnt_gemv_seq_work_bytes(len(CHAIN)))
    xs_ref, ys_ref = _run(Q, fmt, g, xdt, mats, x0, use_noalloc=False, work=work)
    for call in range(2):
        xs, ys = _run(Q, fmt, g, xdt, mats, x0, use_noalloc=True)
        for i, ((ref, _, _), x, y, yr) in enumerate(zip(mats, xs, ys, ys_ref)):
            xb = x.cpu().view(torch.int16).numpy().view(np.uint16)[None, :]
            assert np.array_equal(xb, (x0 if i == 0 else ys_ref[i - 1][:CHAIN[i][1]]).cpu().view(torch.int16)
                                  .numpy().view(np.uint16)[None, :]), f"call {call} step {i}: inputs differ"
            _, aref = orc.gemm(ref, xb, xdt)
            H.assert_within_tol(H.y_to_f64(y[None, :], xdt), H.y_to_f64(yr[None, :], xdt), aref,
                                f"noalloc call {call} step {i} vs workspace entry point", xdt)


def test_noalloc_rejects_too_many_steps():
    Q = H.q()
    A = 1 << 20
    d = Q.desc(Q.QNT_INT4_ASYM, 64, 256, 128)
    steps = Q.seq_steps([(d, A, A, A, A, 0)] * (Q.QNT_SEQ_NOALLOC_MAX_STEPS + 1))
    assert Q.qnt_gemv_seq_noalloc(steps, Q.QNT_F16, check=False, stream=0) == Q.QNT_ERR_ARG
