"""Dependent calls on one stream with no host synchronization in between.

The batch-1 GEMV kernels start before the preceding kernel on the stream has
finished (programmatic dependent launch) and request their weights at once;
only the reads of x and the writes of y wait.  The sequence kernel
(qnt_gemv_seq) orders its steps with completion counters instead.  These tests
chain calls so that each GEMV's x is the previous GEMV's y, poison every y with
NaN beforehand (a read that races its producer shows up as NaN or a wrong
value), and check every step against the CPU oracle evaluated on the x that the
step actually consumed (read back after the chain).  Also: quantize followed by
a GEMV on the fresh codes, and the same chains captured in CUDA graphs.
"""
import numpy as np
import pytest
import torch

from dequant_gemv_rtn_b200 import synth
from oracle import oracle as orc
from tests import gpu_helpers as H

pytestmark = pytest.mark.gpu

FOUR = [orc.INT4, orc.FP4, orc.AFPQ, orc.RAZER]
NAN16 = 0x7E00


def _packed(fmt, N, K, g, seed):
    W = synth.llama_like(N, K, seed=seed)
    ref = orc.quantize(fmt, W, g)
    pc, pm = orc.pack(ref)
    return ref, torch.from_numpy(pc).cuda(), torch.from_numpy(pm).cuda()


def _bits(t: torch.Tensor) -> np.ndarray:
    return t.cpu().view(torch.int16).numpy().view(np.uint16)


# A chain of shapes where x_{i+1} = y_i[:K_{i+1}] (several tiles, a ragged N,
# a tail of K that is not a whole work item).
CHAIN = [(1536, 1024), (1032, 1536), (4224, 1024), (640, 4224), (2048, 640)]


def _chain_buffers(fmt, g, xdt, seed0):
    mats = [_packed(fmt, N, K, g, seed0 + i) for i, (N, K) in enumerate(CHAIN)]
    x0 = torch.from_numpy(H.to_x_bits(synth.activations(1, CHAIN[0][1], seed=seed0), xdt).view(np.int16)).cuda()
    ys = [torch.full((N,), NAN16, dtype=torch.int16, device="cuda") for N, _ in CHAIN]
    xs = [x0] + [ys[i][:CHAIN[i + 1][1]] for i in range(len(CHAIN) - 1)]
    return mats, xs, ys


def _check_chain(mats, xs, ys, xdt, ctx):
    for i, ((ref, _, _), x, y) in enumerate(zip(mats, xs, ys)):
        xb = _bits(x)[None, :]
        assert np.all((xb & 0x7FFF) < (0x7F80 if xdt else 0x7C00)), f"{ctx}: step {i} input not finite"
        yref, aref = orc.gemm(ref, xb, xdt)
        H.assert_within_tol(H.y_to_f64(y[None, :], xdt), yref, aref, f"{ctx} step {i}", xdt)


@pytest.mark.parametrize("fmt", FOUR)
@pytest.mark.parametrize("xdt", [0, 1])
def test_gemv_chain_back_to_back(fmt, xdt):
    Q = H.q()
    g = 128
    mats, xs, ys = _chain_buffers(fmt, g, xdt, seed0=10 * fmt + xdt)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    torch.cuda.synchronize()
    for (ref, pc, pm), x, y, (N, K) in zip(mats, xs, ys, CHAIN):
        Q.qnt_gemv(Q.desc(fmt, N, K, g), pc, pm, x, y, xdt, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    _check_chain(mats, xs, ys, xdt, f"chain fmt={fmt} xdt={xdt}")


@pytest.mark.parametrize("fmt", [orc.INT4, orc.RAZER])
def test_gemv_chain_in_cuda_graph(fmt):
    Q = H.q()
    g, xdt = 128, 0
    mats, xs, ys = _chain_buffers(fmt, g, xdt, seed0=77 + fmt)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    s = torch.cuda.Stream()

    def run(stream):
        for (ref, pc, pm), x, y, (N, K) in zip(mats, xs, ys, CHAIN):
            Q.qnt_gemv(Q.desc(fmt, N, K, g), pc, pm, x, y, xdt, st, stream)

    with torch.cuda.stream(s):
        run(s)                         # eager first: per-kernel attributes are set outside capture
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=s):
        run(torch.cuda.current_stream())
    for rep in range(3):
        for y in ys:
            y.fill_(NAN16)
        torch.cuda.synchronize()
        graph.replay()
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        _check_chain(mats, xs, ys, xdt, f"graph fmt={fmt} replay {rep}")


@pytest.mark.parametrize("fmt", FOUR)
def test_quantize_then_gemv_without_sync(fmt):
    """qnt_gemv requests its codes before it waits for the preceding kernel;
    qnt_quantize ends with an empty kernel so the fresh codes are what it reads.
    The codes and metadata buffers start as garbage from an earlier matrix."""
    Q = H.q()
    N, K, g = 4096, 4096, 128
    W1 = synth.llama_like_device(N, K, seed=900 + fmt)
    W2 = synth.llama_like_device(N, K, seed=901 + fmt)
    d = Q.desc(fmt, N, K, g)
    codes = H.dev_bytes(Q.qnt_codes_bytes(d))
    meta = H.dev_bytes(Q.qnt_meta_bytes(d))
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    Q.qnt_quantize(d, W1, codes, meta, st)
    torch.cuda.synchronize()
    xb = H.to_x_bits(synth.activations(1, K, seed=fmt), 0)
    x = H.x_tensor(xb)
    y = torch.full((N,), NAN16, dtype=torch.int16, device="cuda")
    Q.qnt_quantize(d, W2, codes, meta, st)       # no synchronization before the GEMV
    Q.qnt_gemv(d, codes, meta, x, y, 0, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    rows = np.array(sorted(set(range(8)) | set(range(N - 8, N)) | set(range(0, N, 97))))
    ref = orc.quantize(fmt, W2[torch.from_numpy(rows).cuda()].cpu().numpy(), g)
    H.assert_quant_equal(H.unpack_rows(fmt, N, K, g, codes, meta, rows), ref, "fresh codes")
    yref, aref = orc.gemm(ref, xb, 0)
    H.assert_within_tol(H.y_to_f64(y[None, :], 0)[:, rows], yref, aref, f"quantize->gemv fmt={fmt}")


# ------------------------------------------------------------------ the sequence kernel
@pytest.mark.parametrize("fmt", FOUR)
@pytest.mark.parametrize("g", [128, 64, 32])
def test_gemv_seq_chain(fmt, g):
    Q = H.q()
    xdt = 1 if g == 64 else 0
    mats, xs, ys = _chain_buffers(fmt, g, xdt, seed0=200 + 3 * fmt + g)
    items = [(Q.desc(fmt, N, K, g), pc, pm, x, y, 1 if i else 0)
             for i, ((ref, pc, pm), x, y, (N, K)) in enumerate(zip(mats, xs, ys, CHAIN))]
    steps = Q.seq_steps(items)
    work = H.dev_bytes(Q.qnt_gemv_seq_work_bytes(len(items)))
    work.fill_(0xAB)                     # the call clears its workspace itself
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    torch.cuda.synchronize()
    Q.qnt_gemv_seq(steps, xdt, work, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    _check_chain(mats, xs, ys, xdt, f"seq fmt={fmt} g={g}")


def test_gemv_seq_independent_steps_and_tiny_shapes():
    """Steps that do not wait (own inputs), N = 1 and N < 8 (fewer row groups than
    CTAs), and a dependent step after them; two calls in a row reuse the workspace."""
    Q = H.q()
    fmt, g, xdt = orc.INT4, 128, 0
    shapes = [(1, 128), (5, 256), (3000, 128), (7, 3000 // 8 * 8 // 128 * 128)]
    mats = [_packed(fmt, N, K, g, 300 + i) for i, (N, K) in enumerate(shapes)]
    xs = [H.x_tensor(H.to_x_bits(synth.activations(1, K, seed=i), xdt)) for i, (_, K) in enumerate(shapes[:3])]
    ys = [torch.full((N,), NAN16, dtype=torch.int16, device="cuda") for N, _ in shapes]
    xs.append(ys[2][:shapes[3][1]])
    items = [(Q.desc(fmt, N, K, g), pc, pm, x, y, 1 if i == 3 else 0)
             for i, ((ref, pc, pm), x, y, (N, K)) in enumerate(zip(mats, xs, ys, shapes))]
    steps = Q.seq_steps(items)
    work = H.dev_bytes(Q.qnt_gemv_seq_work_bytes(len(items)))
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    for rep in range(2):
        for y in ys:
            y.fill_(NAN16)
        Q.qnt_gemv_seq(steps, xdt, work, st)
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        _check_chain(mats, xs, ys, xdt, f"independent rep {rep}")


@pytest.mark.parametrize("fmt,g", [(orc.INT4, 128), (orc.AFPQ, 128), (orc.RAZER, 64), (orc.FP4, 32)])
def test_gemv_seq_shared_x_and_waits_back(fmt, g):
    """Steps that read the same x with no new dependency keep one activation
    image (the second and third step on x0, the fifth after the fourth), one of
    them with rows on few CTAs (N = 40); steps that wait several steps back
    (step 3 for step 0, step 4 for step 0 as well, step 6 for step 4); a step
    with a larger K than the others in between (8192).  Two calls in a row;
    every y poisoned with NaN before each."""
    Q = H.q()
    xdt = 0
    #            (N, K),       x source,        wait
    plan = [((1200, 2048), "x0", 0), ((40, 2048), "x0", 0), ((1000, 2048), "x0", 0),
            ((2048, 1024), ("y", 0), 3), ((512, 1024), ("y", 0), 4), ((256, 8192), "xb", 0),
            ((300, 512), ("y", 4), 2)]
    mats = [_packed(fmt, N, K, g, 700 + i) for i, ((N, K), _, _) in enumerate(plan)]
    x0 = H.x_tensor(H.to_x_bits(synth.activations(1, 2048, seed=70), xdt))
    xb = H.x_tensor(H.to_x_bits(synth.activations(1, 8192, seed=71), xdt))
    ys = [torch.full((N,), NAN16, dtype=torch.int16, device="cuda") for (N, _), _, _ in plan]
    xs = []
    for (N, K), src, _ in plan:
        xs.append(x0 if src == "x0" else xb if src == "xb" else ys[src[1]][:K])
        assert xs[-1].numel() == K
    items = [(Q.desc(fmt, N, K, g), pc, pm, x, y, w)
             for ((ref, pc, pm), x, y, ((N, K), _, w)) in zip(mats, xs, ys, plan)]
    steps = Q.seq_steps(items)
    work = H.dev_bytes(Q.qnt_gemv_seq_work_bytes(len(items)))
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    for rep in range(2):
        for y in ys:
            y.fill_(NAN16)
        Q.qnt_gemv_seq(steps, xdt, work, st)
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        _check_chain(mats, xs, ys, xdt, f"continuing steps fmt={fmt} g={g} rep {rep}")


def test_gemv_seq_llama_layers_in_cuda_graph():
    """Two Llama-7B decode layers (qkv 12288x4096, o 4096^2, gate / up 11008x4096,
    down 4096x11008; INT4 g128) as one sequence: o reads the first 4096 outputs
    of qkv, gate and up read o's output, down reads gate's, the next layer's qkv
    reads down's.  Quantized on the GPU; checked on sampled rows, on the x each
    step consumed.  Each step waits only for its producer (up: two steps back).
    Captured in a CUDA graph and replayed."""
    Q = H.q()
    fmt, g, xdt = orc.INT4, 128, 0
    shapes = [("qkv", 12288, 4096), ("o", 4096, 4096), ("gate", 11008, 4096), ("up", 11008, 4096),
              ("down", 4096, 11008)] * 2
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    mods = []
    for i, (name, N, K) in enumerate(shapes):
        d = Q.desc(fmt, N, K, g)
        W = synth.llama_like_device(N, K, seed=4000 + i)
        codes, meta = H.dev_bytes(Q.qnt_codes_bytes(d)), H.dev_bytes(Q.qnt_meta_bytes(d))
        Q.qnt_quantize(d, W, codes, meta, st)
        rows = np.array(sorted(set(range(4)) | set(range(N - 4, N)) | set(range(0, N, 509))))
        mods.append((d, codes, meta, rows, orc.quantize(fmt, W[torch.from_numpy(rows).cuda()].cpu().numpy(), g)))
        del W
    x0 = H.x_tensor(H.to_x_bits(synth.activations(1, 4096, seed=5), xdt))
    ys = [torch.full((N,), NAN16, dtype=torch.int16, device="cuda") for _, N, _ in shapes]
    src = {"qkv": None, "o": 0, "gate": 1, "up": 1, "down": 2}   # offset of the producing step in the layer
    xs = []
    for i, (name, N, K) in enumerate(shapes):
        if i == 0:
            xs.append(x0)
        elif name == "qkv":
            xs.append(ys[i - 1][:K])
        else:
            xs.append(ys[5 * (i // 5) + src[name]][:K])
    back = {"qkv": 1, "o": 1, "gate": 1, "up": 2, "down": 1}    # steps back to the producer
    items = [(d, c, m, x, y, 0 if i == 0 else back[shapes[i][0]])
             for i, ((d, c, m, _, _), x, y) in enumerate(zip(mods, xs, ys))]
    steps = Q.seq_steps(items)
    work = H.dev_bytes(Q.qnt_gemv_seq_work_bytes(len(items)))
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        Q.qnt_gemv_seq(steps, xdt, work, st, s)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=s):
        Q.qnt_gemv_seq(steps, xdt, work, st, torch.cuda.current_stream())
    for rep in range(2):
        for y in ys:
            y.fill_(NAN16)
        torch.cuda.synchronize()
        graph.replay()
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        for i, ((d, _, _, rows, ref), x, y) in enumerate(zip(mods, xs, ys)):
            xb = _bits(x)[None, :]
            yref, aref = orc.gemm(ref, xb, xdt)
            H.assert_within_tol(H.y_to_f64(y[None, :], xdt)[:, rows], yref, aref, f"layers rep {rep} step {i}", xdt)
