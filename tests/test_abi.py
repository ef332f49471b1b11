"""C-ABI checks that need no GPU: the library loads, exports every function that
include/*.h declares, validates arguments on the host (returning error codes
without launching anything), sizes buffers like the layout text says, and the
selective-precision table resolves module names."""
import ctypes
import glob
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        for m in re.finditer(r"\b(qnt_\w+)\s*\(", text):
            names.add(m.group(1))
    return sorted(names)


@pytest.fixture(scope="module")
def q():
    from dequant_gemv_rtn_b200 import build
    build.build()
    from dequant_gemv_rtn_b200 import qnt
    return qnt


def test_exports_every_declared_symbol(q):
    names = _declared_functions()
    assert "qnt_gemv" in names and "qnt_quantize" in names and "qnt_gemm" in names
    lib = ctypes.CDLL(q.LIB_PATH)
    missing = [n for n in names if not hasattr(lib, n)]
    assert not missing, missing


def test_version_and_strerror(q):
    assert q.qnt_version() == 3
    for c in range(8):
        assert q.qnt_strerror(c)
    assert "unknown" in q.qnt_strerror(99)


@pytest.mark.parametrize("fmt", [1, 2, 3, 4, 5, 6])
@pytest.mark.parametrize("shape", [(256, 512, 32), (4096, 11008, 128), (33, 384, 64), (1, 128, 128)])
def test_buffer_sizes_match_layout_text(q, orc, fmt, shape):
    N, K, g = shape
    d = q.desc(fmt, N, K, g)
    assert q.qnt_check_desc(d) == 0
    assert q.qnt_codes_bytes(d) == orc.codes_bytes(fmt, N, K)
    assert q.qnt_meta_bytes(d) == orc.meta_bytes(fmt, N, K, g)


def test_shape_validation(q):
    bad = [q.desc(1, 0, 128, 128), q.desc(1, 16, 100, 32), q.desc(1, 16, 256, 16), q.desc(2, 16, 256, 256),
           q.desc(7, 16, 256, 128), q.desc(0, 16, 256, 128)]
    codes = [q.qnt_check_desc(d) for d in bad]
    assert codes == [q.QNT_ERR_SHAPE, q.QNT_ERR_SHAPE, q.QNT_ERR_SHAPE, q.QNT_ERR_SHAPE, q.QNT_ERR_ARG, q.QNT_ERR_ARG]
    d = q.qnt_desc(5, 16, 256, 128)   # INT8 needs group == K
    assert q.qnt_check_desc(d) == q.QNT_ERR_SHAPE
    for d in bad:
        assert q.qnt_codes_bytes(d) == 0 and q.qnt_meta_bytes(d) == 0


def test_calls_reject_bad_arguments_without_launching(q):
    d = q.desc(1, 64, 256, 128)
    A = 1 << 20   # fake, 16-byte aligned addresses: validation fails before any CUDA call
    assert q.qnt_gemv(d, None, A, A, A, check=False, stream=0) == q.QNT_ERR_ARG
    assert q.qnt_gemv(d, A, A, A + 2, A, check=False, stream=0) == q.QNT_ERR_ALIGN
    assert q.qnt_gemv(d, A, A, A, A, xdtype=5, check=False, stream=0) == q.QNT_ERR_ARG
    assert q.qnt_gemm(d, A, A, A, A, 0, check=False, stream=0) == q.QNT_ERR_ARG
    assert q.qnt_gemm(d, A, A, A, A, 129, check=False, stream=0) == q.QNT_ERR_ARG
    assert q.qnt_gemm(d, A, A + 8, A, A, 4, check=False, stream=0) == q.QNT_ERR_ALIGN
    assert q.qnt_quantize(d, A, None, A, check=False, stream=0) == q.QNT_ERR_ARG
    assert q.qnt_quantize(d, A + 4, A, A, check=False, stream=0) == q.QNT_ERR_ALIGN
    assert q.qnt_quantize(q.desc(1, 64, 200, 128), A, A, A, check=False, stream=0) == q.QNT_ERR_SHAPE
    with pytest.raises(q.QntError):
        q.qnt_gemv(d, None, A, A, A, stream=0)


def test_selective_precision_table(q):
    """Llama-2-7B style policy: INT4 g128 default, INT8 per-channel down_proj in
    the first two and last two layers, FP16 lm_head."""
    t = q.qnt_table_create(q.QNT_INT4_ASYM, 128)
    for layer in (0, 1, 30, 31):
        t.set(f"model.layers.{layer}.mlp.down_proj", q.QNT_INT8_PERCHAN, 0)
    t.set("lm_head", q.QNT_FP16, 0)
    t.set("*.self_attn.?_proj", q.QNT_INT4_ASYM, 64)
    assert len(t) == 6
    assert t.lookup("model.layers.0.mlp.down_proj") == (q.QNT_INT8_PERCHAN, 0)
    assert t.lookup("model.layers.2.mlp.down_proj") == (q.QNT_INT4_ASYM, 128)
    assert t.lookup("model.layers.31.mlp.down_proj") == (q.QNT_INT8_PERCHAN, 0)
    assert t.lookup("lm_head") == (q.QNT_FP16, 0)
    assert t.lookup("model.layers.7.self_attn.q_proj") == (q.QNT_INT4_ASYM, 64)
    assert t.lookup("model.layers.7.self_attn.o_proj") == (q.QNT_INT4_ASYM, 64)
    assert t.lookup("model.layers.7.mlp.up_proj") == (q.QNT_INT4_ASYM, 128)
    # first match wins
    t.set("model.layers.*", q.QNT_FP16, 0)
    assert t.lookup("model.layers.0.mlp.down_proj") == (q.QNT_INT8_PERCHAN, 0)
    assert t.lookup("model.layers.5.mlp.gate_proj") == (q.QNT_FP16, 0)
    with pytest.raises(q.QntError):
        t.set("x", q.QNT_FP4_E2M1, 48)
    with pytest.raises(q.QntError):
        t.set("x", 9, 128)
    t.close()
    with pytest.raises(q.QntError):
        q.qnt_table_create(q.QNT_INT4_ASYM, 100)


def test_glob_edge_cases(q):
    t = q.qnt_table_create(q.QNT_FP4_E2M1, 32)
    t.set("a*b*c", q.QNT_INT8_PERCHAN, 0)
    t.set("", q.QNT_FP16, 0)
    assert t.lookup("abc")[0] == q.QNT_INT8_PERCHAN
    assert t.lookup("aXXbYYc")[0] == q.QNT_INT8_PERCHAN
    assert t.lookup("aXXbYY")[0] == q.QNT_FP4_E2M1
    assert t.lookup("")[0] == q.QNT_FP16
    assert t.lookup("abcc")[0] == q.QNT_INT8_PERCHAN


def test_gemv_k_bound(q):
    """K above QNT_MAX_GEMV_K (the activation vector is staged in shared memory)
    is a shape error for the GEMV calls, not a launch failure; quantize takes it."""
    A = 1 << 20
    big = q.desc(1, 64, q.QNT_MAX_GEMV_K + 128, 128)
    assert q.qnt_check_desc(big) == q.QNT_OK
    assert q.qnt_gemv(big, A, A, A, A, check=False, stream=0) == q.QNT_ERR_SHAPE
    assert q.qnt_gemm(big, A, A, A, A, 4, check=False, stream=0) == q.QNT_ERR_SHAPE
    steps = q.seq_steps([(big, A, A, A, A, 0)])
    assert q.qnt_gemv_seq(steps, q.QNT_F16, A, check=False, stream=0) == q.QNT_ERR_SHAPE


def test_seq_work_bytes(q):
    assert q.qnt_gemv_seq_work_bytes(0) == 0
    assert q.qnt_gemv_seq_work_bytes(q.QNT_SEQ_MAX_STEPS + 1) == 0
    for n in (1, 3, 4, 160, q.QNT_SEQ_MAX_STEPS):
        b = q.qnt_gemv_seq_work_bytes(n)
        assert b >= 4 * (n + 1) and b % 16 == 0


def test_seq_rejects_bad_arguments_without_launching(q):
    A = 1 << 20
    d4 = q.desc(1, 64, 256, 128)
    ok = (d4, A, A, A, A, 0)
    assert q.qnt_gemv_seq(q.seq_steps([]), 0, A, check=False, stream=0) == q.QNT_ERR_ARG
    assert q.qnt_gemv_seq(q.seq_steps([ok] * (q.QNT_SEQ_MAX_STEPS + 1)), 0, A, check=False, stream=0) == q.QNT_ERR_ARG
    cases = [
        ([ok, (q.desc(2, 64, 256, 128), A, A, A, A, 1)], 0, A, q.QNT_ERR_ARG),     # formats differ
        ([ok, (q.desc(1, 64, 256, 64), A, A, A, A, 1)], 0, A, q.QNT_ERR_ARG),      # groups differ
        ([(d4, A, A, A, A, 0), ok, (d4, A, A, A, A, 2)], 0, None, q.QNT_ERR_ARG),  # (valid waits, no workspace)
        ([(q.desc(5, 64, 256, 256), A, A, A, A, 0)], 0, A, q.QNT_ERR_ARG),         # not 4-bit
        ([ok, (d4, A, A, None, A, 1)], 0, A, q.QNT_ERR_ARG),                       # null x
        ([ok, (d4, A, A, A, A, 2)], 0, A, q.QNT_ERR_ARG),                          # waits past step 0
        ([(d4, A, A, A, A, 1)], 0, A, q.QNT_ERR_ARG),                              # step 0 cannot wait
        ([ok, (d4, A, A, A, A, -1)], 0, A, q.QNT_ERR_ARG),                         # negative wait
        ([ok], 7, A, q.QNT_ERR_ARG),                                               # dtype
        ([ok], 0, None, q.QNT_ERR_ARG),                                            # no workspace
        ([ok, (d4, A, A + 8, A, A, 1)], 0, A, q.QNT_ERR_ALIGN),                    # metadata alignment
        ([ok], 0, A + 4, q.QNT_ERR_ALIGN),                                         # workspace alignment
        ([(q.desc(1, 64, 100, 32), A, A, A, A, 0)], 0, A, q.QNT_ERR_SHAPE),        # K % 128
    ]
    for items, xdt, work, want in cases:
        assert q.qnt_gemv_seq(q.seq_steps(items), xdt, work, check=False, stream=0) == want, (items, want)
