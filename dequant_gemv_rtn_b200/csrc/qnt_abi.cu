// qnt_abi.cu -- the C ABI of libqnt: argument validation, buffer sizes and
// kernel dispatch.  Nothing here allocates memory; every launch goes to the
// caller's stream.
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <cuda_runtime.h>
#include "qnt.h"

#include <cstdlib>
#include "kernels.h"

namespace {

thread_local char g_last_error[256] = "";

// Map a CUDA status to the ABI's code, remembering the text of a failure.
int cuda_rc(cudaError_t e) {
  if (e == cudaSuccess) return QNT_OK;
  snprintf(g_last_error, sizeof(g_last_error), "%s: %s", cudaGetErrorName(e), cudaGetErrorString(e));
  return QNT_ERR_CUDA;
}

bool is_4bit(int f) { return f == QNT_INT4_ASYM || f == QNT_FP4_E2M1 || f == QNT_FP4_AFPQ || f == QNT_FP4_RAZER; }

long round_up(long v, long a) { return (v + a - 1) / a * a; }

long n_groups(const qnt_desc& d) { return is_4bit(d.fmt) ? (long)d.N * (d.K / d.group) : (long)d.N; }

// Start of the zero / selector plane inside the metadata buffer.
long zero_plane(const qnt_desc& d) { return round_up(2 * n_groups(d), 256); }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check(const qnt_desc* d) {
  if (!d) return QNT_ERR_ARG;
  if (d->fmt < QNT_INT4_ASYM || d->fmt > QNT_FP16) return QNT_ERR_ARG;
  if (d->N < 1 || d->K < 128 || d->K % 128 != 0) return QNT_ERR_SHAPE;
  if (d->K > (1 << 20) || d->N > (1 << 24)) return QNT_ERR_SHAPE;
  if (is_4bit(d->fmt)) {
    if (d->group != 32 && d->group != 64 && d->group != 128) return QNT_ERR_SHAPE;
  } else if (d->group != d->K) {
    return QNT_ERR_SHAPE;
  }
  return QNT_OK;
}

// Y[m] = W x[m], m < M.  Kernel choice (measured on B200 with L2-cold weights):
//   one vector, 4-bit formats       -> batch-1 kernel (mma.sync tensor cores)
//   2..8 vectors, 4-bit formats, group 128, K a multiple of 1024
//                                   -> the batch-1 kernel, the vectors sharing its MMAs
//   3..128 vectors otherwise        -> tcgen05 GEMM, one pass over the weights
//   2 vectors otherwise, INT8, FP16 -> CUDA-core multi-vector kernel (passes of 8)
// QNT_FORCE_SIMT=1 selects the CUDA-core multi-vector kernel everywhere (used to
// test every path on the same inputs).
cudaError_t dispatch_gemm(const qnt_desc& d, const void* codes, const void* meta, const void* X, void* Y, int M,
                          int xbf16, int* st, cudaStream_t s) {
  static const bool force_simt = [] {
    const char* a = std::getenv("QNT_FORCE_SIMT");
    return a && a[0] == '1';
  }();
  const long z0 = zero_plane(d);
  bool handled = false;
  cudaError_t e = cudaSuccess;
  if (!force_simt && M == 1) {
    e = qnt::launch_gemv4_one(d, codes, meta, z0, X, Y, xbf16, st, s, &handled);
    if (handled || e != cudaSuccess) return e;
  }
  if (!force_simt && M >= 2 && M <= 8) {
    e = qnt::launch_gemv1_multi(d, codes, meta, X, Y, M, xbf16, st, s, &handled);
    if (handled || e != cudaSuccess) return e;
  }
  if (!force_simt && M >= 3) {
    e = qnt::launch_gemm_tc(d, codes, meta, z0, X, Y, M, xbf16, st, s, &handled);
    if (handled || e != cudaSuccess) return e;
  }
  return qnt::launch_gemv_simt(d, codes, meta, z0, X, Y, M, xbf16, st, s);
}

}  // namespace

extern "C" {

int qnt_version(void) { return QNT_VERSION; }

int qnt_check_desc(const qnt_desc* desc) { return check(desc); }

size_t qnt_codes_bytes(const qnt_desc* d) {
  if (check(d) != QNT_OK) return 0;
  const size_t nk = (size_t)d->N * (size_t)d->K;
  if (d->fmt == QNT_INT8_PERCHAN) return nk;
  if (d->fmt == QNT_FP16) return 2 * nk;
  return ((size_t)d->N + 7) / 8 * 8 * (size_t)d->K / 2;   // 4-bit: whole row groups of eight
}

size_t qnt_meta_bytes(const qnt_desc* d) {
  if (check(d) != QNT_OK) return 0;
  const long P = n_groups(*d);
  switch (d->fmt) {
    case QNT_INT4_ASYM: return (size_t)(zero_plane(*d) + round_up((P + 1) / 2, 16));
    case QNT_FP4_E2M1: return (size_t)round_up(2 * P, 16);
    case QNT_FP4_AFPQ: return (size_t)round_up(4 * P, 16);
    case QNT_FP4_RAZER: return (size_t)(zero_plane(*d) + round_up((P + 3) / 4, 16));
    case QNT_INT8_PERCHAN: return (size_t)round_up(2L * d->N, 16);
    default: return 0;
  }
}

const char* qnt_last_error(void) { return g_last_error; }

const char* qnt_strerror(int code) {
  switch (code) {
    case QNT_OK: return "ok";
    case QNT_ERR_ARG: return "invalid argument (null pointer, unknown format or dtype, M out of range)";
    case QNT_ERR_SHAPE: return "invalid shape (N >= 1, K a positive multiple of 128, group 32/64/128 for 4-bit, K otherwise)";
    case QNT_ERR_ALIGN: return "buffer not 16-byte aligned";
    case QNT_ERR_CUDA: return "CUDA launch failed";
    case QNT_ERR_TIMEOUT: return "device: a bounded wait for an asynchronous copy expired";
    case QNT_ERR_NONFINITE: return "device: NaN or Inf in the weights";
    case QNT_ERR_RANGE: return "device: a scale or FP16 code overflowed fp16";
    default: return "unknown error code";
  }
}

int qnt_quantize(const qnt_desc* desc, const float* d_W, void* d_codes, void* d_meta, int* d_status, void* stream) {
  int e = check(desc);
  if (e != QNT_OK) return e;
  if (!d_W || !d_codes || (desc->fmt != QNT_FP16 && !d_meta)) return QNT_ERR_ARG;
  if (!aligned16(d_W) || !aligned16(d_codes) || (d_meta && !aligned16(d_meta))) return QNT_ERR_ALIGN;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const long z0 = zero_plane(*desc);
  if (desc->fmt == QNT_INT4_ASYM || desc->fmt == QNT_FP4_RAZER) {
    // the zero / selector plane is filled with atomic ORs: clear it first
    const size_t tail = qnt_meta_bytes(desc) - (size_t)z0;   /* a multiple of 16 bytes */
    const int rc = cuda_rc(cudaMemsetAsync(static_cast<uint8_t*>(d_meta) + z0, 0, tail, s));
    if (rc != QNT_OK) return rc;
  }
  const int rc = cuda_rc(qnt::launch_quantize(*desc, d_W, d_codes, d_meta, z0, d_status, s));
  if (rc != QNT_OK) return rc;
  // a GEMV right after this call requests the codes before it waits for the
  // preceding kernel: put a kernel in between that starts only after this one
  return cuda_rc(qnt::launch_stream_fence(s));
}

}  // extern "C"

namespace {
// Validation of the steps of qnt_gemv_seq_noalloc (the rules of qnt_gemv_seq).
int check_seq(const qnt_seq_step* steps, int nsteps, int xdtype) {
  if (xdtype != QNT_F16 && xdtype != QNT_BF16) return QNT_ERR_ARG;
  for (int i = 0; i < nsteps; ++i) {
    const qnt_seq_step& t = steps[i];
    const int e = check(&t.desc);
    if (e != QNT_OK) return e;
    if (!is_4bit(t.desc.fmt) || t.desc.fmt != steps[0].desc.fmt || t.desc.group != steps[0].desc.group)
      return QNT_ERR_ARG;
    if (t.wait < 0 || t.wait > i) return QNT_ERR_ARG;
    if (t.desc.K > QNT_MAX_GEMV_K) return QNT_ERR_SHAPE;
    if (!t.codes || !t.meta || !t.x || !t.y) return QNT_ERR_ARG;
    if (!aligned16(t.codes) || !aligned16(t.meta) || !aligned16(t.x) || !aligned16(t.y)) return QNT_ERR_ALIGN;
  }
  return QNT_OK;
}
}  // namespace

extern "C" {

size_t qnt_gemv_seq_work_bytes(int nsteps) {
  if (nsteps < 1 || nsteps > QNT_SEQ_MAX_STEPS) return 0;
  return (size_t)round_up(4L * (nsteps + 1), 16);   // a counter per step, then an abort word
}

int qnt_gemv_seq_noalloc(const qnt_seq_step* steps, int nsteps, int xdtype, int* d_status, void* stream) {
  if (!steps || nsteps < 1 || nsteps > QNT_SEQ_NOALLOC_MAX_STEPS) return QNT_ERR_ARG;
  const int v = check_seq(steps, nsteps, xdtype);
  if (v != QNT_OK) return v;
  bool handled = false;
  const int rc = cuda_rc(qnt::launch_gemv_seq_noalloc(steps, nsteps, xdtype == QNT_BF16, d_status,
                                                      static_cast<cudaStream_t>(stream), &handled));
  if (rc != QNT_OK) return rc;
  return handled ? QNT_OK : QNT_ERR_SHAPE;
}

int qnt_gemv_seq(const qnt_seq_step* steps, int nsteps, int xdtype, void* d_work, int* d_status, void* stream) {
  if (!steps || nsteps < 1 || nsteps > QNT_SEQ_MAX_STEPS) return QNT_ERR_ARG;
  if (xdtype != QNT_F16 && xdtype != QNT_BF16) return QNT_ERR_ARG;
  if (!d_work) return QNT_ERR_ARG;
  for (int i = 0; i < nsteps; ++i) {
    const qnt_seq_step& t = steps[i];
    const int e = check(&t.desc);
    if (e != QNT_OK) return e;
    if (!is_4bit(t.desc.fmt) || t.desc.fmt != steps[0].desc.fmt || t.desc.group != steps[0].desc.group)
      return QNT_ERR_ARG;
    if (t.wait < 0 || t.wait > i) return QNT_ERR_ARG;
    if (t.desc.K > QNT_MAX_GEMV_K) return QNT_ERR_SHAPE;
    if (!t.codes || !t.meta || !t.x || !t.y) return QNT_ERR_ARG;
    if (!aligned16(t.codes) || !aligned16(t.meta) || !aligned16(t.x) || !aligned16(t.y)) return QNT_ERR_ALIGN;
  }
  if (!aligned16(d_work)) return QNT_ERR_ALIGN;
  bool handled = false;
  const int rc = cuda_rc(qnt::launch_gemv_seq(steps, nsteps, xdtype == QNT_BF16, d_work, d_status,
                                              static_cast<cudaStream_t>(stream), &handled));
  if (rc != QNT_OK) return rc;
  return handled ? QNT_OK : QNT_ERR_SHAPE;
}

int qnt_gemm(const qnt_desc* desc, const void* d_codes, const void* d_meta, const void* d_X, void* d_Y, int M,
             int xdtype, int* d_status, void* stream) {
  int e = check(desc);
  if (e != QNT_OK) return e;
  if (desc->K > QNT_MAX_GEMV_K) return QNT_ERR_SHAPE;
  if (M < 1 || M > 128) return QNT_ERR_ARG;
  if (xdtype != QNT_F16 && xdtype != QNT_BF16) return QNT_ERR_ARG;
  if (!d_codes || !d_X || !d_Y || (desc->fmt != QNT_FP16 && !d_meta)) return QNT_ERR_ARG;
  if (!aligned16(d_codes) || !aligned16(d_X) || !aligned16(d_Y) || (d_meta && !aligned16(d_meta))) return QNT_ERR_ALIGN;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  return cuda_rc(dispatch_gemm(*desc, d_codes, d_meta, d_X, d_Y, M, xdtype == QNT_BF16, d_status, s));
}

int qnt_gemv(const qnt_desc* desc, const void* d_codes, const void* d_meta, const void* d_x, void* d_y, int xdtype,
             int* d_status, void* stream) {
  int e = check(desc);
  if (e != QNT_OK) return e;
  if (desc->K > QNT_MAX_GEMV_K) return QNT_ERR_SHAPE;
  if (xdtype != QNT_F16 && xdtype != QNT_BF16) return QNT_ERR_ARG;
  if (!d_codes || !d_x || !d_y || (desc->fmt != QNT_FP16 && !d_meta)) return QNT_ERR_ARG;
  if (!aligned16(d_codes) || !aligned16(d_x) || !aligned16(d_y) || (d_meta && !aligned16(d_meta))) return QNT_ERR_ALIGN;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  return cuda_rc(dispatch_gemm(*desc, d_codes, d_meta, d_x, d_y, 1, xdtype == QNT_BF16, d_status, s));
}

}  // extern "C"

#ifdef QNT_TEST_FAULTS
// Test builds only (libqnt_test.so, never the product library): qnt_gemv_seq
// with a fault injected and a short wait limit, so that a test can watch a
// bounded wait expire.  fault 1: CTA 0 never reports step 0 complete, so every
// step that waits for step 0 gives up after timeout_ns and the kernel reports
// QNT_ERR_TIMEOUT, drains its copies and returns.
extern "C" int qnt_test_gemv_seq_fault(const qnt_seq_step* steps, int nsteps, int xdtype, void* d_work,
                                       int* d_status, void* stream, int fault, unsigned long long timeout_ns) {
  qnt::set_test_fault(fault, timeout_ns);
  const int rc = qnt_gemv_seq(steps, nsteps, xdtype, d_work, d_status, stream);
  qnt::set_test_fault(0, 2000000000ull);
  return rc;
}

// Test builds only: qnt_gemm (M >= 3, 4-bit formats: the tcgen05 GEMM) with a
// fault injected and a short wait limit.  fault 1: in CTA 0 one decode warp
// never reports stage 0 decoded, so the MMA issuers' wait for it gives up after
// timeout_ns; the kernel reports QNT_ERR_TIMEOUT, lets the copies it issued
// land, frees its tensor memory and returns.
extern "C" int qnt_test_gemm_fault(const qnt_desc* desc, const void* d_codes, const void* d_meta, const void* d_X,
                                   void* d_Y, int M, int xdtype, int* d_status, void* stream, int fault,
                                   unsigned long long timeout_ns) {
  qnt::set_test_gemm_fault(fault, timeout_ns);
  const int rc = qnt_gemm(desc, d_codes, d_meta, d_X, d_Y, M, xdtype, d_status, stream);
  qnt::set_test_gemm_fault(0, 2000000000ull);
  return rc;
}
#endif
