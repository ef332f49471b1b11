// kernels.h -- host-side entry points of the libqnt kernels (internal; the C
// ABI in qnt_abi.cu validates arguments and dispatches to these).
#pragma once
#include <cuda_runtime.h>
#include "qnt.h"

namespace qnt {

// Streaming multiprocessors of the current device (cached per device).
int num_sms();
// Dynamic shared memory that one CTA may request on sm_100.
constexpr int kMaxDynSmem = 227 * 1024;
// Raise a kernel's dynamic shared-memory limit once per process and device;
// later launches make no attribute calls, so they are safe inside stream capture.
cudaError_t configure_smem(const void* fn);

// RTN quantization (quantize.cu).
cudaError_t launch_quantize(const qnt_desc& d, const float* W, void* codes, void* meta, long z0, int* st,
                            cudaStream_t s);

// Y[m] = W x[m] for m < M on CUDA cores, any format (gemv.cu).
cudaError_t launch_gemv_simt(const qnt_desc& d, const void* codes, const void* meta, long z0, const void* X,
                             void* Y, int M, int xbf16, int* st, cudaStream_t s);

// y = W x for one activation vector, 4-bit formats, on the tensor cores with
// mma.sync straight from the packed codes (gemv1.cu).  *handled = false when it
// does not apply (the activation vector and a weight ring do not fit in shared
// memory).
cudaError_t launch_gemv4_one(const qnt_desc& d, const void* codes, const void* meta, long z0, const void* X, void* Y,
                             int xbf16, int* st, cudaStream_t s, bool* handled);

// Two to eight vectors of the 4-bit formats, group 128, K a multiple of 1024:
// the batch-1 kernel with the vectors sharing every MMA (gemv1.cu).
// *handled = false when the case is not covered or does not fit.
cudaError_t launch_gemv1_multi(const qnt_desc& d, const void* codes, const void* meta, const void* X, void* Y, int M,
                              int xbf16, int* st, cudaStream_t s, bool* handled);

// A sequence of batch-1 GEMVs (4-bit formats) in one cooperative launch
// (gemv1.cu); clears the workspace first.  *handled = false when the
// activation vector and a weight ring do not fit in shared memory.
cudaError_t launch_gemv_seq(const qnt_seq_step* steps, int n, int xbf16, void* work, int* st, cudaStream_t s,
                            bool* handled);

// qnt_gemv_seq with the completion counters in a library-owned device array
// (gemv1.cu); n <= QNT_SEQ_NOALLOC_MAX_STEPS.
cudaError_t launch_gemv_seq_noalloc(const qnt_seq_step* steps, int n, int xbf16, int* st, cudaStream_t s,
                                    bool* handled);

#ifdef QNT_TEST_FAULTS
// Test builds only (gemv1.cu): inject `fault` into this thread's next batch-1 /
// sequence launches and use `timeout_ns` as their wait limit.
void set_test_fault(int fault, unsigned long long timeout_ns);
// Test builds only (gemm_tc.cu): the same for this thread's next tcgen05 GEMM launches.
void set_test_gemm_fault(int fault, unsigned long long timeout_ns);
#endif

// An empty kernel: the next kernel in the stream cannot overlap the ones before it.
cudaError_t launch_stream_fence(cudaStream_t s);

// Y[m] = W x[m] for 1 <= M <= 128 on the tensor cores in one pass over the
// weights (gemm_tc.cu, 4-bit formats).  *handled = false when it does not apply.
cudaError_t launch_gemm_tc(const qnt_desc& d, const void* codes, const void* meta, long z0, const void* X, void* Y,
                           int M, int xbf16, int* st, cudaStream_t s, bool* handled);

}  // namespace qnt
