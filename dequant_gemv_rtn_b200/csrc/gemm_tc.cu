// gemm_tc.cu -- small-batch fused-dequant GEMM on the tensor cores (tcgen05).
#include "common.cuh"

namespace qnt {

// Returns with *handled = false when the tensor-core path does not take this
// shape; the caller then uses the CUDA-core multi-vector kernel.
cudaError_t launch_gemm_tc(const qnt_desc& d, const void* codes, const void* meta, long z0, const void* X, void* Y,
                           int M, int xbf16, int* st, cudaStream_t s, bool* handled) {
  (void)d; (void)codes; (void)meta; (void)z0; (void)X; (void)Y; (void)M; (void)xbf16; (void)st; (void)s;
  *handled = false;
  return cudaSuccess;
}

}  // namespace qnt
