// gemv.cu -- fused-dequant GEMV on CUDA cores: the multi-vector kernel (all
// formats; the batch-1 tensor-core kernel for 4-bit formats is in gemv1.cu).
//
// The decode-time kernel the RTN page ("Is (Selective) Round-To-Nearest
// Quantization All You Need?", English abstract: token-generation throughput of
// RTN with fused-dequant kernels) and the RaZeR page ("The Power of Negative
// Zero", English abstract and method section: a GEMV that turns 4-bit codes
// into FP16 with bit-level operations, fused with the dot product) describe:
//   y[m][n] = sum_k dq(code[n][k], meta[n][k/g]) * x[m][k].
//
// The CUDA-core multi-vector kernel: INT8 and FP16 weights at any batch and
// the 4-bit formats at batch 2 take it.  One CTA of 16 warps per SM owns a
// contiguous range of rows.
//  * Activations are staged once per CTA with bulk copies; bf16 vectors are
//    rescaled by an exact power of two into fp16 range.
//  * A work item is (2 rows) x (2048 bytes of each row); each warp streams its
//    items through a 2-deep ring of 1-D TMA bulk copies, and lane l reads the
//    16-byte chunks l, l+32, l+64, l+96 of the range.  Per-(row, range)
//    partial sums are combined in a fixed order (deterministic results).
//  * Decode in registers; products by the sm_100 mixed-precision FMA
//    (fma.rn.f32.f16: exact fp16 x fp16 product, fp32 accumulation):
//      INT4: a nibble masked into the low bits of an fp16 half is the fp16
//            subnormal q * 2^-24 (a nibble at bits 4..7 gives 16 q * 2^-24),
//            exact; the zero point is applied once per group as -s z sum(x),
//            from a per-CTA table of group sums.
//      FP4 / RaZeR: cvt.rn.f16x2.e2m1x2; RaZeR codes 0b1000 (decoded as -0)
//            are found with a nibble test and add sv * x separately.  AFPQ
//            splits positive / negative parts and applies s+ and s-.
//      INT8: PRMT into 0x64xx fp16 patterns and one subtract; FP16: direct.
#include <mutex>
#include "common.cuh"
#include "gemv_common.cuh"
#include "kernels.h"

namespace qnt {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kStages = 2;                  // ring depth per warp
constexpr int kRangeBytes = 2048;           // bytes of one row per work item
constexpr int kItemBytes = 2 * kRangeBytes; // 2 rows
constexpr int kCtrlBytes = 1024;            // barriers + reduction scratch
constexpr int kRingBytes = kWarps * kStages * kItemBytes;

// ------------------------------------------------------------------ shared prologue
// Waits for the MB staged activation vectors (fp16 or bf16, [MB][K]) in xs;
// bf16 vectors are rescaled by an exact power of two into fp16 range
// (xscale = 2^e undoes it on the output).  Returns false on a staging timeout
// (status reported; the caller must return).
template <int MB>
__device__ bool stage_activations(uint64_t* xbar, float* red, __half* xs, int K, int xbf16,
                                  float (&xscale)[MB], int* d_status) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  bool ok = mbar_wait(xbar, 0);
  if (__syncthreads_or(!ok)) {
    if (tid == 0) report(d_status, QNT_ERR_TIMEOUT);
    mbar_wait(xbar, 0);
    return false;
  }
#pragma unroll
  for (int m = 0; m < MB; ++m) xscale[m] = 1.0f;
  if (xbf16) {
#pragma unroll 1
    for (int m = 0; m < MB; ++m) {
      const __nv_bfloat16* xb = reinterpret_cast<const __nv_bfloat16*>(xs + (size_t)m * K);
      float am = 0.0f;
      for (int k = tid; k < K; k += kThreads) am = fmaxf(am, fabsf(__bfloat162float(xb[k])));
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, o));
      if (lane == 0) red[warp] = am;
      __syncthreads();
      am = red[0];
      for (int i = 1; i < kWarps; ++i) am = fmaxf(am, red[i]);
      int e = 0;
      if (am > 0.0f && isfinite(am)) e = min(max(ilogbf(am) - 14, -100), 100);
      const float down = __int_as_float((127 - e) << 23);   // 2^-e
#pragma unroll
      for (int mm = 0; mm < MB; ++mm) if (mm == m) xscale[mm] = __int_as_float((127 + e) << 23);
      __syncthreads();
      for (int k = tid; k < K; k += kThreads) {
        const float v = __bfloat162float(xb[k]) * down;
        reinterpret_cast<__half*>(xs + (size_t)m * K)[k] = __float2half_rn(v);
      }
    }
    __syncthreads();
  }
  return true;
}

// ------------------------------------------------------------------ per-chunk dot products
// One 16-byte chunk c of a 4-bit row (32 weights, order as in the layout) with
// the activations xk of its first weight.  acc[0..3]: INT4 [0,1] nibbles at bit
// 0 of a half (scale 1), [2,3] nibbles at bit 4 (scale 16); FP4 / RaZeR [0,1];
// AFPQ [0,1] positive part, [2,3] negative part.  corr (RaZeR): the sum of x
// over weights coded 0b1000.
template <int FMT>
__device__ __forceinline__ void dot_chunk4(const uint4& c, const __half* xk, float (&acc)[4], float& corr) {
  const uint32_t w[4] = {c.x, c.y, c.z, c.w};
  if (FMT == QNT_INT4_ASYM) {
    // word j: low nibbles -> chunk weights 4j..4j+3, high nibbles -> 16+4j..19+4j
    const uint4 xa0 = lds128(xk), xa1 = lds128(xk + 8), xb0 = lds128(xk + 16), xb1 = lds128(xk + 24);
    const uint32_t xl[8] = {xa0.x, xa0.y, xa0.z, xa0.w, xa1.x, xa1.y, xa1.z, xa1.w};
    const uint32_t xh[8] = {xb0.x, xb0.y, xb0.z, xb0.w, xb1.x, xb1.y, xb1.z, xb1.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t w8 = w[j] >> 8;
      fma_mixed2(w[j] & 0x000F000Fu, xl[2 * j], acc[0], acc[1]);
      fma_mixed2(w8 & 0x000F000Fu, xl[2 * j + 1], acc[0], acc[1]);
      fma_mixed2(w[j] & 0x00F000F0u, xh[2 * j], acc[2], acc[3]);
      fma_mixed2(w8 & 0x00F000F0u, xh[2 * j + 1], acc[2], acc[3]);
    }
  } else {
#pragma unroll
    for (int j = 0; j < 4; ++j) {   // word j: chunk weights 8j..8j+7, two per byte
      const uint4 x4 = lds128(xk + 8 * j);
      uint32_t h[4];
      cvt_e2m1x8(w[j], h[0], h[1], h[2], h[3]);
      if (FMT == QNT_FP4_AFPQ) {
#pragma unroll
        for (int p = 0; p < 4; ++p) {
          const uint32_t vp = hmax2(h[p], 0u);
          const uint32_t vn = hsub2(h[p], vp);   // min(v, 0), exact
          fma_mixed2(vp, (&x4.x)[p], acc[0], acc[1]);
          fma_mixed2(vn, (&x4.x)[p], acc[2], acc[3]);
        }
      } else {
#pragma unroll
        for (int p = 0; p < 4; ++p) fma_mixed2(h[p], (&x4.x)[p], acc[0], acc[1]);
        if (FMT == QNT_FP4_RAZER) {
          // nibbles equal to 0b1000: low three bits zero and the sign bit set
          const uint32_t t = (w[j] & 0x77777777u) + 0x77777777u;
          uint32_t spec = lop3<0x20>(w[j], t, 0x88888888u);   // w & ~t & 0x88888888
          while (spec) {
            const int bit = __ffs(spec) - 1;
            spec &= spec - 1;
            corr += __half2float(xk[8 * j + (bit >> 2)]);
          }
        }
      }
    }
  }
}

// Chunk partial scaled by its group's metadata.
template <int FMT>
__device__ __forceinline__ float chunk_value(const GroupMeta& md, const float (&a)[4], float corr) {
  if (FMT == QNT_INT4_ASYM) return md.s * ((a[0] + a[1]) + 0.0625f * (a[2] + a[3]));
  if (FMT == QNT_FP4_AFPQ) return md.s * (a[0] + a[1]) + md.t * (a[2] + a[3]);
  if (FMT == QNT_FP4_RAZER) return md.s * ((a[0] + a[1]) + md.t * corr);
  return md.s * (a[0] + a[1]);
}


// Work ranges: 4-bit formats stream row groups of eight in ranges of 1024
// weights (4 KB, one contiguous run of the layout); INT8 / FP16 stream pairs of
// rows in 2048-byte ranges of each row.
constexpr int kRange4 = 1024;
__host__ __device__ inline int simt_ranges(int fmt, int K) {
  if (fmt == QNT_INT8_PERCHAN) return (K + kRangeBytes - 1) / kRangeBytes;
  if (fmt == QNT_FP16) return (2 * K + kRangeBytes - 1) / kRangeBytes;
  return (K + kRange4 - 1) / kRange4;
}

// Shared-memory carve-up (byte offsets), used by the kernel and the launcher.
struct SmemSimt { size_t xs, xg, part, ms, total; };
// meta_bytes: size of the staged metadata copy (0: read from global memory)
__host__ __device__ inline SmemSimt smem_simt_layout(int fmt, int MB, int K, int group, int rows_cap,
                                                      size_t meta_bytes) {
  const int KR = simt_ranges(fmt, K);
  SmemSimt L;
  L.xs = (size_t)kCtrlBytes + kRingBytes;
  L.xg = align16(L.xs + (size_t)MB * K * 2);
  L.part = align16(L.xg + (fmt == QNT_INT4_ASYM ? (size_t)MB * (K / group) * 4 : 0));
  L.ms = align16(L.part + (size_t)MB * rows_cap * KR * 4);
  L.total = align16(L.ms + meta_bytes);
  return L;
}

// ------------------------------------------------------------------ kernel
// G: group size (4-bit formats; 0 for INT8 / FP16).
template <int FMT, int G, int MB>
__global__ void __launch_bounds__(kThreads, 1)
gemv_simt_kernel(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ meta, long z0,
                 const void* __restrict__ X, void* __restrict__ Y, int N, int K, int ldy, int xbf16,
                 int rows_cap, int meta_bytes, int* d_status) {
  constexpr bool Q4 = FMT != QNT_INT8_PERCHAN && FMT != QNT_FP16;
  constexpr int Gd = G > 0 ? G : 1;                         // group size as a divisor (G = 0: INT8 / FP16)
  constexpr int WPC = FMT == QNT_INT8_PERCHAN ? 16 : 8;   // weights per 16-byte chunk (INT8 / FP16)
  extern __shared__ __align__(1024) uint8_t smem[];
  uint64_t* xbar = reinterpret_cast<uint64_t*>(smem);
  uint64_t* rbar = reinterpret_cast<uint64_t*>(smem + 64);
  float* red = reinterpret_cast<float*>(smem + 512);
  uint8_t* ring = smem + kCtrlBytes;
  const SmemSimt L = smem_simt_layout(FMT, MB, K, Q4 ? G : K, rows_cap, (size_t)meta_bytes);
  __half* xs = reinterpret_cast<__half*>(smem + L.xs);
  float* xg = reinterpret_cast<float*>(smem + L.xg);         // [MB][K/G] group sums (INT4)
  float* part = reinterpret_cast<float*>(smem + L.part);     // [MB][rows_cap][KR]
  uint8_t* ms = smem + L.ms;                                  // staged metadata (4-bit formats)
  const long rowbytes = FMT == QNT_INT8_PERCHAN ? (long)K : 2L * K;   // INT8 / FP16
  const int KR = simt_ranges(FMT, K);
  const int GK = Q4 ? K / G : 1;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  long r_lo, r_hi;
  simt_rows(FMT, N, blockIdx.x, gridDim.x, &r_lo, &r_hi);
  const int nrows = (int)(r_hi - r_lo);
  const int nunits = Q4 ? (nrows + 7) / 8 : (nrows + 1) / 2;   // row groups / row pairs
  const int nitems = nunits * KR;
  uint64_t* mybar = rbar + warp * kStages;
  uint8_t* myring = ring + (size_t)warp * kStages * kItemBytes;

  if (tid == 0) {
    mbar_init(xbar, 1);
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  }
  if (lane == 0)
    for (int s = 0; s < kStages; ++s) mbar_init(mybar + s, 1);
  __syncthreads();
  MetaWin mw = {0, 0, 0, 0, 0};
  if (Q4) mw = meta_window<Q4 ? FMT : QNT_FP4_E2M1>(r_lo, r_hi, GK, z0, rows_cap);
  if (tid == 0) {
    const uint32_t xbytes = (uint32_t)K * 2u;
    const bool stage_meta = Q4 && meta_bytes > 0 && r_hi > r_lo;
    mbar_expect_tx(xbar, xbytes * MB + (stage_meta ? (uint32_t)((mw.a1 - mw.a0) + (mw.b1 - mw.b0)) : 0u));
    if (stage_meta) {
      bulk_g2s(ms, meta + mw.a0, (uint32_t)(mw.a1 - mw.a0), xbar);
      if (mw.b1 > mw.b0) bulk_g2s(ms + mw.bpl, meta + mw.b0, (uint32_t)(mw.b1 - mw.b0), xbar);
    }
    // programmatic dependent launch: the activations (and, after them, every
    // write of Y) wait for the previous kernel in the stream; weights and
    // metadata, which no kernel of this library writes, are already requested
    asm volatile("griddepcontrol.wait;" ::: "memory");
    for (int m = 0; m < MB; ++m)
      bulk_g2s(xs + (size_t)m * K, static_cast<const uint8_t*>(X) + (size_t)m * xbytes, xbytes, xbar);
  }
  const uint64_t pol = l2_evict_first_policy();
  auto issue = [&](int t, int stage) {
    const int un = t / KR, kr = t - un * KR;
    uint8_t* dst = myring + (size_t)stage * kItemBytes;
    if (Q4) {   // row group r_lo/8 + un, blocks 8kr .. 8kr+7: one contiguous run
      const uint32_t nb = (uint32_t)min(8, K / 128 - 8 * kr) * 512u;
      mbar_expect_tx(mybar + stage, nb);
      bulk_g2s_hint(dst, codes + (r_lo / 8 + un) * 4L * K + (long)kr * 4096, nb, mybar + stage, pol);
    } else {
      const long ra = r_lo + 2 * un;
      const int nrow = (ra + 1 < r_hi) ? 2 : 1;
      const long off = (long)kr * kRangeBytes;
      const uint32_t nb = (uint32_t)min((long)kRangeBytes, rowbytes - off);
      mbar_expect_tx(mybar + stage, nb * (uint32_t)nrow);
      for (int r = 0; r < nrow; ++r)
        bulk_g2s_hint(dst + r * kRangeBytes, codes + (ra + r) * rowbytes + off, nb, mybar + stage, pol);
    }
  };
  if (lane == 0)
    for (int s = 0; s < kStages; ++s)
      if (warp + s * kWarps < nitems) issue(warp + s * kWarps, s);

  float xscale[MB];
  if (!stage_activations<MB>(xbar, red, xs, K, xbf16, xscale, d_status)) {
    if (lane == 0)
      for (int s = 0; s < kStages; ++s)
        if (warp + s * kWarps < nitems) mbar_wait(mybar + s, 0);
    return;
  }
  if (FMT == QNT_INT4_ASYM) {   // per-CTA table of group sums of x (fixed summation order)
    for (int idx = tid; idx < MB * GK; idx += kThreads) {
      const __half* xp = xs + (size_t)(idx / GK) * K + (size_t)(idx % GK) * G;
      float sum = 0.0f;
      for (int k = 0; k < G; ++k) sum += __half2float(xp[k]);
      xg[idx] = sum;
    }
    __syncthreads();
  }

  bool failed = false;
  int j = 0;
  for (int t = warp; t < nitems; t += kWarps, ++j) {
    const int stage = j % kStages;
    const uint32_t phase = (uint32_t)(j / kStages) & 1u;
    const int un = t / KR, kr = t - un * KR;
    if (!mbar_wait(mybar + stage, phase)) { failed = true; break; }
    const uint8_t* st = myring + (size_t)stage * kItemBytes;
    if (Q4) {
      // lane l: row i8 = l % 8 of the group, blocks hq = l / 8 and hq + 4 of the
      // range (whole 128-weight blocks, so a G = 128 group is one lane's); the
      // eight lanes of a shared-memory phase read one chunk of eight rows
      // (conflict-free by the layout's swizzle) and the same activations
      const int i8 = lane & 7, hq = lane >> 3;
      const long row = r_lo + 8 * un + i8;
      const int nblk = min(8, K / 128 - 8 * kr);
      float acc[MB];
#pragma unroll
      for (int m = 0; m < MB; ++m) acc[m] = 0.0f;
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const int h = hq + 4 * hh;
        if (h < nblk) {
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const uint4 v = lds128(st + 512 * h + 64 * i8 + 16 * (c ^ ((i8 >> 1) & 3)));
            const long k0 = (long)kr * kRange4 + 128 * h + 32 * c;   // first weight of the chunk
            GroupMeta md = {0.0f, 0.0f};
            if (row < r_hi)
              md = meta_bytes > 0 ? group_meta_s<FMT>(ms, mw, z0, row * GK + k0 / Gd)
                                  : group_meta<FMT>(meta, z0, row * GK + k0 / Gd);
#pragma unroll
            for (int m = 0; m < MB; ++m) {
              float a[4] = {0.0f, 0.0f, 0.0f, 0.0f};
              float corr = 0.0f;
              dot_chunk4<FMT>(v, xs + (size_t)m * K + k0, a, corr);
              float val = chunk_value<FMT>(md, a, corr);
              if (FMT == QNT_INT4_ASYM && (k0 % Gd) == 0) val -= md.t * xg[(size_t)m * GK + k0 / Gd];
              acc[m] += val;
            }
          }
        }
      }
      __syncwarp();
      if (lane == 0 && t + kStages * kWarps < nitems) {
        fence_proxy_async();
        issue(t + kStages * kWarps, stage);
      }
#pragma unroll
      for (int m = 0; m < MB; ++m) {
        float y4 = acc[m];
        y4 += __shfl_xor_sync(0xffffffffu, y4, 8);
        y4 += __shfl_xor_sync(0xffffffffu, y4, 16);
        if (hq == 0 && row < r_hi) part[((size_t)m * rows_cap + (row - r_lo)) * KR + kr] = y4;
      }
      continue;
    }
    const int nch = (int)(min((long)kRangeBytes, rowbytes - (long)kr * kRangeBytes) / 16);   // chunks in range
    float acc[2][MB][2];
#pragma unroll
    for (int r = 0; r < 2; ++r)
#pragma unroll
      for (int m = 0; m < MB; ++m) acc[r][m][0] = acc[r][m][1] = 0.0f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int ch = lane + 32 * i;
      if (ch < nch) {
        const long k0 = ((long)kr * (kRangeBytes / 16) + ch) * WPC;   // first weight of the chunk
        const uint4 va = lds128(st + 16 * ch);
        const uint4 vb = lds128(st + kRangeBytes + 16 * ch);
#pragma unroll
        for (int m = 0; m < MB; ++m) {
          const __half* xk = xs + (size_t)m * K + k0;
          if (FMT == QNT_FP16) {
            const uint4 x4 = lds128(xk);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              fma_mixed2((&va.x)[q], (&x4.x)[q], acc[0][m][0], acc[0][m][1]);
              fma_mixed2((&vb.x)[q], (&x4.x)[q], acc[1][m][0], acc[1][m][1]);
            }
          } else {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const uint4 x4 = lds128(xk + 8 * h);   // weights 8h..8h+7 of the chunk
#pragma unroll
              for (int jj = 0; jj < 2; ++jj) {
                const int q = 2 * h + jj;           // code word q = weights 4q..4q+3
#pragma unroll
                for (int r = 0; r < 2; ++r) {
                  const uint32_t w = (r == 0 ? (&va.x)[q] : (&vb.x)[q]) ^ 0x80808080u;
                  uint32_t lo = prmt(w, 0x64646464u, 0x4140u);   // bytes 0,1 -> 1024 + (q + 128)
                  uint32_t hi = prmt(w, 0x64646464u, 0x4342u);   // bytes 2,3
                  lo = hsub2(lo, 0x64806480u);                   // - 1152 -> q exactly
                  hi = hsub2(hi, 0x64806480u);
                  fma_mixed2(lo, (&x4.x)[2 * jj], acc[r][m][0], acc[r][m][1]);
                  fma_mixed2(hi, (&x4.x)[2 * jj + 1], acc[r][m][0], acc[r][m][1]);
                }
              }
            }
          }
        }
      }
    }
    __syncwarp();
    if (lane == 0 && t + kStages * kWarps < nitems) {
      fence_proxy_async();
      issue(t + kStages * kWarps, stage);
    }
#pragma unroll
    for (int m = 0; m < MB; ++m) {
      const bool upper = lane & 16;
      const float ya = acc[0][m][0] + acc[0][m][1], yb = acc[1][m][0] + acc[1][m][1];
      float keep = upper ? yb : ya;
      const float send = upper ? ya : yb;
      keep += __shfl_xor_sync(0xffffffffu, send, 16);
#pragma unroll
      for (int o = 8; o > 0; o >>= 1) keep += __shfl_xor_sync(0xffffffffu, keep, o);
      const int rl = 2 * un + (upper ? 1 : 0);
      if ((lane & 15) == 0 && rl < nrows) part[((size_t)m * rows_cap + rl) * KR + kr] = keep;
    }
  }
  if (failed && lane == 0) {
    report(d_status, QNT_ERR_TIMEOUT);
    for (int s = 0; s < kStages; ++s) { mbar_wait(mybar + s, 0); mbar_wait(mybar + s, 1); }
  }
  __syncthreads();

  for (int idx = tid; idx < MB * nrows; idx += kThreads) {
    const int m = idx / nrows, rl = idx - m * nrows;
    const float* pp = part + ((size_t)m * rows_cap + rl) * KR;
    float v = 0.0f;
    for (int kr = 0; kr < KR; ++kr) v += pp[kr];
    float sc = 1.0f;
#pragma unroll
    for (int mm = 0; mm < MB; ++mm) if (mm == m) sc = xscale[mm];
    if (FMT == QNT_INT8_PERCHAN) sc *= h2f(ldg_u16(meta + 2 * (r_lo + rl)));
    v *= sc;
    const size_t o = (size_t)m * ldy + r_lo + rl;
    if (xbf16) reinterpret_cast<__nv_bfloat16*>(Y)[o] = __float2bfloat16_rn(v);
    else reinterpret_cast<__half*>(Y)[o] = __float2half_rn(v);
  }
}

// ------------------------------------------------------------------ launchers
int num_sms() {
  static int sms[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) dev = 0;
  if (sms[dev] == 0) {
    int v = 0;
    cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
    sms[dev] = v > 0 ? v : 148;
  }
  return sms[dev];
}


cudaError_t configure_smem(const void* fn) {
  struct Entry { const void* fn; int dev; };
  static Entry done[256];
  static int ndone = 0;
  static std::mutex mu;
  std::lock_guard<std::mutex> lock(mu);
  int dev = 0;
  cudaGetDevice(&dev);
  for (int i = 0; i < ndone; ++i)
    if (done[i].fn == fn && done[i].dev == dev) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxDynSmem);
  if (e == cudaSuccess && ndone < 256) done[ndone++] = {fn, dev};
  return e;
}

static int simt_rows_cap(const qnt_desc& d, int grid) {
  if (d.fmt == QNT_INT8_PERCHAN || d.fmt == QNT_FP16) return (d.N + grid - 1) / grid;
  const int NG = (d.N + 7) / 8;
  return 8 * ((NG + grid - 1) / grid);
}

static int simt_grid(const qnt_desc& d) {
  const int units = (d.fmt == QNT_INT8_PERCHAN || d.fmt == QNT_FP16) ? d.N : (d.N + 7) / 8;
  return units < num_sms() ? units : num_sms();
}

static size_t simt_meta_bytes(const qnt_desc& d, int rows_cap) {
  const long GK = d.K / d.group;
  switch (d.fmt) {
    case QNT_INT4_ASYM: return meta_stage_bytes<QNT_INT4_ASYM>(rows_cap, GK);
    case QNT_FP4_E2M1: return meta_stage_bytes<QNT_FP4_E2M1>(rows_cap, GK);
    case QNT_FP4_AFPQ: return meta_stage_bytes<QNT_FP4_AFPQ>(rows_cap, GK);
    case QNT_FP4_RAZER: return meta_stage_bytes<QNT_FP4_RAZER>(rows_cap, GK);
    default: return 0;
  }
}

// Shared memory of a launch; *meta_bytes: the staged metadata copy, or 0 when
// it would not fit (the kernel then reads metadata from global memory).
static size_t simt_smem(const qnt_desc& d, int MB, int grid, size_t* meta_bytes) {
  const int rows_cap = simt_rows_cap(d, grid);
  size_t mb = simt_meta_bytes(d, rows_cap);
  size_t total = smem_simt_layout(d.fmt, MB, d.K, d.group, rows_cap, mb).total;
  if (total > (size_t)kMaxDynSmem) {
    mb = 0;
    total = smem_simt_layout(d.fmt, MB, d.K, d.group, rows_cap, 0).total;
  }
  if (meta_bytes) *meta_bytes = mb;
  return total;
}

size_t gemv_smem_bytes(const qnt_desc& d, int MB, int grid) { return simt_smem(d, MB, grid, nullptr); }

template <int FMT, int G, int MB>
static cudaError_t launch_simt(const qnt_desc& d, const void* codes, const void* meta, long z0, const void* X, void* Y,
                               int ldy, int xbf16, int* st, cudaStream_t s) {
  const int grid = simt_grid(d);
  size_t meta_bytes = 0;
  const size_t smem = simt_smem(d, MB, grid, &meta_bytes);
  auto kfn = gemv_simt_kernel<FMT, G, MB>;
  cudaError_t e = configure_smem(reinterpret_cast<const void*>(kfn));
  if (e != cudaSuccess) return e;
  const int rows_cap = simt_rows_cap(d, grid);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kfn, static_cast<const uint8_t*>(codes), static_cast<const uint8_t*>(meta), z0, X, Y,
                            d.N, d.K, ldy, xbf16, rows_cap, (int)meta_bytes, st);
}

template <int MB>
static cudaError_t dispatch_mb(const qnt_desc& d, const void* codes, const void* meta, long z0, const void* X, void* Y,
                               int ldy, int xbf16, int* st, cudaStream_t s) {
#define QNT_G(FMT)                                                                           \
  switch (d.group) {                                                                         \
    case 32: return launch_simt<FMT, 32, MB>(d, codes, meta, z0, X, Y, ldy, xbf16, st, s);   \
    case 64: return launch_simt<FMT, 64, MB>(d, codes, meta, z0, X, Y, ldy, xbf16, st, s);   \
    default: return launch_simt<FMT, 128, MB>(d, codes, meta, z0, X, Y, ldy, xbf16, st, s);  \
  }
  switch (d.fmt) {
    case QNT_INT4_ASYM: QNT_G(QNT_INT4_ASYM)
    case QNT_FP4_E2M1: QNT_G(QNT_FP4_E2M1)
    case QNT_FP4_AFPQ: QNT_G(QNT_FP4_AFPQ)
    case QNT_FP4_RAZER: QNT_G(QNT_FP4_RAZER)
    case QNT_INT8_PERCHAN: return launch_simt<QNT_INT8_PERCHAN, 0, MB>(d, codes, meta, z0, X, Y, ldy, xbf16, st, s);
    case QNT_FP16: return launch_simt<QNT_FP16, 0, MB>(d, codes, meta, z0, X, Y, ldy, xbf16, st, s);
    default: return cudaErrorInvalidValue;
  }
#undef QNT_G
}

// Largest vectors-per-pass whose staging fits in shared memory (0: none).
int gemv_max_mb(const qnt_desc& d) {
  const int grid = simt_grid(d);
  int best = 0;
  for (int mb : {1, 2, 4, 8})
    if (gemv_smem_bytes(d, mb, grid) <= (size_t)kMaxDynSmem) best = mb;
  return best;
}

cudaError_t launch_gemv_simt(const qnt_desc& d, const void* codes, const void* meta, long z0, const void* X, void* Y,
                             int M, int xbf16, int* st, cudaStream_t s) {
  const int mbmax = gemv_max_mb(d);
  if (mbmax < 1) return cudaErrorInvalidValue;   // K too large to stage one activation vector
  int m0 = 0;
  while (m0 < M) {
    const int left = M - m0;
    int mb = 1;
    for (int c : {8, 4, 2}) if (c <= mbmax && c <= left) { mb = c; break; }
    const void* Xm = static_cast<const uint8_t*>(X) + (size_t)m0 * d.K * 2;
    void* Ym = static_cast<uint8_t*>(Y) + (size_t)m0 * d.N * 2;
    cudaError_t e;
    switch (mb) {
      case 8: e = dispatch_mb<8>(d, codes, meta, z0, Xm, Ym, d.N, xbf16, st, s); break;
      case 4: e = dispatch_mb<4>(d, codes, meta, z0, Xm, Ym, d.N, xbf16, st, s); break;
      case 2: e = dispatch_mb<2>(d, codes, meta, z0, Xm, Ym, d.N, xbf16, st, s); break;
      default: e = dispatch_mb<1>(d, codes, meta, z0, Xm, Ym, d.N, xbf16, st, s); break;
    }
    if (e != cudaSuccess) return e;
    m0 += mb;
  }
  return cudaSuccess;
}

}  // namespace qnt
