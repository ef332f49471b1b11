// gemv.cu -- fused-dequant GEMV (batch 1) and CUDA-core multi-vector GEMV.
//
// The decode-time kernel the RTN page ("Is (Selective) Round-To-Nearest
// Quantization All You Need?", English abstract: token-generation throughput of
// RTN with fused-dequant kernels) and the RaZeR page ("The Power of Negative
// Zero", English abstract and method section: a GEMV that turns 4-bit codes
// into FP16 with bit-level operations, fused with the dot product) describe:
//   y[m][n] = sum_k dq(code[n][k], meta[n][k/g]) * x[m][k].
//
// B200 design.  One CTA of 16 warps per SM owns a contiguous range of rows.
//  * Weights stream HBM -> shared memory through per-warp rings of 1-D TMA bulk
//    copies (cp.async.bulk, mbarrier completion): bytes in flight cost no
//    registers, and every warp keeps its next items loading while it computes.
//  * Activations are staged once per CTA (one bulk copy), then each slot's 16
//    16-byte units are XOR-swizzled in place so that the 32 lanes of a warp,
//    which read the same unit of 32 different 128-weight slots, hit distinct
//    bank groups.
//  * A work item is (2 rows) x (32 slots of 128 weights); lane l owns slot
//    32*ks + l.  Items are dealt to warps round-robin; per-(row, K-step)
//    partial sums are combined in a fixed order, so results are deterministic.
//  * Dequantization in registers, products by the sm_100 mixed-precision FMA
//    (fma.rn.f32.f16: exact fp16 x fp16 product, fp32 accumulation):
//      INT4: a nibble masked into the low bits of an fp16 half is the fp16
//            subnormal q * 2^-24 (bits 4..7 give 16 q * 2^-24), exact; the
//            products q * x * 2^-24 are exact in fp32, so one LOP3 per two
//            weights plus one FMA per weight is the whole inner loop.  The
//            zero point is applied once per group as -z * sum(x over the
//            group), a per-CTA table shared by every row.
//      FP4 / RaZeR: cvt.rn.f16x2.e2m1x2 (two codes -> fp16x2); RaZeR codes
//            0b1000 (decoded as -0) are found with a nibble test and add
//            sv * x separately.  AFPQ splits positive / negative parts
//            (max / subtract) and applies s+ and s- per group.
//      INT8: PRMT into 0x64xx fp16 patterns and one subtract; FP16: direct.
#include <mutex>
#include "common.cuh"

namespace qnt {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kStages = 2;                  // ring depth per warp
constexpr int kRowChunkBytes = 512;         // one chunk of 32 slots / 512 bytes of a wide row
constexpr int kItemBytes = 2 * 4 * kRowChunkBytes;  // 2 rows x 4 chunks x 512 B
constexpr int kCtrlBytes = 1024;            // barriers + reduction scratch
constexpr int kRingBytes = kWarps * kStages * kItemBytes;

__device__ __forceinline__ void fence_proxy_async() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

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

// ------------------------------------------------------------------ metadata
struct Meta {
  float s[4];     // INT4: s * 2^24; FP4 / RaZeR: s; AFPQ: s+
  float t[4];     // INT4: s * z;   AFPQ: s-;  RaZeR: special value
};

template <int FMT, int G>
__device__ __forceinline__ void load_meta(const uint8_t* __restrict__ meta, long z0, long f0, Meta& m) {
  constexpr int NG = kSlot / G;
#pragma unroll
  for (int q = 0; q < NG; ++q) {
    const long f = f0 + q;
    if (FMT == QNT_FP4_AFPQ) {
      const uint32_t w = ldg_u32(meta + 4 * f);
      m.s[q] = h2f(w & 0xFFFFu);
      m.t[q] = h2f(w >> 16);
    } else {
      const float s = h2f(ldg_u16(meta + 2 * f));
      if (FMT == QNT_INT4_ASYM) {
        const uint32_t z = (ldg_u8(meta + z0 + f / 2) >> (4 * (f & 1))) & 15u;
        m.s[q] = s * 16777216.0f;          // 2^24 undoes the subnormal encoding
        m.t[q] = s * (float)z;
      } else if (FMT == QNT_FP4_RAZER) {
        const uint32_t sel = (ldg_u8(meta + z0 + f / 4) >> (2 * (f & 3))) & 3u;
        const float sv = (sel & 2u) ? 8.0f : 5.0f;
        m.s[q] = s;
        m.t[q] = (sel & 1u) ? -sv : sv;
      } else {
        m.s[q] = s;
        m.t[q] = 0.0f;
      }
    }
  }
}

// ------------------------------------------------------------------ per-word dot products
// acc[0..3]: fp32 accumulators.  INT4: [0,1] weights whose nibbles sit at bit 0
// of a half (x1), [2,3] nibbles at bit 4 (x16).  FP4 / RaZeR: [0,1].  AFPQ:
// [0,1] positive part, [2,3] negative part.
template <int FMT>
__device__ __forceinline__ void dot_word(uint32_t w, const uint4& x4, float (&acc)[4], uint32_t& spec) {
  if (FMT == QNT_INT4_ASYM) {
    const uint32_t w8 = w >> 8;
    fma_mixed2(w & 0x000F000Fu, x4.x, acc[0], acc[1]);    // weights 0,1: q * 2^-24
    fma_mixed2(w8 & 0x000F000Fu, x4.z, acc[0], acc[1]);   // weights 4,5
    fma_mixed2(w & 0x00F000F0u, x4.y, acc[2], acc[3]);    // weights 2,3: 16 q * 2^-24
    fma_mixed2(w8 & 0x00F000F0u, x4.w, acc[2], acc[3]);   // weights 6,7
  } else if (FMT == QNT_FP4_E2M1 || FMT == QNT_FP4_RAZER) {
    uint32_t h0, h1, h2, h3;
    cvt_e2m1x8(w, h0, h1, h2, h3);
    fma_mixed2(h0, x4.x, acc[0], acc[1]);
    fma_mixed2(h1, x4.y, acc[0], acc[1]);
    fma_mixed2(h2, x4.z, acc[0], acc[1]);
    fma_mixed2(h3, x4.w, acc[0], acc[1]);
    if (FMT == QNT_FP4_RAZER) {
      // nibbles equal to 0b1000: low three bits zero and the sign bit set
      const uint32_t t = (w & 0x77777777u) + 0x77777777u;
      spec = lop3<0x20>(w, t, 0x88888888u);   // w & ~t & 0x88888888
    }
  } else if (FMT == QNT_FP4_AFPQ) {
    uint32_t h[4];
    cvt_e2m1x8(w, h[0], h[1], h[2], h[3]);
    const uint32_t xv[4] = {x4.x, x4.y, x4.z, x4.w};
#pragma unroll
    for (int p = 0; p < 4; ++p) {
      const uint32_t vp = hmax2(h[p], 0u);
      const uint32_t vn = hsub2(h[p], vp);   // min(v, 0), exact
      fma_mixed2(vp, xv[p], acc[0], acc[1]);
      fma_mixed2(vn, xv[p], acc[2], acc[3]);
    }
  }
}

// ------------------------------------------------------------------ 4-bit kernel
// MB activation vectors per pass (MB = 1: the batch-1 GEMV).
template <int FMT, int G, int MB>
__global__ void __launch_bounds__(kThreads, 1)
gemv4_kernel(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ meta, long z0,
             const void* __restrict__ X, void* __restrict__ Y, int N, int K, int ldy, int xbf16,
             int rows_cap, int* d_status) {
  constexpr int NG = kSlot / G;
  extern __shared__ __align__(1024) uint8_t smem[];
  uint64_t* xbar = reinterpret_cast<uint64_t*>(smem);
  uint64_t* rbar = reinterpret_cast<uint64_t*>(smem + 64);              // [kWarps][kStages]
  float* red = reinterpret_cast<float*>(smem + 512);
  uint8_t* ring = smem + kCtrlBytes;                                    // [kWarps][kStages][kItemBytes]
  __half* xs = reinterpret_cast<__half*>(smem + kCtrlBytes + kRingBytes);      // [MB][K] (swizzled)
  const int S = K / kSlot;
  const int KS = (S + 31) / 32;
  float* xg = reinterpret_cast<float*>(xs + (size_t)MB * K);            // [MB][K/G] group sums of x
  float* part = xg + (size_t)MB * (K / G);                               // [MB][rows_cap][KS]

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const long r_lo = (long)blockIdx.x * N / gridDim.x;
  const long r_hi = (long)(blockIdx.x + 1) * N / gridDim.x;
  const int nrows = (int)(r_hi - r_lo);
  const int npairs = (nrows + 1) / 2;
  const int nitems = npairs * KS;
  const long rowbytes = K / 2;
  uint64_t* mybar = rbar + warp * kStages;
  uint8_t* myring = ring + (size_t)warp * kStages * kItemBytes;

  if (tid == 0) mbar_init(xbar, 1);
  if (lane == 0)
    for (int s = 0; s < kStages; ++s) mbar_init(mybar + s, 1);
  __syncthreads();
  if (tid == 0) {
    const uint32_t xbytes = (uint32_t)K * 2u;
    mbar_expect_tx(xbar, xbytes * MB);
    for (int m = 0; m < MB; ++m)
      bulk_g2s(xs + (size_t)m * K, static_cast<const uint8_t*>(X) + (size_t)m * xbytes, xbytes, xbar);
  }
  // item t -> stage: 2 rows x 4 chunks, each chunk = 16 * nsl bytes of 32 slots
  auto issue = [&](int t, int stage) {
    const int rp = t / KS, ks = t - rp * KS;
    const long ra = r_lo + 2 * rp;
    const int nrow = (ra + 1 < r_hi) ? 2 : 1;
    const int nsl = min(32, S - 32 * ks);
    const uint32_t cb = 16u * (uint32_t)nsl;
    mbar_expect_tx(mybar + stage, cb * 4u * (uint32_t)nrow);
    uint8_t* dst = myring + (size_t)stage * kItemBytes;
    for (int r = 0; r < nrow; ++r)
      for (int i = 0; i < 4; ++i)
        bulk_g2s(dst + (r * 4 + i) * kRowChunkBytes, codes + (ra + r) * rowbytes + 16L * ((long)i * S + 32 * ks), cb,
                 mybar + stage);
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

  // ---- group sums of x (INT4 zero points) and the in-place swizzle: one thread per slot
  for (int t = tid; t < MB * S; t += kThreads) {
    const int m = t / S, sl = t - m * S;
    uint4* base = reinterpret_cast<uint4*>(xs + (size_t)m * K + (size_t)sl * kSlot);
    const int sw = sl & 7;
    float gsum = 0.0f;
#pragma unroll
    for (int h = 0; h < 16; h += 8) {       // c ^ sw stays inside its half (sw < 8)
      uint4 v[8];
#pragma unroll
      for (int c = 0; c < 8; ++c) v[c] = base[h + c];
      if (FMT == QNT_INT4_ASYM) {
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const uint32_t u[4] = {v[c].x, v[c].y, v[c].z, v[c].w};
#pragma unroll
          for (int p = 0; p < 4; ++p) {
            const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&u[p]));
            gsum += f.x;
            gsum += f.y;
          }
          if (((h + c + 1) * 8) % G == 0) {  // last 16-byte unit of a group
            xg[(size_t)m * (K / G) + ((size_t)sl * kSlot + (h + c) * 8) / G] = gsum;
            gsum = 0.0f;
          }
        }
      }
      if (sw) {
#pragma unroll
        for (int c = 0; c < 8; ++c) base[h + (c ^ sw)] = v[c];
      }
    }
  }
  __syncthreads();

  // ---- main loop
  Meta mnext[2];
  auto meta_for = [&](int t, Meta (&mm)[2]) {
    const int rp = t / KS, ks = t - rp * KS;
    const long ra = r_lo + 2 * rp;
    const int slot = ks * 32 + lane;
    if (slot < S) {
      load_meta<FMT, G>(meta, z0, ra * (K / G) + (long)slot * NG, mm[0]);
      if (ra + 1 < r_hi) load_meta<FMT, G>(meta, z0, (ra + 1) * (K / G) + (long)slot * NG, mm[1]);
    }
  };
  if (warp < nitems) meta_for(warp, mnext);
  bool failed = false;
  int j = 0;
  for (int t = warp; t < nitems; t += kWarps, ++j) {
    const int stage = j % kStages;
    const uint32_t phase = (uint32_t)(j / kStages) & 1u;
    Meta md[2] = {mnext[0], mnext[1]};
    if (t + kWarps < nitems) meta_for(t + kWarps, mnext);
    const int rp = t / KS, ks = t - rp * KS;
    const int slot = ks * 32 + lane;
    const bool act = slot < S;
    const int sw = slot & 7;
    if (!mbar_wait(mybar + stage, phase)) { failed = true; break; }
    const uint8_t* st = myring + (size_t)stage * kItemBytes + 16 * lane;

    float ysum[2][MB];
#pragma unroll
    for (int r = 0; r < 2; ++r)
#pragma unroll
      for (int m = 0; m < MB; ++m) ysum[r][m] = 0.0f;
    if (act) {
      const __half* xslot = xs + (size_t)slot * kSlot;
      float acc[2][MB][4];
      float corr[2][MB];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        constexpr int CPG = G / kChunk;     // chunks per group
        const int q = i / CPG;
        if (i % CPG == 0) {
#pragma unroll
          for (int r = 0; r < 2; ++r)
#pragma unroll
            for (int m = 0; m < MB; ++m) {
              acc[r][m][0] = acc[r][m][1] = acc[r][m][2] = acc[r][m][3] = 0.0f;
              corr[r][m] = 0.0f;
            }
        }
        const uint4 ca = lds128(st + i * kRowChunkBytes);
        const uint4 cb = lds128(st + (4 + i) * kRowChunkBytes);
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
          const int unit = (4 * i + jj) ^ sw;
#pragma unroll
          for (int m = 0; m < MB; ++m) {
            const uint4 x4 = lds128(xslot + (size_t)m * K + 8 * unit);
#pragma unroll
            for (int r = 0; r < 2; ++r) {
              const uint32_t w = r == 0 ? (&ca.x)[jj] : (&cb.x)[jj];
              uint32_t spec = 0;
              dot_word<FMT>(w, x4, acc[r][m], spec);
              if (FMT == QNT_FP4_RAZER) {
                while (spec) {   // weights coded as the group's special value
                  const int bit = __ffs(spec) - 1;
                  spec &= spec - 1;
                  corr[r][m] += __half2float(xslot[(size_t)m * K + 8 * unit + (bit >> 2)]);
                }
              }
            }
          }
        }
        if (i % CPG == CPG - 1) {
#pragma unroll
          for (int r = 0; r < 2; ++r)
#pragma unroll
            for (int m = 0; m < MB; ++m) {
              const float* a = acc[r][m];
              float v;
              if (FMT == QNT_INT4_ASYM)
                v = md[r].s[q] * ((a[0] + a[1]) + 0.0625f * (a[2] + a[3])) -
                    md[r].t[q] * xg[(size_t)m * (K / G) + ((size_t)slot * kSlot) / G + q];
              else if (FMT == QNT_FP4_AFPQ) v = md[r].s[q] * (a[0] + a[1]) + md[r].t[q] * (a[2] + a[3]);
              else if (FMT == QNT_FP4_RAZER) v = md[r].s[q] * ((a[0] + a[1]) + md[r].t[q] * corr[r][m]);
              else v = md[r].s[q] * (a[0] + a[1]);
              ysum[r][m] += v;
            }
        }
      }
    }
    // ---- release the stage: every lane has consumed its shared-memory reads
    __syncwarp();
    if (lane == 0 && t + kStages * kWarps < nitems) {
      fence_proxy_async();
      issue(t + kStages * kWarps, stage);
    }
    // ---- reduce the two rows across the warp: halves exchange, then butterfly
#pragma unroll
    for (int m = 0; m < MB; ++m) {
      const bool upper = lane & 16;
      float keep = upper ? ysum[1][m] : ysum[0][m];
      const float send = upper ? ysum[0][m] : ysum[1][m];
      keep += __shfl_xor_sync(0xffffffffu, send, 16);
#pragma unroll
      for (int o = 8; o > 0; o >>= 1) keep += __shfl_xor_sync(0xffffffffu, keep, o);
      const int rl = 2 * rp + (upper ? 1 : 0);
      if ((lane & 15) == 0 && rl < nrows) part[((size_t)m * rows_cap + rl) * KS + ks] = keep;
    }
  }
  if (failed && lane == 0) {
    // a bulk copy did not complete within the bound: report, then give any copy
    // still in flight a bounded chance to land before the CTA exits
    report(d_status, QNT_ERR_TIMEOUT);
    for (int s = 0; s < kStages; ++s) { mbar_wait(mybar + s, 0); mbar_wait(mybar + s, 1); }
  }
  __syncthreads();

  // ---- epilogue: sum K-step partials in order, undo the activation scale, round, store
  for (int idx = tid; idx < MB * nrows; idx += kThreads) {
    const int m = idx / nrows, rl = idx - m * nrows;
    const float* pp = part + ((size_t)m * rows_cap + rl) * KS;
    float v = 0.0f;
    for (int ks = 0; ks < KS; ++ks) v += pp[ks];
    float sc = 1.0f;
#pragma unroll
    for (int mm = 0; mm < MB; ++mm) if (mm == m) sc = xscale[mm];
    v *= sc;
    const size_t o = (size_t)m * ldy + r_lo + rl;
    if (xbf16) reinterpret_cast<__nv_bfloat16*>(Y)[o] = __float2bfloat16_rn(v);
    else reinterpret_cast<__half*>(Y)[o] = __float2half_rn(v);
  }
}

// ------------------------------------------------------------------ INT8 / FP16 kernel
// Row-major codes.  Item = (2 rows) x (2048-byte range of each row); lane l
// reads 16-byte chunks l, l+32, l+64, l+96 of the range.
template <int FMT, int MB>
__global__ void __launch_bounds__(kThreads, 1)
gemv_wide_kernel(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ meta,
                 const void* __restrict__ X, void* __restrict__ Y, int N, int K, int ldy, int xbf16,
                 int rows_cap, int* d_status) {
  constexpr int WPC = (FMT == QNT_INT8_PERCHAN) ? 16 : 8;   // weights per 16-byte chunk
  constexpr int RANGE = 4 * kRowChunkBytes;                  // bytes of one row per item
  extern __shared__ __align__(1024) uint8_t smem[];
  uint64_t* xbar = reinterpret_cast<uint64_t*>(smem);
  uint64_t* rbar = reinterpret_cast<uint64_t*>(smem + 64);
  float* red = reinterpret_cast<float*>(smem + 512);
  uint8_t* ring = smem + kCtrlBytes;
  __half* xs = reinterpret_cast<__half*>(smem + kCtrlBytes + kRingBytes);
  const long rowbytes = (FMT == QNT_INT8_PERCHAN) ? (long)K : 2L * K;
  const int KR = (int)((rowbytes + RANGE - 1) / RANGE);
  float* part = reinterpret_cast<float*>(xs + (size_t)MB * K);   // [MB][rows_cap][KR]

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const long r_lo = (long)blockIdx.x * N / gridDim.x;
  const long r_hi = (long)(blockIdx.x + 1) * N / gridDim.x;
  const int nrows = (int)(r_hi - r_lo);
  const int npairs = (nrows + 1) / 2;
  const int nitems = npairs * KR;
  uint64_t* mybar = rbar + warp * kStages;
  uint8_t* myring = ring + (size_t)warp * kStages * kItemBytes;

  if (tid == 0) mbar_init(xbar, 1);
  if (lane == 0)
    for (int s = 0; s < kStages; ++s) mbar_init(mybar + s, 1);
  __syncthreads();
  if (tid == 0) {
    const uint32_t xbytes = (uint32_t)K * 2u;
    mbar_expect_tx(xbar, xbytes * MB);
    for (int m = 0; m < MB; ++m)
      bulk_g2s(xs + (size_t)m * K, static_cast<const uint8_t*>(X) + (size_t)m * xbytes, xbytes, xbar);
  }
  auto issue = [&](int t, int stage) {
    const int rp = t / KR, kr = t - rp * KR;
    const long ra = r_lo + 2 * rp;
    const int nrow = (ra + 1 < r_hi) ? 2 : 1;
    const long off = (long)kr * RANGE;
    const uint32_t nb = (uint32_t)min((long)RANGE, rowbytes - off);
    mbar_expect_tx(mybar + stage, nb * (uint32_t)nrow);
    uint8_t* dst = myring + (size_t)stage * kItemBytes;
    for (int r = 0; r < nrow; ++r) bulk_g2s(dst + r * RANGE, codes + (ra + r) * rowbytes + off, nb, mybar + stage);
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

  bool failed = false;
  int j = 0;
  for (int t = warp; t < nitems; t += kWarps, ++j) {
    const int stage = j % kStages;
    const uint32_t phase = (uint32_t)(j / kStages) & 1u;
    const int rp = t / KR, kr = t - rp * KR;
    const int nch = (int)(min((long)RANGE, rowbytes - (long)kr * RANGE) / 16);   // chunks in this range
    if (!mbar_wait(mybar + stage, phase)) { failed = true; break; }
    const uint8_t* st = myring + (size_t)stage * kItemBytes;
    float acc[2][MB][2];
#pragma unroll
    for (int r = 0; r < 2; ++r)
#pragma unroll
      for (int m = 0; m < MB; ++m) acc[r][m][0] = acc[r][m][1] = 0.0f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int ch = lane + 32 * i;
      if (ch < nch) {
        const uint4 va = lds128(st + 16 * ch);
        const uint4 vb = lds128(st + RANGE + 16 * ch);
        const long k0 = (long)kr * (RANGE / (16 / WPC)) + (long)ch * WPC;   // first weight of the chunk
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
      const int rl = 2 * rp + (upper ? 1 : 0);
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
static int num_sms() {
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

constexpr int kMaxDynSmem = 227 * 1024;

// Raise a kernel's dynamic shared-memory limit once (per process and device);
// later launches make no attribute calls, so they are safe inside stream capture.
static cudaError_t configure_smem(const void* fn) {
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

static bool wide_fmt(int f) { return f == QNT_INT8_PERCHAN || f == QNT_FP16; }

size_t gemv_smem_bytes(const qnt_desc& d, int MB, int grid) {
  const int rows_cap = (d.N + grid - 1) / grid;
  size_t b = (size_t)kCtrlBytes + kRingBytes + (size_t)MB * d.K * 2;
  if (wide_fmt(d.fmt)) {
    const long rowbytes = d.fmt == QNT_INT8_PERCHAN ? d.K : 2L * d.K;
    const int KR = (int)((rowbytes + 4 * kRowChunkBytes - 1) / (4 * kRowChunkBytes));
    b += (size_t)MB * rows_cap * KR * sizeof(float);
  } else {
    const int S = d.K / kSlot, KS = (S + 31) / 32;
    b += (size_t)MB * (d.K / d.group) * sizeof(float) + (size_t)MB * rows_cap * KS * sizeof(float);
  }
  return b;
}

template <int FMT, int G, int MB>
static cudaError_t launch4(const qnt_desc& d, const void* codes, const void* meta, long z0, const void* X, void* Y,
                           int ldy, int xbf16, int* st, cudaStream_t s) {
  const int grid = d.N < num_sms() ? d.N : num_sms();
  const size_t smem = gemv_smem_bytes(d, MB, grid);
  auto kfn = gemv4_kernel<FMT, G, MB>;
  cudaError_t e = configure_smem(reinterpret_cast<const void*>(kfn));
  if (e != cudaSuccess) return e;
  const int rows_cap = (d.N + grid - 1) / grid;
  kfn<<<grid, kThreads, smem, s>>>(static_cast<const uint8_t*>(codes), static_cast<const uint8_t*>(meta), z0, X, Y,
                                   d.N, d.K, ldy, xbf16, rows_cap, st);
  return cudaGetLastError();
}

template <int FMT, int MB>
static cudaError_t launch_wide(const qnt_desc& d, const void* codes, const void* meta, const void* X, void* Y,
                               int ldy, int xbf16, int* st, cudaStream_t s) {
  const int grid = d.N < num_sms() ? d.N : num_sms();
  const size_t smem = gemv_smem_bytes(d, MB, grid);
  auto kfn = gemv_wide_kernel<FMT, MB>;
  cudaError_t e = configure_smem(reinterpret_cast<const void*>(kfn));
  if (e != cudaSuccess) return e;
  const int rows_cap = (d.N + grid - 1) / grid;
  kfn<<<grid, kThreads, smem, s>>>(static_cast<const uint8_t*>(codes), static_cast<const uint8_t*>(meta), X, Y,
                                   d.N, d.K, ldy, xbf16, rows_cap, st);
  return cudaGetLastError();
}

template <int MB>
static cudaError_t dispatch_mb(const qnt_desc& d, const void* codes, const void* meta, long z0, const void* X, void* Y,
                               int ldy, int xbf16, int* st, cudaStream_t s) {
#define QNT_G(FMT)                                                                       \
  switch (d.group) {                                                                     \
    case 32: return launch4<FMT, 32, MB>(d, codes, meta, z0, X, Y, ldy, xbf16, st, s);   \
    case 64: return launch4<FMT, 64, MB>(d, codes, meta, z0, X, Y, ldy, xbf16, st, s);   \
    default: return launch4<FMT, 128, MB>(d, codes, meta, z0, X, Y, ldy, xbf16, st, s);  \
  }
  switch (d.fmt) {
    case QNT_INT4_ASYM: QNT_G(QNT_INT4_ASYM)
    case QNT_FP4_E2M1: QNT_G(QNT_FP4_E2M1)
    case QNT_FP4_AFPQ: QNT_G(QNT_FP4_AFPQ)
    case QNT_FP4_RAZER: QNT_G(QNT_FP4_RAZER)
    case QNT_INT8_PERCHAN: return launch_wide<QNT_INT8_PERCHAN, MB>(d, codes, meta, X, Y, ldy, xbf16, st, s);
    case QNT_FP16: return launch_wide<QNT_FP16, MB>(d, codes, meta, X, Y, ldy, xbf16, st, s);
    default: return cudaErrorInvalidValue;
  }
#undef QNT_G
}

// Largest vectors-per-pass whose staging fits in shared memory (0: none).
int gemv_max_mb(const qnt_desc& d) {
  const int grid = d.N < num_sms() ? d.N : num_sms();
  int best = 0;
  for (int mb : {1, 2, 4, 8})
    if (gemv_smem_bytes(d, mb, grid) <= (size_t)kMaxDynSmem) best = mb;
  return best;
}

// Y[m] = W x[m] for m < M, in passes of up to 8 vectors.
cudaError_t launch_gemv(const qnt_desc& d, const void* codes, const void* meta, long z0, const void* X, void* Y,
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
