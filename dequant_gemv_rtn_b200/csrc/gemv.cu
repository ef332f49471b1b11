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
// Metadata planes of the 4-bit formats (bytes per entry of plane A; bits per
// entry of plane B, the zero / selector plane starting at z0; 0 = none).
template <int FMT> struct MetaPlanes {
  static constexpr int A = (FMT == QNT_FP4_AFPQ) ? 4 : 2;
  static constexpr int B = (FMT == QNT_INT4_ASYM) ? 4 : (FMT == QNT_FP4_RAZER ? 2 : 0);
};

// 16-byte-aligned byte ranges of the metadata of rows [r_lo, r_hi) (G groups
// per row); every metadata buffer is padded to 16 bytes, so the ranges stay
// inside it.
struct MetaRange { long a0, a1, b0, b1; };
template <int FMT>
__host__ __device__ inline MetaRange meta_range(long r_lo, long r_hi, long G, long z0) {
  using MP = MetaPlanes<FMT>;
  MetaRange m;
  m.a0 = (MP::A * r_lo * G) & ~15L;
  m.a1 = (MP::A * r_hi * G + 15) & ~15L;
  if (MP::B) {
    m.b0 = (z0 + (r_lo * G * MP::B) / 8) & ~15L;
    m.b1 = (z0 + (r_hi * G * MP::B + 7) / 8 + 15) & ~15L;
  } else {
    m.b0 = m.b1 = 0;
  }
  return m;
}

struct GroupMeta {
  float s;   // INT4: s * 2^24; FP4 / RaZeR: s; AFPQ: s+
  float t;   // INT4: s * z;   AFPQ: s-;  RaZeR: special value
};

// Metadata of group f from the CTA's staged copy (ma: plane A, mb: plane B).
template <int FMT>
__device__ __forceinline__ GroupMeta group_meta(const uint8_t* ma, const uint8_t* mb, const MetaRange& mr, long z0,
                                                long f) {
  GroupMeta g;
  if (FMT == QNT_FP4_AFPQ) {
    const uint32_t w = lds_u32(ma + (4 * f - mr.a0));
    g.s = h2f(w & 0xFFFFu);
    g.t = h2f(w >> 16);
    return g;
  }
  const float s = h2f(lds_u16(ma + (2 * f - mr.a0)));
  if (FMT == QNT_INT4_ASYM) {
    const uint32_t z = (lds_u8(mb + (z0 + f / 2 - mr.b0)) >> (4 * (f & 1))) & 15u;
    g.s = s * 16777216.0f;     // 2^24 undoes the subnormal encoding
    g.t = s * (float)z;
  } else if (FMT == QNT_FP4_RAZER) {
    const uint32_t sel = (lds_u8(mb + (z0 + f / 4 - mr.b0)) >> (2 * (f & 3))) & 3u;
    const float sv = (sel & 2u) ? 8.0f : 5.0f;
    g.s = s;
    g.t = (sel & 1u) ? -sv : sv;
  } else {
    g.s = s;
    g.t = 0.0f;
  }
  return g;
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

// Shared-memory carve-up of the 4-bit kernel (byte offsets).
struct Smem4 {
  size_t xs, xg, part, ma, mb, total;
};
__host__ __device__ inline size_t align16(size_t v) { return (v + 15) & ~size_t(15); }
template <int FMT>
__host__ __device__ inline Smem4 smem4_layout(int MB, int K, int G, int rows_cap, int KS) {
  using MP = MetaPlanes<FMT>;
  Smem4 L;
  L.xs = kCtrlBytes + kRingBytes;
  L.xg = align16(L.xs + (size_t)MB * K * 2);
  L.part = align16(L.xg + (size_t)MB * G * 4);
  L.ma = align16(L.part + (size_t)MB * rows_cap * KS * 4);
  L.mb = align16(L.ma + (size_t)MP::A * rows_cap * G + 32);
  L.total = align16(L.mb + (MP::B ? ((size_t)rows_cap * G * MP::B + 7) / 8 + 48 : 0));
  return L;
}

// ------------------------------------------------------------------ 4-bit kernel
// MB activation vectors per pass (MB = 1: the batch-1 GEMV).  A work item is
// (2 rows) x (one 32-slot tile); its codes are one contiguous 2 KB run per row.
template <int FMT, int G, int MB>
__global__ void __launch_bounds__(kThreads, 1)
gemv4_kernel(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ meta, long z0,
             const void* __restrict__ X, void* __restrict__ Y, int N, int K, int ldy, int xbf16,
             int rows_cap, int* d_status) {
  constexpr int NG = kSlot / G;
  using MP = MetaPlanes<FMT>;
  extern __shared__ __align__(1024) uint8_t smem[];
  const int S = K / kSlot;
  const int KS = (S + 31) / 32;
  const int GK = K / G;
  const Smem4 L = smem4_layout<FMT>(MB, K, GK, rows_cap, KS);
  uint64_t* xbar = reinterpret_cast<uint64_t*>(smem);
  uint64_t* rbar = reinterpret_cast<uint64_t*>(smem + 64);              // [kWarps][kStages]
  float* red = reinterpret_cast<float*>(smem + 512);
  uint8_t* ring = smem + kCtrlBytes;                                    // [kWarps][kStages][kItemBytes]
  __half* xs = reinterpret_cast<__half*>(smem + L.xs);                  // [MB][K] (swizzled)
  float* xg = reinterpret_cast<float*>(smem + L.xg);                    // [MB][GK] group sums of x
  float* part = reinterpret_cast<float*>(smem + L.part);                // [MB][rows_cap][KS]
  uint8_t* ma = smem + L.ma;                                            // staged metadata plane A
  uint8_t* mb = smem + L.mb;                                            // staged metadata plane B

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const long r_lo = (long)blockIdx.x * N / gridDim.x;
  const long r_hi = (long)(blockIdx.x + 1) * N / gridDim.x;
  const int nrows = (int)(r_hi - r_lo);
  const int npairs = (nrows + 1) / 2;
  const long rowbytes = K / 2;
  const MetaRange mr = meta_range<FMT>(r_lo, r_hi, GK, z0);
  const bool whole_rows = (KS == 1 && S == 32);   // a tile is a whole row: 2 rows = 1 copy
  uint64_t* mybar = rbar + warp * kStages;
  uint8_t* myring = ring + (size_t)warp * kStages * kItemBytes;

  if (tid == 0) mbar_init(xbar, 1);
  if (lane == 0)
    for (int s = 0; s < kStages; ++s) mbar_init(mybar + s, 1);
  __syncthreads();
  if (tid == 0) {   // activations + this CTA's metadata, ahead of the weight copies
    const uint32_t xbytes = (uint32_t)K * 2u;
    mbar_expect_tx(xbar, xbytes * MB + (uint32_t)(mr.a1 - mr.a0) + (uint32_t)(mr.b1 - mr.b0));
    for (int m = 0; m < MB; ++m)
      bulk_g2s(xs + (size_t)m * K, static_cast<const uint8_t*>(X) + (size_t)m * xbytes, xbytes, xbar);
    bulk_g2s(ma, meta + mr.a0, (uint32_t)(mr.a1 - mr.a0), xbar);
    if (MP::B) bulk_g2s(mb, meta + mr.b0, (uint32_t)(mr.b1 - mr.b0), xbar);
  }
  const uint64_t pol = l2_evict_first_policy();
  // item cursor (row pair rp, tile ks) advanced by kWarps items at a time
  auto advance = [&](int& rp, int& ks) {
    ks += kWarps;
    while (ks >= KS) { ks -= KS; ++rp; }
  };
  auto issue = [&](int rp, int ks, int stage) {
    const long ra = r_lo + 2 * rp;
    const int nrow = (ra + 1 < r_hi) ? 2 : 1;
    const int nsl = min(32, S - 32 * ks);
    const uint32_t rb = 64u * (uint32_t)nsl;          // bytes of one row's tile
    mbar_expect_tx(mybar + stage, rb * (uint32_t)nrow);
    uint8_t* dst = myring + (size_t)stage * kItemBytes;
    const uint8_t* src = codes + ra * rowbytes + 2048L * ks;
    if (whole_rows) {
      bulk_g2s_hint(dst, src, rb * (uint32_t)nrow, mybar + stage, pol);
    } else {
      for (int r = 0; r < nrow; ++r) bulk_g2s_hint(dst + r * 2048, src + r * rowbytes, rb, mybar + stage, pol);
    }
  };
  int is_rp = 0, is_ks = 0;    // issue cursor: this warp's first item
  is_ks = warp;
  while (is_ks >= KS) { is_ks -= KS; ++is_rp; }
  const int first_rp = is_rp, first_ks = is_ks;
  int nissued = 0;
  if (lane == 0)
    for (int s = 0; s < kStages; ++s) {
      if (is_rp < npairs) { issue(is_rp, is_ks, s); ++nissued; }
      advance(is_rp, is_ks);
    }
  else
    for (int s = 0; s < kStages; ++s) advance(is_rp, is_ks);

  float xscale[MB];
  if (!stage_activations<MB>(xbar, red, xs, K, xbf16, xscale, d_status)) {
    if (lane == 0)
      for (int s = 0; s < nissued; ++s) mbar_wait(mybar + s, 0);
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
            xg[(size_t)m * GK + ((size_t)sl * kSlot + (h + c) * 8) / G] = gsum;
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

  // ---- main loop over this warp's items
  bool failed = false;
  int j = 0;
  for (int rp = first_rp, ks = first_ks; rp < npairs; advance(rp, ks), ++j) {
    const int stage = j % kStages;
    const uint32_t phase = (uint32_t)(j / kStages) & 1u;
    const int rl0 = 2 * rp;
    const int nsl = min(32, S - 32 * ks);
    const int slot = ks * 32 + lane;
    const bool act = lane < nsl;
    const int sw = slot & 7;
    GroupMeta md[2][NG];
#pragma unroll
    for (int r = 0; r < 2; ++r)
#pragma unroll
      for (int q = 0; q < NG; ++q) {
        md[r][q].s = md[r][q].t = 0.0f;
        if (act && rl0 + r < nrows)
          md[r][q] = group_meta<FMT>(ma, mb, mr, z0, (r_lo + rl0 + r) * GK + (long)slot * NG + q);
      }
    if (!mbar_wait(mybar + stage, phase)) { failed = true; break; }
    const uint8_t* st = myring + (size_t)stage * kItemBytes + 16 * lane;
    const int cstride = 16 * nsl;            // bytes between chunks of one row's tile

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
        const uint4 ca = lds128(st + i * cstride);
        const uint4 cb = lds128(st + 2048 + i * cstride);
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
                v = md[r][q].s * ((a[0] + a[1]) + 0.0625f * (a[2] + a[3])) -
                    md[r][q].t * xg[(size_t)m * GK + (size_t)slot * NG + q];
              else if (FMT == QNT_FP4_AFPQ) v = md[r][q].s * (a[0] + a[1]) + md[r][q].t * (a[2] + a[3]);
              else if (FMT == QNT_FP4_RAZER) v = md[r][q].s * ((a[0] + a[1]) + md[r][q].t * corr[r][m]);
              else v = md[r][q].s * (a[0] + a[1]);
              ysum[r][m] += v;
            }
        }
      }
    }
    // ---- release the stage: every lane has consumed its shared-memory reads
    __syncwarp();
    if (lane == 0 && is_rp < npairs) {
      fence_proxy_async();
      issue(is_rp, is_ks, stage);
      ++nissued;
    }
    advance(is_rp, is_ks);
    // ---- reduce the two rows across the warp: halves exchange, then butterfly
#pragma unroll
    for (int m = 0; m < MB; ++m) {
      const bool upper = lane & 16;
      float keep = upper ? ysum[1][m] : ysum[0][m];
      const float send = upper ? ysum[0][m] : ysum[1][m];
      keep += __shfl_xor_sync(0xffffffffu, send, 16);
#pragma unroll
      for (int o = 8; o > 0; o >>= 1) keep += __shfl_xor_sync(0xffffffffu, keep, o);
      const int rl = rl0 + (upper ? 1 : 0);
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

  // ---- epilogue: sum K-tile partials in order, undo the activation scale, round, store
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

// ------------------------------------------------------------------ 4-bit kernel, K <= 4096
// When a row fits in one tile (K <= 4096, S <= 32 slots) every lane owns the
// same slot in every row, so it keeps its 128 activations (and, for INT4, its
// group sums) in registers for the whole kernel.  Work item = one row; each
// warp streams its rows through a ring of row copies (deep enough, where shared
// memory allows, to request all of its rows at once) and writes each row's
// output itself, so the kernel has no closing barrier.  The activation and
// metadata copies are queued before any row copy, so the first row never waits
// behind the weight stream.
constexpr int kRowMaxStages = 8;       // ring depth per warp is chosen at launch, at most this
constexpr int kRowSlotBytes = 2048;   // ring slot: one row of at most 4096 weights
constexpr int kXPitch = 272;          // padded bytes per slot of activations (256 + 16)
constexpr int kRowCtrlBytes = 2048;   // barriers [1 + kWarps * kRowMaxStages] + reduction scratch

// Shared-memory carve-up of the row kernel (byte offsets), used by the kernel
// and by the launcher's size computation alike.  GK = groups per row; the ring
// (nst stages of one row per warp) comes last.
struct SmemRow { size_t xp, xg, ma, mb, ring, total; };
template <int FMT>
__host__ __device__ inline SmemRow smem_row_layout(int S, int GK, int rows_cap, int nst) {
  using MP = MetaPlanes<FMT>;
  SmemRow L;
  L.xp = kRowCtrlBytes;
  L.xg = align16(L.xp + (size_t)S * kXPitch);
  L.ma = align16(L.xg + (size_t)GK * 4);
  L.mb = L.ma + align16((size_t)MP::A * rows_cap * GK + 32);
  L.ring = align16(L.mb + (MP::B ? ((size_t)rows_cap * GK * MP::B + 7) / 8 + 48 : 0));
  L.total = L.ring + (size_t)kWarps * nst * kRowSlotBytes;
  return L;
}

template <int FMT, int G>
__global__ void __launch_bounds__(kThreads, 1)
gemv4_row_kernel(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ meta, long z0,
                 const void* __restrict__ X, void* __restrict__ Y, int N, int K, int xbf16, int rows_cap,
                 int nst, int* d_status) {
  constexpr int NG = kSlot / G;
  constexpr int RowBytes = kRowSlotBytes;
  constexpr int XPitch = kXPitch;
  using MP = MetaPlanes<FMT>;
  extern __shared__ __align__(1024) uint8_t smem[];
  const int S = K / kSlot;
  const int GK = K / G;                       // groups per row (G is the group size)
  const SmemRow L = smem_row_layout<FMT>(S, GK, rows_cap, nst);
  uint64_t* xbar = reinterpret_cast<uint64_t*>(smem);
  uint64_t* rbar = reinterpret_cast<uint64_t*>(smem + 64);              // [kWarps][nst]
  float* red = reinterpret_cast<float*>(smem + 64 + 8 * kWarps * kRowMaxStages);
  uint8_t* xp = smem + L.xp;                                            // [S][XPitch] activations
  float* xg = reinterpret_cast<float*>(smem + L.xg);                    // [GK] group sums of x (INT4)
  uint8_t* ma = smem + L.ma;                                            // staged metadata plane A
  uint8_t* mb = smem + L.mb;                                            // staged metadata plane B
  uint8_t* ring = smem + L.ring;                                        // [kWarps][nst][RowBytes]

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const long r_lo = (long)blockIdx.x * N / gridDim.x;
  const long r_hi = (long)(blockIdx.x + 1) * N / gridDim.x;
  const int nrows = (int)(r_hi - r_lo);
  const long rowbytes = K / 2;
  const MetaRange mr = meta_range<FMT>(r_lo, r_hi, GK, z0);
  uint64_t* mybar = rbar + warp * nst;
  uint8_t* myring = ring + (size_t)warp * nst * RowBytes;

  if (tid == 0) mbar_init(xbar, 1);
  if (lane == 0)
    for (int s = 0; s < nst; ++s) mbar_init(mybar + s, 1);
  __syncthreads();
  if (warp == 0) {   // activations (one 256-byte copy per slot, padded pitch) + this CTA's metadata
    if (lane == 0)
      mbar_expect_tx(xbar, (uint32_t)K * 2u + (uint32_t)(mr.a1 - mr.a0) + (uint32_t)(mr.b1 - mr.b0));
    __syncwarp();
    if (lane < S) bulk_g2s(xp + (size_t)lane * XPitch, static_cast<const uint8_t*>(X) + 256 * lane, 256u, xbar);
    if (lane == 0) {
      bulk_g2s(ma, meta + mr.a0, (uint32_t)(mr.a1 - mr.a0), xbar);
      if (MP::B) bulk_g2s(mb, meta + mr.b0, (uint32_t)(mr.b1 - mr.b0), xbar);
    }
  }
  __syncthreads();   // the activation / metadata copies enter the copy queue before any row copy
  const uint64_t pol = l2_evict_first_policy();
  auto issue = [&](int rl, int stage) {
    mbar_expect_tx(mybar + stage, (uint32_t)rowbytes);
    bulk_g2s_hint(myring + (size_t)stage * RowBytes, codes + (r_lo + rl) * rowbytes, (uint32_t)rowbytes,
                  mybar + stage, pol);
  };
  int nissued = 0;
  if (lane == 0)
    for (int s = 0; s < nst; ++s)
      if (warp + s * kWarps < nrows) { issue(warp + s * kWarps, s); ++nissued; }

  // ---- activations landed?  (bounded wait; on timeout no copy may be left in flight)
  const bool ok = mbar_wait(xbar, 0);
  if (__syncthreads_or(!ok)) {
    if (tid == 0) report(d_status, QNT_ERR_TIMEOUT);
    mbar_wait(xbar, 0);
    if (lane == 0)
      for (int s = 0; s < nissued; ++s) mbar_wait(mybar + s, 0);
    return;
  }
  // bf16 activations: exact power-of-two rescale into fp16 range, in place
  float xscale = 1.0f;
  if (xbf16) {
    float am = 0.0f;
    for (int k = tid; k < K; k += kThreads) {
      const uint16_t b = *reinterpret_cast<const uint16_t*>(xp + (k >> 7) * XPitch + 2 * (k & 127));
      am = fmaxf(am, fabsf(__uint_as_float((uint32_t)b << 16)));
    }
    am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 16));
    am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 8));
    am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 4));
    am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 2));
    am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 1));
    if (lane == 0) red[warp] = am;
    __syncthreads();
    am = red[0];
    for (int i = 1; i < kWarps; ++i) am = fmaxf(am, red[i]);
    int e = 0;
    if (am > 0.0f && isfinite(am)) e = min(max(ilogbf(am) - 14, -100), 100);
    const float down = __int_as_float((127 - e) << 23);
    xscale = __int_as_float((127 + e) << 23);
    for (int k = tid; k < K; k += kThreads) {
      uint16_t* p = reinterpret_cast<uint16_t*>(xp + (k >> 7) * XPitch + 2 * (k & 127));
      *p = __half_as_ushort(__float2half_rn(__uint_as_float((uint32_t)*p << 16) * down));
    }
    __syncthreads();
  }
  // INT4 zero points need the sum of x over each group: computed once per CTA
  // (one thread per 8 activations, groups summed in a fixed order)
  if (FMT == QNT_INT4_ASYM) {
    for (int gi = tid; gi < GK; gi += kThreads) {
      float sum = 0.0f;
      const int k0 = gi * G;
      for (int u = 0; u < G / 8; ++u) {
        const int k = k0 + 8 * u;
        const uint4 v = lds128(xp + (size_t)(k >> 7) * XPitch + 2 * (k & 127));
        const uint32_t uu[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int p = 0; p < 4; ++p) {
          const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&uu[p]));
          sum += f.x;
          sum += f.y;
        }
      }
      xg[gi] = sum;
    }
    __syncthreads();
  }
  // this lane's slot: 128 activations in registers, plus its group sums
  const bool act = lane < S;
  uint4 xr[16];
  float xgs[NG];
#pragma unroll
  for (int q = 0; q < NG; ++q) xgs[q] = (FMT == QNT_INT4_ASYM && act) ? xg[lane * NG + q] : 0.0f;
#pragma unroll
  for (int u = 0; u < 16; ++u) xr[u] = act ? lds128(xp + (size_t)lane * XPitch + 16 * u) : make_uint4(0, 0, 0, 0);

  bool failed = false;
  int j = 0;
  for (int rl = warp; rl < nrows; rl += kWarps, ++j) {
    const int stage = j % nst;
    const uint32_t phase = (uint32_t)(j / nst) & 1u;
    const long row = r_lo + rl;
    GroupMeta md[NG];
#pragma unroll
    for (int q = 0; q < NG; ++q) {
      md[q].s = md[q].t = 0.0f;
      if (act) md[q] = group_meta<FMT>(ma, mb, mr, z0, row * GK + (long)lane * NG + q);
    }
    if (!mbar_wait(mybar + stage, phase)) { failed = true; break; }
    const uint8_t* st = myring + (size_t)stage * RowBytes + 16 * lane;
    float ysum = 0.0f;
    if (act) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        constexpr int CPG = G / kChunk;
        const int q = i / CPG;
        float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
        float corr = 0.0f;
        const uint4 c = lds128(st + i * 16 * S);
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
          uint32_t spec = 0;
          dot_word<FMT>((&c.x)[jj], xr[4 * i + jj], acc, spec);
          if (FMT == QNT_FP4_RAZER) {
            while (spec) {   // weights coded as the group's special value
              const int bit = __ffs(spec) - 1;
              spec &= spec - 1;
              const uint16_t xb =
                  *reinterpret_cast<const uint16_t*>(xp + (size_t)lane * XPitch + 2 * (32 * i + 8 * jj + (bit >> 2)));
              corr += __half2float(__ushort_as_half(xb));
            }
          }
        }
        // chunk partial scaled by its group's metadata (linear in the group sum)
        float v;
        if (FMT == QNT_INT4_ASYM) {
          v = md[q].s * ((acc[0] + acc[1]) + 0.0625f * (acc[2] + acc[3]));
          if (i % CPG == CPG - 1) v -= md[q].t * xgs[q];
        } else if (FMT == QNT_FP4_AFPQ) {
          v = md[q].s * (acc[0] + acc[1]) + md[q].t * (acc[2] + acc[3]);
        } else if (FMT == QNT_FP4_RAZER) {
          v = md[q].s * ((acc[0] + acc[1]) + md[q].t * corr);
        } else {
          v = md[q].s * (acc[0] + acc[1]);
        }
        ysum += v;
      }
    }
    __syncwarp();
    const int next = rl + nst * kWarps;
    if (lane == 0 && next < nrows) {
      fence_proxy_async();
      issue(next, stage);
      ++nissued;
    }
    ysum = warp_sum(ysum);
    if (lane == 0) {
      const float v = ysum * xscale;
      if (xbf16) reinterpret_cast<__nv_bfloat16*>(Y)[row] = __float2bfloat16_rn(v);
      else reinterpret_cast<__half*>(Y)[row] = __float2half_rn(v);
    }
  }
  if (failed && lane == 0) {
    report(d_status, QNT_ERR_TIMEOUT);
    for (int s = 0; s < nst; ++s) { mbar_wait(mybar + s, 0); mbar_wait(mybar + s, 1); }
  }
}

template <int FMT>
static size_t smem_row_bytes(const qnt_desc& d, int grid, int nst) {
  const int rows_cap = (d.N + grid - 1) / grid;
  return smem_row_layout<FMT>(d.K / kSlot, d.K / d.group, rows_cap, nst).total;
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
  const uint64_t pol = l2_evict_first_policy();
  auto issue = [&](int t, int stage) {
    const int rp = t / KR, kr = t - rp * KR;
    const long ra = r_lo + 2 * rp;
    const int nrow = (ra + 1 < r_hi) ? 2 : 1;
    const long off = (long)kr * RANGE;
    const uint32_t nb = (uint32_t)min((long)RANGE, rowbytes - off);
    mbar_expect_tx(mybar + stage, nb * (uint32_t)nrow);
    uint8_t* dst = myring + (size_t)stage * kItemBytes;
    for (int r = 0; r < nrow; ++r)
      bulk_g2s_hint(dst + r * RANGE, codes + (ra + r) * rowbytes + off, nb, mybar + stage, pol);
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

template <int FMT>
static size_t smem4_bytes(const qnt_desc& d, int MB, int grid) {
  const int rows_cap = (d.N + grid - 1) / grid;
  const int S = d.K / kSlot, KS = (S + 31) / 32;
  return smem4_layout<FMT>(MB, d.K, d.K / d.group, rows_cap, KS).total;
}

size_t gemv_smem_bytes(const qnt_desc& d, int MB, int grid) {
  const int rows_cap = (d.N + grid - 1) / grid;
  if (wide_fmt(d.fmt)) {
    const long rowbytes = d.fmt == QNT_INT8_PERCHAN ? d.K : 2L * d.K;
    const int KR = (int)((rowbytes + 4 * kRowChunkBytes - 1) / (4 * kRowChunkBytes));
    return (size_t)kCtrlBytes + kRingBytes + (size_t)MB * d.K * 2 + (size_t)MB * rows_cap * KR * sizeof(float);
  }
  switch (d.fmt) {
    case QNT_INT4_ASYM: return smem4_bytes<QNT_INT4_ASYM>(d, MB, grid);
    case QNT_FP4_AFPQ: return smem4_bytes<QNT_FP4_AFPQ>(d, MB, grid);
    case QNT_FP4_RAZER: return smem4_bytes<QNT_FP4_RAZER>(d, MB, grid);
    default: return smem4_bytes<QNT_FP4_E2M1>(d, MB, grid);
  }
}

// Grid for a pass: one CTA per SM, or (when the per-CTA metadata would not
// fit) a multiple of the SM count so that each CTA holds fewer rows.
static int gemv_grid(const qnt_desc& d, int MB) {
  int grid = d.N < num_sms() ? d.N : num_sms();
  while (gemv_smem_bytes(d, MB, grid) > (size_t)kMaxDynSmem && grid < d.N && grid < 64 * num_sms()) grid *= 2;
  if (grid > d.N) grid = d.N;
  return grid;
}

template <int FMT, int G>
static cudaError_t launch_row(const qnt_desc& d, const void* codes, const void* meta, long z0, const void* X, void* Y,
                              int xbf16, int* st, cudaStream_t s) {
  int grid = d.N < num_sms() ? d.N : num_sms();
  while (smem_row_bytes<FMT>(d, grid, 2) > (size_t)kMaxDynSmem && grid < d.N) grid = grid * 2 < d.N ? grid * 2 : d.N;
  const int rows_cap = (d.N + grid - 1) / grid;
  // ring depth: enough stages to request all of a warp's rows at once, as far as
  // shared memory allows (at least 2, at most kRowMaxStages)
  int nst = (rows_cap + kWarps - 1) / kWarps;
  nst = nst < 2 ? 2 : (nst > kRowMaxStages ? kRowMaxStages : nst);
  while (nst > 2 && smem_row_bytes<FMT>(d, grid, nst) > (size_t)kMaxDynSmem) --nst;
  const size_t smem = smem_row_bytes<FMT>(d, grid, nst);
  auto kfn = gemv4_row_kernel<FMT, G>;
  cudaError_t e = configure_smem(reinterpret_cast<const void*>(kfn));
  if (e != cudaSuccess) return e;
  kfn<<<grid, kThreads, smem, s>>>(static_cast<const uint8_t*>(codes), static_cast<const uint8_t*>(meta), z0, X, Y,
                                   d.N, d.K, xbf16, rows_cap, nst, st);
  return cudaGetLastError();
}

template <int FMT, int G, int MB>
static cudaError_t launch4(const qnt_desc& d, const void* codes, const void* meta, long z0, const void* X, void* Y,
                           int ldy, int xbf16, int* st, cudaStream_t s) {
  // a single activation vector and rows of at most one tile: the row kernel
  if (MB == 1 && d.K <= 32 * kSlot) return launch_row<FMT, G>(d, codes, meta, z0, X, Y, xbf16, st, s);
  const int grid = gemv_grid(d, MB);
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
  int best = 0;
  for (int mb : {1, 2, 4, 8})
    if (gemv_smem_bytes(d, mb, gemv_grid(d, mb)) <= (size_t)kMaxDynSmem) best = mb;
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
