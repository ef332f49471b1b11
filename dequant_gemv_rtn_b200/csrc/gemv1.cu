// gemv1.cu -- batch-1 fused-dequant GEMV for the 4-bit formats on the tensor
// cores (mma.sync), launched once per GEMV (qnt_gemv), once for a whole
// sequence of GEMVs (qnt_gemv_seq, a persistent kernel), or once for 2 to 8
// activation vectors (qnt_gemm).
//
// What it computes is the decode-time GEMV of the RTN page ("Is (Selective)
// Round-To-Nearest Quantization All You Need?", English abstract: token
// generation with fused-dequant RTN kernels) and of the RaZeR page ("The Power
// of Negative Zero", English abstract and method section: a GEMV that turns
// 4-bit codes into FP16 with bit operations inside the product):
//   y[n] = sum_k dq(code[n][k], meta[n][k/g]) * x[k].
//
// Structure (one CTA of 16 warps per SM; every warp computes):
//  * A work item is one row group of eight rows x 8 blocks of 128 weights of
//    K (4 KB), one contiguous run of the packed layout.  Each
//    warp takes every 16th item of the CTA and keeps the next few of its own
//    items in flight in a small ring of its own, issued with 1-D bulk copies
//    (TMA) by its lane 0: no warp waits for another to fetch, and the copies of
//    a warp's next items, those of the next GEMV of a sequence included, are
//    under way while it computes, so weights keep streaming while a GEMV ends.
//  * MMA mapping (mma.sync m16n8k16, fp16 in, fp32 accumulate): lane 4g + r holds
//    chunk r (16 bytes) of row g of a block; word j of the chunk is MMA j's A
//    fragment (row g: the word's first K segment, row g + 8: its second), so a
//    lane spends five bit operations on the A operand of eight INT4 weights
//    (fp16 subnormals q 2^-24; bits 4..7 meet x / 16 in B) or four cvt on FP4.
//  * Blocks are processed in sets of S = 4 / (128 / g) blocks that share the
//    B registers: the B column pair hp = lane / 8 belongs to block hp / (128/g)
//    of the set (group hp % (128/g)), and each block of the set has its own
//    accumulator.  So a lane loads its activations once per set, the four
//    column pairs are all useful for g = 128, and after the set lane 4g + r
//    finds, in accumulator r / (128/g), row g's dot product over one
//    (block, group) pair: the scale / zero-point epilogue runs once per set in
//    all 32 lanes.  The products that pair one block's weights with another
//    block's activations land in accumulator entries that are never read.
//  * Activations: each warp reads its blocks of x from global memory (at L2:
//    in a sequence another SM may have just written x) and writes them as the
//    B-operand image (each block scaled by an exact power of two that puts its
//    maximum in [2^14, 2^15), undone in fp32 by the epilogue) with, per
//    (block, group), the scale factor and the group sum of x (INT4 zero point:
//    -s z sum x).
//  * Sequence: each step may wait for every earlier step of the launch (its x is
//    then an earlier step's y): one thread polls the per-step completion
//    counters in the caller's workspace (acquire), and each CTA bumps the counter
//    of a step after storing its rows of y (release).  The counters need every
//    CTA resident: the sequence kernel is a cooperative launch.
//  * qnt_gemv: the same kernel with one step and programmatic dependent launch;
//    the weights are requested before griddepcontrol.wait, the activations
//    after it.
//  * qnt_gemm with 2 to 8 vectors (template parameter MV = 2, 4, 8; g = 128, K a
//    multiple of 1024): the B column pairs that batch 1 spends on several blocks
//    of one vector carry the vectors instead (MV = 8: two B operands per decoded
//    word), each vector with its own image, factor table and partial sums, so
//    the decode and the codes traffic per weight stay those of batch 1.
// Every wait is bounded by the global timer; on expiry the kernel reports
// QNT_ERR_TIMEOUT, stops issuing work, drains its copies and returns.
#include <cstring>
#include <mutex>
#include "common.cuh"
#include "gemv_common.cuh"
#include "kernels.h"

namespace qnt {

constexpr int kB1Blocks = 8;                     // blocks of 128 weights per work item (4 KB)
constexpr int kB1Warps = 16;
constexpr int kB1Threads = 32 * kB1Warps;
constexpr int kB1MaxDepth = 8;                   // ring slots per warp, at most
constexpr int kB1Ctrl = 2048;                    // barriers and flags
constexpr unsigned long long kB1TimeoutNs = 2000000000ull;   // 2 s per wait

struct B1Step {
  const uint8_t* codes;
  const uint8_t* meta;
  const void* x;
  void* y;
  long z0;       // zero / selector plane offset in meta
  int N, K;
  int wait;      // k >= 1: read x only after step (this - k) and every step before it have stored y
  int rot;       // rotation of the row-group split over the CTAs (balances remainders)
  int NG, KB, KBR, GK;   // row groups, blocks and item runs per row, groups per row
  int rows_cap;  // rows of the busiest CTA
  int reuse_x;   // 1: x is the previous step's x and cannot have changed since: keep its image
};

template <int MAXS>
struct B1Params {
  B1Step s[MAXS];
  int nsteps;
  int xbf16;
  int depth;        // ring slots per warp
  int kmax;
  int meta_cap;     // bytes of one staged metadata window
  int part_cap;     // floats of the per-row partial-sum table
  int fault;        // test builds only: an injected fault (0: none)
  unsigned* done;   // [nsteps] completion counters, then one abort word (sequence only)
  int* status;
  unsigned long long timeout_ns;
  int nvec;         // activation vectors of a several-vector launch (MV > 1), else 1
};

// The weight rings, the activation image with its table of per-(block, group)
// factors, the per-row partial sums and the staged metadata window.
// With mv activation vectors (several-vector launches) the image, the factor
// table and the partial sums are held once per vector, one after another.
struct B1Smem { size_t ring, ximg, xs2, part, meta, total; };
constexpr int kB1SlotBytes = kB1Blocks * 512;
__host__ __device__ inline B1Smem b1_smem(int depth, int kmax, int gpb, int part_cap, int meta_cap, int mv = 1) {
  B1Smem L;
  L.ring = kB1Ctrl;
  L.ximg = L.ring + (size_t)kB1Warps * depth * kB1SlotBytes;
  L.xs2 = align16(L.ximg + (size_t)mv * kmax * 2);
  L.part = align16(L.xs2 + (size_t)mv * (kmax / 128) * gpb * 8);
  L.meta = align16(L.part + (size_t)mv * part_cap * 4);
  L.total = align16(L.meta + (size_t)meta_cap);
  return L;
}

// Rows [lo, hi) of the CTA in a step: whole row groups of eight, a balanced
// split of the N/8 row groups over the grid, rotated by `rot`.
__host__ __device__ inline void b1_rows(long N, int cta, int grid, int rot, long* lo, long* hi) {
  const long NG = (N + 7) / 8;
  const long c = (cta + rot) % grid;
  *lo = 8 * (c * NG / grid);
  const long h = 8 * ((c + 1) * NG / grid);
  *hi = h < N ? h : N;
}
__host__ __device__ inline int b1_rows_cap(long N, int grid) { return (int)(8 * (((N + 7) / 8 + grid - 1) / grid)); }
// The same split from a step's constants, in 32-bit arithmetic (NG < 2^22, grid < 2^10).
__device__ __forceinline__ void b1_rows_s(const B1Step& st, int cta, int grid, int* lo, int* hi) {
  int c = cta + st.rot;
  if (c >= grid) c -= grid;
  *lo = 8 * (c * st.NG / grid);
  const int h = 8 * ((c + 1) * st.NG / grid);
  *hi = h < st.N ? h : st.N;
}

// ------------------------------------------------------------------ device helpers
__device__ __forceinline__ uint64_t gtimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Bounded wait for phase `parity` of an mbarrier: gives up `timeout` ns after
// the first unsuccessful try, or early when the CTA's abort flag is raised.
// Between tries the thread sleeps ~32 ns (a suspend-time hint on try_wait
// instead was measured to wake threads up to microseconds after the phase
// completed; this form measured 1.4 % faster on the decode stack).
__device__ __forceinline__ bool mbar_wait_to(uint64_t* bar, uint32_t parity, uint64_t timeout, volatile int* abort_s) {
  const uint32_t a = smem_addr(bar);
  uint64_t deadline = 0;
  for (;;) {
    uint32_t done;
    asm volatile("{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\tselp.u32 %0, 1, 0, p;\n\t}"
                 : "=r"(done) : "r"(a), "r"(parity) : "memory");
    if (done) return true;
    if (abort_s && *abort_s) return false;
    const uint64_t now = gtimer();
    if (deadline == 0) deadline = now + timeout;
    else if (now > deadline) return false;
    __nanosleep(32);
  }
}

__device__ __forceinline__ unsigned ld_acquire_gpu(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void consumer_bar(int nthreads) {
  asm volatile("bar.sync 1, %0;" :: "r"(nthreads) : "memory");
}
// Barrier of the consumer warps that also ORs a flag over them, so that every
// consumer takes the same decision (the producer may raise the abort flag at
// any time, and a plain read after a barrier could differ between warps).
__device__ __forceinline__ bool consumer_bar_or(int nthreads, bool flag) {
  uint32_t r;
  asm volatile("{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\t"
               "bar.red.or.pred q, 1, %2, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
               : "=r"(r) : "r"((uint32_t)flag), "r"(nthreads) : "memory");
  return r != 0;
}

// D = A B (no accumulator input)
__device__ __forceinline__ void mma_16816_z(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                            uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%10,%10,%10,%10};"
      : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "f"(0.0f));
}
// D += A B
__device__ __forceinline__ void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                          uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Byte offset in the activation image of the B entry for block b, chunk r,
// segment s, MMA j, half hf (b0: hf = 0, b1: hf = 1).  A lane reads its (s, r)
// entry of a block with two 16-byte loads (MMAs 0, 1 and 2, 3).
__device__ __forceinline__ uint32_t xf_off(int b, int r, int s, int j, int hf) {
  return (uint32_t)(256 * b + 128 * (j >> 1) + 16 * (4 * s + r) + 8 * (j & 1) + 4 * hf);
}

// Build blocks b0 and b1 (b1 < 0: none) of the B-operand image at ximg from the
// activations in global memory (read at L2, since they may have just been
// written by other CTAs).  Lane l takes x[128b + 4l .. 4l + 3].  The weight at chunk
// offset o = 16 hf + 4j + 2s + e (INT4) or 8j + 4hf + 2s + e (FP4 family) meets
// B half hf, segment s of MMA j.  Per (block, group h) xs2 gets (c / 2^e, sum of x
// over the group), c = 2^24 for INT4 (undoes the subnormal encoding), else 1.
template <int FMT, int G>
__device__ __forceinline__ void build_x(const uint8_t* xg, uint32_t ximg, uint32_t xs2, int b0, int b1, int xbf16,
                                        int lane, bool zero = false) {
  constexpr int GPB = 128 / G;
  const int bb[2] = {b0, b1 >= 0 ? b1 : b0};
  float v[2][4], sg[2];
  uint32_t am[2];
  uint2 raws[2];
#pragma unroll
  for (int q = 0; q < 2; ++q)   // L2: x may be another CTA's y; zero: an image of zeros (no vector)
    raws[q] = zero ? make_uint2(0u, 0u) : ldg_cg64(xg + 256 * bb[q] + 8 * lane);
#pragma unroll
  for (int q = 0; q < 2; ++q) {
    const uint2 raw = raws[q];
    if (xbf16) {
      v[q][0] = __uint_as_float(raw.x << 16); v[q][1] = __uint_as_float(raw.x & 0xFFFF0000u);
      v[q][2] = __uint_as_float(raw.y << 16); v[q][3] = __uint_as_float(raw.y & 0xFFFF0000u);
    } else {
      v[q][0] = h2f(raw.x & 0xFFFFu); v[q][1] = h2f(raw.x >> 16);
      v[q][2] = h2f(raw.y & 0xFFFFu); v[q][3] = h2f(raw.y >> 16);
    }
    // |x| bit patterns order like the magnitudes (non-negative floats)
    const uint32_t m01 = max(__float_as_uint(v[q][0]) & 0x7FFFFFFFu, __float_as_uint(v[q][1]) & 0x7FFFFFFFu);
    const uint32_t m23 = max(__float_as_uint(v[q][2]) & 0x7FFFFFFFu, __float_as_uint(v[q][3]) & 0x7FFFFFFFu);
    am[q] = __reduce_max_sync(0xffffffffu, max(m01, m23));
    sg[q] = (v[q][0] + v[q][1]) + (v[q][2] + v[q][3]);
  }
  if (FMT == QNT_INT4_ASYM) {
#pragma unroll
    for (int o = 1; o < G / 4; o <<= 1)
#pragma unroll
      for (int q = 0; q < 2; ++q) sg[q] += __shfl_xor_sync(0xffffffffu, sg[q], o);
  }
  __syncwarp();
  const int r = lane >> 3, o = 4 * (lane & 7);
  int j, hf;
  if (FMT == QNT_INT4_ASYM) {
    hf = o >> 4;
    j = (o & 15) >> 2;
  } else {
    j = o >> 3;
    hf = (o >> 2) & 1;
  }
#pragma unroll
  for (int q = 0; q < 2; ++q) {
    if (q == 1 && b1 < 0) break;
    int e = 0;
    const uint32_t ex = (am[q] >> 23) & 255u;
    if (am[q] != 0u && ex != 255u) e = min(max(14 - (int)ex + 127, -126), 126);
    const float f = __uint_as_float((uint32_t)(127 + e) << 23);
    const float fs = (FMT == QNT_INT4_ASYM && hf) ? f * 0.0625f : f;   // INT4 bits 4..7 decode 16x too large
    const __half2 p0 = __floats2half2_rn(v[q][0] * fs, v[q][1] * fs), p1 = __floats2half2_rn(v[q][2] * fs, v[q][3] * fs);
    sts32a(ximg + xf_off(bb[q], r, 0, j, hf), *reinterpret_cast<const uint32_t*>(&p0));
    sts32a(ximg + xf_off(bb[q], r, 1, j, hf), *reinterpret_cast<const uint32_t*>(&p1));
    if ((lane & (G / 4 - 1)) == 0)
      sts64fa(xs2 + 8 * (bb[q] * GPB + lane / (G / 4)),
              __uint_as_float((uint32_t)(127 - e) << 23) * (FMT == QNT_INT4_ASYM ? 16777216.0f : 1.0f),
              FMT == QNT_INT4_ASYM ? sg[q] : 0.0f);
  }
}

// Metadata of the CTA's rows from the staged shared copy, by window-relative
// group index fr = (row - r_lo) * K/g + group: ms_a addresses scale 0 of row
// r_lo, mz_a the byte of the zero / selector plane that holds group 0 of row
// r_lo (r_lo is a multiple of 8, so the nibble / 2-bit position of fr is that
// of the absolute group index).
struct MetaRef { uint32_t ms_a, mz_a; };
__device__ __forceinline__ float meta_scale(const MetaRef& M, uint32_t fr) { return h2f(lds16a(M.ms_a + 2u * fr)); }
__device__ __forceinline__ uint32_t meta_afpq(const MetaRef& M, uint32_t fr) { return lds32a(M.ms_a + 4u * fr); }
__device__ __forceinline__ uint32_t meta_zero4(const MetaRef& M, uint32_t fr) {
  return (lds8a(M.mz_a + (fr >> 1)) >> (4u * (fr & 1u))) & 15u;
}
__device__ __forceinline__ uint32_t meta_sel2(const MetaRef& M, uint32_t fr) {
  return (lds8a(M.mz_a + (fr >> 2)) >> (2u * (fr & 3u))) & 3u;
}

// Decode word j of a lane's chunk and run MMA j of its block into d (and, for
// AFPQ, the negative part into dn); MMA 0 starts the accumulators from zero.
// bx: the lane's eight B registers; sv16: RaZeR: twice the special value of this
// lane's chunk group, as an fp16 pair.
template <int FMT>
__device__ __forceinline__ void word_mma(uint32_t w, int j, const uint32_t (&bx)[8], float (&d)[4], float (&dn)[4],
                                         uint32_t sv16) {
  const uint32_t b0 = bx[2 * j], b1 = bx[2 * j + 1];
  if (FMT == QNT_INT4_ASYM) {
    const uint32_t w8 = w >> 8;
    if (j == 0) mma_16816_z(d, w & 0x000F000Fu, w8 & 0x000F000Fu, w & 0x00F000F0u, w8 & 0x00F000F0u, b0, b1);
    else mma_16816(d, w & 0x000F000Fu, w8 & 0x000F000Fu, w & 0x00F000F0u, w8 & 0x00F000F0u, b0, b1);
    return;
  }
  uint32_t h[4];
  cvt_e2m1x8(w, h[0], h[1], h[2], h[3]);
  if (FMT == QNT_FP4_RAZER) {
    // codes 0b1000 decode to -0 and take the group's special value sv, branch
    // free: nibbles 0b0001 exactly where the code is 0b1000 convert to 0.5, and
    // -0 + 0.5 * 2sv = sv, x + 0 * 2sv = x (sv16: the pair 2sv, 2sv)
    const uint32_t tt = (w & 0x77777777u) + 0x77777777u;
    const uint32_t spec = lop3<0x20>(w, tt, 0x88888888u);   // bit 3 of every nibble equal to 0b1000
    uint32_t ind[4];
    cvt_e2m1x8(spec >> 3, ind[0], ind[1], ind[2], ind[3]);
#pragma unroll
    for (int pp = 0; pp < 4; ++pp) h[pp] = hfma2(ind[pp], sv16, h[pp]);
  }
  if (FMT == QNT_FP4_AFPQ) {
    uint32_t hp[4], hn[4];
#pragma unroll
    for (int pp = 0; pp < 4; ++pp) { hp[pp] = hmax2(h[pp], 0u); hn[pp] = hsub2(h[pp], hp[pp]); }
    if (j == 0) {
      mma_16816_z(d, hp[0], hp[1], hp[2], hp[3], b0, b1);
      mma_16816_z(dn, hn[0], hn[1], hn[2], hn[3], b0, b1);
    } else {
      mma_16816(d, hp[0], hp[1], hp[2], hp[3], b0, b1);
      mma_16816(dn, hn[0], hn[1], hn[2], hn[3], b0, b1);
    }
  } else {
    if (FMT != QNT_FP4_AFPQ && j == 0) {
#pragma unroll
      for (int e = 0; e < 4; ++e) dn[e] = 0.0f;
    }
    if (j == 0) mma_16816_z(d, h[0], h[1], h[2], h[3], b0, b1);
    else mma_16816(d, h[0], h[1], h[2], h[3], b0, b1);
  }
}

// word_mma for two B operands (eight vectors: vectors 0-3 in bxa, 4-7 in bxb):
// the word is decoded once and feeds both MMAs.
template <int FMT>
__device__ __forceinline__ void word_mma2(uint32_t w, int j, const uint32_t (&bxa)[8], const uint32_t (&bxb)[8],
                                          float (&da)[4], float (&dna)[4], float (&db)[4], float (&dnb)[4],
                                          uint32_t sv16) {
  uint32_t h[4];
  if (FMT == QNT_INT4_ASYM) {
    const uint32_t w8 = w >> 8;
    h[0] = w & 0x000F000Fu; h[1] = w8 & 0x000F000Fu; h[2] = w & 0x00F000F0u; h[3] = w8 & 0x00F000F0u;
  } else {
    cvt_e2m1x8(w, h[0], h[1], h[2], h[3]);
    if (FMT == QNT_FP4_RAZER) {   // as in word_mma
      const uint32_t tt = (w & 0x77777777u) + 0x77777777u;
      const uint32_t spec = lop3<0x20>(w, tt, 0x88888888u);
      uint32_t ind[4];
      cvt_e2m1x8(spec >> 3, ind[0], ind[1], ind[2], ind[3]);
#pragma unroll
      for (int pp = 0; pp < 4; ++pp) h[pp] = hfma2(ind[pp], sv16, h[pp]);
    }
  }
  if (FMT == QNT_FP4_AFPQ) {
    uint32_t hp[4], hn[4];
#pragma unroll
    for (int pp = 0; pp < 4; ++pp) { hp[pp] = hmax2(h[pp], 0u); hn[pp] = hsub2(h[pp], hp[pp]); }
    if (j == 0) {
      mma_16816_z(da, hp[0], hp[1], hp[2], hp[3], bxa[0], bxa[1]);
      mma_16816_z(dna, hn[0], hn[1], hn[2], hn[3], bxa[0], bxa[1]);
      mma_16816_z(db, hp[0], hp[1], hp[2], hp[3], bxb[0], bxb[1]);
      mma_16816_z(dnb, hn[0], hn[1], hn[2], hn[3], bxb[0], bxb[1]);
    } else {
      mma_16816(da, hp[0], hp[1], hp[2], hp[3], bxa[2 * j], bxa[2 * j + 1]);
      mma_16816(dna, hn[0], hn[1], hn[2], hn[3], bxa[2 * j], bxa[2 * j + 1]);
      mma_16816(db, hp[0], hp[1], hp[2], hp[3], bxb[2 * j], bxb[2 * j + 1]);
      mma_16816(dnb, hn[0], hn[1], hn[2], hn[3], bxb[2 * j], bxb[2 * j + 1]);
    }
  } else {
    if (j == 0) {
      mma_16816_z(da, h[0], h[1], h[2], h[3], bxa[0], bxa[1]);
      mma_16816_z(db, h[0], h[1], h[2], h[3], bxb[0], bxb[1]);
    } else {
      mma_16816(da, h[0], h[1], h[2], h[3], bxa[2 * j], bxa[2 * j + 1]);
      mma_16816(db, h[0], h[1], h[2], h[3], bxb[2 * j], bxb[2 * j + 1]);
    }
  }
}

// ------------------------------------------------------------------ kernel
template <int FMT, int G, int MAXS, int MV>
__global__ void __launch_bounds__(kB1Threads, 1)
gemv1_kernel(const __grid_constant__ B1Params<MAXS> P) {
  constexpr int GPB = 128 / G;        // groups per block
  constexpr int MVc = MV > 4 ? 4 : MV;   // vectors per B operand (eight vectors: two B operands)
  constexpr int S = 4 / (GPB * MVc);  // blocks per set (accumulators)
  constexpr int NQ = kB1Blocks / S;   // sets per full item
  constexpr int RB = kB1Blocks;
  constexpr int C = kB1Warps;
  constexpr int ZSH = FMT == QNT_FP4_RAZER ? 2 : 1;   // zero / selector plane: fr >> ZSH is the byte
  extern __shared__ __align__(1024) uint8_t smem[];
  uint64_t* full = reinterpret_cast<uint64_t*>(smem);      // [C * depth] ring slots
  uint64_t* mfull = full + C * kB1MaxDepth;                // staged metadata landed
  volatile int* abort_s = reinterpret_cast<volatile int*>(smem + 1280);
  const int D = P.depth;
  const B1Smem L = b1_smem(D, P.kmax, GPB, P.part_cap, P.meta_cap, MV);
  const uint32_t sbase = smem_addr(smem);
  const uint32_t ximg_a = sbase + (uint32_t)L.ximg, xs2_a = sbase + (uint32_t)L.xs2;
  float* part = reinterpret_cast<float*>(smem + L.part);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int grid = gridDim.x;
  const int nct = kB1Threads;
  unsigned* abort_g = P.done ? P.done + P.nsteps : nullptr;

  if (tid == 0) {
    for (int i = 0; i < C * D; ++i) mbar_init_nofence(full + i, 1);
    mbar_init_nofence(mfull, 1);
    mbar_init_fence();
    *abort_s = 0;
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  }
  __syncthreads();

  auto fail = [&](int code) {
    *abort_s = 1;
    if (abort_g) atomicExch(abort_g, 1u);
    report(P.status, code);
  };
  // staged metadata window of step j (thread 32); its barrier completes phase j
  int nmeta_issued = 0;
  auto issue_meta = [&](int j) {
    const B1Step& st = P.s[j];
    int r_lo, r_hi;
    b1_rows_s(st, blockIdx.x, grid, &r_lo, &r_hi);
    uint64_t* bar = mfull;
    if (r_hi > r_lo) {
      const MetaWin mw = meta_window<FMT>(r_lo, r_hi, st.GK, st.z0, st.rows_cap);
      uint8_t* mdst = smem + L.meta;
      mbar_expect_tx(bar, (uint32_t)((mw.a1 - mw.a0) + (mw.b1 - mw.b0)));
      bulk_g2s(mdst, st.meta + mw.a0, (uint32_t)(mw.a1 - mw.a0), bar);
      if (mw.b1 > mw.b0) bulk_g2s(mdst + mw.bpl, st.meta + mw.b0, (uint32_t)(mw.b1 - mw.b0), bar);
    } else {
      asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" :: "r"(smem_addr(bar)) : "memory");
    }
    ++nmeta_issued;
  };

  // This warp's items: the CTA's items of all steps in order (a step's items are
  // its row groups x runs of 8 blocks of K), every C-th one starting at the
  // warp's index; the warp's k-th item goes to its ring slot k % D.  The issue
  // cursor walks them ahead of the computation, across step boundaries.
  struct Cursor {
    int j;           // step
    int left;        // items of this warp left in the step, this one included
    int u, br;       // row group and K run of the current item
    int KB, KBR, du, dbr;   // blocks, runs per row group, advance per item (C items)
    int skip;        // offset of the warp's first item in the next step
    const uint8_t* base;
    long rs;
  };
  // position the cursor at the warp's first item of step c.j, given that
  // `first` items of the step precede it (the warp's share starts there)
  auto cursor_step = [&](Cursor& c, int first) {
    for (; c.j < P.nsteps; ++c.j) {
      const B1Step& st = P.s[c.j];
      int r_lo, r_hi;
      b1_rows_s(st, blockIdx.x, grid, &r_lo, &r_hi);
      c.KB = st.KB;
      c.KBR = st.KBR;
      const int n = (r_hi - r_lo + 7) / 8 * c.KBR;
      c.rs = 4L * st.K;
      c.base = st.codes + (r_lo / 8) * c.rs;
      c.du = C / c.KBR;
      c.dbr = C - c.du * c.KBR;
      if (first < n) {
        c.left = (n - first + C - 1) / C;
        c.u = first / c.KBR;
        c.br = first - c.u * c.KBR;
        // the next step's share starts at (first + C * left) - n
        c.skip = first + C * c.left - n;
        return;
      }
      first -= n;
    }
  };
  auto cursor_next = [&](Cursor& c) {
    if (--c.left > 0) {
      c.u += c.du;
      c.br += c.dbr;
      if (c.br >= c.KBR) { c.br -= c.KBR; ++c.u; }
    } else {
      ++c.j;
      cursor_step(c, c.skip);
    }
  };
  Cursor ic = {0, 0, 0, 0, 0, 0, 0, 0, 0, nullptr, 0};
  int k_issued = 0, islot = 0;
  const uint64_t pol = l2_evict_first_policy();
  auto issue_next = [&]() {   // lane 0: issue the cursor's item into slot islot
    if (ic.j >= P.nsteps) return;
    const int nb = min(RB, ic.KB - RB * ic.br);
    uint64_t* bar = full + warp * D + islot;
    mbar_expect_tx(bar, (uint32_t)nb * 512u);
    bulk_g2s_hint(smem + L.ring + (size_t)(warp * D + islot) * kB1SlotBytes,
                  ic.base + ic.u * ic.rs + (long)ic.br * (RB * 512), (uint32_t)nb * 512u, bar, pol);
    ++k_issued;
    if (++islot == D) islot = 0;
    cursor_next(ic);
  };
  // weights and metadata do not depend on the preceding kernel: request them first
  if (tid == 32) issue_meta(0);
  if (lane == 0) {
    cursor_step(ic, warp);
    for (int i = 0; i < D; ++i) issue_next();
  }

  const int g = lane >> 2, r = lane & 3;
  const int hp = lane >> 3;                                    // B column pair of this lane
  const bool bload = (r * GPB) / 4 == hp % GPB;                // this lane's chunk lies in the pair's group
  const int bsel = hp / (GPB * MVc);                           // block of the set that feeds the pair
  const int ei = r / (GPB * MVc), eh = r % GPB;                // epilogue: accumulator, group in block
  // several vectors (MV > 1, g = 128): column pair hp carries vector hp % MV of
  // block hp / MV of the set, and lane 4g + r's result belongs to vector r % MV
  const int vb = hp % MVc, ve = r % MVc;
  const int IMGV = 2 * P.kmax, XSV = (P.kmax / 128) * GPB * 8;   // bytes per vector: image, factor table
  const uint32_t coff = 64u * g + 16u * (uint32_t)(r ^ ((g >> 1) & 3));
  const uint32_t xoff = 16u * (uint32_t)(4 * ((lane >> 2) & 1) + r);
  const uint32_t rz = (uint32_t)((r * GPB) / 4);              // group of this lane's chunk within a block
  int T0 = 0;                                                  // items of the CTA in earlier steps
  int cslot = 0;                                               // ring slot of the warp's next item
  uint32_t cphase = 0;                                         // its barrier phase parity
  int k_done = 0;
  for (int j = 0; j < P.nsteps; ++j) {
    const B1Step& st = P.s[j];
    int r_lo, r_hi;
    b1_rows_s(st, blockIdx.x, grid, &r_lo, &r_hi);
    const int KB = st.KB, KBR = st.KBR, GK = st.GK;
    const int nrows = r_hi - r_lo;
    const int nitems = (nrows + 7) / 8 * KBR;
    // -- dependency (thread 32: thread 0 may still be releasing the previous
    // step's completion, which this overlaps)
    if (tid == 32) {
      if (j == 0) {
        asm volatile("griddepcontrol.wait;" ::: "memory");
      } else if (st.wait > 0 && P.done) {
        const unsigned* cnt = P.done + (j - st.wait);
        uint64_t dl = 0;
        for (;;) {
          if (ld_acquire_gpu(cnt) >= (unsigned)grid) break;
          if (*abort_s || (abort_g && *(volatile unsigned*)abort_g)) { *abort_s = 1; break; }
          const uint64_t now = gtimer();
          if (dl == 0) dl = now + P.timeout_ns;
          else if (now > dl) { fail(QNT_ERR_TIMEOUT); break; }
          __nanosleep(32);
        }
      }
    }
    if (consumer_bar_or(nct, *abort_s != 0)) break;
    // -- the activation image, straight from global memory (after the barrier:
    // ordered after thread 32's acquire of the producing step's completion)
    if (!st.reuse_x) {
      if constexpr (MV == 1) {
        for (int b = 2 * warp; b < KB; b += 2 * C)
          build_x<FMT, G>(static_cast<const uint8_t*>(st.x), ximg_a, xs2_a, b, b + 1 < KB ? b + 1 : -1, P.xbf16, lane);
      } else {   // vector v of x is row v of [M][K]; vectors past M get an image of zeros
        for (int v = 0; v < MV; ++v)
          for (int b = 2 * warp; b < KB; b += 2 * C)
            build_x<FMT, G>(static_cast<const uint8_t*>(st.x) + (size_t)v * 2 * st.K, ximg_a + (uint32_t)(v * IMGV),
                            xs2_a + (uint32_t)(v * XSV), b, b + 1 < KB ? b + 1 : -1, P.xbf16, lane, v >= P.nvec);
      }
    }
    if (!mbar_wait_to(mfull, (uint32_t)j & 1u, P.timeout_ns, abort_s)) {
      if (!*abort_s) fail(QNT_ERR_TIMEOUT);
    }
    if (consumer_bar_or(nct, *abort_s != 0)) break;

    // -- metadata of this step's rows (window-relative addressing)
    MetaRef M = {0u, 0u};
    if (nrows > 0) {
      const MetaWin mw = meta_window<FMT>(r_lo, r_hi, GK, st.z0, st.rows_cap);
      const uint32_t mbase = sbase + (uint32_t)L.meta;
      const long f_lo = (long)r_lo * GK;                       // group index of row r_lo's group 0
      M.ms_a = mbase + (uint32_t)((FMT == QNT_FP4_AFPQ ? 4 : 2) * f_lo - mw.a0);
      M.mz_a = mbase + (uint32_t)(mw.bpl + st.z0 + (f_lo >> ZSH) - mw.b0);
    }

    // -- this warp's items of the step: t = tfirst, tfirst + C, ...
    const int tfirst = ((warp - T0 % C) % C + C) % C;
    const int du = C / KBR, dbr = C - (C / KBR) * KBR;
    int u = tfirst / KBR, br = tfirst - (tfirst / KBR) * KBR;
    for (int t = tfirst; t < nitems; t += C) {
      const int rl = 8 * u + g;                                // row within the CTA's rows
      const bool rowok = rl < nrows;
      const int nb = min(RB, KB - RB * br);
      const int b0 = RB * br;
      const int slot = warp * D + cslot;
      // window-relative group index of (this lane's epilogue row, block b0, group eh)
      const uint32_t fr0 = (uint32_t)((rowok ? rl : 0) * GK + b0 * GPB + eh);
      if (!mbar_wait_to(full + slot, cphase, P.timeout_ns, abort_s)) {
        if (!*abort_s) fail(QNT_ERR_TIMEOUT);
        break;
      }
      const uint32_t ca = sbase + (uint32_t)L.ring + (uint32_t)slot * (uint32_t)kB1SlotBytes + coff;
      float yacc = 0.0f, yacc2 = 0.0f;   // yacc2: eight vectors, the lane's second one (r + 4)
      // AFPQ's full items at g = 128 take the vector-general path below at any MV
      constexpr bool kGeneral = MV > 1 || (FMT == QNT_FP4_AFPQ && G == 128);
      if (MV > 1 || (nb == RB && G == 128 && (FMT == QNT_FP4_AFPQ || (GK & 1) == 0))) {
       if constexpr (!kGeneral) {
        // ---- full item, g = 128, an even number of groups per row: the lane's
        // epilogue blocks are ei * NQ + q, q < NQ (two consecutive groups of its
        // row, the first of even index, so both scales are one aligned 32-bit
        // word and both zero points one byte): their scales, zero points and
        // activation factors are loaded once for the item
        static_assert(NQ == 2 || G != 128, "two sets per item at g = 128");
        const uint32_t fe = fr0 + (uint32_t)(NQ * ei);        // the lane's first epilogue group
        const uint32_t s2 = lds32a(M.ms_a + 2u * fe);         // two fp16 scales (fe is even)
        const float4 sc = lds128fa(xs2_a + 8u * (uint32_t)(b0 + NQ * ei));   // (c/2^e, sum x) of both blocks
        float ea[NQ], eb[NQ];
        ea[0] = h2f(s2 & 0xFFFFu) * sc.x;
        ea[1] = h2f(s2 >> 16) * sc.z;
        if (FMT == QNT_INT4_ASYM) {
          const uint32_t zb = lds8a(M.mz_a + (fe >> 1));      // both zero points (fe is even)
          eb[0] = h2f(s2 & 0xFFFFu) * (float)(zb & 15u) * sc.y;
          eb[1] = h2f(s2 >> 16) * (float)(zb >> 4) * sc.w;
        } else {
          eb[0] = eb[1] = 0.0f;
        }
        const uint32_t xa = ximg_a + 256u * (uint32_t)(b0 + NQ * bsel) + xoff;
#pragma unroll
        for (int q = 0; q < NQ; ++q) {
          uint4 cv[S];
#pragma unroll
          for (int i = 0; i < S; ++i) cv[i] = lds128a(ca + 512u * (uint32_t)(q + NQ * i));
          const uint4 x0 = lds128a(xa + 256u * q), x1 = lds128a(xa + 256u * q + 128u);
          const uint32_t bx[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
          uint32_t sv16[S];
#pragma unroll
          for (int i = 0; i < S; ++i) {
            sv16[i] = 0u;
            if (FMT == QNT_FP4_RAZER) {
              const uint32_t sel = meta_sel2(M, fr0 - eh + (uint32_t)(q + NQ * i) + rz);
              const uint32_t sv2 = ((sel & 2u) ? 0x4C00u : 0x4900u) | ((sel & 1u) ? 0x8000u : 0u);   // 2 sv: +-16 or +-10
              sv16[i] = sv2 | (sv2 << 16);
            }
          }
          float d[S][4], dn[S][4];
#pragma unroll
          for (int jj = 0; jj < 4; ++jj)
#pragma unroll
            for (int i = 0; i < S; ++i) word_mma<FMT>((&cv[i].x)[jj], jj, bx, d[i], dn[i], sv16[i]);
          float v = d[0][0] + d[0][3];
#pragma unroll
          for (int i = 1; i < S; ++i)
            if (ei == i) v = d[i][0] + d[i][3];
          yacc += ea[q] * v - eb[q];
        }
       } else if constexpr (MV == 8) {
        // ---- eight vectors (g = 128, full items): two B operands, vectors 0-3
        // and 4-7, column pair hp carries vectors hp and hp + 4 of block q of set
        // q (one block per set), every code word is decoded once for both MMAs,
        // and lane 4g + r ends with vectors r and r + 4 of its row.
        const uint32_t fe = fr0;                               // the item's 8 groups of the row
        const uint32_t xs0 = xs2_a + (uint32_t)(r * XSV) + 8u * (uint32_t)b0;
        const uint32_t xs1 = xs2_a + (uint32_t)((r + 4) * XSV) + 8u * (uint32_t)b0;
        const uint32_t xa0 = ximg_a + (uint32_t)(hp * IMGV) + 256u * (uint32_t)b0 + xoff;
        const uint32_t xa1 = ximg_a + (uint32_t)((hp + 4) * IMGV) + 256u * (uint32_t)b0 + xoff;
#pragma unroll 2
        for (int q = 0; q < 8; ++q) {
          const uint4 cv = lds128a(ca + 512u * (uint32_t)q);
          const uint4 a0 = lds128a(xa0 + 256u * q), a1 = lds128a(xa0 + 256u * q + 128u);
          const uint4 c0 = lds128a(xa1 + 256u * q), c1 = lds128a(xa1 + 256u * q + 128u);
          const uint32_t bxa[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
          const uint32_t bxb[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
          uint32_t sv16 = 0u;
          if (FMT == QNT_FP4_RAZER) {
            const uint32_t sel = meta_sel2(M, fr0 + (uint32_t)q);
            const uint32_t sv2 = ((sel & 2u) ? 0x4C00u : 0x4900u) | ((sel & 1u) ? 0x8000u : 0u);   // 2 sv: +-16 or +-10
            sv16 = sv2 | (sv2 << 16);
          }
          float da[4], dna[4], db[4], dnb[4];
#pragma unroll
          for (int jj = 0; jj < 4; ++jj) word_mma2<FMT>((&cv.x)[jj], jj, bxa, bxb, da, dna, db, dnb, sv16);
          const float v0 = da[0] + da[3], v1 = db[0] + db[3];
          const float2 sc0 = lds64fa(xs0 + 8u * q), sc1 = lds64fa(xs1 + 8u * q);
          if (FMT == QNT_FP4_AFPQ) {
            const uint32_t w2 = lds32a(M.ms_a + 4u * (fe + (uint32_t)q));
            const float sp = h2f(w2 & 0xFFFFu), sn = h2f(w2 >> 16);
            yacc += sc0.x * (sp * v0 + sn * (dna[0] + dna[3]));
            yacc2 += sc1.x * (sp * v1 + sn * (dnb[0] + dnb[3]));
          } else {
            const float sq = meta_scale(M, fe + (uint32_t)q);
            const float zq = FMT == QNT_INT4_ASYM ? (float)meta_zero4(M, fe + (uint32_t)q) : 0.0f;
            yacc += sq * (sc0.x * v0 - zq * sc0.y);
            yacc2 += sq * (sc1.x * v1 - zq * sc1.y);
          }
        }
        if (!rowok) yacc = yacc2 = 0.0f;
       } else {
        // ---- several vectors (g = 128, full items: the launcher's conditions),
        // or AFPQ's full items at g = 128.
        // Set q holds blocks q + NQ i (i < S); the lane's epilogue blocks are
        // NQ ei + q, q < NQ: NQ consecutive groups of its row whose scales (and
        // INT4 zero points) are aligned loads, as the group index of the first
        // is a multiple of NQ (K is a multiple of 1024).
        static_assert(G == 128, "several vectors: g = 128");
        const uint32_t fe = fr0 + (uint32_t)(NQ * ei);
        uint32_t sw[NQ / 2] = {};                              // the NQ fp16 scales, two per word (AFPQ: per set)
        if constexpr (FMT != QNT_FP4_AFPQ) {
          if constexpr (NQ == 8) {
            const uint4 t = lds128a(M.ms_a + 2u * fe);
            sw[0] = t.x; sw[1] = t.y; sw[2] = t.z; sw[3] = t.w;
          } else {
            const uint2 t = lds64a(M.ms_a + 2u * fe);
            sw[0] = t.x; sw[1] = t.y;
          }
        }
        uint32_t zw = 0u;                                      // INT4: the NQ zero points, a nibble each
        if (FMT == QNT_INT4_ASYM) zw = NQ == 8 ? lds32a(M.mz_a + (fe >> 1)) : lds16a(M.mz_a + (fe >> 1));
        const uint32_t xsv = xs2_a + (uint32_t)(ve * XSV) + 8u * (uint32_t)(b0 + NQ * ei);   // vector ve's factors
        const uint32_t xa = ximg_a + (uint32_t)(vb * IMGV) + 256u * (uint32_t)(b0 + NQ * bsel) + xoff;
        // AFPQ with one or two vectors: both parts of a set's blocks are 32 or 16
        // accumulators; one set at a time keeps them in registers (no spills;
        // measured 3.5 % faster at batch 1, 1.5 % slower at batch 2)
        constexpr int kSetUnroll = (FMT == QNT_FP4_AFPQ && MV <= 2) ? 1 : NQ;
#pragma unroll kSetUnroll
        for (int q = 0; q < NQ; ++q) {
          uint4 cv[S];
#pragma unroll
          for (int i = 0; i < S; ++i) cv[i] = lds128a(ca + 512u * (uint32_t)(q + NQ * i));
          const uint4 x0 = lds128a(xa + 256u * q), x1 = lds128a(xa + 256u * q + 128u);
          const uint32_t bx[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
          uint32_t sv16[S];
#pragma unroll
          for (int i = 0; i < S; ++i) {
            sv16[i] = 0u;
            if (FMT == QNT_FP4_RAZER) {
              const uint32_t sel = meta_sel2(M, fr0 + (uint32_t)(q + NQ * i));
              const uint32_t sv2 = ((sel & 2u) ? 0x4C00u : 0x4900u) | ((sel & 1u) ? 0x8000u : 0u);   // 2 sv: +-16 or +-10
              sv16[i] = sv2 | (sv2 << 16);
            }
          }
          float d[S][4], dn[S][4];
#pragma unroll
          for (int jj = 0; jj < 4; ++jj)
#pragma unroll
            for (int i = 0; i < S; ++i) word_mma<FMT>((&cv[i].x)[jj], jj, bx, d[i], dn[i], sv16[i]);
          float v = d[0][0] + d[0][3], vn = dn[0][0] + dn[0][3];
#pragma unroll
          for (int i = 1; i < S; ++i)
            if (ei == i) { v = d[i][0] + d[i][3]; vn = dn[i][0] + dn[i][3]; }
          const float2 sc = lds64fa(xsv + 8u * q);             // (c / 2^e, group sum of x) of vector ve
          if (FMT == QNT_FP4_AFPQ) {                             // positive part times s+, negative times s-
            const uint32_t w2 = lds32a(M.ms_a + 4u * (fe + (uint32_t)q));
            yacc += sc.x * (h2f(w2 & 0xFFFFu) * v + h2f(w2 >> 16) * vn);
          } else {
            const float sq = h2f((sw[q >> 1] >> (16 * (q & 1))) & 0xFFFFu);
            const float zq = FMT == QNT_INT4_ASYM ? (float)((zw >> (4 * q)) & 15u) : 0.0f;
            yacc += sq * (sc.x * v - zq * sc.y);
          }
        }
        if (!rowok) yacc = 0.0f;
       }
      } else {
       if constexpr (MV == 1) {
        // ---- general item (g < 128, AFPQ, or the last run of K of a row)
        auto set_epilogue = [&](int q, const float (&d)[S][4], const float (&dn)[S][4]) {
          // accumulator ei holds this lane's (row g, block q + NQ ei, group eh)
          float v = d[0][0] + d[0][3], vn = dn[0][0] + dn[0][3];
#pragma unroll
          for (int i = 1; i < S; ++i)
            if (ei == i) { v = d[i][0] + d[i][3]; vn = dn[i][0] + dn[i][3]; }
          const int be = q + NQ * ei;
          if (rowok && be < nb) {
            const uint32_t fr = fr0 + (uint32_t)(be * GPB);
            const float2 sc = lds64fa(xs2_a + 8u * (uint32_t)((b0 + be) * GPB + eh));   // (c / 2^e, group sum of x)
            float c;
            if (FMT == QNT_INT4_ASYM) {
              c = meta_scale(M, fr) * (sc.x * v - (float)meta_zero4(M, fr) * sc.y);
            } else if (FMT == QNT_FP4_AFPQ) {
              const uint32_t w2 = meta_afpq(M, fr);
              c = sc.x * (h2f(w2 & 0xFFFFu) * v + h2f(w2 >> 16) * vn);
            } else {
              c = meta_scale(M, fr) * sc.x * v;
            }
            yacc += c;
          }
        };
#pragma unroll 1
        for (int q = 0; q < NQ && q < nb; ++q) {
          uint32_t bx[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
          const int bl = q + NQ * bsel;                        // block of the item that feeds this lane's pair
          if (bload && bl < nb) {
            const uint32_t xa = ximg_a + 256u * (uint32_t)(b0 + bl) + xoff;
            const uint4 x0 = lds128a(xa), x1 = lds128a(xa + 128u);
            bx[0] = x0.x; bx[1] = x0.y; bx[2] = x0.z; bx[3] = x0.w;
            bx[4] = x1.x; bx[5] = x1.y; bx[6] = x1.z; bx[7] = x1.w;
          }
          float d[S][4], dn[S][4];
#pragma unroll
          for (int i = 0; i < S; ++i) {
            const int blk = q + NQ * i;
#pragma unroll
            for (int e = 0; e < 4; ++e) d[i][e] = dn[i][e] = 0.0f;
            if (blk < nb) {
              const uint4 cv = lds128a(ca + 512u * (uint32_t)blk);
              uint32_t sv = 0u;
              if (FMT == QNT_FP4_RAZER) {
                const uint32_t sel = meta_sel2(M, fr0 - eh + (uint32_t)(blk * GPB) + rz);
                const uint32_t sv2 = ((sel & 2u) ? 0x4C00u : 0x4900u) | ((sel & 1u) ? 0x8000u : 0u);   // 2 sv: +-16 or +-10
                sv = sv2 | (sv2 << 16);
              }
#pragma unroll
              for (int jj = 0; jj < 4; ++jj) word_mma<FMT>((&cv.x)[jj], jj, bx, d[i], dn[i], sv);
            }
          }
          set_epilogue(q, d, dn);
        }
       }
      }
      // the slot is read: refill it with this warp's item D ahead
      __syncwarp();
      ++k_done;
      if (++cslot == D) { cslot = 0; cphase ^= 1u; }
      if (lane == 0) {
        fence_proxy_async();
        issue_next();
      }
      if constexpr (MV == 1) {
        yacc += __shfl_xor_sync(0xffffffffu, yacc, 1);
        yacc += __shfl_xor_sync(0xffffffffu, yacc, 2);
        if (r == 0 && rowok) part[rl * KBR + br] = yacc;
      } else if constexpr (MV == 8) {   // lane r ends with vectors r and r + 4
        if (rowok) {
          part[r * P.part_cap + rl * KBR + br] = yacc;
          part[(r + 4) * P.part_cap + rl * KBR + br] = yacc2;
        }
      } else {   // lanes r and r ^ 2 hold the same vector when MV = 2; lane r < MV ends with vector r
        if (MV == 2) yacc += __shfl_xor_sync(0xffffffffu, yacc, 2);
        if (r < MV && rowok) part[r * P.part_cap + rl * KBR + br] = yacc;
      }
      u += du;
      br += dbr;
      if (br >= KBR) { br -= KBR; ++u; }
    }
    if (consumer_bar_or(nct, *abort_s != 0)) break;
    // every warp is done with this step's metadata: request the next step's,
    // which lands while the step's completion propagates
    if (tid == 32 && j + 1 < P.nsteps) issue_meta(j + 1);
    // -- this CTA's rows of y, the partial sums combined in a fixed order
    if constexpr (MV == 1) {
      for (int rr = tid; rr < nrows; rr += nct) {
        float v = 0.0f;
        for (int b = 0; b < KBR; ++b) v += part[rr * KBR + b];
        if (P.xbf16) reinterpret_cast<__nv_bfloat16*>(st.y)[r_lo + rr] = __float2bfloat16_rn(v);
        else reinterpret_cast<__half*>(st.y)[r_lo + rr] = __float2half_rn(v);
      }
    } else {   // vector v's outputs are row v of [M][N]
      for (int rr = tid; rr < nrows; rr += nct)
        for (int vv = 0; vv < P.nvec; ++vv) {
          float v = 0.0f;
          for (int b = 0; b < KBR; ++b) v += part[vv * P.part_cap + rr * KBR + b];
          const long o = (long)vv * st.N + r_lo + rr;
          if (P.xbf16) reinterpret_cast<__nv_bfloat16*>(st.y)[o] = __float2bfloat16_rn(v);
          else reinterpret_cast<__half*>(st.y)[o] = __float2half_rn(v);
        }
    }
    consumer_bar(nct);
#ifdef QNT_TEST_FAULTS
    // test builds: CTA 0 never reports step 0 complete, so every wait for it expires
    const bool skip_signal = P.fault == 1 && j == 0 && blockIdx.x == 0;
#else
    constexpr bool skip_signal = false;
#endif
    if (P.done && tid == 0 && !skip_signal)   // release: every y store of the CTA (ordered by the barrier) comes first
      asm volatile("red.release.gpu.global.add.u32 [%0], 1;" :: "l"(P.done + j) : "memory");
    T0 += nitems;
  }
  // drain: every issued copy has landed before the CTA exits
  if (lane == 0)
    for (int k = k_done; k < k_issued; ++k)
      mbar_wait_to(full + warp * D + k % D, (uint32_t)(k / D) & 1u, P.timeout_ns, nullptr);
  if (tid == 32 && nmeta_issued > 0) mbar_wait_to(mfull, (uint32_t)(nmeta_issued - 1) & 1u, P.timeout_ns, nullptr);
  __syncthreads();
}

// ------------------------------------------------------------------ launchers
#ifdef QNT_TEST_FAULTS
// Test builds only: a fault to inject into the next launches of this thread and
// the wait limit to use (set by qnt_test_gemv_seq_fault).
static thread_local int t_fault = 0;
static thread_local unsigned long long t_timeout_ns = kB1TimeoutNs;
void set_test_fault(int fault, unsigned long long timeout_ns) {
  t_fault = fault;
  t_timeout_ns = timeout_ns;
}
#define QNT_B1_FAULT t_fault
#define QNT_B1_TIMEOUT t_timeout_ns
#else
#define QNT_B1_FAULT 0
#define QNT_B1_TIMEOUT kB1TimeoutNs
#endif

namespace {

// Shared-memory plan of a launch: the deepest per-warp ring that fits with the
// activation image and two staged metadata windows.  depth = 0 if it does not fit.
struct B1Plan { int depth, kmax, meta_cap, part_cap; size_t smem; };
template <int FMT, int G, int MV>
B1Plan b1_plan(const qnt_seq_step* steps, int n, int grid) {
  B1Plan p = {0, 0, 0, 0, 0};
  size_t meta = 0;
  for (int i = 0; i < n; ++i) {
    const qnt_desc& d = steps[i].desc;
    p.kmax = p.kmax > d.K ? p.kmax : d.K;
    const int KBR = (d.K / 128 + kB1Blocks - 1) / kB1Blocks;
    const int pc = b1_rows_cap(d.N, grid) * KBR;
    p.part_cap = p.part_cap > pc ? p.part_cap : pc;
    const size_t mb = meta_stage_bytes<FMT>(b1_rows_cap(d.N, grid), d.K / G);
    meta = meta > mb ? meta : mb;
  }
  p.meta_cap = (int)align16(meta);
  constexpr int GPB = 128 / G;
  for (int dp = kB1MaxDepth; dp >= 1; --dp) {
    const size_t tot = b1_smem(dp, p.kmax, GPB, p.part_cap, p.meta_cap, MV).total;
    if (tot <= (size_t)kMaxDynSmem) {
      p.depth = dp;
      p.smem = tot;
      return p;
    }
  }
  return p;
}

// MV > 1: one step whose x is [nvec][K] and y [nvec][N] (nvec <= MV).  A plan
// with a single ring slot per warp is still taken: measured on B200 it beats the
// other kernels (M = 4 on K = 8192, N = 28672: 33 us against 71 on tcgen05).
template <int FMT, int G, int MAXS, int MV = 1>
cudaError_t b1_launch(const qnt_seq_step* steps, int n, int xbf16, unsigned* done, int* st, cudaStream_t s,
                      bool cooperative, bool* handled, int nvec = 1) {
  const int sms = num_sms();
  long maxng = 1;
  for (int i = 0; i < n; ++i) maxng = maxng > (steps[i].desc.N + 7) / 8 ? maxng : (steps[i].desc.N + 7) / 8;
  const int grid = cooperative ? sms : (int)(maxng < sms ? maxng : sms);
  static B1Params<MAXS> P;   // large: built in static storage, copied by the launch
  static std::mutex mu;
  std::lock_guard<std::mutex> lock(mu);
  const B1Plan p = b1_plan<FMT, G, MV>(steps, n, grid);
  if (!p.depth) return cudaSuccess;   // not handled: the activations and metadata do not fit
  auto kfn = gemv1_kernel<FMT, G, MAXS, MV>;
  cudaError_t e = configure_smem(reinterpret_cast<const void*>(kfn));
  if (e != cudaSuccess) return e;
  std::memset(&P, 0, sizeof(P));
  long rot = 0;
  for (int i = 0; i < n; ++i) {
    B1Step& b = P.s[i];
    const qnt_desc& d = steps[i].desc;
    b.codes = static_cast<const uint8_t*>(steps[i].codes);
    b.meta = static_cast<const uint8_t*>(steps[i].meta);
    b.x = steps[i].x;
    b.y = steps[i].y;
    b.z0 = (long)((2L * d.N * (d.K / d.group) + 255) / 256 * 256);
    b.N = d.N;
    b.K = d.K;
    b.wait = steps[i].wait;
    b.rot = (int)(rot % grid);
    b.NG = (d.N + 7) / 8;
    b.KB = d.K / 128;
    b.KBR = (b.KB + kB1Blocks - 1) / kB1Blocks;
    b.GK = d.K / d.group;
    b.rows_cap = b1_rows_cap(d.N, grid);
    rot += (d.N + 7) / 8;   // rotate the remainder CTAs from step to step
    // The activation image of step i - 1 serves step i when both read the same
    // x and step i waits for no step that step i - 1 did not already wait for:
    // x is then unchanged since it was imaged (a step that writes x must be
    // waited for by the steps that read it).
    const int dep = steps[i].wait > 0 ? i - steps[i].wait : -1;
    const int dep_prev = i > 0 && steps[i - 1].wait > 0 ? i - 1 - steps[i - 1].wait : -1;
    b.reuse_x = i > 0 && steps[i].x == steps[i - 1].x && d.K == steps[i - 1].desc.K && dep <= dep_prev ? 1 : 0;
  }
  P.nsteps = n;
  P.xbf16 = xbf16;
  P.depth = p.depth;
  P.kmax = p.kmax;
  P.meta_cap = p.meta_cap;
  P.part_cap = p.part_cap;
  P.done = done;
  P.status = st;
  P.fault = QNT_B1_FAULT;
  P.timeout_ns = QNT_B1_TIMEOUT;
  P.nvec = nvec;
  *handled = true;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kB1Threads);
  cfg.dynamicSmemBytes = p.smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  if (cooperative) {
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
  } else {
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
  }
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kfn, P);
}

template <int MAXS>
cudaError_t b1_dispatch(const qnt_seq_step* steps, int n, int xbf16, unsigned* done, int* st, cudaStream_t s,
                        bool cooperative, bool* handled) {
#define QNT_B1G(FMT)                                                                             \
  switch (steps[0].desc.group) {                                                                 \
    case 32: return b1_launch<FMT, 32, MAXS>(steps, n, xbf16, done, st, s, cooperative, handled);  \
    case 64: return b1_launch<FMT, 64, MAXS>(steps, n, xbf16, done, st, s, cooperative, handled);  \
    default: return b1_launch<FMT, 128, MAXS>(steps, n, xbf16, done, st, s, cooperative, handled); \
  }
  switch (steps[0].desc.fmt) {
    case QNT_INT4_ASYM: QNT_B1G(QNT_INT4_ASYM)
    case QNT_FP4_E2M1: QNT_B1G(QNT_FP4_E2M1)
    case QNT_FP4_AFPQ: QNT_B1G(QNT_FP4_AFPQ)
    case QNT_FP4_RAZER: QNT_B1G(QNT_FP4_RAZER)
    default: return cudaSuccess;
  }
#undef QNT_B1G
}

}  // namespace

cudaError_t launch_gemv4_one(const qnt_desc& d, const void* codes, const void* meta, long /*z0*/, const void* X,
                             void* Y, int xbf16, int* st, cudaStream_t s, bool* handled) {
  *handled = false;
  qnt_seq_step one = {};
  one.desc = d;
  one.codes = codes;
  one.meta = meta;
  one.x = X;
  one.y = Y;
  one.wait = 0;
  return b1_dispatch<1>(&one, 1, xbf16, nullptr, st, s, false, handled);
}

cudaError_t launch_gemv1_multi(const qnt_desc& d, const void* codes, const void* meta, const void* X, void* Y, int M,
                              int xbf16, int* st, cudaStream_t s, bool* handled) {
  *handled = false;
  if (M < 2 || M > 8 || d.group != 128 || d.K % 1024 != 0) return cudaSuccess;
  qnt_seq_step one = {};
  one.desc = d;
  one.codes = codes;
  one.meta = meta;
  one.x = X;
  one.y = Y;
  one.wait = 0;
#define QNT_B1M(FMT)                                                                                       \
  return M == 2   ? b1_launch<FMT, 128, 1, 2>(&one, 1, xbf16, nullptr, st, s, false, handled, M)          \
         : M <= 4 ? b1_launch<FMT, 128, 1, 4>(&one, 1, xbf16, nullptr, st, s, false, handled, M)          \
                  : b1_launch<FMT, 128, 1, 8>(&one, 1, xbf16, nullptr, st, s, false, handled, M);
  switch (d.fmt) {
    case QNT_INT4_ASYM: QNT_B1M(QNT_INT4_ASYM)
    case QNT_FP4_E2M1: QNT_B1M(QNT_FP4_E2M1)
    case QNT_FP4_AFPQ: QNT_B1M(QNT_FP4_AFPQ)
    case QNT_FP4_RAZER: QNT_B1M(QNT_FP4_RAZER)
    default: return cudaSuccess;
  }
#undef QNT_B1M
}

cudaError_t launch_gemv_seq(const qnt_seq_step* steps, int n, int xbf16, void* work, int* st, cudaStream_t s,
                            bool* handled) {
  *handled = false;
  cudaError_t e = cudaMemsetAsync(work, 0, qnt_gemv_seq_work_bytes(n), s);
  if (e != cudaSuccess) return e;
  return b1_dispatch<QNT_SEQ_MAX_STEPS>(steps, n, xbf16, static_cast<unsigned*>(work), st, s, true, handled);
}

// ------------------------------------------------------------------ the same, with a library-owned workspace
// For callers that cannot allocate device memory (qnt_gemv_seq_noalloc): the
// completion counters live in this array, which the CUDA runtime places in the
// device memory of every GPU that loads the library, for the life of the
// process.  Host code must not pass the array's name to a kernel (on the host
// it is only a stand-in); its device address is looked up once per device.
static __device__ __align__(256) unsigned g_seq_counters[QNT_SEQ_NOALLOC_MAX_STEPS + 1];

// Device address of g_seq_counters on the current device, looked up on the
// first call for each device.
static cudaError_t seq_counters_address(unsigned** out) {
  static unsigned* addr[64] = {nullptr};
  static std::mutex mu;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_seq_counters);
    if (e != cudaSuccess) return e;
    addr[dev] = static_cast<unsigned*>(p);
  }
  *out = addr[dev];
  return cudaSuccess;
}

cudaError_t launch_gemv_seq_noalloc(const qnt_seq_step* steps, int n, int xbf16, int* st, cudaStream_t s,
                                    bool* handled) {
  *handled = false;
  unsigned* counters = nullptr;
  cudaError_t e = seq_counters_address(&counters);
  if (e != cudaSuccess) return e;
  // every call starts from zeroed counters (the array keeps the last call's)
  e = cudaMemsetAsync(counters, 0, sizeof(unsigned) * (size_t)(n + 1), s);
  if (e != cudaSuccess) return e;
  return b1_dispatch<QNT_SEQ_MAX_STEPS>(steps, n, xbf16, counters, st, s, true, handled);
}

}  // namespace qnt
