// gemm_tc.cu -- small-batch fused-dequant GEMM on the 5th-generation tensor
// cores (tcgen05), in one pass over the weights for 3 <= M <= 128 activation
// rows: Y[m][n] = sum_k dq(code[n][k], meta[n][k/g]) * X[m][k].
//
// The GEMM of the RTN page ("Is (Selective) Round-To-Nearest Quantization All
// You Need?", English abstract: fused-dequant RTN kernels and their throughput)
// and of the RaZeR page ("The Power of Negative Zero", method section: 4-bit
// codes turned into FP16 with bit operations, fused with the product), for the
// small batches of a decode step.
//
// Structure: one CTA per tile of 128 weight rows (tensor-memory lanes), the
// whole of K in stages of 128 weights:
//  * warp 0 requests each stage with two kinds of TMA tile copies: the
//    stage's 512-byte block of each of the tile's 16 row groups as one box of a
//    2-D tensor map over the codes (row groups x 32-bit words), and the stage's
//    slice of X as two 64-column boxes of a tensor map with 128-byte swizzle
//    (rows of X beyond M read as zeros), so X is the canonical K-major B
//    operand.  The shared-memory ring holds up to 16 stages;
//  * the decode warps, in groups of four (one per tensor-memory lane quarter),
//    take the stages in turn (group j: stages j, j + groups, ...): each thread
//    owns one weight row (its tensor-memory lane) and turns the stage's 128
//    weights of it into the MMA's A operand with the group scale folded in (one
//    rounding per weight: fp16 (q - z) exactly, times the scale times a per-row
//    power of two that keeps the products in fp16 range; bf16 the same product
//    rounded once, through a split of the scale into bf16 high and low parts),
//    and writes it to one of the A slots in tensor memory (the 64-column slots
//    the accumulators leave, 4 or 6) with tcgen05.st;
//  * one thread in each of warps 1..4 (2 or 4 of them, by M) issues a share of
//    each stage's eight tcgen05.mma (M = 128, N = M rounded up to 16, K = 16;
//    A from tensor memory, B from shared memory) into its own fp32
//    accumulator in tensor memory, and commits them to the stage's barriers,
//    which free the stage's shared memory and its A slot.  A single issuing
//    thread is not enough: each small-N MMA occupies it for ~60 cycles, longer
//    than the HBM time of the 2048 weights it consumes;
//  * the decode warps then sum the accumulators (tcgen05.ld), undo the row's
//    power of two and store Y.
// Waiting threads sleep between tries (nanosleep backoff), so the waiting warps
// take few issue slots from the decode warps.
// Programmatic dependent launch: the codes of the first stages are requested
// before griddepcontrol.wait, X after it.  Every wait is bounded; on expiry the
// kernel reports QNT_ERR_TIMEOUT, lets every copy and MMA it issued finish,
// frees tensor memory and returns.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <mutex>
#include "common.cuh"
#include "kernels.h"

namespace qnt {
namespace {

constexpr int kGtRows = 128;            // weight rows per tile (tensor-memory lanes)
constexpr int kGtStageK = 128;          // weights of each row per stage (one block)
constexpr int kGtCodeBytes = 16 * 512;  // codes of one stage: 16 row groups x one block
constexpr int kGtMmaWarp0 = 1;          // warps 1..4: MMA issuers
constexpr int kGtMaxIssuers = 4;
constexpr int kGtDecodeWarp0 = 5;       // then the decode warps, in groups of four (one per lane quarter)
#ifndef QNT_GT_DECODE_GROUPS
#define QNT_GT_DECODE_GROUPS 2
#endif
constexpr int kGtGroups = QNT_GT_DECODE_GROUPS;   // decode groups: group j decodes stages j, j + kGtGroups, ...
constexpr int kGtThreads = 32 * (kGtDecodeWarp0 + 4 * kGtGroups);
constexpr int kGtMaxStages = 16;        // shared-memory ring
constexpr int kGtMaxASlots = 8;         // A slots in tensor memory, at most
constexpr uint32_t kGtTmemCols = 512;   // accumulators first, then the A slots, 64 columns each
constexpr int kGtCtrl = 1024;
constexpr unsigned long long kGtTimeoutNs = 2000000000ull;

struct GtArgs {
  const uint8_t* meta;
  void* Y;
  long z0;
  int N, K, M, Mpad;
  int nstages;        // shared-memory stages in flight
  int nissuers;       // MMA issuing threads (accumulators): 4 for M <= 64, else 2
  int naslots;        // A slots: the tensor-memory columns the accumulators leave, 64 each, at most 8
  int cola;           // first column of the A slots
  int xbf16;
  int* status;
  unsigned long long timeout_ns;   // limit of every wait
  int fault;                       // test builds only: an injected fault (0: none)
  int split;                       // CTAs per tile (a cluster), each over a share of K
};

struct GtSmem { size_t stage0, stage_bytes, xoff, total; };
__host__ __device__ inline GtSmem gt_smem(int Mpad, int nst) {
  GtSmem L;
  L.stage0 = kGtCtrl;                                         // 1024-aligned (swizzle atoms)
  L.xoff = kGtCodeBytes;                                      // X after the codes in a stage
  L.stage_bytes = (size_t)kGtCodeBytes + (size_t)Mpad * 256;  // two boxes of Mpad rows x 128 bytes
  L.total = L.stage0 + (size_t)nst * L.stage_bytes;
  return L;
}

// ------------------------------------------------------------------ PTX wrappers
__device__ __forceinline__ uint64_t gt_now() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
// Bounded wait (gives up `timeout` ns after the first unsuccessful try, or
// when the abort flag is raised).  max_sleep > 0: between tries the thread
// sleeps, 32 ns at first, doubling up to max_sleep ns, so a waiting warp takes
// few issue slots from the decode warps that share its scheduler and sees the
// phase complete at most ~max_sleep ns late.  max_sleep = 0: it spins, looking
// at the flag and the clock every 64 tries (the MMA issuers, whose waits are on
// the critical path).  (A suspend-time hint on try_wait instead was measured to
// wake the thread up to microseconds after the phase completed.)
__device__ __forceinline__ bool gt_wait(uint64_t* bar, uint32_t parity, volatile int* abort_s, uint64_t timeout,
                                        uint32_t max_sleep, bool cluster_scope = false) {
  const uint32_t a = smem_addr(bar);
  uint64_t deadline = 0;
  for (uint32_t n = 0, ns = 0;; ++n) {
    uint32_t done;
    if (cluster_scope)   // the phase was completed by arrivals (with release) from other CTAs of the cluster
      asm volatile("{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
                   "selp.u32 %0, 1, 0, p;\n\t}" : "=r"(done) : "r"(a), "r"(parity) : "memory");
    else
      asm volatile("{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\tselp.u32 %0, 1, 0, p;\n\t}"
                   : "=r"(done) : "r"(a), "r"(parity) : "memory");
    if (done) return true;
    if (max_sleep == 0 && (n & 63u) != 63u) continue;
    if (abort_s && *abort_s) return false;
    const uint64_t now = gt_now();
    if (deadline == 0) deadline = now + timeout;
    else if (now > deadline) return false;
    if (max_sleep) {
      if (ns) __nanosleep(ns);
      ns = ns ? (ns < max_sleep ? 2 * ns : max_sleep) : 32;
    }
  }
}
// Position in a ring of n slots: slot index and the parity of its current use.
struct GtRing {
  int slot = 0;
  uint32_t phase = 0;
  __device__ __forceinline__ void next(int n) {
    if (++slot == n) {
      slot = 0;
      phase ^= 1u;
    }
  }
  __device__ __forceinline__ void adv(int k, int n) {   // k <= n
    slot += k;
    if (slot >= n) {
      slot -= n;
      phase ^= 1u;
    }
  }
};
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
               :: "r"(smem_addr(bar)) : "memory");
}
// D[128 x N] (+)= A[128 x 16] (tensor memory) * B[16 x N] (shared memory, descriptor)
__device__ __forceinline__ void tc_mma_tmem_a(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                              uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, {%5, %5, %5, %5}, p;\n\t}"
      :: "r"(d_tmem), "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(0u) : "memory");
}
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};"
      :: "r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
         "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&d)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3]), "=r"(d[4]), "=r"(d[5]), "=r"(d[6]), "=r"(d[7]),
        "=r"(d[8]), "=r"(d[9]), "=r"(d[10]), "=r"(d[11]), "=r"(d[12]), "=r"(d[13]), "=r"(d[14]), "=r"(d[15])
      : "r"(taddr) : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Shared-memory descriptor of a K-major operand with 128-byte swizzle: rows of
// 128 bytes, 8-row groups 1024 bytes apart (LBO unused: 1), sm_100 version 1.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)1u << 16) | ((uint64_t)(1024u >> 4) << 32) |
         (1ull << 46) | (2ull << 61);
}
// Instruction descriptor of kind::f16: fp32 accumulator, A and B fp16 (or
// both bf16), K-major, M = 128, N = n.
__device__ __forceinline__ uint32_t f16_idesc(int n, int bf16) {
  return (1u << 4) | (bf16 ? ((1u << 7) | (1u << 10)) : 0u) | ((uint32_t)(n >> 3) << 17) | ((128u >> 4) << 24);
}
// 2-D tiled TMA loads (no multicast) of a box at (c0, c1) into shared memory.
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int c0, int c1, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
      :: "r"(smem_addr(dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(smem_addr(bar))
      : "memory");
}
__device__ __forceinline__ void tma_load_2d_hint(void* dst, const CUtensorMap* map, int c0, int c1, uint64_t* bar,
                                                 uint64_t pol) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3}], [%4], %5;"
      :: "r"(smem_addr(dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(smem_addr(bar)), "l"(pol)
      : "memory");
}

// Cluster helpers (split of K over the CTAs of a cluster; no multicast).
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Address of this CTA's shared-memory location `a` in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t cluster_map(uint32_t a, uint32_t rank) {
  uint32_t d;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(rank));
  return d;
}
__device__ __forceinline__ void cluster_arrive(uint32_t bar_cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" :: "r"(bar_cluster_addr) : "memory");
}
__device__ __forceinline__ float lds32f(uint32_t a) {
  float v;
  asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(a) : "memory");
  return v;
}
__device__ __forceinline__ void cluster_st_f32(uint32_t a, float v) {
  asm volatile("st.shared::cluster.f32 [%0], %1;" :: "r"(a), "f"(v) : "memory");
}

// packed bf16 arithmetic (one rounding each)
__device__ __forceinline__ uint32_t bsub2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
__device__ __forceinline__ uint32_t bmul2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
__device__ __forceinline__ uint32_t bfma2(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("fma.rn.bf16x2 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}
__device__ __forceinline__ uint32_t hmul2_(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
__device__ __forceinline__ uint32_t pack2(uint32_t lo16, uint32_t hi16) { return (lo16 & 0xFFFFu) | (hi16 << 16); }
__device__ __forceinline__ uint32_t f2bf_pair(float a, float b) {
  uint32_t d;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(b), "f"(a));
  return d;
}

// Per-group constants of the decode of one row (see gt_decode_chunk).
struct GtGroup {
  uint32_t zlo, zhi;   // INT4: (1024 + z), (1024 + 16 z) fp16 pairs; bf16: (128 + z) bf16 pair
  uint32_t s1, s2;     // fp16: scale pair (low / high nibble); bf16: scale high part; AFPQ: s+ / s-
  uint32_t s3;         // bf16: scale low part
  float fs, fs2;       // FP4 family with bf16: fp32 scale(s)
  uint32_t sv;         // RaZeR: twice the special value, as an fp16 pair
};

// Raw metadata of group f: AFPQ the (s+, s-) word; otherwise the fp16 scale in
// bits 0..15 and the INT4 zero / RaZeR selector in bits 16..19.
template <int FMT>
__device__ __forceinline__ uint32_t gt_meta_raw(const uint8_t* meta, long z0, long f) {
  if (FMT == QNT_FP4_AFPQ) return ldg_u32(meta + 4 * f);
  uint32_t v = ldg_u16(meta + 2 * f);
  if (FMT == QNT_INT4_ASYM) v |= ((ldg_u8(meta + z0 + f / 2) >> (4 * (f & 1))) & 15u) << 16;
  if (FMT == QNT_FP4_RAZER) v |= ((ldg_u8(meta + z0 + f / 4) >> (2 * (f & 3))) & 3u) << 16;
  return v;
}

// Decode constants of a group from its raw metadata; pw = 2^f of the row
// (fp16 products), 1 for bf16.
template <int FMT, bool BF16>
__device__ __forceinline__ GtGroup gt_group(uint32_t raw, float pw) {
  GtGroup c = {};
  if (FMT == QNT_FP4_AFPQ) {
    const float sp = h2f(raw & 0xFFFFu) * pw, sn = h2f(raw >> 16) * pw;
    if (BF16) {
      c.fs = sp;
      c.fs2 = sn;
    } else {
      const uint32_t hp = __half_as_ushort(__float2half_rn(sp)), hn = __half_as_ushort(__float2half_rn(sn));
      c.s1 = pack2(hp, hp);
      c.s2 = pack2(hn, hn);
    }
    return c;
  }
  const float s = h2f(raw & 0xFFFFu) * pw;
  const uint32_t extra = raw >> 16;
  if (FMT == QNT_INT4_ASYM) {
    const uint32_t z = extra;
    if (BF16) {
      c.zlo = pack2(0x4300u + z, 0x4300u + z);                   // bf16 128 + z
      const uint32_t bits = __float_as_uint(s);
      const uint32_t hi = (bits & 0xFFFF0000u) >> 16;             // bf16 with the low mantissa bits cut
      const float lo = s - __uint_as_float(bits & 0xFFFF0000u);    // exact, <= 3 significant bits
      const uint32_t lob = __float_as_uint(lo) >> 16;
      c.s1 = pack2(hi, hi);
      c.s3 = pack2(lob, lob);
    } else {
      c.zlo = pack2(0x6400u + z, 0x6400u + z);                   // fp16 1024 + z
      c.zhi = pack2(0x6400u + 16u * z, 0x6400u + 16u * z);       // fp16 1024 + 16 z
      const uint32_t h1 = __half_as_ushort(__float2half_rn(s));
      const uint32_t h16 = __half_as_ushort(__float2half_rn(s * 0.0625f));
      c.s1 = pack2(h1, h1);
      c.s2 = pack2(h16, h16);
    }
    return c;
  }
  if (FMT == QNT_FP4_RAZER) {   // the pair (2 sv, 2 sv): +-16 or +-10
    const uint32_t sv2 = ((extra & 2u) ? 0x4C00u : 0x4900u) | ((extra & 1u) ? 0x8000u : 0u);
    c.sv = sv2 | (sv2 << 16);
  }
  if (BF16) {
    c.fs = s;
  } else {
    const uint32_t h = __half_as_ushort(__float2half_rn(s));
    c.s1 = pack2(h, h);
  }
  return c;
}

// One 16-byte chunk (32 weights of the row, chunk-local k = 0..31) -> 16
// registers of A in k order (register i: k = 2i, 2i + 1).
template <int FMT, bool BF16>
__device__ __forceinline__ void gt_decode_chunk(const uint4& cv, const GtGroup& c, uint32_t (&a)[16]) {
  const uint32_t w[4] = {cv.x, cv.y, cv.z, cv.w};
  if constexpr (FMT == QNT_INT4_ASYM) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      // nibbles p = 0..7 of word j: chunk weights 16(p%2) + 4j + 2((p/2)%2) + p/4
      if (BF16) {
        const uint32_t q0 = and_or(w[j], 0x000F000Fu, 0x43004300u);          // k = 4j, 4j+1
        const uint32_t q1 = and_or(w[j] >> 8, 0x000F000Fu, 0x43004300u);     // k = 4j+2, 4j+3
        const uint32_t q2 = and_or(w[j] >> 4, 0x000F000Fu, 0x43004300u);     // k = 16+4j, 17+4j
        const uint32_t q3 = and_or(w[j] >> 12, 0x000F000Fu, 0x43004300u);    // k = 18+4j, 19+4j
        const uint32_t d0 = bsub2(q0, c.zlo), d1 = bsub2(q1, c.zlo), d2 = bsub2(q2, c.zlo), d3 = bsub2(q3, c.zlo);
        a[2 * j] = bfma2(d0, c.s1, bmul2(d0, c.s3));
        a[2 * j + 1] = bfma2(d1, c.s1, bmul2(d1, c.s3));
        a[8 + 2 * j] = bfma2(d2, c.s1, bmul2(d2, c.s3));
        a[8 + 2 * j + 1] = bfma2(d3, c.s1, bmul2(d3, c.s3));
      } else {
        const uint32_t w8 = w[j] >> 8;
        a[2 * j] = hmul2_(hsub2(and_or(w[j], 0x000F000Fu, 0x64006400u), c.zlo), c.s1);
        a[2 * j + 1] = hmul2_(hsub2(and_or(w8, 0x000F000Fu, 0x64006400u), c.zlo), c.s1);
        a[8 + 2 * j] = hmul2_(hsub2(and_or(w[j], 0x00F000F0u, 0x64006400u), c.zhi), c.s2);
        a[8 + 2 * j + 1] = hmul2_(hsub2(and_or(w8, 0x00F000F0u, 0x64006400u), c.zhi), c.s2);
      }
    }
  } else {
  // FP4 family: byte b of word j holds chunk weights 8j + 2b, 8j + 2b + 1
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    uint32_t h[4];
    cvt_e2m1x8(w[j], h[0], h[1], h[2], h[3]);
    if (FMT == QNT_FP4_RAZER) {
      // codes 0b1000 (decoded as -0) take the group's special value, branch
      // free: -0 + 0.5 * 2 sv = sv where the code is 0b1000, x + 0 elsewhere
      const uint32_t tt = (w[j] & 0x77777777u) + 0x77777777u;
      const uint32_t spec = lop3<0x20>(w[j], tt, 0x88888888u);   // bit 3 of every nibble equal to 0b1000
      uint32_t ind[4];
      cvt_e2m1x8(spec >> 3, ind[0], ind[1], ind[2], ind[3]);
#pragma unroll
      for (int p = 0; p < 4; ++p) h[p] = hfma2(ind[p], c.sv, h[p]);
    }
#pragma unroll
    for (int p = 0; p < 4; ++p) {
      if (BF16) {
        const float v0 = h2f(h[p] & 0xFFFFu), v1 = h2f(h[p] >> 16);
        if (FMT == QNT_FP4_AFPQ)
          a[4 * j + p] = f2bf_pair(v0 * (v0 > 0.0f ? c.fs : c.fs2), v1 * (v1 > 0.0f ? c.fs : c.fs2));
        else
          a[4 * j + p] = f2bf_pair(v0 * c.fs, v1 * c.fs);
      } else if (FMT == QNT_FP4_AFPQ) {
        const uint32_t vp = hmax2(h[p], 0u);
        const uint32_t vn = hsub2(h[p], vp);                     // min(v, 0), exact
        a[4 * j + p] = hfma2(vn, c.s2, hmul2_(vp, c.s1));         // one product is zero: one rounding
      } else {
        a[4 * j + p] = hmul2_(h[p], c.s1);
      }
    }
  }
  }
}

// ------------------------------------------------------------------ kernel
template <int FMT, int G, bool BF16>
__global__ void __launch_bounds__(kGtThreads, 1)
gemm_tc_kernel(const __grid_constant__ CUtensorMap xmap, const __grid_constant__ CUtensorMap cmap, const GtArgs A) {
  extern __shared__ __align__(1024) uint8_t smem[];
  uint64_t* full = reinterpret_cast<uint64_t*>(smem);       // [nst] codes + X landed
  // [nst] the stage's MMAs are complete: frees its shared-memory slot and (for
  // stage s + nA) its A slot; one commit per issuer and stage
  uint64_t* empty = full + kGtMaxStages;
  uint64_t* afull = empty + kGtMaxStages;                    // [A slots] A written to tensor memory
  uint64_t* dfull = afull + kGtMaxASlots;                    // all MMAs complete
  uint64_t* tmem_ready = dfull + 1;
  uint64_t* red_ready = tmem_ready + 1;                      // split: the leader's ring is free for partial sums
  uint64_t* red_full = red_ready + 1;                        // split, leader: every other CTA's partial sums landed
  uint32_t* tbase_p = reinterpret_cast<uint32_t*>(smem + 512);
  volatile int* abort_s = reinterpret_cast<volatile int*>(smem + 520);
  const int nst = A.nstages, nI = A.nissuers, nA = A.naslots;
  const GtSmem L = gt_smem(A.Mpad, nst);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int GK = A.K / G;
  // split of K: the A.split CTAs of a cluster share a tile, CTA `crank` takes
  // stages [s0, s0 + KB) of it; the leader (rank 0) sums the partial results
  const int S = A.split;
  const int crank = S > 1 ? (int)cluster_rank() : 0;
  const int tile = blockIdx.x / S;
  const int KBt = A.K / 128;
  const int s0 = crank * KBt / S, KB = (crank + 1) * KBt / S - s0;

  if (tid == 0) {
    for (int i = 0; i < nst; ++i) {
      mbar_init_nofence(full + i, 1);
      mbar_init_nofence(empty + i, nI);
    }
    for (int i = 0; i < nA; ++i) mbar_init_nofence(afull + i, 4);
    mbar_init_nofence(dfull, nI);
    mbar_init_nofence(tmem_ready, 1);
    mbar_init_nofence(red_ready, 1);
    mbar_init_nofence(red_full, S > 1 ? S - 1 : 1);
    mbar_init_fence();
    *abort_s = 0;
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  }
  __syncthreads();
  if (S > 1) cluster_sync();   // every CTA's barriers are initialized before any remote arrival
  if (warp == kGtMmaWarp0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 :: "r"(smem_addr(tbase_p)), "r"(kGtTmemCols) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    tc_fence_before();
    __syncwarp();
    if (lane == 0) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" :: "r"(smem_addr(tmem_ready)) : "memory");
  }
  auto fail = [&]() {
    *abort_s = 1;
    report(A.status, QNT_ERR_TIMEOUT);
  };
  auto wait = [&](uint64_t* bar, uint32_t parity, volatile int* ab, uint32_t max_sleep = 128, bool cluster_scope = false) {
    return gt_wait(bar, parity, ab, A.timeout_ns, max_sleep, cluster_scope);
  };

  if (warp == 0) {
    // ---------------------------------------------------------------- producer
    if (lane == 0) {
      const uint64_t pol = l2_evict_first_policy();
      const uint32_t stage_tx = (uint32_t)kGtCodeBytes + (uint32_t)A.Mpad * 256u;   // full boxes, zero-filled past the ends
      auto stage_ptr = [&](int s) { return smem + L.stage0 + (size_t)(s % nst) * L.stage_bytes; };
      auto issue_codes = [&](int s) {
        mbar_expect_tx(full + s % nst, stage_tx);
        tma_load_2d_hint(stage_ptr(s), &cmap, (s0 + s) * 128, tile * 16, full + s % nst, pol);
      };
      auto issue_x = [&](int s) {
        uint8_t* st = stage_ptr(s);
        tma_load_2d(st + L.xoff, &xmap, (s0 + s) * kGtStageK, 0, full + s % nst);
        tma_load_2d(st + L.xoff + (size_t)A.Mpad * 128, &xmap, (s0 + s) * kGtStageK + 64, 0, full + s % nst);
      };
      // the first stages' codes do not depend on the preceding kernel; X does
      const int pre = min(nst, KB);
      int s = 0;
      for (; s < pre; ++s) issue_codes(s);
      asm volatile("griddepcontrol.wait;" ::: "memory");
      for (int i = 0; i < pre; ++i) issue_x(i);
      GtRing er;   // the stage whose slot stage s reuses: s - nst
      for (; s < KB; ++s) {
        if (!wait(empty + er.slot, er.phase, abort_s, 512)) {
          if (!*abort_s) fail();
          break;
        }
        er.next(nst);
        issue_codes(s);
        issue_x(s);
      }
      // drain: the copies of every issued stage have landed
      for (int i = (s > nst ? s - nst : 0); i < s; ++i) wait(full + i % nst, (uint32_t)(i / nst) & 1u, nullptr);
    }
  } else if (warp < kGtMmaWarp0 + kGtMaxIssuers) {
    // ---------------------------------------------------------------- MMA issuers
    const int me = warp - kGtMmaWarp0;
    if (lane == 0 && me < nI) {
      if (!wait(tmem_ready, 0, abort_s)) {
        if (!*abort_s) fail();
      } else {
        tc_fence_after();
        const uint32_t tbase = *tbase_p;
        const uint32_t dcol = tbase + (uint32_t)(me * A.Mpad);
        const uint32_t idesc = f16_idesc(A.Mpad, BF16 ? 1 : 0);
        const uint32_t st0 = smem_addr(smem + L.stage0);
        const int per = 8 / nI, kk0 = me * per;
        GtRing fr, ar;
        for (int s = 0; s < KB; ++s) {
          const int slot = fr.slot, as = ar.slot;
          if (!wait(full + slot, fr.phase, abort_s, 0) || !wait(afull + as, ar.phase, abort_s, 0)) {
            if (!*abort_s) fail();
            break;
          }
          fr.next(nst);
          ar.next(nA);
          tc_fence_after();
          const uint32_t xs = st0 + (uint32_t)(slot * L.stage_bytes + L.xoff);
          const uint32_t acol = tbase + (uint32_t)A.cola + 64u * (uint32_t)as;
          for (int kk = kk0; kk < kk0 + per; ++kk) {
            const uint32_t b_addr = xs + (uint32_t)((kk >> 2) * A.Mpad * 128) + 32u * (uint32_t)(kk & 3);
            tc_mma_tmem_a(dcol, acol + 8u * (uint32_t)kk, sw128_desc(b_addr), idesc, (s > 0 || kk > kk0) ? 1u : 0u);
          }
          tc_commit(empty + slot);
        }
      }
      tc_commit(dfull);   // arrives once every MMA this thread issued has completed
    }
  } else {
    // ---------------------------------------------------------------- decode and epilogue
    const int dw = warp - kGtDecodeWarp0;
    const int quarter = warp & 3;                              // tensor-memory lanes 32 quarter ..
    const int grp = dw >> 2;                                   // stages grp, grp + kGtGroups, ...
    const int r = 32 * quarter + lane;                         // row of the tile
    const long row = (long)tile * kGtRows + r;
    const bool rowok = row < A.N;
    const long rowm = rowok ? row : (long)tile * kGtRows;      // a row with metadata
    const int rg = r >> 3, i8 = r & 7;
    // the row's power of two: fp16 products (q - z) s 2^f stay below 2^15
    float pw = 1.0f, unpw = 1.0f;
    if (!BF16) {
      float smax = 0.0f;
#pragma unroll 8
      for (int gi = 0; gi < GK; ++gi) {
        const long f = rowm * GK + gi;
        if (FMT == QNT_FP4_AFPQ) {
          const uint32_t w = ldg_u32(A.meta + 4 * f);
          smax = fmaxf(smax, fmaxf(h2f(w & 0xFFFFu), h2f(w >> 16)));
        } else {
          smax = fmaxf(smax, h2f(ldg_u16(A.meta + 2 * f)));
        }
      }
      const float vmax = FMT == QNT_INT4_ASYM ? 15.0f : (FMT == QNT_FP4_RAZER ? 8.0f : 6.0f);
      int e = 0;
      const float top = smax * vmax;
      if (top > 0.0f && isfinite(top)) e = min(max(14 - ((int)((__float_as_uint(top) >> 23) & 255u) - 127), -24), 24);
      pw = __uint_as_float((uint32_t)(127 + e) << 23);
      unpw = __uint_as_float((uint32_t)(127 - e) << 23);
    }
    uint32_t tbase = 0;
    bool ok = wait(tmem_ready, 0, abort_s);
    if (ok) {
      tc_fence_after();
      tbase = *tbase_p;
    } else if (!*abort_s) {
      fail();
    }
    const uint32_t tlane = (uint32_t)(32 * quarter) << 16;
    const uint32_t st0 = smem_addr(smem + L.stage0);
    // raw metadata of the row's groups in a stage, requested kPf of this
    // group's stages ahead
    constexpr int kGps = 128 / G;   // groups per stage
    constexpr int kPf = 2;
    uint32_t raw[kPf][kGps];
    auto load_raw = [&](int s, uint32_t (&out)[kGps]) {
      if (s >= KB) return;
#pragma unroll
      for (int h = 0; h < kGps; ++h) out[h] = gt_meta_raw<FMT>(A.meta, A.z0, rowm * GK + (long)(s0 + s) * kGps + h);
    };
#pragma unroll
    for (int u = 0; u < kPf; ++u) load_raw(grp + u * kGtGroups, raw[u]);
    // ring positions of this group's next stage; nst and nA are multiples of
    // kGtGroups, so the stage that last used a slot was this group's own
    GtRing fr, ar, er;   // er: the stage s - nA whose completion frees stage s's A slot
    bool er_set = false;
    fr.adv(grp, nst);
    ar.adv(grp, nA);
    for (int s0 = grp; s0 < KB && ok; s0 += kGtGroups * kPf) {
#pragma unroll
      for (int u = 0; u < kPf; ++u) {
        const int s = s0 + u * kGtGroups;
        if (s >= KB || !ok) break;
        GtGroup c[kGps];
#pragma unroll
        for (int h = 0; h < kGps; ++h) c[h] = gt_group<FMT, BF16>(raw[u][h], pw);
        load_raw(s + kGtGroups * kPf, raw[u]);
        const int slot = fr.slot, as = ar.slot;
        // the A slot is free once stage s - nA's MMAs are complete
        if (s >= nA && !er_set) {
          er.slot = (s - nA) % nst;
          er.phase = (uint32_t)((s - nA) / nst) & 1u;
          er_set = true;
        }
        if ((s >= nA && !wait(empty + er.slot, er.phase, abort_s)) || !wait(full + slot, fr.phase, abort_s)) {
          if (!*abort_s) fail();
          ok = false;
          break;
        }
        fr.adv(kGtGroups, nst);
        ar.adv(kGtGroups, nA);
        if (er_set) er.adv(kGtGroups, nst);
        tc_fence_after();
        const uint32_t cbase = st0 + (uint32_t)(slot * L.stage_bytes) + (uint32_t)(rg * 512 + 64 * i8);
        const uint32_t abase = tbase + tlane + (uint32_t)A.cola + 64u * (uint32_t)as;
#pragma unroll
        for (int chunk = 0; chunk < 4; ++chunk) {
          const uint4 cv = lds128a(cbase + 16u * (uint32_t)(chunk ^ ((i8 >> 1) & 3)));
          uint32_t av[16];
          gt_decode_chunk<FMT, BF16>(cv, c[chunk * 32 / G], av);
          tmem_st16(abase + 16u * (uint32_t)chunk, av);
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
#ifdef QNT_TEST_FAULTS
        // fault 1 (test builds): in CTA 0 the warp of lane quarter 0 never reports
        // stage 0 decoded, so the MMA issuers' wait for it expires
        const bool skip = A.fault == 1 && tile == 0 && s == 0 && quarter == 0;
#else
        constexpr bool skip = false;
#endif
        if (lane == 0 && !skip)
          asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" :: "r"(smem_addr(afull + as)) : "memory");
      }
    }
    // epilogue: 16-column chunks of the accumulator rows, dealt out to the
    // groups, summed over the accumulators (and, split, over the cluster's CTAs)
    const bool have = ok && wait(dfull, 0, abort_s);
    if (have) tc_fence_after();
    else if (!*abort_s) fail();
    auto tmem_sum = [&](int cc, float (&acc)[16]) {
#pragma unroll
      for (int e = 0; e < 16; ++e) acc[e] = 0.0f;
      for (int i = 0; i < nI; ++i) {
        uint32_t d[16];
        tmem_ld16(tbase + tlane + (uint32_t)(i * A.Mpad + cc), d);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 16; ++e) acc[e] += __uint_as_float(d[e]);
      }
    };
    // partial sums of CTA k > 0 in the leader's ring: float [k - 1][column][row]
    const uint32_t red0 = st0;
    if (S > 1 && crank != 0) {
      // wait until the leader's ring is free, write this CTA's partial sums
      // there, then tell the leader (one arrival per CTA, after all decode warps)
      const bool can = have && wait(red_ready, 0, abort_s, 512, true);
      if (have && !can && !*abort_s) fail();
      if (can) {
        const uint32_t dst0 = cluster_map(red0, 0u);
        for (int cc = 16 * grp; cc < A.Mpad; cc += 16 * kGtGroups) {
          float acc[16];
          tmem_sum(cc, acc);
#pragma unroll
          for (int e = 0; e < 16; ++e)
            cluster_st_f32(dst0 + 4u * (uint32_t)((((crank - 1) * A.Mpad) + cc + e) * kGtRows + r), acc[e]);
        }
      }
      asm volatile("bar.sync 2, %0;" :: "r"(32 * 4 * kGtGroups) : "memory");   // the decode warps
      if (dw == 0 && lane == 0) {
        asm volatile("fence.acq_rel.cluster;" ::: "memory");
        cluster_arrive(cluster_map(smem_addr(red_full), 0u));
      }
    } else if (have) {
      if (S > 1 && dw == 0 && lane == 0)   // the ring is read: the other CTAs may write their partial sums
        for (int k = 1; k < S; ++k) cluster_arrive(cluster_map(smem_addr(red_ready), (uint32_t)k));
      bool red_ok = true;
      if (S > 1) {
        red_ok = wait(red_full, 0, abort_s, 512, true);
        if (!red_ok && !*abort_s) fail();
      }
      if (red_ok) {
        for (int cc = 16 * grp; cc < A.Mpad; cc += 16 * kGtGroups) {
          float acc[16];
          tmem_sum(cc, acc);
          for (int k = 1; k < S; ++k)
#pragma unroll
            for (int e = 0; e < 16; ++e)
              acc[e] += lds32f(red0 + 4u * (uint32_t)((((k - 1) * A.Mpad) + cc + e) * kGtRows + r));
          if (rowok) {
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              const int m = cc + e;
              if (m < A.M) {
                const float v = acc[e] * unpw;
                const size_t o = (size_t)m * A.N + row;
                if (A.xbf16) reinterpret_cast<__nv_bfloat16*>(A.Y)[o] = __float2bfloat16_rn(v);
                else reinterpret_cast<__half*>(A.Y)[o] = __float2half_rn(v);
              }
            }
          }
        }
      }
    }
  }
  // teardown: every MMA issued has completed before tensor memory is freed
  __syncthreads();
  if (warp == kGtMmaWarp0) {
    if (lane == 0 && *abort_s) wait(dfull, 0, nullptr);   // each issuer's final commit follows its MMAs
    __syncwarp();
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" :: "r"(*tbase_p), "r"(kGtTmemCols) : "memory");
  }
  // split: no CTA leaves while another may still write into its shared memory
  // or arrive on its barriers (every path above reaches this point: all waits
  // are bounded)
  if (S > 1) {
    __syncthreads();
    cluster_sync();
  }
}

// ------------------------------------------------------------------ host
#ifdef QNT_TEST_FAULTS
static thread_local int t_gt_fault = 0;
static thread_local unsigned long long t_gt_timeout_ns = kGtTimeoutNs;
#define QNT_GT_FAULT t_gt_fault
#define QNT_GT_TIMEOUT t_gt_timeout_ns
#else
#define QNT_GT_FAULT 0
#define QNT_GT_TIMEOUT kGtTimeoutNs
#endif
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

template <int FMT, int G, bool BF16>
cudaError_t gt_launch(const qnt_desc& d, const void* codes, const void* meta, long z0, const void* X, void* Y, int M,
                      int* st, cudaStream_t s, bool* handled) {
  const int Mpad = (M + 15) / 16 * 16;
  int nst = 0;
  for (int k = kGtMaxStages / kGtGroups * kGtGroups; k >= 2 * kGtGroups && !nst; k -= kGtGroups)
    if (gt_smem(Mpad, k).total <= (size_t)kMaxDynSmem) nst = k;
  if (!nst) return cudaSuccess;
  auto enc = encode_fn();
  if (!enc) return cudaSuccess;
  // X: [M][K] fp16 / bf16, boxes of 64 columns x Mpad rows, 128-byte swizzle
  CUtensorMap xmap, cmap;
  {
    const cuuint64_t dims[2] = {(cuuint64_t)d.K, (cuuint64_t)M};
    const cuuint64_t strides[1] = {(cuuint64_t)d.K * 2};
    const cuuint32_t box[2] = {64u, (cuuint32_t)Mpad};
    const cuuint32_t estr[2] = {1u, 1u};
    if (enc(&xmap, BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(X),
            dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaSuccess;   // not handled
  }
  // codes: row groups of 4K bytes = K 32-bit words; boxes of one block (128
  // words) x 16 row groups, no swizzle (the layout's own chunk swizzle stays)
  {
    const cuuint64_t dims[2] = {(cuuint64_t)d.K, (cuuint64_t)((d.N + 7) / 8)};
    const cuuint64_t strides[1] = {(cuuint64_t)d.K * 4};
    const cuuint32_t box[2] = {128u, 16u};
    const cuuint32_t estr[2] = {1u, 1u};
    if (enc(&cmap, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<void*>(codes), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaSuccess;
  }
  auto kfn = gemm_tc_kernel<FMT, G, BF16>;
  cudaError_t e = configure_smem(reinterpret_cast<const void*>(kfn));
  if (e != cudaSuccess) return e;
  GtArgs a;
  a.meta = static_cast<const uint8_t*>(meta);
  a.Y = Y;
  a.z0 = z0;
  a.N = d.N;
  a.K = d.K;
  a.M = M;
  a.Mpad = Mpad;
  a.nstages = nst;
#ifndef QNT_GT_ISSUERS
#define QNT_GT_ISSUERS 4
#endif
  // MMA issuers (one accumulator of Mpad columns each): a small-N MMA keeps its
  // issuing thread ~60 cycles, so four threads share each stage's eight MMAs
  // (measured on 8192 x 28672, M = 16: one issuer 104 us, two 82, four 72)
  a.nissuers = min(QNT_GT_ISSUERS, Mpad <= 64 ? 4 : 2);
  a.cola = a.nissuers * Mpad;
  a.naslots = min(kGtMaxASlots, ((int)kGtTmemCols - a.cola) / 64) / kGtGroups * kGtGroups;
  a.xbf16 = BF16 ? 1 : 0;
  a.status = st;
  a.timeout_ns = QNT_GT_TIMEOUT;
  a.fault = QNT_GT_FAULT;
  // Split K over a cluster of `split` CTAs per tile when the tiles alone would
  // leave at least half of the SMs idle: a power of two up to 8, each CTA with
  // at least 4 stages, and the partial sums of the other CTAs fitting in the
  // leader's ring.
  const int tiles = (d.N + kGtRows - 1) / kGtRows, KBt = d.K / kGtStageK;
  const size_t ring = (size_t)nst * gt_smem(Mpad, nst).stage_bytes, part = (size_t)Mpad * kGtRows * 4;
  int split = 1;
  while (split < 8 && 2 * split * tiles <= num_sms() && KBt / (2 * split) >= 4 && (size_t)(2 * split - 1) * part <= ring)
    split *= 2;
  a.split = split;
  *handled = true;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(tiles * split);
  cfg.blockDim = dim3(kGtThreads);
  cfg.dynamicSmemBytes = gt_smem(Mpad, nst).total;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = (unsigned)split;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = split > 1 ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, kfn, xmap, cmap, a);
}

}  // namespace

// 1..128 activation rows (dispatched for 9..128, and for 3..8 where the batch-1 kernel's
// activation images do not fit), 4-bit formats, one pass over the weights.
cudaError_t launch_gemm_tc(const qnt_desc& d, const void* codes, const void* meta, long z0, const void* X, void* Y,
                           int M, int xbf16, int* st, cudaStream_t s, bool* handled) {
  *handled = false;
  if (M < 1 || M > 128) return cudaSuccess;
#define QNT_GT(FMT, BF)                                                                                     \
  switch (d.group) {                                                                                        \
    case 32: return gt_launch<FMT, 32, BF>(d, codes, meta, z0, X, Y, M, st, s, handled);                    \
    case 64: return gt_launch<FMT, 64, BF>(d, codes, meta, z0, X, Y, M, st, s, handled);                    \
    default: return gt_launch<FMT, 128, BF>(d, codes, meta, z0, X, Y, M, st, s, handled);                   \
  }
  if (xbf16) {
    switch (d.fmt) {
      case QNT_INT4_ASYM: QNT_GT(QNT_INT4_ASYM, true)
      case QNT_FP4_E2M1: QNT_GT(QNT_FP4_E2M1, true)
      case QNT_FP4_AFPQ: QNT_GT(QNT_FP4_AFPQ, true)
      case QNT_FP4_RAZER: QNT_GT(QNT_FP4_RAZER, true)
      default: return cudaSuccess;
    }
  }
  switch (d.fmt) {
    case QNT_INT4_ASYM: QNT_GT(QNT_INT4_ASYM, false)
    case QNT_FP4_E2M1: QNT_GT(QNT_FP4_E2M1, false)
    case QNT_FP4_AFPQ: QNT_GT(QNT_FP4_AFPQ, false)
    case QNT_FP4_RAZER: QNT_GT(QNT_FP4_RAZER, false)
    default: return cudaSuccess;
  }
#undef QNT_GT
}

#ifdef QNT_TEST_FAULTS
void set_test_gemm_fault(int fault, unsigned long long timeout_ns) {
  t_gt_fault = fault;
  t_gt_timeout_ns = timeout_ns;
}
#endif

}  // namespace qnt
