// gemv_tc.cu -- fused-dequant GEMV / small-batch GEMM on the 5th-generation
// tensor cores (tcgen05), for the 4-bit formats INT4, FP4 (E2M1) and RaZeR and
// batches of up to 16 activation vectors.
//
// Computes what the RTN page ("Is (Selective) Round-To-Nearest Quantization
// All You Need?", English abstract: fused-dequant RTN kernels for token
// generation) and the RaZeR page ("The Power of Negative Zero", method section:
// 4-bit codes turned into FP16 with bit operations, fused with the product)
// describe:  y[m][n] = sum_k dq(code[n][k], meta[n][k/g]) * x[m][k].
//
// Why tensor cores for a memory-bound product: on CUDA cores every weight costs
// one FMA issue slot on top of its decode, so decode + FMA alone run at about
// the HBM rate and any overhead makes the kernel compute-bound.  Here the
// weights are decoded to fp16 by CUDA cores and written to tensor memory, and
// the multiply-accumulate runs on the tensor pipe, so each 8 weights cost 5
// bit operations (INT4) plus a share of one tensor-memory store.
//
// Structure (12 warps, one CTA per SM):
//  * rows: the CTA owns blocks of up to 128 rows (a balanced split of N over
//    the SMs); row r of a block is lane r of tensor memory, so the A operand
//    of tcgen05.mma (M = 128) is the block's weights, decoded.
//  * warp 0 streams the codes through a ring of shared-memory slots: a stage
//    is 256 weights of every row of the block, i.e. one contiguous 1 KB run per
//    row group of eight in the packed layout, so each stage is a few 1-D bulk
//    copies (TMA) issued by the warp's lanes in parallel; the same warp copies
//    the stage's activation slices and each row block's metadata.
//  * warp 3: builds each stage's activation images in shared memory: x of
//    every (vector, group) scaled by an exact power of two 2^e(m,g) that puts
//    the group maximum in [2^14, 2^15), as fp16 (bf16 inputs included), in the
//    K-major layout the MMA B descriptor reads; INT4 also gets a copy scaled by
//    1/16 and the group sums of x.
//  * warps 4-11: decode; warps 4+q and 8+q own tensor-memory lanes 32q..32q+31
//    and split every stage (chunks 0-3 / 4-7 and their groups); each decodes
//    stage s before finishing the epilogue of stage s-1, so the MMAs of a stage
//    overlap CUDA-core work.  INT4: a nibble masked into bits 0..3 of an fp16
//    half is the subnormal q * 2^-24 (bits 4..7 give 16 q * 2^-24, multiplied
//    by the 1/16 activation copy), exact.  FP4 / RaZeR: cvt.rn.f16x2.e2m1x2;
//    RaZeR codes 0b1000 are replaced by the group's special value.  The fp16
//    pairs go to tensor memory with tcgen05.st; after the MMAs, the same warps
//    read each group's accumulator (tcgen05.ld), apply scale / zero point and
//    2^-e, and accumulate y in registers.
//  * warps 1 and 2: one thread each issues the MMAs of half a stage (M = 128,
//    N = 16, K = 16, fp32 accumulation in tensor memory, one accumulator region
//    per group) and commits them to mbarriers; a single thread issues a
//    small-N MMA only every ~57 cycles, two of them about every 33.
//  * programmatic dependent launch: each CTA lets the next kernel in the stream
//    launch early, and queues its first weight and metadata copies before it
//    waits for the previous kernel (griddepcontrol.wait); only the activation
//    copies, and so every read of x and write of y, come after that wait.
//  Every wait is bounded; on a timeout the kernel reports QNT_ERR_TIMEOUT,
//  stops issuing work, drains what it issued and frees tensor memory.
#include "common.cuh"
#include "kernels.h"

namespace qnt {
namespace {

constexpr int kRowsTile = 128;                    // tensor-memory lanes = rows per block
constexpr int kStageK = 256;                      // weights of each row per stage
constexpr int kPiece = 8 * kStageK / 2;          // bytes of one row group per stage (1 KB)
constexpr int kCopyStages = 4;                    // stages per codes copy: one 4 KB run per row group
constexpr int kCPiece = kCopyStages * kPiece;     // 4 KB
constexpr int kMaxSlots = 64;                     // activation slots (one stage each)
constexpr int kMaxRingSlots = 8;                  // activation ring depth when they are not all resident
constexpr int kMaxCSlots = 4;                     // codes slots (kCopyStages stages each)
constexpr int kThreadsTc = 384;                   // 12 warps
constexpr int kMmaWarp1 = 1, kMmaWarp2 = 2;       // MMA issuers (chunks 0..3 / 4..7 of a stage)
constexpr int kPrepWarp = 3;
constexpr int kDecodeWarp0 = 4;
constexpr int kNumDecodeWarps = 8;                // two per lane quarter, each half of every stage
constexpr uint32_t kTmemCols = 512;               // A: 2 x 128 columns, D: 2 x 128 columns
constexpr uint32_t kColA = 0, kColD = 256;
constexpr int kCtrlBytesTc = 2048;               // barriers, tensor-memory base, abort flag

// ------------------------------------------------------------------ shared-memory plan
struct TcPlan {
  int MBp;            // B-operand rows per 16-byte k-chunk of the images: batch bucket x K splits
  int nslot;          // activation slots (one stage each)
  int ncs;            // codes slots (kCopyStages stages each)
  size_t cslot_bytes; // one codes slot: a 4 KB run for every (split, row group)
  size_t codes, ximg, xtab, meta, ybuf, total;
  size_t ximg_bytes;  // one activation image (x or x/16) of one slot, with read slack
  size_t xraw_bytes;  // raw activation slices of one slot ([MBp][256] fp16 / bf16), copied by TMA
  size_t slot_x;      // bytes per slot: raw slices, images, tables
  size_t meta_cap;
};

template <int FMT>
struct MetaPlanesTc {
  static constexpr int A = 2;                                           // fp16 scale per group
  static constexpr int B = (FMT == QNT_INT4_ASYM) ? 4 : (FMT == QNT_FP4_RAZER ? 2 : 0);   // bits per group
};

template <int FMT>
__host__ __device__ inline size_t meta_cap_bytes(int rows_cap, int GK) {
  using MP = MetaPlanesTc<FMT>;
  size_t a = ((size_t)MP::A * rows_cap * GK + 32 + 15) & ~size_t(15);
  size_t b = MP::B ? ((((size_t)rows_cap * GK * MP::B + 7) / 8 + 48 + 15) & ~size_t(15)) : 0;
  return a + b;
}

template <int FMT>
__host__ __device__ inline TcPlan tc_plan(int MB, int MBp, int nslot, int ncs, int npieces, int rows_cap, int GK) {
  TcPlan p;
  p.MBp = MBp;
  p.nslot = nslot;
  p.ncs = ncs;
  p.cslot_bytes = (size_t)npieces * kCPiece;
  p.ximg_bytes = (size_t)(kStageK / 8) * MBp * 16 + 256;
  p.xraw_bytes = (size_t)MBp * kStageK * 2;
  // raw slices, x image, x/16 image, then [MBp][8] group sums + [MBp][8] 2^-e
  p.slot_x = p.xraw_bytes + 2 * p.ximg_bytes + (size_t)MBp * 8 * 2 * 4;
  p.codes = kCtrlBytesTc;
  p.ximg = p.codes + (size_t)ncs * p.cslot_bytes;
  p.xtab = 0;  // per slot, inside the image block
  p.meta = (p.ximg + (size_t)nslot * p.slot_x + 15) & ~size_t(15);
  p.meta_cap = meta_cap_bytes<FMT>(rows_cap, GK);
  p.ybuf = (p.meta + p.meta_cap + 15) & ~size_t(15);
  p.total = p.ybuf + (size_t)2 * kRowsTile * MB * 4;   // partial y of every lane, per half
  return p;
}

// 16-byte-aligned metadata superset of rows [r_lo, r_hi) with GK groups per row.
struct MetaWin { long a0, a1, b0, b1; };
template <int FMT>
__device__ inline MetaWin meta_window(long r_lo, long r_hi, long GK, long z0) {
  using MP = MetaPlanesTc<FMT>;
  MetaWin m;
  m.a0 = (MP::A * r_lo * GK) & ~15L;
  m.a1 = (MP::A * r_hi * GK + 15) & ~15L;
  if (MP::B) {
    m.b0 = (z0 + (r_lo * GK * MP::B) / 8) & ~15L;
    m.b1 = (z0 + (r_hi * GK * MP::B + 7) / 8 + 15) & ~15L;
  } else {
    m.b0 = m.b1 = 0;
  }
  return m;
}

// ------------------------------------------------------------------ PTX wrappers
__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
// Bounded wait on phase `parity` without a suspend-time hint: the handoffs in
// this kernel (MMA commits, arrivals by other warps) are short, and a
// suspended waiter can sleep for its whole hint.  Gives up after about 2 s.
__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity) {
  const uint32_t a = smem_addr(bar);
  uint64_t t0 = 0;
  for (uint32_t it = 0;; ++it) {
    uint32_t done;
    asm volatile("{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\tselp.u32 %0, 1, 0, p;\n\t}"
                 : "=r"(done) : "r"(a), "r"(parity) : "memory");
    if (done) return true;
    if ((it & 255u) == 0) {
      const uint64_t t = global_ns();
      if (it == 0) t0 = t;
      else if (t - t0 > 2000000000ull) return false;
    }
  }
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
               :: "r"(smem_addr(bar)) : "memory");
}
// D[128 x 16] (+)= A[128 x 16] (tensor memory) * B[16 x 16] (shared memory, descriptor)
__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
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
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Load MB consecutive accumulator columns (fp32) of this thread's lane.
template <int MB>
__device__ __forceinline__ void tmem_ld(uint32_t taddr, uint32_t (&d)[MB]) {
  if constexpr (MB == 1) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x1.b32 {%0}, [%1];" : "=r"(d[0]) : "r"(taddr) : "memory");
  } else if constexpr (MB == 4) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3]) : "r"(taddr) : "memory");
  } else {
    static_assert(MB == 16, "batch buckets are 1, 4 and 16");
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3]), "=r"(d[4]), "=r"(d[5]), "=r"(d[6]), "=r"(d[7]),
          "=r"(d[8]), "=r"(d[9]), "=r"(d[10]), "=r"(d[11]), "=r"(d[12]), "=r"(d[13]), "=r"(d[14]), "=r"(d[15])
        : "r"(taddr) : "memory");
  }
}

// Shared-memory matrix descriptor: K-major, no swizzle; lbo = byte step between
// the two 8-element k-chunks of a K = 16 slice, sbo = byte step between groups of
// 8 rows (batch vectors).
__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46);
}

// Instruction descriptor of kind::f16: fp32 accumulator, fp16 A and B, both
// K-major, N = 16, M = 128.
constexpr uint32_t kIdesc = (1u << 4) | ((16u >> 3) << 17) | ((128u >> 4) << 24);

// ------------------------------------------------------------------ the kernel
template <int FMT, int G, int MB>
__global__ void __launch_bounds__(kThreadsTc, 1)
gemv_tc_kernel(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ meta, long z0,
               const void* __restrict__ X, void* __restrict__ Y, int N, int K, int M, int ldy, int xbf16,
               int rows_cap, int nslot, int ncs, int sk, int rcp, int Ks, int xres, int* d_status) {
  using MP = MetaPlanesTc<FMT>;
  constexpr int GPS = kStageK / G;          // groups per stage
  extern __shared__ __align__(1024) uint8_t smem[];
  const int GK = K / G;
  // K splits: tensor-memory lane v holds row v % rcp of the block for split
  // j = v / rcp (weights j*Ks .. j*Ks + Ks - 1), and B column j*MB + m holds the
  // matching slice of activation vector m, so one MMA serves all splits.
  const int MBp = MB * sk;
  const TcPlan P = tc_plan<FMT>(MB, MBp, nslot, ncs, (rows_cap / 8) * sk, rows_cap, GK);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem);            // [kMaxSlots] activation slices landed
  uint64_t* empty = full + kMaxSlots;                             // [kMaxSlots] activation slot consumed (MMAs + epilogue)
  uint64_t* xready = empty + kMaxSlots;                           // [kMaxSlots] activation images built
  uint64_t* cfull = xready + kMaxSlots;                           // [kMaxCSlots] codes landed
  uint64_t* cempty = cfull + kMaxCSlots;                          // [kMaxCSlots] codes decoded
  uint64_t* afull = cempty + kMaxCSlots;                          // [2] A buffer written
  uint64_t* mdone = afull + 2;                                    // [2] MMAs of a stage complete
  uint64_t* metafull = mdone + 2;                                 // row block metadata landed
  uint64_t* metafree = metafull + 1;                              // row block metadata no longer read
  uint64_t* mmafin = metafree + 1;                                // [2] all MMAs of an issuer complete (teardown)
  uint64_t* tmem_ready = mmafin + 2;                              // tensor memory allocated
  uint32_t* tbase_p = reinterpret_cast<uint32_t*>(smem + 1984);
  volatile int* abort_p = reinterpret_cast<volatile int*>(smem + 1988);
  uint8_t* codes_s = smem + P.codes;
  uint8_t* ximg_s = smem + P.ximg;
  uint8_t* meta_s = smem + P.meta;
  float* ybuf = reinterpret_cast<float*>(smem + P.ybuf);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nks = Ks / kStageK;                                   // stages per row block
  const int nblk_total = (N + rows_cap - 1) / rows_cap;          // rows_cap is a multiple of 8
  const int nblk = blockIdx.x < nblk_total ? (nblk_total - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
  const int nstages = nblk * nks;
  const int ncks = (nks + kCopyStages - 1) / kCopyStages;        // codes copies per row block
  // Activation images: with xres every stage of a row has its own slot (built
  // once, reused by every row block); otherwise a ring of nslot slots.
  auto xslot_of = [&](int s) { return xres ? s % nks : s % nslot; };
  auto xphase_of = [&](int s) { return xres ? 0u : (uint32_t)(s / nslot) & 1u; };

  if (tid == 0) {
    auto init = [](uint64_t* bar, uint32_t count) {   // one fence after all of them (below)
      asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" :: "r"(smem_addr(bar)), "r"(count));
    };
    for (int i = 0; i < nslot; ++i) { init(full + i, 1); init(empty + i, 2 + kNumDecodeWarps); init(xready + i, 1); }
    for (int i = 0; i < kMaxCSlots; ++i) { init(cfull + i, 1); init(cempty + i, kNumDecodeWarps); }
    for (int i = 0; i < 2; ++i) { init(afull + i, kNumDecodeWarps); init(mdone + i, 2); }
    init(metafull, 1);
    init(metafree, kNumDecodeWarps);
    init(mmafin, 1);
    init(mmafin + 1, 1);
    init(tmem_ready, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    *abort_p = 0;
  }
  __syncthreads();
  // Tensor memory is allocated by warp 1 while warp 0 already streams weights:
  // a CTA that starts on an SM still running the previous kernel's CTA waits
  // here until that CTA frees its columns, but its copies are under way.
  if (warp == kMmaWarp1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 :: "r"(smem_addr(tbase_p)), "r"(kTmemCols) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    tc_fence_before();
    __syncwarp();
    if (lane == 0) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" :: "r"(smem_addr(tmem_ready)) : "memory");
  }
  uint32_t tbase = 0;
  auto get_tmem = [&]() -> bool {   // bounded wait for the allocation
    if (!wait_bar(tmem_ready, 0)) return false;
    tc_fence_after();
    tbase = *tbase_p;
    return true;
  };

  auto fail = [&]() {
    *abort_p = 1;
    report(d_status, QNT_ERR_TIMEOUT);
  };
  auto block_of = [&](int p) { return (int)blockIdx.x + p * (int)gridDim.x; };
  // start of the zero / selector plane inside the staged metadata
  const size_t bplane = ((size_t)MP::A * rows_cap * GK + 32 + 15) & ~size_t(15);

  if (warp == 0) {
    // ---------------------------------------------------------------- producer: codes, activations, metadata
    const uint64_t pol = l2_evict_first_policy();
    const long NG = (N + 7) / 8;                    // row groups in the codes buffer
    const int gpb = rows_cap / 8;                   // row groups per block
    const int ncstages = nblk * ncks;
    auto issue_meta = [&](int p) {   // lane 0
      const long r0 = (long)block_of(p) * rows_cap;
      const long r1 = r0 + rows_cap < N ? r0 + rows_cap : N;
      const MetaWin w = meta_window<FMT>(r0, r1, GK, z0);
      mbar_expect_tx(metafull, (uint32_t)((w.a1 - w.a0) + (w.b1 - w.b0)));
      bulk_g2s(meta_s, meta + w.a0, (uint32_t)(w.a1 - w.a0), metafull);
      if (MP::B) bulk_g2s(meta_s + bplane, meta + w.b0, (uint32_t)(w.b1 - w.b0), metafull);
    };
    // codes copy cg: lanes 0..15 each copy the 4 KB run of one (split j, row group g)
    auto issue_codes = [&](int cg) {
      const int p = cg / ncks, cs = cg - p * ncks, cslot = cg % ncs;
      const long g0 = (long)block_of(p) * gpb;
      uint32_t nb = 0;
      const uint8_t* src = nullptr;
      uint8_t* dst = nullptr;
      if (lane < 16) {
        const int j = lane / gpb, g = lane - j * gpb;
        const long k = (long)j * Ks + (long)cs * kCopyStages * kStageK;
        const long kend = min((long)K, (long)(j + 1) * Ks);
        if (j < sk && g0 + g < NG && k < kend) {
          nb = (uint32_t)(min(kend - k, (long)kCopyStages * kStageK) / 128 * 512);
          src = codes + (g0 + g) * 4L * K + k / 128 * 512;
          dst = codes_s + (size_t)cslot * P.cslot_bytes + (size_t)(j * gpb + g) * kCPiece;
        }
      }
      uint32_t tot = nb;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) tot += __shfl_xor_sync(0xffffffffu, tot, o);
      if (lane == 0) mbar_expect_tx(cfull + cslot, tot);
      __syncwarp();
      if (nb) bulk_g2s_hint(dst, src, nb, cfull + cslot, pol);
    };
    // activation slices of stage s: lanes 16..31 each copy B row n (split j, vector m)
    auto issue_x = [&](int s) {
      const int p = s / nks, ks = s - p * nks, xslot = xslot_of(s);
      (void)p;
      uint32_t nb = 0;
      const uint8_t* src = nullptr;
      uint8_t* dst = nullptr;
      if (lane >= 16) {
        const int n = lane - 16, j = n / MB, m = n - j * MB;
        const long k = (long)j * Ks + (long)ks * kStageK;
        if (n < MBp && m < M && k < K) {
          nb = (uint32_t)((K - k < kStageK ? K - k : kStageK) * 2);
          src = static_cast<const uint8_t*>(X) + ((size_t)m * K + k) * 2;
          dst = ximg_s + (size_t)xslot * P.slot_x + (size_t)n * kStageK * 2;
        }
      }
      uint32_t tot = nb;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) tot += __shfl_xor_sync(0xffffffffu, tot, o);
      if (lane == 0) mbar_expect_tx(full + xslot, tot);
      __syncwarp();
      if (nb) bulk_g2s(dst, src, nb, full + xslot);
    };
    // Metadata and the first codes copies do not depend on the previous kernel:
    // they are requested before the dependency wait.
    if (lane == 0 && nblk > 0) issue_meta(0);
    int cg_next = 0;
    for (; cg_next < ncstages && cg_next < ncs; ++cg_next) issue_codes(cg_next);
    asm volatile("griddepcontrol.wait;" ::: "memory");
    int xissued = 0;
    if (xres && nstages > 0) {
      for (int ks = 0; ks < nks; ++ks) issue_x(ks);
      xissued = nks;
    }
    for (int s = 0; s < nstages && !*abort_p; ++s) {
      const int p = s / nks, ks = s - p * nks;
      bool ok = true;
      if (ks == 0 && p > 0) {   // row block metadata, after the previous block's readers are done
        if (lane == 0) {
          ok = wait_bar(metafree, (uint32_t)(p - 1) & 1u);
          if (ok) issue_meta(p);
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) { if (lane == 0) fail(); break; }
      }
      if (ks % kCopyStages == 0) {   // keep ncs codes copies in flight
        const int want = p * ncks + ks / kCopyStages + ncs - 1;
        while (ok && cg_next <= want && cg_next < ncstages) {
          if (lane == 0 && cg_next >= ncs) ok = wait_bar(cempty + cg_next % ncs, (uint32_t)(cg_next / ncs - 1) & 1u);
          ok = __shfl_sync(0xffffffffu, ok, 0);
          if (ok) issue_codes(cg_next++);
        }
        if (!ok) { if (lane == 0) fail(); break; }
      }
      if (!xres) {
        const int xslot = s % nslot;
        if (lane == 0 && s >= nslot) ok = wait_bar(empty + xslot, (uint32_t)(s / nslot - 1) & 1u);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) { if (lane == 0) fail(); break; }
        issue_x(s);
        xissued = s + 1;
      }
    }
    // drain: every issued copy must land before the CTA exits
    if (*abort_p && lane == 0) {
      for (int c = (cg_next > ncs ? cg_next - ncs : 0); c < cg_next; ++c) wait_bar(cfull + c % ncs, (uint32_t)(c / ncs) & 1u);
      for (int t = (xissued > nslot ? xissued - nslot : 0); t < xissued; ++t) wait_bar(full + xslot_of(t), xphase_of(t));
    }
  } else if (warp == kMmaWarp1 || warp == kMmaWarp2) {
    // ---------------------------------------------------------------- MMA issuers (half a stage each)
    const int half = warp == kMmaWarp1 ? 0 : 1;
    if (lane == 0 && !get_tmem()) fail();
    if (lane == 0 && !*abort_p) {
      const uint32_t img0 = smem_addr(ximg_s);
      const uint32_t lbo = 16u * MBp, sbo = 128u;
      for (int s = 0; s < nstages && !*abort_p; ++s) {
        const int slot = xslot_of(s), b = s & 1;
        if (!wait_bar(afull + b, (uint32_t)(s >> 1) & 1u)) { fail(); break; }
        if (!wait_bar(xready + slot, xphase_of(s))) { fail(); break; }
        tc_fence_after();
        const uint32_t x1 = img0 + (uint32_t)(slot * P.slot_x + P.xraw_bytes);
        const uint32_t x2 = x1 + (uint32_t)(FMT == QNT_INT4_ASYM ? P.ximg_bytes : 0);
        const uint32_t dcol = tbase + kColD + 128u * b, acol = tbase + kColA + 128u * b;
        // descriptor start addresses are in 16-byte units in the low bits: a chunk
        // (32 weights = 4 k-chunks of the image) advances them by 4 * MBp
        const uint64_t desc1 = smem_desc(x1, lbo, sbo), desc2 = smem_desc(x2 + 32u * MBp, lbo, sbo);
#pragma unroll
        for (int c = 4 * half; c < 4 * half + 4; ++c) {   // groups never straddle the halves (G <= 128)
          const uint32_t d = dcol + 16u * ((32 * c) / G);
          tc_mma(d, acol + 16u * c, desc1 + (uint64_t)(4 * c * MBp), kIdesc, ((32 * c) % G) != 0);
          tc_mma(d, acol + 16u * c + 8u, desc2 + (uint64_t)(4 * c * MBp), kIdesc, 1u);
        }
        tc_commit(mdone + b);
        if (!xres) tc_commit(empty + slot);
      }
      tc_commit(mmafin + half);   // tracks every MMA this thread issued
      if (!wait_bar(mmafin + half, 0)) fail();
    }
  } else if (warp == kPrepWarp) {
    // ---------------------------------------------------------------- activation images
    for (int s = 0; s < (xres ? (nstages > 0 ? nks : 0) : nstages); ++s) {
      if (*abort_p) break;
      const int ks = s % nks, slot = xslot_of(s);
      // the slot's copies have landed (and so its previous stage is fully consumed)
      if (!wait_bar(full + slot, xphase_of(s))) { fail(); break; }
      const uint8_t* xraw = ximg_s + (size_t)slot * P.slot_x;
      uint8_t* img1 = ximg_s + (size_t)slot * P.slot_x + P.xraw_bytes;
      uint8_t* img2 = img1 + P.ximg_bytes;
      float* xgs = reinterpret_cast<float*>(img1 + 2 * P.ximg_bytes);   // [MBp][8] group sums of x
      float* inv = xgs + MBp * 8;                                       // [MBp][8] 2^-e
      for (int n = 0; n < MBp; ++n) {                                   // B row n: split j, vector m
        const int j = n / MB, m = n - j * MB;
        const long k = (long)j * Ks + (long)ks * kStageK + 8 * lane;   // this lane's 8 activations
        float v[8];
        if (m < M && k < K) {
          const uint4 raw = lds128(xraw + (size_t)n * kStageK * 2 + 16 * lane);
          const uint32_t r4[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            if (xbf16) {
              v[2 * i] = __uint_as_float(r4[i] << 16);
              v[2 * i + 1] = __uint_as_float(r4[i] & 0xFFFF0000u);
            } else {
              v[2 * i] = h2f(r4[i] & 0xFFFFu);
              v[2 * i + 1] = h2f(r4[i] >> 16);
            }
          }
        } else {
#pragma unroll
          for (int i = 0; i < 8; ++i) v[i] = 0.0f;
        }
        float am = 0.0f, sum = 0.0f;
#pragma unroll
        for (int i = 0; i < 8; ++i) { am = fmaxf(am, fabsf(v[i])); sum += v[i]; }
#pragma unroll
        for (int o = 1; o < G / 8; o <<= 1) {
          am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, o));
          sum += __shfl_xor_sync(0xffffffffu, sum, o);
        }
        // e: exact power of two putting the group maximum into [2^14, 2^15)
        // (the maximum's binary exponent read from its bits; 0 for an all-zero group)
        int e = 0;
        if (am > 0.0f && isfinite(am)) e = min(max(14 - (int)((__float_as_uint(am) >> 23) & 255u) + 127, -122), 126);
        const float f1 = __uint_as_float((uint32_t)(127 + e) << 23);       // 2^e
        const float f16 = __uint_as_float((uint32_t)(123 + e) << 23);      // 2^(e-4)
        uint32_t o1[4], o2[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const __half2 a = __floats2half2_rn(v[2 * i] * f1, v[2 * i + 1] * f1);
          o1[i] = *reinterpret_cast<const uint32_t*>(&a);
          if (FMT == QNT_INT4_ASYM) {
            const __half2 b2 = __floats2half2_rn(v[2 * i] * f16, v[2 * i + 1] * f16);
            o2[i] = *reinterpret_cast<const uint32_t*>(&b2);
          }
        }
        const size_t off = ((size_t)lane * MBp + n) * 16;
        *reinterpret_cast<uint4*>(img1 + off) = make_uint4(o1[0], o1[1], o1[2], o1[3]);
        if (FMT == QNT_INT4_ASYM) *reinterpret_cast<uint4*>(img2 + off) = make_uint4(o2[0], o2[1], o2[2], o2[3]);
        if ((lane % (G / 8)) == 0) {
          const int gl = lane / (G / 8);
          xgs[n * 8 + gl] = sum;
          inv[n * 8 + gl] = __uint_as_float((uint32_t)(127 - e) << 23);   // 2^-e
        }
      }
      fence_proxy_async();   // make the images visible to the tensor core (async proxy)
      __syncwarp();
      if (lane == 0) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" :: "r"(smem_addr(xready + slot)) : "memory");
    }
  } else {
    // ---------------------------------------------------------------- decode + epilogue
    const int q = (warp - kDecodeWarp0) & 3;         // lane quarter
    const int hf = (warp - kDecodeWarp0) >> 2;       // half of every stage: chunks 4hf..4hf+3
    const int v = 32 * q + lane;                     // tensor-memory lane
    const int j = v / rcp, r = v - j * rcp;          // K split and row within the block
    const long kj = (long)j * Ks;                    // first weight of this lane's split
    const int i8 = v & 7;                            // row within its row group
    if (!get_tmem()) fail();
    const uint32_t lane_base = tbase + ((uint32_t)(32 * q) << 16);
    float y[MB];
#pragma unroll
    for (int m = 0; m < MB; ++m) y[m] = 0.0f;
    for (int p = 0; p < nblk; ++p) {
      const long r0 = (long)block_of(p) * rows_cap;
      const long r1 = r0 + rows_cap < N ? r0 + rows_cap : N;
      const long row = r0 + r;
      const bool live = j < sk && r < rows_cap && row < r1;
      const bool wlive = __any_sync(0xffffffffu, live);   // warp has work in this block
      const MetaWin mw = meta_window<FMT>(r0, r1, GK, z0);
      if (!*abort_p && !wait_bar(metafull, (uint32_t)p & 1u)) fail();

      // epilogue of stage t: per-group accumulators -> y, then release its slot
      auto epilogue = [&](int t) -> bool {
        const int kt = t - p * nks, slot = xslot_of(t), b = t & 1;
        if (!wait_bar(mdone + b, (uint32_t)(t >> 1) & 1u)) return false;
        tc_fence_after();
        const float* xgs = reinterpret_cast<const float*>(ximg_s + (size_t)slot * P.slot_x + P.xraw_bytes + 2 * P.ximg_bytes);
        const float* inv = xgs + MBp * 8;
        constexpr int GPH = GPS / 2;                   // groups of this half
#pragma unroll
        for (int gg = 0; gg < (wlive ? GPH : 0); ++gg) {
          const int gl = hf * GPH + gg;
          uint32_t d16[16];
          __syncwarp();
          tmem_ld<16>(lane_base + kColD + 128u * b + 16u * gl, d16);
          tmem_wait_ld();
          uint32_t dv[MB];   // columns j*MB .. j*MB + MB - 1 belong to this lane's split
#pragma unroll
          for (int m = 0; m < MB; ++m) dv[m] = d16[m];
          if (MB < 16) {
#pragma unroll
            for (int jj = 1; jj < 16 / MB && jj < 4; ++jj)
              if (j == jj) {
#pragma unroll
                for (int m = 0; m < MB; ++m) dv[m] = d16[(jj * MB + m) & 15];
              }
          }
          const long gi = (kj + (long)kt * kStageK) / G + gl;
          if (live && gi < GK) {
            const long f = row * GK + gi;
            const float sc = h2f(lds_u16(meta_s + (size_t)(2 * f - mw.a0)));
            float mul = sc, tz = 0.0f;
            if (FMT == QNT_INT4_ASYM) {
              const uint32_t z = (lds_u8(meta_s + bplane + (size_t)(z0 + f / 2 - mw.b0)) >> (4 * (f & 1))) & 15u;
              mul = sc * 16777216.0f;   // 2^24 undoes the subnormal encoding
              tz = sc * (float)z;
            }
#pragma unroll
            for (int m = 0; m < MB; ++m) {
              const int n = j * MB + m;
              y[m] = fmaf(mul * inv[n * 8 + gl], __uint_as_float(dv[m]), y[m]);
              if (FMT == QNT_INT4_ASYM) y[m] = fmaf(-tz, xgs[n * 8 + gl], y[m]);
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (!xres && lane == 0) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" :: "r"(smem_addr(empty + slot)) : "memory");
        return true;
      };

      // stage s is decoded before the epilogue of stage s-1 runs, so the MMAs of
      // s-1 execute while this warp decodes; A buffer s%2 was last read by the
      // MMAs of stage s-2, whose completion the epilogue of s-2 observed
      int pending = -1;
      for (int s = p * nks; s < (p + 1) * nks; ++s) {
        const int ks = s - p * nks;
        if (*abort_p) break;
        const int b = s & 1;
        const int cg = p * ncks + ks / kCopyStages, cslot = cg % ncs, sub = ks % kCopyStages;
        if (!wait_bar(cfull + cslot, (uint32_t)(cg / ncs) & 1u)) { fail(); break; }
        // ---- decode 8 chunks of this lane's row / split into A buffer b
        // row i8 of run v / 8 (stage sub at 1 KB sub): block h = c / 4 at 512 h,
        // row at 64 i8, chunk u = c % 4 at position u ^ (i8 / 2 % 4)
        // (lanes without a row read the slot start: the slot holds only the block's runs)
        const uint8_t* src = codes_s + (size_t)cslot * P.cslot_bytes +
                             (live ? (size_t)(v >> 3) * kCPiece + (size_t)sub * kPiece + 64 * i8 : 0);
#pragma unroll 4
        for (int c = 4 * hf; c < (wlive ? 4 * hf + 4 : 0); ++c) {
          const uint4 cw = lds128(src + (live ? 512 * (c >> 2) + (((c & 3) ^ ((i8 >> 1) & 3)) << 4) : 0));
          const uint32_t w[4] = {cw.x, cw.y, cw.z, cw.w};
          uint32_t a[16];
          if (FMT == QNT_INT4_ASYM) {
#pragma unroll
            for (int jw = 0; jw < 4; ++jw) {
              const uint32_t w8 = w[jw] >> 8;
              a[2 * jw] = w[jw] & 0x000F000Fu;          // chunk weights 4j, 4j+1   (q * 2^-24)
              a[2 * jw + 1] = w8 & 0x000F000Fu;         // 4j+2, 4j+3
              a[8 + 2 * jw] = w[jw] & 0x00F000F0u;      // 16+4j, 17+4j (16 q * 2^-24)
              a[8 + 2 * jw + 1] = w8 & 0x00F000F0u;     // 18+4j, 19+4j
            }
          } else {
#pragma unroll
            for (int jw = 0; jw < 4; ++jw) cvt_e2m1x8(w[jw], a[4 * jw], a[4 * jw + 1], a[4 * jw + 2], a[4 * jw + 3]);
            if (FMT == QNT_FP4_RAZER) {
              // codes 0b1000 take the group's special value (+5, -5, +8, -8 by selector)
              uint32_t spec[4];
              uint32_t any = 0;
#pragma unroll
              for (int jw = 0; jw < 4; ++jw) {
                const uint32_t t = (w[jw] & 0x77777777u) + 0x77777777u;
                spec[jw] = lop3<0x20>(w[jw], t, 0x88888888u);
                any |= spec[jw];
              }
              if (any && live) {
                const long f = row * GK + (kj + (long)ks * kStageK + 32 * c) / G;
                const uint32_t sel = (lds_u8(meta_s + bplane + (size_t)(z0 + f / 4 - mw.b0)) >> (2 * (f & 3))) & 3u;
                const uint32_t svb = (sel & 2u) ? 0x4800u : 0x4500u;
                const uint32_t sv16 = svb | ((sel & 1u) << 15);
#pragma unroll
                for (int jw = 0; jw < 4; ++jw) {
                  uint32_t sp = spec[jw];
                  while (sp) {
                    const int nib = (__ffs(sp) - 1) >> 2;   // nibble 0..7 of word jw
                    sp &= sp - 1;
                    uint32_t& h = a[4 * jw + (nib >> 1)];
                    h = (nib & 1) ? ((h & 0x0000FFFFu) | (sv16 << 16)) : ((h & 0xFFFF0000u) | sv16);
                  }
                }
              }
            }
          }
          __syncwarp();
          tmem_st16(lane_base + kColA + 128u * b + 16u * c, a);
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" :: "r"(smem_addr(afull + b)) : "memory");
        if ((sub == kCopyStages - 1 || ks == nks - 1) && lane == 0)   // this warp is done with the codes run
          asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" :: "r"(smem_addr(cempty + cslot)) : "memory");
        if (pending >= 0 && !epilogue(pending)) { fail(); pending = -1; break; }
        pending = s;
      }
      if (pending >= 0 && !*abort_p && !epilogue(pending)) fail();

      // ---- row block done: sum the partials of all splits of each row, write
      // y, release the metadata
#pragma unroll
      for (int m = 0; m < MB; ++m) ybuf[(hf * kRowsTile + v) * MB + m] = y[m];
      asm volatile("bar.sync 1, %0;" :: "r"(32 * kNumDecodeWarps) : "memory");
      if (hf == 0) {
        const int u = v;                              // row u of the block
        if (u < rows_cap && r0 + u < r1 && !*abort_p) {
          for (int m = 0; m < M && m < MB; ++m) {
            float acc = 0.0f;
            for (int jj = 0; jj < sk; ++jj)
              acc += ybuf[(jj * rcp + u) * MB + m] + ybuf[(kRowsTile + jj * rcp + u) * MB + m];
            const size_t o = (size_t)m * ldy + r0 + u;
            if (xbf16) reinterpret_cast<__nv_bfloat16*>(Y)[o] = __float2bfloat16_rn(acc);
            else reinterpret_cast<__half*>(Y)[o] = __float2half_rn(acc);
          }
        }
      }
#pragma unroll
      for (int m = 0; m < MB; ++m) y[m] = 0.0f;
      asm volatile("bar.sync 1, %0;" :: "r"(32 * kNumDecodeWarps) : "memory");
      if (lane == 0) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" :: "r"(smem_addr(metafree)) : "memory");
    }
  }

  // ---------------------------------------------------------------- teardown
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kMmaWarp1) {   // the allocating warp frees the columns (it always allocated them)
    const uint32_t t = *tbase_p;
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" :: "r"(t), "r"(kTmemCols) : "memory");
  }
}

// ------------------------------------------------------------------ host side
struct TcConfig { int rows_cap, grid, nslot, ncs, sk, rcp, Ks, xres; size_t smem; };

template <int FMT>
bool tc_config(const qnt_desc& d, int MB, TcConfig* c) {
  const int sms = num_sms();
  const int GK = d.K / d.group;
  const int NG = (d.N + 7) / 8;
  for (int passes = (NG + sms * 16 - 1) / (sms * 16); passes <= 64; ++passes) {
    const int rows_cap = 8 * ((NG + sms * passes - 1) / (sms * passes));   // whole row groups
    if (rows_cap > kRowsTile) continue;
    // K splits fill the tensor-memory lanes that the rows leave idle; each split
    // keeps at least two stages of work
    const int rcp = rows_cap;
    int sk = 1;
    for (int cand : {4, 2})
      if (MB * cand <= 16 && rcp * cand <= kRowsTile && d.K >= 2 * kStageK * cand) { sk = cand; break; }
    const int Ks = ((d.K + sk - 1) / sk + kStageK - 1) / kStageK * kStageK;
    const int nks = Ks / kStageK;
    auto take = [&](int ns, int ncs, int xres, size_t total) {
      const int nblk = (d.N + rows_cap - 1) / rows_cap;
      c->rows_cap = rows_cap;
      c->grid = nblk < sms ? nblk : sms;
      c->nslot = ns;
      c->ncs = ncs;
      c->sk = sk;
      c->rcp = rcp;
      c->Ks = Ks;
      c->xres = xres;
      c->smem = total;
    };
    // every stage's activation image resident, with the deepest codes ring that fits
    if (nks <= kMaxSlots)
      for (int ncs = kMaxCSlots; ncs >= 2; --ncs) {
        const TcPlan p = tc_plan<FMT>(MB, MB * sk, nks, ncs, (rows_cap / 8) * sk, rows_cap, GK);
        if (p.total <= (size_t)kMaxDynSmem) { take(nks, ncs, 1, p.total); return true; }
      }
    // else rings for both
    for (int ncs = kMaxCSlots; ncs >= 2; --ncs)
      for (int ns = kMaxRingSlots; ns >= 3; --ns) {
        const TcPlan p = tc_plan<FMT>(MB, MB * sk, ns, ncs, (rows_cap / 8) * sk, rows_cap, GK);
        if (p.total <= (size_t)kMaxDynSmem) { take(ns, ncs, 0, p.total); return true; }
      }
  }
  return false;
}

template <int FMT, int G, int MB>
cudaError_t launch_tc(const qnt_desc& d, const void* codes, const void* meta, long z0, const void* X, void* Y, int M,
                      int xbf16, int* st, cudaStream_t s, bool* handled) {
  TcConfig c;
  if (!tc_config<FMT>(d, MB, &c)) return cudaSuccess;   // not handled
  auto kfn = gemv_tc_kernel<FMT, G, MB>;
  cudaError_t e = configure_smem(reinterpret_cast<const void*>(kfn));
  if (e != cudaSuccess) return e;
  *handled = true;
  // programmatic dependent launch: the kernel orders its reads of X and writes
  // of Y after griddepcontrol.wait, so it may start before the previous kernel ends
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(c.grid);
  cfg.blockDim = dim3(kThreadsTc);
  cfg.dynamicSmemBytes = c.smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kfn, static_cast<const uint8_t*>(codes), static_cast<const uint8_t*>(meta), z0, X, Y,
                            d.N, d.K, M, d.N, xbf16, c.rows_cap, c.nslot, c.ncs, c.sk, c.rcp, c.Ks, c.xres, st);
}

template <int FMT, int MB>
cudaError_t launch_tc_g(const qnt_desc& d, const void* codes, const void* meta, long z0, const void* X, void* Y, int M,
                        int xbf16, int* st, cudaStream_t s, bool* handled) {
  switch (d.group) {
    case 32: return launch_tc<FMT, 32, MB>(d, codes, meta, z0, X, Y, M, xbf16, st, s, handled);
    case 64: return launch_tc<FMT, 64, MB>(d, codes, meta, z0, X, Y, M, xbf16, st, s, handled);
    default: return launch_tc<FMT, 128, MB>(d, codes, meta, z0, X, Y, M, xbf16, st, s, handled);
  }
}

template <int FMT>
cudaError_t launch_tc_mb(const qnt_desc& d, const void* codes, const void* meta, long z0, const void* X, void* Y, int M,
                         int xbf16, int* st, cudaStream_t s, bool* handled) {
  if (M == 1) return launch_tc_g<FMT, 1>(d, codes, meta, z0, X, Y, M, xbf16, st, s, handled);
  if (M <= 4) return launch_tc_g<FMT, 4>(d, codes, meta, z0, X, Y, M, xbf16, st, s, handled);
  return launch_tc_g<FMT, 16>(d, codes, meta, z0, X, Y, M, xbf16, st, s, handled);
}

}  // namespace

cudaError_t launch_gemv_tc(const qnt_desc& d, const void* codes, const void* meta, long z0, const void* X, void* Y,
                           int M, int xbf16, int* st, cudaStream_t s, bool* handled) {
  *handled = false;
  if (M < 1 || M > 16) return cudaSuccess;
  switch (d.fmt) {
    case QNT_INT4_ASYM: return launch_tc_mb<QNT_INT4_ASYM>(d, codes, meta, z0, X, Y, M, xbf16, st, s, handled);
    case QNT_FP4_E2M1: return launch_tc_mb<QNT_FP4_E2M1>(d, codes, meta, z0, X, Y, M, xbf16, st, s, handled);
    case QNT_FP4_RAZER: return launch_tc_mb<QNT_FP4_RAZER>(d, codes, meta, z0, X, Y, M, xbf16, st, s, handled);
    default: return cudaSuccess;
  }
}

}  // namespace qnt
