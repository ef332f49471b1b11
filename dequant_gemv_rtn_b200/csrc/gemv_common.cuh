// gemv_common.cuh -- metadata access and row partitioning shared by the GEMV
// kernels (gemv.cu: CUDA-core multi-vector kernel; gemv1.cu: batch-1 and
// sequence kernel on mma.sync).  Layout of the metadata planes: include/qnt.h.
#pragma once
#include "common.cuh"

namespace qnt {

__host__ __device__ inline size_t align16(size_t v) { return (v + 15) & ~size_t(15); }

// ------------------------------------------------------------------ metadata
struct GroupMeta {
  float s;   // INT4: s * 2^24; FP4 / RaZeR: s; AFPQ: s+
  float t;   // INT4: s * z;   AFPQ: s-;  RaZeR: special value
};

// Metadata of group f (= row * groups_per_row + group) from global memory.
template <int FMT>
__device__ __forceinline__ GroupMeta group_meta(const uint8_t* meta, long z0, long f) {
  GroupMeta g;
  if (FMT == QNT_FP4_AFPQ) {
    const uint32_t w = ldg_u32(meta + 4 * f);
    g.s = h2f(w & 0xFFFFu);
    g.t = h2f(w >> 16);
    return g;
  }
  const float s = h2f(ldg_u16(meta + 2 * f));
  if (FMT == QNT_INT4_ASYM) {
    const uint32_t z = (ldg_u8(meta + z0 + f / 2) >> (4 * (f & 1))) & 15u;
    g.s = s * 16777216.0f;     // 2^24 undoes the subnormal encoding
    g.t = s * (float)z;
  } else if (FMT == QNT_FP4_RAZER) {
    const uint32_t sel = (ldg_u8(meta + z0 + f / 4) >> (2 * (f & 3))) & 3u;
    const float sv = (sel & 2u) ? 8.0f : 5.0f;
    g.s = s;
    g.t = (sel & 1u) ? -sv : sv;
  } else {
    g.s = s;
    g.t = 0.0f;
  }
  return g;
}

// The metadata of a CTA's rows, staged in shared memory: 16-byte-aligned
// supersets of the scale plane (A bytes per group) and of the zero / selector
// plane (B bits per group) that the rows [r_lo, r_hi) use.
template <int FMT> struct MetaPlanes {
  static constexpr int A = (FMT == QNT_FP4_AFPQ) ? 4 : 2;
  static constexpr int B = (FMT == QNT_INT4_ASYM) ? 4 : (FMT == QNT_FP4_RAZER ? 2 : 0);
};
struct MetaWin { long a0, a1, b0, b1, bpl; };
template <int FMT>
__host__ __device__ inline MetaWin meta_window(long r_lo, long r_hi, long GK, long z0, long rows_cap) {
  using MP = MetaPlanes<FMT>;
  MetaWin m;
  m.a0 = (MP::A * r_lo * GK) & ~15L;
  m.a1 = (MP::A * r_hi * GK + 15) & ~15L;
  m.bpl = (MP::A * rows_cap * GK + 32 + 15) & ~15L;   // plane B's offset in the staged copy
  if (MP::B) {
    m.b0 = (z0 + (r_lo * GK * MP::B) / 8) & ~15L;
    m.b1 = (z0 + (r_hi * GK * MP::B + 7) / 8 + 15) & ~15L;
  } else {
    m.b0 = m.b1 = 0;
  }
  return m;
}
template <int FMT>
__host__ __device__ inline size_t meta_stage_bytes(long rows_cap, long GK) {
  using MP = MetaPlanes<FMT>;
  const size_t a = ((size_t)MP::A * rows_cap * GK + 32 + 15) & ~size_t(15);
  return a + (MP::B ? ((((size_t)rows_cap * GK * MP::B + 7) / 8 + 48 + 15) & ~size_t(15)) : 0);
}
// Metadata of group f from the staged copy.
template <int FMT>
__device__ __forceinline__ GroupMeta group_meta_s(const uint8_t* ms, const MetaWin& w, long z0, long f) {
  GroupMeta g;
  if (FMT == QNT_FP4_AFPQ) {
    const uint32_t v = lds_u32(ms + (4 * f - w.a0));
    g.s = h2f(v & 0xFFFFu);
    g.t = h2f(v >> 16);
    return g;
  }
  const float s = h2f(lds_u16(ms + (2 * f - w.a0)));
  if (FMT == QNT_INT4_ASYM) {
    const uint32_t z = (lds_u8(ms + w.bpl + (z0 + f / 2 - w.b0)) >> (4 * (f & 1))) & 15u;
    g.s = s * 16777216.0f;
    g.t = s * (float)z;
  } else if (FMT == QNT_FP4_RAZER) {
    const uint32_t sel = (lds_u8(ms + w.bpl + (z0 + f / 4 - w.b0)) >> (2 * (f & 3))) & 3u;
    const float sv = (sel & 2u) ? 8.0f : 5.0f;
    g.s = s;
    g.t = (sel & 1u) ? -sv : sv;
  } else {
    g.s = s;
    g.t = 0.0f;
  }
  return g;
}


// Rows of CTA b out of `grid`: 4-bit formats split whole row groups of eight.
__host__ __device__ inline void simt_rows(int fmt, long N, int b, int grid, long* r_lo, long* r_hi) {
  if (fmt == QNT_INT8_PERCHAN || fmt == QNT_FP16) {
    *r_lo = (long)b * N / grid;
    *r_hi = (long)(b + 1) * N / grid;
  } else {
    const long NG = (N + 7) / 8;
    *r_lo = 8 * ((long)b * NG / grid);
    const long hi = 8 * ((long)(b + 1) * NG / grid);
    *r_hi = hi < N ? hi : N;
  }
}

}  // namespace qnt
