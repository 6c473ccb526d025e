// Device helpers: exact FP4 indexer scores from tensor-core accumulators,
// ranking keys, block maxima, status flags.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "internal.cuh"

namespace csa2 {

// Programmatic dependent launch (every kernel here is launched with it, see
// launch_k): launch_dependents lets the stream's next kernel be scheduled and
// run its prologue while this one still works; grid_wait blocks until every
// prerequisite grid has completed and its memory writes are visible.  Each
// kernel calls grid_wait in every CTA before its first global access, so the
// usual stream order holds for all data (and completes transitively).
__device__ __forceinline__ void launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void grid_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

__device__ __forceinline__ void set_status(uint32_t* status, uint32_t flag) {
  if (status) atomicOr(status, flag);
}

// Checked visible length of segment s: negative lengths count as 0, lengths
// above the host bound are clamped (CSA2_DEV_LENGTH), and a misaligned or
// out-of-capacity row range makes the segment empty (CSA2_DEV_ROW_LAYOUT).
// In the paged layout a length beyond the segment's page-table row makes
// the segment empty (CSA2_DEV_ROW_LAYOUT); page ids are checked where they
// are used (paged_row).
__device__ __forceinline__ int64_t seg_len_checked(const SegDesc& sd, int s, uint32_t* status) {
  int64_t L = sd.len[s];
  if (L < 0) L = 0;
  if (L > sd.max_len) {
    set_status(status, CSA2_DEV_LENGTH);
    L = sd.max_len;
  }
  if (sd.pages) {
    if (L > (int64_t(sd.max_pages) << sd.page_shift)) {
      set_status(status, CSA2_DEV_ROW_LAYOUT);
      L = 0;
    }
    return L;
  }
  const int64_t off = sd.row_off ? sd.row_off[s] : sd.row0;
  if ((off & 7) != 0 || off < 0 || off + L > sd.cache_rows) {
    set_status(status, CSA2_DEV_ROW_LAYOUT);
    L = 0;
  }
  return L;
}

// Cache row of position t (< the checked length) of a sequence whose
// page-table row is `row`: a page id outside the cache is reported
// (CSA2_DEV_ROW_LAYOUT) and read as page 0, so no access leaves the cache.
__device__ __forceinline__ int64_t paged_row(const int32_t* row, int shift, int64_t cache_rows, int64_t t,
                                             uint32_t* status) {
  int64_t pg = __ldg(row + (t >> shift));
  if (pg < 0 || ((pg + 1) << shift) > cache_rows) {
    set_status(status, CSA2_DEV_ROW_LAYOUT);
    pg = 0;
  }
  return (pg << shift) + (t & ((int64_t(1) << shift) - 1));
}

// Cache row of position t of segment s (either layout).
__device__ __forceinline__ int64_t seg_row(const SegDesc& sd, int s, int64_t t, uint32_t* status) {
  if (sd.pages)
    return paged_row(sd.pages + int64_t(s) * sd.max_pages, sd.page_shift, sd.cache_rows, t, status);
  return (sd.row_off ? sd.row_off[s] : sd.row0) + t;
}

// Test controls of the tensor-core kernels (see kCtlWaitUs): the pipeline
// wait limit in ns (the built-in `dflt` unless word 2 is set) and whether the
// producer withholds its first work item (word 3).
struct PipeCtl {
  uint64_t wait_ns;
  bool withhold;
};
__device__ __forceinline__ PipeCtl pipe_ctl(const uint32_t* status, uint64_t dflt) {
  PipeCtl c{dflt, false};
  if (status) {
    const uint32_t us = __ldcg(status + kCtlWaitUs);
    if (us) c.wait_ns = uint64_t(us) * 1000ull;
    c.withhold = __ldcg(status + kCtlWithhold) != 0u;
  }
  return c;
}

// Order-preserving map of an fp32 score to a uint32 key; -0 ranks as +0.
// Every NaN (whatever its sign and payload) maps to key 1, below every
// number including -inf (key 0x007FFFFF), so NaN positions rank last and
// among themselves by position.  Key 0 is reserved for "absent".
__device__ __forceinline__ uint32_t rank_key(float s) {
  if (s != s) return 1u;
  if (s == 0.0f) s = 0.0f;
  uint32_t u = __float_as_uint(s);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// 2^e as a double for e in [-1022, 1023] (exact).
__device__ __forceinline__ double pow2d(int e) {
  return __longlong_as_double(static_cast<long long>(e + 1023) << 52);
}

// Scale context of one indexer query for the tensor-core epilogues:
// qsh[h][b] = (E8M0 byte - 127) << 23 (an fp32 exponent-field offset), the
// head weights, and the range of the query's block exponents.
struct IdxQCtx {
  uint32_t qsh[kHi][4];
  float w[kHi];
  int qlo, qhi, qspread;
};

__device__ __forceinline__ void make_qctx(IdxQCtx& c, const uint8_t* q_scales /*[4][4]*/, const float* w /*[4]*/) {
  c.qlo = 255;
  c.qhi = 0;
  c.qspread = 0;
#pragma unroll
  for (int h = 0; h < kHi; ++h) {
    int mn = 255, mx = 0;
#pragma unroll
    for (int bb = 0; bb < 4; ++bb) {
      const int q = q_scales[h * 4 + bb];
      c.qsh[h][bb] = uint32_t(q - 127) << 23;
      mn = min(mn, q);
      mx = max(mx, q);
    }
    c.qlo = min(c.qlo, mn);
    c.qhi = max(c.qhi, mx);
    c.qspread = max(c.qspread, mx - mn);
    c.w[h] = w[h];
  }
}

// Exact score of one position from its 16 tensor-core accumulators
// v[4h+b] = D_{h,b}/4 (the block dot of doubled E2M1 values, exact in fp32)
// and its key's E8M0 scale word sw (block b in byte b):
//   d_h = fp32( sum_b D_{h,b} * 2^(eq+ek-2) )  (summed in order b = 0..3),
//   s = w0*d0, then s = fma(w_h, d_h, s); -0 -> +0.
// When the block exponents lie within 9 of each other (and away from the
// fp32 range limits) every term and partial sum is exact in fp32, so the sum
// is done there; otherwise in fp64 as the definition states.
// Key side of the score: the four block exponents of one indexer-K row.
struct KeyScale {
  int kb[4];
  int kmin, kmax;
};

__device__ __forceinline__ KeyScale key_scale(uint32_t sw) {
  KeyScale k;
  k.kb[0] = int(sw & 255u);
  k.kb[1] = int((sw >> 8) & 255u);
  k.kb[2] = int((sw >> 16) & 255u);
  k.kb[3] = int(sw >> 24);
  k.kmin = min(min(k.kb[0], k.kb[1]), min(k.kb[2], k.kb[3]));
  k.kmax = max(max(k.kb[0], k.kb[1]), max(k.kb[2], k.kb[3]));
  return k;
}

__device__ __forceinline__ float exact_score(const uint32_t (&v)[16], const KeyScale& ks, const IdxQCtx& q) {
  const bool fast = (ks.kmax - ks.kmin + q.qspread <= 9) && (q.qlo + ks.kmin - 254 >= -100) &&
                    (q.qhi + ks.kmax - 254 <= 100);
  float d[kHi];
  if (fast) {
#pragma unroll
    for (int h = 0; h < kHi; ++h) {
      float acc = __fmul_rn(__uint_as_float(v[4 * h]), __uint_as_float(q.qsh[h][0] + (uint32_t(ks.kb[0]) << 23)));
#pragma unroll
      for (int bb = 1; bb < 4; ++bb)
        acc = __fmaf_rn(__uint_as_float(v[4 * h + bb]), __uint_as_float(q.qsh[h][bb] + (uint32_t(ks.kb[bb]) << 23)),
                        acc);
      d[h] = acc;
    }
  } else {
#pragma unroll
    for (int h = 0; h < kHi; ++h) {
      double acc = 0.0;
#pragma unroll
      for (int bb = 0; bb < 4; ++bb) {
        const int e = int(int32_t(q.qsh[h][bb]) >> 23) + ks.kb[bb] - 127;  // eq + ek
        acc = __dadd_rn(acc, __dmul_rn(double(__uint_as_float(v[4 * h + bb])), pow2d(e)));
      }
      d[h] = __double2float_rn(acc);
    }
  }
  float sc = __fmul_rn(q.w[0], d[0]);
#pragma unroll
  for (int h = 1; h < kHi; ++h) sc = __fmaf_rn(q.w[h], d[h], sc);
  if (sc == 0.0f) sc = 0.0f;
  return sc;
}

__device__ __forceinline__ float exact_score(const uint32_t (&v)[16], uint32_t sw, const IdxQCtx& q) {
  return exact_score(v, key_scale(sw), q);
}

// Max over aligned groups of 8 lanes; every lane of the group gets it.
__device__ __forceinline__ uint32_t group8_max(uint32_t v) {
  v = max(v, __shfl_xor_sync(0xffffffffu, v, 1));
  v = max(v, __shfl_xor_sync(0xffffffffu, v, 2));
  v = max(v, __shfl_xor_sync(0xffffffffu, v, 4));
  return v;
}

}  // namespace csa2
