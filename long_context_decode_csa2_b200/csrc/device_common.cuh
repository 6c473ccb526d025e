// Device helpers: FP4 indexer scoring on CUDA cores, ranking keys, status.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "internal.cuh"

namespace csa2 {

__device__ __forceinline__ void set_status(uint32_t* status, uint32_t flag) {
  if (status) atomicOr(status, flag);
}

// Order-preserving map of an fp32 score to a uint32 key; -0 ranks as +0.
// Key 0 is reserved for "absent" (only a negative NaN would map there).
__device__ __forceinline__ uint32_t rank_key(float s) {
  if (s == 0.0f) s = 0.0f;
  uint32_t u = __float_as_uint(s);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// 2^e as a double for e in [-1022, 1023] (exact).
__device__ __forceinline__ double pow2d(int e) {
  return __longlong_as_double(static_cast<long long>(e + 1023) << 52);
}

// Doubled E2M1 value of a code: {0,1,2,3,4,6,8,12} with sign.
__device__ __forceinline__ int e2m1_twice(uint32_t code) {
  const uint32_t mag = (0xC8643210u >> (4 * (code & 7))) & 15u;  // nibbles 0,1,2,3,4,6,8,12
  return (code & 8) ? -static_cast<int>(mag) : static_cast<int>(mag);
}

// One indexer query prepared for dp4a scoring:
//   qp[h][m] packs the doubled values of elements 4m..4m+3 (signed bytes),
//   qn[h][m] the same bytes negated; eq[h][b] = block-scale exponent (byte-127);
//   w[h] the head weights.
struct IdxQueryPrep {
  uint32_t qp[kHi][32];
  uint32_t qn[kHi][32];
  int eq[kHi][4];
  float w[kHi];
};

// Fill `qs` from the raw query (call with all threads of the block, then sync).
__device__ __forceinline__ void prep_query(IdxQueryPrep& qs, const uint8_t* q_codes /*[4][64]*/,
                                           const uint8_t* q_scales /*[4][4]*/, const float* w, int tid,
                                           int nthreads) {
  for (int i = tid; i < kHi * 32; i += nthreads) {
    const int h = i / 32, m = i % 32;
    const uint8_t b0 = q_codes[h * 64 + 2 * m], b1 = q_codes[h * 64 + 2 * m + 1];
    const int v0 = e2m1_twice(b0 & 15), v1 = e2m1_twice(b0 >> 4);
    const int v2 = e2m1_twice(b1 & 15), v3 = e2m1_twice(b1 >> 4);
    qs.qp[h][m] = (uint32_t(v0) & 255u) | ((uint32_t(v1) & 255u) << 8) | ((uint32_t(v2) & 255u) << 16) |
                  ((uint32_t(v3) & 255u) << 24);
    qs.qn[h][m] = (uint32_t(-v0) & 255u) | ((uint32_t(-v1) & 255u) << 8) | ((uint32_t(-v2) & 255u) << 16) |
                  ((uint32_t(-v3) & 255u) << 24);
  }
  for (int i = tid; i < kHi * 4; i += nthreads) qs.eq[i / 4][i % 4] = int(q_scales[i]) - 127;
  for (int i = tid; i < kHi; i += nthreads) qs.w[i] = w[i];
}

// Exact block dot products D[h][b] (doubled-E2M1 integers) of one 128-element
// key row (16 code words) with the prepared query.
__device__ __forceinline__ void block_dots(const IdxQueryPrep& q, const uint32_t (&kw)[16], int (&D)[kHi][4]) {
#pragma unroll
  for (int h = 0; h < kHi; ++h)
#pragma unroll
    for (int b = 0; b < 4; ++b) D[h][b] = 0;
#pragma unroll
  for (int wd = 0; wd < 16; ++wd) {
    const uint32_t c = kw[wd];
    const uint32_t lo = c & 0xFFFFu, hi = c >> 16;
    const uint32_t mlo = __byte_perm(0x03020100u, 0x0C080604u, lo & 0x7777u);
    const uint32_t mhi = __byte_perm(0x03020100u, 0x0C080604u, hi & 0x7777u);
    const uint32_t slo = 0x3210u | ((lo & 0x8888u) >> 1);
    const uint32_t shi = 0x3210u | ((hi & 0x8888u) >> 1);
#pragma unroll
    for (int h = 0; h < kHi; ++h) {
      const uint32_t a0 = __byte_perm(q.qp[h][2 * wd], q.qn[h][2 * wd], slo);
      const uint32_t a1 = __byte_perm(q.qp[h][2 * wd + 1], q.qn[h][2 * wd + 1], shi);
      D[h][wd / 4] = __dp4a(int(a0), int(mlo), D[h][wd / 4]);
      D[h][wd / 4] = __dp4a(int(a1), int(mhi), D[h][wd / 4]);
    }
  }
}

// Score from exact block dots: per head the four terms D*2^(eq+ek-2) are
// summed in double in block order and rounded once to float; heads combine
// with an fp32 fma chain.  Explicit _rn intrinsics keep nvcc from contracting.
__device__ __forceinline__ float combine_score(const IdxQueryPrep& q, const int (&D)[kHi][4], uint32_t kscale_word) {
  float d[kHi];
#pragma unroll
  for (int h = 0; h < kHi; ++h) {
    double acc = 0.0;
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      const int ek = int((kscale_word >> (8 * b)) & 255u) - 127;
      const double term = __dmul_rn(static_cast<double>(D[h][b]), pow2d(q.eq[h][b] + ek - 2));
      acc = __dadd_rn(acc, term);
    }
    d[h] = __double2float_rn(acc);
  }
  float s = __fmul_rn(q.w[0], d[0]);
#pragma unroll
  for (int h = 1; h < kHi; ++h) s = __fmaf_rn(q.w[h], d[h], s);
  if (s == 0.0f) s = 0.0f;
  return s;
}

__device__ __forceinline__ void load_key_row(const uint8_t* kcodes, int64_t row, uint32_t (&kw)[16]) {
  const uint4* p = reinterpret_cast<const uint4*>(kcodes + row * kIdxCodeBytes);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint4 v = __ldg(p + i);
    kw[4 * i + 0] = v.x;
    kw[4 * i + 1] = v.y;
    kw[4 * i + 2] = v.z;
    kw[4 * i + 3] = v.w;
  }
}

__device__ __forceinline__ float score_row(const IdxQueryPrep& q, const uint8_t* kcodes, const uint8_t* kscales,
                                           int64_t row) {
  uint32_t kw[16];
  load_key_row(kcodes, row, kw);
  const uint32_t sw = __ldg(reinterpret_cast<const uint32_t*>(kscales) + row);
  int D[kHi][4];
  block_dots(q, kw, D);
  return combine_score(q, D, sw);
}

// Max over aligned groups of 8 lanes; every lane of the group gets it.
__device__ __forceinline__ uint32_t group8_max(uint32_t v) {
  v = max(v, __shfl_xor_sync(0xffffffffu, v, 1));
  v = max(v, __shfl_xor_sync(0xffffffffu, v, 2));
  v = max(v, __shfl_xor_sync(0xffffffffu, v, 4));
  return v;
}

}  // namespace csa2
