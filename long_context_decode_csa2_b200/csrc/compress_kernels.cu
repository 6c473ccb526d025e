// Pair compression (ratio 2) / pass-through (ratio 1), optional indexer-K
// projection, and OCP MXFP4 encoding of the new cache entries.
//
// "DeepSeek-V4.1-Flash: Pushing the Limits of KV Cache Compression": the
// architecture figure caption (ratio 2 in the encoder, 1 in the decoder),
// section "三个方向一起压小缓存" (disjoint sources, no absolute position
// encoding, indexer K projected from the main KV, MXFP4 after positional
// encoding) and section "后 20 层干脆共用一份 KV" (per-layer compression
// weights).  Every floating-point step is an explicit _rn intrinsic so that
// nvcc cannot contract it; the exp is this library's own (Cody & Waite
// reduction by ln 2, Taylor series of degree 14) so results are reproducible
// bit for bit on any IEEE-754 implementation taking the same steps.
#include "device_common.cuh"

namespace csa2 {

// ln 2 split into an exactly representable 24-bit head and a tail.
__device__ __constant__ double kLn2Head = 0.6931471824645996;   // 11629080 * 2^-24
__device__ __constant__ double kLn2Tail = -1.904654299957768e-09;
__device__ __constant__ double kInvLn2 = 1.4426950408889634;

__device__ double own_exp(double x) {
  if (x < -745.0) return 0.0;
  if (x > 709.0) return __longlong_as_double(0x7FF0000000000000LL);
  const double k = rint(__dmul_rn(x, kInvLn2));  // nearest, ties to even
  const double r = __dsub_rn(__dsub_rn(x, __dmul_rn(k, kLn2Head)), __dmul_rn(k, kLn2Tail));
  // Taylor coefficients 1/n!, n = 14 .. 0 (Horner)
  double p = 1.0 / 87178291200.0;
  p = __fma_rn(p, r, 1.0 / 6227020800.0);
  p = __fma_rn(p, r, 1.0 / 479001600.0);
  p = __fma_rn(p, r, 1.0 / 39916800.0);
  p = __fma_rn(p, r, 1.0 / 3628800.0);
  p = __fma_rn(p, r, 1.0 / 362880.0);
  p = __fma_rn(p, r, 1.0 / 40320.0);
  p = __fma_rn(p, r, 1.0 / 5040.0);
  p = __fma_rn(p, r, 1.0 / 720.0);
  p = __fma_rn(p, r, 1.0 / 120.0);
  p = __fma_rn(p, r, 1.0 / 24.0);
  p = __fma_rn(p, r, 1.0 / 6.0);
  p = __fma_rn(p, r, 1.0 / 2.0);
  p = __fma_rn(p, r, 1.0);
  p = __fma_rn(p, r, 1.0);
  const int ki = static_cast<int>(k);
  if (ki >= -1020) return __dmul_rn(p, pow2d(ki));
  return __dmul_rn(__dmul_rn(p, pow2d(ki + 1000)), pow2d(-1000));  // one rounding
}

__device__ __forceinline__ float bf16f(uint16_t b) { return __uint_as_float(uint32_t(b) << 16); }

// OCP MXFP4 block exponent X = floor(log2 amax) - 2, clamped to [-127, 127];
// amax == 0 gives -127.
__device__ __forceinline__ int mx_block_exp(float amax) {
  const uint32_t bits = __float_as_uint(amax);
  if (bits == 0u) return -127;
  const int e = int((bits >> 23) & 255u);
  int fl;
  if (e == 0) fl = -149 + (31 - __clz(int(bits & 0x7FFFFFu)));
  else fl = e - 127;
  return max(-127, min(127, fl - 2));
}

// 2^-X as float (X in [-127, 127]).
__device__ __forceinline__ float pow2f_neg(int X) {
  const int e = -X;  // in [-127, 127]
  return e >= -126 ? __uint_as_float(uint32_t(e + 127) << 23) : __uint_as_float(0x00400000u);
}

// E2M1 code of x at block exponent X: nearest magnitude, ties to the even
// mantissa, saturating at 6; the sign bit is x's sign bit.
__device__ __forceinline__ uint32_t e2m1_code(float x, float inv_scale) {
  const float a = fabsf(__fmul_rn(x, inv_scale));
  const uint32_t idx = uint32_t(a > 0.25f) + uint32_t(a >= 0.75f) + uint32_t(a > 1.25f) + uint32_t(a >= 1.75f) +
                       uint32_t(a > 2.5f) + uint32_t(a >= 3.5f) + uint32_t(a > 5.0f);
  return idx | ((__float_as_uint(x) >> 28) & 8u);
}

constexpr int kCompWarps = 8;
constexpr int kCompEntries = 16;                       // entries per CTA (two per warp)
constexpr int kCompGroups = kCompWarps * 32 / kDi;     // one-chain projection: entry groups of the CTA (2)
// Projection of a full CTA: thread t owns columns 2(t % 64), 2(t % 64) + 1
// of the entries e = 4q + t / 64 (q = 0..3), eight chains, and reads two
// consecutive terms of an entry's merged row per 16-byte shared load, so a
// shared load feeds four FMAs; W_idx rows are loaded one block ahead of their
// use.  (For 262144 tokens at ratio 2: one shared load per FMA, with each
// W_idx load just before its use, 1.36 ms; this, 1.11 ms; W_idx widened to
// fp64 once per call and read as doubles, 1.21 ms: twice the L2 bytes cost
// more than the conversions it saves.)
constexpr int kProjCols = 2;                                   // columns per projecting thread
constexpr int kProjGroups = kCompWarps * 32 * kProjCols / kDi; // entry groups (4)
constexpr int kProjEntries = kCompEntries / kProjGroups;       // entries per projecting thread (4)
constexpr int kProjRows = 4;                                   // W_idx rows per prefetched block
static_assert(kD % kProjRows == 0 && kProjRows % 2 == 0, "whole blocks of row pairs");

// Writes one MXFP4 row of 32*V elements held V per lane (lane: elements
// V*lane .. V*lane+V-1), blocks of 32 = 32/V lanes.
template <int V>
__device__ __forceinline__ void encode_row(const float (&x)[V], uint8_t* codes, uint8_t* scales, int lane) {
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < V; ++i) amax = fmaxf(amax, fabsf(x[i]));
#pragma unroll
  for (int o = 1; o < 32 / V; o <<= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  const int X = mx_block_exp(amax);
  const float inv = pow2f_neg(X);
  if constexpr (V == 16) {
    uint32_t lo = 0, hi = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) lo |= e2m1_code(x[i], inv) << (4 * i);
#pragma unroll
    for (int i = 0; i < 8; ++i) hi |= e2m1_code(x[8 + i], inv) << (4 * i);
    *reinterpret_cast<uint2*>(codes + 8 * lane) = make_uint2(lo, hi);
  } else {
    uint32_t v = 0;
#pragma unroll
    for (int i = 0; i < V; ++i) v |= e2m1_code(x[i], inv) << (4 * i);
    *reinterpret_cast<uint16_t*>(codes + 2 * lane) = uint16_t(v);
  }
  if ((lane % (32 / V)) == 0) scales[lane / (32 / V)] = uint8_t(X + 127);
}

// Token s of sequence b's stream: the pending token (s < pn) or raw token
// tok0 + s - pn of this call.
struct TokenSrc {
  const CompressArgs& a;
  int b, pn;
  int64_t tok0;
  __device__ const uint16_t* row(int64_t s) const {
    return s < pn ? a.pend_raw + int64_t(b) * kD : a.raw + (tok0 + s - pn) * kD;
  }
  __device__ const uint16_t* idx_row(int64_t s) const {
    return s < pn ? a.pend_idx + int64_t(b) * kDi : a.idx_raw + (tok0 + s - pn) * kDi;
  }
  __device__ double logit(int64_t s) const { return s < pn ? a.pend_logit[b] : a.logits[tok0 + s - pn]; }
};

// Pair weights w = softmax(z0, z1) in double with the own exp.
__device__ __forceinline__ void pair_weights(double z0, double z1, double& w0, double& w1) {
  const double m = fmax(z0, z1);
  const double e0 = own_exp(__dsub_rn(z0, m)), e1 = own_exp(__dsub_rn(z1, m));
  const double sum = __dadd_rn(e0, e1);
  w0 = __ddiv_rn(e0, sum);
  w1 = __ddiv_rn(e1, sum);
}

// grid = (ceil(max_new / 16), B), block = 256.  Each warp merges and encodes
// two entries' main rows; the optional W_idx projection is shared by the CTA
// (thread t: columns 2(t % 64) and 2(t % 64) + 1 of the entries
// e = 4q + t / 64, eight fma chains), and each warp then encodes its
// two indexer rows.  Streaming mode (a.pend_n != null): the sequence's token
// stream starts with its pending token, the last CTA of the sequence to
// finish keeps an odd trailing token as the new pending one and writes the
// new lengths (all CTAs have read the old ones by then).
__global__ void __launch_bounds__(kCompWarps * 32, 3) k_compress(CompressArgs a) {
  // merged rows, widened once for the projection; projected rows
  extern __shared__ __align__(16) unsigned char csm[];
  double (*cbuf)[kD] = reinterpret_cast<double (*)[kD]>(csm);
  float (*rbuf)[kDi] = reinterpret_cast<float (*)[kDi]>(csm + sizeof(double) * kCompEntries * kD);
  __shared__ int last_cta;
  launch_dependents();
  grid_wait();
  const int b = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool streaming = a.pend_n != nullptr;
  const int64_t tok0 = a.tok_off[b];
  const int64_t ntok = max(int64_t(0), a.tok_off[b + 1] - tok0);
  const int pn = streaming ? (a.pend_n[b] != 0 ? 1 : 0) : 0;
  const int64_t nstream = ntok + pn;
  const int64_t nnew_all = nstream / a.ratio;
  // entries beyond the host's bound max_new (the grid) are not written: flagged
  const int64_t nnew = min(nnew_all, a.max_new);
  const int32_t len_in = a.seq_len_in[b];
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    if (nnew_all > a.max_new) set_status(a.status, CSA2_DEV_LENGTH);
    if (!streaming) a.seq_len_out[b] = len_in + int32_t(nnew_all);
  }
  const TokenSrc src{a, b, pn, tok0};
  const int64_t j0 = int64_t(blockIdx.x) * kCompEntries;

  if (j0 < nnew) {  // uniform for the whole CTA
    const int nvalid = int(min(int64_t(kCompEntries), nnew - j0));
    // ---- phase 1: merge + encode the main rows (entries warp, warp + 8) ----
    bool ok[2];
    int64_t rows[2];
    double w0s[2], w1s[2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int e = warp + kCompWarps * u;
      const int64_t j = j0 + e;
      ok[u] = j < nnew;
      int64_t row = -1;
      if (ok[u]) {
        if (a.pages) {
          const int64_t t = int64_t(len_in) + j;
          if (len_in < 0 || t >= (int64_t(a.max_pages) << a.page_shift)) {
            if (lane == 0) set_status(a.status, CSA2_DEV_ROW_LAYOUT);
            ok[u] = false;
          } else {
            row = paged_row(a.pages + int64_t(b) * a.max_pages, a.page_shift, min(a.mrows, a.irows), t, a.status);
          }
        } else {
          row = a.seq_row_off[b] + len_in + j;
        }
      }
      if (ok[u] && (row < 0 || row >= a.mrows || row >= a.irows)) {
        if (lane == 0) set_status(a.status, CSA2_DEV_ROW_LAYOUT);
        ok[u] = false;
      }
      rows[u] = row;
      w0s[u] = 1.0;
      w1s[u] = 0.0;
      float c[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) c[i] = 0.0f;
      if (ok[u]) {
        const int64_t s0 = a.ratio * j;  // first stream token of the entry
        if (a.ratio == 2) pair_weights(src.logit(s0), src.logit(s0 + 1), w0s[u], w1s[u]);
        // lane holds elements 16*lane .. 16*lane+15
        const uint4* p0 = reinterpret_cast<const uint4*>(src.row(s0) + 16 * lane);
        const uint4 u0 = __ldg(p0), u1 = __ldg(p0 + 1);
        const uint32_t x0w[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
        if (a.ratio == 2) {
          const uint4* p1 = reinterpret_cast<const uint4*>(src.row(s0 + 1) + 16 * lane);
          const uint4 v0 = __ldg(p1), v1 = __ldg(p1 + 1);
          const uint32_t x1w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const double x0 = bf16f(uint16_t(x0w[i / 2] >> (16 * (i & 1))));
            const double x1 = bf16f(uint16_t(x1w[i / 2] >> (16 * (i & 1))));
            c[i] = __double2float_rn(__fma_rn(w0s[u], x0, __dmul_rn(w1s[u], x1)));
          }
        } else {
#pragma unroll
          for (int i = 0; i < 16; ++i) c[i] = bf16f(uint16_t(x0w[i / 2] >> (16 * (i & 1))));
        }
        encode_row<16>(c, a.mcodes + row * kMainCodeBytes, a.mscales + row * kMainScaleBytes, lane);
      }
      if (a.w_idx) {
#pragma unroll
        for (int i = 0; i < 16; ++i) cbuf[e][16 * lane + i] = double(c[i]);
      }
    }

    // ---- phase 2: indexer rows r = W_idx^T c (fp64 chain over i = 0..511) ----
    if (a.w_idx) {
      __syncthreads();
      const int col = threadIdx.x % kDi, grp = threadIdx.x / kDi;
      if (nvalid <= kCompGroups) {
        // one entry per group (a decode append): a single chain per thread;
        // W_idx is read 64 rows at a time, so the chain waits for one L2
        // round trip per 64 terms rather than per few
        if (grp < nvalid) {
          double acc = 0.0;
          for (int i0 = 0; i0 < kD; i0 += 64) {
            float wv[64];
#pragma unroll
            for (int u = 0; u < 64; ++u) wv[u] = __ldg(a.w_idx + (i0 + u) * kDi + col);
#pragma unroll
            for (int u = 0; u < 64; ++u) acc = __fma_rn(cbuf[grp][i0 + u], double(wv[u]), acc);
          }
          rbuf[grp][col] = __double2float_rn(acc);
        }
      } else {
        const int c0 = kProjCols * (threadIdx.x % (kDi / kProjCols)), pg = threadIdx.x / (kDi / kProjCols);
        double acc[kProjEntries][kProjCols];
#pragma unroll
        for (int q = 0; q < kProjEntries; ++q) acc[q][0] = acc[q][1] = 0.0;
        // W_idx rows come from L2 one block of kProjRows ahead of their use
        const float2* wp = reinterpret_cast<const float2*>(a.w_idx + c0);
        float2 wc[kProjRows], wn[kProjRows];
#pragma unroll
        for (int r = 0; r < kProjRows; ++r) wc[r] = __ldg(wp + r * (kDi / 2));
        for (int i0 = 0; i0 < kD; i0 += kProjRows) {
          const int nxt = min(i0 + kProjRows, kD - kProjRows);  // the last block reloads itself
#pragma unroll
          for (int r = 0; r < kProjRows; ++r) wn[r] = __ldg(wp + (nxt + r) * (kDi / 2));
#pragma unroll
          for (int r = 0; r < kProjRows; r += 2) {
#pragma unroll
            for (int q = 0; q < kProjEntries; ++q) {
              const double2 x = *reinterpret_cast<const double2*>(&cbuf[q * kProjGroups + pg][i0 + r]);
              acc[q][0] = __fma_rn(x.x, double(wc[r].x), acc[q][0]);
              acc[q][1] = __fma_rn(x.x, double(wc[r].y), acc[q][1]);
              acc[q][0] = __fma_rn(x.y, double(wc[r + 1].x), acc[q][0]);
              acc[q][1] = __fma_rn(x.y, double(wc[r + 1].y), acc[q][1]);
            }
          }
#pragma unroll
          for (int r = 0; r < kProjRows; ++r) wc[r] = wn[r];
        }
#pragma unroll
        for (int q = 0; q < kProjEntries; ++q) {
          rbuf[q * kProjGroups + pg][c0] = __double2float_rn(acc[q][0]);
          rbuf[q * kProjGroups + pg][c0 + 1] = __double2float_rn(acc[q][1]);
        }
      }
      __syncthreads();
    }

    // ---- phase 3: encode the indexer rows (lane holds 4*lane .. 4*lane+3) ----
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      if (!ok[u]) continue;
      const int e = warp + kCompWarps * u;
      const int64_t s0 = a.ratio * (j0 + e), row = rows[u];
      float r[4];
      if (a.w_idx) {
#pragma unroll
        for (int i = 0; i < 4; ++i) r[i] = rbuf[e][4 * lane + i];
      } else {
        const uint2 uu = __ldg(reinterpret_cast<const uint2*>(src.idx_row(s0) + 4 * lane));
        const uint32_t x0w[2] = {uu.x, uu.y};
        if (a.ratio == 2) {
          const uint2 v = __ldg(reinterpret_cast<const uint2*>(src.idx_row(s0 + 1) + 4 * lane));
          const uint32_t x1w[2] = {v.x, v.y};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const double x0 = bf16f(uint16_t(x0w[i / 2] >> (16 * (i & 1))));
            const double x1 = bf16f(uint16_t(x1w[i / 2] >> (16 * (i & 1))));
            r[i] = __double2float_rn(__fma_rn(w0s[u], x0, __dmul_rn(w1s[u], x1)));
          }
        } else {
#pragma unroll
          for (int i = 0; i < 4; ++i) r[i] = bf16f(uint16_t(x0w[i / 2] >> (16 * (i & 1))));
        }
      }
      encode_row<4>(r, a.icodes + row * kIdxCodeBytes, a.iscales + row * kIdxScaleBytes, lane);
    }
  }
  if (!streaming) return;

  // ---- streaming: the last CTA of the sequence updates the pending token ----
  // The barrier orders this CTA's reads of the pending token and of the
  // lengths before thread 0's release-acquire arrival (gpu scope).
  __syncthreads();
  if (threadIdx.x == 0) {
    unsigned old;
    asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], 1;" : "=r"(old) : "l"(a.arrive + b) : "memory");
    last_cta = old == gridDim.x - 1;
  }
  __syncthreads();
  if (!last_cta) return;
  const int64_t keep = nstream - nnew_all * a.ratio;  // 0 or 1 trailing tokens
  const int64_t s_last = nstream - 1;
  if (keep == 1 && s_last >= pn) {  // a raw token of this call becomes the pending one
    const uint32_t* from = reinterpret_cast<const uint32_t*>(src.row(s_last));
    uint32_t* to = reinterpret_cast<uint32_t*>(a.pend_raw + int64_t(b) * kD);
    for (int i = threadIdx.x; i < kD / 2; i += blockDim.x) to[i] = __ldcg(from + i);
    if (a.pend_idx) {
      const uint32_t* fi = reinterpret_cast<const uint32_t*>(src.idx_row(s_last));
      uint32_t* ti = reinterpret_cast<uint32_t*>(a.pend_idx + int64_t(b) * kDi);
      for (int i = threadIdx.x; i < kDi / 2; i += blockDim.x) ti[i] = __ldcg(fi + i);
    }
    if (threadIdx.x == 0) a.pend_logit[b] = a.logits[tok0 + s_last - pn];
  }
  if (threadIdx.x == 0) {
    a.pend_n[b] = int32_t(keep);
    if (a.seq_len_out) a.seq_len_out[b] = len_in + int32_t(nnew_all);
    a.arrive[b] = 0u;  // ready for the next call
  }
}

void launch_compress(const CompressArgs& a, cudaStream_t st) {
  if (a.B == 0) return;
  const int64_t gx = a.max_new > 0 ? (a.max_new + kCompEntries - 1) / kCompEntries : 1;
  const size_t smem = sizeof(double) * kCompEntries * kD + sizeof(float) * kCompEntries * kDi;
  cudaFuncSetAttribute(k_compress, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  launch_k(k_compress, dim3(static_cast<unsigned>(gx), a.B), dim3(kCompWarps * 32), smem, st, a);
}

}  // namespace csa2
