// Sparse attention over the selected MXFP4 main-KV rows plus the FP8 sliding
// window, one softmax per head ("DeepSeek-V4.1-Flash: Pushing the Limits of
// KV Cache Compression", section "三个方向一起压小缓存": 512 entries per layer,
// MXFP4 main KV, FP8 window; section "后 20 层干脆共用一份 KV": 128-token window).
//
// Work split: ceil(k/128) chunks of selected rows plus one window chunk per
// segment.  A CTA gathers its <= 128 key rows, dequantises them exactly into
// fp16 in shared memory (E2M1 x 2^X and raw E4M3 are exact in fp16 inside the
// range checked below), and runs both products on the tensor cores with
// warp-level mma (fp16 inputs, fp32 accumulation):
//   S = Q K^T  (16 heads x 128 keys),  P = exp(S*scale - max),  O = P V.
// The window's fp32 scale multiplies its logits and its partial output in
// fp32, never the fp16 values.  Each CTA writes an unnormalised partial
// (O, max, sum) per head; a second kernel combines the chunks in a fixed order.
#include <cuda_fp16.h>

#include "device_common.cuh"

namespace csa2 {

constexpr int kChunk = 128;
constexpr int kAttnThreads = 256;                 // 8 warps
constexpr int kPartFloats = kHq * kD + 2 * kHq;  // O, then m, then l
constexpr int kQS = kD + 8;                       // smem row stride (halves) of Q and K
constexpr int kPS = kChunk + 8;                   // smem row stride (halves) of P

int attn_num_chunks(int k) { return (k + kChunk - 1) / kChunk + 1; }
size_t attn_partial_bytes(int S, int k) {
  return size_t(S) * attn_num_chunks(k) * kPartFloats * sizeof(float);
}

struct AttnSmem {
  __half q[kHq][kQS];
  __half kv[kChunk][kQS];
  __half p[kHq][kPS];
  float red_max[8][kHq];
  float red_sum[8][kHq];
  int valid[kChunk];
};

// fp16 bit patterns of the E2M1 magnitudes {0, .5, 1, 1.5, 2, 3, 4, 6}
__device__ __forceinline__ uint32_t e2m1_half_bits(uint32_t code) {
  const uint32_t lo = 0x3E003C00u, hi = 0x46004400u;  // 1.5|1, 6|4
  const uint32_t mag = code & 7u;
  uint32_t bits;
  if (mag < 2) bits = mag ? 0x3800u : 0u;
  else if (mag < 4) bits = (mag == 2) ? (lo & 0xFFFFu) : (lo >> 16);
  else if (mag < 6) bits = (mag == 4) ? 0x4000u : 0x4200u;
  else bits = (mag == 6) ? (hi & 0xFFFFu) : (hi >> 16);
  return bits | ((code & 8u) << 12);
}

// OCP E4M3 -> fp16 bits (exact: 3 mantissa bits, exponent -9 .. 8).
__device__ __forceinline__ uint32_t e4m3_half_bits(uint32_t b) {
  const uint32_t s = (b & 0x80u) << 8, e = (b >> 3) & 15u, m = b & 7u;
  uint32_t bits;
  if (e == 0) {
    bits = m ? __half_as_ushort(__float2half_rn(float(m) * 0.001953125f)) : 0u;  // m * 2^-9, exact
  } else {
    bits = ((e + 8u) << 10) | (m << 7);  // exponent bias 7 -> 15
  }
  return bits | s;
}

__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(static_cast<uint32_t>(__cvta_generic_to_shared(p))));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t (&r)[4], const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(static_cast<uint32_t>(__cvta_generic_to_shared(p))));
}
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__global__ void __launch_bounds__(kAttnThreads) k_attn_partial(AttnArgs a) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  AttnSmem& sm = *reinterpret_cast<AttnSmem*>(smem_raw);
  const int s = blockIdx.y, c = blockIdx.x, tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, t = lane & 3;
  const int nmain = (a.k + kChunk - 1) / kChunk;
  const bool is_win = (c == nmain);
  const int64_t eff = a.seg_eff[s];
  const int64_t off = a.sd.row_off ? a.sd.row_off[s] : a.sd.row0;
  float* part = a.partial + (int64_t(s) * gridDim.x + c) * kPartFloats;

  int nkeys;
  float kscale = 1.0f;
  const uint8_t* win_base = nullptr;
  if (!is_win) {
    nkeys = min(kChunk, a.k - c * kChunk);
  } else if (a.q_pos == nullptr) {
    nkeys = max(0, min(kWin, a.win_len[s]));
    kscale = a.win_scale[s];
    win_base = a.win + int64_t(s) * kWin * kD;
  } else {
    int64_t p = a.q_pos[s];
    if (p >= a.n_raw) {
      set_status(a.status, CSA2_DEV_LENGTH);
      p = a.n_raw - 1;
    }
    const int64_t lo = p - (kWin - 1) > 0 ? p - (kWin - 1) : 0;
    nkeys = p >= 0 ? int(p - lo + 1) : 0;
    kscale = a.raw_scale;
    win_base = a.raw_win + lo * kD;
  }
  if (nkeys == 0) {
    for (int i = tid; i < kHq * kD; i += kAttnThreads) part[i] = 0.0f;
    if (tid < kHq) {
      part[kHq * kD + tid] = -INFINITY;
      part[kHq * kD + kHq + tid] = 0.0f;
    }
    return;
  }

  // Q: bf16 -> fp16 (exact for |q| in [2^-14, 65504]; smaller values keep 2^-24 resolution)
  for (int i = tid; i < kHq * kD / 2; i += kAttnThreads) {
    const uint32_t w2 = reinterpret_cast<const uint32_t*>(a.q + int64_t(s) * kHq * kD)[i];
    const float lo = __uint_as_float(w2 << 16), hi = __uint_as_float(w2 & 0xFFFF0000u);
    if (fabsf(lo) > 65504.0f || fabsf(hi) > 65504.0f) set_status(a.status, CSA2_DEV_FP16_RANGE);
    const int h = (2 * i) / kD, d = (2 * i) % kD;
    *reinterpret_cast<__half2*>(&sm.q[h][d]) = __floats2half2_rn(lo, hi);
  }
  // keys: thread -> one row r (lanes on consecutive rows, which keeps the
  // shared-memory stores conflict-free) and 8 of its 16 blocks
  const int r = tid & (kChunk - 1);
  int64_t tpos = -1;
  if (!is_win && r < nkeys) {
    tpos = a.topk[int64_t(s) * a.k + c * kChunk + r];
    if (tpos >= eff) {
      if (tid < kChunk) set_status(a.status, CSA2_DEV_INDEX_RANGE);
      tpos = -1;
    }
  }
  const bool row_ok = (r < nkeys) && (is_win || tpos >= 0);
  if (tid < kChunk) sm.valid[r] = row_ok;
  for (int b = tid >> 7; b < 16; b += kAttnThreads / kChunk) {
    const bool ok = row_ok;
    uint4 out[4];
    if (!is_win) {
      if (ok) {
        const int64_t row = off + tpos;
        const uint4 cw = __ldg(reinterpret_cast<const uint4*>(a.mcodes + row * kMainCodeBytes) + b);
        const uint32_t sb = a.mscales[row * kMainScaleBytes + b];
        // fp16-exact iff the block exponent X = sb - 127 lies in [-23, 13]
        if (sb < 104u || sb > 140u) set_status(a.status, CSA2_DEV_FP16_RANGE);
        const int X = int(sb) - 127;
        const __half2 sc2 = __half2half2(__ushort_as_half(
            X >= -14 ? uint16_t((X + 15) << 10) : uint16_t(1u << (X + 24 > 0 ? X + 24 : 0))));
        const uint32_t w4[4] = {cw.x, cw.y, cw.z, cw.w};
        uint32_t hv[16];
#pragma unroll
        for (int q = 0; q < 4; ++q)
#pragma unroll
          for (int n = 0; n < 4; ++n) {
            const uint32_t c0 = (w4[q] >> (8 * n)) & 15u, c1 = (w4[q] >> (8 * n + 4)) & 15u;
            const uint32_t pair = e2m1_half_bits(c0) | (e2m1_half_bits(c1) << 16);
            const __half2 v = __hmul2(*reinterpret_cast<const __half2*>(&pair), sc2);
            hv[4 * q + n] = *reinterpret_cast<const uint32_t*>(&v);
          }
#pragma unroll
        for (int q = 0; q < 4; ++q) out[q] = make_uint4(hv[4 * q], hv[4 * q + 1], hv[4 * q + 2], hv[4 * q + 3]);
      }
    } else if (ok) {
      const uint4* src = reinterpret_cast<const uint4*>(win_base + int64_t(r) * kD + 32 * b);
      const uint4 v0 = __ldg(src), v1 = __ldg(src + 1);
      const uint32_t w8[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
      uint32_t hv[16];
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        hv[2 * q] = e4m3_half_bits(w8[q] & 255u) | (e4m3_half_bits((w8[q] >> 8) & 255u) << 16);
        hv[2 * q + 1] = e4m3_half_bits((w8[q] >> 16) & 255u) | (e4m3_half_bits(w8[q] >> 24) << 16);
      }
#pragma unroll
      for (int q = 0; q < 4; ++q) out[q] = make_uint4(hv[4 * q], hv[4 * q + 1], hv[4 * q + 2], hv[4 * q + 3]);
    }
    if (!ok)
#pragma unroll
      for (int q = 0; q < 4; ++q) out[q] = make_uint4(0, 0, 0, 0);
    uint4* dst = reinterpret_cast<uint4*>(&sm.kv[r][32 * b]);
#pragma unroll
    for (int q = 0; q < 4; ++q) dst[q] = out[q];
  }
  __syncthreads();

  // ---- S = Q K^T: warp w owns keys 16w .. 16w+15 (two n-tiles of 8) ----
  float sacc[2][4] = {{0, 0, 0, 0}, {0, 0, 0, 0}};
  {
    const int kr = 16 * warp + (lane & 7) + 8 * (lane >> 4);  // key row for the B matrices
    const int kc = 8 * ((lane >> 3) & 1);
    const int qr = (lane & 7) + 8 * ((lane >> 3) & 1);        // head row for the A matrices
    const int qc = 8 * (lane >> 4);
#pragma unroll 4
    for (int k0 = 0; k0 < kD; k0 += 16) {
      uint32_t af[4], bf[4];
      ldsm_x4(af, &sm.q[qr][k0 + qc]);
      ldsm_x4(bf, &sm.kv[kr][k0 + kc]);
      mma16816(sacc[0], af, bf[0], bf[1]);
      mma16816(sacc[1], af, bf[2], bf[3]);
    }
  }
  // ---- softmax over the chunk's keys (per head) ----
  const float lscale = a.sm_scale * kscale;
  float mx[2] = {-INFINITY, -INFINITY};  // heads g, g+8
#pragma unroll
  for (int nt = 0; nt < 2; ++nt)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int key = 16 * warp + 8 * nt + 2 * t + (j & 1);
      const float v = sm.valid[key] ? sacc[nt][j] * lscale : -INFINITY;
      sacc[nt][j] = v;
      mx[j >> 1] = fmaxf(mx[j >> 1], v);
    }
#pragma unroll
  for (int hh = 0; hh < 2; ++hh) {
    mx[hh] = fmaxf(mx[hh], __shfl_xor_sync(0xffffffffu, mx[hh], 1));
    mx[hh] = fmaxf(mx[hh], __shfl_xor_sync(0xffffffffu, mx[hh], 2));
  }
  if (t == 0) {
    sm.red_max[warp][g] = mx[0];
    sm.red_max[warp][g + 8] = mx[1];
  }
  __syncthreads();
  float m[2], sum[2] = {0.0f, 0.0f};
#pragma unroll
  for (int hh = 0; hh < 2; ++hh) {
    float v = -INFINITY;
#pragma unroll
    for (int w = 0; w < 8; ++w) v = fmaxf(v, sm.red_max[w][g + 8 * hh]);
    m[hh] = v;
  }
#pragma unroll
  for (int nt = 0; nt < 2; ++nt)
#pragma unroll
    for (int j = 0; j < 4; j += 2) {
      const int hh = j >> 1;
      const float p0 = (m[hh] == -INFINITY) ? 0.0f : __expf(sacc[nt][j] - m[hh]);
      const float p1 = (m[hh] == -INFINITY) ? 0.0f : __expf(sacc[nt][j + 1] - m[hh]);
      const __half2 ph = __floats2half2_rn(p0, p1);
      const float2 pr = __half22float2(ph);  // the sum uses the rounded fp16 weights
      sum[hh] += pr.x + pr.y;
      *reinterpret_cast<__half2*>(&sm.p[g + 8 * hh][16 * warp + 8 * nt + 2 * t]) = ph;
    }
#pragma unroll
  for (int hh = 0; hh < 2; ++hh) {
    sum[hh] += __shfl_xor_sync(0xffffffffu, sum[hh], 1);
    sum[hh] += __shfl_xor_sync(0xffffffffu, sum[hh], 2);
  }
  if (t == 0) {
    sm.red_sum[warp][g] = sum[0];
    sm.red_sum[warp][g + 8] = sum[1];
  }
  __syncthreads();

  // ---- O = P V: warp w owns dims 64w .. 64w+63 (eight n-tiles of 8) ----
  float oacc[8][4];
#pragma unroll
  for (int nt = 0; nt < 8; ++nt)
#pragma unroll
    for (int j = 0; j < 4; ++j) oacc[nt][j] = 0.0f;
  {
    const int pr_ = (lane & 7) + 8 * ((lane >> 3) & 1);
    const int pc = 8 * (lane >> 4);
    const int vr = (lane & 7) + 8 * ((lane >> 3) & 1);  // key row within the k-step
    const int vc = 8 * (lane >> 4);                     // dim offset within the n-tile pair
    const int kend = (nkeys + 15) & ~15;
    for (int k0 = 0; k0 < kend; k0 += 16) {
      uint32_t af[4];
      ldsm_x4(af, &sm.p[pr_][k0 + pc]);
#pragma unroll
      for (int np = 0; np < 4; ++np) {
        uint32_t bf[4];
        ldsm_x4_t(bf, &sm.kv[k0 + vr][64 * warp + 16 * np + vc]);
        mma16816(oacc[2 * np], af, bf[0], bf[1]);
        mma16816(oacc[2 * np + 1], af, bf[2], bf[3]);
      }
    }
  }
  // ---- partial out (window values carry their fp32 scale) ----
#pragma unroll
  for (int nt = 0; nt < 8; ++nt) {
    const int d = 64 * warp + 8 * nt + 2 * t;
    *reinterpret_cast<float2*>(&part[g * kD + d]) = make_float2(oacc[nt][0] * kscale, oacc[nt][1] * kscale);
    *reinterpret_cast<float2*>(&part[(g + 8) * kD + d]) = make_float2(oacc[nt][2] * kscale, oacc[nt][3] * kscale);
  }
  if (tid < kHq) {
    float l = 0.0f;
#pragma unroll
    for (int w = 0; w < 8; ++w) l += sm.red_sum[w][tid];
    float mm = -INFINITY;
#pragma unroll
    for (int w = 0; w < 8; ++w) mm = fmaxf(mm, sm.red_max[w][tid]);
    part[kHq * kD + tid] = mm;
    part[kHq * kD + kHq + tid] = l;
  }
}

// Combine the chunk partials of one segment in chunk order.  grid = S,
// block = 512 (thread = output dim); per-head factors computed once in smem.
__global__ void __launch_bounds__(512) k_attn_combine(AttnArgs a, int nchunks) {
  constexpr int kMaxChunks = CSA2_MAX_TOPK / kChunk + 1;
  __shared__ float fac[kMaxChunks][kHq];  // exp(m_c - M) / L per chunk and head
  __shared__ float lse_s[kHq];
  const int s = blockIdx.x, d = threadIdx.x;
  const float* base = a.partial + int64_t(s) * nchunks * kPartFloats;
  if (d < kHq) {
    float M = -INFINITY;
    for (int c = 0; c < nchunks; ++c) M = fmaxf(M, base[c * kPartFloats + kHq * kD + d]);
    float L = 0.0f;
    for (int c = 0; c < nchunks; ++c) {
      const float mc = base[c * kPartFloats + kHq * kD + d];
      const float f = (mc == -INFINITY) ? 0.0f : __expf(mc - M);
      fac[c][d] = f;
      L += base[c * kPartFloats + kHq * kD + kHq + d] * f;
    }
    for (int c = 0; c < nchunks; ++c) fac[c][d] = (M == -INFINITY) ? 0.0f : fac[c][d] / L;
    lse_s[d] = (M == -INFINITY) ? -INFINITY : M + logf(L);
  }
  __syncthreads();
#pragma unroll 4
  for (int h = 0; h < kHq; ++h) {
    float o = 0.0f;
    for (int c = 0; c < nchunks; ++c) o = fmaf(base[c * kPartFloats + h * kD + d], fac[c][h], o);
    a.out[(int64_t(s) * kHq + h) * kD + d] = o;
  }
  if (a.lse && d < kHq) a.lse[int64_t(s) * kHq + d] = lse_s[d];
}

void launch_attention(const AttnArgs& a, cudaStream_t st) {
  if (a.S == 0) return;
  const int nchunks = attn_num_chunks(a.k);
  const size_t smem = sizeof(AttnSmem);
  cudaFuncSetAttribute(k_attn_partial, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  k_attn_partial<<<dim3(nchunks, a.S), kAttnThreads, smem, st>>>(a);
  k_attn_combine<<<a.S, 512, 0, st>>>(a, nchunks);
}

}  // namespace csa2
