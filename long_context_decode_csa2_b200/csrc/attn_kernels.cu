// Sparse attention over the selected MXFP4 main-KV rows plus the FP8 sliding
// window, one softmax per head ("DeepSeek-V4.1-Flash: Pushing the Limits of
// KV Cache Compression", section "三个方向一起压小缓存": 512 entries per layer,
// MXFP4 main KV, FP8 window; section "后 20 层干脆共用一份 KV": 128-token window).
//
// Split over chunks of 128 keys (ceil(k/128) main chunks + 1 window chunk):
// each CTA writes an unnormalised partial (m, l, O) per head; a second kernel
// combines the chunks in a fixed order (deterministic).
#include "device_common.cuh"

namespace csa2 {

constexpr int kChunk = 128;
constexpr int kSub = 32;
constexpr int kAttnThreads = 512;
constexpr int kPartFloats = kHq * kD + 2 * kHq;  // O, then m, then l

int attn_num_chunks(int k) { return (k + kChunk - 1) / kChunk + 1; }
size_t attn_partial_bytes(int S, int k) {
  return size_t(S) * attn_num_chunks(k) * kPartFloats * sizeof(float);
}

__device__ __forceinline__ float e2m1_val(uint32_t code) {
  const float mag = 0.5f * float((0xC8643210u >> (4 * (code & 7))) & 15u);
  return (code & 8) ? -mag : mag;
}

// 2^(byte-127); byte 0 is the subnormal 2^-127 (byte 255 is never stored).
__device__ __forceinline__ float e8m0_val(uint32_t byte) {
  return byte ? __uint_as_float(byte << 23) : __uint_as_float(0x00400000u);
}

__device__ __forceinline__ float e4m3_val(uint32_t b) {
  const uint32_t e = (b >> 3) & 15u, m = b & 7u;
  float v = (e == 0) ? float(m) * 0.001953125f /* m/8 * 2^-6 */
                     : __uint_as_float(((e + 120u) << 23) | (m << 20));
  return (b & 128u) ? -v : v;
}

struct AttnSmem {
  float qf[kHq][kD];
  float kf[kSub][kD + 1];
  float p[kHq][kSub];
  float corr[kHq];
  float m[kHq];
  float l[kHq];
  int valid[kSub];
};

__global__ void __launch_bounds__(kAttnThreads) k_attn_partial(AttnArgs a) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  AttnSmem& sm = *reinterpret_cast<AttnSmem*>(smem_raw);
  const int s = blockIdx.y, c = blockIdx.x, tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5;
  const int nmain = (a.k + kChunk - 1) / kChunk;
  const bool is_win = (c == nmain);
  const int64_t eff = a.seg_eff[s];
  const int64_t off = a.sd.row_off ? a.sd.row_off[s] : a.sd.row0;

  // key list of this chunk
  int nkeys;
  int64_t win_lo = 0;
  float kscale = 1.0f;
  const uint8_t* win_base = nullptr;
  if (!is_win) {
    nkeys = min(kChunk, a.k - c * kChunk);
  } else if (a.q_pos == nullptr) {
    int wl = a.win_len[s];
    nkeys = max(0, min(kWin, wl));
    kscale = a.win_scale[s];
    win_base = a.win + int64_t(s) * kWin * kD;
  } else {
    int64_t p = a.q_pos[s];
    if (p >= a.n_raw) {
      set_status(a.status, CSA2_DEV_LENGTH);
      p = a.n_raw - 1;
    }
    win_lo = p - (kWin - 1) > 0 ? p - (kWin - 1) : 0;
    nkeys = p >= 0 ? int(p - win_lo + 1) : 0;
    kscale = a.raw_scale;
    win_base = a.raw_win + win_lo * kD;
  }

  for (int i = tid; i < kHq * kD; i += kAttnThreads) {
    const uint32_t bits = uint32_t(a.q[int64_t(s) * kHq * kD + i]) << 16;
    sm.qf[i / kD][i % kD] = __uint_as_float(bits);
  }
  if (tid < kHq) {
    sm.m[tid] = -INFINITY;
    sm.l[tid] = 0.0f;
  }
  float acc[kHq];
#pragma unroll
  for (int h = 0; h < kHq; ++h) acc[h] = 0.0f;
  __syncthreads();

  const float lscale = a.sm_scale * kscale;
  for (int j0 = 0; j0 < nkeys; j0 += kSub) {
    // dequantise 32 keys: thread -> (row r = lane, 32-element block b = warp)
    {
      const int r = lane, b = warp;
      const int j = j0 + r;
      bool ok = j < nkeys;
      if (!is_win) {
        int64_t t = ok ? a.topk[int64_t(s) * a.k + c * kChunk + j] : -1;
        if (t >= eff) {
          if (b == 0) set_status(a.status, CSA2_DEV_INDEX_RANGE);
          t = -1;
        }
        ok = ok && t >= 0;
        if (ok) {
          const int64_t row = off + t;
          const uint4 cw = __ldg(reinterpret_cast<const uint4*>(a.mcodes + row * kMainCodeBytes) + b);
          const float sc = e8m0_val(a.mscales[row * kMainScaleBytes + b]);
          const uint32_t w4[4] = {cw.x, cw.y, cw.z, cw.w};
#pragma unroll
          for (int q = 0; q < 4; ++q)
#pragma unroll
            for (int n = 0; n < 8; ++n) sm.kf[r][32 * b + 8 * q + n] = e2m1_val((w4[q] >> (4 * n)) & 15u) * sc;
        }
      } else if (ok) {
        const uint4* src = reinterpret_cast<const uint4*>(win_base + int64_t(j) * kD + 32 * b);
        const uint4 v0 = __ldg(src), v1 = __ldg(src + 1);
        const uint32_t w8[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
#pragma unroll
        for (int q = 0; q < 8; ++q)
#pragma unroll
          for (int n = 0; n < 4; ++n) sm.kf[r][32 * b + 4 * q + n] = e4m3_val((w8[q] >> (8 * n)) & 255u);
      }
      if (!ok)
        for (int n = 0; n < 32; ++n) sm.kf[r][32 * b + n] = 0.0f;
      if (b == 0) sm.valid[r] = ok;
    }
    __syncthreads();
    // logits: warp = head, lane = key
    {
      const int h = warp, j = lane;
      float dot = 0.0f;
#pragma unroll 8
      for (int d = 0; d < kD; ++d) dot = fmaf(sm.qf[h][d], sm.kf[j][d], dot);
      const float lg = sm.valid[j] ? dot * lscale : -INFINITY;
      float mx = lg;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      const float mold = sm.m[h];
      const float mnew = fmaxf(mold, mx);
      const float pj = (mnew == -INFINITY || !sm.valid[j]) ? 0.0f : expf(lg - mnew);
      float ps = pj;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, o);
      __syncwarp();
      if (lane == 0) {
        const float corr = (mold == -INFINITY) ? 0.0f : expf(mold - mnew);
        sm.corr[h] = corr;
        sm.l[h] = sm.l[h] * corr + ps;
        sm.m[h] = mnew;
      }
      sm.p[h][j] = pj * kscale;  // values carry the FP8 scale in fp32
    }
    __syncthreads();
    {
      const int d = tid;
#pragma unroll
      for (int h = 0; h < kHq; ++h) {
        float v = acc[h] * sm.corr[h];
#pragma unroll 8
        for (int j = 0; j < kSub; ++j) v = fmaf(sm.p[h][j], sm.kf[j][d], v);
        acc[h] = v;
      }
    }
    __syncthreads();
  }
  float* part = a.partial + (int64_t(s) * gridDim.x + c) * kPartFloats;
#pragma unroll
  for (int h = 0; h < kHq; ++h) part[h * kD + tid] = acc[h];
  if (tid < kHq) {
    part[kHq * kD + tid] = sm.m[tid];
    part[kHq * kD + kHq + tid] = sm.l[tid];
  }
}

__global__ void __launch_bounds__(kAttnThreads) k_attn_combine(AttnArgs a, int nchunks) {
  const int s = blockIdx.x, d = threadIdx.x;
  const float* base = a.partial + int64_t(s) * nchunks * kPartFloats;
  for (int h = 0; h < kHq; ++h) {
    float M = -INFINITY;
    for (int c = 0; c < nchunks; ++c) M = fmaxf(M, base[c * kPartFloats + kHq * kD + h]);
    float o = 0.0f, L = 0.0f;
    if (M != -INFINITY) {
      for (int c = 0; c < nchunks; ++c) {
        const float mc = base[c * kPartFloats + kHq * kD + h];
        if (mc == -INFINITY) continue;
        const float f = expf(mc - M);
        L += base[c * kPartFloats + kHq * kD + kHq + h] * f;
        o += base[c * kPartFloats + h * kD + d] * f;
      }
      o = o / L;
    }
    a.out[(int64_t(s) * kHq + h) * kD + d] = o;
    if (a.lse && d == 0) a.lse[int64_t(s) * kHq + h] = (M == -INFINITY) ? -INFINITY : M + logf(L);
  }
}

void launch_attention(const AttnArgs& a, cudaStream_t st) {
  if (a.S == 0) return;
  const int nchunks = attn_num_chunks(a.k);
  const size_t smem = sizeof(AttnSmem);
  cudaFuncSetAttribute(k_attn_partial, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  k_attn_partial<<<dim3(nchunks, a.S), kAttnThreads, smem, st>>>(a);
  k_attn_combine<<<a.S, kAttnThreads, 0, st>>>(a, nchunks);
}

}  // namespace csa2
