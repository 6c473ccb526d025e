// Pieces of a context-parallel decode step, where each of G shards (GPUs)
// holds a contiguous range of every long sequence's entries: the exact rank
// keys of listed positions or blocks (so that shards can compare their local
// winners), the exact merge of the shards' candidate lists, and the merge of
// the shards' attention partials.
//
// "DeepSeek-V4.1-Flash: Pushing the Limits of KV Cache Compression", section
// "三个方向一起压小缓存": the pool and every Top-512 are best-first selections
// by score, so the global winners are among the union of each shard's own
// winners under the same order (score desc, position asc); attention over
// the union of disjoint key sets is the lse-weighted mix of the per-set
// softmaxes.
#include "device_common.cuh"

namespace csa2 {

namespace {

// Doubled E2M1 value of a 4-bit code: magnitudes {0,1,2,3,4,6,8,12}, sign in bit 3.
__device__ __forceinline__ int dbl_e2m1(uint32_t nib) {
  const int m = int((0xC8643210u >> (4u * (nib & 7u))) & 15u);
  return (nib & 8u) ? -m : m;
}

// grid (ceil(n * blk / 256), B), block 256.  Thread = (listed id i, offset o
// < blk): the exact score of position id*blk + o from the 68-byte key row,
// reduced to the key of the id (block maximum for blk = 8).  The block dots
// are integer dp4a over doubled E2M1 values (|value| <= 12 fits int8).
__global__ void __launch_bounds__(256) k_score_positions(const uint8_t* kcodes, const uint8_t* kscales, SegDesc sd,
                                                         const uint8_t* q_codes, const uint8_t* q_scales,
                                                         const float* w, const int32_t* ids, int n, int blk,
                                                         uint32_t* keys_out, uint32_t* status) {
  __shared__ uint32_t qw[kHi][kDi / 4];  // query: int8x4 of elements 4i .. 4i+3 per head
  __shared__ uint16_t lut[256];          // code byte -> two int8 doubled values (low nibble first)
  __shared__ IdxQCtx qc;
  launch_dependents();
  grid_wait();
  const int b = blockIdx.y;
  {
    const int t = threadIdx.x;  // 256 threads: one LUT entry each
    const uint32_t lo = uint32_t(dbl_e2m1(t & 15u)) & 255u, hi = uint32_t(dbl_e2m1(uint32_t(t) >> 4)) & 255u;
    lut[t] = uint16_t(lo | (hi << 8));
  }
  __syncthreads();
  if (threadIdx.x < kHi * kDi / 4) {  // 128 words: two query code bytes each
    const int h = threadIdx.x / (kDi / 4), i = threadIdx.x % (kDi / 4);
    const uint8_t* qc8 = q_codes + int64_t(b) * kHi * 64 + h * 64 + 2 * i;
    qw[h][i] = uint32_t(lut[qc8[0]]) | (uint32_t(lut[qc8[1]]) << 16);
  }
  if (threadIdx.x == 0) make_qctx(qc, q_scales + int64_t(b) * kHi * 4, w + int64_t(b) * kHi);
  __syncthreads();
  const int64_t L = seg_len_checked(sd, b, status);
  const int64_t g = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t i = g / blk;
  const int o = int(g % blk);
  uint32_t key = 0;
  if (i < n) {
    const int32_t id = ids[int64_t(b) * n + i];
    const int64_t t = int64_t(id) * blk + o;
    if (id >= 0 && int64_t(id) * blk >= L && o == 0) set_status(status, CSA2_DEV_INDEX_RANGE);
    if (id >= 0 && t < L) {
      const int64_t row = seg_row(sd, b, t, status);
      const uint4* kr = reinterpret_cast<const uint4*>(kcodes + row * kIdxCodeBytes);
      int D[kHi][4];
#pragma unroll
      for (int h = 0; h < kHi; ++h)
#pragma unroll
        for (int bb = 0; bb < 4; ++bb) D[h][bb] = 0;
#pragma unroll
      for (int bb = 0; bb < 4; ++bb) {  // block bb: 16 bytes = 32 codes
        const uint4 c = __ldg(kr + bb);
        const uint32_t words[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
        for (int wd = 0; wd < 4; ++wd) {  // bytes 4wd .. 4wd+3 = elements 8wd .. 8wd+7 of the block
          const uint32_t x = words[wd];
          const int k0 = int(uint32_t(lut[x & 255u]) | (uint32_t(lut[(x >> 8) & 255u]) << 16));
          const int k1 = int(uint32_t(lut[(x >> 16) & 255u]) | (uint32_t(lut[x >> 24]) << 16));
          const int qi = 8 * bb + 2 * wd;  // word index of element 32bb + 8wd
#pragma unroll
          for (int h = 0; h < kHi; ++h) {
            D[h][bb] = __dp4a(k0, int(qw[h][qi]), D[h][bb]);
            D[h][bb] = __dp4a(k1, int(qw[h][qi + 1]), D[h][bb]);
          }
        }
      }
      // the tensor-core accumulator of a block is D / 4, exact in fp32
      uint32_t v[16];
#pragma unroll
      for (int h = 0; h < kHi; ++h)
#pragma unroll
        for (int bb = 0; bb < 4; ++bb) v[4 * h + bb] = __float_as_uint(float(D[h][bb]) * 0.25f);
      const uint32_t sw = __ldg(reinterpret_cast<const uint32_t*>(kscales) + row);
      key = rank_key(exact_score(v, sw, qc));
    }
  }
  if (blk == kBlk) key = group8_max(key);
  if (i < n && o == 0) keys_out[int64_t(b) * n + i] = key;
}

// keys / ids [G][B][n] (ids local to their shard, -1 = none) -> [B][G*n]
// with ids made global by the shard's offset src_off[g][b] (or as given).
__global__ void k_merge_gather(const uint32_t* keys, const int32_t* ids, const int64_t* src_off, int G, int B, int n,
                               uint32_t* keys_t, int32_t* ids_t, uint32_t* status) {
  launch_dependents();
  grid_wait();
  const int b = blockIdx.y;
  const int64_t c = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;  // candidate g * n + i of segment b
  if (c >= int64_t(G) * n) return;
  const int g = int(c / n), i = int(c % n);
  const int64_t src = (int64_t(g) * B + b) * n + i;
  const int32_t id = ids[src];
  int64_t gid = -1;
  if (id >= 0) {
    gid = int64_t(id) + (src_off ? src_off[int64_t(g) * B + b] : 0);
    if (gid > INT32_MAX) {
      set_status(status, CSA2_DEV_INDEX_RANGE);
      gid = -1;
    }
  }
  ids_t[int64_t(b) * G * n + c] = int32_t(gid);
  keys_t[int64_t(b) * G * n + c] = gid >= 0 ? keys[src] : 0u;
}

// out_local[b][j] = out[b][j] - lo[b] where lo[b] <= out[b][j] < hi[b], else -1.
__global__ void k_localize(const int32_t* out, int B, int k, const int64_t* lo, const int64_t* hi,
                           int32_t* out_local) {
  launch_dependents();
  grid_wait();
  const int b = blockIdx.y;
  const int j = blockIdx.x * blockDim.x + threadIdx.x;
  if (j >= k) return;
  const int32_t id = out[int64_t(b) * k + j];
  out_local[int64_t(b) * k + j] = (id >= 0 && id >= lo[b] && id < hi[b]) ? int32_t(id - lo[b]) : -1;
}

// grid B, block 512 (warp h = head h; lane = 16 of the 512 dimensions).
// out = sum_g exp(lse_g - M) out_g / sum_g exp(lse_g - M), lse = M + log(sum).
__global__ void __launch_bounds__(512) k_attn_combine(const float* out_parts, const float* lse_parts, int G, int B,
                                                      float* out, float* lse) {
  launch_dependents();
  grid_wait();
  const int b = blockIdx.x, h = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float M = -INFINITY;
  for (int g = 0; g < G; ++g) M = fmaxf(M, lse_parts[(int64_t(g) * B + b) * kHq + h]);
  float4 acc[4];
#pragma unroll
  for (int m = 0; m < 4; ++m) acc[m] = make_float4(0.f, 0.f, 0.f, 0.f);
  float sum = 0.0f;
  if (M != -INFINITY) {
    for (int g = 0; g < G; ++g) {
      const float l = lse_parts[(int64_t(g) * B + b) * kHq + h];
      if (l == -INFINITY) continue;
      const float f = __expf(l - M);
      sum += f;
      const float4* src = reinterpret_cast<const float4*>(out_parts + ((int64_t(g) * B + b) * kHq + h) * kD);
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const float4 x = src[lane + 32 * m];
        acc[m].x += f * x.x, acc[m].y += f * x.y, acc[m].z += f * x.z, acc[m].w += f * x.w;
      }
    }
  }
  const float inv = sum > 0.0f ? 1.0f / sum : 0.0f;
  float4* dst = reinterpret_cast<float4*>(out + (int64_t(b) * kHq + h) * kD);
#pragma unroll
  for (int m = 0; m < 4; ++m)
    dst[lane + 32 * m] = make_float4(acc[m].x * inv, acc[m].y * inv, acc[m].z * inv, acc[m].w * inv);
  if (lse && lane == 0) lse[int64_t(b) * kHq + h] = (M == -INFINITY) ? -INFINITY : M + logf(sum);
}

}  // namespace

void launch_score_positions(const uint8_t* kcodes, const uint8_t* kscales, const SegDesc& sd, const uint8_t* q_codes,
                            const uint8_t* q_scales, const float* w, const int32_t* ids, int B, int n, int blk,
                            uint32_t* keys_out, uint32_t* status, cudaStream_t st) {
  if (B == 0 || n == 0) return;
  const int64_t threads = int64_t(n) * blk;
  launch_k(k_score_positions, dim3(unsigned((threads + 255) / 256), B), dim3(256), 0, st, kcodes, kscales, sd, q_codes,
           q_scales, w, ids, n, blk, keys_out, status);
}

void launch_merge_gather(const uint32_t* keys, const int32_t* ids, const int64_t* src_off, int G, int B, int n,
                         uint32_t* keys_t, int32_t* ids_t, uint32_t* status, cudaStream_t st) {
  const int64_t c = int64_t(G) * n;
  if (B == 0 || c == 0) return;
  launch_k(k_merge_gather, dim3(unsigned((c + 255) / 256), B), dim3(256), 0, st, keys, ids, src_off, G, B, n, keys_t,
           ids_t, status);
}

void launch_localize(const int32_t* out, int B, int k, const int64_t* lo, const int64_t* hi, int32_t* out_local,
                     cudaStream_t st) {
  if (B == 0 || k == 0) return;
  launch_k(k_localize, dim3(unsigned((k + 255) / 256), B), dim3(256), 0, st, out, B, k, lo, hi, out_local);
}

void launch_attn_combine(const float* out_parts, const float* lse_parts, int G, int B, float* out, float* lse,
                         cudaStream_t st) {
  if (B == 0) return;
  launch_k(k_attn_combine, dim3(B), dim3(512), 0, st, out_parts, lse_parts, G, B, out, lse);
}

}  // namespace csa2
