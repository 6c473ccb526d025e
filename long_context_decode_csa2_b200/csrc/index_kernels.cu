// Indexer kernels: segment checks, full-context scan with fused block max,
// pool-candidate scoring, causal prefill scan, and deterministic radix
// selection (Top-k by key desc / index asc, output ascending).
//
// Score definition and selection rule: "DeepSeek-V4.1-Flash: Pushing the
// Limits of KV Cache Compression", section "三个方向一起压小缓存" (hierarchical
// sparse indexer, 8-position blocks ranked by their maximum, pool of at most
// 2048 blocks, Top-512 per layer, FP4 indexer q/k).
#include "device_common.cuh"

namespace csa2 {

// ---------------------------------------------------------------------------
// Segment checks: effective visible length (0 for a bad layout).
// ---------------------------------------------------------------------------
__global__ void k_seg_check(SegDesc sd, int S, int32_t* seg_eff, uint32_t* status) {
  const int s = blockIdx.x * blockDim.x + threadIdx.x;
  if (s >= S) return;
  int64_t L = sd.len[s];
  const int64_t off = sd.row_off ? sd.row_off[s] : sd.row0;
  if (L < 0) L = 0;
  if (L > sd.max_len) {
    set_status(status, CSA2_DEV_LENGTH);
    L = sd.max_len;
  }
  if ((off & 7) != 0 || off < 0 || off + L > sd.cache_rows) {
    set_status(status, CSA2_DEV_ROW_LAYOUT);
    L = 0;
  }
  seg_eff[s] = static_cast<int32_t>(L);
}

void launch_seg_check(const SegDesc& sd, int S, int32_t* seg_eff, uint32_t* status, cudaStream_t st) {
  k_seg_check<<<(S + 255) / 256, 256, 0, st>>>(sd, S, seg_eff, status);
}

// ---------------------------------------------------------------------------
// Full-context scan (CUDA cores): one thread per position, block max fused.
// grid = (ceil(max_len/256), S), block = 256.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) k_scan(const uint8_t* __restrict__ kcodes, const uint8_t* __restrict__ kscales,
                                              SegDesc sd, const int32_t* __restrict__ seg_eff,
                                              const uint8_t* __restrict__ q_codes, const uint8_t* __restrict__ q_scales,
                                              const float* __restrict__ w, uint32_t* __restrict__ bkeys,
                                              int64_t nb_stride, float* __restrict__ scores, int64_t score_stride) {
  __shared__ IdxQueryPrep q;
  const int s = blockIdx.y;
  const int64_t L = seg_eff[s];
  const int64_t t0 = int64_t(blockIdx.x) * 256;
  if (t0 >= L) return;
  prep_query(q, q_codes + int64_t(s) * kHi * 64, q_scales + int64_t(s) * kHi * 4, w + int64_t(s) * kHi,
             threadIdx.x, 256);
  __syncthreads();
  const int64_t t = t0 + threadIdx.x;
  const int64_t off = sd.row_off ? sd.row_off[s] : sd.row0;
  uint32_t key = 0;
  if (t < L) {
    const float sc = score_row(q, kcodes, kscales, off + t);
    key = rank_key(sc);
    if (scores) scores[int64_t(s) * score_stride + t] = sc;
  }
  key = group8_max(key);
  if ((threadIdx.x & 7) == 0 && t < L) bkeys[int64_t(s) * nb_stride + t / kBlk] = key;
}

void launch_scan(const uint8_t* kcodes, const uint8_t* kscales, const SegDesc& sd, const int32_t* seg_eff, int S,
                 const uint8_t* q_codes, const uint8_t* q_scales, const float* w, uint32_t* bkeys, int64_t nb_stride,
                 float* scores, int64_t score_stride, cudaStream_t st) {
  if (S == 0 || sd.max_len == 0) return;
  dim3 grid(static_cast<unsigned>((sd.max_len + 255) / 256), S);
  k_scan<<<grid, 256, 0, st>>>(kcodes, kscales, sd, seg_eff, q_codes, q_scales, w, bkeys, nb_stride, scores,
                               score_stride);
}

// ---------------------------------------------------------------------------
// Pool candidates: keys [S][P*8]; candidate i is position 8*pool[i/8] + i%8.
// grid = (ceil(P*8/256), S), block = 256.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) k_pool_score(const uint8_t* __restrict__ kcodes,
                                                    const uint8_t* __restrict__ kscales, SegDesc sd,
                                                    const int32_t* __restrict__ seg_eff,
                                                    const uint8_t* __restrict__ q_codes,
                                                    const uint8_t* __restrict__ q_scales, const float* __restrict__ w,
                                                    const int32_t* __restrict__ pool, int P,
                                                    uint32_t* __restrict__ ckeys, uint32_t* status) {
  __shared__ IdxQueryPrep q;
  const int s = blockIdx.y;
  prep_query(q, q_codes + int64_t(s) * kHi * 64, q_scales + int64_t(s) * kHi * 4, w + int64_t(s) * kHi,
             threadIdx.x, 256);
  __syncthreads();
  const int i = blockIdx.x * 256 + threadIdx.x;
  if (i >= P * kBlk) return;
  const int64_t L = seg_eff[s];
  const int32_t blk = pool[int64_t(s) * P + i / kBlk];
  const int64_t t = int64_t(blk) * kBlk + (i % kBlk);
  uint32_t key = 0;
  if (blk >= 0) {
    if (int64_t(blk) * kBlk >= L) {
      if ((i % kBlk) == 0) set_status(status, CSA2_DEV_INDEX_RANGE);
    } else if (t < L) {
      const int64_t off = sd.row_off ? sd.row_off[s] : sd.row0;
      key = rank_key(score_row(q, kcodes, kscales, off + t));
    }
  }
  ckeys[int64_t(s) * P * kBlk + i] = key;
}

void launch_pool_score(const uint8_t* kcodes, const uint8_t* kscales, const SegDesc& sd, const int32_t* seg_eff,
                       int S, const uint8_t* q_codes, const uint8_t* q_scales, const float* w, const int32_t* pool,
                       int P, uint32_t* ckeys, uint32_t* status, cudaStream_t st) {
  if (S == 0) return;
  dim3 grid((P * kBlk + 255) / 256, S);
  k_pool_score<<<grid, 256, 0, st>>>(kcodes, kscales, sd, seg_eff, q_codes, q_scales, w, pool, P, ckeys, status);
}

// ---------------------------------------------------------------------------
// Prefill: visible entry counts, then the multi-query scan.
// ---------------------------------------------------------------------------
__global__ void k_prefill_vis(const int32_t* q_pos, int T, int ratio, int64_t n_entries, int32_t* vis,
                              uint32_t* status) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= T) return;
  int64_t p = q_pos[i];
  if (p < 0) {
    set_status(status, CSA2_DEV_LENGTH);
    p = -1;
  }
  int64_t v = (p + 1) / ratio;
  if (v > n_entries) v = n_entries;
  vis[i] = static_cast<int32_t>(v);
}

void launch_prefill_vis(const int32_t* q_pos, int T, int ratio, int64_t n_entries, int32_t* vis, uint32_t* status,
                        cudaStream_t st) {
  if (T == 0) return;
  k_prefill_vis<<<(T + 255) / 256, 256, 0, st>>>(q_pos, T, ratio, n_entries, vis, status);
}

// grid = (ceil(max_vis/256), ceil(T/kPQ)), block = 256.  Each thread unpacks
// its key row once and scores it against kPQ queries.
constexpr int kPQ = 16;
__global__ void __launch_bounds__(256) k_prefill_scan(const uint8_t* __restrict__ kcodes,
                                                      const uint8_t* __restrict__ kscales, int64_t row0,
                                                      const int32_t* __restrict__ vis, int T,
                                                      const uint8_t* __restrict__ q_codes,
                                                      const uint8_t* __restrict__ q_scales,
                                                      const float* __restrict__ w, uint32_t* __restrict__ bkeys,
                                                      int64_t nb_stride) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  IdxQueryPrep* qs = reinterpret_cast<IdxQueryPrep*>(smem_raw);
  const int i0 = blockIdx.y * kPQ;
  const int nq = min(kPQ, T - i0);
  const int64_t t0 = int64_t(blockIdx.x) * 256;
  __shared__ int any_vis;
  if (threadIdx.x == 0) {
    int a = 0;
    for (int j = 0; j < nq; ++j) a |= (vis[i0 + j] > t0);
    any_vis = a;
  }
  __syncthreads();
  if (!any_vis) return;
  for (int j = 0; j < nq; ++j)
    prep_query(qs[j], q_codes + int64_t(i0 + j) * kHi * 64, q_scales + int64_t(i0 + j) * kHi * 4,
               w + int64_t(i0 + j) * kHi, threadIdx.x, 256);
  __syncthreads();
  const int64_t t = t0 + threadIdx.x;
  uint32_t kw[16];
  uint32_t sw = 0;
  const int64_t row = row0 + t;
  // rows beyond the longest visibility of this query tile are never used
  int maxv = 0;
  for (int j = 0; j < nq; ++j) maxv = max(maxv, vis[i0 + j]);
  const bool live = t < maxv;
  if (live) {
    load_key_row(kcodes, row, kw);
    sw = __ldg(reinterpret_cast<const uint32_t*>(kscales) + row);
  } else {
#pragma unroll
    for (int m = 0; m < 16; ++m) kw[m] = 0;
  }
  for (int j = 0; j < nq; ++j) {
    const int64_t v = vis[i0 + j];
    uint32_t key = 0;
    if (t < v) {
      int D[kHi][4];
      block_dots(qs[j], kw, D);
      key = rank_key(combine_score(qs[j], D, sw));
    }
    key = group8_max(key);
    if ((threadIdx.x & 7) == 0 && t < v) bkeys[int64_t(i0 + j) * nb_stride + t / kBlk] = key;
  }
}

void launch_prefill_scan(const uint8_t* kcodes, const uint8_t* kscales, int64_t row0, const int32_t* vis, int T,
                         int64_t max_vis, const uint8_t* q_codes, const uint8_t* q_scales, const float* w,
                         uint32_t* bkeys, int64_t nb_stride, cudaStream_t st) {
  if (T == 0 || max_vis == 0) return;
  dim3 grid(static_cast<unsigned>((max_vis + 255) / 256), (T + kPQ - 1) / kPQ);
  const size_t smem = sizeof(IdxQueryPrep) * kPQ;
  cudaFuncSetAttribute(k_prefill_scan, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  k_prefill_scan<<<grid, 256, smem, st>>>(kcodes, kscales, row0, vis, T, q_codes, q_scales, w, bkeys, nb_stride);
}

// ---------------------------------------------------------------------------
// Selection: one CTA (1024 threads) per segment.
//   1) radix select (4 passes of 8 bits over keys != 0) for the threshold key
//      T and the number `rem` of keys equal to T that are taken;
//   2) an ordered pass over tiles of 4096 keys: key > T, or key == T among the
//      first `rem` equal keys in index order, is written at
//      (#greater before) + min(#equal before, rem).
// ---------------------------------------------------------------------------
constexpr int kSelThreads = 1024;

template <int KIND>
__device__ __forceinline__ uint32_t sel_key(const void* in, int64_t base, int64_t i, int64_t n) {
  if (i >= n) return 0u;
  if (KIND == kSelScores) return rank_key(static_cast<const float*>(in)[base + i]);
  return static_cast<const uint32_t*>(in)[base + i];
}

// Block-wide exclusive scan of one uint32 per thread; returns the exclusive
// prefix and writes the total to *total.
__device__ __forceinline__ uint32_t block_exclusive_scan(uint32_t v, uint32_t* warp_sums, uint32_t* total) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  uint32_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_sums[wid] = x;
  __syncthreads();
  if (wid == 0) {
    uint32_t ws = (lane < (kSelThreads / 32)) ? warp_sums[lane] : 0u;
    uint32_t z = ws;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, z, o);
      if (lane >= o) z += y;
    }
    warp_sums[lane] = z - ws;  // exclusive prefix of warp totals
    if (lane == 31) *total = z;
  }
  __syncthreads();
  const uint32_t r = warp_sums[wid] + x - v;
  __syncthreads();
  return r;
}

template <int KIND>
__global__ void __launch_bounds__(kSelThreads) k_select(const void* __restrict__ in, int64_t in_stride,
                                                        const int32_t* __restrict__ seg_eff, int P,
                                                        const int32_t* __restrict__ pool, int k,
                                                        int32_t* __restrict__ out) {
  __shared__ uint32_t hist[256];
  __shared__ uint32_t warp_sums[32];
  __shared__ uint32_t sh_total;
  __shared__ uint32_t sh_digit, sh_rem;
  const int s = blockIdx.x;
  const int tid = threadIdx.x;
  int64_t n;
  if (KIND == kSelBlockKeys) n = (int64_t(seg_eff[s]) + kBlk - 1) / kBlk;
  else if (KIND == kSelScores) n = seg_eff[s];
  else n = int64_t(P) * kBlk;
  const int64_t base = int64_t(s) * in_stride;
  int32_t* o = out + int64_t(s) * k;

  // pass 0 counts the present keys; passes 1..4 narrow the threshold
  uint32_t prefix = 0, pmask = 0, rem = uint32_t(k);
  uint32_t present = 0;
  for (int64_t i = tid; i < n; i += kSelThreads) present += (sel_key<KIND>(in, base, i, n) != 0u);
  block_exclusive_scan(present, warp_sums, &sh_total);
  const uint32_t total = sh_total;
  uint32_t T = 0;
  if (total <= uint32_t(k)) {
    T = 0;
    rem = 0;
  } else {
    for (int shift = 24; shift >= 0; shift -= 8) {
      for (int i = tid; i < 256; i += kSelThreads) hist[i] = 0;
      __syncthreads();
      for (int64_t i = tid; i < n; i += kSelThreads) {
        const uint32_t key = sel_key<KIND>(in, base, i, n);
        if (key != 0u && (key & pmask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
      }
      __syncthreads();
      if (tid == 0) {
        uint32_t cum = 0;
        int d = 255;
        for (; d > 0; --d) {
          if (cum + hist[d] >= rem) break;
          cum += hist[d];
        }
        sh_digit = uint32_t(d);
        sh_rem = rem - cum;
      }
      __syncthreads();
      prefix |= sh_digit << shift;
      pmask |= 255u << shift;
      rem = sh_rem;
      __syncthreads();
    }
    T = prefix;
  }

  // ordered output pass
  uint32_t run_gt = 0, run_eq = 0;
  for (int64_t t0 = 0; t0 < n; t0 += 4 * kSelThreads) {
    uint32_t kk[4];
    uint32_t gt = 0, eq = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      kk[j] = sel_key<KIND>(in, base, t0 + 4 * tid + j, n);
      gt += (kk[j] > T);
      eq += (kk[j] == T && kk[j] != 0u);
    }
    const uint32_t packed = (gt << 16) | eq;
    const uint32_t ex = block_exclusive_scan(packed, warp_sums, &sh_total);
    const uint32_t tot = sh_total;
    uint32_t g = run_gt + (ex >> 16), e = run_eq + (ex & 0xFFFFu);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int64_t i = t0 + 4 * tid + j;
      const uint32_t key = kk[j];
      int64_t id;
      if (KIND == kSelPoolCand) id = (i < n) ? int64_t(pool[int64_t(s) * P + i / kBlk]) * kBlk + (i % kBlk) : -1;
      else id = i;
      if (key > T) {
        o[g + min(e, rem)] = static_cast<int32_t>(id);
        ++g;
      } else if (key == T && key != 0u) {
        if (e < rem) o[g + e] = static_cast<int32_t>(id);
        ++e;
      }
    }
    run_gt += tot >> 16;
    run_eq += tot & 0xFFFFu;
    __syncthreads();
  }
  const uint32_t nsel = run_gt + min(run_eq, rem);
  for (int j = int(nsel) + tid; j < k; j += kSelThreads) o[j] = -1;
}

void launch_select(SelectKind kind, const void* in, int64_t in_stride, const int32_t* seg_eff, int S, int P,
                   const int32_t* pool, int k, int32_t* out, cudaStream_t st) {
  if (S == 0) return;
  switch (kind) {
    case kSelBlockKeys:
      k_select<kSelBlockKeys><<<S, kSelThreads, 0, st>>>(in, in_stride, seg_eff, P, pool, k, out);
      break;
    case kSelScores:
      k_select<kSelScores><<<S, kSelThreads, 0, st>>>(in, in_stride, seg_eff, P, pool, k, out);
      break;
    case kSelPoolCand:
      k_select<kSelPoolCand><<<S, kSelThreads, 0, st>>>(in, in_stride, seg_eff, P, pool, k, out);
      break;
  }
}

}  // namespace csa2
