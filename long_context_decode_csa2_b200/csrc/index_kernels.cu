// Indexer kernels: segment checks, the multi-query causal prefill scan, and
// deterministic radix selection (Top-k by key desc / index asc, output
// ascending).  The decode scan and the pool scoring run on the tensor cores
// (scan_tc.cu).
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
// Selection: one CTA (1024 threads) per segment finds the k best of n keys
// (key 0 = absent) by (key desc, index asc) and writes their ids ascending.
//   * small n (<= 16384): the keys live in shared memory; radix passes of
//     8 bits and the ordered output pass all read shared memory;
//   * large n: one global pass builds a 15-bit histogram, a second collects
//     the keys of the threshold bucket (<= 12288 of them; otherwise a global
//     radix pass per remaining digit), the exact threshold comes from an
//     in-smem radix over those candidates, and a last global pass writes the
//     selection in index order.
// Output rule: key > T, or key == T among the first `rem` equal keys in
// index order, goes to position (#greater before) + min(#equal before, rem).
// ---------------------------------------------------------------------------
constexpr int kSelThreads = 1024;
constexpr int kSelSmallMax = 16384;
constexpr int kHist1Bits = 15;
constexpr int kHist1Bins = 1 << kHist1Bits;
constexpr int kLowBits = 32 - kHist1Bits;  // 17
constexpr int kCandCap = 12288;

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
    const uint32_t ws = (lane < (kSelThreads / 32)) ? warp_sums[lane] : 0u;
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

struct SelShared {
  uint32_t warp_sums[32];
  uint32_t total;
  uint32_t digit, rem, found;
  uint32_t ncand;
};

// Finds, among `cnt` bins of `hist` scanned from the top, the bin where the
// running count reaches `need`; returns it in sh.digit with the count still
// needed from it in sh.rem.  (Whole block; `hist` in shared memory.)
__device__ __forceinline__ void find_bin(const uint32_t* hist, int nbins, uint32_t need, SelShared& sh) {
  const int per = (nbins + kSelThreads - 1) / kSelThreads;
  // thread j owns bins [nbins - per*(j+1), nbins - per*j) (top bins first)
  const int hi = nbins - per * int(threadIdx.x);
  const int lo = max(0, hi - per);
  uint32_t mine = 0;
  for (int b = lo; b < hi; ++b) mine += hist[b];
  const uint32_t before = block_exclusive_scan(mine, sh.warp_sums, &sh.total);
  if (before < need && before + mine >= need) {
    uint32_t cum = before;
    for (int b = hi - 1; b >= lo; --b) {
      if (cum + hist[b] >= need) {
        sh.digit = uint32_t(b);
        sh.rem = need - cum;
        break;
      }
      cum += hist[b];
    }
  }
  __syncthreads();
}

template <int KIND, bool SMALL>
__device__ __forceinline__ uint32_t get_key(const uint32_t* ks, const void* in, int64_t base, int64_t i, int64_t n) {
  if (SMALL) return i < n ? ks[i] : 0u;
  return sel_key<KIND>(in, base, i, n);
}

template <int KIND, bool SMALL>
__global__ void __launch_bounds__(kSelThreads) k_select(const void* __restrict__ in, int64_t in_stride,
                                                        const int32_t* __restrict__ seg_eff, int P,
                                                        const int32_t* __restrict__ pool, int k,
                                                        int32_t* __restrict__ out) {
  extern __shared__ __align__(16) uint32_t dsm[];
  __shared__ SelShared sh;
  const int s = blockIdx.x;
  const int tid = threadIdx.x;
  int64_t n;
  if (KIND == kSelBlockKeys) n = (int64_t(seg_eff[s]) + kBlk - 1) / kBlk;
  else if (KIND == kSelScores) n = seg_eff[s];
  else n = int64_t(P) * kBlk;
  const int64_t base = int64_t(s) * in_stride;
  int32_t* o = out + int64_t(s) * k;
  uint32_t* ks = dsm;  // small: the keys; large: unused

  uint32_t T = 0, rem = 0, total;
  if (SMALL) {
    // ---- keys into shared memory, present count ----
    uint32_t present = 0;
    for (int64_t i = tid; i < n; i += kSelThreads) {
      const uint32_t key = sel_key<KIND>(in, base, i, n);
      ks[i] = key;
      present += (key != 0u);
    }
    block_exclusive_scan(present, sh.warp_sums, &sh.total);
    total = sh.total;
    if (total > uint32_t(k)) {
      uint32_t* hist = dsm + kSelSmallMax;
      uint32_t prefix = 0, pmask = 0;
      rem = uint32_t(k);
      for (int shift = 24; shift >= 0; shift -= 8) {
        if (tid < 256) hist[tid] = 0;
        __syncthreads();
        for (int64_t i = tid; i < n; i += kSelThreads) {
          const uint32_t key = ks[i];
          if (key != 0u && (key & pmask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
        }
        __syncthreads();
        find_bin(hist, 256, rem, sh);
        prefix |= sh.digit << shift;
        pmask |= 255u << shift;
        rem = sh.rem;
      }
      T = prefix;
    }
  } else {
    // ---- pass A: 15-bit histogram of the present keys ----
    uint32_t* hist = dsm;                        // kHist1Bins
    uint32_t* cand = dsm + kHist1Bins;           // kCandCap low parts
    for (int i = tid; i < kHist1Bins; i += kSelThreads) hist[i] = 0;
    __syncthreads();
    uint32_t present = 0;
    for (int64_t i0 = int64_t(tid) * 4; i0 < n; i0 += int64_t(kSelThreads) * 4) {
      uint32_t kk[4];
      if (KIND == kSelBlockKeys && i0 + 3 < n && ((base + i0) & 3) == 0) {
        const uint4 v = *reinterpret_cast<const uint4*>(static_cast<const uint32_t*>(in) + base + i0);
        kk[0] = v.x, kk[1] = v.y, kk[2] = v.z, kk[3] = v.w;
      } else {
#pragma unroll
        for (int j = 0; j < 4; ++j) kk[j] = sel_key<KIND>(in, base, i0 + j, n);
      }
#pragma unroll
      for (int j = 0; j < 4; ++j)
        if (kk[j] != 0u) {
          ++present;
          atomicAdd(&hist[kk[j] >> kLowBits], 1u);
        }
    }
    block_exclusive_scan(present, sh.warp_sums, &sh.total);
    total = sh.total;
    if (total > uint32_t(k)) {
      find_bin(hist, kHist1Bins, uint32_t(k), sh);
      const uint32_t b1 = sh.digit, need = sh.rem, cnt = hist[b1];
      __syncthreads();
      if (cnt <= uint32_t(kCandCap)) {
        // ---- pass B: collect the low bits of the threshold bucket's keys ----
        if (tid == 0) sh.ncand = 0;
        __syncthreads();
        for (int64_t i = tid; i < n; i += kSelThreads) {
          const uint32_t key = sel_key<KIND>(in, base, i, n);
          if (key != 0u && (key >> kLowBits) == b1) cand[atomicAdd(&sh.ncand, 1u)] = key & ((1u << kLowBits) - 1u);
        }
        __syncthreads();
        const uint32_t nc = sh.ncand;
        // exact threshold among the candidates: digits of 9 and 8 bits
        uint32_t prefix = 0, pmask = 0, r = need;
        uint32_t* h2 = hist;  // reuse (first 512 bins)
        const int shifts[2] = {8, 0};
        const int widths[2] = {9, 8};
        for (int d = 0; d < 2; ++d) {
          const int nb = 1 << widths[d];
          for (int i = tid; i < nb; i += kSelThreads) h2[i] = 0;
          __syncthreads();
          const uint32_t dm = uint32_t(nb - 1);
          for (uint32_t i = tid; i < nc; i += kSelThreads) {
            const uint32_t low = cand[i];
            if ((low & pmask) == prefix) atomicAdd(&h2[(low >> shifts[d]) & dm], 1u);
          }
          __syncthreads();
          find_bin(h2, nb, r, sh);
          prefix |= sh.digit << shifts[d];
          pmask |= dm << shifts[d];
          r = sh.rem;
        }
        T = (b1 << kLowBits) | prefix;
        rem = r;
      } else {
        // more than kCandCap keys share the threshold bucket: finish with
        // global radix passes over the low 17 bits (9 + 8)
        uint32_t prefix = b1 << kLowBits, pmask = ~((1u << kLowBits) - 1u), r = need;
        uint32_t* h2 = hist;
        const int shifts[2] = {8, 0};
        const int widths[2] = {9, 8};
        for (int d = 0; d < 2; ++d) {
          const int nb = 1 << widths[d];
          for (int i = tid; i < nb; i += kSelThreads) h2[i] = 0;
          __syncthreads();
          const uint32_t dm = uint32_t(nb - 1);
          for (int64_t i = tid; i < n; i += kSelThreads) {
            const uint32_t key = sel_key<KIND>(in, base, i, n);
            if (key != 0u && (key & pmask) == prefix) atomicAdd(&h2[(key >> shifts[d]) & dm], 1u);
          }
          __syncthreads();
          find_bin(h2, nb, r, sh);
          prefix |= sh.digit << shifts[d];
          pmask |= dm << shifts[d];
          r = sh.rem;
        }
        T = prefix;
        rem = r;
      }
    }
  }
  if (total <= uint32_t(k)) {
    T = 0;
    rem = 0;
  }

  // ---- ordered output pass ----
  uint32_t run_gt = 0, run_eq = 0;
  for (int64_t t0 = 0; t0 < n; t0 += 4 * kSelThreads) {
    uint32_t kk[4];
    uint32_t gt = 0, eq = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      kk[j] = get_key<KIND, SMALL>(ks, in, base, t0 + 4 * tid + j, n);
      gt += (kk[j] > T);
      eq += (kk[j] == T && kk[j] != 0u);
    }
    const uint32_t packed = (gt << 16) | eq;
    const uint32_t ex = block_exclusive_scan(packed, sh.warp_sums, &sh.total);
    const uint32_t tot = sh.total;
    uint32_t g = run_gt + (ex >> 16), e = run_eq + (ex & 0xFFFFu);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int64_t i = t0 + 4 * tid + j;
      const uint32_t key = kk[j];
      if (key > T || (key == T && key != 0u)) {
        int64_t id;
        if (KIND == kSelPoolCand) id = int64_t(pool[int64_t(s) * P + i / kBlk]) * kBlk + (i % kBlk);
        else id = i;
        if (key > T) {
          o[g + min(e, rem)] = static_cast<int32_t>(id);
          ++g;
        } else {
          if (e < rem) o[g + e] = static_cast<int32_t>(id);
          ++e;
        }
      }
    }
    run_gt += tot >> 16;
    run_eq += tot & 0xFFFFu;
  }
  const uint32_t nsel = run_gt + min(run_eq, rem);
  for (int j = int(nsel) + tid; j < k; j += kSelThreads) o[j] = -1;
}

template <int KIND>
void launch_select_kind(const void* in, int64_t in_stride, const int32_t* seg_eff, int S, int P, const int32_t* pool,
                        int k, int32_t* out, int64_t n_bound, cudaStream_t st) {
  if (n_bound <= kSelSmallMax) {
    const size_t smem = (kSelSmallMax + 256) * sizeof(uint32_t);
    cudaFuncSetAttribute(k_select<KIND, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
    k_select<KIND, true><<<S, kSelThreads, smem, st>>>(in, in_stride, seg_eff, P, pool, k, out);
  } else {
    const size_t smem = (kHist1Bins + kCandCap) * sizeof(uint32_t);
    cudaFuncSetAttribute(k_select<KIND, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
    k_select<KIND, false><<<S, kSelThreads, smem, st>>>(in, in_stride, seg_eff, P, pool, k, out);
  }
}

void launch_select(SelectKind kind, const void* in, int64_t in_stride, const int32_t* seg_eff, int S, int P,
                   const int32_t* pool, int k, int32_t* out, cudaStream_t st) {
  if (S == 0) return;
  // n per segment is at most the row stride of the input
  switch (kind) {
    case kSelBlockKeys:
      launch_select_kind<kSelBlockKeys>(in, in_stride, seg_eff, S, P, pool, k, out, in_stride, st);
      break;
    case kSelScores:
      launch_select_kind<kSelScores>(in, in_stride, seg_eff, S, P, pool, k, out, in_stride, st);
      break;
    case kSelPoolCand:
      launch_select_kind<kSelPoolCand>(in, in_stride, seg_eff, S, P, pool, k, out, in_stride, st);
      break;
  }
}

}  // namespace csa2
