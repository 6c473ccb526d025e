// Indexer kernels: prefill visibility and deterministic radix
// selection (Top-k by key desc / index asc, output ascending).  The scans and
// the pool scoring run on the tensor cores (scan_tc.cu, prefill_tc.cu).
//
// Score definition and selection rule: "DeepSeek-V4.1-Flash: Pushing the
// Limits of KV Cache Compression", section "三个方向一起压小缓存" (hierarchical
// sparse indexer, 8-position blocks ranked by their maximum, pool of at most
// 2048 blocks, Top-512 per layer, FP4 indexer q/k).
#include "device_common.cuh"
#include "sm100.cuh"

namespace csa2 {

// ---------------------------------------------------------------------------
// Prefill: visible entry counts (the scan itself runs on the tensor cores,
// prefill_tc.cu).
// ---------------------------------------------------------------------------
__global__ void k_prefill_vis(const int32_t* q_pos, int T, int ratio, int64_t n_entries, int32_t* vis,
                              uint32_t* status) {
  launch_dependents();
  grid_wait();
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
  launch_k(k_prefill_vis, dim3((T + 255) / 256), dim3(256), 0, st, q_pos, T, ratio, n_entries, vis, status);
}

// ---------------------------------------------------------------------------
// Selection: one CTA (1024 threads) per segment finds the k best of n keys
// (key 0 = absent) by (key desc, index asc) and writes their ids ascending.
// Keys are read in chunks of 16384 (16 consecutive keys per thread, four
// 16-byte loads), so every thread keeps 64 bytes in flight per chunk.
//   * the kernel that wrote the keys may also have histogrammed them (a row
//     per segment in the workspace: 15 bits for block keys, 12 bits for pool
//     candidates); the selection then starts from that row and zeroes it;
//   * small n (<= 16384): one chunk; the keys stay in registers through radix
//     digits of up to 8 bits (shared-memory histograms) and the ordered
//     output;
//   * large n: pass A builds a 15-bit histogram (unless the producer's row is
//     given) and finds the threshold bucket; pass B collects, in index order,
//     the ids of the keys above the bucket and the (low bits, id) of the keys
//     inside it (<= 12288); the exact threshold comes from radix passes over
//     those candidates in shared memory, and the two ordered lists are merged
//     into the output without another pass over the keys.  A bucket with more
//     than 12288 keys falls back to global radix passes and an ordered output
//     pass.
//   * large n from a producer's histogram, few segments: a cluster of two
//     CTAs per segment.  CTA 0 takes the histogram and finds the threshold
//     bucket, and sends it to CTA 1; each CTA collects the lists of one half
//     of the key chunks; CTA 1 writes its lists behind CTA 0's (their total
//     lengths follow from the histogram) and CTA 0 finishes alone.
// Output rule: key > T, or key == T among the first `rem` equal keys in
// index order; ids leave in ascending order.
// ---------------------------------------------------------------------------
constexpr int kSelThreads = 1024;
constexpr int kSelPer = 16;                          // keys per thread per chunk
constexpr int kSelChunk = kSelThreads * kSelPer;     // 16384
constexpr int kSelSmallMax = kSelChunk;
constexpr int kHist1Bits = kSelHistBits;
constexpr int kHist1Bins = kSelHistBins;
constexpr int kLowBits = 32 - kHist1Bits;  // 17
constexpr uint32_t kLowMask = (1u << kLowBits) - 1u;
constexpr int kCandCap = 12288;
constexpr int kSelMaxK = CSA2_MAX_TOPK;
// large-path shared memory: the histogram, later reused for the lists
constexpr int kSelLargeWords = kHist1Bins;
static_assert(kSelMaxK + 2 * kCandCap + 512 + kSelMaxK <= kSelLargeWords, "selection lists exceed the histogram");

template <int KIND>
__device__ __forceinline__ uint32_t sel_key(const void* in, int64_t base, int64_t i, int64_t n) {
  if (i >= n) return 0u;
  if (KIND == kSelScores) return rank_key(static_cast<const float*>(in)[base + i]);
  return static_cast<const uint32_t*>(in)[base + i];
}

// Keys i0 .. i0+15 (0 beyond n); 16-byte loads when the run is whole and aligned.
template <int KIND>
__device__ __forceinline__ void load_keys(const void* in, int64_t base, int64_t i0, int64_t n,
                                          uint32_t (&kk)[kSelPer]) {
  if (i0 + kSelPer <= n && ((base + i0) & 3) == 0) {
    const uint4* p = reinterpret_cast<const uint4*>(static_cast<const uint32_t*>(in) + base + i0);
    uint4 v[kSelPer / 4];
#pragma unroll
    for (int j = 0; j < kSelPer / 4; ++j) v[j] = __ldg(p + j);
#pragma unroll
    for (int j = 0; j < kSelPer / 4; ++j) {
      kk[4 * j] = v[j].x, kk[4 * j + 1] = v[j].y, kk[4 * j + 2] = v[j].z, kk[4 * j + 3] = v[j].w;
      if (KIND == kSelScores) {
#pragma unroll
        for (int e = 0; e < 4; ++e) kk[4 * j + e] = rank_key(__uint_as_float(kk[4 * j + e]));
      }
    }
  } else {
#pragma unroll
    for (int e = 0; e < kSelPer; ++e) kk[e] = sel_key<KIND>(in, base, i0 + e, n);
  }
}

template <int KIND>
__device__ __forceinline__ int32_t sel_id(const int32_t* pool, int s, int P, int64_t i) {
  if (KIND == kSelPoolCand) return pool[int64_t(s) * P + i / kBlk] * kBlk + int32_t(i % kBlk);
  if (KIND == kSelExplicit) return pool[int64_t(s) * P + i];
  return static_cast<int32_t>(i);
}

struct SelShared {
  uint32_t warp_sums[32];
  uint32_t total;
  uint32_t digit, rem;
  int sel_warp;         // find_bin: the warp whose bin range holds the threshold
  uint32_t sel_before;  // and the count above that range
  uint32_t xfer[6];     // cluster: (total, bucket, need, count) to CTA 1, (na, nc) to CTA 0
};

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

// Finds, among `nbins` bins of `hist` scanned from the top, the bin where the
// running count reaches `need`; returns it in sh.digit with the count still
// needed from it in sh.rem.  (Whole block; `hist` in shared memory.)  Large
// histograms are read with consecutive lanes on consecutive bins (no bank
// conflicts): every warp sums a contiguous range of bins, a scan of the warp
// totals picks the range that holds the threshold, and that warp walks its
// range 32 bins at a time.
__device__ __forceinline__ void find_bin(const uint32_t* hist, int nbins, uint32_t need, SelShared& sh) {
  if (threadIdx.x == 0) {  // defined result even for an inconsistent histogram
    sh.digit = 0;
    sh.rem = need;
  }
  if (nbins <= kSelThreads) {
    // thread j owns bin nbins - 1 - j (top bins first)
    const int b = nbins - 1 - int(threadIdx.x);
    const uint32_t mine = b >= 0 ? hist[b] : 0u;
    const uint32_t before = block_exclusive_scan(mine, sh.warp_sums, &sh.total);
    if (before < need && before + mine >= need) {
      sh.digit = uint32_t(b);
      sh.rem = need - before;
    }
    __syncthreads();
    return;
  }
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int per_warp = nbins / (kSelThreads / 32);  // a multiple of 32
  const int whi = nbins - per_warp * warp;          // warp w: bins [whi - per_warp, whi)
  uint32_t t = 0;
  for (int b = whi - per_warp + lane; b < whi; b += 32) t += hist[b];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
  __syncthreads();  // sh.warp_sums may still be read by the caller's previous step
  if (lane == 0) sh.warp_sums[warp] = t;
  __syncthreads();
  if (warp == 0) {
    const uint32_t v = sh.warp_sums[lane];  // lane = warp index, top range first
    uint32_t x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    const uint32_t hit = __ballot_sync(0xffffffffu, x - v < need && x >= need);
    if (lane == 0) sh.sel_warp = hit ? __ffs(hit) - 1 : -1;
    if (hit && lane == __ffs(hit) - 1) sh.sel_before = x - v;
  }
  __syncthreads();
  if (warp == sh.sel_warp) {
    uint32_t cum = sh.sel_before;
    for (int top = whi; top > whi - per_warp; top -= 32) {
      const int b = top - 1 - lane;  // lane 0 holds the highest bin of the group
      const uint32_t v = hist[b];
      uint32_t x = v;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
      }
      const uint32_t hit = __ballot_sync(0xffffffffu, cum + x >= need);
      if (hit) {
        if (lane == __ffs(hit) - 1) {
          sh.digit = uint32_t(b);
          sh.rem = need - (cum + x - v);
        }
        break;
      }
      cum += __shfl_sync(0xffffffffu, x, 31);
    }
  }
  __syncthreads();
}

// Adds one to hist[bin] for an active lane.  (Aggregating equal bins across
// the warp with match.any first was measured slower than the plain atomics.)
__device__ __forceinline__ void hist_add(uint32_t* hist, uint32_t bin, bool active) {
  if (active) atomicAdd(&hist[bin], 1u);
}

// Copies a segment's histogram row (written by the kernel that produced the
// keys) into shared memory and zeroes the row for the next call; returns this
// thread's share of the key count.
template <int NB>
struct HistPart {
  static constexpr int kVec = NB / 4 / kSelThreads;  // uint4 per thread
  static_assert(kVec >= 1 && NB % (4 * kSelThreads) == 0, "histogram rows are whole uint4 per thread");
  uint4 v[kVec];
};

// First half of take_hist: this thread's share of the row, loaded (kept in
// registers so the loads overlap other work).
template <int NB>
__device__ __forceinline__ void load_hist(const uint32_t* __restrict__ gh, HistPart<NB>& hp) {
#pragma unroll
  for (int j = 0; j < HistPart<NB>::kVec; ++j)
    hp.v[j] = __ldcg(reinterpret_cast<const uint4*>(gh) + threadIdx.x + j * kSelThreads);
}

// Second half: into shared memory, and the global row zeroed where non-zero.
template <int NB>
__device__ __forceinline__ void store_hist(uint32_t* __restrict__ gh, uint32_t* __restrict__ hist,
                                           const HistPart<NB>& hp) {
  uint4* g4 = reinterpret_cast<uint4*>(gh);
#pragma unroll
  for (int j = 0; j < HistPart<NB>::kVec; ++j) {
    const uint4 v = hp.v[j];
    reinterpret_cast<uint4*>(hist)[threadIdx.x + j * kSelThreads] = v;
    if ((v.x | v.y | v.z | v.w) != 0u) g4[threadIdx.x + j * kSelThreads] = make_uint4(0, 0, 0, 0);
  }
}

template <int NB>
__device__ __forceinline__ uint32_t take_hist(uint32_t* __restrict__ gh, uint32_t* __restrict__ hist) {
  constexpr int kVec = HistPart<NB>::kVec;
  uint4 v[kVec];
  uint4* g4 = reinterpret_cast<uint4*>(gh);
#pragma unroll
  for (int j = 0; j < kVec; ++j) v[j] = __ldcg(g4 + threadIdx.x + j * kSelThreads);
  uint32_t sum = 0;
#pragma unroll
  for (int j = 0; j < kVec; ++j) {
    reinterpret_cast<uint4*>(hist)[threadIdx.x + j * kSelThreads] = v[j];
    sum += v[j].x + v[j].y + v[j].z + v[j].w;
    if ((v[j].x | v[j].y | v[j].z | v[j].w) != 0u) g4[threadIdx.x + j * kSelThreads] = make_uint4(0, 0, 0, 0);
  }
  return sum;
}

// Position of the first element >= x in the ascending list a[0..n).
__device__ __forceinline__ uint32_t lower_bound_u32(const uint32_t* a, uint32_t n, uint32_t x) {
  uint32_t lo = 0, hi = n;
  while (lo < hi) {
    const uint32_t mid = (lo + hi) >> 1;
    if (a[mid] < x) lo = mid + 1;
    else hi = mid;
  }
  return lo;
}

// Ordered output pass over the keys in global memory (fallback of the large path).
template <int KIND>
__device__ void ordered_output_global(const void* in, int64_t base, int64_t n, uint32_t T, uint32_t rem,
                                      const int32_t* pool, int s, int P, int32_t* o, int k, SelShared& sh) {
  const int tid = threadIdx.x;
  uint32_t run_gt = 0, run_eq = 0;
  for (int64_t c0 = 0; c0 < n; c0 += kSelChunk) {
    uint32_t kk[kSelPer];
    const int64_t i0 = c0 + int64_t(tid) * kSelPer;
    load_keys<KIND>(in, base, i0, n, kk);
    uint32_t gt = 0, eq = 0;
#pragma unroll
    for (int e = 0; e < kSelPer; ++e) {
      gt += (kk[e] > T);
      eq += (kk[e] == T && kk[e] != 0u);
    }
    const uint32_t ex = block_exclusive_scan((gt << 16) | eq, sh.warp_sums, &sh.total);
    const uint32_t tot = sh.total;
    uint32_t g = run_gt + (ex >> 16), q = run_eq + (ex & 0xFFFFu);
#pragma unroll
    for (int e = 0; e < kSelPer; ++e) {
      const uint32_t key = kk[e];
      if (key > T) {
        const uint32_t at = g + min(q, rem);
        if (at < uint32_t(k)) o[at] = sel_id<KIND>(pool, s, P, i0 + e);
        ++g;
      } else if (key == T && key != 0u) {
        if (q < rem && g + q < uint32_t(k)) o[g + q] = sel_id<KIND>(pool, s, P, i0 + e);
        ++q;
      }
    }
    run_gt += tot >> 16;
    run_eq += tot & 0xFFFFu;
  }
  const uint32_t nsel = run_gt + min(run_eq, rem);
  for (int j = int(nsel) + tid; j < k; j += kSelThreads) o[j] = -1;
}

// The selection of segment s = blockIdx.x / CL (whole CTA, or with CL = 2
// the two CTAs of a cluster, large path with a producer histogram only);
// `dsm` is the dynamic shared memory the launch gave.
template <int KIND, bool SMALL, int CL>
__device__ __forceinline__ void select_segment(const void* __restrict__ in, int64_t in_stride,
                                               const int32_t* __restrict__ seg_eff, int P,
                                               const int32_t* __restrict__ pool, int k, int32_t* __restrict__ out,
                                               uint32_t* __restrict__ ghist, uint32_t* __restrict__ status,
                                               uint32_t* dsm, SelShared& sh) {
  static_assert(CL == 1 || (CL == 2 && !SMALL), "clusters serve the large path only");
  const int s = blockIdx.x / CL;
  const uint32_t rank = CL == 1 ? 0u : sm100::cluster_ctarank();
  const int tid = threadIdx.x;
  int64_t n;
  if (KIND == kSelBlockKeys) n = (int64_t(seg_eff[s]) + kBlk - 1) / kBlk;
  else if (KIND == kSelScores) n = seg_eff[s];
  else if (KIND == kSelExplicit) n = P;
  else n = int64_t(P) * kBlk;
  const int64_t base = int64_t(s) * in_stride;
  int32_t* o = out + int64_t(s) * k;

  if (SMALL) {
    // ---- one chunk: this thread's 16 keys stay in registers ----
    constexpr int HB = (KIND == kSelPoolCand) ? kCandHistBits : kHist1Bits;
    constexpr int NB = 1 << HB;
    uint32_t kk[kSelPer];
    const int64_t i0 = int64_t(tid) * kSelPer;
    HistPart<NB> hp;
    if (ghist) load_hist<NB>(ghist + int64_t(s) * NB, hp);  // in flight with the keys
    // pool candidates: the pool ids of this thread's two blocks, loaded with
    // the keys (not one dependent load per selected id at the end)
    constexpr int kIdBlocks = KIND == kSelPoolCand ? kSelPer / kBlk : 1;
    int32_t pid[kIdBlocks];
    if (KIND == kSelPoolCand) {
#pragma unroll
      for (int m = 0; m < kIdBlocks; ++m) {
        const int64_t bi = i0 / kBlk + m;
        pid[m] = bi < P ? __ldg(pool + int64_t(s) * P + bi) : -1;
      }
    }
    auto id_of = [&](int e) -> int32_t {
      if (KIND == kSelPoolCand) return pid[e / kBlk] * kBlk + (e % kBlk);
      return sel_id<KIND>(pool, s, P, i0 + e);
    };
    load_keys<KIND>(in, base, i0, n, kk);
    uint32_t present = 0;
#pragma unroll
    for (int e = 0; e < kSelPer; ++e) present += (kk[e] != 0u);
    block_exclusive_scan(present, sh.warp_sums, &sh.total);
    const uint32_t total = sh.total;
    uint32_t T = 0, rem = 0;
    if (ghist) {
      // the top HB bits from the producer's histogram; the low bits by radix
      // digits of up to 10 bits over the keys of the threshold bucket only
      // (two digits for both histogram widths)
      uint32_t* hist = dsm;       // NB
      uint32_t* h2 = dsm + NB;    // 1024
      store_hist<NB>(ghist + int64_t(s) * NB, hist, hp);
      __syncthreads();
      if (total > uint32_t(k)) {
        find_bin(hist, NB, uint32_t(k), sh);
        uint32_t prefix = sh.digit << (32 - HB), pmask = ~((1u << (32 - HB)) - 1u);
        rem = sh.rem;
        for (int hi = 31 - HB; hi >= 0; hi -= 10) {
          const int width = min(10, hi + 1), shift = hi - width + 1;
          const uint32_t dm = (1u << width) - 1u;
          h2[tid] = 0;  // 1024 threads, 1024 bins
          __syncthreads();
#pragma unroll
          for (int e = 0; e < kSelPer; ++e) {
            const uint32_t key = kk[e];
            hist_add(h2, (key >> shift) & dm, key != 0u && (key & pmask) == prefix);
          }
          __syncthreads();
          find_bin(h2, 1 << width, rem, sh);
          prefix |= sh.digit << shift;
          pmask |= dm << shift;
          rem = sh.rem;
        }
        T = prefix;
      }
    } else if (total > uint32_t(k)) {
      uint32_t* hist = dsm;  // 256 bins
      uint32_t prefix = 0, pmask = 0;
      rem = uint32_t(k);
      for (int shift = 24; shift >= 0; shift -= 8) {
        if (tid < 256) hist[tid] = 0;
        __syncthreads();
#pragma unroll
        for (int e = 0; e < kSelPer; ++e) {
          const uint32_t key = kk[e];
          hist_add(hist, (key >> shift) & 255u, key != 0u && (key & pmask) == prefix);
        }
        __syncthreads();
        find_bin(hist, 256, rem, sh);
        prefix |= sh.digit << shift;
        pmask |= 255u << shift;
        rem = sh.rem;
      }
      T = prefix;
    }
    // ---- ordered output ----
    uint32_t gt = 0, eq = 0;
#pragma unroll
    for (int e = 0; e < kSelPer; ++e) {
      gt += (kk[e] > T);
      eq += (kk[e] == T && kk[e] != 0u);
    }
    const uint32_t ex = block_exclusive_scan((gt << 16) | eq, sh.warp_sums, &sh.total);
    const uint32_t tot = sh.total;
    uint32_t g = ex >> 16, q = ex & 0xFFFFu;
#pragma unroll
    for (int e = 0; e < kSelPer; ++e) {
      const uint32_t key = kk[e];
      if (key > T) {
        const uint32_t at = g + min(q, rem);
        if (at < uint32_t(k)) o[at] = id_of(e);
        ++g;
      } else if (key == T && key != 0u) {
        if (q < rem && g + q < uint32_t(k)) o[g + q] = id_of(e);
        ++q;
      }
    }
    const uint32_t nsel = (tot >> 16) + min(tot & 0xFFFFu, rem);
    for (int j = int(nsel) + tid; j < k; j += kSelThreads) o[j] = -1;
    return;
  }

  // ---- large n, pass A: 15-bit histogram of the present keys ----
  uint32_t* hist = dsm;
  uint32_t present = 0;
  uint32_t total = 0, b1 = 0, need = 0, cnt = 0;
  if (CL == 2) {
    // CTA 0 finds the threshold bucket from the producer's histogram and
    // sends it to CTA 1 (ghist is non-null whenever CL == 2)
    if (rank == 0) {
      present = take_hist<kHist1Bins>(ghist + int64_t(s) * kHist1Bins, hist);
      __syncthreads();
      block_exclusive_scan(present, sh.warp_sums, &sh.total);
      total = sh.total;
      if (total > uint32_t(k)) {
        find_bin(hist, kHist1Bins, uint32_t(k), sh);
        b1 = sh.digit;
        need = sh.rem;
        cnt = hist[b1];
      }
      if (tid < 4) {
        const uint32_t v = tid == 0 ? total : tid == 1 ? b1 : tid == 2 ? need : cnt;
        sm100::st_cluster_u32(sm100::mapa_shared(sm100::smem_u32(&sh.xfer[tid]), 1), v);
      }
    }
    sm100::cluster_sync();
    if (rank == 1) {
      total = sh.xfer[0];
      b1 = sh.xfer[1];
      need = sh.xfer[2];
      cnt = sh.xfer[3];
    }
  } else if (ghist) {
    present = take_hist<kHist1Bins>(ghist + int64_t(s) * kHist1Bins, hist);
  } else {
    for (int i = tid; i < kHist1Bins; i += kSelThreads) hist[i] = 0;
    __syncthreads();
    uint32_t kk[kSelPer], nx[kSelPer];
    load_keys<KIND>(in, base, int64_t(tid) * kSelPer, n, kk);
    for (int64_t c0 = 0; c0 < n; c0 += kSelChunk) {
      if (c0 + kSelChunk < n) load_keys<KIND>(in, base, c0 + kSelChunk + int64_t(tid) * kSelPer, n, nx);
#pragma unroll
      for (int e = 0; e < kSelPer; ++e) {
        present += (kk[e] != 0u);
        hist_add(hist, kk[e] >> kLowBits, kk[e] != 0u);
      }
#pragma unroll
      for (int e = 0; e < kSelPer; ++e) kk[e] = nx[e];
    }
  }
  if (CL == 1) {
    __syncthreads();
    block_exclusive_scan(present, sh.warp_sums, &sh.total);
    total = sh.total;
    if (total > uint32_t(k)) {
      find_bin(hist, kHist1Bins, uint32_t(k), sh);
      b1 = sh.digit;
      need = sh.rem;
      cnt = hist[b1];
    }
  }
  const bool all = total <= uint32_t(k);
  __syncthreads();  // the histogram's memory is reused below

  if (!all && cnt > uint32_t(kCandCap)) {
    if (rank != 0) return;  // (both CTAs of a cluster decide alike; no cluster barrier follows)
    // more than kCandCap keys share the threshold bucket: global radix passes
    // over the low 17 bits (9 + 8), then an ordered pass over the keys
    if (status && tid == 0) atomicAdd(status + kDiagOverfull, 1u);
    uint32_t prefix = b1 << kLowBits, pmask = ~kLowMask, r = need;
    uint32_t* h2 = dsm;
    const int shifts[2] = {8, 0};
    const int widths[2] = {9, 8};
    for (int d = 0; d < 2; ++d) {
      const int nb = 1 << widths[d];
      for (int i = tid; i < nb; i += kSelThreads) h2[i] = 0;
      __syncthreads();
      const uint32_t dm = uint32_t(nb - 1);
      for (int64_t c0 = 0; c0 < n; c0 += kSelChunk) {
        uint32_t kk[kSelPer];
        load_keys<KIND>(in, base, c0 + int64_t(tid) * kSelPer, n, kk);
#pragma unroll
        for (int e = 0; e < kSelPer; ++e)
          hist_add(h2, (kk[e] >> shifts[d]) & dm, kk[e] != 0u && (kk[e] & pmask) == prefix);
      }
      __syncthreads();
      find_bin(h2, nb, r, sh);
      prefix |= sh.digit << shifts[d];
      pmask |= dm << shifts[d];
      r = sh.rem;
    }
    ordered_output_global<KIND>(in, base, n, prefix, r, pool, s, P, o, k, sh);
    return;
  }

  // ---- pass B: ordered lists of the keys above the bucket and inside it ----
  uint32_t* A = dsm;                     // [kSelMaxK] ids above the bucket (all present ids if `all`)
  uint32_t* Clow = A + kSelMaxK;         // [kCandCap] low bits of the bucket's keys
  uint32_t* Cidx = Clow + kCandCap;      // [kCandCap] their ids
  uint32_t* h2 = Cidx + kCandCap;        // [512]
  uint32_t* Csel = h2 + 512;             // [kSelMaxK] selected bucket ids
  uint32_t run_a = 0, run_c = 0;
  {
    // this CTA's keys: all, or (cluster) one half of the chunks
    int64_t lo = 0, hi = n;
    if (CL == 2) {
      const int64_t half = (n + 2 * kSelChunk - 1) / (2 * kSelChunk) * kSelChunk;
      lo = rank == 0 ? 0 : half;
      hi = rank == 0 ? (half < n ? half : n) : n;
    }
    uint32_t kk[kSelPer], nx[kSelPer];
    load_keys<KIND>(in, base, lo + int64_t(tid) * kSelPer, hi, kk);
    for (int64_t c0 = lo; c0 < hi; c0 += kSelChunk) {
      if (c0 + kSelChunk < hi) load_keys<KIND>(in, base, c0 + kSelChunk + int64_t(tid) * kSelPer, hi, nx);
      // most threads hold no key at or above the bucket: one max decides
      uint32_t mx = 0;
#pragma unroll
      for (int e = 0; e < kSelPer; ++e) mx = max(mx, kk[e]);
      const bool hot = mx != 0u && (all || (mx >> kLowBits) >= b1);
      uint32_t na = 0, nc = 0;
      if (hot) {
#pragma unroll
        for (int e = 0; e < kSelPer; ++e) {
          const uint32_t key = kk[e], hi = key >> kLowBits;
          if (key != 0u) {
            if (all || hi > b1) ++na;
            else if (hi == b1) ++nc;
          }
        }
      }
      const uint32_t ex = block_exclusive_scan((na << 16) | nc, sh.warp_sums, &sh.total);
      const uint32_t tot = sh.total;
      uint32_t a = run_a + (ex >> 16), c = run_c + (ex & 0xFFFFu);
      const uint32_t i0 = uint32_t(c0) + uint32_t(tid) * kSelPer;
#pragma unroll
      for (int e = 0; e < kSelPer && hot; ++e) {
        const uint32_t key = kk[e], hi = key >> kLowBits;
        if (key != 0u) {
          if (all || hi > b1) {
            if (a < uint32_t(kSelMaxK)) A[a] = i0 + e;
            ++a;
          } else if (hi == b1) {
            if (c < uint32_t(kCandCap)) {
              Clow[c] = key & kLowMask;
              Cidx[c] = i0 + e;
            }
            ++c;
          }
        }
      }
      run_a += tot >> 16;
      run_c += tot & 0xFFFFu;
#pragma unroll
      for (int e = 0; e < kSelPer; ++e) kk[e] = nx[e];
    }
  }
  __syncthreads();
  if (CL == 2) {
    // CTA 1's lists go behind CTA 0's: the histogram fixes both totals
    const uint32_t na_tot = all ? total : uint32_t(k) - need, nc_tot = all ? 0u : cnt;
    if (rank == 1) {
      const uint32_t a_off = na_tot - min(run_a, na_tot), c_off = nc_tot - min(run_c, nc_tot);
      for (uint32_t i = tid; i < run_a && a_off + i < uint32_t(kSelMaxK); i += kSelThreads)
        sm100::st_cluster_u32(sm100::mapa_shared(sm100::smem_u32(&A[a_off + i]), 0), A[i]);
      for (uint32_t i = tid; i < run_c && c_off + i < uint32_t(kCandCap); i += kSelThreads) {
        sm100::st_cluster_u32(sm100::mapa_shared(sm100::smem_u32(&Clow[c_off + i]), 0), Clow[i]);
        sm100::st_cluster_u32(sm100::mapa_shared(sm100::smem_u32(&Cidx[c_off + i]), 0), Cidx[i]);
      }
      if (tid < 2) sm100::st_cluster_u32(sm100::mapa_shared(sm100::smem_u32(&sh.xfer[4 + tid]), 0),
                                         tid == 0 ? run_a : run_c);
    }
    sm100::cluster_sync();
    if (rank == 1) return;
    // the halves' lengths disagree with the histogram only after a producer
    // failure that already set a flag: no pool then
    if (run_a + sh.xfer[4] != na_tot || run_c + sh.xfer[5] != nc_tot || na_tot > uint32_t(kSelMaxK)) {
      for (int j = tid; j < k; j += kSelThreads) o[j] = -1;
      return;
    }
    run_a = na_tot;
    run_c = nc_tot;
  }
  // (the list lengths only exceed their capacities if the histogram and the
  // keys disagree, i.e. after a producer failure that already set a flag)
  run_a = min(run_a, uint32_t(kSelMaxK));
  if (all) {
    for (uint32_t i = tid; i < run_a; i += kSelThreads)
      if (i < uint32_t(k)) o[i] = sel_id<KIND>(pool, s, P, A[i]);
    for (int j = int(run_a) + tid; j < k; j += kSelThreads) o[j] = -1;
    return;
  }
  // exact threshold inside the bucket: digits of 9 and 8 bits over the candidates
  const uint32_t nc = min(run_c, uint32_t(kCandCap));
  uint32_t prefix = 0, pmask = 0, r = need;
  {
    const int shifts[2] = {8, 0};
    const int widths[2] = {9, 8};
    for (int d = 0; d < 2; ++d) {
      const int nb = 1 << widths[d];
      for (int i = tid; i < nb; i += kSelThreads) h2[i] = 0;
      __syncthreads();
      const uint32_t dm = uint32_t(nb - 1);
      for (uint32_t i0 = 0; i0 < nc; i0 += kSelThreads) {
        const uint32_t i = i0 + tid;
        const uint32_t low = i < nc ? Clow[i] : 0u;
        hist_add(h2, (low >> shifts[d]) & dm, i < nc && (low & pmask) == prefix);
      }
      __syncthreads();
      find_bin(h2, nb, r, sh);
      prefix |= sh.digit << shifts[d];
      pmask |= dm << shifts[d];
      r = sh.rem;
    }
  }
  // the bucket's selected ids in index order: low > prefix, or == prefix among the first r
  {
    const uint32_t per = (nc + kSelThreads - 1) / kSelThreads;
    const uint32_t lo = min(nc, per * tid), hi = min(nc, lo + per);
    uint32_t gt = 0, eq = 0;
    for (uint32_t i = lo; i < hi; ++i) {
      gt += (Clow[i] > prefix);
      eq += (Clow[i] == prefix);
    }
    const uint32_t ex = block_exclusive_scan((gt << 16) | eq, sh.warp_sums, &sh.total);
    uint32_t g = ex >> 16, q = ex & 0xFFFFu;
    for (uint32_t i = lo; i < hi; ++i) {
      if (Clow[i] > prefix) {
        const uint32_t at = g + min(q, r);
        if (at < need) Csel[at] = Cidx[i];
        ++g;
      } else if (Clow[i] == prefix) {
        if (q < r && g + q < need) Csel[g + q] = Cidx[i];
        ++q;
      }
    }
  }
  __syncthreads();
  // merge the two ascending lists: k - need ids above the bucket, need from it
  const uint32_t na = run_a;
  for (uint32_t i = tid; i < na; i += kSelThreads) {
    const uint32_t at = i + lower_bound_u32(Csel, need, A[i]);
    if (at < uint32_t(k)) o[at] = sel_id<KIND>(pool, s, P, A[i]);
  }
  for (uint32_t j = tid; j < need; j += kSelThreads) {
    const uint32_t at = j + lower_bound_u32(A, na, Csel[j]);
    if (at < uint32_t(k)) o[at] = sel_id<KIND>(pool, s, P, Csel[j]);
  }
}

// Adds one to hist[bin] for every active lane, one atomic per distinct bin of
// the warp (the keys near the top of a pool share their high bits, so plain
// shared atomics would serialise on a few bins).
__device__ __forceinline__ void hist_add_warp(uint32_t* hist, uint32_t bin, bool active) {
  const uint32_t am = __ballot_sync(0xffffffffu, active);
  if (!active) return;
  const uint32_t peers = __match_any_sync(am, bin);
  if ((threadIdx.x & 31) == __ffs(peers) - 1) atomicAdd(&hist[bin], uint32_t(__popc(peers)));
}

// After segment s's pool (`o`: n_pool <= 2048 block ids, ascending, then -1)
// is written: its best `kb` blocks by (block key desc, id asc), ascending,
// into tb (-1 padded).  Every one of the kb best positions lies in those
// blocks: each block ranked before the block b of a selected position p
// holds a position ranked before p (its own best; among equal keys the
// lower block holds the lower position), which is then selected too, so
// fewer than kb blocks rank before b.  The position Top-kb is therefore taken
// from the 8 kb positions of these blocks instead of the whole pool's.
// Radix digits of 8 bits start below the bits every pool key shares.
__device__ __forceinline__ void top_blocks_of_pool(const uint32_t* __restrict__ keys, const int32_t* o, int n_pool,
                                                   int kb, int32_t* __restrict__ tb, uint32_t* hist,
                                                   SelShared& sh) {
  __syncthreads();  // the pool written by every thread of the CTA is visible
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  uint32_t kk[2];
  int32_t id[2];
#pragma unroll
  for (int e = 0; e < 2; ++e) {  // entries 2 tid, 2 tid + 1 (ids ascend with the entry)
    const int i = 2 * tid + e;
    id[e] = i < n_pool ? o[i] : -1;
    kk[e] = id[e] >= 0 ? keys[id[e]] : 0u;
  }
  // present count, and the AND / OR of the present keys
  uint32_t cnt = (kk[0] != 0u) + (kk[1] != 0u);
  uint32_t kand = (kk[0] ? kk[0] : ~0u) & (kk[1] ? kk[1] : ~0u), kor = kk[0] | kk[1];
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    cnt += __shfl_xor_sync(0xffffffffu, cnt, off);
    kand &= __shfl_xor_sync(0xffffffffu, kand, off);
    kor |= __shfl_xor_sync(0xffffffffu, kor, off);
  }
  uint32_t* wred = hist;  // 3 x 32 words, before the histogram uses them
  if (lane == 0) {
    wred[wid] = cnt;
    wred[32 + wid] = kand;
    wred[64 + wid] = kor;
  }
  __syncthreads();
  uint32_t total = 0, all_and = ~0u, all_or = 0u;
#pragma unroll 8
  for (int w = 0; w < kSelThreads / 32; ++w) {
    total += wred[w];
    all_and &= wred[32 + w];
    all_or |= wred[64 + w];
  }
  __syncthreads();  // wred is read by everyone before the histogram reuses it
  uint32_t T = 0, rem = 0;
  if (total > uint32_t(kb)) {
    const uint32_t diff = all_and ^ all_or;  // bits on which the present keys differ
    rem = uint32_t(kb);
    if (diff == 0u) {
      T = all_and;  // every present key equal: the lowest ids win
    } else {
      const int top = 31 - __clz(diff);
      const uint32_t common = top == 31 ? 0u : ~((2u << top) - 1u);
      uint32_t prefix = all_and & common, pmask = common;
      for (int hi = top; hi >= 0; hi -= 8) {
        const int width = min(8, hi + 1), shift = hi - width + 1;
        const uint32_t dm = (1u << width) - 1u;
        if (tid < 256) hist[tid] = 0;
        __syncthreads();
#pragma unroll
        for (int e = 0; e < 2; ++e)
          hist_add_warp(hist, (kk[e] >> shift) & dm, kk[e] != 0u && (kk[e] & pmask) == prefix);
        __syncthreads();
        find_bin(hist, 1 << width, rem, sh);
        prefix |= sh.digit << shift;
        pmask |= dm << shift;
        rem = sh.rem;
      }
      T = prefix;
    }
  }
  // ordered output: key > T, or key == T among the first rem (ids ascend with the entry)
  uint32_t gt = 0, eq = 0;
#pragma unroll
  for (int e = 0; e < 2; ++e) {
    gt += (kk[e] > T);
    eq += (kk[e] == T && kk[e] != 0u);
  }
  const uint32_t ex = block_exclusive_scan((gt << 16) | eq, sh.warp_sums, &sh.total);
  const uint32_t tot = sh.total;
  uint32_t g = ex >> 16, q = ex & 0xFFFFu;
#pragma unroll
  for (int e = 0; e < 2; ++e) {
    if (kk[e] > T) {
      const uint32_t at = g + min(q, rem);
      if (at < uint32_t(kb)) tb[at] = id[e];
      ++g;
    } else if (kk[e] == T && kk[e] != 0u) {
      if (q < rem && g + q < uint32_t(kb)) tb[g + q] = id[e];
      ++q;
    }
  }
  const uint32_t nsel = (tot >> 16) + min(tot & 0xFFFFu, rem);
  for (int j = int(nsel) + tid; j < kb; j += kSelThreads) tb[j] = -1;
}

// One CTA (1024 threads) per segment, or a cluster of CL = 2.  Block-key
// selections may also write the best `kb` blocks of each pool into topblk
// [S][kb] (see top_blocks_of_pool).
template <int KIND, bool SMALL, int CL>
__global__ void __launch_bounds__(kSelThreads, 1) k_select(const void* __restrict__ in, int64_t in_stride,
                                                        const int32_t* __restrict__ seg_eff, int P,
                                                        const int32_t* __restrict__ pool, int k,
                                                        int32_t* __restrict__ out, uint32_t* __restrict__ ghist,
                                                        uint32_t* __restrict__ status, int32_t* __restrict__ topblk,
                                                        int kb) {
  extern __shared__ __align__(16) uint32_t dsm[];
  __shared__ SelShared sh;
  launch_dependents();
  grid_wait();
  select_segment<KIND, SMALL, CL>(in, in_stride, seg_eff, P, pool, k, out, ghist, status, dsm, sh);
  if (KIND == kSelBlockKeys && topblk != nullptr && (CL == 1 || sm100::cluster_ctarank() == 0)) {
    const int s = blockIdx.x / CL;
    top_blocks_of_pool(static_cast<const uint32_t*>(in) + int64_t(s) * in_stride, out + int64_t(s) * k, k, kb,
                       topblk + int64_t(s) * kb, dsm, sh);
  }
}

template <int KIND>
void launch_select_kind(const void* in, int64_t in_stride, const int32_t* seg_eff, int S, int P, const int32_t* pool,
                        int k, int32_t* out, uint32_t* hist, int64_t n_bound, cudaStream_t st, uint32_t* status,
                        int32_t* topblk, int kb) {
  if (n_bound <= kSelSmallMax) {
    constexpr int NB = (KIND == kSelPoolCand) ? kCandHistBins : kHist1Bins;
    const size_t smem = (hist ? NB + 1024 : 256) * sizeof(uint32_t);
    cudaFuncSetAttribute(k_select<KIND, true, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         int((NB + 1024) * sizeof(uint32_t)));
    launch_k(k_select<KIND, true, 1>, dim3(S), dim3(kSelThreads), smem, st, in, in_stride, seg_eff, P, pool, k, out,
             hist, status, topblk, kb);
  } else if (hist != nullptr && 2 * int64_t(S) <= num_sms()) {
    // few segments: two CTAs (SMs) each, still one wave
    const size_t smem = kSelLargeWords * sizeof(uint32_t);
    cudaFuncSetAttribute(k_select<KIND, false, 2>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
    launch_k_cluster(k_select<KIND, false, 2>, dim3(2 * S), dim3(kSelThreads), smem, st, 2, in, in_stride, seg_eff, P,
                     pool, k, out, hist, status, topblk, kb);
  } else {
    const size_t smem = kSelLargeWords * sizeof(uint32_t);
    cudaFuncSetAttribute(k_select<KIND, false, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
    launch_k(k_select<KIND, false, 1>, dim3(S), dim3(kSelThreads), smem, st, in, in_stride, seg_eff, P, pool, k, out,
             hist, status, topblk, kb);
  }
}

void launch_select(SelectKind kind, const void* in, int64_t in_stride, const int32_t* seg_eff, int S, int P,
                   const int32_t* pool, int k, int32_t* out, uint32_t* hist, cudaStream_t st, uint32_t* status,
                   int32_t* topblk, int kb) {
  if (S == 0) return;
  // n per segment is at most the row stride of the input
  switch (kind) {
    case kSelBlockKeys:
      launch_select_kind<kSelBlockKeys>(in, in_stride, seg_eff, S, P, pool, k, out, hist, in_stride, st, status, topblk,
                                        kb);
      break;
    case kSelScores:
      launch_select_kind<kSelScores>(in, in_stride, seg_eff, S, P, pool, k, out, hist, in_stride, st, status,
                                     nullptr, 0);
      break;
    case kSelPoolCand:
      launch_select_kind<kSelPoolCand>(in, in_stride, seg_eff, S, P, pool, k, out, hist, in_stride, st, status,
                                       nullptr, 0);
      break;
    case kSelExplicit:
      launch_select_kind<kSelExplicit>(in, in_stride, seg_eff, S, P, pool, k, out, hist, in_stride, st, status,
                                       nullptr, 0);
      break;
  }
}

}  // namespace csa2
