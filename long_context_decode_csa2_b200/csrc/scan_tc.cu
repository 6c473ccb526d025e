// Indexer scoring on the 5th-generation tensor cores (sm_100a): the
// full-context scan (block maxima) and the pool-candidate scoring (one key per
// candidate) share one kernel.
//
// Score definition: "DeepSeek-V4.1-Flash: Pushing the Limits of KV Cache
// Compression", section "三个方向一起压小缓存" (FP4 indexer q/k, block maxima over
// 8 positions, candidate pool of 2048 blocks x 8); see csa2.h for the exact
// rounding rules.
//
// One persistent CTA per SM walks a contiguous range of work items; an item
// is 512 positions of one segment: 512 consecutive rows (scan) or the rows of
// 64 pool blocks (pool scoring).  Per item:
//   * the producer loads the 64-byte code rows and the 4-byte E8M0 scale
//     words.  Scan: warp 0 issues two TMA tile copies of 256 rows (64-byte
//     swizzle) and one bulk copy of the scale words.  Pool: four producer
//     warps each gather 16 of the item's 64 blocks with cp.async (one warp
//     instruction per 512-byte block, the swizzle applied to the
//     destination) from the segment's pool ids held in shared memory; each
//     lane's copies arrive on the stage's barrier as they land
//     (cp.async.mbarrier.arrive), so the producers never wait for them.
//     Warp 0 also writes the item's B operand: the segment's indexer query
//     laid out "one 32-element block per output column" (column 4h+b holds
//     head h's block b, zeros elsewhere);
//   * warp 1 issues eight tcgen05.mma kind::mxf4 (M=128 positions, N=16,
//     K=64) with every block scale = 1: each accumulator is D/4 for an exact
//     integer |D| <= 4608, i.e. exact in fp32;
//   * two teams of four epilogue warps (alternate items) read the 16
//     accumulators of each position from TMEM, apply the E8M0 scales exactly
//     (fp32 when the block exponents are close, else the same fp64 sum as the
//     definition), combine the heads with the fp32 fma chain and emit rank
//     keys: the maximum of every 8 positions (scan) or one key per candidate
//     (pool; 0 for absent candidates), and add each key to its sequence's
//     histogram row for the selection that follows.
// Stages are recycled through mbarriers (smem ring of 4 for the scan, 6 for
// the pool gather; TMEM ring of 3).
// Every wait is time-bounded; on a timeout the kernel sets CSA2_DEV_TIMEOUT,
// drains its own copies and MMAs, frees TMEM and returns.
#include <mutex>

#include "device_common.cuh"
#include "sm100.cuh"

namespace csa2 {

namespace {

constexpr int kTile = 512;             // positions per work item
constexpr int kMT = kTile / 128;       // 128-row MMA tiles per item
// smem ring: 4 stages stream the contiguous scan fastest; the pool gather's
// small copies take longer to land, so it keeps more items in flight
template <bool kPool>
struct Ring {
  static constexpr int kStages = kPool ? 6 : 4;
};
constexpr int kAcc = 3;                // TMEM accumulator ring (16 columns per MMA tile)
constexpr int kAccCols = 16 * kMT;
constexpr int kTmemCols = 256;
constexpr uint32_t kSfCol = 192;       // scale factors (all 0x7F = 2^0) live here
constexpr int kEpiTeams = 2;           // epilogue teams of 4 warps, items round-robin
constexpr int kFirstExtra = 2 + 4 * kEpiTeams;  // first extra producer warp (pool mode)
constexpr int kPoolProducers = 4;      // pool mode: warps sharing the gather of an item
template <bool kPool>
constexpr int threads_of() {           // producer, MMA, epilogue (+ extra producer) warps
  return 32 * (kFirstExtra + (kPool ? kPoolProducers - 1 : 0));
}
constexpr uint32_t kCodeBytes = kTile * kIdxCodeBytes;
constexpr int kBoxRows = 256;          // TMA box height (scan)
constexpr int kPoolSlots = kTile / kBlk;  // pool blocks per item (64)
constexpr int kSlotsPerWarp = kPoolSlots / kPoolProducers;
static_assert(kSlotsPerWarp <= 32 && kPoolSlots % kPoolProducers == 0, "one pool slot per lane at most");
static_assert(kAcc * kAccCols <= int(kSfCol), "TMEM accumulators overlap the scale factors");

template <int kStages>
struct __align__(1024) ScanSmem {
  uint8_t a[kStages][kCodeBytes];      // code rows, 64-byte swizzled
  uint8_t bop[kStages][1024];          // B operand: 16 rows x 64 bytes, swizzled
  uint32_t sc[kStages][kTile];         // E8M0 scale words
  int32_t blk[kStages][kPoolSlots];    // pool mode: block id of each 8-row slot
  int2 info[kStages];                  // (segment, item index within the segment)
  uint64_t full[kStages];
  uint64_t empty[kStages];
  uint64_t tfull[kAcc];
  uint64_t tempty[kAcc];
  uint64_t done;
  uint32_t tmem_base;
  int abort_flag;
  int built[kStages];                  // segment whose B operand each stage holds
  // pool mode: each producer warp's share of the current segment's pool ids
  // (slot i of item j of warp w is pool entry 64 j + kSlotsPerWarp w + i)
  int32_t segpool[kPoolProducers][CSA2_MAX_POOL_BLOCKS / kPoolProducers];
};

struct ScanParams {
  const uint8_t* kcodes;      // code plane (pool gather)
  const uint8_t* kscales;
  const uint8_t* q_codes;
  const uint8_t* q_scales;
  const float* w;
  const int64_t* row_off;     // [S] or null -> row0
  int64_t row0;
  const int32_t* seg_eff;     // checked lengths, or null: computed from sd
  SegDesc sd;
  const int32_t* tile_start;  // scan: [S+1] item prefix
  int S;
  // scan outputs
  uint32_t* bkeys;
  int64_t nb_stride;
  float* scores;
  int64_t score_stride;
  // pool mode
  const int32_t* pool;        // [S][P]
  int P;
  int items_per_seg;
  uint32_t* ckeys;            // [S][P*8]
  uint32_t* hist;             // histogram rows of the emitted keys, or null:
                              // [S][kSelHistBins] (scan), [S][kCandHistBins] (pool)
  uint32_t* status;
};

// Whole warp: the same, with up to 128 prefix entries loaded at once (one
// round trip instead of a chain of them), also returning the segment's first
// item and the next segment's; longer prefixes fall back.
__device__ __forceinline__ int find_seq(const int32_t* tile_start, int S, int item);
__device__ __forceinline__ int find_seq_warp(const int32_t* tile_start, int S, int item, int& start, int& next) {
  if (S + 1 > 128) {
    const int b = find_seq(tile_start, S, item);
    start = __ldg(tile_start + b);
    next = __ldg(tile_start + b + 1);
    return b;
  }
  const int lane = threadIdx.x & 31;
  int32_t v[4];
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const int j = lane + 32 * r;
    v[r] = j <= S ? __ldg(tile_start + j) : INT32_MAX;
  }
  // the last j < S with tile_start[j] <= item (tile_start ascends, [0] = 0)
  int last = 0;
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const uint32_t m = __ballot_sync(0xffffffffu, lane + 32 * r < S && v[r] <= item);
    if (m) last = 32 * r + 31 - __clz(m);
  }
  auto entry = [&](int j) {  // tile_start[j] for j <= S (the same j in every lane)
    const int r = j >> 5;
    const int32_t x = r == 0 ? v[0] : r == 1 ? v[1] : r == 2 ? v[2] : v[3];
    return __shfl_sync(0xffffffffu, x, j & 31);
  };
  start = entry(last);
  next = entry(last + 1);
  return last;
}

__device__ __forceinline__ int find_seq(const int32_t* tile_start, int S, int item) {
  int lo = 0, hi = S;  // tile_start[lo] <= item < tile_start[hi]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (__ldg(tile_start + mid) <= item) lo = mid;
    else hi = mid;
  }
  return lo;
}

template <class Smem>
__device__ __forceinline__ void abort_kernel(Smem& sm, uint32_t* status) {
  set_status(status, CSA2_DEV_TIMEOUT);
  atomicExch(&sm.abort_flag, 1);
}

template <class Smem>
__device__ __forceinline__ bool aborted(Smem& sm) {
  return *reinterpret_cast<volatile int*>(&sm.abort_flag) != 0;
}

__device__ __forceinline__ int64_t seg_row_off(const ScanParams& p, int s) {
  return p.row_off ? p.row_off[s] : p.row0;
}

__device__ __forceinline__ int64_t seg_len(const ScanParams& p, int s) {
  return p.seg_eff ? int64_t(p.seg_eff[s]) : seg_len_checked(p.sd, s, p.status);
}

// Writes the B operand image of a segment's query into `bo` (whole warp).
__device__ __forceinline__ void build_b_operand(uint8_t* bo, uint2 qreg, int lane) {
  *reinterpret_cast<uint4*>(bo + lane * 32) = make_uint4(0, 0, 0, 0);
  *reinterpret_cast<uint4*>(bo + lane * 32 + 16) = make_uint4(0, 0, 0, 0);
  __syncwarp();
  const int head = lane >> 3, part = lane & 7, blk = part >> 1;
  const int n = head * 4 + blk;
  const int phys = n * 64 + ((blk ^ ((n >> 1) & 3)) << 4) + (part & 1) * 8;
  *reinterpret_cast<uint2*>(bo + phys) = qreg;
  sm100::fence_proxy_async_smem();  // generic writes -> MMA (async proxy) reads
}

template <bool kPool>
__global__ void __launch_bounds__(threads_of<kPool>(), 1)
    k_index_tc(const __grid_constant__ CUtensorMap tmap, ScanParams p) {
  constexpr int kStages = Ring<kPool>::kStages;
  using Smem = ScanSmem<kStages>;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  launch_dependents();

  // prologue (touches no global memory): barriers, tensor memory, unit scales
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      // pool: every producer lane arrives when its copies have landed, and
      // lane 0 of each producer warp once more after the warp's writes
      sm100::mbar_init(&sm.full[s], kPool ? kPoolProducers * 33 : 1);
      sm100::mbar_init(&sm.empty[s], 1 + 4);
    }
    for (int a = 0; a < kAcc; ++a) {
      sm100::mbar_init(&sm.tfull[a], 1);
      sm100::mbar_init(&sm.tempty[a], 4);
    }
    sm100::mbar_init(&sm.done, 1);
    sm.abort_flag = 0;
    sm100::fence_mbar_init();
    sm100::tma_prefetch_desc(&tmap);
  }
  if (warp == 1) {
    sm100::tmem_alloc(&sm.tmem_base, kTmemCols);
    sm100::tmem_relinquish();
  }
  sm100::tc_fence_before();
  __syncthreads();
  sm100::tc_fence_after();
  const uint32_t tmem = sm.tmem_base;

  // unit block scales for both operands: fill 64 scale-factor columns with 0x7F
  if (warp >= 2 && warp < 6) {
    const uint32_t lane_base = uint32_t(32 * (warp & 3)) << 16;
#pragma unroll
    for (int c = 0; c < 64; c += 8) sm100::tmem_st8_same(tmem + lane_base + kSfCol + c, 0x7F7F7F7Fu);
    sm100::tmem_st_wait();
  }
  sm100::tc_fence_before();
  __syncthreads();
  sm100::tc_fence_after();
  grid_wait();  // the item prefix, lengths, pool and histograms come from earlier kernels

  const int n_items = kPool ? p.S * p.items_per_seg : __ldg(p.tile_start + p.S);
  // wait limit of the pipeline (2 s unless a test sets it) and, in the scan
  // only, a test's request to withhold the first item's copies
  const PipeCtl ctl = pipe_ctl(p.status, 2000000000ull);
  const bool withhold = ctl.withhold && !kPool;
  const int i0 = int(int64_t(n_items) * blockIdx.x / gridDim.x);
  const int i1 = int(int64_t(n_items) * (blockIdx.x + 1) / gridDim.x);

  if (warp == 0 || warp >= kFirstExtra) {
    // ------------------------------------------------------------ producer(s)
    // pool mode: warp 0 and the extra warps each gather kSlotsPerWarp blocks of
    // every item; warp 0 alone writes the B operand and the item info
    const int pw = warp == 0 ? 0 : warp - kFirstExtra + 1;
    int issued = 0;
    if (warp == 0 && lane < kStages) sm.built[lane] = -1;
    __syncwarp();
    if (i0 < i1) {
      int b, seq_start = 0, next_start = 0;
      if (kPool) {
        b = i0 / p.items_per_seg;
      } else {
        b = find_seq_warp(p.tile_start, p.S, i0, seq_start, next_start);
      }
      int64_t seq_off = seg_row_off(p, b);
      int64_t seq_len = seg_len(p, b);
      int qb = -1;
      uint2 qreg = make_uint2(0, 0);
      int pool_seg = -1;  // segment whose pool ids are in sm.segpool
      for (int it = i0; it < i1; ++it) {
        const int t = it - i0, s = t % kStages, round = t / kStages;
        int j;
        if (kPool) {
          const int nb = it / p.items_per_seg;
          if (nb != b) {
            b = nb;
            seq_off = seg_row_off(p, b);
            seq_len = seg_len(p, b);
          }
          j = it - b * p.items_per_seg;
        } else {
          while (it >= next_start) {
            ++b;
            seq_start = next_start;
            next_start = __ldg(p.tile_start + b + 1);
            seq_off = seg_row_off(p, b);
            seq_len = seg_len(p, b);
          }
          j = it - seq_start;
        }
        const bool ok = round == 0 || sm100::mbar_wait(&sm.empty[s], (round - 1) & 1, ctl.wait_ns);
        if (!__all_sync(0xffffffffu, ok)) {
          if (lane == 0) abort_kernel(sm, p.status);
          break;
        }
        if (__any_sync(0xffffffffu, aborted(sm))) break;
        // pool mode, new segment: this warp's share of its pool ids (one
        // round trip per segment, in flight with the query's codes below);
        // copies already issued carry their own addresses
        constexpr int kPer = CSA2_MAX_POOL_BLOCKS / kPoolProducers / 32;
        int32_t v[kPer];
        const bool new_pool = kPool && pool_seg != b;
        if (new_pool) {
          const int32_t* src = p.pool + int64_t(b) * p.P;
#pragma unroll
          for (int m = 0; m < kPer; ++m) {
            const int e = lane + 32 * m;  // entry (item e / kSlotsPerWarp, slot e % kSlotsPerWarp)
            const int slot = (e / kSlotsPerWarp) * kPoolSlots + pw * kSlotsPerWarp + e % kSlotsPerWarp;
            v[m] = slot < p.P ? __ldg(src + slot) : -1;
          }
        }
        if (pw == 0 && sm.built[s] != b) {
          if (qb != b) {
            qreg = __ldg(reinterpret_cast<const uint2*>(p.q_codes + int64_t(b) * kHi * 64) + lane);
            qb = b;
          }
          build_b_operand(sm.bop[s], qreg, lane);
          __syncwarp();
          if (lane == 0) sm.built[s] = b;
        }
        __syncwarp();
        if (kPool) {
          if (new_pool) {
#pragma unroll
            for (int m = 0; m < kPer; ++m) sm.segpool[pw][lane + 32 * m] = v[m];
            __syncwarp();
            pool_seg = b;
          }
          // lane i < kSlotsPerWarp owns slot pw * kSlotsPerWarp + i of the item
          // (block id and first cache row; -1 = absent)
          int32_t my = -1;
          int64_t myrow = -1;
          if (lane < kSlotsPerWarp) {
            const int32_t bk = sm.segpool[pw][j * kSlotsPerWarp + lane];
            const bool in_range = bk >= 0 && int64_t(bk) * kBlk < seq_len;
            if (bk >= 0 && !in_range) set_status(p.status, CSA2_DEV_INDEX_RANGE);
            my = in_range ? bk : -1;
            if (in_range) myrow = p.sd.pages ? seg_row(p.sd, b, int64_t(bk) * kBlk, p.status) : seq_off + int64_t(bk) * kBlk;
            sm.blk[s][pw * kSlotsPerWarp + lane] = my;
          }
          if (pw == 0 && lane == 0) sm.info[s] = make_int2(b, j);
          // one warp instruction per 512-byte block: lane = (row l/4, chunk l%4),
          // destination in the 64-byte swizzle the MMA descriptor expects
          const int r8 = lane >> 2, ch = lane & 3;
          const int phys = r8 * 64 + ((ch ^ ((r8 >> 1) & 3)) << 4);
          const uint8_t* kbase = p.kcodes + lane * 16;
          uint8_t* abase = sm.a[s] + pw * kSlotsPerWarp * kBlk * kIdxCodeBytes + phys;
#pragma unroll
          for (int i = 0; i < kSlotsPerWarp; ++i) {
            const int64_t row = __shfl_sync(0xffffffffu, myrow, i);
            if (row >= 0) sm100::cp_async16(abase + i * kBlk * kIdxCodeBytes, kbase + row * kIdxCodeBytes);
          }
          // scales: 32 bytes per block, two 16-byte chunks
#pragma unroll
          for (int c0 = 0; c0 < 2 * kSlotsPerWarp; c0 += 32) {
            const int c = c0 + lane, i = (c >> 1) & 31;
            const int64_t row = __shfl_sync(0xffffffffu, myrow, i);
            if (c < 2 * kSlotsPerWarp && row >= 0)
              sm100::cp_async16(&sm.sc[s][(pw * kSlotsPerWarp + i) * kBlk + 4 * (c & 1)],
                                p.kscales + row * 4 + 16 * (c & 1));
          }
          // the stage completes once every lane's copies have landed and
          // lane 0 has arrived after the warp's generic writes (slot blocks,
          // item info, B operand: fenced for the async proxy); the MMA thread
          // fences the landed copies itself after its wait
          sm100::cp_async_mbar_arrive_noinc(&sm.full[s]);
          sm100::fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) sm100::mbar_arrive(&sm.full[s]);
        } else if (lane == 0) {
          sm.info[s] = make_int2(b, j);
          const int64_t rem_rows = seq_len - int64_t(j) * kTile;
          const int rows_valid = rem_rows < kTile ? int(rem_rows) : kTile;
          const uint32_t sbytes = uint32_t((rows_valid + 7) & ~7) * 4u;
          // an item never crosses a page (pages hold a multiple of kTile rows)
          const int64_t row0 =
              p.sd.pages ? seg_row(p.sd, b, int64_t(j) * kTile, p.status) : seq_off + int64_t(j) * kTile;
          if (!(withhold && t == 0)) {  // (a test withholds item 0: stage 0 never fills)
            sm100::mbar_arrive_expect_tx(&sm.full[s], kCodeBytes + sbytes);
#pragma unroll
            for (int bx = 0; bx < kTile / kBoxRows; ++bx)
              sm100::tma_load_2d(sm.a[s] + bx * kBoxRows * kIdxCodeBytes, &tmap, 0, int32_t(row0 + bx * kBoxRows),
                                 &sm.full[s]);
            sm100::bulk_load(sm.sc[s], p.kscales + row0 * 4, sbytes, &sm.full[s]);
          }
        }
        ++issued;
      }
      if (kPool) sm100::cp_async_wait<0>();  // (landed already once the MMA consumed every stage)
    }
    // drain: every copy this warp issued has landed before the CTA exits (a
    // withheld item 0 leaves stage 0 without copies: it is never refilled,
    // since that needs item 0 consumed first)
    if (lane == 0)
      for (int s = 0; s < kStages && s < issued; ++s) {
        if (withhold && s == 0) continue;
        const int last_round = (issued - 1 - s) / kStages;
        if (!sm100::mbar_wait(&sm.full[s], last_round & 1, 200000000ull)) set_status(p.status, CSA2_DEV_TIMEOUT);
      }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = sm100::idesc_mxf4(128, 16);
      const uint32_t sfa = tmem + kSfCol, sfb = tmem + kSfCol + 32;
      for (int it = i0; it < i1; ++it) {
        const int t = it - i0, s = t % kStages, a = t % kAcc;
        if (!sm100::mbar_wait(&sm.full[s], (t / kStages) & 1, ctl.wait_ns)) {
          abort_kernel(sm, p.status);
          break;
        }
        if (t >= kAcc && !sm100::mbar_wait(&sm.tempty[a], ((t / kAcc) - 1) & 1, ctl.wait_ns)) {
          abort_kernel(sm, p.status);
          break;
        }
        if (aborted(sm)) break;
        // pool: the gathered rows were written by cp.async (generic proxy);
        // the barrier made them visible here, the fence orders them before
        // this thread's tensor-core (async proxy) reads
        if (kPool) sm100::fence_proxy_async_smem();
        sm100::tc_fence_after();
        const uint32_t abase = sm100::smem_u32(sm.a[s]);
        const uint32_t bbase = sm100::smem_u32(sm.bop[s]);
#pragma unroll
        for (int half = 0; half < kMT; ++half)
#pragma unroll
          for (int kk = 0; kk < 2; ++kk)
            sm100::mma_mxf4(tmem + a * kAccCols + half * 16, sm100::smem_desc_k64b(abase + half * 8192 + kk * 32),
                            sm100::smem_desc_k64b(bbase + kk * 32), idesc, uint32_t(kk), sfa, sfb);
        sm100::mma_commit(&sm.empty[s]);
        sm100::mma_commit(&sm.tfull[a]);
      }
      // all MMAs of this CTA complete before TMEM is released
      sm100::mma_commit(&sm.done);
      if (!sm100::mbar_wait(&sm.done, 0, 200000000ull)) set_status(p.status, CSA2_DEV_TIMEOUT);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int g = warp & 3;  // TMEM lane quarter of this warp
    const int team = (warp - 2) >> 2;
    const uint32_t lane_base = uint32_t(32 * g) << 16;
    int cur = -1;
    int64_t L = 0;
    IdxQCtx qc;
    for (int it = i0 + team; it < i1; it += kEpiTeams) {
      const int t = it - i0, s = t % kStages, a = t % kAcc;
      const bool ok = sm100::mbar_wait(&sm.full[s], (t / kStages) & 1, ctl.wait_ns) &&
                      sm100::mbar_wait(&sm.tfull[a], (t / kAcc) & 1, ctl.wait_ns);
      if (!__all_sync(0xffffffffu, ok)) {
        if (lane == 0) abort_kernel(sm, p.status);
        break;
      }
      if (__any_sync(0xffffffffu, aborted(sm))) break;
      sm100::tc_fence_after();
      const int2 inf = sm.info[s];
      if (inf.x != cur) {
        cur = inf.x;
        L = seg_len(p, cur);
        make_qctx(qc, p.q_scales + int64_t(cur) * 16, p.w + int64_t(cur) * kHi);
      }
      uint32_t swv[kMT];
      int64_t posv[kMT];
      uint32_t v[kMT][16];
#pragma unroll
      for (int half = 0; half < kMT; ++half) {
        const int pl = 128 * half + 32 * g + lane;  // position within the item
        swv[half] = sm.sc[s][pl];
        if (kPool) {
          const int32_t bk = sm.blk[s][pl >> 3];
          posv[half] = bk >= 0 ? int64_t(bk) * kBlk + (pl & 7) : int64_t(-1);
        } else {
          posv[half] = int64_t(inf.y) * kTile + pl;
        }
        sm100::tmem_ld16(tmem + lane_base + a * kAccCols + half * 16, v[half]);
      }
      sm100::tmem_ld_wait();
      sm100::tc_fence_before();
      sm100::fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        sm100::mbar_arrive(&sm.empty[s]);
        sm100::mbar_arrive(&sm.tempty[a]);
      }
#pragma unroll
      for (int half = 0; half < kMT; ++half) {
        const int64_t pos = posv[half];
        const uint32_t sw = swv[half];
        float sc = 0.0f;
        uint32_t key = 0;
        if (pos >= 0 && pos < L) {
          sc = exact_score(v[half], sw, qc);
          key = rank_key(sc);
          if (!kPool && p.scores) p.scores[int64_t(cur) * p.score_stride + pos] = sc;
        }
        if (kPool) {
          const int64_t ci = int64_t(inf.y) * kTile + 128 * half + 32 * g + lane;  // candidate index
          if (ci < int64_t(p.P) * kBlk) {
            p.ckeys[int64_t(cur) * p.P * kBlk + ci] = key;
            if (p.hist && key != 0u)
              atomicAdd(p.hist + int64_t(cur) * kCandHistBins + (key >> (32 - kCandHistBits)), 1u);
          }
        } else {
          key = group8_max(key);
          if ((lane & 7) == 0 && pos < L) {
            p.bkeys[int64_t(cur) * p.nb_stride + pos / kBlk] = key;
            if (p.hist && key != 0u) atomicAdd(p.hist + int64_t(cur) * kSelHistBins + (key >> (32 - kSelHistBits)), 1u);
          }
        }
      }
    }
  }

  sm100::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    sm100::tc_fence_after();
    sm100::tmem_dealloc(tmem, kTmemCols);
  }
}

// Effective lengths and the exclusive prefix of work items per segment
// (one CTA of 1024 threads, any S).
__global__ void __launch_bounds__(1024) k_seg_prep(SegDesc sd, int S, int32_t* seg_eff, int32_t* tile_start,
                                                    uint32_t* status) {
  __shared__ int32_t warp_sums[32];
  __shared__ int32_t carry;
  launch_dependents();
  grid_wait();
  if (threadIdx.x == 0) carry = 0;
  __syncthreads();
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  for (int base = 0; base < S; base += 1024) {
    const int s = base + threadIdx.x;
    int32_t ntile = 0;
    if (s < S) {
      const int64_t L = seg_len_checked(sd, s, status);
      seg_eff[s] = int32_t(L);
      ntile = int32_t((L + kTile - 1) / kTile);
    }
    int32_t x = ntile;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int32_t y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) warp_sums[wid] = x;
    __syncthreads();
    if (wid == 0) {
      const int32_t ws = warp_sums[lane];
      int32_t z = ws;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int32_t y = __shfl_up_sync(0xffffffffu, z, o);
        if (lane >= o) z += y;
      }
      warp_sums[lane] = z - ws;
    }
    __syncthreads();
    const int32_t excl = carry + warp_sums[wid] + x - ntile;
    if (s < S) tile_start[s] = excl;
    __syncthreads();
    if (threadIdx.x == 1023) carry = excl + ntile;
    __syncthreads();
  }
  if (threadIdx.x == 0) tile_start[S] = carry;
}

}  // namespace

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(f);
  });
  return fn;
}

// Tensor map over the indexer-K code plane: rows of 64 bytes, box of
// `box_rows` rows, 64-byte swizzle, out-of-range rows read as zero.
csa2_status code_map(CUtensorMap* map, const uint8_t* kcodes, int64_t rows, int box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return fail(CSA2_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
  const cuuint64_t dims[2] = {cuuint64_t(kIdxCodeBytes), cuuint64_t(rows)};
  const cuuint64_t strides[1] = {cuuint64_t(kIdxCodeBytes)};
  const cuuint32_t box[2] = {cuuint32_t(kIdxCodeBytes), cuuint32_t(box_rows)};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(kcodes), dims, strides, box,
                         estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(CSA2_ERR_CUDA, "cuTensorMapEncodeTiled failed for the indexer-K codes");
  return CSA2_OK;
}

int num_sms() {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return sms;
}

namespace {

template <bool kPool>
void launch_index_tc(const CUtensorMap& map, const ScanParams& p, int64_t max_items, cudaStream_t st) {
  const size_t smem = sizeof(ScanSmem<Ring<kPool>::kStages>) + 1024;
  cudaFuncSetAttribute(k_index_tc<kPool>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  const int grid = int(std::min<int64_t>(num_sms(), std::max<int64_t>(max_items, 1)));
  launch_k(k_index_tc<kPool>, dim3(grid), dim3(threads_of<kPool>()), smem, st, map, p);
}

}  // namespace

size_t scan_tc_prefix_ints(int S) { return size_t(S) + 1; }

csa2_status launch_scan_tc(const uint8_t* kcodes, const uint8_t* kscales, const SegDesc& sd, int32_t* seg_eff,
                           int32_t* tile_start, int S, const uint8_t* q_codes, const uint8_t* q_scales,
                           const float* w, uint32_t* bkeys, int64_t nb_stride, float* scores, int64_t score_stride,
                           uint32_t* hist, uint32_t* status, cudaStream_t st) {
  if (S == 0) return CSA2_OK;
  launch_k(k_seg_prep, dim3(1), dim3(1024), 0, st, sd, S, seg_eff, tile_start, status);
  if (sd.max_len == 0) return CSA2_OK;
  CUtensorMap map;
  const csa2_status rc = code_map(&map, kcodes, sd.cache_rows, kBoxRows);
  if (rc != CSA2_OK) return rc;
  ScanParams p{};
  p.kscales = kscales;
  p.q_codes = q_codes;
  p.q_scales = q_scales;
  p.w = w;
  p.row_off = sd.row_off;
  p.row0 = sd.row0;
  p.seg_eff = seg_eff;
  p.sd = sd;
  p.tile_start = tile_start;
  p.S = S;
  p.bkeys = bkeys;
  p.nb_stride = nb_stride;
  p.scores = scores;
  p.score_stride = score_stride;
  p.hist = hist;
  p.status = status;
  // the host cannot see the item count; cap the grid by an upper bound of it
  launch_index_tc<false>(map, p, int64_t(S) * ((sd.max_len + kTile - 1) / kTile), st);
  return CSA2_OK;
}

csa2_status launch_pool_tc(const uint8_t* kcodes, const uint8_t* kscales, const SegDesc& sd, const int32_t* seg_eff,
                           int S, const uint8_t* q_codes, const uint8_t* q_scales, const float* w,
                           const int32_t* pool, int P, uint32_t* ckeys, uint32_t* hist, uint32_t* status,
                           cudaStream_t st) {
  if (S == 0) return CSA2_OK;
  CUtensorMap map;
  const csa2_status rc = code_map(&map, kcodes, sd.cache_rows, kBlk);
  if (rc != CSA2_OK) return rc;
  ScanParams p{};
  p.kcodes = kcodes;
  p.kscales = kscales;
  p.q_codes = q_codes;
  p.q_scales = q_scales;
  p.w = w;
  p.row_off = sd.row_off;
  p.row0 = sd.row0;
  p.seg_eff = seg_eff;
  p.sd = sd;
  p.S = S;
  p.pool = pool;
  p.P = P;
  p.items_per_seg = (P * kBlk + kTile - 1) / kTile;
  p.ckeys = ckeys;
  p.hist = hist;
  p.status = status;
  launch_index_tc<true>(map, p, int64_t(S) * p.items_per_seg, st);
  return CSA2_OK;
}

}  // namespace csa2
