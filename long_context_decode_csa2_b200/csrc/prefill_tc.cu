// Causal multi-query indexer scan for prefill on the 5th-generation tensor
// cores (sm_100a): the block-scaled FP4 GEMM of T indexer queries (4 heads x
// 128) against the visible indexer-K rows of one sequence, reduced to block
// maxima per query.
//
// Source: "DeepSeek-V4.1-Flash: Pushing the Limits of KV Cache Compression",
// section "三个方向一起压小缓存" (FP4 indexer q/k; every 8 positions reduced to
// their best score; pool of at most 2048 blocks), with the causal visibility
// of compressed entries to raw query positions (section "后 20 层干脆共用一份
// KV": m raw tokens per entry).
//
// Work item = (group of 8 consecutive queries, tile of 128 positions); items
// run group-major, so a persistent CTA keeps one group's B operand for many
// key tiles.  Per item:
//   * warp 0 loads the tile's 128 code rows with one TMA tile copy (64-byte
//     swizzle) and its 128 scale words with a bulk copy; when the group
//     changes it also writes the group's B operand, 128 rows of which row
//     16j + 4h + b holds block b of head h of query j (zeros elsewhere), and
//     the queries' scale contexts;
//   * warp 1 issues two tcgen05.mma kind::mxf4 (M = 128 positions, N = 128,
//     K = 64) with every block scale = 1, so each accumulator is an exact
//     block dot D/4;
//   * four teams of four epilogue warps (two of the eight queries each) read
//     each position's 16 accumulators per query, form the exact score (the
//     same rounding as the decode scan), mask positions the query cannot see,
//     and write the maximum of every 8 positions as one rank key.
// Items past the visibility of every query of a group are skipped by all
// roles alike.  Every wait is time-bounded (CSA2_DEV_TIMEOUT on expiry).
//
// The same kernel serves a batch of sequences with a few queries each (the
// candidate tokens of a speculative-decoding verification step, section
// "DSpark" of the same page: several positions per request scored in one
// forward): a group is then up to 8 consecutive queries of one sequence,
// read from a group table that k_multi_prep builds, and every item loads its
// group's own sequence rows.
#include <algorithm>
#include <cstddef>

#include "device_common.cuh"
#include "sm100.cuh"

namespace csa2 {

namespace {

constexpr int kQG = 8;                   // queries per group
constexpr int kN = 16 * kQG;             // MMA N: 4 heads x 4 blocks per query
constexpr int kPT = 128;                 // positions per item (MMA M)
constexpr int kSt = 6;                   // smem ring
constexpr int kAc = 3;                   // TMEM accumulator ring, kN columns each
constexpr int kTmemCols = 512;
constexpr uint32_t kSf = 448;            // scale-factor columns (all 2^0)
constexpr int kTeams = 4;                // epilogue teams of 4 warps, all on every item
constexpr int kQPT = kQG / kTeams;       // queries per team and item
constexpr int kEpiWarps = 4 * kTeams;
constexpr int kThr = 64 + 32 * kEpiWarps;  // producer, MMA, epilogue warps
constexpr uint32_t kTileBytes = kPT * kIdxCodeBytes;
static_assert(kAc * kN <= int(kSf), "TMEM accumulators overlap the scale factors");

struct __align__(16) QCtxS {
  IdxQCtx c;
  int vis;  // visible entries of this query (0 past the end of the batch)
};
static_assert(sizeof(QCtxS) == 96, "QCtxS is read as six 16-byte words");

// One query's context from shared memory in six 16-byte loads.
__device__ __forceinline__ QCtxS load_qctx(const QCtxS& src) {
  QCtxS q;
  const uint4* s4 = reinterpret_cast<const uint4*>(&src);
  uint4* d4 = reinterpret_cast<uint4*>(&q);
#pragma unroll
  for (int i = 0; i < 6; ++i) d4[i] = s4[i];
  return q;
}

struct __align__(1024) PfSmem {
  uint8_t a[kSt][kTileBytes];           // code rows, 64-byte swizzled
  uint8_t bop[kSt][kN * kIdxCodeBytes]; // B operand of the stage's group
  uint32_t sc[kSt][kPT];                // E8M0 scale words of the rows
  int2 info[kSt];                       // (group, tile)
  QCtxS qctx[kSt][kQG];
  uint64_t full[kSt];
  uint64_t empty[kSt];
  uint64_t tfull[kAc];
  uint64_t tempty[kAc];
  uint64_t done;
  uint32_t tmem_base;
  int abort_flag;
  int built[kSt];                       // group whose B operand each stage holds
};
// alignment the copies need: TMA tiles and MMA operands (1024 bytes, 64-byte
// swizzle), bulk-copy destinations (16 bytes)
static_assert(offsetof(PfSmem, a) % 1024 == 0 && kTileBytes % 1024 == 0, "code tiles misaligned");
static_assert(offsetof(PfSmem, bop) % 1024 == 0 && (kN * kIdxCodeBytes) % 1024 == 0, "B operand misaligned");
static_assert(offsetof(PfSmem, sc) % 16 == 0 && (kPT * 4) % 16 == 0, "bulk-copy destination misaligned");
static_assert(offsetof(PfSmem, full) % 8 == 0, "mbarriers misaligned");

struct PfParams {
  const int4* groups;       // [n_groups] {sequence, first query, queries, 0}, or null: group g = queries 8g..
  const int64_t* seq_row_off;  // [B] first cache row of each sequence (with groups)
  const uint8_t* kscales;
  const uint8_t* q_codes;   // [T][4][64]
  const uint8_t* q_scales;  // [T][4][4]
  const float* w;           // [T][4]
  const int32_t* vis;       // [T]
  int T;
  int64_t row0;
  int64_t cache_rows;
  int n_groups;             // groups (with a group table: its capacity)
  const int32_t* n_groups_dev;  // with a group table: the groups k_multi_prep wrote, or null
  int n_tiles;
  uint32_t* bkeys;          // [T][nb_stride]
  int64_t nb_stride;
  uint32_t* status;
};

__device__ __forceinline__ void pf_abort(PfSmem& sm, uint32_t* status) {
  set_status(status, CSA2_DEV_TIMEOUT);
  atomicExch(&sm.abort_flag, 1);
}
__device__ __forceinline__ bool pf_aborted(PfSmem& sm) {
  return *reinterpret_cast<volatile int*>(&sm.abort_flag) != 0;
}

// Queries and cache rows of group g.
struct GroupRef {
  int q0, nq;
  int64_t row0;
};
__device__ __forceinline__ GroupRef group_ref(const PfParams& p, int g) {
  if (p.groups) {
    const int4 e = __ldg(p.groups + g);
    return GroupRef{e.y, e.z, e.z > 0 ? __ldg(p.seq_row_off + e.x) : 0};
  }
  const int q0 = g * kQG;
  return GroupRef{q0, min(kQG, p.T - q0), p.row0};
}

// Largest visibility among the group's queries.
__device__ __forceinline__ int group_vis(const PfParams& p, const GroupRef& gr) {
  int m = 0;
  for (int j = 0; j < gr.nq; ++j) m = max(m, __ldg(p.vis + gr.q0 + j));
  return m;
}

// Writes group g's B operand and scale contexts into stage s (whole warp).
__device__ __forceinline__ void build_group(PfSmem& sm, int s, const PfParams& p, const GroupRef& gr, int lane) {
  uint8_t* bo = sm.bop[s];
#pragma unroll
  for (int m = 0; m < kN * kIdxCodeBytes / 16 / 32; ++m)
    *reinterpret_cast<uint4*>(bo + 16 * (lane + 32 * m)) = make_uint4(0, 0, 0, 0);
  __syncwarp();
  // 128 chunks of 16 bytes: chunk c = (query j, head h, block b), 4 per lane
#pragma unroll
  for (int m = 0; m < kN / 32; ++m) {
    const int c = lane + 32 * m;
    const int j = c >> 4, h = (c >> 2) & 3, b = c & 3;
    const int qi = gr.q0 + j;
    if (j < gr.nq) {
      const uint4 v = __ldg(reinterpret_cast<const uint4*>(p.q_codes + int64_t(qi) * kHi * 64 + h * 64 + b * 16));
      const int n = 16 * j + 4 * h + b;
      *reinterpret_cast<uint4*>(bo + n * 64 + ((b ^ ((n >> 1) & 3)) << 4)) = v;
    }
  }
  if (lane < kQG) {
    const int qi = gr.q0 + lane;
    QCtxS& q = sm.qctx[s][lane];
    if (lane < gr.nq) {
      make_qctx(q.c, p.q_scales + int64_t(qi) * 16, p.w + int64_t(qi) * kHi);
      q.vis = __ldg(p.vis + qi);
    } else {
      const uint8_t unit[16] = {127, 127, 127, 127, 127, 127, 127, 127, 127, 127, 127, 127, 127, 127, 127, 127};
      const float zero[4] = {0.f, 0.f, 0.f, 0.f};
      make_qctx(q.c, unit, zero);
      q.vis = 0;
    }
  }
  sm100::fence_proxy_async_smem();  // generic writes -> MMA (async proxy) reads
  __syncwarp();
}

__global__ void __launch_bounds__(kThr, 1) k_prefill_tc(const __grid_constant__ CUtensorMap tmap, PfParams p) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  PfSmem& sm = *reinterpret_cast<PfSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  launch_dependents();

  // prologue (touches no global memory): barriers, tensor memory, unit scales
  if (threadIdx.x == 0) {
    for (int s = 0; s < kSt; ++s) {
      sm100::mbar_init(&sm.full[s], 1);
      sm100::mbar_init(&sm.empty[s], 1 + kEpiWarps);
    }
    for (int a = 0; a < kAc; ++a) {
      sm100::mbar_init(&sm.tfull[a], 1);
      sm100::mbar_init(&sm.tempty[a], kEpiWarps);
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
  if (warp >= 2 && warp < 6) {  // unit block scales in columns kSf .. kSf+63
    const uint32_t lane_base = uint32_t(32 * (warp & 3)) << 16;
#pragma unroll
    for (int c = 0; c < 64; c += 8) sm100::tmem_st8_same(tmem + lane_base + kSf + c, 0x7F7F7F7Fu);
    sm100::tmem_st_wait();
  }
  sm100::tc_fence_before();
  __syncthreads();
  sm100::tc_fence_after();
  grid_wait();  // the group table, visible counts and queries come from earlier kernels

  // items are split over the groups that exist (the table's capacity is a
  // host bound; empty entries past the real count would idle their CTAs)
  const int n_groups = p.n_groups_dev ? min(p.n_groups, max(0, __ldg(p.n_groups_dev))) : p.n_groups;
  const int n_items = n_groups * p.n_tiles;
  // wait limit of the pipeline (2 s unless a test sets it); a test may also
  // have the producer withhold its first item's copies
  const PipeCtl ctl = pipe_ctl(p.status, 2000000000ull);
  const int i0 = int(int64_t(n_items) * blockIdx.x / gridDim.x);
  const int i1 = int(int64_t(n_items) * (blockIdx.x + 1) / gridDim.x);

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane < kSt) sm.built[lane] = -1;
    __syncwarp();
    int issued = 0, cg = -1, gmax = 0;
    GroupRef gr{0, 0, 0};
    for (int it = i0; it < i1; ++it) {
      const int g = it / p.n_tiles, tile = it - g * p.n_tiles;
      if (g != cg) {
        cg = g;
        gr = group_ref(p, g);
        gmax = group_vis(p, gr);
      }
      if (int64_t(tile) * kPT >= gmax) continue;
      const int t = issued, s = t % kSt, round = t / kSt;
      const bool ok = round == 0 || sm100::mbar_wait_sleep(&sm.empty[s], (round - 1) & 1, ctl.wait_ns);
      if (!__all_sync(0xffffffffu, ok)) {
        if (lane == 0) pf_abort(sm, p.status);
        break;
      }
      if (__any_sync(0xffffffffu, pf_aborted(sm))) break;
      if (sm.built[s] != g) {
        build_group(sm, s, p, gr, lane);
        if (lane == 0) sm.built[s] = g;
      }
      __syncwarp();
      if (lane == 0) {
        sm.info[s] = make_int2(g, tile);
        const int64_t row = gr.row0 + int64_t(tile) * kPT;
        const int64_t left = p.cache_rows - row;  // > 0 and a multiple of 8
        const uint32_t sbytes = uint32_t(left < kPT ? left : kPT) * 4u;
        if (!(ctl.withhold && t == 0)) {  // (a test withholds item 0: stage 0 never fills)
          sm100::mbar_arrive_expect_tx(&sm.full[s], kTileBytes + sbytes);
          sm100::tma_load_2d(sm.a[s], &tmap, 0, int32_t(row), &sm.full[s]);
          sm100::bulk_load(sm.sc[s], p.kscales + row * 4, sbytes, &sm.full[s]);
        }
      }
      ++issued;
    }
    // every copy this warp issued has landed before the CTA exits (a withheld
    // item 0 leaves stage 0 without copies; it is never refilled)
    if (lane == 0)
      for (int s = 0; s < kSt && s < issued; ++s) {
        if (ctl.withhold && s == 0) continue;
        const int last_round = (issued - 1 - s) / kSt;
        if (!sm100::mbar_wait_sleep(&sm.full[s], last_round & 1, 200000000ull)) set_status(p.status, CSA2_DEV_TIMEOUT);
      }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = sm100::idesc_mxf4(kPT, kN);
      const uint32_t sfa = tmem + kSf, sfb = tmem + kSf + 32;
      int t = 0, cg = -1, gmax = 0;
      for (int it = i0; it < i1; ++it) {
        const int g = it / p.n_tiles, tile = it - g * p.n_tiles;
        if (g != cg) {
          cg = g;
          gmax = group_vis(p, group_ref(p, g));
        }
        if (int64_t(tile) * kPT >= gmax) continue;
        const int s = t % kSt, a = t % kAc;
        if (!sm100::mbar_wait_sleep(&sm.full[s], (t / kSt) & 1, ctl.wait_ns)) {
          pf_abort(sm, p.status);
          break;
        }
        if (t >= kAc && !sm100::mbar_wait_sleep(&sm.tempty[a], ((t / kAc) - 1) & 1, ctl.wait_ns)) {
          pf_abort(sm, p.status);
          break;
        }
        if (pf_aborted(sm)) break;
        sm100::tc_fence_after();
        const uint32_t abase = sm100::smem_u32(sm.a[s]);
        const uint32_t bbase = sm100::smem_u32(sm.bop[s]);
#pragma unroll
        for (int kk = 0; kk < 2; ++kk)
          sm100::mma_mxf4(tmem + a * kN, sm100::smem_desc_k64b(abase + kk * 32), sm100::smem_desc_k64b(bbase + kk * 32),
                          idesc, uint32_t(kk), sfa, sfb);
        sm100::mma_commit(&sm.empty[s]);
        sm100::mma_commit(&sm.tfull[a]);
        ++t;
      }
      sm100::mma_commit(&sm.done);  // all MMAs complete before TMEM is released
      if (!sm100::mbar_wait_sleep(&sm.done, 0, 200000000ull)) set_status(p.status, CSA2_DEV_TIMEOUT);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int q4 = warp & 3;  // TMEM lane quarter of this warp
    const int team = (warp - 2) >> 2;
    const int j0 = team * kQPT;  // this team's queries of the group
    const uint32_t lane_base = uint32_t(32 * q4) << 16;
    int t = -1, cg = -1, gmax = 0;
    GroupRef gr{0, 0, 0};
    for (int it = i0; it < i1; ++it) {
      const int g = it / p.n_tiles, tile = it - g * p.n_tiles;
      if (g != cg) {
        cg = g;
        gr = group_ref(p, g);
        gmax = group_vis(p, gr);
      }
      if (int64_t(tile) * kPT >= gmax) continue;
      ++t;
      const int s = t % kSt, a = t % kAc;
      const bool ok = sm100::mbar_wait_sleep(&sm.full[s], (t / kSt) & 1, ctl.wait_ns) &&
                      sm100::mbar_wait_sleep(&sm.tfull[a], (t / kAc) & 1, ctl.wait_ns);
      if (!__all_sync(0xffffffffu, ok)) {
        if (lane == 0) pf_abort(sm, p.status);
        break;
      }
      if (__any_sync(0xffffffffu, pf_aborted(sm))) break;
      sm100::tc_fence_after();
      const int pl = 32 * q4 + lane;
      const int64_t pos = int64_t(tile) * kPT + pl;
      const KeyScale ks = key_scale(sm.sc[s][pl]);
      const uint32_t tcol = tmem + lane_base + uint32_t(a * kN);
      uint32_t v[kQPT][16];
#pragma unroll
      for (int jj = 0; jj < kQPT; ++jj) sm100::tmem_ld16(tcol + 16 * (j0 + jj), v[jj]);
#pragma unroll
      for (int jj = 0; jj < kQPT; ++jj) sm100::tmem_ld_wait(v[jj]);
#pragma unroll
      for (int jj = 0; jj < kQPT; ++jj) {
        const int j = j0 + jj;
        const QCtxS q = load_qctx(sm.qctx[s][j]);
        uint32_t key = 0;
        if (pos < q.vis) key = rank_key(exact_score(v[jj], ks, q.c));
        key = group8_max(key);
        if ((lane & 7) == 0 && pos < q.vis)
          p.bkeys[int64_t(gr.q0 + j) * p.nb_stride + pos / kBlk] = key;
      }
      sm100::tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        sm100::mbar_arrive(&sm.empty[s]);
        sm100::mbar_arrive(&sm.tempty[a]);
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

// Group table and per-query rows of a batch of sequences with a few queries
// each (one CTA of 1024 threads).  Sequence b owns queries q_off[b] ..
// q_off[b+1]-1, cut into groups of at most 8; every query gets its
// sequence's first row and its checked visible count (negative -> 0, above
// max_vis -> clamped with CSA2_DEV_LENGTH, outside the cache ->
// 0 with CSA2_DEV_ROW_LAYOUT); queries of no sequence see nothing.
__global__ void __launch_bounds__(1024) k_multi_prep(const int64_t* seq_row_off, const int32_t* q_off,
                                                     const int32_t* q_vis, int B, int Q, int G, int64_t max_vis,
                                                     int64_t cache_rows, int4* groups, int64_t* q_row_off,
                                                     int32_t* vis, int32_t* n_groups, uint32_t* status) {
  __shared__ int32_t warp_sums[32];
  __shared__ int32_t carry;
  launch_dependents();
  grid_wait();
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  for (int q = threadIdx.x; q < Q; q += blockDim.x) {
    vis[q] = 0;
    q_row_off[q] = 0;
  }
  for (int g = threadIdx.x; g < G; g += blockDim.x) groups[g] = make_int4(0, 0, 0, 0);
  if (threadIdx.x == 0) carry = 0;
  // the offsets must be ascending within [0, Q], so that the sequences'
  // query ranges are disjoint; otherwise no query sees anything
  bool ok = true;
  for (int b = threadIdx.x; b <= B; b += blockDim.x) {
    const int32_t v = q_off[b];
    if (v < 0 || v > Q || (b > 0 && q_off[b - 1] > v)) ok = false;
  }
  if (!__syncthreads_and(ok)) {
    if (threadIdx.x == 0) {
      set_status(status, CSA2_DEV_LENGTH);
      *n_groups = 0;
    }
    return;
  }
  for (int base = 0; base < B; base += 1024) {
    const int b = base + threadIdx.x;
    int32_t q0 = 0, nq = 0;
    if (b < B) {
      q0 = q_off[b];
      nq = q_off[b + 1] - q0;
    }
    const int32_t ng = (nq + kQG - 1) / kQG;
    int32_t x = ng;
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
    const int32_t first = carry + warp_sums[wid] + x - ng;
    if (nq > 0) {
      const int64_t off = seq_row_off[b];
      for (int c = 0; c < ng; ++c) {
        if (first + c < G) {
          groups[first + c] = make_int4(b, q0 + kQG * c, min(kQG, nq - kQG * c), 0);
        } else {
          set_status(status, CSA2_DEV_LENGTH);
        }
      }
      for (int i = 0; i < nq; ++i) {
        int64_t v = q_vis[q0 + i];
        if (v < 0) v = 0;
        if (v > max_vis) {
          set_status(status, CSA2_DEV_LENGTH);
          v = max_vis;
        }
        if ((off & 7) != 0 || off < 0 || off + v > cache_rows) {
          set_status(status, CSA2_DEV_ROW_LAYOUT);
          v = 0;
        }
        vis[q0 + i] = int32_t(v);
        q_row_off[q0 + i] = off;
      }
    }
    __syncthreads();
    if (threadIdx.x == 1023) carry = first + ng;
    __syncthreads();
  }
  if (threadIdx.x == 0) *n_groups = min(carry, G);
}

csa2_status launch_groups_tc(const CUtensorMap& map, PfParams& p, int64_t max_vis, cudaStream_t st) {
  p.n_tiles = int((max_vis + kPT - 1) / kPT);
  const int64_t n_items = int64_t(p.n_groups) * p.n_tiles;
  if (n_items > INT32_MAX) return fail(CSA2_ERR_UNSUPPORTED, "csa2 multi-query scan: too many query tiles");
  // more than half of the SM's shared memory, so that one CTA (and one
  // 512-column TMEM allocation) runs per SM
  const size_t smem = std::max<size_t>(sizeof(PfSmem) + 1024, 120 * 1024);
  cudaFuncSetAttribute(k_prefill_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  const int grid = int(std::min<int64_t>(num_sms(), n_items));
  launch_k(k_prefill_tc, dim3(grid), dim3(kThr), smem, st, map, p);
  return CSA2_OK;
}

}  // namespace

int multi_group_bound(int B, int Q) {
  const int64_t g = (int64_t(Q) + 7 * int64_t(B)) / kQG + 1;
  return int(std::min<int64_t>(std::max<int64_t>(g, 1), std::max(Q, 1)));
}

void launch_multi_prep(const int64_t* seq_row_off, const int32_t* q_off, const int32_t* q_vis, int B, int Q, int G,
                       int64_t max_vis, int64_t cache_rows, int4* groups, int64_t* q_row_off, int32_t* vis,
                       int32_t* n_groups, uint32_t* status, cudaStream_t st) {
  launch_k(k_multi_prep, dim3(1), dim3(1024), 0, st, seq_row_off, q_off, q_vis, B, Q, G, max_vis, cache_rows, groups,
           q_row_off, vis, n_groups, status);
}

csa2_status launch_multi_tc(const uint8_t* kcodes, const uint8_t* kscales, int64_t cache_rows,
                            const int64_t* seq_row_off, const int4* groups, int G, const int32_t* n_groups,
                            const int32_t* vis, int Q,
                            int64_t max_vis, const uint8_t* q_codes, const uint8_t* q_scales, const float* w,
                            uint32_t* bkeys, int64_t nb_stride, uint32_t* status, cudaStream_t st) {
  if (Q == 0 || max_vis == 0) return CSA2_OK;
  CUtensorMap map;
  const csa2_status rc = code_map(&map, kcodes, cache_rows, kPT);
  if (rc != CSA2_OK) return rc;
  PfParams p{};
  p.groups = groups;
  p.seq_row_off = seq_row_off;
  p.kscales = kscales;
  p.q_codes = q_codes;
  p.q_scales = q_scales;
  p.w = w;
  p.vis = vis;
  p.T = Q;
  p.row0 = 0;
  p.cache_rows = cache_rows;
  p.n_groups = G;
  p.n_groups_dev = n_groups;
  p.bkeys = bkeys;
  p.nb_stride = nb_stride;
  p.status = status;
  return launch_groups_tc(map, p, max_vis, st);
}

csa2_status launch_prefill_tc(const uint8_t* kcodes, const uint8_t* kscales, int64_t row0, int64_t cache_rows,
                              const int32_t* vis, int T, int64_t max_vis, const uint8_t* q_codes,
                              const uint8_t* q_scales, const float* w, uint32_t* bkeys, int64_t nb_stride,
                              uint32_t* status, cudaStream_t st) {
  if (T == 0 || max_vis == 0) return CSA2_OK;
  CUtensorMap map;
  const csa2_status rc = code_map(&map, kcodes, cache_rows, kPT);
  if (rc != CSA2_OK) return rc;
  PfParams p{};
  p.kscales = kscales;
  p.q_codes = q_codes;
  p.q_scales = q_scales;
  p.w = w;
  p.vis = vis;
  p.T = T;
  p.row0 = row0;
  p.cache_rows = cache_rows;
  p.n_groups = (T + kQG - 1) / kQG;
  p.bkeys = bkeys;
  p.nb_stride = nb_stride;
  p.status = status;
  return launch_groups_tc(map, p, max_vis, st);
}

}  // namespace csa2
