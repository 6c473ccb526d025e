// Sparse attention over the selected MXFP4 main-KV rows plus the FP8 sliding
// window, one softmax per head ("DeepSeek-V4.1-Flash: Pushing the Limits of
// KV Cache Compression", section "三个方向一起压小缓存": 512 entries per layer,
// MXFP4 main KV, FP8 window; section "后 20 层干脆共用一份 KV": 128-token window).
//
// Work split: a segment's keys are chunks (ceil(k/64) chunks of 64 selected
// rows, then four window chunks of 32 rows), and R CTAs share a segment, each
// walking a contiguous run of its chunks (R = 2 x SMs / segments, at most 4:
// two CTAs fit on an SM, and small batches still fill the GPU in one wave).  A CTA loads Q once,
// keeps an online softmax (running max, sum and output per head) across its
// chunks, and while it computes one chunk, cp.async brings the next chunk's
// raw rows (272-byte MXFP4 rows or 512-byte E4M3 rows) into a staging
// buffer; the Top-k ids are loaded one chunk earlier still.  Each chunk's
// rows are dequantised exactly into fp16 in shared memory (E2M1 x 2^X and
// raw E4M3 are exact in fp16 inside the range checked below), and both
// products run on the tensor cores with warp-level mma (fp16 inputs, fp32
// accumulation):
//   S = Q K^T  (16 heads x 64 keys),  P = exp(S*scale - max),  O = P V.
// The window's fp32 scale multiplies its logits and its output in fp32, never
// the fp16 values, so a CTA keeps the window chunks in a partial of their
// own.  Each CTA writes its partials (O, max, sum per head); the last CTA of
// a segment to finish combines them in a fixed order (deterministic) and
// resets the segment's arrival counter.
#include <cuda_fp16.h>

#include <algorithm>

#include "device_common.cuh"
#include "sm100.cuh"

namespace csa2 {

constexpr int kChunk = 64;                         // keys per chunk
constexpr int kAttnThreads = 256;                  // 8 warps
constexpr int kPartFloats = kHq * kD + 2 * kHq;    // O, then m, then l
constexpr int kQS = kD + 8;                        // smem row stride (halves) of Q and K
constexpr int kPS = kChunk + 8;                    // smem row stride (halves) of P
constexpr int kWinRows = 32;                       // window rows per chunk (small staging buffer)
constexpr int kWinChunks = kWin / kWinRows;        // 4
constexpr int kMaxSplits = 4;                      // CTAs per segment at most
constexpr int kMaxSlots = 2 * kMaxSplits;          // partials per segment (main + window per CTA)
constexpr int kRawMain = kMainCodeBytes + kMainScaleBytes;  // 272: codes then scales (row stride 68
                                                            // words: conflict-free 16-byte reads)
constexpr int kRawWin = kD + 16;                   // 528: one E4M3 row + pad

__host__ __device__ inline int attn_main_chunks(int k) { return (k + kChunk - 1) / kChunk; }

int attn_num_chunks(int k) { return attn_main_chunks(k) + kWinChunks; }

// CTAs per segment: the R that minimises (waves of S*R CTAs, two per SM) x
// (chunks per CTA), the fewest CTAs among equals (fewer partials to merge).
int attn_splits(int S, int k) {
  if (S <= 0) return 1;
  const int64_t slots = 2 * int64_t(num_sms());  // two CTAs per SM
  const int nch = attn_num_chunks(k);
  int best = 1;
  int64_t best_cost = INT64_MAX;
  for (int r = 1; r <= std::min(kMaxSplits, nch); ++r) {
    const int64_t waves = (int64_t(S) * r + slots - 1) / slots;
    const int64_t cost = waves * ((nch + r - 1) / r);
    if (cost < best_cost) {
      best_cost = cost;
      best = r;
    }
  }
  return best;
}

size_t attn_partial_bytes(int S, int k) {
  return size_t(S) * 2 * attn_splits(S, k) * kPartFloats * sizeof(float);
}

struct AttnSmem {
  __half q[kHq][kQS];
  __half kv[kChunk][kQS];
  __half p[kHq][kPS];                    // softmax weights, fp16 head ...
  __half plo[kHq][kPS];                  // ... and the fp16 rest (p - head)
  union {
    uint8_t main[kChunk][kRawMain];
    uint8_t win[kWinRows][kRawWin];
  } raw;                                 // staged raw rows of the next chunk
  float red_max[8][kHq];
  float red_sum[8][kHq];
  float m_run[kHq];                      // online softmax state of the current part
  float l_run[kHq];
  int valid[kChunk];
  float fac[kMaxSlots][kHq];
  int last;
};

static_assert(sizeof(AttnSmem) <= 112 * 1024, "two attention CTAs must fit on one SM");

// Rows of chunk c of segment s: how many, where from, and the window scale.
struct ChunkSrc {
  int nkeys;
  bool is_win;
  float kscale;
  const uint8_t* win_base;  // window rows (contiguous), or null
};

__device__ __forceinline__ ChunkSrc chunk_src(const AttnArgs& a, int s, int c) {
  ChunkSrc r;
  const int nmain = attn_main_chunks(a.k);
  r.is_win = (c >= nmain);
  r.kscale = 1.0f;
  r.win_base = nullptr;
  if (!r.is_win) {
    r.nkeys = min(kChunk, a.k - c * kChunk);
    return r;
  }
  const int wc = c - nmain;  // window chunk 0 .. kWinChunks-1
  int nwin;
  const uint8_t* base;
  if (a.q_pos == nullptr) {
    nwin = max(0, min(kWin, a.win_len[s]));
    r.kscale = a.win_scale[s];
    base = a.win + int64_t(s) * kWin * kD;
  } else {
    int64_t p = a.q_pos[s];
    if (p >= a.n_raw) {
      set_status(a.status, CSA2_DEV_LENGTH);
      p = a.n_raw - 1;
    }
    const int64_t lo = p - (kWin - 1) > 0 ? p - (kWin - 1) : 0;
    nwin = p >= 0 ? int(p - lo + 1) : 0;
    r.kscale = a.raw_scale;
    base = a.raw_win + lo * kD;
  }
  r.nkeys = max(0, min(kWinRows, nwin - wc * kWinRows));
  r.win_base = base + int64_t(wc) * kWinRows * kD;
  return r;
}

// Top-k id of this thread's row of chunk c (or -1 when the row is not a
// selected main row).  Issued one chunk ahead of its use.
__device__ __forceinline__ int32_t chunk_tpos(const AttnArgs& a, int s, int c, int r) {
  if (c >= attn_main_chunks(a.k)) return -1;
  const int idx = c * kChunk + r;
  return idx < a.k ? __ldg(a.topk + int64_t(s) * a.k + idx) : -1;
}

// Segment facts every gather needs, read once per CTA: the checked visible
// length and (contiguous layout) the first cache row.
struct SegInfo {
  int64_t eff;
  int64_t row_base;  // -1 in the paged layout
};

__device__ __forceinline__ SegInfo seg_info(const AttnArgs& a, int s) {
  SegInfo g;
  g.eff = a.seg_eff ? int64_t(a.seg_eff[s]) : seg_len_checked(a.sd, s, a.status);
  g.row_base = a.sd.pages ? int64_t(-1) : (a.sd.row_off ? a.sd.row_off[s] : a.sd.row0);
  return g;
}

// Issues the cp.async copies of chunk c's rows into sm.raw (this thread: row
// r = tid % 64, quarter tid / 64 of it) and returns whether row r is present.
__device__ __forceinline__ bool issue_gather(const AttnArgs& a, AttnSmem& sm, int s, int c, int32_t tpos,
                                             const SegInfo& g) {
  const int tid = threadIdx.x, r = tid & (kChunk - 1), qt = tid / kChunk;
  const ChunkSrc src = chunk_src(a, s, c);
  bool ok = r < src.nkeys;
  if (!src.is_win && ok) {
    const int64_t eff = g.eff;
    if (tpos >= eff) {
      if (qt == 0) set_status(a.status, CSA2_DEV_INDEX_RANGE);
      ok = false;
    } else if (tpos < 0) {
      ok = false;
    }
  }
  if (ok) {
    if (!src.is_win) {
      const int64_t row = g.row_base >= 0 ? g.row_base + tpos : seg_row(a.sd, s, tpos, a.status);
      const uint8_t* cs = a.mcodes + row * kMainCodeBytes + qt * (kMainCodeBytes / 4);
      uint8_t* dst = sm.raw.main[r] + qt * (kMainCodeBytes / 4);
#pragma unroll
      for (int i = 0; i < kMainCodeBytes / 4 / 16; ++i) sm100::cp_async16(dst + 16 * i, cs + 16 * i);
      if (qt == 0) sm100::cp_async16(sm.raw.main[r] + kMainCodeBytes, a.mscales + row * kMainScaleBytes);
    } else {  // r < nkeys <= kWinRows
      const uint8_t* ws = src.win_base + int64_t(r) * kD + qt * (kD / 4);
      uint8_t* dst = sm.raw.win[r] + qt * (kD / 4);
#pragma unroll
      for (int i = 0; i < kD / 4 / 16; ++i) sm100::cp_async16(dst + 16 * i, ws + 16 * i);
    }
  }
  return ok;
}

// Two E2M1 codes (low nibble = lower element) -> f16x2, exact.
__device__ __forceinline__ uint32_t cvt_e2m1x2(uint32_t byte) {
  uint32_t r;
  asm("{\n\t.reg .b8 t;\n\tmov.b16 {t, _}, %1;\n\tcvt.rn.f16x2.e2m1x2 %0, t;\n\t}" : "=r"(r) : "h"(uint16_t(byte)));
  return r;
}
// Two E4M3 bytes (low byte = lower element) -> f16x2, exact.
__device__ __forceinline__ uint32_t cvt_e4m3x2(uint32_t two) {
  uint32_t r;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(r) : "h"(uint16_t(two)));
  return r;
}

// Packed f16x2 multiply on raw 32-bit registers (round to nearest).
__device__ __forceinline__ uint32_t hmul2_u32(uint32_t x, uint32_t y) {
  uint32_t r;
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(x), "r"(y));
  return r;
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

// Q of segment s: bf16 -> fp16 into sm.q (exact for |q| in [2^-14, 65504];
// smaller values keep 2^-24 resolution).
__device__ __forceinline__ void load_q(const AttnArgs& a, AttnSmem& sm, int s) {
  const int tid = threadIdx.x;
  constexpr int kQV = kHq * kD / 8 / kAttnThreads;  // 16-byte vectors per thread (4)
  uint4 qv[kQV];
  const uint4* qsrc = reinterpret_cast<const uint4*>(a.q + int64_t(s) * kHq * kD);
#pragma unroll
  for (int m = 0; m < kQV; ++m) qv[m] = __ldg(qsrc + tid + m * kAttnThreads);
#pragma unroll
  for (int m = 0; m < kQV; ++m) {
    const int e = 8 * (tid + m * kAttnThreads);
    const int h = e / kD, d = e % kD;
    const uint32_t w[4] = {qv[m].x, qv[m].y, qv[m].z, qv[m].w};
    uint32_t o[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float lo = __uint_as_float(w[q] << 16), hi = __uint_as_float(w[q] & 0xFFFF0000u);
      if (fabsf(lo) > 65504.0f || fabsf(hi) > 65504.0f) set_status(a.status, CSA2_DEV_FP16_RANGE);
      const __half2 h2 = __floats2half2_rn(lo, hi);
      o[q] = *reinterpret_cast<const uint32_t*>(&h2);
    }
    *reinterpret_cast<uint4*>(&sm.q[h][d]) = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

// Staged raw rows -> fp16 keys in sm.kv (absent rows as zeros) and the
// row-valid flags.  Thread: row r = tid % 64, blocks tid/64 + 4i.
__device__ __forceinline__ void dequant_chunk(const AttnArgs& a, AttnSmem& sm, bool is_win, bool row_ok) {
  const int tid = threadIdx.x;
  const int r = tid & (kChunk - 1);
  constexpr int kBPT = 16 / (kAttnThreads / kChunk);  // blocks per thread (4)
  const int b0 = tid / kChunk;
  if (b0 == 0) sm.valid[r] = row_ok;
#pragma unroll
  for (int i = 0; i < kBPT; ++i) {
    const int b = b0 + 4 * i;
    uint4* dst = reinterpret_cast<uint4*>(&sm.kv[r][32 * b]);
    if (!row_ok) {
#pragma unroll
      for (int q = 0; q < 4; ++q) dst[q] = make_uint4(0, 0, 0, 0);
      continue;
    }
    if (!is_win) {
      // fp16-exact iff the block exponent X = byte - 127 lies in [-23, 13]
      const uint4 cw = *reinterpret_cast<const uint4*>(sm.raw.main[r] + 16 * b);
      const uint32_t sb = sm.raw.main[r][kMainCodeBytes + b];
      if (sb < 104u || sb > 140u) set_status(a.status, CSA2_DEV_FP16_RANGE);
      const int X = int(sb) - 127;
      const uint16_t xb = X >= -14 ? uint16_t((X + 15) << 10) : uint16_t(1u << (X + 24 > 0 ? X + 24 : 0));
      const uint32_t sc2 = uint32_t(xb) | (uint32_t(xb) << 16);
      const uint32_t w4[4] = {cw.x, cw.y, cw.z, cw.w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint32_t hv[4];
#pragma unroll
        for (int n = 0; n < 4; ++n) hv[n] = hmul2_u32(cvt_e2m1x2((w4[q] >> (8 * n)) & 255u), sc2);
        dst[q] = make_uint4(hv[0], hv[1], hv[2], hv[3]);
      }
    } else {
      const uint4 v0 = *reinterpret_cast<const uint4*>(sm.raw.win[r] + 32 * b);
      const uint4 v1 = *reinterpret_cast<const uint4*>(sm.raw.win[r] + 32 * b + 16);
      const uint32_t w8[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
#pragma unroll
      for (int q = 0; q < 4; ++q)
        dst[q] = make_uint4(cvt_e4m3x2(w8[2 * q] & 0xFFFFu), cvt_e4m3x2(w8[2 * q] >> 16),
                            cvt_e4m3x2(w8[2 * q + 1] & 0xFFFFu), cvt_e4m3x2(w8[2 * q + 1] >> 16));
    }
  }
}

__device__ __forceinline__ void ldsm_x2(uint32_t (&r)[2], const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0, %1}, [%2];"
               : "=r"(r[0]), "=r"(r[1])
               : "r"(static_cast<uint32_t>(__cvta_generic_to_shared(p))));
}

// One chunk (keys in sm.kv) into the running softmax state: S = Q K^T for the
// chunk's keys, the running max / sum per head (sm.m_run, sm.l_run) and the
// output accumulator oacc (warp w: dims 64w .. 64w+63, rows g and g+8).
__device__ __forceinline__ void chunk_update(const AttnArgs& a, AttnSmem& sm, float (&oacc)[8][4], int nkeys,
                                             float kscale) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, t = lane & 3;
  // ---- S: warp w owns keys 8w .. 8w+7; two accumulators over alternate k-steps ----
  // four independent accumulators over alternate k-steps (chains of 8 MMAs)
  float sacc[4][4] = {};
  {
    const int kr = 8 * warp + (lane & 7);
    const int kc = 8 * ((lane >> 3) & 1);
    const int qr = (lane & 7) + 8 * ((lane >> 3) & 1);
    const int qc = 8 * (lane >> 4);
#pragma unroll 2
    for (int k0 = 0; k0 < kD; k0 += 64) {
      uint32_t af[4][4], bf[4][2];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        ldsm_x4(af[u], &sm.q[qr][k0 + 16 * u + qc]);
        ldsm_x2(bf[u], &sm.kv[kr][k0 + 16 * u + kc]);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) mma16816(sacc[u], af[u], bf[u][0], bf[u][1]);
    }
  }
  // ---- logits, chunk maxima (per head) ----
  const float lscale = a.sm_scale * kscale;
  float sv[4];
  float mx[2] = {-INFINITY, -INFINITY};  // heads g, g+8
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int key = 8 * warp + 2 * t + (j & 1);
    const float v =
        (key < nkeys && sm.valid[key]) ? ((sacc[0][j] + sacc[1][j]) + (sacc[2][j] + sacc[3][j])) * lscale : -INFINITY;
    sv[j] = v;
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
  // ---- new running max, rescale factor, fp16 weights ----
  float mnew[2], alpha[2], sum[2] = {0.0f, 0.0f};
#pragma unroll
  for (int hh = 0; hh < 2; ++hh) {
    const int h = g + 8 * hh;
    float cm = -INFINITY;
#pragma unroll
    for (int w = 0; w < 8; ++w) cm = fmaxf(cm, sm.red_max[w][h]);
    const float mold = sm.m_run[h];
    mnew[hh] = fmaxf(mold, cm);
    alpha[hh] = (mold == -INFINITY) ? 0.0f : __expf(mold - mnew[hh]);
  }
#pragma unroll
  for (int j = 0; j < 4; j += 2) {
    const int hh = j >> 1;
    const float p0 = (mnew[hh] == -INFINITY) ? 0.0f : __expf(sv[j] - mnew[hh]);
    const float p1 = (mnew[hh] == -INFINITY) ? 0.0f : __expf(sv[j + 1] - mnew[hh]);
    // p = head + rest, both fp16 (the rest is exact in fp32); P V runs on
    // both, so the weights carry about 22 bits and the sum uses exactly the
    // weights the MMAs see
    const __half2 ph = __floats2half2_rn(p0, p1);
    const float2 pr = __half22float2(ph);
    const __half2 pl = __floats2half2_rn(p0 - pr.x, p1 - pr.y);
    const float2 plr = __half22float2(pl);
    sum[hh] += (pr.x + plr.x) + (pr.y + plr.y);
    *reinterpret_cast<__half2*>(&sm.p[g + 8 * hh][8 * warp + 2 * t]) = ph;
    *reinterpret_cast<__half2*>(&sm.plo[g + 8 * hh][8 * warp + 2 * t]) = pl;
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
  if (tid < kHq) {  // running state (read again only after the next chunk's barriers)
    float l = 0.0f;
#pragma unroll
    for (int w = 0; w < 8; ++w) l += sm.red_sum[w][tid];
    float cm = -INFINITY;
#pragma unroll
    for (int w = 0; w < 8; ++w) cm = fmaxf(cm, sm.red_max[w][tid]);
    const float mold = sm.m_run[tid];
    const float mn = fmaxf(mold, cm);
    const float al = (mold == -INFINITY) ? 0.0f : __expf(mold - mn);
    sm.l_run[tid] = sm.l_run[tid] * al + l;
    sm.m_run[tid] = mn;
  }
  // ---- O = alpha O + P V over the chunk's keys ----
#pragma unroll
  for (int nt = 0; nt < 8; ++nt) {
    oacc[nt][0] *= alpha[0];
    oacc[nt][1] *= alpha[0];
    oacc[nt][2] *= alpha[1];
    oacc[nt][3] *= alpha[1];
  }
  {
    const int pr_ = (lane & 7) + 8 * ((lane >> 3) & 1);
    const int pc = 8 * (lane >> 4);
    const int vr = (lane & 7) + 8 * ((lane >> 3) & 1);  // key row within the k-step
    const int vc = 8 * (lane >> 4);                     // dim offset within the n-tile pair
    const int kend = (nkeys + 15) & ~15;
    for (int k0 = 0; k0 < kend; k0 += 16) {
      uint32_t af[4], al[4];
      ldsm_x4(af, &sm.p[pr_][k0 + pc]);
      ldsm_x4(al, &sm.plo[pr_][k0 + pc]);
#pragma unroll
      for (int np = 0; np < 4; ++np) {
        uint32_t bf[4];
        ldsm_x4_t(bf, &sm.kv[k0 + vr][64 * warp + 16 * np + vc]);
        mma16816(oacc[2 * np], af, bf[0], bf[1]);
        mma16816(oacc[2 * np + 1], af, bf[2], bf[3]);
        mma16816(oacc[2 * np], al, bf[0], bf[1]);
        mma16816(oacc[2 * np + 1], al, bf[2], bf[3]);
      }
    }
  }
}

// Writes the running part (O x kscale, max, sum) to partial slot `slot` and
// resets the state.
__device__ __forceinline__ void flush_part(const AttnArgs& a, AttnSmem& sm, float (&oacc)[8][4], int s, int nslots,
                                           int slot, float kscale) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, t = lane & 3;
  float* part = a.partial + (int64_t(s) * nslots + slot) * kPartFloats;
  __syncthreads();  // the running max / sum of the last chunk are written
#pragma unroll
  for (int nt = 0; nt < 8; ++nt) {
    const int d = 64 * warp + 8 * nt + 2 * t;
    *reinterpret_cast<float2*>(&part[g * kD + d]) = make_float2(oacc[nt][0] * kscale, oacc[nt][1] * kscale);
    *reinterpret_cast<float2*>(&part[(g + 8) * kD + d]) = make_float2(oacc[nt][2] * kscale, oacc[nt][3] * kscale);
#pragma unroll
    for (int j = 0; j < 4; ++j) oacc[nt][j] = 0.0f;
  }
  __syncthreads();
  if (tid < kHq) {
    part[kHq * kD + tid] = sm.m_run[tid];
    part[kHq * kD + kHq + tid] = sm.l_run[tid];
    sm.m_run[tid] = -INFINITY;
    sm.l_run[tid] = 0.0f;
  }
}

// An empty partial: max -inf, sum 0 (its O is never read).
__device__ __forceinline__ void empty_part(const AttnArgs& a, int s, int nslots, int slot) {
  float* part = a.partial + (int64_t(s) * nslots + slot) * kPartFloats;
  if (threadIdx.x < kHq) {
    part[kHq * kD + threadIdx.x] = -INFINITY;
    part[kHq * kD + kHq + threadIdx.x] = 0.0f;
  }
}

// Last-arriving CTA of a segment: combine the partials in slot order
// (deterministic), write out / lse, and reset the segment's arrival counter.
__device__ __forceinline__ void combine_if_last(const AttnArgs& a, AttnSmem& sm, int s, int nctas, int nslots) {
  const int tid = threadIdx.x;
  // The barrier orders every thread's partial stores before thread 0's
  // release-acquire arrival (gpu scope); the last arrival therefore sees all
  // of the segment's partials.
  __syncthreads();
  if (tid == 0) {
    int old;
    asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], 1;" : "=r"(old) : "l"(a.counters + s) : "memory");
    sm.last = (old == nctas - 1);
  }
  __syncthreads();
  if (!sm.last) return;
  const float* base = a.partial + int64_t(s) * nslots * kPartFloats;
  if (tid < kHq) {
    float mc[kMaxSlots], lc[kMaxSlots];
    float M = -INFINITY;
#pragma unroll
    for (int c = 0; c < kMaxSlots; ++c) {  // all loads first
      mc[c] = c < nslots ? __ldcg(base + c * kPartFloats + kHq * kD + tid) : -INFINITY;
      lc[c] = c < nslots ? __ldcg(base + c * kPartFloats + kHq * kD + kHq + tid) : 0.0f;
    }
#pragma unroll
    for (int c = 0; c < kMaxSlots; ++c) M = fmaxf(M, mc[c]);
    float L = 0.0f;
#pragma unroll
    for (int c = 0; c < kMaxSlots; ++c) {
      const float f = (mc[c] == -INFINITY) ? 0.0f : __expf(mc[c] - M);
      if (c < nslots) sm.fac[c][tid] = f;
      L += lc[c] * f;
    }
    for (int c = 0; c < nslots; ++c) sm.fac[c][tid] = (M == -INFINITY) ? 0.0f : sm.fac[c][tid] / L;
    if (a.lse) a.lse[int64_t(s) * kHq + tid] = (M == -INFINITY) ? -INFINITY : M + logf(L);
  }
  __syncthreads();
  // 8 float4 per thread; slots whose factor is 0 (empty or negligible) are
  // skipped, so an empty slot's O is never read
  constexpr int kOV = kHq * kD / 4 / kAttnThreads;
  float4 o[kOV];
#pragma unroll
  for (int m = 0; m < kOV; ++m) o[m] = make_float4(0.f, 0.f, 0.f, 0.f);
  // two slots per pass: both slots' loads are in flight together (slot
  // order of the sums unchanged)
  for (int c = 0; c < nslots; c += 2) {
    float4 v[2][kOV];
    float f[2][kOV];
#pragma unroll
    for (int u = 0; u < 2; ++u)
#pragma unroll
      for (int m = 0; m < kOV; ++m) {
        f[u][m] = c + u < nslots ? sm.fac[c + u][(4 * (tid + m * kAttnThreads)) / kD] : 0.0f;
        v[u][m] = f[u][m] != 0.0f
                      ? __ldcg(reinterpret_cast<const float4*>(base + (c + u) * kPartFloats) + tid + m * kAttnThreads)
                      : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
    for (int u = 0; u < 2; ++u)
#pragma unroll
      for (int m = 0; m < kOV; ++m) {
        o[m].x = fmaf(v[u][m].x, f[u][m], o[m].x);
        o[m].y = fmaf(v[u][m].y, f[u][m], o[m].y);
        o[m].z = fmaf(v[u][m].z, f[u][m], o[m].z);
        o[m].w = fmaf(v[u][m].w, f[u][m], o[m].w);
      }
  }
#pragma unroll
  for (int m = 0; m < kOV; ++m) reinterpret_cast<float4*>(a.out + int64_t(s) * kHq * kD)[tid + m * kAttnThreads] = o[m];
  if (tid == 0) a.counters[s] = 0;
}

// grid = (R, S): CTA (r, s) takes chunks [r n / R, (r + 1) n / R) of segment s.
__global__ void __launch_bounds__(kAttnThreads, 2) k_attn(AttnArgs a, int R) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  AttnSmem& sm = *reinterpret_cast<AttnSmem*>(smem_raw);
  const int s = blockIdx.y, r = blockIdx.x, tid = threadIdx.x, row = tid & (kChunk - 1);
  const int n = attn_main_chunks(a.k) + kWinChunks;
  const int c0 = int(int64_t(n) * r / R), c1 = int(int64_t(n) * (r + 1) / R);
  const int nslots = 2 * R;
  launch_dependents();
  float oacc[8][4];
#pragma unroll
  for (int nt = 0; nt < 8; ++nt)
#pragma unroll
    for (int j = 0; j < 4; ++j) oacc[nt][j] = 0.0f;
  if (tid < kHq) {
    sm.m_run[tid] = -INFINITY;
    sm.l_run[tid] = 0.0f;
  }
  grid_wait();  // the Top-k ids, queries and rows may come from the previous kernel
  const SegInfo sg = seg_info(a, s);
  bool ok = false;
  int32_t tnext = -1;
  if (c0 < c1) {
    ok = issue_gather(a, sm, s, c0, chunk_tpos(a, s, c0, row), sg);
    sm100::cp_async_commit();
    tnext = (c0 + 1 < c1) ? chunk_tpos(a, s, c0 + 1, row) : -1;
  }
  load_q(a, sm, s);  // overlaps the first gather
  bool in_win = false, wrote_main = false;
  float win_scale = 1.0f;
  for (int c = c0; c < c1; ++c) {
    const ChunkSrc src = chunk_src(a, s, c);
    if (src.is_win && !in_win) {
      if (c > c0) {  // this CTA's selected rows are done: their partial
        flush_part(a, sm, oacc, s, nslots, 2 * r, 1.0f);
        wrote_main = true;
      }
      in_win = true;
      win_scale = src.kscale;
    }
    sm100::cp_async_wait<0>();
    __syncthreads();  // this chunk's rows (and Q) are in shared memory
    dequant_chunk(a, sm, src.is_win, ok);
    __syncthreads();  // keys ready; the staging buffer is free
    if (c + 1 < c1) {
      ok = issue_gather(a, sm, s, c + 1, tnext, sg);
      sm100::cp_async_commit();
      tnext = (c + 2 < c1) ? chunk_tpos(a, s, c + 2, row) : -1;
    }
    chunk_update(a, sm, oacc, src.nkeys, src.kscale);
  }
  if (in_win) {
    flush_part(a, sm, oacc, s, nslots, 2 * r + 1, win_scale);
  } else if (c0 < c1) {
    flush_part(a, sm, oacc, s, nslots, 2 * r, 1.0f);
    wrote_main = true;
  }
  if (!wrote_main) empty_part(a, s, nslots, 2 * r);
  if (!in_win) empty_part(a, s, nslots, 2 * r + 1);
  sm100::cp_async_wait<0>();
  combine_if_last(a, sm, s, R, nslots);
}

void prepare_attention() {
  // setting the attributes loads the kernel's module on the current device
  cudaFuncSetAttribute(k_attn, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(sizeof(AttnSmem)));
  cudaFuncSetAttribute(k_attn, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
}

void launch_attention(const AttnArgs& a, cudaStream_t st) {
  if (a.S == 0) return;
  const int R = attn_splits(a.S, a.k);
  prepare_attention();
  launch_k(k_attn, dim3(R, a.S), dim3(kAttnThreads), sizeof(AttnSmem), st, a, R);
}

}  // namespace csa2
