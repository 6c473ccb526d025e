// Sparse attention over the selected MXFP4 main-KV rows plus the FP8 sliding
// window, one softmax per head ("DeepSeek-V4.1-Flash: Pushing the Limits of
// KV Cache Compression", section "三个方向一起压小缓存": 512 entries per layer,
// MXFP4 main KV, FP8 window; section "后 20 层干脆共用一份 KV": 128-token window).
//
// Work split: a segment's keys are chunks (ceil(k/64) chunks of 64 selected
// rows, and four window chunks of 32 rows), and R CTAs share a segment
// (R <= 4, the one that minimises waves of CTAs, two per SM, times chunks
// per CTA: 4 at a decode batch of 64, 1 for a prefill chunk of 4096
// queries).  Each CTA takes an even share of
// the window chunks and one of the selected chunks, windows first: the window
// rows are the caller's inputs, so the first of them are staged before the
// wait on the previous kernel.  While a CTA computes one chunk, cp.async
// brings the next chunk's raw rows (272-byte MXFP4 rows or 512-byte E4M3
// rows) into the staging buffer; the Top-k ids are loaded one chunk earlier
// still.
//
// Both products run on the tensor cores with warp-level mma (fp16 inputs,
// fp32 accumulation), and the rows are converted to fp16 once, in registers
// (E2M1 x 2^X and E4M3 are exact in fp16 inside the range checked below):
//   S = Q K^T  (16 heads x 64 keys): warp (h, q) takes the keys of half h
//       and the 128 dims of quarter q, reads their raw bytes, converts them
//       and keeps its Q fragments in registers for the whole kernel; the four
//       quarters' partial scores meet in shared memory and are summed in a
//       fixed order.  Inside each 32-dim scale block the reduction order of
//       the dims is permuted so that a thread's 8 consecutive dims (one
//       32-bit word of E2M1 codes) form its B fragments of two k-steps; Q
//       uses the same permutation.  The converted rows go to shared memory.
//   P = exp(S*scale - max), split into an fp16 head and an fp16 rest.
//   O = P V: warp w owns dims 64w .. 64w+63 and reads V (the same rows)
//       with transposing ldmatrix.
// The window's fp32 scale multiplies its logits and its output in fp32, never
// the fp16 values: a CTA multiplies its accumulated output by it once, when
// its window chunks are done and before its selected chunks, so one running
// softmax state covers all of its chunks.  With R > 1 each CTA writes that
// part (O, max, sum per head) and the last CTA of a segment to finish
// combines the R parts in a fixed order (deterministic) and resets the
// segment's arrival counter; a segment's only CTA (R = 1) divides by the sum
// in registers and writes the output directly.
#include <cuda_fp16.h>

#include <algorithm>

#include "device_common.cuh"
#include "sm100.cuh"

namespace csa2 {

constexpr int kChunk = 64;                         // keys per chunk
constexpr int kAttnThreads = 256;                  // 8 warps
constexpr int kPartFloats = kHq * kD + 2 * kHq;    // O, then m, then l
constexpr int kQS = kD + 8;                        // smem row stride (halves) of the converted rows
constexpr int kPS = kChunk + 8;                    // smem row stride (halves) of P
constexpr int kWinRows = 32;                       // window rows per chunk (small staging buffer)
constexpr int kWinChunks = kWin / kWinRows;        // 4
constexpr int kMaxSplits = 4;                      // CTAs per segment at most
constexpr int kMaxSlots = kMaxSplits;              // partials per segment (one per CTA)
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

// One partial per CTA; a segment's only CTA (R = 1) normalises its output
// in registers and writes none.
size_t attn_partial_bytes(int S, int k) {
  const int R = attn_splits(S, k);
  return R == 1 ? 0 : size_t(S) * R * kPartFloats * sizeof(float);
}

// Staged raw rows of one chunk.  Row strides of 68 and 132 words put the
// rows a warp reads together on different banks.
union RawRows {
  uint8_t main[kChunk][kRawMain];
  uint8_t win[kWinRows][kRawWin];
};

struct AttnSmem {
  __half kv[kChunk][kQS];                // the chunk's rows in fp16
  RawRows raw;                           // staged raw rows of the next chunk
  float4 s_part[2][4][4][32];            // partial scores [key half][dim quarter][n-tile][lane]
  __half p[kHq][kPS];                    // softmax weights, fp16 head ...
  __half plo[kHq][kPS];                  // ... and the fp16 rest (p - head)
  float red_max[8][kHq];
  float red_sum[8][kHq];
  float m_run[kHq];                      // online softmax state of the current part
  float l_run[kHq];
  int valid[2][kChunk];                  // row present (this chunk's and the next one's)
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
// r = tid % 64, quarter tid / 64 of it) and records in sm.valid[vb] whether
// row r is present.  An absent row is written as zeros (codes 0, unit scales), so
// the products read exact zeros from it.
__device__ __forceinline__ void issue_gather(const AttnArgs& a, AttnSmem& sm, int vb, int s, int c, int32_t tpos,
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
  RawRows& rr = sm.raw;
  if (!src.is_win) {
    uint8_t* dst = rr.main[r] + qt * (kMainCodeBytes / 4);
    if (ok) {
      const int64_t row = g.row_base >= 0 ? g.row_base + tpos : seg_row(a.sd, s, tpos, a.status);
      const uint8_t* cs = a.mcodes + row * kMainCodeBytes + qt * (kMainCodeBytes / 4);
#pragma unroll
      for (int i = 0; i < kMainCodeBytes / 4 / 16; ++i) sm100::cp_async16(dst + 16 * i, cs + 16 * i);
      if (qt == 0) sm100::cp_async16(rr.main[r] + kMainCodeBytes, a.mscales + row * kMainScaleBytes);
    } else {
#pragma unroll
      for (int i = 0; i < kMainCodeBytes / 4 / 16; ++i) *reinterpret_cast<uint4*>(dst + 16 * i) = make_uint4(0, 0, 0, 0);
      if (qt == 0)
        *reinterpret_cast<uint4*>(rr.main[r] + kMainCodeBytes) =
            make_uint4(0x7F7F7F7Fu, 0x7F7F7F7Fu, 0x7F7F7F7Fu, 0x7F7F7F7Fu);
    }
    if (qt == 0) sm.valid[vb][r] = ok;
  } else if (r < kWinRows) {
    uint8_t* dst = rr.win[r] + qt * (kD / 4);
    if (ok) {
      const uint8_t* ws = src.win_base + int64_t(r) * kD + qt * (kD / 4);
#pragma unroll
      for (int i = 0; i < kD / 4 / 16; ++i) sm100::cp_async16(dst + 16 * i, ws + 16 * i);
    } else {
#pragma unroll
      for (int i = 0; i < kD / 4 / 16; ++i) *reinterpret_cast<uint4*>(dst + 16 * i) = make_uint4(0, 0, 0, 0);
    }
    if (qt == 0) sm.valid[vb][r] = ok;
  }
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
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t (&r)[4], const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(static_cast<uint32_t>(__cvta_generic_to_shared(p))));
}

// 2^X as an fp16 pair for an E8M0 scale byte (X = byte - 127); exact for X in
// [-24, 15].
__device__ __forceinline__ uint32_t e8m0_f16x2(uint32_t sb) {
  const int X = int(sb) - 127;
  const uint16_t xb = X >= -14 ? uint16_t((X + 15) << 10) : uint16_t(1u << (X + 24 > 0 ? X + 24 : 0));
  return uint32_t(xb) | (uint32_t(xb) << 16);
}

// One 32-bit word of E2M1 codes (8 consecutive dims) times its block scale:
// f[m] = dims 2m, 2m+1 of the word.
__device__ __forceinline__ void conv_fp4_word(uint32_t w, uint32_t sc2, uint32_t (&f)[4]) {
#pragma unroll
  for (int m = 0; m < 4; ++m) f[m] = hmul2_u32(cvt_e2m1x2((w >> (8 * m)) & 255u), sc2);
}
// Eight consecutive E4M3 bytes: f[m] = dims 2m, 2m+1.
__device__ __forceinline__ void conv_e4m3_pair(uint2 v, uint32_t (&f)[4]) {
  f[0] = cvt_e4m3x2(v.x & 0xFFFFu);
  f[1] = cvt_e4m3x2(v.x >> 16);
  f[2] = cvt_e4m3x2(v.y & 0xFFFFu);
  f[3] = cvt_e4m3x2(v.y >> 16);
}

// This thread's Q fragments (lane = 4g + t): for each of the warp's four
// scale blocks (dims 32(4q + j) ..), dims 8t .. 8t+7 of heads g (qa) and g+8
// (qb) as fp16 pairs.  bf16 -> fp16 is exact for |q| in [2^-14, 65504];
// smaller values keep 2^-24 resolution.
struct QFrag {
  uint4 qa[4], qb[4];
};

__device__ __forceinline__ uint4 bf16x8_to_f16x8(uint4 v, uint32_t* status) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t o[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const float lo = __uint_as_float(w[q] << 16), hi = __uint_as_float(w[q] & 0xFFFF0000u);
    if (fabsf(lo) > 65504.0f || fabsf(hi) > 65504.0f) set_status(status, CSA2_DEV_FP16_RANGE);
    const __half2 h2 = __floats2half2_rn(lo, hi);
    o[q] = *reinterpret_cast<const uint32_t*>(&h2);
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

__device__ __forceinline__ void load_q_frag(const AttnArgs& a, int s, int quarter, QFrag& qf) {
  const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  const uint16_t* qs = a.q + int64_t(s) * kHq * kD;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int d = 32 * (4 * quarter + j) + 8 * t;
    qf.qa[j] = __ldg(reinterpret_cast<const uint4*>(qs + g * kD + d));
    qf.qb[j] = __ldg(reinterpret_cast<const uint4*>(qs + (g + 8) * kD + d));
  }
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    qf.qa[j] = bf16x8_to_f16x8(qf.qa[j], a.status);
    qf.qb[j] = bf16x8_to_f16x8(qf.qb[j], a.status);
  }
}

// Partial scores of one chunk: warp (h, q) = (warp / 4, warp % 4) computes
// S over dims of quarter q for the 32 keys of half h (4 n-tiles) and leaves
// them in sm.s_part; the converted rows go to sm.kv.  For k-step (j, e) of
// block j, the thread's B fragment is (dims 4e, 4e+1 | 4e+2, 4e+3 of its
// word) and its A fragment the same dims of Q, so the k order inside the
// block is a permutation of the dims.
__device__ __forceinline__ void qk_partial(const AttnArgs& a, AttnSmem& sm, bool is_win, int nkeys,
                                           const QFrag& qf) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 2, t = lane & 3, kh = warp >> 2, dq = warp & 3;
  if (32 * kh >= nkeys) return;  // (window chunks) no keys in this half
  const RawRows& rr = sm.raw;
  float sacc[4][4] = {};
  if (!is_win) {
    uint32_t wd[4][4], sw[4];
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) {
      const uint8_t* row = rr.main[32 * kh + 8 * nt + g];
#pragma unroll
      for (int j = 0; j < 4; ++j) wd[nt][j] = *reinterpret_cast<const uint32_t*>(row + 16 * (4 * dq + j) + 4 * t);
      sw[nt] = *reinterpret_cast<const uint32_t*>(row + kMainCodeBytes + 4 * dq);
    }
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint32_t sb = (sw[nt] >> (8 * j)) & 255u;
        // fp16-exact iff the block exponent X = byte - 127 lies in [-23, 13]
        if (t == 0 && (sb < 104u || sb > 140u)) set_status(a.status, CSA2_DEV_FP16_RANGE);
      }
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t qa0[4] = {qf.qa[j].x, qf.qb[j].x, qf.qa[j].y, qf.qb[j].y};
      const uint32_t qa1[4] = {qf.qa[j].z, qf.qb[j].z, qf.qa[j].w, qf.qb[j].w};
#pragma unroll
      for (int nt = 0; nt < 4; ++nt) {
        uint32_t f[4];
        conv_fp4_word(wd[nt][j], e8m0_f16x2((sw[nt] >> (8 * j)) & 255u), f);
        mma16816(sacc[nt], qa0, f[0], f[1]);
        mma16816(sacc[nt], qa1, f[2], f[3]);
        *reinterpret_cast<uint4*>(&sm.kv[32 * kh + 8 * nt + g][32 * (4 * dq + j) + 8 * t]) =
            make_uint4(f[0], f[1], f[2], f[3]);
      }
    }
  } else {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t qa0[4] = {qf.qa[j].x, qf.qb[j].x, qf.qa[j].y, qf.qb[j].y};
      const uint32_t qa1[4] = {qf.qa[j].z, qf.qb[j].z, qf.qa[j].w, qf.qb[j].w};
#pragma unroll
      for (int nt = 0; nt < 4; ++nt) {
        const uint8_t* row = rr.win[32 * kh + 8 * nt + g];
        uint32_t f[4];
        conv_e4m3_pair(*reinterpret_cast<const uint2*>(row + 32 * (4 * dq + j) + 8 * t), f);
        mma16816(sacc[nt], qa0, f[0], f[1]);
        mma16816(sacc[nt], qa1, f[2], f[3]);
        *reinterpret_cast<uint4*>(&sm.kv[32 * kh + 8 * nt + g][32 * (4 * dq + j) + 8 * t]) =
            make_uint4(f[0], f[1], f[2], f[3]);
      }
    }
  }
#pragma unroll
  for (int nt = 0; nt < 4; ++nt) sm.s_part[kh][dq][nt][lane] = make_float4(sacc[nt][0], sacc[nt][1], sacc[nt][2], sacc[nt][3]);
}

// The rest of one chunk (partial scores in sm.s_part, rows in sm.kv): the
// running max / sum per head (sm.m_run, sm.l_run) and the output accumulator
// oacc (warp w: dims 64w .. 64w+63, heads g and g+8 of lane 4g + t).
__device__ __forceinline__ void softmax_pv(const AttnArgs& a, AttnSmem& sm, int vb, float (&oacc)[8][4], int nkeys,
                                           float kscale) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, t = lane & 3;
  // ---- S of keys 8w .. 8w+7: the four quarters in order, then the chunk maxima ----
  float sacc[4];
  {
    const int kh = warp >> 2, nt = warp & 3;
    float4 v = sm.s_part[kh][0][nt][lane];
#pragma unroll
    for (int q = 1; q < 4; ++q) {
      const float4 u = sm.s_part[kh][q][nt][lane];
      v.x += u.x, v.y += u.y, v.z += u.z, v.w += u.w;
    }
    sacc[0] = v.x, sacc[1] = v.y, sacc[2] = v.z, sacc[3] = v.w;
  }
  const float lscale = a.sm_scale * kscale;
  float sv[4];
  float mx[2] = {-INFINITY, -INFINITY};  // heads g, g+8
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int key = 8 * warp + 2 * t + (j & 1);
    const float v = (key < nkeys && sm.valid[vb][key]) ? sacc[j] * lscale : -INFINITY;
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

// O *= f (the window rows' fp32 scale, applied once to their output).
__device__ __forceinline__ void scale_acc(float (&oacc)[8][4], float f) {
#pragma unroll
  for (int nt = 0; nt < 8; ++nt)
#pragma unroll
    for (int j = 0; j < 4; ++j) oacc[nt][j] *= f;
}

// Writes the running part (O, max, sum) to partial slot `slot`.
__device__ __forceinline__ void flush_part(const AttnArgs& a, AttnSmem& sm, float (&oacc)[8][4], int s, int nslots,
                                           int slot) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, t = lane & 3;
  float* part = a.partial + (int64_t(s) * nslots + slot) * kPartFloats;
  __syncthreads();  // the running max / sum of the last chunk are written
#pragma unroll
  for (int nt = 0; nt < 8; ++nt) {
    const int d = 64 * warp + 8 * nt + 2 * t;
    *reinterpret_cast<float2*>(&part[g * kD + d]) = make_float2(oacc[nt][0], oacc[nt][1]);
    *reinterpret_cast<float2*>(&part[(g + 8) * kD + d]) = make_float2(oacc[nt][2], oacc[nt][3]);
  }
  if (tid < kHq) {
    part[kHq * kD + tid] = sm.m_run[tid];
    part[kHq * kD + kHq + tid] = sm.l_run[tid];
  }
}

// The only CTA of its segment: out = O / l and lse = max + log l per head,
// from registers (the same factor 1 / l as a one-slot combine).
__device__ __forceinline__ void finish_single(const AttnArgs& a, AttnSmem& sm, float (&oacc)[8][4], int s) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, t = lane & 3;
  __syncthreads();  // the running max / sum of the last chunk are written
  float f[2];
#pragma unroll
  for (int hh = 0; hh < 2; ++hh) {
    const float M = sm.m_run[g + 8 * hh], L = sm.l_run[g + 8 * hh];
    f[hh] = (M == -INFINITY) ? 0.0f : 1.0f / L;
  }
  float* o = a.out + int64_t(s) * kHq * kD;
#pragma unroll
  for (int nt = 0; nt < 8; ++nt) {
    const int d = 64 * warp + 8 * nt + 2 * t;
    *reinterpret_cast<float2*>(&o[g * kD + d]) = make_float2(oacc[nt][0] * f[0], oacc[nt][1] * f[0]);
    *reinterpret_cast<float2*>(&o[(g + 8) * kD + d]) = make_float2(oacc[nt][2] * f[1], oacc[nt][3] * f[1]);
  }
  if (a.lse && tid < kHq) {
    const float M = sm.m_run[tid], L = sm.l_run[tid];
    a.lse[int64_t(s) * kHq + tid] = (M == -INFINITY) ? -INFINITY : M + logf(L);
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

// grid = (R, S): CTA (r, s) takes window chunks [4r/R, 4(r+1)/R) and main
// chunks [m r/R, m (r+1)/R) of segment s (m main chunks), windows first.  The
// window rows, like the queries, are the caller's inputs: the first window
// chunk is staged before the wait on the previous kernel.
__global__ void __launch_bounds__(kAttnThreads, 2) k_attn(AttnArgs a, int R) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  AttnSmem& sm = *reinterpret_cast<AttnSmem*>(smem_raw);
  const int s = blockIdx.y, r = blockIdx.x, tid = threadIdx.x, row = tid & (kChunk - 1);
  const int nmain = attn_main_chunks(a.k);
  const int w0 = kWinChunks * r / R, w1 = kWinChunks * (r + 1) / R;
  const int m0 = int(int64_t(nmain) * r / R), m1 = int(int64_t(nmain) * (r + 1) / R);
  const int nw = w1 - w0, nc = nw + (m1 - m0);
  auto chunk_at = [&](int i) { return i < nw ? nmain + w0 + i : m0 + (i - nw); };
  const int nslots = R;  // one part per CTA: its window rows' output is scaled into the running state
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
  // The queries and the window rows are the caller's inputs, which no kernel
  // of this library writes: they are read while the previous kernel
  // (typically the Top-k selection) still runs.  A kernel that does not
  // trigger its dependents early has completed before this one starts.
  QFrag qf;
  load_q_frag(a, s, (tid >> 5) & 3, qf);
  if (nw > 0) {
    const SegInfo unused{0, -1};  // (window chunks read no cache rows)
    issue_gather(a, sm, 0, s, chunk_at(0), -1, unused);
    sm100::cp_async_commit();
  }
  grid_wait();  // the Top-k ids, lengths and rows may come from the previous kernel
  const SegInfo sg = seg_info(a, s);
  if (nw == 0 && nc > 0) {
    issue_gather(a, sm, 0, s, chunk_at(0), chunk_tpos(a, s, chunk_at(0), row), sg);
    sm100::cp_async_commit();
  }
  int32_t tnext = nc > 1 ? chunk_tpos(a, s, chunk_at(1), row) : -1;
  bool in_win = nw > 0;
  float win_scale = 1.0f;
  for (int i = 0; i < nc; ++i) {
    const int c = chunk_at(i), vb = i & 1;
    const ChunkSrc src = chunk_src(a, s, c);
    if (src.is_win) {
      win_scale = src.kscale;
    } else if (in_win) {  // this CTA's window rows are done: their output takes the window's scale
      scale_acc(oacc, win_scale);
      in_win = false;
    }
    sm100::cp_async_wait<0>();
    __syncthreads();  // this chunk's rows are staged; the last chunk's P V is done
    qk_partial(a, sm, src.is_win, src.nkeys, qf);
    __syncthreads();  // converted rows and partial scores written; the staging buffer is free
    if (i + 1 < nc) {
      issue_gather(a, sm, vb ^ 1, s, chunk_at(i + 1), tnext, sg);
      sm100::cp_async_commit();
      tnext = (i + 2 < nc) ? chunk_tpos(a, s, chunk_at(i + 2), row) : -1;
    }
    softmax_pv(a, sm, vb, oacc, src.nkeys, src.kscale);
  }
  if (in_win) scale_acc(oacc, win_scale);  // (a CTA of window rows only)
  sm100::cp_async_wait<0>();
  if (R == 1) {  // the segment's only CTA: no partial, no combine
    finish_single(a, sm, oacc, s);
    return;
  }
  if (nc > 0) flush_part(a, sm, oacc, s, nslots, r);
  else empty_part(a, s, nslots, r);
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
