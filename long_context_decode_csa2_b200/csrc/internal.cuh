// Internal declarations shared by the CSA2 CUDA sources (sm_100a only).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <string>
#include <utility>

#include "csa2.h"

namespace csa2 {

constexpr int kD = CSA2_MAIN_DIM;      // 512
constexpr int kHq = CSA2_Q_HEADS;      // 16
constexpr int kHi = CSA2_IDX_HEADS;    // 4
constexpr int kDi = CSA2_IDX_DIM;      // 128
constexpr int kBlk = CSA2_BLOCK;       // 8
constexpr int kWin = CSA2_WINDOW;      // 128
constexpr int kIdxCodeBytes = kDi / 2;        // 64
constexpr int kIdxScaleBytes = kDi / 32;      // 4
constexpr int kMainCodeBytes = kD / 2;        // 256
constexpr int kMainScaleBytes = kD / 32;      // 16
constexpr size_t kStatusBytes = 256;          // head of every workspace
// Words of that head: 0 = the device status flags (CSA2_DEV_*); 2 and 3 are
// test controls of the tensor-core kernels, zero (= off) in a zero-filled
// workspace: word 2, if nonzero, replaces their pipeline wait limit (in
// microseconds); word 3, if nonzero, makes each CTA's producer withhold the
// copies of its first work item, so that a wait must run out (tests of the
// timeout path use them).
constexpr int kCtlWaitUs = 2;
constexpr int kCtlWithhold = 3;
// Word 4 is a diagnostic counter: selections that found more than 12288 keys
// in their threshold bucket and fell back to global radix passes add one.
constexpr int kDiagOverfull = 4;

// ---------------------------------------------------------------------------
// Host-side error plumbing (thread-local message, no other global state).
// ---------------------------------------------------------------------------
void set_error(const std::string& msg);
csa2_status fail(csa2_status code, const std::string& msg);
csa2_status check_launch(const char* what);
inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

// Launches `kernel` on `st` with programmatic stream serialisation: it may
// start (and run its prologue up to grid_wait) while the previous kernel of
// the stream finishes.  Errors surface through cudaGetLastError.
template <typename... KArgs, typename... Args>
inline void launch_k(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, Args&&... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}
// launch_k with thread-block clusters of `cluster_x` CTAs along x.
template <typename... KArgs, typename... Args>
inline void launch_k_cluster(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                             int cluster_x, Args&&... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = unsigned(cluster_x);
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}
inline size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
// Row stride (in keys) of the per-block key arrays: whole 16-byte groups, so
// every row starts 16-byte aligned for vector loads.
inline int64_t block_key_stride(int64_t len) { return int64_t(round_up(size_t((len + 7) / 8), 4)); }

// ---------------------------------------------------------------------------
// Segments: a "segment" is one ranking problem (a decode sequence, or one
// prefill query).  Segment s reads cache rows row_off(s) .. + len(s) - 1.
// ---------------------------------------------------------------------------
struct SegDesc {
  const int64_t* row_off;  // [S] or null (then row0 for every segment)
  int64_t row0;
  const int32_t* len;      // [S]
  int64_t max_len;         // host bound
  int64_t cache_rows;      // capacity of the cache
  // paged layout (pages != null): position t of segment s lives in row
  // pages[s * max_pages + (t >> page_shift)] * 2^page_shift + t % 2^page_shift
  const int32_t* pages;
  int page_shift;
  int max_pages;
};

// Selection histograms: one row per segment in the workspace over the top
// bits of the rank keys (15 bits for block keys, 12 bits for the 16384 pool
// candidates, whose row must stay small next to the keys themselves).  The
// kernel that writes the keys adds each present key to its bin; the
// selection reads the row and leaves it zeroed for the next call (the
// workspace starts zero-filled).
constexpr int kSelHistBits = 15;
constexpr int kSelHistBins = 1 << kSelHistBits;
constexpr int kCandHistBits = 12;
constexpr int kCandHistBins = 1 << kCandHistBits;

// ---------------------------------------------------------------------------
// Kernel launchers (each returns after enqueueing on `st`).
// ---------------------------------------------------------------------------
// Tensor-core scan (tcgen05 + TMA): segment checks, work-item prefix
// (tile_start [S+1]), block keys and optional scores.
size_t scan_tc_prefix_ints(int S);
csa2_status launch_scan_tc(const uint8_t* kcodes, const uint8_t* kscales, const SegDesc& sd, int32_t* seg_eff,
                           int32_t* tile_start, int S, const uint8_t* q_codes, const uint8_t* q_scales,
                           const float* w, uint32_t* bkeys, int64_t nb_stride, float* scores, int64_t score_stride,
                           uint32_t* hist, uint32_t* status, cudaStream_t st);

// Scores of pool candidates 8*pool[s][i/8] + i%8 -> keys [S][P*8] (0 = absent),
// on the tensor cores (gathered with cp.async).  seg_eff may be null: the
// kernel then checks each segment's length from sd itself.
csa2_status launch_pool_tc(const uint8_t* kcodes, const uint8_t* kscales, const SegDesc& sd, const int32_t* seg_eff,
                           int S, const uint8_t* q_codes, const uint8_t* q_scales, const float* w,
                           const int32_t* pool, int P, uint32_t* ckeys, uint32_t* hist, uint32_t* status,
                           cudaStream_t st);

// Prefill scan on the tensor cores: block keys [T][nb_stride] of every query
// against the visible prefix (vis[i] entries from row0) of one sequence.
csa2_status launch_prefill_tc(const uint8_t* kcodes, const uint8_t* kscales, int64_t row0, int64_t cache_rows,
                              const int32_t* vis, int T, int64_t max_vis, const uint8_t* q_codes,
                              const uint8_t* q_scales, const float* w, uint32_t* bkeys, int64_t nb_stride,
                              uint32_t* status, cudaStream_t st);

// Multi-query scan (a batch of sequences with a few queries each): the group
// table (at most multi_group_bound(B, Q) groups of <= 8 queries of one
// sequence) with its real group count, each query's first cache row and
// checked visible count, then the block keys [Q][nb_stride] of every query on
// the tensor cores (work split over the real groups only).
int multi_group_bound(int B, int Q);
void launch_multi_prep(const int64_t* seq_row_off, const int32_t* q_off, const int32_t* q_vis, int B, int Q, int G,
                       int64_t max_vis, int64_t cache_rows, int4* groups, int64_t* q_row_off, int32_t* vis,
                       int32_t* n_groups, uint32_t* status, cudaStream_t st);
csa2_status launch_multi_tc(const uint8_t* kcodes, const uint8_t* kscales, int64_t cache_rows,
                            const int64_t* seq_row_off, const int4* groups, int G, const int32_t* n_groups,
                            const int32_t* vis, int Q,
                            int64_t max_vis, const uint8_t* q_codes, const uint8_t* q_scales, const float* w,
                            uint32_t* bkeys, int64_t nb_stride, uint32_t* status, cudaStream_t st);

// Context-parallel pieces (cp_kernels.cu): exact keys of listed positions
// (blk 1) or blocks (blk 8); shards' candidate lists [G][B][n] -> [B][G*n]
// with global ids; ids inside [lo, hi) made local; lse-weighted merge of
// attention partials [G][B].
void launch_score_positions(const uint8_t* kcodes, const uint8_t* kscales, const SegDesc& sd, const uint8_t* q_codes,
                            const uint8_t* q_scales, const float* w, const int32_t* ids, int B, int n, int blk,
                            uint32_t* keys_out, uint32_t* status, cudaStream_t st);
void launch_merge_gather(const uint32_t* keys, const int32_t* ids, const int64_t* src_off, int G, int B, int n,
                         uint32_t* keys_t, int32_t* ids_t, uint32_t* status, cudaStream_t st);
void launch_localize(const int32_t* out, int B, int k, const int64_t* lo, const int64_t* hi, int32_t* out_local,
                     cudaStream_t st);
void launch_attn_combine(const float* out_parts, const float* lse_parts, int G, int B, float* out, float* lse,
                         cudaStream_t st);

// Visible entry counts of prefill queries.
void launch_prefill_vis(const int32_t* q_pos, int T, int ratio, int64_t n_entries, int32_t* vis, uint32_t* status,
                        cudaStream_t st);

// Selection: per segment the k best of n keys (0 = absent) by (key desc,
// index asc), written ascending.  Input kinds below.
enum SelectKind : int {
  kSelBlockKeys = 0,  // u32 keys, n = ceil(seg_eff/8), id = index
  kSelScores = 1,     // fp32 scores, n = seg_eff, id = index
  kSelPoolCand = 2,   // u32 keys, n = P*8, id = 8*pool[i/8] + i%8
  kSelExplicit = 3,   // u32 keys, n = P, id = pool[i] (ids ascending with i)
};
// `hist` (or null): the keys' histogram rows, zeroed on return: [S][kSelHistBins]
// for block keys, [S][kCandHistBins] for pool candidates.
// `status` (or null): the workspace's status block (diagnostic counter).
// Block-key selections (the pool, k = its size) may also write the best `kb`
// blocks of every pool, ascending, into topblk [S][kb]: the blocks that hold
// every one of the segment's kb best positions.
void launch_select(SelectKind kind, const void* in, int64_t in_stride, const int32_t* seg_eff, int S, int P,
                   const int32_t* pool, int k, int32_t* out, uint32_t* hist, cudaStream_t st,
                   uint32_t* status = nullptr, int32_t* topblk = nullptr, int kb = 0);

// Attention partials + combine.
struct AttnArgs {
  const uint16_t* q;            // [S][16][512] bf16
  const uint8_t* mcodes;
  const uint8_t* mscales;
  SegDesc sd;                   // rows of segment s (len = visible count)
  const int32_t* seg_eff;       // checked visible count, or null: checked from sd in the kernel
  const int32_t* topk;          // [S][k]
  int k;
  // decode window
  const uint8_t* win;           // [S][128][512] or null
  const float* win_scale;       // [S]
  const int32_t* win_len;       // [S]
  // prefill window
  const int32_t* q_pos;         // [S] or null
  const uint8_t* raw_win;       // [n_raw][512]
  int64_t n_raw;
  float raw_scale;
  float sm_scale;
  float* out;                   // [S][16][512]
  float* lse;                   // [S][16] or null
  float* partial;               // workspace
  int32_t* counters;            // [S] arrival counters, zero between calls
  uint32_t* status;
  int S;
};
int attn_num_chunks(int k);
size_t attn_partial_bytes(int S, int k);
void launch_attention(const AttnArgs& a, cudaStream_t st);
// Loads the attention kernel on the current device and sets its launch
// attributes (launch_attention does this itself).
void prepare_attention();

// Compression + MXFP4 encode.
struct CompressArgs {
  uint8_t* mcodes;
  uint8_t* mscales;
  int64_t mrows;
  uint8_t* icodes;
  uint8_t* iscales;
  int64_t irows;
  const uint16_t* raw;
  const float* logits;
  const float* w_idx;
  const uint16_t* idx_raw;
  const int64_t* tok_off;
  const int64_t* seq_row_off;
  const int32_t* seq_len_in;
  int32_t* seq_len_out;
  int B;
  int ratio;
  int64_t max_new;
  uint32_t* status;
  // streaming mode (pend_n != null): the pending half-pair of every sequence
  int32_t* pend_n;       // [B] 0 or 1, read and written
  uint16_t* pend_raw;    // [B][512] bf16
  float* pend_logit;     // [B]
  uint16_t* pend_idx;    // [B][128] bf16, or null (W_idx projection)
  uint32_t* arrive;      // [B] arrival counters, zero between calls
  // paged layout (pages != null; then seq_row_off is unused)
  const int32_t* pages;  // [B][max_pages]
  int page_shift;
  int max_pages;
};
void launch_compress(const CompressArgs& a, cudaStream_t st);

}  // namespace csa2
