// C ABI entry points of the CSA2 library: host-side validation, workspace
// carving, and the launch sequence of each call (all on the caller's stream).
#include <cstdio>
#include <string>

#include "internal.cuh"

namespace csa2 {

namespace {
thread_local std::string g_last_error;
}

void set_error(const std::string& msg) { g_last_error = msg; }

csa2_status fail(csa2_status code, const std::string& msg) {
  set_error(msg);
  return code;
}

csa2_status check_launch(const char* what) {
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(CSA2_ERR_CUDA, std::string(what) + ": " + cudaGetErrorString(e));
  return CSA2_OK;
}

// Sequential carving of a workspace into 256-byte aligned pieces.
struct Carve {
  char* base;
  size_t used;
  explicit Carve(void* ws) : base(static_cast<char*>(ws)), used(0) {}
  template <class T>
  T* take(size_t count) {
    T* p = reinterpret_cast<T*>(base ? base + used : nullptr);
    used = round_up(used + count * sizeof(T), 256);
    return p;
  }
};

bool cache_ok(const csa2_mxfp4_cache& c) {
  return c.codes && c.scales && aligned16(c.codes) && aligned16(c.scales) && c.rows >= 0 && (c.rows % 8) == 0;
}

// Paged layout arguments: page_rows a power of two in [512, 2^24] (a scan
// item of 512 rows never crosses a page), every cache a whole number of
// pages.  Sets *shift = log2(page_rows).
bool pages_ok(const int32_t* pages, int page_rows, int max_pages, int64_t rows_a, int64_t rows_b, int* shift) {
  if (!pages || (reinterpret_cast<uintptr_t>(pages) & 3) || max_pages < 1) return false;
  if (page_rows < 512 || page_rows > (1 << 24) || (page_rows & (page_rows - 1))) return false;
  if (rows_a % page_rows != 0 || rows_b % page_rows != 0) return false;
  int sh = 0;
  while ((1 << sh) < page_rows) ++sh;
  *shift = sh;
  return true;
}

SegDesc paged_desc(const int32_t* pages, int shift, int max_pages, const int32_t* len, int64_t max_len,
                   int64_t cache_rows) {
  SegDesc sd{nullptr, 0, len, max_len, cache_rows};
  sd.pages = pages;
  sd.page_shift = shift;
  sd.max_pages = max_pages;
  return sd;
}

struct IndexFullWs {
  uint32_t* status;
  int32_t* seg_eff;
  int32_t* tile_start;
  uint32_t* bkeys;
  uint32_t* ckeys;
  int32_t* topblk;  // [B][k]: the best k blocks of every pool (when P >= k)
  float* scores;
  uint32_t* hist;  // [B][kSelHistBins] (block keys, then candidates), zero between calls
  size_t bytes;
};

IndexFullWs index_full_ws(void* ws, int B, int max_len, int P, int k, bool need_scores) {
  Carve c(ws);
  IndexFullWs w;
  w.status = c.take<uint32_t>(kStatusBytes / 4);
  w.seg_eff = c.take<int32_t>(size_t(B));
  w.tile_start = c.take<int32_t>(scan_tc_prefix_ints(B));
  const size_t nb = size_t(block_key_stride(max_len));
  w.bkeys = c.take<uint32_t>(size_t(B) * nb);
  w.ckeys = (P >= k) ? c.take<uint32_t>(size_t(B) * k * kBlk) : nullptr;
  w.topblk = (P >= k) ? c.take<int32_t>(size_t(B) * k) : nullptr;
  w.scores = need_scores ? c.take<float>(size_t(B) * max_len) : nullptr;
  w.hist = c.take<uint32_t>(size_t(B) * kSelHistBins);
  w.bytes = c.used;
  return w;
}

}  // namespace csa2

using namespace csa2;

extern "C" {

const char* csa2_status_string(csa2_status s) {
  switch (s) {
    case CSA2_OK: return "ok";
    case CSA2_ERR_INVALID_ARG: return "invalid argument";
    case CSA2_ERR_UNSUPPORTED: return "unsupported";
    case CSA2_ERR_WORKSPACE: return "workspace too small";
    case CSA2_ERR_CUDA: return "CUDA error";
    case CSA2_ERR_DEVICE_CHECK: return "device check failed";
    default: return "unknown status";
  }
}

const char* csa2_last_error(void) { return g_last_error.c_str(); }

csa2_status csa2_device_status(void* workspace, void* stream, uint32_t* flags) {
  if (!workspace || !flags) return fail(CSA2_ERR_INVALID_ARG, "csa2_device_status: null argument");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint32_t h = 0;
  cudaError_t e = cudaMemcpyAsync(&h, workspace, sizeof(h), cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e == cudaSuccess) e = cudaMemsetAsync(workspace, 0, sizeof(h), st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return fail(CSA2_ERR_CUDA, std::string("csa2_device_status: ") + cudaGetErrorString(e));
  *flags = h;
  return h ? CSA2_ERR_DEVICE_CHECK : CSA2_OK;
}

// ---------------------------------------------------------------------------
size_t csa2_index_full_workspace_bytes(int B, int max_len, int pool_blocks, int k) {
  if (B < 0 || max_len < 0) return 0;
  return index_full_ws(nullptr, B, max_len, pool_blocks, k, pool_blocks < k).bytes;
}

namespace {
// phases: 1 = scan + block pool, 2 = Top-k (from the workspace state phase 1
// left), 3 = both
csa2_status index_full_impl(const char* fn, csa2_mxfp4_cache idx_k, const uint8_t* q_codes, const uint8_t* q_scales,
                            const float* w, SegDesc sd, int B, int max_len, int pool_blocks, int k, int32_t* pool_out,
                            int32_t* topk_out, float* scores_out, void* workspace, size_t workspace_bytes,
                            void* stream, int phases = 3) {
  if (!q_codes || !q_scales || !w || !sd.len || !pool_out || (!topk_out && (phases & 2)) || !workspace)
    return fail(CSA2_ERR_INVALID_ARG, std::string(fn) + ": null pointer");
  if (!aligned16(q_codes) || (reinterpret_cast<uintptr_t>(workspace) & 255))
    return fail(CSA2_ERR_INVALID_ARG, std::string(fn) + ": q_codes must be 16-byte and workspace 256-byte aligned");
  const bool need_scores = pool_blocks < k && scores_out == nullptr;
  IndexFullWs ws = index_full_ws(workspace, B, max_len, pool_blocks, k, need_scores);
  if (workspace_bytes < ws.bytes) return fail(CSA2_ERR_WORKSPACE, std::string(fn) + ": workspace too small");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int64_t nb = block_key_stride(max_len);
  float* scores = scores_out ? scores_out : ws.scores;
  if (phases & 1) {
    const csa2_status rc = launch_scan_tc(idx_k.codes, idx_k.scales, sd, ws.seg_eff, ws.tile_start, B, q_codes,
                                          q_scales, w, ws.bkeys, nb, scores, max_len, ws.hist, ws.status, st);
    if (rc != CSA2_OK) return rc;
    // the pool, and (P >= k) the best k blocks among it
    launch_select(kSelBlockKeys, ws.bkeys, nb, ws.seg_eff, B, 0, nullptr, pool_blocks, pool_out, ws.hist, st,
                  ws.status, ws.topblk, k);
  }
  if (!(phases & 2)) return check_launch(fn);
  if (pool_blocks >= k) {
    // Every Top-k position's block ranks within the first k blocks, so the
    // Top-k over the positions of those blocks equals the Top-k over all
    // positions: re-score their 8k positions and select.
    const csa2_status rc2 = launch_pool_tc(idx_k.codes, idx_k.scales, sd, ws.seg_eff, B, q_codes, q_scales, w,
                                           ws.topblk, k, ws.ckeys, ws.hist, ws.status, st);
    if (rc2 != CSA2_OK) return rc2;
    launch_select(kSelPoolCand, ws.ckeys, int64_t(k) * kBlk, ws.seg_eff, B, k, ws.topblk, k, topk_out, ws.hist, st);
  } else {
    launch_select(kSelScores, scores, max_len, ws.seg_eff, B, 0, nullptr, k, topk_out, nullptr, st, ws.status);
  }
  return check_launch(fn);
}

csa2_status index_full_args(const char* fn, const csa2_mxfp4_cache& idx_k, int B, int max_len, int pool_blocks,
                            int k) {
  if (B < 0 || max_len < 0) return fail(CSA2_ERR_INVALID_ARG, std::string(fn) + ": negative size");
  if (pool_blocks < 1 || pool_blocks > CSA2_MAX_POOL_BLOCKS || k < 1 || k > CSA2_MAX_TOPK)
    return fail(CSA2_ERR_INVALID_ARG, std::string(fn) + ": pool_blocks and k must be in 1..2048");
  if (B > 0 && !cache_ok(idx_k)) return fail(CSA2_ERR_INVALID_ARG, std::string(fn) + ": bad indexer-K cache");
  return CSA2_OK;
}
}  // namespace

csa2_status csa2_index_full(csa2_mxfp4_cache idx_k, const uint8_t* q_codes, const uint8_t* q_scales, const float* w,
                            const int64_t* seq_row_off, const int32_t* seq_len, int B, int max_len,
                            int pool_blocks, int k, int32_t* pool_out, int32_t* topk_out, float* scores_out,
                            void* workspace, size_t workspace_bytes, void* stream) {
  const char* fn = "csa2_index_full";
  const csa2_status rc = index_full_args(fn, idx_k, B, max_len, pool_blocks, k);
  if (rc != CSA2_OK || B == 0) return rc;
  if (!seq_row_off) return fail(CSA2_ERR_INVALID_ARG, std::string(fn) + ": null pointer");
  return index_full_impl(fn, idx_k, q_codes, q_scales, w, SegDesc{seq_row_off, 0, seq_len, max_len, idx_k.rows}, B,
                         max_len, pool_blocks, k, pool_out, topk_out, scores_out, workspace, workspace_bytes, stream);
}

csa2_status csa2_index_full_pool(csa2_mxfp4_cache idx_k, const uint8_t* q_codes, const uint8_t* q_scales,
                                 const float* w, const int64_t* seq_row_off, const int32_t* seq_len, int B,
                                 int max_len, int pool_blocks, int k, int32_t* pool_out, float* scores_out,
                                 void* workspace, size_t workspace_bytes, void* stream) {
  const char* fn = "csa2_index_full_pool";
  const csa2_status rc = index_full_args(fn, idx_k, B, max_len, pool_blocks, k);
  if (rc != CSA2_OK || B == 0) return rc;
  if (!seq_row_off) return fail(CSA2_ERR_INVALID_ARG, std::string(fn) + ": null pointer");
  return index_full_impl(fn, idx_k, q_codes, q_scales, w, SegDesc{seq_row_off, 0, seq_len, max_len, idx_k.rows}, B,
                         max_len, pool_blocks, k, pool_out, nullptr, scores_out, workspace, workspace_bytes, stream,
                         1);
}

csa2_status csa2_index_full_topk(csa2_mxfp4_cache idx_k, const uint8_t* q_codes, const uint8_t* q_scales,
                                 const float* w, const int64_t* seq_row_off, const int32_t* seq_len, int B,
                                 int max_len, int pool_blocks, int k, const int32_t* pool, int32_t* topk_out,
                                 float* scores_out, void* workspace, size_t workspace_bytes, void* stream) {
  const char* fn = "csa2_index_full_topk";
  const csa2_status rc = index_full_args(fn, idx_k, B, max_len, pool_blocks, k);
  if (rc != CSA2_OK || B == 0) return rc;
  if (!seq_row_off) return fail(CSA2_ERR_INVALID_ARG, std::string(fn) + ": null pointer");
  return index_full_impl(fn, idx_k, q_codes, q_scales, w, SegDesc{seq_row_off, 0, seq_len, max_len, idx_k.rows}, B,
                         max_len, pool_blocks, k, const_cast<int32_t*>(pool), topk_out, scores_out, workspace,
                         workspace_bytes, stream, 2);
}

csa2_status csa2_index_full_paged(csa2_mxfp4_cache idx_k, const uint8_t* q_codes, const uint8_t* q_scales,
                                  const float* w, const int32_t* pages, int page_rows, int max_pages,
                                  const int32_t* seq_len, int B, int max_len, int pool_blocks, int k,
                                  int32_t* pool_out, int32_t* topk_out, float* scores_out, void* workspace,
                                  size_t workspace_bytes, void* stream) {
  const char* fn = "csa2_index_full_paged";
  const csa2_status rc = index_full_args(fn, idx_k, B, max_len, pool_blocks, k);
  if (rc != CSA2_OK || B == 0) return rc;
  int shift = 0;
  if (!pages_ok(pages, page_rows, max_pages, idx_k.rows, idx_k.rows, &shift))
    return fail(CSA2_ERR_INVALID_ARG, std::string(fn) + ": bad page table or page size");
  return index_full_impl(fn, idx_k, q_codes, q_scales, w,
                         paged_desc(pages, shift, max_pages, seq_len, max_len, idx_k.rows), B, max_len, pool_blocks,
                         k, pool_out, topk_out, scores_out, workspace, workspace_bytes, stream);
}

// ---------------------------------------------------------------------------
size_t csa2_index_reindex_workspace_bytes(int B, int pool_blocks, int k) {
  (void)k;
  Carve c(nullptr);
  c.take<uint32_t>(kStatusBytes / 4);
  c.take<int32_t>(size_t(B));
  c.take<uint32_t>(size_t(B) * pool_blocks * kBlk);
  c.take<uint32_t>(size_t(B) * kCandHistBins);
  return c.used;
}

namespace {
csa2_status reindex_args(const char* fn, const csa2_mxfp4_cache& idx_k, int B, int pool_blocks, int k) {
  if (B < 0) return fail(CSA2_ERR_INVALID_ARG, std::string(fn) + ": negative size");
  if (pool_blocks < 1 || pool_blocks > CSA2_MAX_POOL_BLOCKS || k < 1 || k > CSA2_MAX_TOPK)
    return fail(CSA2_ERR_INVALID_ARG, std::string(fn) + ": pool_blocks and k must be in 1..2048");
  if (B > 0 && !cache_ok(idx_k)) return fail(CSA2_ERR_INVALID_ARG, std::string(fn) + ": bad indexer-K cache");
  return CSA2_OK;
}

csa2_status reindex_impl(const char* fn, csa2_mxfp4_cache idx_k, const uint8_t* q_codes, const uint8_t* q_scales,
                         const float* w, SegDesc sd, const int32_t* pool, int B, int pool_blocks, int k,
                         int32_t* topk_out, void* workspace, size_t workspace_bytes, void* stream) {
  if (!q_codes || !q_scales || !w || !sd.len || !pool || !topk_out || !workspace)
    return fail(CSA2_ERR_INVALID_ARG, std::string(fn) + ": null pointer");
  if (reinterpret_cast<uintptr_t>(workspace) & 255)
    return fail(CSA2_ERR_INVALID_ARG, std::string(fn) + ": workspace must be 256-byte aligned");
  if (workspace_bytes < csa2_index_reindex_workspace_bytes(B, pool_blocks, k))
    return fail(CSA2_ERR_WORKSPACE, std::string(fn) + ": workspace too small");
  Carve c(workspace);
  uint32_t* status = c.take<uint32_t>(kStatusBytes / 4);
  int32_t* seg_eff = c.take<int32_t>(size_t(B));
  uint32_t* ckeys = c.take<uint32_t>(size_t(B) * pool_blocks * kBlk);
  uint32_t* hist = c.take<uint32_t>(size_t(B) * kCandHistBins);  // zero between calls
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  (void)seg_eff;  // lengths are checked inside the kernels
  const csa2_status rc = launch_pool_tc(idx_k.codes, idx_k.scales, sd, nullptr, B, q_codes, q_scales, w, pool,
                                        pool_blocks, ckeys, hist, status, st);
  if (rc != CSA2_OK) return rc;
  launch_select(kSelPoolCand, ckeys, int64_t(pool_blocks) * kBlk, nullptr, B, pool_blocks, pool, k, topk_out, hist,
                st);
  return check_launch(fn);
}
}  // namespace

csa2_status csa2_index_reindex(csa2_mxfp4_cache idx_k, const uint8_t* q_codes, const uint8_t* q_scales,
                               const float* w, const int64_t* seq_row_off, const int32_t* seq_len,
                               const int32_t* pool, int B, int pool_blocks, int k, int32_t* topk_out,
                               void* workspace, size_t workspace_bytes, void* stream) {
  const char* fn = "csa2_index_reindex";
  const csa2_status rc = reindex_args(fn, idx_k, B, pool_blocks, k);
  if (rc != CSA2_OK || B == 0) return rc;
  if (!seq_row_off) return fail(CSA2_ERR_INVALID_ARG, std::string(fn) + ": null pointer");
  return reindex_impl(fn, idx_k, q_codes, q_scales, w, SegDesc{seq_row_off, 0, seq_len, INT32_MAX, idx_k.rows}, pool,
                      B, pool_blocks, k, topk_out, workspace, workspace_bytes, stream);
}

csa2_status csa2_index_reindex_paged(csa2_mxfp4_cache idx_k, const uint8_t* q_codes, const uint8_t* q_scales,
                                     const float* w, const int32_t* pages, int page_rows, int max_pages,
                                     const int32_t* seq_len, const int32_t* pool, int B, int pool_blocks, int k,
                                     int32_t* topk_out, void* workspace, size_t workspace_bytes, void* stream) {
  const char* fn = "csa2_index_reindex_paged";
  const csa2_status rc = reindex_args(fn, idx_k, B, pool_blocks, k);
  if (rc != CSA2_OK || B == 0) return rc;
  int shift = 0;
  if (!pages_ok(pages, page_rows, max_pages, idx_k.rows, idx_k.rows, &shift))
    return fail(CSA2_ERR_INVALID_ARG, std::string(fn) + ": bad page table or page size");
  return reindex_impl(fn, idx_k, q_codes, q_scales, w, paged_desc(pages, shift, max_pages, seq_len, INT32_MAX, idx_k.rows),
                      pool, B, pool_blocks, k, topk_out, workspace, workspace_bytes, stream);
}

// ---------------------------------------------------------------------------
size_t csa2_sparse_attn_decode_workspace_bytes(int B, int k) {
  Carve c(nullptr);
  c.take<uint32_t>(kStatusBytes / 4);
  c.take<int32_t>(size_t(B));
  c.take<int32_t>(size_t(B));
  c.take<char>(attn_partial_bytes(B, k));
  return c.used;
}

namespace {
csa2_status attn_decode_args(const char* fn, const csa2_mxfp4_cache& main_kv, int B, int k) {
  if (B < 0 || k < 1 || k > CSA2_MAX_TOPK) return fail(CSA2_ERR_INVALID_ARG, std::string(fn) + ": bad B or k");
  if (B > 0 && !cache_ok(main_kv)) return fail(CSA2_ERR_INVALID_ARG, std::string(fn) + ": bad main-KV cache");
  return CSA2_OK;
}

csa2_status attn_decode_impl(const char* fn, const uint16_t* q, csa2_mxfp4_cache main_kv, SegDesc sd,
                             const int32_t* topk, int k, const uint8_t* win, const float* win_scale,
                             const int32_t* win_len, float sm_scale, float* out, float* lse, int B, void* workspace,
                             size_t workspace_bytes, void* stream) {
  if (!q || !sd.len || !topk || !win || !win_scale || !win_len || !out || !workspace)
    return fail(CSA2_ERR_INVALID_ARG, std::string(fn) + ": null pointer");
  if (!aligned16(win) || !aligned16(q) || (reinterpret_cast<uintptr_t>(workspace) & 255))
    return fail(CSA2_ERR_INVALID_ARG, std::string(fn) + ": q/win must be 16-byte, workspace 256-byte aligned");
  if (workspace_bytes < csa2_sparse_attn_decode_workspace_bytes(B, k))
    return fail(CSA2_ERR_WORKSPACE, std::string(fn) + ": workspace too small");
  Carve c(workspace);
  AttnArgs a{};
  a.status = c.take<uint32_t>(kStatusBytes / 4);
  int32_t* seg_eff = c.take<int32_t>(size_t(B));
  a.counters = c.take<int32_t>(size_t(B));
  a.partial = reinterpret_cast<float*>(c.take<char>(attn_partial_bytes(B, k)));
  a.q = q;
  a.mcodes = main_kv.codes;
  a.mscales = main_kv.scales;
  a.sd = sd;
  a.seg_eff = nullptr;  // checked per segment inside the kernel
  (void)seg_eff;
  a.topk = topk;
  a.k = k;
  a.win = win;
  a.win_scale = win_scale;
  a.win_len = win_len;
  a.sm_scale = sm_scale;
  a.out = out;
  a.lse = lse;
  a.S = B;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  launch_attention(a, st);
  return check_launch(fn);
}
}  // namespace

csa2_status csa2_sparse_attn_decode(const uint16_t* q, csa2_mxfp4_cache main_kv, const int64_t* seq_row_off,
                                    const int32_t* seq_len, const int32_t* topk, int k, const uint8_t* win,
                                    const float* win_scale, const int32_t* win_len, float sm_scale, float* out,
                                    float* lse, int B, void* workspace, size_t workspace_bytes, void* stream) {
  const char* fn = "csa2_sparse_attn_decode";
  const csa2_status rc = attn_decode_args(fn, main_kv, B, k);
  if (rc != CSA2_OK || B == 0) return rc;
  if (!seq_row_off) return fail(CSA2_ERR_INVALID_ARG, std::string(fn) + ": null pointer");
  return attn_decode_impl(fn, q, main_kv, SegDesc{seq_row_off, 0, seq_len, INT32_MAX, main_kv.rows}, topk, k, win,
                          win_scale, win_len, sm_scale, out, lse, B, workspace, workspace_bytes, stream);
}

csa2_status csa2_sparse_attn_decode_paged(const uint16_t* q, csa2_mxfp4_cache main_kv, const int32_t* pages,
                                          int page_rows, int max_pages, const int32_t* seq_len, const int32_t* topk,
                                          int k, const uint8_t* win, const float* win_scale, const int32_t* win_len,
                                          float sm_scale, float* out, float* lse, int B, void* workspace,
                                          size_t workspace_bytes, void* stream) {
  const char* fn = "csa2_sparse_attn_decode_paged";
  const csa2_status rc = attn_decode_args(fn, main_kv, B, k);
  if (rc != CSA2_OK || B == 0) return rc;
  int shift = 0;
  if (!pages_ok(pages, page_rows, max_pages, main_kv.rows, main_kv.rows, &shift))
    return fail(CSA2_ERR_INVALID_ARG, std::string(fn) + ": bad page table or page size");
  return attn_decode_impl(fn, q, main_kv, paged_desc(pages, shift, max_pages, seq_len, INT32_MAX, main_kv.rows), topk,
                          k, win, win_scale, win_len, sm_scale, out, lse, B, workspace, workspace_bytes, stream);
}

// ---------------------------------------------------------------------------
size_t csa2_compress_append_workspace_bytes(int B) {
  (void)B;
  return kStatusBytes;
}

csa2_status csa2_compress_append(csa2_mxfp4_cache main_kv, csa2_mxfp4_cache idx_k, const uint16_t* raw,
                                 const float* logits, const float* w_idx, const uint16_t* idx_raw,
                                 const int64_t* tok_off, const int64_t* seq_row_off, const int32_t* seq_len_in,
                                 int32_t* seq_len_out, int B, int ratio, int64_t n_tok, int64_t max_new,
                                 void* workspace, size_t workspace_bytes, void* stream) {
  const char* fn = "csa2_compress_append";
  if (B < 0 || n_tok < 0 || max_new < 0) return fail(CSA2_ERR_INVALID_ARG, std::string(fn) + ": negative size");
  if (ratio != 1 && ratio != 2) return fail(CSA2_ERR_INVALID_ARG, std::string(fn) + ": ratio must be 1 or 2");
  if (B == 0) return CSA2_OK;
  if (!cache_ok(main_kv) || !cache_ok(idx_k)) return fail(CSA2_ERR_INVALID_ARG, std::string(fn) + ": bad cache");
  if (!raw || !tok_off || !seq_row_off || !seq_len_in || !seq_len_out || !workspace)
    return fail(CSA2_ERR_INVALID_ARG, std::string(fn) + ": null pointer");
  if (ratio == 2 && !logits) return fail(CSA2_ERR_INVALID_ARG, std::string(fn) + ": ratio 2 needs logits");
  if ((w_idx == nullptr) == (idx_raw == nullptr))
    return fail(CSA2_ERR_INVALID_ARG, std::string(fn) + ": give exactly one of w_idx and idx_raw");
  if (!aligned16(raw) || (idx_raw && (reinterpret_cast<uintptr_t>(idx_raw) & 7)) ||
      (w_idx && (reinterpret_cast<uintptr_t>(w_idx) & 7)))
    return fail(CSA2_ERR_INVALID_ARG, std::string(fn) + ": raw must be 16-byte, idx_raw and w_idx 8-byte aligned");
  if (reinterpret_cast<uintptr_t>(workspace) & 255)
    return fail(CSA2_ERR_INVALID_ARG, std::string(fn) + ": workspace must be 256-byte aligned");
  if (workspace_bytes < csa2_compress_append_workspace_bytes(B))
    return fail(CSA2_ERR_WORKSPACE, std::string(fn) + ": workspace too small");
  CompressArgs a{};
  a.mcodes = main_kv.codes;
  a.mscales = main_kv.scales;
  a.mrows = main_kv.rows;
  a.icodes = idx_k.codes;
  a.iscales = idx_k.scales;
  a.irows = idx_k.rows;
  a.raw = raw;
  a.logits = logits;
  a.w_idx = w_idx;
  a.idx_raw = idx_raw;
  a.tok_off = tok_off;
  a.seq_row_off = seq_row_off;
  a.seq_len_in = seq_len_in;
  a.seq_len_out = seq_len_out;
  a.B = B;
  a.ratio = ratio;
  a.max_new = max_new;
  a.status = static_cast<uint32_t*>(workspace);
  launch_compress(a, static_cast<cudaStream_t>(stream));
  return check_launch(fn);
}

size_t csa2_compress_stream_workspace_bytes(int B) {
  return kStatusBytes + round_up(size_t(B > 0 ? B : 0) * sizeof(uint32_t), 256);
}

namespace {
// seq_row_off (contiguous layout) or pages / shift / max_pages (paged)
csa2_status compress_stream_impl(const char* fn, csa2_mxfp4_cache main_kv, csa2_mxfp4_cache idx_k,
                                 const uint16_t* raw, const float* logits, const float* w_idx,
                                 const uint16_t* idx_raw, const int64_t* tok_off, const int64_t* seq_row_off,
                                 const int32_t* pages, int shift, int max_pages, const int32_t* seq_len_in,
                                 int32_t* seq_len_out, int32_t* pend_n, uint16_t* pend_raw, float* pend_logit,
                                 uint16_t* pend_idx, int B, int64_t n_tok, int64_t max_new, void* workspace,
                                 size_t workspace_bytes, void* stream) {
  if (!tok_off || !(seq_row_off || pages) || !seq_len_in || !pend_n || !pend_raw || !pend_logit || !logits ||
      !workspace)
    return fail(CSA2_ERR_INVALID_ARG, std::string(fn) + ": null pointer");
  if (n_tok > 0 && !raw) return fail(CSA2_ERR_INVALID_ARG, std::string(fn) + ": null raw");
  if ((w_idx == nullptr) == (idx_raw == nullptr && pend_idx == nullptr))
    return fail(CSA2_ERR_INVALID_ARG, std::string(fn) + ": give w_idx, or idx_raw with pend_idx");
  if (w_idx && (idx_raw || pend_idx))
    return fail(CSA2_ERR_INVALID_ARG, std::string(fn) + ": w_idx excludes idx_raw and pend_idx");
  if (!w_idx && (!pend_idx || (n_tok > 0 && !idx_raw)))
    return fail(CSA2_ERR_INVALID_ARG, std::string(fn) + ": idx_raw needs pend_idx");
  if ((raw && !aligned16(raw)) || !aligned16(pend_raw) || (idx_raw && (reinterpret_cast<uintptr_t>(idx_raw) & 7)) ||
      (pend_idx && (reinterpret_cast<uintptr_t>(pend_idx) & 7)) || (w_idx && (reinterpret_cast<uintptr_t>(w_idx) & 7)))
    return fail(CSA2_ERR_INVALID_ARG,
                std::string(fn) + ": raw and pend_raw must be 16-byte, idx_raw, pend_idx and w_idx 8-byte aligned");
  if (reinterpret_cast<uintptr_t>(workspace) & 255)
    return fail(CSA2_ERR_INVALID_ARG, std::string(fn) + ": workspace must be 256-byte aligned");
  if (workspace_bytes < csa2_compress_stream_workspace_bytes(B))
    return fail(CSA2_ERR_WORKSPACE, std::string(fn) + ": workspace too small");
  CompressArgs a{};
  a.mcodes = main_kv.codes;
  a.mscales = main_kv.scales;
  a.mrows = main_kv.rows;
  a.icodes = idx_k.codes;
  a.iscales = idx_k.scales;
  a.irows = idx_k.rows;
  a.raw = raw;
  a.logits = logits;
  a.w_idx = w_idx;
  a.idx_raw = idx_raw;
  a.tok_off = tok_off;
  a.seq_row_off = seq_row_off;
  a.seq_len_in = seq_len_in;
  a.seq_len_out = seq_len_out;
  a.B = B;
  a.ratio = 2;
  a.max_new = max_new;
  a.status = static_cast<uint32_t*>(workspace);
  a.pend_n = pend_n;
  a.pend_raw = pend_raw;
  a.pend_logit = pend_logit;
  a.pend_idx = pend_idx;
  a.arrive = reinterpret_cast<uint32_t*>(static_cast<char*>(workspace) + kStatusBytes);
  a.pages = pages;
  a.page_shift = shift;
  a.max_pages = max_pages;
  launch_compress(a, static_cast<cudaStream_t>(stream));
  return check_launch(fn);
}

csa2_status compress_stream_args(const char* fn, const csa2_mxfp4_cache& main_kv, const csa2_mxfp4_cache& idx_k,
                                 int B, int64_t n_tok, int64_t max_new) {
  if (B < 0 || n_tok < 0 || max_new < 0) return fail(CSA2_ERR_INVALID_ARG, std::string(fn) + ": negative size");
  if (B > 0 && (!cache_ok(main_kv) || !cache_ok(idx_k)))
    return fail(CSA2_ERR_INVALID_ARG, std::string(fn) + ": bad cache");
  return CSA2_OK;
}
}  // namespace

csa2_status csa2_compress_stream(csa2_mxfp4_cache main_kv, csa2_mxfp4_cache idx_k, const uint16_t* raw,
                                 const float* logits, const float* w_idx, const uint16_t* idx_raw,
                                 const int64_t* tok_off, const int64_t* seq_row_off, const int32_t* seq_len_in,
                                 int32_t* seq_len_out, int32_t* pend_n, uint16_t* pend_raw, float* pend_logit,
                                 uint16_t* pend_idx, int B, int64_t n_tok, int64_t max_new, void* workspace,
                                 size_t workspace_bytes, void* stream) {
  const char* fn = "csa2_compress_stream";
  const csa2_status rc = compress_stream_args(fn, main_kv, idx_k, B, n_tok, max_new);
  if (rc != CSA2_OK || B == 0) return rc;
  if (!seq_row_off) return fail(CSA2_ERR_INVALID_ARG, std::string(fn) + ": null pointer");
  return compress_stream_impl(fn, main_kv, idx_k, raw, logits, w_idx, idx_raw, tok_off, seq_row_off, nullptr, 0, 0,
                              seq_len_in, seq_len_out, pend_n, pend_raw, pend_logit, pend_idx, B, n_tok, max_new,
                              workspace, workspace_bytes, stream);
}

csa2_status csa2_compress_stream_paged(csa2_mxfp4_cache main_kv, csa2_mxfp4_cache idx_k, const uint16_t* raw,
                                       const float* logits, const float* w_idx, const uint16_t* idx_raw,
                                       const int64_t* tok_off, const int32_t* pages, int page_rows, int max_pages,
                                       const int32_t* seq_len_in, int32_t* seq_len_out, int32_t* pend_n,
                                       uint16_t* pend_raw, float* pend_logit, uint16_t* pend_idx, int B, int64_t n_tok,
                                       int64_t max_new, void* workspace, size_t workspace_bytes, void* stream) {
  const char* fn = "csa2_compress_stream_paged";
  const csa2_status rc = compress_stream_args(fn, main_kv, idx_k, B, n_tok, max_new);
  if (rc != CSA2_OK || B == 0) return rc;
  int shift = 0;
  if (!pages_ok(pages, page_rows, max_pages, main_kv.rows, idx_k.rows, &shift))
    return fail(CSA2_ERR_INVALID_ARG, std::string(fn) + ": bad page table or page size");
  return compress_stream_impl(fn, main_kv, idx_k, raw, logits, w_idx, idx_raw, tok_off, nullptr, pages, shift,
                              max_pages, seq_len_in, seq_len_out, pend_n, pend_raw, pend_logit, pend_idx, B, n_tok,
                              max_new, workspace, workspace_bytes, stream);
}

// ---------------------------------------------------------------------------
namespace {
struct PrefillWs {
  uint32_t* status;
  int32_t* vis;
  uint32_t* bkeys;
  uint32_t* ckeys;
  int32_t* topblk;  // [T][k]: the best k blocks of every pool
  float* scores;
  size_t bytes;
};
PrefillWs prefill_ws(void* ws, int T, int64_t n_entries, int P, int k) {
  Carve c(ws);
  PrefillWs w;
  w.status = c.take<uint32_t>(kStatusBytes / 4);
  w.vis = c.take<int32_t>(size_t(T));
  const size_t nb = size_t(block_key_stride(n_entries));
  w.bkeys = c.take<uint32_t>(size_t(T) * nb);
  w.ckeys = c.take<uint32_t>(size_t(T) * k * kBlk);
  w.topblk = c.take<int32_t>(size_t(T) * k);
  (void)P;
  w.scores = nullptr;
  w.bytes = c.used;
  return w;
}
}  // namespace

size_t csa2_index_prefill_workspace_bytes(int T, int64_t n_entries, int pool_blocks, int k) {
  if (T < 0 || n_entries < 0) return 0;
  return prefill_ws(nullptr, T, n_entries, pool_blocks, k).bytes;
}

csa2_status csa2_index_prefill(csa2_mxfp4_cache idx_k, const uint8_t* q_codes, const uint8_t* q_scales,
                               const float* w, const int32_t* q_pos, int T, int64_t row0, int64_t n_entries,
                               int ratio, int pool_blocks, int k, int32_t* pool_out, int32_t* topk_out,
                               void* workspace, size_t workspace_bytes, void* stream) {
  const char* fn = "csa2_index_prefill";
  if (T < 0 || n_entries < 0 || row0 < 0) return fail(CSA2_ERR_INVALID_ARG, std::string(fn) + ": negative size");
  if (ratio != 1 && ratio != 2) return fail(CSA2_ERR_INVALID_ARG, std::string(fn) + ": ratio must be 1 or 2");
  if (pool_blocks < 1 || pool_blocks > CSA2_MAX_POOL_BLOCKS || k < 1 || k > CSA2_MAX_TOPK)
    return fail(CSA2_ERR_INVALID_ARG, std::string(fn) + ": pool_blocks and k must be in 1..2048");
  if (pool_blocks < k)
    return fail(CSA2_ERR_UNSUPPORTED, std::string(fn) + ": prefill needs pool_blocks >= k");
  if (T == 0) return CSA2_OK;
  if (!cache_ok(idx_k) || (row0 % 8) != 0 || row0 + n_entries > idx_k.rows || n_entries > INT32_MAX)
    return fail(CSA2_ERR_INVALID_ARG, std::string(fn) + ": bad cache, row0 or n_entries");
  if (!q_codes || !q_scales || !w || !q_pos || !pool_out || !topk_out || !workspace)
    return fail(CSA2_ERR_INVALID_ARG, std::string(fn) + ": null pointer");
  if (!aligned16(q_codes) || (reinterpret_cast<uintptr_t>(workspace) & 255))
    return fail(CSA2_ERR_INVALID_ARG, std::string(fn) + ": q_codes must be 16-byte and workspace 256-byte aligned");
  PrefillWs ws = prefill_ws(workspace, T, n_entries, pool_blocks, k);
  if (workspace_bytes < ws.bytes) return fail(CSA2_ERR_WORKSPACE, std::string(fn) + ": workspace too small");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int64_t nb = block_key_stride(n_entries);
  launch_prefill_vis(q_pos, T, ratio, n_entries, ws.vis, ws.status, st);
  const csa2_status rc0 = launch_prefill_tc(idx_k.codes, idx_k.scales, row0, idx_k.rows, ws.vis, T, n_entries, q_codes,
                                            q_scales, w, ws.bkeys, nb, ws.status, st);
  if (rc0 != CSA2_OK) return rc0;
  // the pool, the best k blocks among it, and the Top-k over their positions
  launch_select(kSelBlockKeys, ws.bkeys, nb, ws.vis, T, 0, nullptr, pool_blocks, pool_out, nullptr, st, ws.status,
                ws.topblk, k);
  SegDesc sd{nullptr, row0, ws.vis, n_entries, idx_k.rows};
  const csa2_status rc = launch_pool_tc(idx_k.codes, idx_k.scales, sd, ws.vis, T, q_codes, q_scales, w, ws.topblk, k,
                                        ws.ckeys, nullptr, ws.status, st);
  if (rc != CSA2_OK) return rc;
  launch_select(kSelPoolCand, ws.ckeys, int64_t(k) * kBlk, ws.vis, T, k, ws.topblk, k, topk_out, nullptr, st);
  return check_launch(fn);
}

// ---------------------------------------------------------------------------
namespace {
struct MultiWs {
  uint32_t* status;
  int32_t* vis;
  int64_t* q_row_off;
  int4* groups;
  int32_t* n_groups;
  uint32_t* bkeys;
  uint32_t* ckeys;
  int32_t* topblk;  // [Q][k]: the best k blocks of every pool
  size_t bytes;
};
MultiWs multi_ws(void* ws, int B, int Q, int64_t max_vis, int k) {
  Carve c(ws);
  MultiWs w;
  w.status = c.take<uint32_t>(kStatusBytes / 4);
  w.vis = c.take<int32_t>(size_t(Q));
  w.q_row_off = c.take<int64_t>(size_t(Q));
  w.groups = c.take<int4>(size_t(multi_group_bound(B, Q)));
  w.n_groups = c.take<int32_t>(1);
  w.bkeys = c.take<uint32_t>(size_t(Q) * size_t(block_key_stride(max_vis)));
  w.ckeys = c.take<uint32_t>(size_t(Q) * k * kBlk);
  w.topblk = c.take<int32_t>(size_t(Q) * k);
  w.bytes = c.used;
  return w;
}
}  // namespace

size_t csa2_index_multi_workspace_bytes(int B, int Q, int64_t max_vis, int pool_blocks, int k) {
  (void)k;
  if (B < 0 || Q < 0 || max_vis < 0 || pool_blocks < 0) return 0;
  return multi_ws(nullptr, B, Q, max_vis, k).bytes;
}

csa2_status csa2_index_multi(csa2_mxfp4_cache idx_k, const uint8_t* q_codes, const uint8_t* q_scales, const float* w,
                             const int64_t* seq_row_off, const int32_t* q_off, const int32_t* q_vis, int B, int Q,
                             int64_t max_vis, int pool_blocks, int k, int32_t* pool_out, int32_t* topk_out,
                             int64_t* q_row_off_out, void* workspace, size_t workspace_bytes, void* stream) {
  const char* fn = "csa2_index_multi";
  if (B < 0 || Q < 0 || max_vis < 0) return fail(CSA2_ERR_INVALID_ARG, std::string(fn) + ": negative size");
  if (pool_blocks < 1 || pool_blocks > CSA2_MAX_POOL_BLOCKS || k < 1 || k > CSA2_MAX_TOPK)
    return fail(CSA2_ERR_INVALID_ARG, std::string(fn) + ": pool_blocks and k must be in 1..2048");
  if (pool_blocks < k)
    return fail(CSA2_ERR_UNSUPPORTED, std::string(fn) + ": the multi-query indexer needs pool_blocks >= k");
  if (Q == 0) return CSA2_OK;
  if (B == 0) return fail(CSA2_ERR_INVALID_ARG, std::string(fn) + ": queries without sequences");
  if (!cache_ok(idx_k) || max_vis > idx_k.rows || max_vis > INT32_MAX)
    return fail(CSA2_ERR_INVALID_ARG, std::string(fn) + ": bad cache or max_vis");
  if (!q_codes || !q_scales || !w || !seq_row_off || !q_off || !q_vis || !pool_out || !topk_out || !workspace)
    return fail(CSA2_ERR_INVALID_ARG, std::string(fn) + ": null pointer");
  if (!aligned16(q_codes) || (reinterpret_cast<uintptr_t>(workspace) & 255) ||
      (q_row_off_out && (reinterpret_cast<uintptr_t>(q_row_off_out) & 7)))
    return fail(CSA2_ERR_INVALID_ARG, std::string(fn) + ": q_codes must be 16-byte and workspace 256-byte aligned");
  MultiWs ws = multi_ws(workspace, B, Q, max_vis, k);
  if (workspace_bytes < ws.bytes) return fail(CSA2_ERR_WORKSPACE, std::string(fn) + ": workspace too small");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int64_t* row_off = q_row_off_out ? q_row_off_out : ws.q_row_off;
  const int G = multi_group_bound(B, Q);
  const int64_t nb = block_key_stride(max_vis);
  launch_multi_prep(seq_row_off, q_off, q_vis, B, Q, G, max_vis, idx_k.rows, ws.groups, row_off, ws.vis,
                    ws.n_groups, ws.status, st);
  const csa2_status rc0 = launch_multi_tc(idx_k.codes, idx_k.scales, idx_k.rows, seq_row_off, ws.groups, G,
                                          ws.n_groups, ws.vis, Q, max_vis, q_codes, q_scales, w, ws.bkeys, nb,
                                          ws.status, st);
  if (rc0 != CSA2_OK) return rc0;
  // the pool, the best k blocks among it, and the Top-k over their positions
  launch_select(kSelBlockKeys, ws.bkeys, nb, ws.vis, Q, 0, nullptr, pool_blocks, pool_out, nullptr, st, ws.status,
                ws.topblk, k);
  SegDesc sd{row_off, 0, ws.vis, max_vis, idx_k.rows};
  const csa2_status rc = launch_pool_tc(idx_k.codes, idx_k.scales, sd, ws.vis, Q, q_codes, q_scales, w, ws.topblk, k,
                                        ws.ckeys, nullptr, ws.status, st);
  if (rc != CSA2_OK) return rc;
  launch_select(kSelPoolCand, ws.ckeys, int64_t(k) * kBlk, ws.vis, Q, k, ws.topblk, k, topk_out, nullptr, st);
  return check_launch(fn);
}

// ---------------------------------------------------------------------------
size_t csa2_score_positions_workspace_bytes(int B) {
  (void)B;
  return kStatusBytes;
}

csa2_status csa2_score_positions(csa2_mxfp4_cache idx_k, const uint8_t* q_codes, const uint8_t* q_scales,
                                 const float* w, const int64_t* seq_row_off, const int32_t* seq_len,
                                 const int32_t* ids, int B, int n, int block, uint32_t* keys_out, void* workspace,
                                 size_t workspace_bytes, void* stream) {
  const char* fn = "csa2_score_positions";
  if (B < 0 || n < 0) return fail(CSA2_ERR_INVALID_ARG, std::string(fn) + ": negative size");
  if (block != 1 && block != kBlk) return fail(CSA2_ERR_INVALID_ARG, std::string(fn) + ": block must be 1 or 8");
  if (B == 0 || n == 0) return CSA2_OK;
  if (!cache_ok(idx_k)) return fail(CSA2_ERR_INVALID_ARG, std::string(fn) + ": bad indexer-K cache");
  if (!q_codes || !q_scales || !w || !seq_row_off || !seq_len || !ids || !keys_out || !workspace)
    return fail(CSA2_ERR_INVALID_ARG, std::string(fn) + ": null pointer");
  if (workspace_bytes < kStatusBytes) return fail(CSA2_ERR_WORKSPACE, std::string(fn) + ": workspace too small");
  SegDesc sd{seq_row_off, 0, seq_len, INT32_MAX, idx_k.rows};
  launch_score_positions(idx_k.codes, idx_k.scales, sd, q_codes, q_scales, w, ids, B, n, block, keys_out,
                         static_cast<uint32_t*>(workspace), static_cast<cudaStream_t>(stream));
  return check_launch(fn);
}

size_t csa2_topk_merge_workspace_bytes(int G, int B, int n) {
  if (G < 0 || B < 0 || n < 0) return 0;
  Carve c(nullptr);
  c.take<uint32_t>(kStatusBytes / 4);
  c.take<uint32_t>(size_t(B) * G * n);
  c.take<int32_t>(size_t(B) * G * n);
  return c.used;
}

csa2_status csa2_topk_merge(const uint32_t* keys, const int32_t* ids, const int64_t* src_off, int G, int B, int n,
                            int k, const int64_t* lo, const int64_t* hi, int32_t* out, int32_t* out_local,
                            void* workspace, size_t workspace_bytes, void* stream) {
  const char* fn = "csa2_topk_merge";
  if (G < 1 || B < 0 || n < 0 || k < 1 || k > CSA2_MAX_TOPK)
    return fail(CSA2_ERR_INVALID_ARG, std::string(fn) + ": bad G, B, n or k");
  if (int64_t(G) * n > (int64_t(1) << 24)) return fail(CSA2_ERR_UNSUPPORTED, std::string(fn) + ": too many candidates");
  if (B == 0) return CSA2_OK;
  if (!keys || !ids || !out || !workspace || (out_local && (!lo || !hi)))
    return fail(CSA2_ERR_INVALID_ARG, std::string(fn) + ": null pointer");
  if (reinterpret_cast<uintptr_t>(workspace) & 255)
    return fail(CSA2_ERR_INVALID_ARG, std::string(fn) + ": workspace must be 256-byte aligned");
  if (workspace_bytes < csa2_topk_merge_workspace_bytes(G, B, n))
    return fail(CSA2_ERR_WORKSPACE, std::string(fn) + ": workspace too small");
  Carve c(workspace);
  uint32_t* status = c.take<uint32_t>(kStatusBytes / 4);
  uint32_t* keys_t = c.take<uint32_t>(size_t(B) * G * n);
  int32_t* ids_t = c.take<int32_t>(size_t(B) * G * n);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  launch_merge_gather(keys, ids, src_off, G, B, n, keys_t, ids_t, status, st);
  launch_select(kSelExplicit, keys_t, int64_t(G) * n, nullptr, B, G * n, ids_t, k, out, nullptr, st);
  if (out_local) launch_localize(out, B, k, lo, hi, out_local, st);
  return check_launch(fn);
}

csa2_status csa2_attn_combine(const float* out_parts, const float* lse_parts, int G, int B, float* out, float* lse,
                              void* stream) {
  const char* fn = "csa2_attn_combine";
  if (G < 1 || B < 0) return fail(CSA2_ERR_INVALID_ARG, std::string(fn) + ": bad G or B");
  if (B == 0) return CSA2_OK;
  if (!out_parts || !lse_parts || !out) return fail(CSA2_ERR_INVALID_ARG, std::string(fn) + ": null pointer");
  if (!aligned16(out_parts) || !aligned16(out))
    return fail(CSA2_ERR_INVALID_ARG, std::string(fn) + ": out_parts and out must be 16-byte aligned");
  launch_attn_combine(out_parts, lse_parts, G, B, out, lse, static_cast<cudaStream_t>(stream));
  return check_launch(fn);
}

// ---------------------------------------------------------------------------
size_t csa2_sparse_attn_prefill_workspace_bytes(int T, int k) {
  Carve c(nullptr);
  c.take<uint32_t>(kStatusBytes / 4);
  c.take<int32_t>(size_t(T));
  c.take<int32_t>(size_t(T));
  c.take<char>(attn_partial_bytes(T, k));
  return c.used;
}

csa2_status csa2_sparse_attn_prefill(const uint16_t* q, const int32_t* q_pos, int T, csa2_mxfp4_cache main_kv,
                                     int64_t row0, int64_t n_entries, int ratio, const int32_t* topk, int k,
                                     const uint8_t* raw_win, int64_t n_raw, float win_scale, float sm_scale,
                                     float* out, float* lse, void* workspace, size_t workspace_bytes,
                                     void* stream) {
  const char* fn = "csa2_sparse_attn_prefill";
  if (T < 0 || k < 1 || k > CSA2_MAX_TOPK || n_entries < 0 || n_raw < 0 || row0 < 0)
    return fail(CSA2_ERR_INVALID_ARG, std::string(fn) + ": bad size");
  if (ratio != 1 && ratio != 2) return fail(CSA2_ERR_INVALID_ARG, std::string(fn) + ": ratio must be 1 or 2");
  if (T == 0) return CSA2_OK;
  if (!cache_ok(main_kv) || row0 + n_entries > main_kv.rows || n_entries > INT32_MAX)
    return fail(CSA2_ERR_INVALID_ARG, std::string(fn) + ": bad cache, row0 or n_entries");
  if (!q || !q_pos || !topk || !raw_win || !out || !workspace)
    return fail(CSA2_ERR_INVALID_ARG, std::string(fn) + ": null pointer");
  if (!aligned16(q) || !aligned16(raw_win) || (reinterpret_cast<uintptr_t>(workspace) & 255))
    return fail(CSA2_ERR_INVALID_ARG, std::string(fn) + ": q/raw_win must be 16-byte, workspace 256-byte aligned");
  if (workspace_bytes < csa2_sparse_attn_prefill_workspace_bytes(T, k))
    return fail(CSA2_ERR_WORKSPACE, std::string(fn) + ": workspace too small");
  Carve c(workspace);
  AttnArgs a{};
  a.status = c.take<uint32_t>(kStatusBytes / 4);
  int32_t* vis = c.take<int32_t>(size_t(T));
  a.counters = c.take<int32_t>(size_t(T));
  a.partial = reinterpret_cast<float*>(c.take<char>(attn_partial_bytes(T, k)));
  a.q = q;
  a.mcodes = main_kv.codes;
  a.mscales = main_kv.scales;
  a.sd = SegDesc{nullptr, row0, vis, n_entries, main_kv.rows};
  a.seg_eff = vis;
  a.topk = topk;
  a.k = k;
  a.q_pos = q_pos;
  a.raw_win = raw_win;
  a.n_raw = n_raw;
  a.raw_scale = win_scale;
  a.sm_scale = sm_scale;
  a.out = out;
  a.lse = lse;
  a.S = T;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  launch_prefill_vis(q_pos, T, ratio, n_entries, vis, a.status, st);
  launch_attention(a, st);
  return check_launch(fn);
}

}  // extern "C"
