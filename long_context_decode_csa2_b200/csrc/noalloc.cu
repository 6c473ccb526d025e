// csa2_sparse_attn_decode_noalloc: the sparse-attention decode call with no
// workspace argument and no device allocation of its own.
//
// Who needs it: callers that are not allowed to allocate device memory when
// they run.  Examples are plugins executed inside another inference runtime
// (the host runtime owns every allocation and forbids cudaMalloc inside its
// enqueue callback), serving loops that must keep a fixed, pre-planned memory
// footprint, and code that cannot afford the implicit device synchronisation
// that cudaMalloc / cudaFree can cause.  Such a caller passes only its inputs
// and outputs; the scratch this call needs lives in a fixed array of the
// library's own device memory, declared below.
//
// When that memory is committed: the array belongs to this file's device
// module.  Under CUDA's lazy module loading (the default) a module is loaded,
// and its device memory committed, the first time the process touches it on a
// device, here the address lookup of the array.  The attention kernel's own
// module loads at its first launch in the same way.  So the first call on a
// device may allocate (once); a call with B = 0 does only that set-up and
// launches nothing, so a caller can make it before entering the region where
// it may not allocate.
#include <mutex>
#include <string>

#include "internal.cuh"

namespace csa2 {
namespace {

// Limits of this variant (the regular call has none besides k <= 2048).
constexpr int kNoAllocMaxSeqs = 64;
constexpr int kNoAllocMaxTopk = 512;
constexpr size_t kNoAllocStatusBytes = 256;                       // device status word
constexpr size_t kNoAllocCounterBytes = 256;                      // 64 arrival counters (self-resetting)
constexpr size_t kNoAllocSlots = 4;                               // partials per sequence: one per CTA,
                                                                  // up to 4 CTAs
constexpr size_t kNoAllocPartialBytes =                           // split-KV partials
    size_t(kNoAllocMaxSeqs) * kNoAllocSlots * (kHq * kD + 2 * kHq) * sizeof(float);
constexpr size_t kNoAllocScratchBytes =
    kNoAllocStatusBytes + kNoAllocCounterBytes + kNoAllocPartialBytes;
static_assert(kNoAllocScratchBytes == 8421888, "the documented scratch size");

// The scratch: 8,421,888 bytes of device memory that every GPU on which this
// library's device code is loaded keeps until the process exits.  All calls
// on a device share it and it keeps whatever the last call left in it.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Host code cannot use g_noalloc_scratch as a pointer (on the host the name
// is only a stand-in for the device symbol), so its device address is looked
// up once per device, with that device current, and cached here.  The cache
// assumes the device's context lives as long as the process: after a
// cudaDeviceReset the module may reload elsewhere, so the library must not be
// used across a reset.
constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_addr[kMaxDevices] = {};

csa2_status scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(CSA2_ERR_CUDA, std::string("cudaGetDevice: ") + cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices) return fail(CSA2_ERR_UNSUPPORTED, "device ordinal beyond 63");
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr)
      return fail(CSA2_ERR_CUDA, std::string("cudaGetSymbolAddress of the static scratch: ") + cudaGetErrorString(e));
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return CSA2_OK;
}

}  // namespace
}  // namespace csa2

using namespace csa2;

extern "C" csa2_status csa2_sparse_attn_decode_noalloc(const uint16_t* q, csa2_mxfp4_cache main_kv,
                                                       const int64_t* seq_row_off, const int32_t* seq_len,
                                                       const int32_t* topk, int k, const uint8_t* win,
                                                       const float* win_scale, const int32_t* win_len, float sm_scale,
                                                       float* out, float* lse, uint32_t* flags_out, int B,
                                                       void* stream) {
  const char* fn = "csa2_sparse_attn_decode_noalloc";
  if (B < 0) return fail(CSA2_ERR_INVALID_ARG, std::string(fn) + ": negative B");
  if (B == 0) {
    // set-up only: load this file's module (the scratch) and the attention
    // kernel's module on the current device, launch nothing
    void* base = nullptr;
    const csa2_status rc = scratch_address(&base);
    if (rc != CSA2_OK) return rc;
    prepare_attention();
    return check_launch(fn);
  }
  if (k < 1) return fail(CSA2_ERR_INVALID_ARG, std::string(fn) + ": bad k");
  if (B > kNoAllocMaxSeqs || k > kNoAllocMaxTopk)
    return fail(CSA2_ERR_UNSUPPORTED, std::string(fn) + ": at most 64 sequences and k <= 512 (fixed scratch of " +
                                          std::to_string(kNoAllocScratchBytes) + " bytes); use csa2_sparse_attn_decode");
  if (!(main_kv.codes && main_kv.scales && aligned16(main_kv.codes) && aligned16(main_kv.scales) && main_kv.rows >= 0 &&
        main_kv.rows % 8 == 0))
    return fail(CSA2_ERR_INVALID_ARG, std::string(fn) + ": bad main-KV cache");
  if (!q || !seq_row_off || !seq_len || !topk || !win || !win_scale || !win_len || !out)
    return fail(CSA2_ERR_INVALID_ARG, std::string(fn) + ": null pointer");
  if (!aligned16(win) || !aligned16(q))
    return fail(CSA2_ERR_INVALID_ARG, std::string(fn) + ": q and win must be 16-byte aligned");
  if (attn_partial_bytes(B, k) > kNoAllocPartialBytes)
    return fail(CSA2_ERR_UNSUPPORTED, std::string(fn) + ": problem does not fit the fixed scratch");
  void* base = nullptr;
  const csa2_status rc = scratch_address(&base);
  if (rc != CSA2_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  char* p = static_cast<char*>(base);
  AttnArgs a{};
  a.status = reinterpret_cast<uint32_t*>(p);
  a.counters = reinterpret_cast<int32_t*>(p + kNoAllocStatusBytes);
  a.partial = reinterpret_cast<float*>(p + kNoAllocStatusBytes + kNoAllocCounterBytes);
  // The status word must start at zero for this call.  The arrival counters
  // are zero when the module loads and every call leaves them at zero; the
  // partials are fully written before they are read.
  cudaError_t e = cudaMemsetAsync(a.status, 0, sizeof(uint32_t), st);
  if (e != cudaSuccess) return fail(CSA2_ERR_CUDA, std::string(fn) + ": " + cudaGetErrorString(e));
  a.q = q;
  a.mcodes = main_kv.codes;
  a.mscales = main_kv.scales;
  a.sd = SegDesc{seq_row_off, 0, seq_len, INT32_MAX, main_kv.rows};
  a.seg_eff = nullptr;  // lengths are checked per segment inside the kernel
  a.topk = topk;
  a.k = k;
  a.win = win;
  a.win_scale = win_scale;
  a.win_len = win_len;
  a.sm_scale = sm_scale;
  a.out = out;
  a.lse = lse;
  a.S = B;
  launch_attention(a, st);
  if (flags_out) {
    e = cudaMemcpyAsync(flags_out, a.status, sizeof(uint32_t), cudaMemcpyDeviceToDevice, st);
    if (e != cudaSuccess) return fail(CSA2_ERR_CUDA, std::string(fn) + ": " + cudaGetErrorString(e));
  }
  return check_launch(fn);
}
