// Peak probes for the roofline denominators that a plain copy and a cuBLAS
// GEMM do not give (bench.py --peaks): the read-only HBM stream with 128-bit
// loads and with bulk asynchronous copies, the block-scaled FP4 tensor-core
// rate (tcgen05.mma kind::mxf4, M = 128, N = 16 and N = 128, K = 64 per
// instruction) and the FP64 FMA rate.  Each probe only launches; bench.py
// times it with CUDA events.  Every wait is bounded and reports through
// `err` instead of spinning forever.
#include <cuda_runtime.h>
#include <stdint.h>

#include "long_context_decode_csa2_b200/csrc/sm100.cuh"

namespace {

using namespace csa2;

// ---------------------------------------------------------------- read, ld.global.nc
__global__ void __launch_bounds__(512) k_read_ldg(const uint4* __restrict__ p, long long n, unsigned* sink) {
  uint32_t x = 0;
  const long long stride = (long long)gridDim.x * blockDim.x;
  long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  for (; i + 3 * stride < n; i += 4 * stride) {
    const uint4 a = __ldg(p + i), b = __ldg(p + i + stride), c = __ldg(p + i + 2 * stride), d = __ldg(p + i + 3 * stride);
    x ^= a.x ^ a.y ^ a.z ^ a.w ^ b.x ^ b.y ^ b.z ^ b.w ^ c.x ^ c.y ^ c.z ^ c.w ^ d.x ^ d.y ^ d.z ^ d.w;
  }
  for (; i < n; i += stride) {
    const uint4 a = __ldg(p + i);
    x ^= a.x ^ a.y ^ a.z ^ a.w;
  }
  if (x == 0x9E3779B9u) sink[blockIdx.x] = x;  // keeps the loads; practically never taken
}

// ---------------------------------------------------------------- read, bulk copies into shared memory
constexpr int kBulkStages = 6;
constexpr uint32_t kBulkBytes = 32768;

__global__ void __launch_bounds__(32, 1) k_read_bulk(const uint8_t* __restrict__ p, long long chunks, int* err) {
  extern __shared__ __align__(128) uint8_t buf[];
  __shared__ __align__(8) uint64_t full[kBulkStages];
  const long long c0 = chunks * blockIdx.x / gridDim.x, c1 = chunks * (blockIdx.x + 1) / gridDim.x;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kBulkStages; ++s) sm100::mbar_init(&full[s], 1);
    sm100::fence_mbar_init();
    long long issued = c0, done = c0;
    while (done < c1) {
      // chunk c uses stage (c - c0) % kBulkStages, phase (c - c0) / kBulkStages
      while (issued < c1 && issued - done < kBulkStages) {
        const int s = int((issued - c0) % kBulkStages);
        sm100::mbar_arrive_expect_tx(&full[s], kBulkBytes);
        sm100::bulk_load(buf + size_t(s) * kBulkBytes, p + issued * kBulkBytes, kBulkBytes, &full[s]);
        ++issued;
      }
      const int s = int((done - c0) % kBulkStages);
      if (!sm100::mbar_wait(&full[s], uint32_t((done - c0) / kBulkStages) & 1u, 1000000000ull)) {
        atomicExch(err, 1);
        // wait (bounded) for the copies still in flight, then stop
        for (long long d = done + 1; d < issued; ++d)
          sm100::mbar_wait(&full[(d - c0) % kBulkStages], uint32_t((d - c0) / kBulkStages) & 1u, 100000000ull);
        break;
      }
      ++done;
    }
  }
}

// ---------------------------------------------------------------- tcgen05 kind::mxf4, unit scales
constexpr uint32_t kMmaSf = 448;  // scale-factor columns (2^0 everywhere)

template <int N>
__global__ void __launch_bounds__(128, 1) k_mma_mxf4(int iters, int* err) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* a = sm;               // 128 rows x 64 B (one K = 128 FP4 block pair), zeros
  uint8_t* b = sm + 128 * 64;    // N rows x 64 B
  __shared__ __align__(8) uint64_t done;
  __shared__ uint32_t tmem_base;
  const int warp = threadIdx.x >> 5;
  for (int i = threadIdx.x; i < (128 + N) * 64 / 16; i += blockDim.x)
    reinterpret_cast<uint4*>(sm)[i] = make_uint4(0, 0, 0, 0);
  sm100::fence_proxy_async_smem();
  if (threadIdx.x == 0) {
    sm100::mbar_init(&done, 1);
    sm100::fence_mbar_init();
  }
  if (warp == 0) {
    sm100::tmem_alloc(&tmem_base, 512);
    sm100::tmem_relinquish();
  }
  sm100::tc_fence_before();
  __syncthreads();
  sm100::tc_fence_after();
  const uint32_t tmem = tmem_base;
  {
    const uint32_t lane_base = uint32_t(32 * warp) << 16;
#pragma unroll
    for (int c = 0; c < 64; c += 8) sm100::tmem_st8_same(tmem + lane_base + kMmaSf + c, 0x7F7F7F7Fu);
    sm100::tmem_st_wait();
  }
  sm100::tc_fence_before();
  __syncthreads();
  sm100::tc_fence_after();
  if (threadIdx.x == 0) {
    constexpr uint32_t idesc = sm100::idesc_mxf4(128, N);
    const uint32_t abase = sm100::smem_u32(a), bbase = sm100::smem_u32(b);
    for (int it = 0; it < iters; ++it) {
      const uint32_t kk = uint32_t(it & 1);
      const uint32_t d = tmem + uint32_t((it >> 1) & 1) * N;  // two accumulators
      sm100::mma_mxf4(d, sm100::smem_desc_k64b(abase + kk * 32), sm100::smem_desc_k64b(bbase + kk * 32), idesc,
                      it > 1 ? 1u : kk, tmem + kMmaSf, tmem + kMmaSf + 32);
    }
    sm100::mma_commit(&done);
    if (!sm100::mbar_wait(&done, 0, 2000000000ull)) atomicExch(err, 1);
  }
  sm100::tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    sm100::tc_fence_after();
    sm100::tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------- FP64 FMA
__global__ void __launch_bounds__(256) k_fma64(int iters, double* sink) {
  double x[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) x[j] = 1.0 + 1e-9 * (threadIdx.x + j);
  const double m = 0.999999999, c = 1e-12;
  for (int it = 0; it < iters; ++it) {
#pragma unroll
    for (int j = 0; j < 8; ++j) x[j] = __fma_rn(x[j], m, c);
  }
  double s = 0;
#pragma unroll
  for (int j = 0; j < 8; ++j) s += x[j];
  if (s == 12345.0) sink[blockIdx.x] = s;  // keeps the chains
}

int sms() {
  int dev = 0, n = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n;
}

}  // namespace

extern "C" {

int peaks_num_sms(void) { return sms(); }

// Reads n16 16-byte words once; grid = 8 CTAs of 512 threads per SM.
int peaks_read_ldg(const void* buf, long long n16, unsigned* sink, void* stream) {
  k_read_ldg<<<sms() * 8, 512, 0, static_cast<cudaStream_t>(stream)>>>(static_cast<const uint4*>(buf), n16, sink);
  return int(cudaGetLastError());
}

// Streams `bytes` (a multiple of 32 KiB) into shared memory with bulk copies,
// one CTA of one warp per SM, six 32 KiB stages in flight each.
int peaks_read_bulk(const void* buf, long long bytes, int* err, void* stream) {
  const size_t smem = size_t(kBulkStages) * kBulkBytes;
  cudaFuncSetAttribute(k_read_bulk, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  k_read_bulk<<<sms(), 32, smem, static_cast<cudaStream_t>(stream)>>>(static_cast<const uint8_t*>(buf),
                                                                      bytes / kBulkBytes, err);
  return int(cudaGetLastError());
}

// `iters` back-to-back tcgen05.mma kind::mxf4 (M = 128, N = 16 or 128,
// K = 64) per SM, one CTA per SM.
int peaks_mma_mxf4(int n, int iters, int* err, void* stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (n == 16) {
    cudaFuncSetAttribute(k_mma_mxf4<16>, cudaFuncAttributeMaxDynamicSharedMemorySize, 120 * 1024);
    k_mma_mxf4<16><<<sms(), 128, 120 * 1024, st>>>(iters, err);
  } else if (n == 128) {
    cudaFuncSetAttribute(k_mma_mxf4<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, 120 * 1024);
    k_mma_mxf4<128><<<sms(), 128, 120 * 1024, st>>>(iters, err);
  } else {
    return -1;
  }
  return int(cudaGetLastError());
}

// 8 independent FMA chains of `iters` steps per thread, 8 CTAs of 256 per SM.
int peaks_fma64(int iters, double* sink, void* stream) {
  k_fma64<<<sms() * 8, 256, 0, static_cast<cudaStream_t>(stream)>>>(iters, sink);
  return int(cudaGetLastError());
}

}  // extern "C"
