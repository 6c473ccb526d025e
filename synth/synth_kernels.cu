// GPU twin of synth/__init__.py: the same SplitMix64 counter streams and the
// same integer tables, so large synthetic caches can be generated on the
// device and still equal the NumPy generator byte for byte.  Holds none of
// the CSA2 method's arithmetic (no quantisation, scoring or selection).
#include <cuda_runtime.h>
#include <stdint.h>

namespace {

__device__ __forceinline__ uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

__device__ __forceinline__ uint64_t draw(uint64_t key, uint64_t i) {
  return mix64(key + (i + 1ull) * 0x9E3779B97F4A7C15ull);
}

__device__ __forceinline__ uint32_t e2m1_mag_index(uint32_t v /*0..127*/) {
  const uint32_t cum[8] = {13, 38, 60, 79, 101, 118, 127, 128};
  uint32_t n = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) n += (cum[i] <= v);
  return n;
}

__device__ __forceinline__ int rownorm_shift(uint32_t u /*0..255*/) {
  const uint32_t cum[5] = {5, 63, 193, 251, 256};
  int n = 0;
#pragma unroll
  for (int i = 0; i < 5; ++i) n += (cum[i] <= u);
  return n - 2;
}

// codes: one thread per draw (8 elements -> 4 code bytes)
__global__ void k_mxfp4_codes(uint8_t* codes, uint64_t key, int64_t r0, int64_t nrows, int n) {
  const int64_t per_row = n / 8;
  const int64_t g = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (g >= nrows * per_row) return;
  const int64_t r = g / per_row, m = g % per_row;
  const uint64_t h = draw(key, uint64_t((r0 + r) * per_row + m));
  uint32_t out = 0;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const uint32_t b = uint32_t(h >> (8 * j)) & 255u;
    const uint32_t code = e2m1_mag_index(b & 127u) | ((b >> 7) << 3);
    out |= code << (4 * j);
  }
  reinterpret_cast<uint32_t*>(codes + r * (n / 2))[m] = out;
}

// scales: one thread per row
__global__ void k_mxfp4_scales(uint8_t* scales, uint64_t key, uint64_t norm_key, int has_norm, int64_t r0,
                               int64_t nrows, int n) {
  const int64_t r = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (r >= nrows) return;
  const int nb = n / 32;
  const int nh = (nb + 7) / 8;
  const int shift = has_norm ? rownorm_shift(uint32_t(draw(norm_key, uint64_t(r0 + r))) & 255u) : 0;
  for (int i = 0; i < nb; ++i) {
    const uint64_t h = draw(key, uint64_t((r0 + r) * nh + i / 8));
    const uint32_t u = uint32_t(h >> (8 * (i % 8))) & 255u;
    const int byte = (u < 64u ? 125 : (u < 243u ? 126 : 127)) + shift;
    scales[r * nb + i] = uint8_t(byte);
  }
}

// E4M3 rows: one thread per draw (4 values)
__global__ void k_e4m3_rows(uint8_t* out, uint64_t key, int64_t r0, int64_t nrows, int n) {
  const int64_t per_row = n / 4;
  const int64_t g = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (g >= nrows * per_row) return;
  const int64_t r = g / per_row, m = g % per_row;
  const uint64_t h = draw(key, uint64_t((r0 + r) * per_row + m));
  const uint32_t cum[7] = {16, 40, 64, 123, 205, 253, 256};
  uint32_t word = 0;
#pragma unroll
  for (int v = 0; v < 4; ++v) {
    const uint32_t lo = uint32_t(h >> (16 * v)) & 255u, hi = uint32_t(h >> (16 * v + 8)) & 255u;
    uint32_t cat = 0;
#pragma unroll
    for (int i = 0; i < 7; ++i) cat += (cum[i] <= hi);
    const uint32_t field = 9 + cat;
    uint32_t mant = lo & 7u;
    if (field == 15 && mant == 7) mant = 6;
    word |= (((lo >> 7) << 7) | (field << 3) | mant) << (8 * v);
  }
  reinterpret_cast<uint32_t*>(out + r * n)[m] = word;
}

// ~N(0,1) bf16: (sum of twelve uniform bytes - 1530) / 256, rounded to
// nearest-even bf16 (two draws per value, bytes 0..7 and 0..3).
__global__ void k_normal_bf16(uint16_t* out, uint64_t key, int64_t start, int64_t count) {
  const int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= count) return;
  const uint64_t h0 = draw(key, uint64_t(2 * (start + i))), h1 = draw(key, uint64_t(2 * (start + i) + 1));
  int sum = 0;
#pragma unroll
  for (int j = 0; j < 8; ++j) sum += int((h0 >> (8 * j)) & 255u);
#pragma unroll
  for (int j = 0; j < 4; ++j) sum += int((h1 >> (8 * j)) & 255u);
  const float v = float(sum - 1530) * (1.0f / 256.0f);
  const uint32_t u = __float_as_uint(v);
  out[i] = uint16_t((u + 0x7FFFu + ((u >> 16) & 1u)) >> 16);
}

}  // namespace

extern "C" {

int synth_normal_bf16(uint16_t* out, uint64_t key, int64_t start, int64_t count, void* stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (count > 0) k_normal_bf16<<<unsigned((count + 255) / 256), 256, 0, st>>>(out, key, start, count);
  return int(cudaGetLastError());
}


int synth_mxfp4_rows(uint8_t* codes, uint8_t* scales, uint64_t key_codes, uint64_t key_scales, uint64_t key_norm,
                     int has_norm, int64_t r0, int64_t nrows, int n, void* stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int64_t nd = nrows * (n / 8);
  if (nd > 0) k_mxfp4_codes<<<unsigned((nd + 255) / 256), 256, 0, st>>>(codes, key_codes, r0, nrows, n);
  if (nrows > 0)
    k_mxfp4_scales<<<unsigned((nrows + 255) / 256), 256, 0, st>>>(scales, key_scales, key_norm, has_norm, r0, nrows,
                                                                  n);
  return int(cudaGetLastError());
}

int synth_e4m3_rows(uint8_t* out, uint64_t key, int64_t r0, int64_t nrows, int n, void* stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int64_t nd = nrows * (n / 4);
  if (nd > 0) k_e4m3_rows<<<unsigned((nd + 255) / 256), 256, 0, st>>>(out, key, r0, nrows, n);
  return int(cudaGetLastError());
}

}  // extern "C"
