// Casts for the unscaled FP8 attention path on B200 (sm_100a): 16-bit Q / K
// to e4m3, and 16-bit V to e4m3 transposed to [B, Hkv, d, pitch] (key index
// innermost), the layout whose tiles are the K-major B operand of O += P V.
//
// What is computed: the flashdreams.accelerated developer guide,
// "OptimizedImplConfig" (quantized_sdpa): Q, K and V are cast directly,
// without scales, to float8_e4m3fn. Each value is rounded to the nearest e4m3
// value (ties to even) and saturated at +-448, the largest finite e4m3 value.
// Both passes are elementwise and bound by HBM bandwidth.

#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "attn.h"

namespace hasb_f8 {

template <bool BF16>
__device__ __forceinline__ float to_f32(uint16_t h) {
  if (BF16) return __uint_as_float(static_cast<uint32_t>(h) << 16);
  return __half2float(__ushort_as_half(h));
}

__device__ __forceinline__ uint32_t e4m3x2(float lo, float hi) {
  unsigned short r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

// n elements, 8 per thread (16 bytes in, 8 bytes out); n % 8 == 0.
template <bool BF16>
__global__ void __launch_bounds__(256) cast_kernel(const uint4* __restrict__ x, uint2* __restrict__ y,
                                                   long long n8) {
  for (long long i = blockIdx.x * 256LL + threadIdx.x; i < n8; i += 256LL * gridDim.x) {
    const uint4 v = x[i];
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    float f[8];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      f[2 * e] = to_f32<BF16>(static_cast<uint16_t>(w[e] & 0xFFFFu));
      f[2 * e + 1] = to_f32<BF16>(static_cast<uint16_t>(w[e] >> 16));
    }
    y[i] = make_uint2(e4m3x2(f[0], f[1]) | (e4m3x2(f[2], f[3]) << 16),
                      e4m3x2(f[4], f[5]) | (e4m3x2(f[6], f[7]) << 16));
  }
}

// One 64-key x 64-feature tile of one (batch, head): read coalesced along d,
// written coalesced along keys. vt[b, h, c, j] = e4m3(v[b, j, h, c]).
template <bool BF16>
__global__ void __launch_bounds__(256) cast_vt_kernel(const uint16_t* __restrict__ v,
                                                      uint8_t* __restrict__ vt, int Lk, int H, int d,
                                                      int pitch) {
  __shared__ float tile[64][65];
  const int j0 = blockIdx.x * 64, c0 = blockIdx.y * 64;
  const int bh = blockIdx.z, b = bh / H, h = bh % H;
  const int tx = threadIdx.x % 64, ty = threadIdx.x / 64;  // 64 x 4
  for (int r = ty; r < 64; r += 4) {
    const int j = j0 + r;
    tile[r][tx] = j < Lk ? to_f32<BF16>(v[((static_cast<size_t>(b) * Lk + j) * H + h) * d + c0 + tx]) : 0.f;
  }
  __syncthreads();
  // each thread writes 4 consecutive keys of one feature row
  const int c = threadIdx.x / 16, jj = (threadIdx.x % 16) * 4;
  for (int cc = c; cc < 64; cc += 16) {
    const int j = j0 + jj;
    if (j >= Lk) continue;
    uint8_t* dst = vt + ((static_cast<size_t>(b) * H + h) * d + c0 + cc) * pitch + j;
    const uint32_t w = e4m3x2(tile[jj][cc], tile[jj + 1][cc]) | (e4m3x2(tile[jj + 2][cc], tile[jj + 3][cc]) << 16);
    if (j + 4 <= Lk) {
      *reinterpret_cast<uint32_t*>(dst) = w;  // pitch and j are multiples of 4
    } else {
      for (int e = 0; e < Lk - j; ++e) dst[e] = static_cast<uint8_t>(w >> (8 * e));
    }
  }
}

}  // namespace hasb_f8

using namespace hasb_f8;

namespace {
bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }
bool overlap(const void* a, size_t na, const void* b, size_t nb) {
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return x < y + nb && y < x + na;
}
}  // namespace

extern "C" int attn_fp8_cast(const void* x, void* y, long long n, int dtype, void* stream) {
  if (x == nullptr || y == nullptr || n < 0 || n % 8 != 0) return ATTN_ERR_INVALID_ARG;
  if (dtype != ATTN_DTYPE_BF16 && dtype != ATTN_DTYPE_FP16) return ATTN_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(y, 8)) return ATTN_ERR_INVALID_ARG;
  if (overlap(x, static_cast<size_t>(n) * 2, y, static_cast<size_t>(n))) return ATTN_ERR_INVALID_ARG;
  if (n == 0) return ATTN_OK;
  const long long n8 = n / 8;
  const unsigned grid = static_cast<unsigned>(n8 / 256 + 1 < 148 * 16 ? n8 / 256 + 1 : 148 * 16);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  (void)cudaGetLastError();
  if (dtype == ATTN_DTYPE_BF16)
    cast_kernel<true><<<grid, 256, 0, s>>>(static_cast<const uint4*>(x), static_cast<uint2*>(y), n8);
  else
    cast_kernel<false><<<grid, 256, 0, s>>>(static_cast<const uint4*>(x), static_cast<uint2*>(y), n8);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

extern "C" int attn_fp8_cast_vt(const void* v, void* vt, int B, int Lk, int Hkv, int d, int pitch,
                                int dtype, void* stream) {
  if (v == nullptr || vt == nullptr) return ATTN_ERR_INVALID_ARG;
  if (dtype != ATTN_DTYPE_BF16 && dtype != ATTN_DTYPE_FP16) return ATTN_ERR_INVALID_ARG;
  if (B < 1 || Lk < 1 || Hkv < 1 || d < 64 || d % 64 != 0 || pitch < Lk || pitch % 16 != 0)
    return ATTN_ERR_INVALID_ARG;
  if (!aligned(v, 16) || !aligned(vt, 16)) return ATTN_ERR_INVALID_ARG;
  const size_t nv = 2ull * B * Lk * Hkv * d, nvt = 1ull * B * Hkv * d * pitch;
  if (overlap(v, nv, vt, nvt)) return ATTN_ERR_INVALID_ARG;
  if (static_cast<long long>(B) * Hkv > 65535) return ATTN_ERR_INVALID_ARG;
  dim3 grid((Lk + 63) / 64, d / 64, B * Hkv);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  (void)cudaGetLastError();
  if (dtype == ATTN_DTYPE_BF16)
    cast_vt_kernel<true><<<grid, 256, 0, s>>>(static_cast<const uint16_t*>(v), static_cast<uint8_t*>(vt),
                                              Lk, Hkv, d, pitch);
  else
    cast_vt_kernel<false><<<grid, 256, 0, s>>>(static_cast<const uint16_t*>(v), static_cast<uint8_t*>(vt),
                                               Lk, Hkv, d, pitch);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}
