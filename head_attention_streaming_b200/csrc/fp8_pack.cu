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

// Debug build (-DATTN_DEBUG): the site number of the first index check that
// failed in this file's kernels (0: none); a failed check skips the access.
// In the release build a check is `true` and compiles away.
__device__ unsigned int g_debug_site = 0;
__device__ __forceinline__ bool debug_check(bool ok, unsigned int site) {
  if (!ok) atomicCAS(&g_debug_site, 0u, site);
  return ok;
}
#ifdef ATTN_DEBUG
#define ATTN_CHECK(cond, site) (debug_check((cond), (site)))
#else
#define ATTN_CHECK(cond, site) true
#endif

// Reads (and with `clear` resets) this file's debug site word.
unsigned int debug_site_read(bool clear) {
  unsigned int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_debug_site, sizeof(v)) != cudaSuccess) return 0;
  if (clear) {
    const unsigned int zero = 0;
    (void)cudaMemcpyToSymbol(g_debug_site, &zero, sizeof(zero));
  }
  return v;
}


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
    tile[r][tx] = (j < Lk && c0 + tx < d)
                      ? to_f32<BF16>(v[((static_cast<size_t>(b) * Lk + j) * H + h) * d + c0 + tx])
                      : 0.f;
  }
  __syncthreads();
  // each thread writes 4 consecutive keys of one feature row
  const int c = threadIdx.x / 16, jj = (threadIdx.x % 16) * 4;
  for (int cc = c; cc < 64; cc += 16) {
    const int j = j0 + jj;
    if (j >= Lk || c0 + cc >= d) continue;
    uint8_t* dst = vt + ((static_cast<size_t>(b) * H + h) * d + c0 + cc) * pitch + j;
    const uint32_t w = e4m3x2(tile[jj][cc], tile[jj + 1][cc]) | (e4m3x2(tile[jj + 2][cc], tile[jj + 3][cc]) << 16);
    // site 31: the four keys stay inside the row's pitch, 4-byte aligned
    if (!ATTN_CHECK(Lk <= pitch && (pitch & 3) == 0 && (j & 3) == 0, 31)) continue;
    if (j + 4 <= Lk) {
      *reinterpret_cast<uint32_t*>(dst) = w;  // pitch and j are multiples of 4
    } else {
      for (int e = 0; e < Lk - j; ++e) dst[e] = static_cast<uint8_t>(w >> (8 * e));
    }
  }
}

// ---- per-token / per-channel scaled quantization (developer guide,
// "Quantization Toolkit": s = max(max |x| / 448, eps) in float32 over the
// slice, code = e4m3(x / s) with x / s clipped to +-448; eps = 2^-126, the
// smallest normal float32). Both divisions are IEEE round-to-nearest, so the
// codes are those of any float32 implementation of the same definition.

constexpr float kE4m3Max = 448.f;
constexpr float kScaleFloor = 1.17549435e-38f;  // 2^-126

__device__ __forceinline__ float slice_scale(float amax) {
  return fmaxf(__fdiv_rn(amax, kE4m3Max), kScaleFloor);
}

// One row of d values per G = d / 8 adjacent lanes (8 values a lane).
template <bool BF16>
__global__ void __launch_bounds__(256) quantize_tokens_kernel(const uint4* __restrict__ x,
                                                              uint2* __restrict__ y, float* __restrict__ s,
                                                              long long n_rows, int L, int H, int G,
                                                              int s_pitch) {
  const int rows_per_block = 256 / G;
  const int sub = threadIdx.x % G;
  for (long long row = blockIdx.x * static_cast<long long>(rows_per_block) + threadIdx.x / G;
       row - threadIdx.x / G < n_rows; row += static_cast<long long>(gridDim.x) * rows_per_block) {
    const bool live = row < n_rows;
    float f[8];
    float amax = 0.f;
    if (live) {
      const uint4 v = x[row * G + sub];
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        f[2 * e] = to_f32<BF16>(static_cast<uint16_t>(w[e] & 0xFFFFu));
        f[2 * e + 1] = to_f32<BF16>(static_cast<uint16_t>(w[e] >> 16));
      }
#pragma unroll
      for (int e = 0; e < 8; ++e) amax = fmaxf(amax, fabsf(f[e]));
    }
    for (int off = G / 2; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
    if (!live) continue;
    const float sc = slice_scale(amax);
    float g[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) g[e] = __fdiv_rn(f[e], sc);
    y[row * G + sub] = make_uint2(e4m3x2(g[0], g[1]) | (e4m3x2(g[2], g[3]) << 16),
                                  e4m3x2(g[4], g[5]) | (e4m3x2(g[6], g[7]) << 16));
    if (sub == 0) {
      const long long h = row % H, l = (row / H) % L, b = row / (static_cast<long long>(H) * L);
      // site 32: the token's scale lies inside its [pitch] row
      if (ATTN_CHECK(l < s_pitch, 32)) s[(b * H + h) * s_pitch + l] = sc;
    }
  }
}

// Column maxima of V [B, Lk, H, d] over keys: block (key chunk, b * H + h),
// 8 channels a thread; folded into amax_bits (float bits of |v|, which order
// like the floats for non-negative values) with atomicMax.
template <bool BF16>
__global__ void __launch_bounds__(256) column_amax_kernel(const uint4* __restrict__ v,
                                                          unsigned* __restrict__ amax_bits, int Lk, int H,
                                                          int G, int keys_per_block) {
  __shared__ float part[256][9];
  const int bh = blockIdx.y, b = bh / H, h = bh % H;
  const int sub = threadIdx.x % G, lanes = 256 / G;
  float m[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  const int j_end = min(Lk, (blockIdx.x + 1) * keys_per_block);
  for (int j = blockIdx.x * keys_per_block + threadIdx.x / G; j < j_end; j += lanes) {
    const uint4 q = v[((static_cast<size_t>(b) * Lk + j) * H + h) * G + sub];
    const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      m[2 * e] = fmaxf(m[2 * e], fabsf(to_f32<BF16>(static_cast<uint16_t>(w[e] & 0xFFFFu))));
      m[2 * e + 1] = fmaxf(m[2 * e + 1], fabsf(to_f32<BF16>(static_cast<uint16_t>(w[e] >> 16))));
    }
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) part[threadIdx.x][e] = m[e];
  __syncthreads();
  const int d = 8 * G;
  if (threadIdx.x < d) {  // channel c = threadIdx.x: thread sub = c / 8 of every key lane
    const int c = threadIdx.x, sc = c / 8, e = c % 8;
    float a = 0.f;
    for (int r = 0; r < lanes; ++r) a = fmaxf(a, part[r * G + sc][e]);
    atomicMax(amax_bits + static_cast<size_t>(bh) * d + c, __float_as_uint(a));
  }
}

// cast_vt_kernel with each channel divided by its scale (from the column max).
template <bool BF16>
__global__ void __launch_bounds__(256) quantize_vt_kernel(const uint16_t* __restrict__ v,
                                                          uint8_t* __restrict__ vt,
                                                          const unsigned* __restrict__ amax_bits, int Lk,
                                                          int H, int d, int pitch) {
  __shared__ float tile[64][65];
  const int j0 = blockIdx.x * 64, c0 = blockIdx.y * 64;
  const int bh = blockIdx.z, b = bh / H, h = bh % H;
  const int tx = threadIdx.x % 64, ty = threadIdx.x / 64;
  for (int r = ty; r < 64; r += 4) {
    const int j = j0 + r;
    tile[r][tx] = (j < Lk && c0 + tx < d)
                      ? to_f32<BF16>(v[((static_cast<size_t>(b) * Lk + j) * H + h) * d + c0 + tx])
                      : 0.f;
  }
  __syncthreads();
  const int c = threadIdx.x / 16, jj = (threadIdx.x % 16) * 4;
  for (int cc = c; cc < 64; cc += 16) {
    const int j = j0 + jj;
    if (j >= Lk || c0 + cc >= d) continue;
    const float sc = slice_scale(__uint_as_float(amax_bits[static_cast<size_t>(bh) * d + c0 + cc]));
    uint8_t* dst = vt + ((static_cast<size_t>(b) * H + h) * d + c0 + cc) * pitch + j;
    if (!ATTN_CHECK(Lk <= pitch && (pitch & 3) == 0 && (j & 3) == 0, 33)) continue;
    const uint32_t w = e4m3x2(__fdiv_rn(tile[jj][cc], sc), __fdiv_rn(tile[jj + 1][cc], sc)) |
                       (e4m3x2(__fdiv_rn(tile[jj + 2][cc], sc), __fdiv_rn(tile[jj + 3][cc], sc)) << 16);
    if (j + 4 <= Lk) {
      *reinterpret_cast<uint32_t*>(dst) = w;
    } else {
      for (int e = 0; e < Lk - j; ++e) dst[e] = static_cast<uint8_t>(w >> (8 * e));
    }
  }
}

// Column maxima (float bits) to scales, in place.
__global__ void __launch_bounds__(256) amax_to_scale_kernel(float* __restrict__ sv, int n) {
  const int i = blockIdx.x * 256 + threadIdx.x;
  if (i < n) sv[i] = slice_scale(sv[i]);
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
  if (B < 1 || Lk < 1 || Hkv < 1 || d < 16 || d > 256 || (d & (d - 1)) != 0 || pitch < Lk || pitch % 16 != 0)
    return ATTN_ERR_INVALID_ARG;
  if (!aligned(v, 16) || !aligned(vt, 16)) return ATTN_ERR_INVALID_ARG;
  const size_t nv = 2ull * B * Lk * Hkv * d, nvt = 1ull * B * Hkv * d * pitch;
  if (overlap(v, nv, vt, nvt)) return ATTN_ERR_INVALID_ARG;
  if (static_cast<long long>(B) * Hkv > 65535) return ATTN_ERR_INVALID_ARG;
  dim3 grid((Lk + 63) / 64, (d + 63) / 64, B * Hkv);
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

extern "C" int attn_fp8_quantize_tokens(const void* x, void* y, float* s, int B, int L, int H, int d,
                                        int s_pitch, int dtype, void* stream) {
  if (x == nullptr || y == nullptr || s == nullptr) return ATTN_ERR_INVALID_ARG;
  if (dtype != ATTN_DTYPE_BF16 && dtype != ATTN_DTYPE_FP16) return ATTN_ERR_INVALID_ARG;
  if (B < 1 || L < 1 || H < 1 || d < 16 || d > 256 || (d & (d - 1)) != 0 || s_pitch < L)
    return ATTN_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(y, 8) || !aligned(s, 4)) return ATTN_ERR_INVALID_ARG;
  const size_t n = 1ull * B * L * H * d, ns = 4ull * B * H * s_pitch;
  if (overlap(x, 2 * n, y, n) || overlap(x, 2 * n, s, ns) || overlap(y, n, s, ns)) return ATTN_ERR_INVALID_ARG;
  const int G = d / 8;
  const long long n_rows = 1ll * B * L * H;
  const long long blocks = (n_rows + 256 / G - 1) / (256 / G);
  const unsigned grid = static_cast<unsigned>(blocks < 148 * 16 ? blocks : 148 * 16);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  (void)cudaGetLastError();
  if (dtype == ATTN_DTYPE_BF16)
    quantize_tokens_kernel<true><<<grid, 256, 0, st>>>(static_cast<const uint4*>(x), static_cast<uint2*>(y), s,
                                                       n_rows, L, H, G, s_pitch);
  else
    quantize_tokens_kernel<false><<<grid, 256, 0, st>>>(static_cast<const uint4*>(x), static_cast<uint2*>(y), s,
                                                        n_rows, L, H, G, s_pitch);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

extern "C" int attn_fp8_quantize_vt(const void* v, void* vt, float* sv, int B, int Lk, int Hkv, int d,
                                    int pitch, int dtype, void* stream) {
  if (v == nullptr || vt == nullptr || sv == nullptr) return ATTN_ERR_INVALID_ARG;
  if (dtype != ATTN_DTYPE_BF16 && dtype != ATTN_DTYPE_FP16) return ATTN_ERR_INVALID_ARG;
  if (B < 1 || Lk < 1 || Hkv < 1 || d < 16 || d > 256 || (d & (d - 1)) != 0 || pitch < Lk || pitch % 16 != 0)
    return ATTN_ERR_INVALID_ARG;
  if (!aligned(v, 16) || !aligned(vt, 16) || !aligned(sv, 4)) return ATTN_ERR_INVALID_ARG;
  if (static_cast<long long>(B) * Hkv > 65535) return ATTN_ERR_INVALID_ARG;
  const size_t nv = 2ull * B * Lk * Hkv * d, nvt = 1ull * B * Hkv * d * pitch, ns = 4ull * B * Hkv * d;
  if (overlap(v, nv, vt, nvt) || overlap(v, nv, sv, ns) || overlap(vt, nvt, sv, ns)) return ATTN_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  (void)cudaGetLastError();
  if (cudaMemsetAsync(sv, 0, ns, st) != cudaSuccess) return ATTN_ERR_CUDA;
  const int G = d / 8, kpb = 256;
  const dim3 agrid((Lk + kpb - 1) / kpb, B * Hkv);
  const dim3 qgrid((Lk + 63) / 64, (d + 63) / 64, B * Hkv);
  unsigned* bits = reinterpret_cast<unsigned*>(sv);
  const int n = B * Hkv * d;
  if (dtype == ATTN_DTYPE_BF16) {
    column_amax_kernel<true><<<agrid, 256, 0, st>>>(static_cast<const uint4*>(v), bits, Lk, Hkv, G, kpb);
    quantize_vt_kernel<true><<<qgrid, 256, 0, st>>>(static_cast<const uint16_t*>(v), static_cast<uint8_t*>(vt),
                                                    bits, Lk, Hkv, d, pitch);
  } else {
    column_amax_kernel<false><<<agrid, 256, 0, st>>>(static_cast<const uint4*>(v), bits, Lk, Hkv, G, kpb);
    quantize_vt_kernel<false><<<qgrid, 256, 0, st>>>(static_cast<const uint16_t*>(v), static_cast<uint8_t*>(vt),
                                                     bits, Lk, Hkv, d, pitch);
  }
  amax_to_scale_kernel<<<(n + 255) / 256, 256, 0, st>>>(sv, n);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}
