// Q/K prologue for B200 (sm_100a): RMS normalisation, then rotary position
// embedding, of Q and of the new K chunk, in one launch.
//
// What is computed: the flashdreams.accelerated developer guide, "Multi Head
// Attention Definition": RMSNorm_gamma(z) = gamma * z / sqrt(mean(z^2) + eps)
// over each head (head scope, m = d) or over all heads of a token (inner
// scope, m = H d); then RoPE rotates feature pair r of the token at sequence
// index p by the angle rope_freqs[p, a_r], pairs (2r, 2r + 1) (interleaved) or
// (r, r + d/2) (split-half). Normalisation comes first, as on that page. V is
// neither normalised nor rotated.
//
// The work is an elementwise pass bound by HBM bandwidth: each element is read
// once and written once. One 128-thread block per token. The token's H d
// features are cut into 16-feature items, d / 16 per head; thread t handles
// items t, t + 128, ... An item is two 16-byte vectors of one head: features
// [o, o + 8) and [o + d/2, o + d/2 + 8) for split-half RoPE (so both features
// of every pair sit in one thread), [o, o + 16) otherwise. The d / 16 items of
// a head sit on adjacent lanes of one warp, so the head's sum of squares is a
// butterfly over those lanes. The rotation angles depend on the token's
// position and the feature only, not on the head: the block computes the d / 2
// cosines and sines once per token into shared memory and every head reuses
// them. Arithmetic in fp32; one rounding to the 16-bit type at the end.

#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>

#include "attn.h"

namespace hasb_pro {

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


constexpr int kWarps = 4;
constexpr int kThreads = 32 * kWarps;

// One input tensor [B, L, H, d] and where its tokens go: token (b, l) is
// written to token b * ystride + yoff + l of the output (ystride = L, yoff = 0
// for a plain [B, L, H, d] output; a cache slot range otherwise).
struct ProTensor {
  const void* x;
  void* y;
  const float* gamma;   // [m] or nullptr (all ones)
  const float* angles;  // [L, d] or nullptr (no RoPE)
  int L, H;
  int ystride, yoff;
  int raw;              // copy only: neither normalised nor rotated (V)
  // angle row of token position l: rows[l] when rows is set (a per-token
  // position map, e.g. cache slot -> cache-relative position), else l + row_off;
  // clamped to the table's n_rows rows
  const int* rows;
  int row_off, n_rows;
  int xstride;  // tokens per batch of the input (L, or a cache's S)
};

struct ProParams {
  ProTensor t[3];
  int tok_end[3];  // cumulative token counts: block i serves the first tensor with i < tok_end
  int d;
  float eps;  // normalisation scope and RoPE style are template arguments of the kernel
};

template <bool BF16>
__device__ __forceinline__ void unpack8(const uint4& v, float (&f)[8]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    if (BF16) {
      f[2 * i] = __uint_as_float(w[i] << 16);
      f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    } else {
      const __half2 h = *reinterpret_cast<const __half2*>(&w[i]);
      const float2 t = __half22float2(h);
      f[2 * i] = t.x;
      f[2 * i + 1] = t.y;
    }
  }
}

template <bool BF16>
__device__ __forceinline__ uint4 pack8(const float (&f)[8]) {
  uint32_t w[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    uint32_t r;
    if (BF16)
      asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(f[2 * i + 1]), "f"(f[2 * i]));
    else
      asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(f[2 * i + 1]), "f"(f[2 * i]));
    w[i] = r;
  }
  return make_uint4(w[0], w[1], w[2], w[3]);
}

// Feature index of element e (0..15) of item-offset o within its head.
__device__ __forceinline__ int item_feature(int o, int e, int d, bool split) {
  return split ? (e < 8 ? o + e : o + d / 2 + e - 8) : o + e;
}

// Which tensor, position and batch block-level token index `bid` names.
struct TokenAt {
  ProTensor T;
  int pos, bat;
};

__device__ __forceinline__ TokenAt token_at(const ProParams& p, int bid) {
  TokenAt a;
  const int which = bid < p.tok_end[0] ? 0 : (bid < p.tok_end[1] ? 1 : 2);
  a.T = which == 0 ? p.t[0] : (which == 1 ? p.t[1] : p.t[2]);
  const int token = bid - (which == 0 ? 0 : p.tok_end[which - 1]);  // b * L + l
  a.pos = token % a.T.L;                                            // sequence index l
  a.bat = token / a.T.L;
  return a;
}

__device__ __forceinline__ int angle_row(const ProTensor& T, int pos) {
  const int r = T.rows != nullptr ? __ldg(T.rows + pos) : pos + T.row_off;
  return r < 0 ? 0 : (r >= T.n_rows ? T.n_rows - 1 : r);
}

// One token (all its heads) of one tensor, by the whole block: `x` holds the
// token's H d input values and `ang` its d-entry angle row (either in global
// memory or staged in shared memory; `ang` unused without RoPE).
template <bool BF16, int SCOPE, int STYLE>
__device__ __forceinline__ void token_body(const ProParams& p, const ProTensor& T, int pos, int bat,
                                           const uint16_t* x, const float* ang, float* red, float* cs_s,
                                           float* sn_s) {
  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const bool raw = T.raw != 0;
  const int d = p.d;
  constexpr bool split = STYLE == ATTN_ROPE_SPLIT;
  // site 21: the token and its output slot lie inside the tensor and the cache's rows
  // (block-uniform: a failed check skips the whole token, barriers included)
  if (!ATTN_CHECK(pos >= 0 && pos < T.L && pos < T.xstride && T.yoff >= 0 && T.yoff + pos < T.ystride, 21))
    return;
  const int per_head = d / 16;                  // items per head
  const int sh = __ffs(per_head) - 1;           // log2(per_head)
  const int items = T.H * per_head;             // items of the token
  uint16_t* y = static_cast<uint16_t*>(T.y) +
                (static_cast<size_t>(bat) * T.ystride + T.yoff + pos) * T.H * d;
  // intra-head item index is the same for every item this thread handles
  // (128 is a multiple of d / 16)
  const int io = threadIdx.x % per_head;
  const int o = split ? 8 * io : 16 * io;       // first feature of the item in its head

  if constexpr (STYLE != ATTN_ROPE_NONE) {
    // pair r: first feature a_r = 2r (interleaved) or r (split-half)
    if (!raw && threadIdx.x < d / 2) {
      const int a = split ? threadIdx.x : 2 * threadIdx.x;
      sincosf(ang[a], &sn_s[threadIdx.x], &cs_s[threadIdx.x]);
    }
  }
  float ghead[16];
  if (SCOPE == ATTN_NORM_HEAD && !raw) {
#pragma unroll
    for (int e = 0; e < 16; ++e)
      ghead[e] = T.gamma != nullptr ? T.gamma[item_feature(o, e, d, split)] : 1.f;
  }

  auto load_item = [&](int it, float (&f)[16]) {
    const int h = it >> sh;
    const uint16_t* src = x + h * d + o;
    unpack8<BF16>(*reinterpret_cast<const uint4*>(src), *reinterpret_cast<float(*)[8]>(&f[0]));
    unpack8<BF16>(*reinterpret_cast<const uint4*>(src + (split ? d / 2 : 8)),
                  *reinterpret_cast<float(*)[8]>(&f[8]));
  };

  // inner scope: one sum of squares over the whole token first
  float inv_token = 1.f;
  if (SCOPE == ATTN_NORM_INNER && !raw) {
    float ss = 0.f;
    for (int it = threadIdx.x; it < items; it += kThreads) {
      float f[16];
      load_item(it, f);
#pragma unroll
      for (int e = 0; e < 16; ++e) ss = fmaf(f[e], f[e], ss);
    }
#pragma unroll
    for (int s = 16; s > 0; s >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, s);
    if (lane == 0) red[warp] = ss;
  }
  __syncthreads();  // cos / sin table and partial sums visible
  if (SCOPE == ATTN_NORM_INNER && !raw) {
    const float tot = (red[0] + red[1]) + (red[2] + red[3]);
    inv_token = rsqrtf(tot / static_cast<float>(T.H * d) + p.eps);
  }
  float c8[8], s8[8];
  if (STYLE != ATTN_ROPE_NONE && !raw) {
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      // split: element e and e + 8 form pair o/1 + e; interleaved: elements
      // 2m, 2m + 1 form pair o/2 + m
      const int r = split ? o + e : o / 2 + e;
      c8[e] = cs_s[r];
      s8[e] = sn_s[r];
    }
  }

  const int rounds = (items + kThreads - 1) / kThreads;
  for (int k = 0; k < rounds; ++k) {
    const int it = threadIdx.x + k * kThreads;
    const bool live = it < items;
    float2 f[8];  // f[m] = (element 2m, element 2m + 1) of the item
    if (live) {
      load_item(it, *reinterpret_cast<float(*)[16]>(f));
    } else {
#pragma unroll
      for (int m = 0; m < 8; ++m) f[m] = make_float2(0.f, 0.f);
    }
    if (raw) {
      // copy only
    } else if (SCOPE == ATTN_NORM_HEAD) {
      float2 ss2 = make_float2(0.f, 0.f);
#pragma unroll
      for (int m = 0; m < 8; ++m) ss2 = __ffma2_rn(f[m], f[m], ss2);
      float ss = ss2.x + ss2.y;
      for (int q = 1; q < per_head; q <<= 1) ss += __shfl_xor_sync(0xffffffffu, ss, q);
      const float inv = rsqrtf(ss / static_cast<float>(d) + p.eps);
      const float2 inv2 = make_float2(inv, inv);
#pragma unroll
      for (int m = 0; m < 8; ++m)
        f[m] = __fmul2_rn(make_float2(ghead[2 * m], ghead[2 * m + 1]), __fmul2_rn(f[m], inv2));
    } else if (SCOPE == ATTN_NORM_INNER) {
      const float* g = (T.gamma != nullptr && live) ? T.gamma + (it >> sh) * d : nullptr;
      const float2 inv2 = make_float2(inv_token, inv_token);
#pragma unroll
      for (int m = 0; m < 8; ++m) {
        const float2 gg = g != nullptr ? make_float2(g[item_feature(o, 2 * m, d, split)],
                                                     g[item_feature(o, 2 * m + 1, d, split)])
                                       : make_float2(1.f, 1.f);
        f[m] = __fmul2_rn(gg, __fmul2_rn(f[m], inv2));
      }
    }
    if (raw) {
    } else if constexpr (split) {
      // element e (< 8) pairs with element e + 8: f[m] holds elements 2m, 2m+1
      // of the first vector, f[m + 4] the same two of the second
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const float2 a = f[m], b = f[m + 4];
        const float2 c = make_float2(c8[2 * m], c8[2 * m + 1]);
        const float2 sn = make_float2(s8[2 * m], s8[2 * m + 1]);
        f[m] = __ffma2_rn(a, c, __fmul2_rn(make_float2(-b.x, -b.y), sn));
        f[m + 4] = __ffma2_rn(a, sn, __fmul2_rn(b, c));
      }
    } else if (STYLE == ATTN_ROPE_INTERLEAVED) {
#pragma unroll
      for (int m = 0; m < 8; ++m) {
        const float a = f[m].x, b = f[m].y;
        f[m] = make_float2(a * c8[m] - b * s8[m], a * s8[m] + b * c8[m]);
      }
    }
    if (live) {
      uint16_t* dst = y + (it >> sh) * d + o;
      *reinterpret_cast<uint4*>(dst) = pack8<BF16>(*reinterpret_cast<const float(*)[8]>(&f[0]));
      *reinterpret_cast<uint4*>(dst + (split ? d / 2 : 8)) =
          pack8<BF16>(*reinterpret_cast<const float(*)[8]>(&f[4]));
    }
  }
}



// One block per token, operands read straight from global memory.
template <bool BF16, int SCOPE, int STYLE>
__global__ void __launch_bounds__(kThreads) qk_prologue_kernel(const ProParams p) {
  __shared__ float red[kWarps];
  __shared__ float cs_s[128], sn_s[128];  // cos / sin of the token's d/2 pair angles
  const TokenAt a = token_at(p, blockIdx.x);
  const uint16_t* x = static_cast<const uint16_t*>(a.T.x) +
                      (static_cast<size_t>(a.bat) * a.T.xstride + a.pos) * a.T.H * p.d;
  const float* ang = (STYLE != ATTN_ROPE_NONE && a.T.raw == 0)
                         ? a.T.angles + static_cast<size_t>(angle_row(a.T, a.pos)) * p.d
                         : nullptr;
  token_body<BF16, SCOPE, STYLE>(p, a.T, a.pos, a.bat, x, ang, red, cs_s, sn_s);
}

__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gmem_src) {
  const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(smem_dst));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d), "l"(gmem_src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }

// Persistent blocks, one token at a time, with the next token's bytes (and
// its angle row) copied into the other of two shared-memory buffers by
// cp.async while the current one is processed: the HBM round trip of a token
// hides behind the work on the previous one without holding registers.
// `buf` bytes per buffer: the largest token (H d 16-bit values) and an angle row.
#ifndef PRO_NBUF
#define PRO_NBUF 2
#endif
#ifndef PRO_MINB
#define PRO_MINB 1
#endif
constexpr int kStageBufs = PRO_NBUF;  // tokens in flight per block: the current one and the next ones

template <bool BF16, int SCOPE, int STYLE>
__global__ void __launch_bounds__(kThreads, PRO_MINB) qk_prologue_staged_kernel(const ProParams p, int buf) {
  extern __shared__ __align__(16) uint8_t stage[];
  __shared__ float red[kWarps];
  __shared__ float cs_s[128], sn_s[128];
  const int total = p.tok_end[2];
  const int d = p.d;
  auto issue = [&](int t, int b) {
    const TokenAt a = token_at(p, t);
    const uint8_t* src = static_cast<const uint8_t*>(a.T.x) +
                         (static_cast<size_t>(a.bat) * a.T.xstride + a.pos) * a.T.H * d * 2;
    uint8_t* dst = stage + b * buf;
    const int chunks = a.T.H * d * 2 / 16;
    for (int k = threadIdx.x; k < chunks; k += kThreads) cp_async16(dst + 16 * k, src + 16 * k);
    if (STYLE != ATTN_ROPE_NONE && a.T.raw == 0) {
      const float* arow = a.T.angles + static_cast<size_t>(angle_row(a.T, a.pos)) * d;
      uint8_t* adst = dst + buf - d * 4;
      for (int k = threadIdx.x; k < d / 4; k += kThreads) cp_async16(adst + 16 * k, arow + 4 * k);
    }
  };
  int t = blockIdx.x;
  if (t >= total) return;
#pragma unroll
  for (int q = 0; q < kStageBufs - 1; ++q) {  // the first tokens
    const int tq = t + q * static_cast<int>(gridDim.x);
    if (tq < total) issue(tq, q);
    cp_async_commit();
  }
  for (int n = 0; t < total; ++n, t += gridDim.x) {
    const int b = n % kStageBufs;
    const int ahead = t + (kStageBufs - 1) * static_cast<int>(gridDim.x);
    if (ahead < total) issue(ahead, (n + kStageBufs - 1) % kStageBufs);
    cp_async_commit();  // one group per token (empty past the last)
    // this thread's copies of token t have landed (only the newer groups may pend) ...
    asm volatile("cp.async.wait_group %0;" ::"n"(kStageBufs - 1) : "memory");
    __syncthreads();    // ... and so have everyone's
    const TokenAt a = token_at(p, t);
    const uint8_t* sb = stage + b * buf;
    token_body<BF16, SCOPE, STYLE>(p, a.T, a.pos, a.bat, reinterpret_cast<const uint16_t*>(sb),
                                   reinterpret_cast<const float*>(sb + buf - d * 4), red, cs_s, sn_s);
    __syncthreads();  // buffer b is read out before the next round refills it
  }
}

}  // namespace hasb_pro

using namespace hasb_pro;

namespace {

int sm_count() {
  static int sms = 0;
  if (sms == 0) {
    int dev = 0, n = 0;
    sms = (cudaGetDevice(&dev) == cudaSuccess &&
           cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && n > 0)
              ? n
              : 148;
  }
  return sms;
}

// `buf` > 0: the staged persistent kernel (as many blocks as fit on every SM,
// never more than tokens); 0: one block per token.
template <bool BF16, int SCOPE, int STYLE>
void launch_kernel(const ProParams& p, unsigned tokens, int buf, cudaStream_t s) {
  if (buf == 0) {
    qk_prologue_kernel<BF16, SCOPE, STYLE><<<tokens, kThreads, 0, s>>>(p);
    return;
  }
  auto kern = qk_prologue_staged_kernel<BF16, SCOPE, STYLE>;
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kThreads, kStageBufs * buf) != cudaSuccess ||
      per_sm < 1)
    per_sm = 1;
  const unsigned g = static_cast<unsigned>(sm_count() * per_sm);
  kern<<<tokens < g ? tokens : g, kThreads, kStageBufs * buf, s>>>(p, buf);
}

template <bool BF16, int SCOPE>
void launch_style(const ProParams& p, int style, unsigned tokens, int buf, cudaStream_t s) {
  if (style == ATTN_ROPE_NONE)
    launch_kernel<BF16, SCOPE, ATTN_ROPE_NONE>(p, tokens, buf, s);
  else if (style == ATTN_ROPE_INTERLEAVED)
    launch_kernel<BF16, SCOPE, ATTN_ROPE_INTERLEAVED>(p, tokens, buf, s);
  else
    launch_kernel<BF16, SCOPE, ATTN_ROPE_SPLIT>(p, tokens, buf, s);
}

template <bool BF16>
void launch_scope(const ProParams& p, int scope, int style, unsigned tokens, int buf, cudaStream_t s) {
  if (scope == ATTN_NORM_NONE)
    launch_style<BF16, ATTN_NORM_NONE>(p, style, tokens, buf, s);
  else if (scope == ATTN_NORM_HEAD)
    launch_style<BF16, ATTN_NORM_HEAD>(p, style, tokens, buf, s);
  else
    launch_style<BF16, ATTN_NORM_INNER>(p, style, tokens, buf, s);
}

// Staging buffer bytes for the tensors of `p` (the largest token plus an
// angle row, 16-byte multiple), or 0 when a token is too large for two
// buffers in 48 KB or an angle table is not 16-byte aligned.
int staging_bytes(const ProParams& p, int style) {
  int tok = 0;
  for (int i = 0; i < 3; ++i) {
    const int n = (i == 0 ? p.tok_end[0] : p.tok_end[i] - p.tok_end[i - 1]);
    if (n <= 0) continue;
    const ProTensor& T = p.t[i];
    tok = T.H * p.d * 2 > tok ? T.H * p.d * 2 : tok;
    if (style != ATTN_ROPE_NONE && !T.raw && (reinterpret_cast<uintptr_t>(T.angles) & 15u) != 0) return 0;
  }
  const int buf = (tok + p.d * 4 + 15) / 16 * 16;
  return kStageBufs * buf <= 48 * 1024 ? buf : 0;
}

void launch_prologue(const ProParams& p, bool bf16, int scope, int style, unsigned tokens,
                     cudaStream_t s) {
  const int buf = staging_bytes(p, style);
  if (bf16)
    launch_scope<true>(p, scope, style, tokens, buf, s);
  else
    launch_scope<false>(p, scope, style, tokens, buf, s);
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

bool overlap(const void* a, size_t na, const void* b, size_t nb) {
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return x < y + nb && y < x + na;
}

}  // namespace

extern "C" int attn_qk_prologue(const void* q, void* q_out, const void* k, void* k_out,
                                const float* gamma_q, const float* gamma_k, const float* angles_q,
                                const float* angles_k, int B, int Lq, int Lk, int Hq, int Hkv, int d,
                                int norm_scope, float eps, int rope_style, int dtype, void* stream) {
  // ---- arguments (all checked before any CUDA call)
  if (q == nullptr || q_out == nullptr) return ATTN_ERR_INVALID_ARG;
  if ((k == nullptr) != (k_out == nullptr)) return ATTN_ERR_INVALID_ARG;
  if (dtype != ATTN_DTYPE_BF16 && dtype != ATTN_DTYPE_FP16) return ATTN_ERR_INVALID_ARG;
  if (norm_scope < ATTN_NORM_NONE || norm_scope > ATTN_NORM_INNER) return ATTN_ERR_INVALID_ARG;
  if (rope_style < ATTN_ROPE_NONE || rope_style > ATTN_ROPE_SPLIT) return ATTN_ERR_INVALID_ARG;
  if (!(eps >= 0.f) || !std::isfinite(eps)) return ATTN_ERR_INVALID_ARG;
  if (B < 1 || Lq < 1 || Hq < 1) return ATTN_ERR_INVALID_ARG;
  if (k != nullptr && (Lk < 1 || Hkv < 1)) return ATTN_ERR_INVALID_ARG;
  if (d < 16 || d > 256 || (d & (d - 1)) != 0) return ATTN_ERR_UNSUPPORTED;
  if ((rope_style != ATTN_ROPE_NONE) != (angles_q != nullptr)) return ATTN_ERR_INVALID_ARG;
  if (k != nullptr && (rope_style != ATTN_ROPE_NONE) != (angles_k != nullptr)) return ATTN_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(q_out, 16) || (k && (!aligned(k, 16) || !aligned(k_out, 16))))
    return ATTN_ERR_INVALID_ARG;
  for (const float* f : {gamma_q, gamma_k, angles_q, angles_k})
    if (f != nullptr && !aligned(f, 4)) return ATTN_ERR_INVALID_ARG;
  const long long nq = 1LL * B * Lq * Hq * d, nk = k ? 1LL * B * Lk * Hkv * d : 0;
  const long long tokens = 1LL * B * Lq + (k ? 1LL * B * Lk : 0);
  if (tokens > 0x7fffffffLL || 1LL * Hq * d > (1 << 20) || 1LL * Hkv * d > (1 << 20))
    return ATTN_ERR_INVALID_ARG;
  // outputs may be their own input (in place) but may not overlap anything else
  if (q_out != q && overlap(q_out, nq * 2, q, nq * 2)) return ATTN_ERR_INVALID_ARG;
  if (k != nullptr) {
    if (k_out != k && overlap(k_out, nk * 2, k, nk * 2)) return ATTN_ERR_INVALID_ARG;
    if (overlap(q_out, nq * 2, k, nk * 2) || overlap(k_out, nk * 2, q, nq * 2) ||
        overlap(q_out, nq * 2, k_out, nk * 2))
      return ATTN_ERR_INVALID_ARG;
  }

  ProParams p{};
  p.t[0] = ProTensor{q, q_out, norm_scope ? gamma_q : nullptr, angles_q, Lq, Hq, Lq, 0, 0, nullptr, 0, Lq, Lq};
  p.t[1] = ProTensor{k, k_out, norm_scope ? gamma_k : nullptr, angles_k, Lk, Hkv, Lk, 0, 0, nullptr, 0, Lk, Lk};
  p.tok_end[0] = B * Lq;
  p.tok_end[1] = p.tok_end[2] = static_cast<int>(tokens);
  p.d = d;
  p.eps = eps;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  (void)cudaGetLastError();
  launch_prologue(p, dtype == ATTN_DTYPE_BF16, norm_scope, rope_style, static_cast<unsigned>(tokens), s);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

extern "C" int attn_stream_update(const void* q, void* q_out, const void* k, const void* v,
                                  void* k_cache, void* v_cache, const float* gamma_q,
                                  const float* gamma_k, const float* angles_q, const float* angles_k,
                                  int B, int L, int S, int slot, int Hq, int Hkv, int d,
                                  int norm_scope, float eps, int rope_style, int dtype, void* stream) {
  // ---- arguments (all checked before any CUDA call)
  if (k == nullptr || v == nullptr || k_cache == nullptr || v_cache == nullptr)
    return ATTN_ERR_INVALID_ARG;
  if ((q == nullptr) != (q_out == nullptr)) return ATTN_ERR_INVALID_ARG;
  if (dtype != ATTN_DTYPE_BF16 && dtype != ATTN_DTYPE_FP16) return ATTN_ERR_INVALID_ARG;
  if (norm_scope < ATTN_NORM_NONE || norm_scope > ATTN_NORM_INNER) return ATTN_ERR_INVALID_ARG;
  if (rope_style < ATTN_ROPE_NONE || rope_style > ATTN_ROPE_SPLIT) return ATTN_ERR_INVALID_ARG;
  if (!(eps >= 0.f) || !std::isfinite(eps)) return ATTN_ERR_INVALID_ARG;
  if (B < 1 || L < 1 || Hkv < 1 || (q != nullptr && Hq < 1)) return ATTN_ERR_INVALID_ARG;
  if (slot < 0 || S < 1 || L > S || slot > S - L) return ATTN_ERR_INVALID_ARG;
  if (d < 16 || d > 256 || (d & (d - 1)) != 0) return ATTN_ERR_UNSUPPORTED;
  if ((rope_style != ATTN_ROPE_NONE) != (angles_k != nullptr)) return ATTN_ERR_INVALID_ARG;
  if (q != nullptr && (rope_style != ATTN_ROPE_NONE) != (angles_q != nullptr)) return ATTN_ERR_INVALID_ARG;
  for (const void* t : {q, static_cast<const void*>(q_out), k, v, static_cast<const void*>(k_cache),
                        static_cast<const void*>(v_cache)})
    if (t != nullptr && !aligned(t, 16)) return ATTN_ERR_INVALID_ARG;
  for (const float* f : {gamma_q, gamma_k, angles_q, angles_k})
    if (f != nullptr && !aligned(f, 4)) return ATTN_ERR_INVALID_ARG;
  const long long tok_q = q ? 1LL * B * L : 0, tok_kv = 1LL * B * L;
  if (tok_q + 2 * tok_kv > 0x7fffffffLL || 1LL * Hq * d > (1 << 20) || 1LL * Hkv * d > (1 << 20))
    return ATTN_ERR_INVALID_ARG;
  const size_t nq = static_cast<size_t>(tok_q) * Hq * d * 2, nkv = static_cast<size_t>(tok_kv) * Hkv * d * 2;
  const size_t ncache = static_cast<size_t>(B) * S * Hkv * d * 2;
  // the caches are written: they may overlap no input and not each other; q_out
  // may be q (in place) and may overlap nothing else
  if (overlap(k_cache, ncache, v_cache, ncache)) return ATTN_ERR_INVALID_ARG;
  for (const void* c : {static_cast<const void*>(k_cache), static_cast<const void*>(v_cache)}) {
    if (overlap(c, ncache, k, nkv) || overlap(c, ncache, v, nkv)) return ATTN_ERR_INVALID_ARG;
    if (q != nullptr && (overlap(c, ncache, q, nq) || overlap(c, ncache, q_out, nq)))
      return ATTN_ERR_INVALID_ARG;
  }
  if (q != nullptr) {
    if (q_out != q && overlap(q_out, nq, q, nq)) return ATTN_ERR_INVALID_ARG;
    if (overlap(q_out, nq, k, nkv) || overlap(q_out, nq, v, nkv)) return ATTN_ERR_INVALID_ARG;
  }

  ProParams p{};
  p.t[0] = ProTensor{q, q_out, norm_scope ? gamma_q : nullptr, angles_q, L, Hq, L, 0, 0, nullptr, 0, L, L};
  p.t[1] = ProTensor{k, k_cache, norm_scope ? gamma_k : nullptr, angles_k, L, Hkv, S, slot, 0, nullptr, 0, L, L};
  p.t[2] = ProTensor{v, v_cache, nullptr, nullptr, L, Hkv, S, slot, 1, nullptr, 0, 0, L};
  p.tok_end[0] = static_cast<int>(tok_q);
  p.tok_end[1] = static_cast<int>(tok_q + tok_kv);
  p.tok_end[2] = static_cast<int>(tok_q + 2 * tok_kv);
  p.d = d;
  p.eps = eps;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  (void)cudaGetLastError();
  launch_prologue(p, dtype == ATTN_DTYPE_BF16, norm_scope, rope_style,
                  static_cast<unsigned>(p.tok_end[2]), s);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

extern "C" int attn_rope_after_cache(const void* q, void* q_out, const void* k_cache, void* k_rot,
                                     const float* angles, int n_angle_rows, int q_row0,
                                     const int* k_rows, int B, int Lq, int Lk, int S, int Hq, int Hkv,
                                     int d, int rope_style, int dtype, void* stream) {
  // ---- arguments (all checked before any CUDA call)
  if (q == nullptr || q_out == nullptr || k_cache == nullptr || k_rot == nullptr || angles == nullptr)
    return ATTN_ERR_INVALID_ARG;
  if (dtype != ATTN_DTYPE_BF16 && dtype != ATTN_DTYPE_FP16) return ATTN_ERR_INVALID_ARG;
  if (rope_style != ATTN_ROPE_INTERLEAVED && rope_style != ATTN_ROPE_SPLIT) return ATTN_ERR_INVALID_ARG;
  if (B < 1 || Lq < 1 || Lk < 1 || S < Lk || Hq < 1 || Hkv < 1 || n_angle_rows < 1) return ATTN_ERR_INVALID_ARG;
  if (q_row0 < 0 || static_cast<long long>(q_row0) + Lq > n_angle_rows) return ATTN_ERR_INVALID_ARG;
  if (k_rows == nullptr && Lk > n_angle_rows) return ATTN_ERR_INVALID_ARG;
  if (d < 16 || d > 256 || (d & (d - 1)) != 0) return ATTN_ERR_UNSUPPORTED;
  if (!aligned(q, 16) || !aligned(q_out, 16) || !aligned(k_cache, 16) || !aligned(k_rot, 16) ||
      !aligned(angles, 4) || (k_rows != nullptr && !aligned(k_rows, 4)))
    return ATTN_ERR_INVALID_ARG;
  const long long nq = 1LL * B * Lq * Hq * d, nk = 1LL * B * S * Hkv * d;
  if (1LL * B * (Lq + Lk) > 0x7fffffffLL || 1LL * Hq * d > (1 << 20) || 1LL * Hkv * d > (1 << 20))
    return ATTN_ERR_INVALID_ARG;
  if (q_out != q && overlap(q_out, nq * 2, q, nq * 2)) return ATTN_ERR_INVALID_ARG;
  if (overlap(k_rot, nk * 2, k_cache, nk * 2) || overlap(q_out, nq * 2, k_rot, nk * 2) ||
      overlap(q_out, nq * 2, k_cache, nk * 2) || overlap(k_rot, nk * 2, q, nq * 2))
    return ATTN_ERR_INVALID_ARG;

  ProParams p{};
  p.t[0] = ProTensor{q, q_out, nullptr, angles, Lq, Hq, Lq, 0, 0, nullptr, q_row0, n_angle_rows, Lq};
  // the first Lk slots of each batch's cache, in storage order, to the same slots of k_rot
  p.t[1] = ProTensor{k_cache, k_rot, nullptr, angles, Lk, Hkv, S, 0, 0, k_rows, 0, n_angle_rows, S};
  p.tok_end[0] = B * Lq;
  p.tok_end[1] = p.tok_end[2] = B * (Lq + Lk);
  p.d = d;
  p.eps = 0.f;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  (void)cudaGetLastError();
  launch_prologue(p, dtype == ATTN_DTYPE_BF16, ATTN_NORM_NONE, rope_style, static_cast<unsigned>(p.tok_end[2]),
                  st);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}
