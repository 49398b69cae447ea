// Fused attention forward for B200 (sm_100a): TMA-fed K/V ring, tcgen05 MMAs
// accumulating in tensor memory, warp-specialised load / MMA / softmax roles,
// exp2 online softmax with lazy O rescaling, mask-tile skipping, GQA indexing.
//
// What is computed: the per-head scaled dot-product attention of the
// flashdreams.accelerated developer guide ("Multi Head Attention Definition",
// the equation for A_h), O = softmax(scale * Q K^T + mask) V, for token-major
// [B, L, H, d] tensors, plus the per-row log-sum-exp. The skill page
// "optimizing-attention-flash" ("Quick start") names the IO-aware tiling this
// kernel uses: scores never leave the chip; each KV tile updates a running row
// max / row sum and the output accumulator (the exact online rewrite of the
// softmax).
//
// CTA organisation (one persistent CTA per SM, 384 threads):
//   warps 0-3   softmax for query tile 0 (rows r0 .. r0+127 of a work unit)
//   warps 4-7   softmax for query tile 1 (rows r0+128 .. r0+255)
//   warp  8     TMA producer: Q tiles, then K_0, V_0, K_1, V_1, ... into a ring
//               (at d = 256: K_0, K_1, V_0, K_2, V_1, ..., K one tile ahead)
//   warps 9, 10 MMA issuers (one thread each), warp 9 + t for query tile t:
//               S_t = Q_t K^T and O_t += P_t V
//   warp  11    O store: staged O tiles to global memory by TMA
// A work unit is (batch, query head, 256-row pair of query tiles). Tensor
// memory holds S_0, S_1 (128 fp32 columns each, P aliased as packed 16-bit in
// the first 64 columns) and O_0, O_1 (d columns each). At d = 256 a unit is
// one query tile: warps 0-3 run its softmax, warp 9 issues Q K^T into two
// alternating S buffers, warp 10 issues P V, and the softmax stores O.

#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "attn.h"
#include "sm100_ptx.cuh"

#ifndef POLY_PAIRS_PER8
#define POLY_PAIRS_PER8 0
#endif

namespace hasb {

// Device fault word: bit set by a kernel whose bounded wait ran out.
__device__ unsigned int g_fault_bits = 0;
// Debug build (-DATTN_DEBUG): the site number of the first index check that
// failed in this file's kernels (0: none).
__device__ unsigned int g_debug_site = 0;

enum FaultBit : unsigned int {
  kFaultLoadQEmpty = 1u << 0,
  kFaultLoadKvEmpty = 1u << 1,
  kFaultMmaQFull = 1u << 2,
  kFaultMmaKvFull = 1u << 3,
  kFaultMmaPFull = 1u << 4,
  kFaultSoftmaxSFull = 1u << 5,
  kFaultSoftmaxOFull = 1u << 6,
  kFaultSoftmaxTurn = 1u << 7,
  kFaultStore = 1u << 9,
  kFaultSelftest = 1u << 8,
  kFaultMmaSFree = 1u << 10,
  kFaultBounds = 1u << 11,  // debug build: an index check failed (site in attn_debug_fault_site)
};

// Index checks of the debug build (-DATTN_DEBUG): a check that fails sets
// kFaultBounds, records its site number (the first failure wins) and makes
// the caller skip the access; the kernel goes on, so no wait of another role
// is left without its arrival. In the release build a check is `true` and
// compiles away.
__device__ __forceinline__ bool debug_check(bool ok, unsigned int site) {
  if (!ok) {
    atomicOr(&g_fault_bits, kFaultBounds);
    atomicCAS(&g_debug_site, 0u, site);
  }
  return ok;
}
#ifdef ATTN_DEBUG
#define ATTN_CHECK(cond, site) (::hasb::debug_check((cond), (site)))
#else
#define ATTN_CHECK(cond, site) true
#endif

constexpr int kThreads = 384;
// Register split: 384 threads x 168 launch registers = 64512. The producer
// warpgroup (warps 8-11) drops to 72, the two softmax warpgroups rise to 216:
// 128 x 72 + 256 x 216 = 64512.
constexpr int kRegsProducer = 72;
constexpr int kRegsSoftmax = 216;
constexpr int kTileRows = 128;         // query rows per softmax tile = keys per KV tile
constexpr float kRescaleTau = 8.0f;    // lazy rescale threshold, log2 units (P <= 256)
constexpr float kLn2 = 0.69314718055994531f;
constexpr float kLog2e = 1.4426950408889634f;

template <int D, int F8 = 0>
struct Cfg {
  static constexpr int kChunks = D / 64;              // 128-byte swizzle chunks per row
  static constexpr int kChunkBytes = kTileRows * 128;  // one chunk of a 128-row tile
  static constexpr int kTileBytes = kTileRows * D * 2;
  static constexpr int kStages = (D == 128) ? 4 : 8;   // K/V ring depth (128 KB)
  static constexpr int kOffQ = 0;
  static constexpr int kOffKV = 2 * kTileBytes;
  static constexpr int kOffStg = kOffKV + kStages * kTileBytes;  // O staging for the TMA store
  static constexpr int kOffBar = kOffStg + kTileBytes;
  static constexpr int kOffMl = kOffBar + 512;  // pair-split merge: slot 1's (reference, row sum) per row
  static constexpr int kSmemBytes = kOffMl + 1024 + 1024;  // + 1 KB alignment slack
  // tensor-memory columns of S_t (P_t aliased) and O_t
  static __device__ __forceinline__ uint32_t col_s(int t) { return t ? 128u : 0u; }
  static __device__ __forceinline__ uint32_t col_o(int t) { return t ? 256u + D : 256u; }
  static constexpr uint32_t kTmemCols = 512;
  static_assert(256 + 2 * D <= 512, "S_0, S_1, O_0, O_1 must fit the 512 tensor-memory columns");
  static constexpr int kOChunks = D / 64;  // 64-column chunks of the 16-bit O staging tile
  static constexpr int kOffP = 0;          // P lives in tensor memory
  static constexpr int kOffSk = 0;         // no key scales
};

// d = 256: one 128-row query tile per unit. Tensor memory holds two S buffers
// (128 columns each, alternating over KV tiles, P aliased as for the other
// head dims) and O (256 columns); shared memory holds the Q tile (64 KB) and a
// two-stage K/V ring (64 KB a tile). O goes from registers straight to global
// memory, so there is no staging buffer.
template <>
struct Cfg<256, 0> {
  static constexpr int kChunks = 4;
  static constexpr int kChunkBytes = kTileRows * 128;
  static constexpr int kTileBytes = kTileRows * 256 * 2;
  static constexpr int kStages = 2;
  static constexpr int kOffQ = 0;
  static constexpr int kOffKV = kTileBytes;
  static constexpr int kOffStg = 0;
  static constexpr int kOffBar = kOffKV + kStages * kTileBytes;
  static constexpr int kSmemBytes = kOffBar + 512 + 1024;
  static __device__ __forceinline__ uint32_t col_s(int buf) { return buf ? 128u : 0u; }
  static __device__ __forceinline__ uint32_t col_o(int) { return 256u; }
  static constexpr uint32_t kTmemCols = 512;
  static constexpr int kOChunks = 4;
  static constexpr int kOffP = 0;
  static constexpr int kOffSk = 0;
};

// e4m3 operands, d = 128: a Q / K row is one 128-byte swizzle chunk (16 KB per
// 128-row tile), V arrives transposed (a tile is 128 d-rows of 128 keys) so
// both P V operands are K-major, and P goes through shared memory (two 16 KB
// buffers, K-major with the same swizzle) instead of tensor memory. MODE 2
// (per-token scales) adds one 512-byte buffer of key scales per softmax warp
// and gives up one ring stage for it.
template <int MODE>
struct CfgE4m3 {
  static constexpr int kChunks = 1;
  static constexpr int kChunkBytes = kTileRows * 128;
  static constexpr int kTileBytes = kTileRows * 128;
  static constexpr int kStages = MODE == 2 ? 7 : 8;
  static constexpr int kOChunks = 2;
  static constexpr int kOffQ = 0;
  static constexpr int kOffKV = 2 * kTileBytes;
  static constexpr int kOffP = kOffKV + kStages * kTileBytes;
  static constexpr int kOffStg = kOffP + 2 * kTileBytes;
  static constexpr int kOffSk = kOffStg + kOChunks * kChunkBytes;
  static constexpr int kOffBar = kOffSk + (MODE == 2 ? 8 * 512 : 0);
  static constexpr int kSmemBytes = kOffBar + 512 + 1024;
  static __device__ __forceinline__ uint32_t col_s(int t) { return t ? 128u : 0u; }
  static __device__ __forceinline__ uint32_t col_o(int t) { return t ? 384u : 256u; }
  static constexpr uint32_t kTmemCols = 512;
};
template <>
struct Cfg<128, 1> : CfgE4m3<1> {};
// e4m3 at d = 256: one query tile per unit as for 16-bit d = 256; a Q / K row
// is two 128-byte chunks (32 KB per tile), a V^T tile 256 d-rows of 128 keys;
// P for each of the two S buffers in shared memory (16 KB each).
template <>
struct Cfg<256, 1> {
  static constexpr int kChunks = 2;
  static constexpr int kChunkBytes = kTileRows * 128;
  static constexpr int kTileBytes = 2 * kChunkBytes;
  static constexpr int kStages = 4;
  static constexpr int kOChunks = 4;
  static constexpr int kOffQ = 0;
  static constexpr int kOffKV = kTileBytes;
  static constexpr int kOffP = kOffKV + kStages * kTileBytes;
  static constexpr int kOffStg = 0;
  static constexpr int kOffSk = 0;
  static constexpr int kOffBar = kOffP + 2 * kChunkBytes;
  static constexpr int kSmemBytes = kOffBar + 512 + 1024;
  static __device__ __forceinline__ uint32_t col_s(int buf) { return buf ? 128u : 0u; }
  static __device__ __forceinline__ uint32_t col_o(int) { return 256u; }
  static constexpr uint32_t kTmemCols = 512;
};
// per-token scales at d = 256: the key scales of the current tile, one
// 512-byte copy per softmax warp
template <>
struct Cfg<256, 2> : Cfg<256, 1> {
  static constexpr int kOffSk = Cfg<256, 1>::kOffBar;
  static constexpr int kOffBar = kOffSk + 4 * 512;
  static constexpr int kSmemBytes = kOffBar + 512 + 1024;
};
template <>
struct Cfg<128, 2> : CfgE4m3<2> {};

// barrier slots (8 bytes each) in the barrier area
enum Bar : int {
  kBarQFull = 0,    // [2] TMA -> MMA: Q tile t landed
  kBarQEmpty = 2,   // [2] MMA -> TMA: last S_t of the unit done, Q tile t reusable
  kBarSFull = 4,    // [2] MMA -> softmax t: S_t ready (also: previous PV_t done)
  kBarPFull = 6,    // [2] softmax t -> MMA: all of P_t written (one arrival per warp)
  kBarOFull = 8,    // [2] MMA -> softmax t: O_t final for the unit
  kBarDrain = 10,   // [2] MMA issuer t, abort path: all its MMAs done
  kBarPHalf = 12,   // [2] softmax t -> MMA: first half of P_t (keys 0-63) written
  kBarTurn = 14,    // [2] softmax 1-t -> softmax t: t may run its exponentials now
  kBarKvFull = 16,  // [kStages] TMA -> MMA
  kBarKvEmpty = 24, // [kStages] both MMA issuers -> TMA
  kBarStgFull = 32, //     softmax t -> store warp: O tile t staged (one arrival per warp)
  kBarStgFree = 34, // [2] store warp -> softmax t: staging buffer is t's to fill
  kBarSFree = 36,   // [2] d = 256, P V issuer -> Q K^T issuer: the P V that read S buffer b is done
  kBarMerge1 = 38,  //     pair split, softmax 1 -> softmax 0: slot 1's (reference, row sum) written
  kBarMerged = 39,  //     pair split, softmax 0 -> softmax 1: the merge has read slot 1's O and row state
};

// Exponentials of the softmax: kPolyPairsPer8 of every 8 score pairs take
// exp2_poly_x2 on the FMA pipe instead of the MUFU (16 ex2 per clock per SM).
// Measured on B200 the exponential loop is bound by instruction issue, not by
// the MUFU, so the default is 0; the polynomial stays available (and tested)
// for shapes where the MUFU saturates.
constexpr int kPolyPairsPer8 = POLY_PAIRS_PER8;
// The same split for the e4m3 path, whose GEMMs take half the time.
#ifndef F8_PACKED_KEY_SCALE
#define F8_PACKED_KEY_SCALE 1
#endif
#ifndef F8_POLY_PAIRS_PER8
#define F8_POLY_PAIRS_PER8 0
#endif
constexpr int kF8PolyPairsPer8 = F8_POLY_PAIRS_PER8;

// 2^x for a pair of floats on the FMA pipe: x = j + f with j = round(x) and
// f in [-1/2, 1/2]; 2^f from a degree-3 polynomial minimising the maximum
// relative error on that interval (7.5e-5; coefficients from
// gen_exp2_poly.py), 2^j added into the exponent field. x is clamped below at
// -125, so results under 2^-125 come out near 2^-125 (masked keys are zeroed
// by the caller; every other P is far above that).
__device__ __forceinline__ uint64_t exp2_poly_x2(uint64_t x2) {
  constexpr float c0 = 0.9999280571937561f, c1 = 0.6932609677314758f;
  constexpr float c2 = 0.2426111251115799f, c3 = 0.0551716685295105f;
  constexpr float kRound = 12582912.0f;  // 1.5 * 2^23: x + kRound holds round(x) in its low bits
  float a, b;
  f2_unpack(x2, a, b);
  x2 = f2_pack(fmaxf(a, -125.f), fmaxf(b, -125.f));
  const uint64_t t = f2_add(x2, f2_pack(kRound, kRound));
  const uint64_t j = f2_add(t, f2_pack(-kRound, -kRound));  // round(x), as float
  const uint64_t f = f2_fma(j, f2_pack(-1.f, -1.f), x2);     // x - round(x), exact
  uint64_t q = f2_fma(f2_pack(c3, c3), f, f2_pack(c2, c2));
  q = f2_fma(q, f, f2_pack(c1, c1));
  q = f2_fma(q, f, f2_pack(c0, c0));
  float q0, q1, t0, t1;
  f2_unpack(q, q0, q1);
  f2_unpack(t, t0, t1);
  // the bits of t are 0x4B400000 + j; shifted left by 23 only j << 23 remains
  const uint32_t r0 = __float_as_uint(q0) + (__float_as_uint(t0) << 23);
  const uint32_t r1 = __float_as_uint(q1) + (__float_as_uint(t1) << 23);
  return f2_pack_bits(r0, r1);
}

struct FwdParams {
  void* o;
  float* lse;
  int B, Lq, Lk, Hq, Hkv, group, kv_offset;
  int kv_limit;      // keys visible to every row (masks 0 and 2): Lk or kv_offset + Lq
  int n_pairs;       // ceil(Lq / 256)
  int n_units;       // B * Hq * n_pairs * n_splits
  float sl2;         // scale * log2(e)
  unsigned long long timeout_ns;
  // key split (masks 0 and 2 only): unit s of a query pair covers KV tiles
  // s * split_tiles .. (s + 1) * split_tiles - 1 and writes float32 O / l and
  // LSE of its keys to o_part [n_splits, B, Hq, Lq, d], lse_part [n_splits, B, Hq, Lq]
  int n_splits, split_tiles;
  float* o_part;
  float* lse_part;
  // sliding window (left, right; -1 = unbounded): row i sees keys
  // p - left <= j <= p + right, p = kv_offset + i
  int win_left, win_right;
  // per-token scaled e4m3: the score of (row i, key j) is
  // scale * sq[b, hq, i] * sk[b, hkv, j] * (q8_i . k8_j); O column c is
  // multiplied by sv[b, hkv, c] (nullptr: 1)
  const float* sq;
  const float* sk;
  const float* sv;
  int sq_pitch, sk_pitch;
  // head dim of the tensors (<= D): d = 16 and 32 run the D = 64 kernel on
  // 64-wide TMA boxes whose columns >= d load as zero and are not stored
  int d;
};

// KV tiles of a work unit: the loader streams tiles j0 .. j0 + nu - 1 (the
// union of both query tiles' ranges); query tile t uses n_t of them, starting
// s_t tiles in. Without a window both ranges start at j0 and n0 <= n1 = nu.
struct Unit {
  int b, hq, hkv, r0, n0, n1;
  int j0, split;  // first KV tile, key split index
  int s0, s1, nu;
};

__device__ __forceinline__ int cdiv(int a, int b) { return (a + b - 1) / b; }

// The k-th work unit of this CTA, or -1 once none is left. Units are dealt in
// rounds of gridDim.x, alternately forward and backward: with units ordered
// longest first (causal), the CTA that takes one of the longest units of a
// round takes one of the shortest of the next. Every role of a CTA walks the
// same sequence. A partial round is always the last, so the walk stops at
// the first unit past the end.
__device__ __forceinline__ int cta_unit(int k, int n_units) {
  const int g = static_cast<int>(gridDim.x), c = static_cast<int>(blockIdx.x);
  const long long u = (k & 1) ? 1LL * (k + 1) * g - 1 - c : 1LL * k * g + c;
  return u < n_units ? static_cast<int>(u) : -1;
}

// Pair-split work unit (causal problems with fewer row pairs than SMs): u ->
// (b, hq, one 128-row query tile) whose n visible KV tiles are split between
// the CTA's two slots, slot 0 taking KV tiles [0, n0), slot 1 [n0, n),
// n0 = ceil(n / 2); the two partial results are merged by their row maxima
// and sums (the regrouped softmax) before the store. Units run longest first
// over all heads (the tile index varies slowest); p.n_pairs counts the tiles.
__device__ __forceinline__ Unit decode_pair(const FwdParams& p, int u) {
  Unit x;
  x.split = 0;
  const int bh = p.B * p.Hq;
  const int rank = u / bh;
  int t = u % bh;
  const int g = t % p.group;
  t /= p.group;
  x.hkv = t % p.Hkv;
  x.b = t / p.Hkv;
  x.hq = x.hkv * p.group + g;
  x.r0 = (p.n_pairs - 1 - rank) * kTileRows;
  const int n = cdiv(min(p.Lk, p.kv_offset + x.r0 + kTileRows), kTileRows);
  x.j0 = 0;
  x.n0 = (n + 1) / 2;
  x.n1 = n - x.n0;
  x.s0 = 0;
  x.s1 = x.n0;
  x.nu = n;
  return x;
}
// The two slots' KV tiles are streamed interleaved (0, n0, 1, n0 + 1, ...),
// slot 0's extra tile (n0 = n1 + 1) last: stream position of slot t's k-th
// tile, and the KV tile at a stream position.
__device__ __forceinline__ int pair_pos(const Unit& x, int t, int k) {
  return k < x.n1 ? 2 * k + t : x.n1 + k;
}
__device__ __forceinline__ int pair_tile(const Unit& x, int pos) {
  return pos < 2 * x.n1 ? ((pos & 1) ? x.n0 + pos / 2 : pos / 2) : pos - x.n1;
}

// Work unit u -> (b, hq, row pair). Query heads of one GQA group are adjacent
// and the row pairs of one head are adjacent, so CTAs running together read
// the same K/V head (L2 reuse). Causal units run longest first.
// d = 256: unit u -> (b, hq, 128-row tile); p.n_pairs counts tiles here.
// Same order as decode_unit (GQA group heads adjacent, causal longest first).
template <bool CAUSAL, bool SPLIT, bool WINDOW>
__device__ __forceinline__ Unit decode_single(const FwdParams& p, int u) {
  Unit x;
  if constexpr (SPLIT) {
    x.split = u % p.n_splits;
    u /= p.n_splits;
  } else {
    x.split = 0;
  }
  int tile = u % p.n_pairs;
  int t = u / p.n_pairs;
  const int g = t % p.group;
  t /= p.group;
  x.hkv = t % p.Hkv;
  x.b = t / p.Hkv;
  x.hq = x.hkv * p.group + g;
  if (CAUSAL) tile = p.n_pairs - 1 - tile;
  x.r0 = tile * kTileRows;
  x.s0 = x.s1 = 0;
  if constexpr (WINDOW) {
    // key range of the tile from its first and last real rows
    const int first = min(x.r0, p.Lq - 1), last = min(x.r0 + kTileRows - 1, p.Lq - 1);
    const int lo = p.win_left < 0 ? 0 : max(0, p.kv_offset + first - p.win_left);
    const int hi = p.win_right < 0 ? p.Lk : min(p.Lk, p.kv_offset + last + p.win_right + 1);
    x.j0 = lo / kTileRows;
    x.n0 = x.n1 = x.nu = cdiv(hi, kTileRows) - x.j0;
    return x;
  }
  const int lim = cdiv(CAUSAL ? min(p.Lk, p.kv_offset + x.r0 + kTileRows) : p.kv_limit, kTileRows);
  if constexpr (SPLIT) {
    // this split's tiles the tile can see (0 under the causal mask when the
    // split starts past its last row's limit)
    x.j0 = x.split * p.split_tiles;
    x.n0 = x.n1 = x.nu = max(0, min(lim, x.j0 + p.split_tiles) - x.j0);
  } else {
    x.j0 = 0;
    x.n0 = x.n1 = x.nu = lim;
  }
  return x;
}

template <bool CAUSAL, bool SPLIT, bool WINDOW>
__device__ __forceinline__ Unit decode_unit(const FwdParams& p, int u) {
  Unit x;
  if constexpr (SPLIT) {
    x.split = u % p.n_splits;
    u /= p.n_splits;
  } else {
    x.split = 0;
  }
  int pt = u % p.n_pairs;
  int t = u / p.n_pairs;
  int g = t % p.group;
  t /= p.group;
  x.hkv = t % p.Hkv;
  x.b = t / p.Hkv;
  x.hq = x.hkv * p.group + g;
  if (CAUSAL) pt = p.n_pairs - 1 - pt;
  x.r0 = pt * 2 * kTileRows;
  x.s0 = x.s1 = 0;
  if constexpr (WINDOW) {
    // key range of each query tile from its first and last real rows
    int a[2], e[2];
    for (int t = 0; t < 2; ++t) {
      const int first = min(x.r0 + t * kTileRows, p.Lq - 1);
      const int last = min(x.r0 + t * kTileRows + kTileRows - 1, p.Lq - 1);
      const int lo = p.win_left < 0 ? 0 : max(0, p.kv_offset + first - p.win_left);
      const int hi = p.win_right < 0 ? p.Lk : min(p.Lk, p.kv_offset + last + p.win_right + 1);
      a[t] = lo / kTileRows;
      e[t] = cdiv(hi, kTileRows);
    }
    x.j0 = a[0];  // a[0] <= a[1] and e[0] <= e[1]: tile 1's rows come later
    x.s0 = 0;
    x.s1 = a[1] - a[0];
    x.n0 = e[0] - a[0];
    x.n1 = e[1] - a[1];
    x.nu = e[1] - a[0];
    return x;
  }
  if (CAUSAL) {
    const int lim0 = cdiv(min(p.Lk, p.kv_offset + x.r0 + kTileRows), kTileRows);
    const int lim1 = cdiv(min(p.Lk, p.kv_offset + x.r0 + 2 * kTileRows), kTileRows);
    if constexpr (SPLIT) {
      // this split's tiles a tile can see; 0 when the split starts past its
      // last row's limit (its partial is then empty: O = 0, LSE = -inf)
      x.j0 = x.split * p.split_tiles;
      x.n0 = max(0, min(lim0, x.j0 + p.split_tiles) - x.j0);
      x.n1 = max(0, min(lim1, x.j0 + p.split_tiles) - x.j0);
    } else {
      x.n0 = lim0;
      x.n1 = lim1;
      x.j0 = 0;
    }
  } else if constexpr (SPLIT) {
    const int total = cdiv(p.kv_limit, kTileRows);
    x.j0 = x.split * p.split_tiles;
    x.n0 = x.n1 = min(total, x.j0 + p.split_tiles) - x.j0;  // >= 1: the host never makes an empty split
  } else {
    x.j0 = 0;
    x.n0 = x.n1 = cdiv(p.kv_limit, kTileRows);
  }
  x.nu = x.n1;
  return x;
}

// Bounded barrier wait. Fast path: one probe. Slow path: poll until the phase
// completes, another role has aborted, or the time limit passes (then record
// `bit`, raise the CTA's abort flag and return false).
__device__ __forceinline__ bool mbar_wait_slow(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                            unsigned int bit, unsigned long long timeout_ns) {
  const uint64_t t0 = global_timer_ns();
  // iteration cap as a second bound, should the timer not advance
  const unsigned long long max_iters = (timeout_ns >> 4) + (1ull << 20);
  for (unsigned long long it = 0;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (((it & 63u) == 63u && global_timer_ns() - t0 > timeout_ns) || it > max_iters) {
      atomicOr(&g_fault_bits, bit);
      *abort_flag = 1;
      return false;
    }
  }
}

__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                          unsigned int bit, unsigned long long timeout_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  return mbar_wait_slow(bar, parity, abort_flag, bit, timeout_ns);
}

// Abort path: wait a short, fixed time for a phase, ignoring the abort flag.
__device__ __forceinline__ void mbar_drain(uint32_t bar, uint32_t parity) {
  const uint64_t t0 = global_timer_ns();
  for (uint32_t it = 0; !mbar_try_wait(bar, parity); ++it) {
    if (global_timer_ns() - t0 > 200000000ull || it > (1u << 24)) return;  // ~200 ms
  }
}

// S[tmem] = Q K^T over head_dim D: D/16 MMAs of 128x128x16, fully unrolled (a
// single thread issues every MMA; a rolled loop leaves the tensor core idle).
// Q and K tiles are K-major with the 128-byte swizzle (TMA boxes of 64 elements
// x 128 rows): 16 elements = 32 bytes along K inside a chunk, then the next
// chunk. Descriptor address fields count 16-byte units.
// e4m3 Q K^T: D/32 MMAs of 128x128x32 (kind::f8f6f4), 32 bytes along K each,
// inside the single 128-byte swizzle chunk of a row.
template <int D>
__device__ __forceinline__ void issue_qk_f8(uint32_t d_tmem, uint32_t q_lo, uint32_t k_lo) {
  constexpr uint32_t idesc = mma_idesc_f16(false, 128, 128, false, false);
#pragma unroll
  for (int kk = 0; kk < D / 32; ++kk) {
    // 4 steps of 32 bytes per 128-byte chunk, chunks kTileRows * 128 bytes apart
    const uint32_t off = static_cast<uint32_t>(((kk >> 2) * kTileRows * 128 + (kk & 3) * 32) >> 4);
    mma_f8_ss_lo_flag(d_tmem, q_lo + off, k_lo + off, idesc, kk > 0 ? 1u : 0u);
  }
}

// e4m3 O += P V for half HALF of the 128 keys: A = P (shared memory, K-major),
// B = V^T (K-major): two MMAs of 128xDx32, 32 keys (bytes) each.
template <int D, int HALF>
__device__ __forceinline__ void issue_pv_half_f8(uint32_t d_tmem, uint32_t p_lo, uint32_t vt_lo,
                                                 uint32_t accumulate) {
  constexpr uint32_t idesc = mma_idesc_f16(false, 128, D, false, false);
#pragma unroll
  for (int kk = 2 * HALF; kk < 2 * HALF + 2; ++kk)
    mma_f8_ss_lo_flag(d_tmem, p_lo + 2 * kk, vt_lo + 2 * kk, idesc, kk == 0 ? accumulate : 1u);
}

template <int D, bool BF16>
__device__ __forceinline__ void issue_qk(uint32_t d_tmem, uint32_t q_lo, uint32_t k_lo) {
  constexpr uint32_t idesc = mma_idesc_f16(BF16, 128, 128, false, false);
  mma_f16_ss_lo<false>(d_tmem, q_lo, k_lo, idesc);
#pragma unroll
  for (int kk = 1; kk < D / 16; ++kk) {
    const uint32_t off = static_cast<uint32_t>(((kk >> 2) * Cfg<D>::kChunkBytes + (kk & 3) * 32) >> 4);
    mma_f16_ss_lo<true>(d_tmem, q_lo + off, k_lo + off, idesc);
  }
}

// O[tmem] (+)= P[tmem] V over 128 keys: 8 MMAs of 128xDx16, issued as two halves
// of 64 keys so the first half can start while the softmax still writes the
// second. P is packed 16-bit in tensor memory (two keys per column); V is
// MN-major (d contiguous): 8-key groups 1024 bytes apart (SBO), 64-column d
// chunks one chunk apart (LBO), so 16 keys advance the start address by 2048 B.
template <int D, bool BF16, int HALF>
__device__ __forceinline__ void issue_pv_half(uint32_t d_tmem, uint32_t p_tmem, uint32_t v_lo,
                                              uint32_t accumulate) {
  constexpr uint32_t idesc = mma_idesc_f16(BF16, 128, D, false, true);
  if constexpr (HALF == 0) {
    mma_f16_ts_lo_flag(d_tmem, p_tmem, v_lo, idesc, accumulate);
  } else {
    mma_f16_ts_lo<true>(d_tmem, p_tmem + 32, v_lo + 4 * (2048 >> 4), idesc);
  }
#pragma unroll
  for (int kk = HALF * 4 + 1; kk < HALF * 4 + 4; ++kk)
    mma_f16_ts_lo<true>(d_tmem, p_tmem + kk * 8, v_lo + kk * (2048 >> 4), idesc);
}

template <int D, bool BF16>
__device__ __forceinline__ void issue_pv(uint32_t d_tmem, uint32_t p_tmem, uint32_t v_lo,
                                         uint32_t accumulate) {
  issue_pv_half<D, BF16, 0>(d_tmem, p_tmem, v_lo, accumulate);
  issue_pv_half<D, BF16, 1>(d_tmem, p_tmem, v_lo, 1u);
}

template <int D, bool BF16, bool CAUSAL, bool SPLIT, bool WINDOW, int F8, bool PAIR = false>
__device__ __forceinline__ void load_role(const CUtensorMap* tm_q, const CUtensorMap* tm_k,
                                          const CUtensorMap* tm_v, const FwdParams& p,
                                          uint32_t sQ, uint32_t sKV, uint32_t bars,
                                          volatile int* abort_flag) {
  using C = Cfg<D, F8>;
  const uint64_t pol_q = l2_policy_evict_first();
  const uint64_t pol_kv = l2_policy_evict_last();
  int kv_it = 0, uit = 0;
  // abort drain: the ring index of the last load issued into each slot, and
  // the phase parity of the last load of each Q tile (-1: none issued)
  int slot_last[C::kStages];
#pragma unroll
  for (int i = 0; i < C::kStages; ++i) slot_last[i] = -1;
  int q_last[2] = {-1, -1};
  bool aborted = false;
  for (int u = cta_unit(0, p.n_units); u >= 0 && !aborted; u = cta_unit(++uit, p.n_units)) {
    Unit x;
    if constexpr (PAIR) x = decode_pair(p, u);
    else if constexpr (D == 256) x = decode_single<CAUSAL, SPLIT, WINDOW>(p, u);
    else x = decode_unit<CAUSAL, SPLIT, WINDOW>(p, u);
    // query tile t of the unit into its Q buffer, once the previous unit's
    // last Q K^T of that tile is done
    auto load_q = [&](int t) -> bool {
      const uint32_t bq = bars + 8 * (kBarQEmpty + t);
      if (!mbar_wait(bq, (uit & 1) ^ 1, abort_flag, kFaultLoadQEmpty, p.timeout_ns)) return false;
      const uint32_t bf = bars + 8 * (kBarQFull + t);
      mbar_arrive_expect_tx(bf, C::kTileBytes);
      // site 1: the Q tile's head, batch and first row lie inside q
      (void)ATTN_CHECK(x.hq >= 0 && x.hq < p.Hq && x.b >= 0 && x.b < p.B && x.r0 >= 0 &&
                           x.r0 + (PAIR ? 0 : t * kTileRows) < p.Lq + kTileRows,
                       1);
#pragma unroll
      for (int c = 0; c < C::kChunks; ++c)  // 128 bytes a chunk: 64 16-bit or 128 e4m3 elements
        tma_load_4d(sQ + t * C::kTileBytes + c * C::kChunkBytes, tm_q, bf, c * (F8 != 0 ? 128 : 64), x.hq,
                    x.r0 + (PAIR ? 0 : t * kTileRows), x.b, pol_q);  // pair split: both slots, the same rows
      q_last[t] = uit & 1;
      return true;
    };
    // one K or V tile into its ring slot (ring index kv_it + 2 jj + kv); pair
    // split: stream position jj holds KV tile pair_tile(jj)
    auto load_one = [&](int jj, int kv) -> bool {
      const int idx = kv_it + 2 * jj + kv;
      const int tile = PAIR ? pair_tile(x, jj) : jj;
      // site 2: the K / V tile starts inside the keys of its head and batch
      (void)ATTN_CHECK(x.hkv >= 0 && x.hkv < p.Hkv && tile >= 0 && (x.j0 + tile) * kTileRows < p.Lk, 2);
      const int slot = idx % C::kStages;
      const uint32_t be = bars + 8 * (kBarKvEmpty + slot);
      if (!mbar_wait(be, ((idx / C::kStages) & 1) ^ 1, abort_flag, kFaultLoadKvEmpty, p.timeout_ns))
        return false;
      const uint32_t bf = bars + 8 * (kBarKvFull + slot);
      mbar_arrive_expect_tx(bf, C::kTileBytes);
      if constexpr (F8 != 0) {
        // K: (d, head, key, batch); transposed V: (key, d, head, batch)
#pragma unroll
        for (int c = 0; c < C::kChunks; ++c) {  // V^T: 128 d-rows a chunk; K: 128 bytes a chunk
          if (kv)
            tma_load_4d(sKV + slot * C::kTileBytes + c * C::kChunkBytes, tm_v, bf, (x.j0 + jj) * kTileRows,
                        c * 128, x.hkv, x.b, pol_kv);
          else
            tma_load_4d(sKV + slot * C::kTileBytes + c * C::kChunkBytes, tm_k, bf, c * 128, x.hkv,
                        (x.j0 + jj) * kTileRows, x.b, pol_kv);
        }
      } else {
#pragma unroll
        for (int c = 0; c < C::kChunks; ++c)
          tma_load_4d(sKV + slot * C::kTileBytes + c * C::kChunkBytes, kv ? tm_v : tm_k, bf,
                      c * 64, x.hkv, (x.j0 + tile) * kTileRows, x.b, pol_kv);
      }
      slot_last[slot] = idx;
      return true;
    };
    // 16-bit, two query tiles: Q_0, then K_0, then Q_1. The first Q K^T needs
    // only the first two, and at the start of a launch they come from HBM
    // (1 % on the 1785-token DiT shape against loading both Q tiles first).
    // Tile 0 may then enter a unit while tile 1 is still finishing the
    // previous one; the softmax turn hand-back keeps their turns in order.
    // e4m3 loads both Q tiles first and has no hand-back (both measured
    // slower there); then tile 0 cannot start a unit before tile 1 has issued
    // its last Q K^T of the previous one, which leaves tile 1 far more time to
    // take its last turn than tile 0 needs to offer the next.
    constexpr bool kQ0K0Q1 = D != 256 && F8 == 0;
    bool ok = load_q(0);
    bool k0 = false;
    if constexpr (kQ0K0Q1) {
      if (ok && x.nu > 0) {
        ok = load_one(0, 0);
        k0 = true;
      }
      ok = ok && load_q(1);
    } else if constexpr (D != 256) {
      ok = ok && load_q(1);
    }
    if constexpr (D == 256) {
      // K one tile ahead of V (K_0, K_1, V_0, K_2, V_1, ...): K and V have
      // slots of their own, so K_{j+1} (its slot free once Q K_j^T is done)
      // no longer queues behind V_j (whose slot frees only when P_{j-1} V_{j-1}
      // is done), and Q K_{j+1}^T may run as soon as its S buffer is free.
      // Measured 1260 against 1189 TFLOPS on 8192 x 8192 x 16 heads.
      static_assert(D != 256 || C::kStages % 2 == 0, "K and V slots must not mix");
      if (ok && x.nu > 0) ok = load_one(0, 0);
      for (int j = 0; j < x.nu && ok; ++j) {
        if (j + 1 < x.nu) ok = load_one(j + 1, 0);
        ok = ok && load_one(j, 1);
      }
    } else {
      for (int j = 0; j < x.nu && ok; ++j)
        for (int kv = 0; kv < 2 && ok; ++kv)
          if (j != 0 || kv != 0 || !k0) ok = load_one(j, kv);
    }
    if (!ok) aborted = true;
    else kv_it += 2 * x.nu;
  }
  if (aborted) {
    // let the copies already issued land before the CTA exits: the newest load
    // of each ring slot (its full barrier completes that load's phase; every
    // older load of the slot completed before it could be issued) and of each
    // Q tile that was loaded at all
#pragma unroll 1
    for (int slot = 0; slot < C::kStages; ++slot)
      if (slot_last[slot] >= 0)
        mbar_drain(bars + 8 * (kBarKvFull + slot), (slot_last[slot] / C::kStages) & 1);
    for (int t = 0; t < 2; ++t)
      if (q_last[t] >= 0) mbar_drain(bars + 8 * (kBarQFull + t), q_last[t]);
  }
}

// One MMA issuer per query tile t (warps 9 and 10). A single issuing thread
// serialises both tiles: every tcgen05.mma holds its thread about as long as the
// tensor core takes to run it, so one thread cannot wait for one tile's P while
// issuing the other's GEMMs. With one thread per tile, the tensor core runs
// whichever tile has work. Both threads read the same K/V ring slots; each slot
// use is released by both (kv_empty takes two arrivals).
template <int D, bool BF16, bool CAUSAL, bool SPLIT, bool WINDOW, int F8, bool PAIR = false>
__device__ __forceinline__ void mma_role(const int t, const FwdParams& p, uint32_t tmem, uint32_t sQ,
                                         uint32_t sKV, uint32_t sP, uint32_t bars,
                                         volatile int* abort_flag) {
  using C = Cfg<D, F8>;
  // e4m3: P_t in shared memory (K-major, 128-byte swizzle)
  const uint32_t p_lo = smem_desc_lo(sP + t * C::kTileBytes, 16);
  auto bar = [&](int i) { return bars + 8 * i; };
  // low descriptor halves: Q and K tiles K-major (LBO unused, 16), V tiles MN-major (LBO = chunk)
  const uint32_t q_lo = smem_desc_lo(sQ + t * C::kTileBytes, 16);
  auto k_lo = [&](int idx) { return smem_desc_lo(sKV + (idx % C::kStages) * C::kTileBytes, 16); };
  auto v_lo = [&](int idx) {
    return smem_desc_lo(sKV + (idx % C::kStages) * C::kTileBytes, C::kChunkBytes);
  };
  // K/V tiles are written by TMA (async proxy) and read by the MMA (async proxy):
  // the barrier's transaction count orders them, no tcgen05 fence is needed
  auto kv_full = [&](int idx) {
    return mbar_wait(bar(kBarKvFull + idx % C::kStages), (idx / C::kStages) & 1, abort_flag,
                     kFaultMmaKvFull, p.timeout_ns);
  };
  const uint32_t s_t = tmem + C::col_s(t), o_t = tmem + C::col_o(t);
  int kv_it = 0, uit = 0, pcnt = 0;
  bool ok = true;
  for (int u = cta_unit(0, p.n_units); u >= 0 && ok; u = cta_unit(++uit, p.n_units)) {
    Unit x;
    if constexpr (PAIR) x = decode_pair(p, u);
    else x = decode_unit<CAUSAL, SPLIT, WINDOW>(p, u);
    const int n = t ? x.n1 : x.n0;  // KV tiles this query tile uses
    const int s = WINDOW ? (t ? x.s1 : x.s0) : 0;  // ... starting this many tiles into the stream
    ok = mbar_wait(bar(kBarQFull + t), uit & 1, abort_flag, kFaultMmaQFull, p.timeout_ns);
    if ((CAUSAL && SPLIT || PAIR) && n == 0) {
      // no key of this split is visible to the tile (pair split: slot 1 of a
      // one-tile range): release Q and pass the unit's tiles through. O is
      // neither written nor signalled: the softmax decodes the same empty tile
      // and writes the empty partial (pair split: an empty row state) itself (an
      // O-full commit here, with no hand-shake from the softmax, could complete
      // the barrier's phase twice before the softmax looked at it)
      if (!ok) break;
      mma_commit(bar(kBarQEmpty + t));
      for (int j = 0; j < x.nu && ok; ++j) {
        for (int kv = 0; kv < 2 && ok; ++kv) {
          const int idx = kv_it + 2 * j + kv;
          if (!kv_full(idx)) { ok = false; break; }
          mbar_arrive(bar(kBarKvEmpty + idx % C::kStages));
        }
      }
      kv_it += 2 * x.nu;
      continue;
    }
    if constexpr (WINDOW) {
      // tiles before this query tile's range pass through the ring; release
      // this thread's share once each has landed
      for (int j = 0; j < s && ok; ++j) {
        for (int kv = 0; kv < 2 && ok; ++kv) {
          const int idx = kv_it + 2 * j + kv;
          if (!kv_full(idx)) { ok = false; break; }
          mbar_arrive(bar(kBarKvEmpty + idx % C::kStages));
        }
      }
    }
    // ring index of this query tile's j-th K (pair split: its stream position)
    auto kring = [&](int j) { return kv_it + 2 * (PAIR ? pair_pos(x, t, j) : s + j); };
    // pair split: release the other slot's stream positions [a, b) (K and V)
    auto pass_positions = [&](int a, int b) {
      for (int q = 2 * a; q < 2 * b && ok; ++q) {
        const int idx = kv_it + q;
        if (!kv_full(idx)) { ok = false; break; }
        mbar_arrive(bar(kBarKvEmpty + idx % C::kStages));
      }
    };
    if constexpr (PAIR) pass_positions(0, pair_pos(x, t, 0));
    const int kb = kring(0);  // ring index of this query tile's first K
    ok = ok && kv_full(kb);
    if (!ok) break;
    // S_t(0) = Q_t K_0^T
    if constexpr (F8 != 0) issue_qk_f8<D>(s_t, q_lo, k_lo(kb));
    else issue_qk<D, BF16>(s_t, q_lo, k_lo(kb));
    mma_commit(bar(kBarSFull + t));
    mma_commit(bar(kBarKvEmpty + kb % C::kStages));
    if (n == 1) mma_commit(bar(kBarQEmpty + t));
    for (int j = 0; j < n; ++j) {
      const int vidx = kring(j) + 1;                  // V_j
      const int knext = j + 1 < n ? kring(j + 1) : 0;  // K_{j+1}
      // O_t += P_t V_j: the first 64 keys as soon as their half of P is in
      // tensor memory, the rest once all of P is
      if (!kv_full(vidx) ||
          !mbar_wait(bar(kBarPHalf + t), pcnt & 1, abort_flag, kFaultMmaPFull, p.timeout_ns)) {
        ok = false;
        break;
      }
      tc_fence_after_sync();
      if constexpr (F8 != 0) issue_pv_half_f8<D, 0>(o_t, p_lo, k_lo(vidx), j > 0 ? 1u : 0u);
      else issue_pv_half<D, BF16, 0>(o_t, s_t, v_lo(vidx), j > 0 ? 1u : 0u);
      if (!mbar_wait(bar(kBarPFull + t), pcnt & 1, abort_flag, kFaultMmaPFull, p.timeout_ns)) {
        ok = false;
        break;
      }
      ++pcnt;
      tc_fence_after_sync();
      if constexpr (F8 != 0) issue_pv_half_f8<D, 1>(o_t, p_lo, k_lo(vidx), 1u);
      else issue_pv_half<D, BF16, 1>(o_t, s_t, v_lo(vidx), 1u);
      mma_commit(bar(kBarKvEmpty + vidx % C::kStages));
      if (j == n - 1) {
        mma_commit(bar(kBarOFull + t));
      } else {
        if constexpr (PAIR) {
          pass_positions(pair_pos(x, t, j) + 1, pair_pos(x, t, j + 1));
          if (!ok) break;
        }
        if (!kv_full(knext)) { ok = false; break; }
        if constexpr (F8 != 0) issue_qk_f8<D>(s_t, q_lo, k_lo(knext));
        else issue_qk<D, BF16>(s_t, q_lo, k_lo(knext));
        mma_commit(bar(kBarSFull + t));
        mma_commit(bar(kBarKvEmpty + knext % C::kStages));
        if (j + 1 == n - 1) mma_commit(bar(kBarQEmpty + t));
      }
    }
    // causal / window: tiles after this query tile's range still pass through
    // the ring; release this thread's share once each has landed (waiting for
    // the landing keeps the arrival in the slot's current phase)
    if constexpr (PAIR) pass_positions(pair_pos(x, t, n - 1) + 1, x.nu);
    for (int j = PAIR ? x.nu : s + n; j < x.nu && ok; ++j) {
      for (int kv = 0; kv < 2 && ok; ++kv) {
        const int idx = kv_it + 2 * j + kv;
        if (!kv_full(idx)) { ok = false; break; }
        mbar_arrive(bar(kBarKvEmpty + idx % C::kStages));
      }
    }
    kv_it += 2 * x.nu;
  }
  if (!ok) {
    // every MMA this thread issued must finish before tensor memory is freed
    mma_commit(bar(kBarDrain + t));
    mbar_drain(bar(kBarDrain + t), 0);
  }
}

// P = exp2(s * sl2 - ref) for one row's 128 scores, packed to 16 bits into
// the first 64 columns of S in two halves of 64 keys, each handed to the MMA
// issuer (one arrival per warp) as soon as it is in tensor memory; the turn
// goes to the other softmax warpgroup once the exponentials are done. The
// scale-and-shift and the row sums run as packed f32x2 FMA / add (one
// instruction per two scores: scalar FP32 arithmetic issues at half the
// packed rate on B200; +2-3 % measured on the 1785- and 20480-token
// workloads). MASKED: keys c >= lim are zeroed after the exponential (their
// -inf scores times a zero scale, or -inf + inf when the row has no visible
// key yet, would give NaN).
// e4m3 variant of exp_tile: P = exp2(s * sl2 - ref) rounded to e4m3 (four keys
// per 32-bit word) into this row of the P_t buffer in shared memory (128 bytes
// per row, K-major with the 128-byte swizzle: 16-byte unit u of row r at
// r * 128 + ((u ^ (r % 8)) * 16)), in two halves of 64 keys, each handed to the
// MMA issuer once it is visible to the tensor core (proxy fence). The row sum
// uses the unrounded P.
template <bool MASKED>
__device__ __forceinline__ void exp_tile_f8(const uint32_t (&r)[128], float sl2, float nref, int lim,
                                            int lim_lo, float (&sum)[4], uint32_t prow, int r_in,
                                            uint32_t bar_half, uint32_t bar_full, uint32_t bar_turn_other,
                                            bool hand_over, int lane) {
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    uint32_t w[16];
#pragma unroll
    for (int cc = 0; cc < 16; ++cc) {
      float pv[4];
#pragma unroll
      for (int pr = 0; pr < 2; ++pr) {
        const int c = 64 * h + 4 * cc + 2 * pr;
        float p0, p1;
        if (((2 * cc + pr) & 7) >= 8 - kF8PolyPairsPer8) {
          f2_unpack(exp2_poly_x2(f2_pack(fmaf(__uint_as_float(r[c]), sl2, nref),
                                         fmaf(__uint_as_float(r[c + 1]), sl2, nref))), p0, p1);
        } else {
          p0 = ex2_approx(fmaf(__uint_as_float(r[c]), sl2, nref));
          p1 = ex2_approx(fmaf(__uint_as_float(r[c + 1]), sl2, nref));
        }
        if (MASKED) {
          p0 = (c < lim && c >= lim_lo) ? p0 : 0.f;
          p1 = (c + 1 < lim && c + 1 >= lim_lo) ? p1 : 0.f;
        }
        sum[2 * pr] += p0;
        sum[2 * pr + 1] += p1;
        pv[2 * pr] = p0;
        pv[2 * pr + 1] = p1;
      }
      w[cc] = pack_e4m3x2(pv[0], pv[1]) | (pack_e4m3x2(pv[2], pv[3]) << 16);
    }
    if (h == 1 && hand_over) {  // exponentials done: hand over the turn
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_turn_other);
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const uint32_t unit = static_cast<uint32_t>((4 * h + u) ^ (r_in & 7));
      asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(prow + unit * 16), "r"(w[4 * u]),
                   "r"(w[4 * u + 1]), "r"(w[4 * u + 2]), "r"(w[4 * u + 3])
                   : "memory");
    }
    fence_proxy_async_smem();
    tc_fence_before_sync();
    __syncwarp();
    if (lane == 0) mbar_arrive(h == 0 ? bar_half : bar_full);
  }
}

// Four key scales of one 128-key tile (keys key .. key + 3 of a per-head
// scale row; keys >= Lk read as 0: they are masked anyway).
__device__ __forceinline__ float4 load_key_scales(const float* row, int key, int Lk) {
  if (key + 3 < Lk) return __ldg(reinterpret_cast<const float4*>(row + key));
  float4 v;
  v.x = key < Lk ? __ldg(row + key) : 0.f;
  v.y = key + 1 < Lk ? __ldg(row + key + 1) : 0.f;
  v.z = key + 2 < Lk ? __ldg(row + key + 2) : 0.f;
  v.w = 0.f;
  return v;
}

template <bool BF16, bool MASKED>
__device__ __forceinline__ void exp_tile(const uint32_t (&r)[128], float sl2, float nref, int lim, int lim_lo,
                                         float (&sum)[4], uint32_t tS, uint32_t bar_half,
                                         uint32_t bar_full, uint32_t bar_turn_other, bool hand_over,
                                         int lane) {
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    uint32_t pk[32];
    uint64_t acc0 = f2_pack(sum[0], sum[1]), acc1 = f2_pack(sum[2], sum[3]);
    const uint64_t s2 = f2_pack(sl2, sl2), n2 = f2_pack(nref, nref);
#pragma unroll
    for (int cc = 0; cc < 32; ++cc) {
      const int c = 64 * h + 2 * cc;
      const uint64_t x2 = f2_fma(f2_pack_bits(r[c], r[c + 1]), s2, n2);
      float p0, p1;
      if ((cc & 7) >= 8 - kPolyPairsPer8) {
        f2_unpack(exp2_poly_x2(x2), p0, p1);
      } else {
        float a, b;
        f2_unpack(x2, a, b);
        p0 = ex2_approx(a);
        p1 = ex2_approx(b);
      }
      if (MASKED) {
        p0 = (c < lim && c >= lim_lo) ? p0 : 0.f;
        p1 = (c + 1 < lim && c + 1 >= lim_lo) ? p1 : 0.f;
      }
      if (cc & 1) acc1 = f2_add(acc1, f2_pack(p0, p1));
      else acc0 = f2_add(acc0, f2_pack(p0, p1));
      pk[cc] = pack2<BF16>(p0, p1);
    }
    f2_unpack(acc0, sum[0], sum[1]);
    f2_unpack(acc1, sum[2], sum[3]);
    if (h == 1 && hand_over) {  // exponentials done: hand over the turn
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_turn_other);
    }
    tmem_st_32x32b_x32(tS + 32 * h, pk);
    tmem_wait_st();
    tc_fence_before_sync();
    __syncwarp();
    if (lane == 0) mbar_arrive(h == 0 ? bar_half : bar_full);
  }
}

// Warp 11 (one thread): writes each finished O tile from the shared staging
// buffer to global memory with a TMA store (rows past Lq are clipped by the
// tensor map), then hands the buffer to the other query tile. Order per unit:
// tile 0, then tile 1, the same order the softmax warpgroups fill it in.
template <int D, bool BF16, bool CAUSAL, bool SPLIT, bool WINDOW, int F8, bool PAIR = false>
__device__ __forceinline__ void store_role(const CUtensorMap* tm_o, const FwdParams& p, uint32_t sStg,
                                           uint32_t bars, volatile int* abort_flag) {
  using C = Cfg<D, F8>;
  int scnt = 0;
  bool ok = true;
  int k = 0;
  for (int u = cta_unit(0, p.n_units); u >= 0 && ok; u = cta_unit(++k, p.n_units)) {
    Unit x;
    if constexpr (PAIR) x = decode_pair(p, u);
    else x = decode_unit<CAUSAL, SPLIT, WINDOW>(p, u);
    for (int t = 0; t < (PAIR ? 1 : 2) && ok; ++t) {  // pair split: one merged tile per unit
      ok = mbar_wait(bars + 8 * kBarStgFull, scnt & 1, abort_flag, kFaultStore, p.timeout_ns);
      if (!ok) break;
      ++scnt;
      const int dt = p.d > 0 ? p.d : D;  // a chunk wholly past the tensor's head dim is not stored
      // site 3: a TMA store never starts at a negative coordinate
      const bool st_ok = ATTN_CHECK(x.r0 >= 0 && x.hq >= 0 && x.hq < p.Hq && x.b >= 0 && x.b < p.B, 3);
#pragma unroll
      for (int c = 0; c < C::kOChunks; ++c)
        if (c * 64 < dt && st_ok)
          tma_store_4d(tm_o, sStg + c * C::kChunkBytes, c * 64, x.hq, x.r0 + t * kTileRows, x.b);
      bulk_commit_group();
      bulk_wait_group_read0();
      mbar_arrive(bars + 8 * (kBarStgFree + (PAIR ? 0 : 1 - t)));
    }
  }
  bulk_wait_group0();  // every store complete before the CTA exits
}

template <int D, bool BF16, bool CAUSAL, bool SPLIT, bool WINDOW, int F8, bool PAIR = false>
__device__ __forceinline__ void softmax_role(const int t, const FwdParams& p, uint32_t tmem,
                                             uint32_t bars, uint32_t sstg, uint32_t sP, uint32_t sSk,
                                             uint32_t sMl, volatile int* abort_flag) {
  using C = Cfg<D, F8>;
  const uint32_t prow = sP + t * C::kTileBytes + (threadIdx.x % kTileRows) * 128;  // e4m3 P row
  // per-token scales: this warp's copy of the current KV tile's 128 key scales
  const uint32_t skw = sSk + (threadIdx.x / 32) * 512;
  const int warp = threadIdx.x / 32;
  const int r_in = threadIdx.x % kTileRows;                      // row in tile = TMEM lane
  const uint32_t lane_bits = static_cast<uint32_t>((warp % 4) * 32) << 16;
  const uint32_t tS = tmem + lane_bits + C::col_s(t);
  const uint32_t tO = tmem + lane_bits + C::col_o(t);
  const uint32_t bar_s = bars + 8 * (kBarSFull + t);
  const uint32_t bar_p = bars + 8 * (kBarPFull + t);
  const uint32_t bar_ph = bars + 8 * (kBarPHalf + t);
  const uint32_t bar_turn_mine = bars + 8 * (kBarTurn + t);
  const uint32_t bar_turn_other = bars + 8 * (kBarTurn + (1 - t));
  const uint32_t bar_stg_full = bars + 8 * kBarStgFull;
  const uint32_t bar_stg_free = bars + 8 * (kBarStgFree + t);
  const uint32_t stg = sstg;
  int tcnt = 0;
  bool turn_back = false;  // tile 0: tile 1 owes the turn back from an earlier unit
  const int lane = threadIdx.x % 32;
  const uint32_t bar_o = bars + 8 * (kBarOFull + t);
  const float sl2 = p.sl2;
  int scnt = 0, ocnt = 0;
  int o1cnt = 0;  // pair split: units whose slot 1 had KV tiles (phases of slot 1's O-full barrier)
  // (WINDOW || PAIR): per-slot KV ranges, tile 0 may have more steps than tile 1
  constexpr bool kRanges = WINDOW || PAIR;
  // the turn hand-back at the end of a unit (16-bit; e4m3 relies on the
  // loader's order, see load_role)
  constexpr bool kHandBack = F8 == 0;

  int k = 0;
  for (int u = cta_unit(0, p.n_units); u >= 0; u = cta_unit(++k, p.n_units)) {
    Unit x;
    if constexpr (PAIR) x = decode_pair(p, u);
    else x = decode_unit<CAUSAL, SPLIT, WINDOW>(p, u);
    const int n = t ? x.n1 : x.n0;
    const int s = kRanges ? (t ? x.s1 : x.s0) : 0;  // first KV tile of this query tile, relative to x.j0
    const int row = x.r0 + (PAIR ? 0 : t * kTileRows) + r_in;  // pair split: both slots, the same rows
    if constexpr (PAIR) {
      // slot 1 reuses its O and row-state buffers only once slot 0 has merged the previous unit
      if (t == 1 && k > 0) {
        const bool okm = mbar_wait(bars + 8 * kBarMerged, (k - 1) & 1, abort_flag, kFaultSoftmaxOFull,
                                   p.timeout_ns);
        if (!__all_sync(0xffffffffu, okm)) return;
      }
    }
    // visible keys of this row: [row_lo, row_lim)
    int row_lim = CAUSAL ? min(p.Lk, p.kv_offset + row + 1) : p.kv_limit;
    int row_lo = 0;
    if constexpr (WINDOW) {
      const int pos = p.kv_offset + row;
      row_lo = p.win_left < 0 ? 0 : max(0, pos - p.win_left);
      row_lim = p.win_right < 0 ? p.Lk : min(p.Lk, pos + p.win_right + 1);
    }
    // the unit ends with tile 0 handing the turn to tile 1 (tile 0 has steps and
    // no more of them than tile 1): tile 1 then hands it back after its step
    // n0 - 1, and tile 0 waits for that before its next unit's first step
    const bool ret = kHandBack && x.n0 >= 1 && x.n0 <= x.n1;
    float ref = -INFINITY;  // scaled (log2) max the exponentials are taken against
    float l = 0.f;          // running row sum of exp2(s * sl2 - ref)
    // per-token scales: the row's Q scale joins the log2 factor; each lane
    // fetches 4 of the next KV tile's key scales one tile ahead
    float sl2r = sl2;
    const float* skrow = nullptr;
    float4 skv = make_float4(0.f, 0.f, 0.f, 0.f);
    if constexpr (F8 == 2) {
      const size_t qs = (static_cast<size_t>(x.b) * p.Hq + x.hq) * p.sq_pitch + row;
      // site 6: the row's and the head's scales lie inside [B, H, pitch]
      const bool sok = ATTN_CHECK(x.b < p.B && x.hq < p.Hq && x.hkv < p.Hkv && p.Lq <= p.sq_pitch &&
                                      p.Lk <= p.sk_pitch,
                                  6);
      sl2r = sl2 * (row < p.Lq && sok ? __ldg(p.sq + qs) : 1.f);
      skrow = p.sk + (static_cast<size_t>(x.b) * p.Hkv + x.hkv) * p.sk_pitch;
      skv = load_key_scales(skrow, (x.j0 + s) * kTileRows + 4 * lane, p.Lk);
    }

    for (int j = 0; j < n; ++j) {
      if constexpr (F8 == 2) {
        __syncwarp();  // every lane is done with the previous tile's scales
        st_shared_v4f(skw + 16 * lane, skv);
        __syncwarp();
        if (j + 1 < n) skv = load_key_scales(skrow, (x.j0 + s + j + 1) * kTileRows + 4 * lane, p.Lk);
      }
      bool ok = mbar_wait(bar_s, scnt & 1, abort_flag, kFaultSoftmaxSFull, p.timeout_ns);
      if (!__all_sync(0xffffffffu, ok)) return;
      ++scnt;
      tc_fence_after_sync();

      uint32_t r[128];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld_32x32b_x32(tS + 32 * c, r + 32 * c);
      tmem_wait_ld_x128(r);

      if constexpr (F8 == 2) {
        // raw code product times the key's scale (before masking: an invisible
        // key's -inf must not meet a scale)
#pragma unroll
        for (int c = 0; c < 128; c += 4) {
          const float4 k4 = ld_shared_v4f(skw + 4 * c);
#if F8_PACKED_KEY_SCALE
          float a0, a1, a2, a3;
          f2_unpack(f2_mul(f2_pack_bits(r[c], r[c + 1]), f2_pack(k4.x, k4.y)), a0, a1);
          f2_unpack(f2_mul(f2_pack_bits(r[c + 2], r[c + 3]), f2_pack(k4.z, k4.w)), a2, a3);
          r[c] = __float_as_uint(a0);
          r[c + 1] = __float_as_uint(a1);
          r[c + 2] = __float_as_uint(a2);
          r[c + 3] = __float_as_uint(a3);
#else
          r[c] = __float_as_uint(__uint_as_float(r[c]) * k4.x);
          r[c + 1] = __float_as_uint(__uint_as_float(r[c + 1]) * k4.y);
          r[c + 2] = __float_as_uint(__uint_as_float(r[c + 2]) * k4.z);
          r[c + 3] = __float_as_uint(__uint_as_float(r[c + 3]) * k4.w);
#endif
        }
      }
      const int key0 = (x.j0 + s + j) * kTileRows;  // first key of this tile
      const int lim = row_lim - key0;                // keys c < lim of this tile are visible ...
      const int lim_lo = WINDOW ? row_lo - key0 : 0;  // ... and c >= lim_lo
      const bool partial = lim < kTileRows || lim_lo > 0;
      if (partial) {
#pragma unroll
        for (int c = 0; c < 128; ++c)
          if (c >= lim || c < lim_lo) r[c] = __float_as_uint(-INFINITY);
      }
      // row max: a three-input max tree (depth 5) over the 128 scores
      float m_tile;
      {
        float a[43];
#pragma unroll
        for (int i = 0; i < 42; ++i)
          a[i] = fmax3(__uint_as_float(r[3 * i]), __uint_as_float(r[3 * i + 1]), __uint_as_float(r[3 * i + 2]));
        a[42] = fmaxf(__uint_as_float(r[126]), __uint_as_float(r[127]));
        float b[15];
#pragma unroll
        for (int i = 0; i < 14; ++i) b[i] = fmax3(a[3 * i], a[3 * i + 1], a[3 * i + 2]);
        b[14] = a[42];
        float c5[5];
#pragma unroll
        for (int i = 0; i < 5; ++i) c5[i] = fmax3(b[3 * i], b[3 * i + 1], b[3 * i + 2]);
        m_tile = fmaxf(fmax3(c5[0], c5[1], c5[2]), fmaxf(c5[3], c5[4]));
      }
      const float m_scaled = (m_tile == -INFINITY) ? -INFINITY : m_tile * sl2r;

      // lazy rescale: move the reference only when the max grew by > tau; after
      // the first tiles of a row this almost never fires, so the warp takes the
      // branch only when one of its rows needs it
      const bool rescale = m_scaled > ref + kRescaleTau;
      if (__any_sync(0xffffffffu, rescale)) {
        float alpha = 1.f;
        if (rescale) {
          alpha = ex2_approx(ref - m_scaled);
          ref = m_scaled;
          l *= alpha;
        }
        if (j > 0) {
          const uint64_t a2 = f2_pack(alpha, alpha);
#pragma unroll 1
          for (int c = 0; c < D / 32; ++c) {
            uint32_t ov[32];
            tmem_ld_32x32b_x32(tO + 32 * c, ov);
            tmem_wait_ld_x32(ov);
#pragma unroll
            for (int e = 0; e < 32; e += 2) {
              float lo, hi;
              f2_unpack(f2_mul(f2_pack_bits(ov[e], ov[e + 1]), a2), lo, hi);
              ov[e] = __float_as_uint(lo);
              ov[e + 1] = __float_as_uint(hi);
            }
            tmem_st_32x32b_x32(tO + 32 * c, ov);
          }
          tmem_wait_st();
        }
      }

      // Ping-pong: the two softmax warpgroups take turns for their exponentials
      // (tile 0 of KV tile j, then tile 1 of j, then tile 0 of j + 1, ...), so
      // the MUFU serves one of them at a time and each tile's GEMMs run on the
      // tensor core while the other tile computes. Step j of tile 0 hands over
      // if tile 1 has a step j; step j of tile 1 hands over if tile 0 has a
      // step j + 1, and at the end of a unit that tile 0 ends by handing over
      // (`ret`), tile 1's step n0 - 1 hands the turn back; each waits exactly
      // for the hand-overs it is owed (tile 0's first step of a unit for the
      // hand-back of an earlier one). So the hand-overs on each barrier
      // alternate with its waits across units too, and no barrier can complete
      // a phase twice before its waiter has seen the first (n0 > n1 can happen
      // with a window: tile 0 then ends the unit by receiving the turn).
      bool wait_turn = kRanges ? (t == 0 ? (j >= 1 && j - 1 < x.n1) : j < x.n0)
                               : (t == 0 ? j >= 1 : j < x.n0);  // n0 <= n1 without ranges
      if (kHandBack && t == 0 && j == 0) wait_turn = turn_back;
      if (wait_turn) {
        bool ok_turn = mbar_wait(bar_turn_mine, tcnt & 1, abort_flag, kFaultSoftmaxTurn, p.timeout_ns);
        if (!__all_sync(0xffffffffu, ok_turn)) return;
        ++tcnt;
      }
      if (kHandBack && t == 0 && j == 0) turn_back = false;

      const float nref = -ref;
      const bool hand_over = (kRanges ? (t == 0 ? j < x.n1 : j + 1 < x.n0) : (t == 0 || j + 1 < x.n0)) ||
                             (kHandBack && t == 1 && ret && j == x.n0 - 1);
      float sum[4] = {0.f, 0.f, 0.f, 0.f};
      // the masked variant is a separate instantiation so full tiles carry no
      // per-score compare/select. exp_tile holds warp-collective instructions
      // (tcgen05.st, __syncwarp), so the choice must be the same for the whole
      // warp: rows of one warp can differ (causal), and a lane whose keys are
      // all visible is unaffected by the masked variant.
      if constexpr (F8 != 0) {
        if (__any_sync(0xffffffffu, partial)) {
          exp_tile_f8<true>(r, sl2r, nref, lim, lim_lo, sum, prow, r_in, bar_ph, bar_p, bar_turn_other,
                            hand_over, lane);
        } else {
          exp_tile_f8<false>(r, sl2r, nref, lim, lim_lo, sum, prow, r_in, bar_ph, bar_p, bar_turn_other,
                             hand_over, lane);
        }
      } else if (__any_sync(0xffffffffu, partial)) {
        exp_tile<BF16, true>(r, sl2, nref, lim, lim_lo, sum, tS, bar_ph, bar_p, bar_turn_other, hand_over,
                             lane);
      } else {
        exp_tile<BF16, false>(r, sl2, nref, lim, lim_lo, sum, tS, bar_ph, bar_p, bar_turn_other, hand_over,
                              lane);
      }
      l += (sum[0] + sum[1]) + (sum[2] + sum[3]);
    }
    if (kHandBack && t == 0 && ret) turn_back = true;

    if constexpr (SPLIT) {
      // key split: float32 O / l of this split's keys, each thread its own
      // row (d contiguous floats), straight from registers; LSE of the split
      if (CAUSAL && n == 0) {
        // the tile sees no key of this split (the MMA issuer left O alone)
        const int row_e = x.r0 + t * kTileRows + r_in;
        // site 5: the partial's row lies inside [n_splits, B, Hq, Lq]
        if (row_e < p.Lq && ATTN_CHECK(x.split < p.n_splits && x.b < p.B && x.hq < p.Hq, 5)) {
          const size_t prow = ((static_cast<size_t>(x.split) * p.B + x.b) * p.Hq + x.hq) * p.Lq + row_e;
          float* dst = p.o_part + prow * D;
#pragma unroll 1
          for (int c = 0; c < D; c += 4) *reinterpret_cast<float4*>(dst + c) = make_float4(0.f, 0.f, 0.f, 0.f);
          p.lse_part[prow] = -INFINITY;
        }
        continue;
      }
      bool ok = mbar_wait(bar_o, ocnt & 1, abort_flag, kFaultSoftmaxOFull, p.timeout_ns);
      if (!__all_sync(0xffffffffu, ok)) return;
      ++ocnt;
      tc_fence_after_sync();
      // a row that sees no key of this split (causal) leaves O = 0, LSE = -inf
      const bool empty = !(l > 0.f);
      const float inv_l = empty ? 0.f : 1.f / l;
      const bool in_range = row < p.Lq && ATTN_CHECK(x.split < p.n_splits && x.b < p.B && x.hq < p.Hq, 5);
      const size_t prow = ((static_cast<size_t>(x.split) * p.B + x.b) * p.Hq + x.hq) * p.Lq + row;
      float* dst = p.o_part + prow * D;
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        uint32_t ov[32];
        tmem_ld_32x32b_x32(tO + 32 * c, ov);
        tmem_wait_ld_x32(ov);
        if (in_range) {
#pragma unroll
          for (int e = 0; e < 32; e += 4)
            *reinterpret_cast<float4*>(dst + 32 * c + e) =
                make_float4(__uint_as_float(ov[e]) * inv_l, __uint_as_float(ov[e + 1]) * inv_l,
                            __uint_as_float(ov[e + 2]) * inv_l, __uint_as_float(ov[e + 3]) * inv_l);
        }
      }
      if (in_range) p.lse_part[prow] = empty ? -INFINITY : (ref + log2f(l)) * kLn2;
      // every TMEM read of O_t is complete (wait::ld) before the next unit's
      // P V overwrites it: that MMA waits for this warpgroup's next P
      continue;
    }

    // pair split: slot 1 hands its row state to slot 0, which merges the two
    // partial results (each relative to its own reference):
    // O = (2^(ref0 - m) O_0 + 2^(ref1 - m) O_1) / (2^(ref0 - m) l_0 + 2^(ref1 - m) l_1),
    // m = max(ref0, ref1); slot 1's O_1 is read from tensor memory (same lanes)
    float a0 = 1.f, a1 = 0.f;  // the two slots' weights in the merge (pair split, slot 0)
    if constexpr (PAIR) {
      const uint32_t ml = sMl + r_in * 8;
      if (t == 1) {
        // a slot with no KV tile (one-tile range) leaves ref = -inf, l = 0: weight 0
        asm volatile("st.shared.v2.f32 [%0], {%1, %2};" ::"r"(ml), "f"(ref), "f"(l) : "memory");
        __syncwarp();
        if (lane == 0) mbar_arrive(bars + 8 * kBarMerge1);
        continue;
      }
      bool okm = mbar_wait(bars + 8 * kBarMerge1, k & 1, abort_flag, kFaultSoftmaxOFull, p.timeout_ns);
      if (x.n1 > 0)
        okm = okm && mbar_wait(bars + 8 * (kBarOFull + 1), o1cnt & 1, abort_flag, kFaultSoftmaxOFull,
                               p.timeout_ns);
      if (!__all_sync(0xffffffffu, okm)) return;
      float ref1, l1;
      asm volatile("ld.shared.v2.f32 {%0, %1}, [%2];" : "=f"(ref1), "=f"(l1) : "r"(ml) : "memory");
      const float m = fmaxf(ref, ref1);  // slot 0 always sees key 0: ref is finite
      a0 = ex2_approx(ref - m);
      a1 = x.n1 > 0 ? ex2_approx(ref1 - m) : 0.f;  // ex2(-inf) = 0 for rows slot 1 did not reach
      l = a0 * l + a1 * l1;
      ref = m;
    }

    // epilogue: O / l to 16 bits into the shared staging tile (128-byte
    // swizzle, the layout of the TMA box), handed to the store warp; LSE.
    // The staging buffer alternates between the two query tiles: tile t fills
    // it once the store warp has read out the other tile's previous O.
    bool ok = mbar_wait(bar_o, ocnt & 1, abort_flag, kFaultSoftmaxOFull, p.timeout_ns) &&
              mbar_wait(bar_stg_free, (ocnt & 1) ^ (t == 0 ? 1 : 0), abort_flag, kFaultStore,
                        p.timeout_ns);
    if (!__all_sync(0xffffffffu, ok)) return;
    ++ocnt;
    tc_fence_after_sync();
    const float inv_l = 1.f / l;
    const bool in_range = row < p.Lq;
    const uint32_t tO1 = tmem + lane_bits + C::col_o(1);  // pair split: slot 1's O
#pragma unroll 1
    for (int c = 0; c < D / 32; ++c) {
      uint32_t ov[32];
      tmem_ld_32x32b_x32(tO + 32 * c, ov);
      tmem_wait_ld_x32(ov);
      if constexpr (F8 == 2) {
        // site 7: V's per-channel scales of this head lie inside [B, Hkv, d]
        if (p.sv != nullptr && 32 * c < p.d && ATTN_CHECK(x.b < p.B && x.hkv < p.Hkv && 32 * c + 32 <= p.d, 7)) {
          const float4* sv4 =
              reinterpret_cast<const float4*>(p.sv + (static_cast<size_t>(x.b) * p.Hkv + x.hkv) * p.d + 32 * c);
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const float4 f = __ldg(sv4 + e);
            ov[4 * e] = __float_as_uint(__uint_as_float(ov[4 * e]) * f.x);
            ov[4 * e + 1] = __float_as_uint(__uint_as_float(ov[4 * e + 1]) * f.y);
            ov[4 * e + 2] = __float_as_uint(__uint_as_float(ov[4 * e + 2]) * f.z);
            ov[4 * e + 3] = __float_as_uint(__uint_as_float(ov[4 * e + 3]) * f.w);
          }
        }
      }
      if constexpr (PAIR) {
        if (x.n1 > 0) {  // add slot 1's partial, weighted
          uint32_t o1[32];
          tmem_ld_32x32b_x32(tO1 + 32 * c, o1);
          tmem_wait_ld_x32(o1);
#pragma unroll
          for (int e = 0; e < 32; ++e)
            ov[e] = __float_as_uint(fmaf(__uint_as_float(o1[e]), a1, __uint_as_float(ov[e]) * a0));
        }
      }
      uint32_t pk[16];
#pragma unroll
      for (int e = 0; e < 16; ++e)
        pk[e] = pack2<BF16>(__uint_as_float(ov[2 * e]) * inv_l, __uint_as_float(ov[2 * e + 1]) * inv_l);
      // 32 columns = 4 units of 16 bytes in the 64-column box (c / 2); unit u of
      // row r sits at r * 128 + ((u ^ (r % 8)) * 16)
      const uint32_t box = stg + (c >> 1) * C::kChunkBytes + r_in * 128;
      // site 8: the staged row lies inside the staging tile
      if (!ATTN_CHECK((c >> 1) < C::kOChunks && r_in < kTileRows, 8)) continue;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const uint32_t unit = static_cast<uint32_t>(((c & 1) * 4 + e) ^ (r_in & 7));
        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(box + unit * 16),
                     "r"(pk[4 * e]), "r"(pk[4 * e + 1]), "r"(pk[4 * e + 2]), "r"(pk[4 * e + 3])
                     : "memory");
      }
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) mbar_arrive(bar_stg_full);
    if constexpr (PAIR) {
      // slot 1's O and row state have been read (tcgen05.wait::ld above): it may go on
      if (x.n1 > 0) ++o1cnt;
      tc_fence_before_sync();
      if (lane == 0) mbar_arrive(bars + 8 * kBarMerged);
    }
    // site 4: the LSE index lies inside [B, Hq, Lq]
    if (p.lse != nullptr && in_range &&
        ATTN_CHECK(x.b < p.B && x.hq < p.Hq && row >= 0 && row < p.Lq, 4))
      p.lse[(static_cast<size_t>(x.b) * p.Hq + x.hq) * p.Lq + row] = (ref + log2f(l)) * kLn2;
  }
}

// ----------------------------------------------------------------- d = 256
// The MMAs of the one query tile at d = 256, split over two issuing threads:
// role 0 runs S_j = Q K_j^T into S buffer j % 2, role 1 runs O += P_j V_j. One
// thread issuing both (Q K_{j+1}^T, then P_j V_j) measured 0.79x the speed
// of the split on 8192 x 8192 x 16 heads: in program order P_j V_j then sat
// behind Q K_{j+1}^T, which waited for K_{j+1} to land, so the tensor pipe
// idled while both P_j and V_j were ready.
// Hand-offs: S_full[b] (role 0 -> softmax), P_half / P_full (softmax -> role
// 1), O_full after every P V (role 1 -> softmax: O may be rescaled or read
// out), S_free[b] after every P V (role 1 -> role 0: P_j's buffer may take
// S_{j+2}). S_free has one barrier per buffer, so the completion role 0 waits
// for is the latest one that can have happened (P V_{j+2} needs S_{j+2}
// first) and a parity wait cannot be a phase behind. Each K/V ring slot is
// released by its one reader.
template <bool BF16, bool CAUSAL, bool SPLIT, bool WINDOW, int F8>
__device__ __forceinline__ void mma_role_single(const int role, const FwdParams& p, uint32_t tmem,
                                                uint32_t sQ, uint32_t sKV, uint32_t sP, uint32_t bars,
                                                volatile int* abort_flag) {
  using C = Cfg<256, F8>;
  // e4m3: P of S buffer b in shared memory (K-major, 128-byte swizzle)
  auto p_lo = [&](int b) { return smem_desc_lo(sP + b * kTileRows * 128, 16); };
  auto bar = [&](int i) { return bars + 8 * i; };
  const uint32_t q_lo = smem_desc_lo(sQ, 16);
  auto k_lo = [&](int idx) { return smem_desc_lo(sKV + (idx % C::kStages) * C::kTileBytes, 16); };
  auto v_lo = [&](int idx) {
    return smem_desc_lo(sKV + (idx % C::kStages) * C::kTileBytes, C::kChunkBytes);
  };
  auto kv_full = [&](int idx) {
    return mbar_wait(bar(kBarKvFull + idx % C::kStages), (idx / C::kStages) & 1, abort_flag,
                     kFaultMmaKvFull, p.timeout_ns);
  };
  const uint32_t o_t = tmem + C::col_o(0);
  int kv_it = 0, uit = 0, pcnt = 0;
  int sc = 0;  // KV tiles issued so far by this thread, over all units: tile sc uses S buffer sc % 2
  bool ok = true;
  for (int u = cta_unit(0, p.n_units); u >= 0 && ok; u = cta_unit(++uit, p.n_units)) {
    const Unit x = decode_single<CAUSAL, SPLIT, WINDOW>(p, u);
    const int n = x.n0;
    if (role == 0) {
      ok = mbar_wait(bar(kBarQFull), uit & 1, abort_flag, kFaultMmaQFull, p.timeout_ns);
      if (!ok) break;
      if (SPLIT && n == 0) {
        // (causal key split) no key of this range is visible: release Q; O is
        // neither written nor signalled, the softmax writes the empty partial
        mma_commit(bar(kBarQEmpty));
      }
      for (int j = 0; j < n; ++j) {
        const int b = sc & 1;
        if (sc >= 2) {
          // P V of the tile two back (this unit's or an earlier one's) is done with buffer b
          ok = mbar_wait(bar(kBarSFree + b), ((sc >> 1) - 1) & 1, abort_flag, kFaultMmaSFree,
                         p.timeout_ns);
          if (!ok) break;
          tc_fence_after_sync();
        }
        const int kidx = kv_it + 2 * j;  // K_j
        if (!kv_full(kidx)) { ok = false; break; }
        if constexpr (F8 != 0) issue_qk_f8<256>(tmem + C::col_s(b), q_lo, k_lo(kidx));
        else issue_qk<256, BF16>(tmem + C::col_s(b), q_lo, k_lo(kidx));
        mma_commit(bar(kBarSFull + b));
        mma_commit(bar(kBarKvEmpty + kidx % C::kStages));
        if (j == n - 1) mma_commit(bar(kBarQEmpty));
        ++sc;
      }
    } else {
      for (int j = 0; j < n; ++j) {
        const int b = sc & 1;
        const int vidx = kv_it + 2 * j + 1;  // V_j
        const uint32_t s_j = tmem + C::col_s(b);
        // O += P_j V_j in two halves of 64 keys
        if (!kv_full(vidx) ||
            !mbar_wait(bar(kBarPHalf), pcnt & 1, abort_flag, kFaultMmaPFull, p.timeout_ns)) {
          ok = false;
          break;
        }
        tc_fence_after_sync();
        if constexpr (F8 != 0) issue_pv_half_f8<256, 0>(o_t, p_lo(b), k_lo(vidx), j > 0 ? 1u : 0u);
        else issue_pv_half<256, BF16, 0>(o_t, s_j, v_lo(vidx), j > 0 ? 1u : 0u);
        if (!mbar_wait(bar(kBarPFull), pcnt & 1, abort_flag, kFaultMmaPFull, p.timeout_ns)) {
          ok = false;
          break;
        }
        ++pcnt;
        tc_fence_after_sync();
        if constexpr (F8 != 0) issue_pv_half_f8<256, 1>(o_t, p_lo(b), k_lo(vidx), 1u);
        else issue_pv_half<256, BF16, 1>(o_t, s_j, v_lo(vidx), 1u);
        mma_commit(bar(kBarKvEmpty + vidx % C::kStages));
        mma_commit(bar(kBarOFull));
        mma_commit(bar(kBarSFree + b));
        ++sc;
      }
    }
    kv_it += 2 * x.nu;
  }
  if (!ok) {
    // every MMA this thread issued must finish before tensor memory is freed
    mma_commit(bar(kBarDrain + role));
    mbar_drain(bar(kBarDrain + role), 0);
  }
}

// The softmax of the one query tile (warps 0-3, one thread per row). Per KV
// tile: wait for S_j; row max; wait until P_{j-1} V_{j-1} is done (O may then
// be rescaled and S_j's buffer partner is free); exponentials into P_j. End of
// a unit: wait for the last P V, O / l to 16 bits straight to global memory.
template <bool BF16, bool CAUSAL, bool SPLIT, bool WINDOW, int F8>
__device__ __forceinline__ void softmax_role_single(const FwdParams& p, uint32_t tmem, uint32_t bars,
                                                    uint32_t sP, uint32_t sSk, volatile int* abort_flag) {
  using C = Cfg<256, F8>;
  constexpr int D = 256;
  const uint32_t skw = sSk + (threadIdx.x / 32) * 512;  // per-token scales: this warp's key scales
  const int warp = threadIdx.x / 32;
  const int r_in = threadIdx.x % kTileRows;
  const int lane = threadIdx.x % 32;
  const uint32_t lane_bits = static_cast<uint32_t>((warp % 4) * 32) << 16;
  const uint32_t tO = tmem + lane_bits + C::col_o(0);
  const uint32_t bar_p = bars + 8 * kBarPFull;
  const uint32_t bar_ph = bars + 8 * kBarPHalf;
  const uint32_t bar_o = bars + 8 * kBarOFull;
  const float sl2 = p.sl2;
  int sc = 0, ocnt = 0;
  int k = 0;
  for (int u = cta_unit(0, p.n_units); u >= 0; u = cta_unit(++k, p.n_units)) {
    const Unit x = decode_single<CAUSAL, SPLIT, WINDOW>(p, u);
    const int n = x.n0;
    const int row = x.r0 + r_in;
    int row_lim = CAUSAL ? min(p.Lk, p.kv_offset + row + 1) : p.kv_limit;
    int row_lo = 0;
    if constexpr (WINDOW) {
      const int pos = p.kv_offset + row;
      row_lo = p.win_left < 0 ? 0 : max(0, pos - p.win_left);
      row_lim = p.win_right < 0 ? p.Lk : min(p.Lk, pos + p.win_right + 1);
    }
    float ref = -INFINITY;
    float l = 0.f;
    float sl2r = sl2;  // per-token scales: times the row's Q scale
    const float* skrow = nullptr;
    float4 skv = make_float4(0.f, 0.f, 0.f, 0.f);
    if constexpr (F8 == 2) {
      const size_t qs = (static_cast<size_t>(x.b) * p.Hq + x.hq) * p.sq_pitch + row;
      sl2r = sl2 * (row < p.Lq ? __ldg(p.sq + qs) : 1.f);
      skrow = p.sk + (static_cast<size_t>(x.b) * p.Hkv + x.hkv) * p.sk_pitch;
      skv = load_key_scales(skrow, x.j0 * kTileRows + 4 * lane, p.Lk);
    }
    for (int j = 0; j < n; ++j) {
      if constexpr (F8 == 2) {
        __syncwarp();  // every lane is done with the previous tile's scales
        st_shared_v4f(skw + 16 * lane, skv);
        __syncwarp();
        if (j + 1 < n) skv = load_key_scales(skrow, (x.j0 + j + 1) * kTileRows + 4 * lane, p.Lk);
      }
      const int buf = sc & 1;
      const uint32_t tS = tmem + lane_bits + C::col_s(buf);
      bool ok = mbar_wait(bars + 8 * (kBarSFull + buf), (sc >> 1) & 1, abort_flag, kFaultSoftmaxSFull,
                          p.timeout_ns);
      if (!__all_sync(0xffffffffu, ok)) return;
      ++sc;
      tc_fence_after_sync();
      uint32_t r[128];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld_32x32b_x32(tS + 32 * c, r + 32 * c);
      tmem_wait_ld_x128(r);
      if constexpr (F8 == 2) {
#pragma unroll
        for (int c = 0; c < 128; c += 4) {
          const float4 k4 = ld_shared_v4f(skw + 4 * c);
          float a0, a1, a2, a3;
          f2_unpack(f2_mul(f2_pack_bits(r[c], r[c + 1]), f2_pack(k4.x, k4.y)), a0, a1);
          f2_unpack(f2_mul(f2_pack_bits(r[c + 2], r[c + 3]), f2_pack(k4.z, k4.w)), a2, a3);
          r[c] = __float_as_uint(a0);
          r[c + 1] = __float_as_uint(a1);
          r[c + 2] = __float_as_uint(a2);
          r[c + 3] = __float_as_uint(a3);
        }
      }
      const int key0 = (x.j0 + j) * kTileRows;
      const int lim = row_lim - key0;
      const int lim_lo = WINDOW ? row_lo - key0 : 0;
      const bool partial = lim < kTileRows || lim_lo > 0;
      if (partial) {
#pragma unroll
        for (int c = 0; c < 128; ++c)
          if (c >= lim || c < lim_lo) r[c] = __float_as_uint(-INFINITY);
      }
      float m_tile;
      {  // three-input max tree
        float a[43];
#pragma unroll
        for (int i = 0; i < 42; ++i)
          a[i] = fmax3(__uint_as_float(r[3 * i]), __uint_as_float(r[3 * i + 1]), __uint_as_float(r[3 * i + 2]));
        a[42] = fmaxf(__uint_as_float(r[126]), __uint_as_float(r[127]));
        float b[15];
#pragma unroll
        for (int i = 0; i < 14; ++i) b[i] = fmax3(a[3 * i], a[3 * i + 1], a[3 * i + 2]);
        b[14] = a[42];
        float c5[5];
#pragma unroll
        for (int i = 0; i < 5; ++i) c5[i] = fmax3(b[3 * i], b[3 * i + 1], b[3 * i + 2]);
        m_tile = fmaxf(fmax3(c5[0], c5[1], c5[2]), fmaxf(c5[3], c5[4]));
      }
      const float m_scaled = (m_tile == -INFINITY) ? -INFINITY : m_tile * sl2r;
      if (j > 0) {
        // P_{j-1} V_{j-1} done: O may be rescaled
        ok = mbar_wait(bar_o, ocnt & 1, abort_flag, kFaultSoftmaxOFull, p.timeout_ns);
        if (!__all_sync(0xffffffffu, ok)) return;
        ++ocnt;
        tc_fence_after_sync();
      }
      const bool rescale = m_scaled > ref + kRescaleTau;
      if (__any_sync(0xffffffffu, rescale)) {
        float alpha = 1.f;
        if (rescale) {
          alpha = ex2_approx(ref - m_scaled);
          ref = m_scaled;
          l *= alpha;
        }
        if (j > 0) {
#pragma unroll 1
          for (int c = 0; c < D / 32; ++c) {
            uint32_t ov[32];
            tmem_ld_32x32b_x32(tO + 32 * c, ov);
            tmem_wait_ld_x32(ov);
#pragma unroll
            for (int e = 0; e < 32; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * alpha);
            tmem_st_32x32b_x32(tO + 32 * c, ov);
          }
          tmem_wait_st();
        }
      }
      float sum[4] = {0.f, 0.f, 0.f, 0.f};
      if constexpr (F8 != 0) {
        const uint32_t prow = sP + buf * kTileRows * 128 + r_in * 128;  // e4m3 P row of this S buffer
        if (__any_sync(0xffffffffu, partial))
          exp_tile_f8<true>(r, sl2r, -ref, lim, lim_lo, sum, prow, r_in, bar_ph, bar_p, 0u, false, lane);
        else
          exp_tile_f8<false>(r, sl2r, -ref, lim, lim_lo, sum, prow, r_in, bar_ph, bar_p, 0u, false, lane);
      } else if (__any_sync(0xffffffffu, partial)) {
        exp_tile<BF16, true>(r, sl2, -ref, lim, lim_lo, sum, tS, bar_ph, bar_p, 0u, false, lane);
      } else {
        exp_tile<BF16, false>(r, sl2, -ref, lim, lim_lo, sum, tS, bar_ph, bar_p, 0u, false, lane);
      }
      l += (sum[0] + sum[1]) + (sum[2] + sum[3]);
    }
    if constexpr (SPLIT) {
      // float32 O / l and the LSE of this key range; a row (or the whole
      // tile) that sees no key of the range writes O = 0, LSE = -inf
      const bool in_range = row < p.Lq && ATTN_CHECK(x.split < p.n_splits && x.b < p.B && x.hq < p.Hq, 5);
      const size_t prow = ((static_cast<size_t>(x.split) * p.B + x.b) * p.Hq + x.hq) * p.Lq + row;
      float* dst = p.o_part + prow * D;
      if (n == 0) {
        if (in_range) {
#pragma unroll 1
          for (int c = 0; c < D; c += 4) *reinterpret_cast<float4*>(dst + c) = make_float4(0.f, 0.f, 0.f, 0.f);
          p.lse_part[prow] = -INFINITY;
        }
        continue;
      }
      bool ok = mbar_wait(bar_o, ocnt & 1, abort_flag, kFaultSoftmaxOFull, p.timeout_ns);
      if (!__all_sync(0xffffffffu, ok)) return;
      ++ocnt;
      tc_fence_after_sync();
      const bool empty = !(l > 0.f);
      const float inv_l = empty ? 0.f : 1.f / l;
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        uint32_t ov[32];
        tmem_ld_32x32b_x32(tO + 32 * c, ov);
        tmem_wait_ld_x32(ov);
        if (in_range) {
#pragma unroll
          for (int e = 0; e < 32; e += 4)
            *reinterpret_cast<float4*>(dst + 32 * c + e) =
                make_float4(__uint_as_float(ov[e]) * inv_l, __uint_as_float(ov[e + 1]) * inv_l,
                            __uint_as_float(ov[e + 2]) * inv_l, __uint_as_float(ov[e + 3]) * inv_l);
        }
      }
      if (in_range) p.lse_part[prow] = empty ? -INFINITY : (ref + log2f(l)) * kLn2;
      continue;
    }
    // the last P V, then O / l straight to global memory
    bool ok = mbar_wait(bar_o, ocnt & 1, abort_flag, kFaultSoftmaxOFull, p.timeout_ns);
    if (!__all_sync(0xffffffffu, ok)) return;
    ++ocnt;
    tc_fence_after_sync();
    const float inv_l = 1.f / l;
    const bool in_range = row < p.Lq;
    uint16_t* dst = static_cast<uint16_t*>(p.o) + ((static_cast<size_t>(x.b) * p.Lq + row) * p.Hq + x.hq) * D;
    // site 9: the output row lies inside [B, Lq, Hq, D]
    const bool dst_ok = ATTN_CHECK(x.b < p.B && x.hq < p.Hq && (row < p.Lq || !in_range), 9);
#pragma unroll 1
    for (int c = 0; c < D / 32; ++c) {
      uint32_t ov[32];
      tmem_ld_32x32b_x32(tO + 32 * c, ov);
      tmem_wait_ld_x32(ov);
      if (in_range && dst_ok) {
        if constexpr (F8 == 2) {
          if (p.sv != nullptr) {  // V's per-channel scales
            const float4* sv4 = reinterpret_cast<const float4*>(
                p.sv + (static_cast<size_t>(x.b) * p.Hkv + x.hkv) * D + 32 * c);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const float4 f = __ldg(sv4 + e);
              ov[4 * e] = __float_as_uint(__uint_as_float(ov[4 * e]) * f.x);
              ov[4 * e + 1] = __float_as_uint(__uint_as_float(ov[4 * e + 1]) * f.y);
              ov[4 * e + 2] = __float_as_uint(__uint_as_float(ov[4 * e + 2]) * f.z);
              ov[4 * e + 3] = __float_as_uint(__uint_as_float(ov[4 * e + 3]) * f.w);
            }
          }
        }
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e)
          pk[e] = pack2<BF16>(__uint_as_float(ov[2 * e]) * inv_l, __uint_as_float(ov[2 * e + 1]) * inv_l);
#pragma unroll
        for (int e = 0; e < 4; ++e)
          *reinterpret_cast<uint4*>(dst + 32 * c + 8 * e) =
              make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
      }
    }
    if (p.lse != nullptr && in_range &&
        ATTN_CHECK(x.b < p.B && x.hq < p.Hq && row >= 0 && row < p.Lq, 4))
      p.lse[(static_cast<size_t>(x.b) * p.Hq + x.hq) * p.Lq + row] = (ref + log2f(l)) * kLn2;
    // every TMEM read of O is complete (wait::ld) before the next unit's first
    // P V overwrites it: that MMA waits for this warpgroup's next P
  }
}

template <int D, bool BF16, bool CAUSAL, bool SPLIT, bool WINDOW, int F8, bool PAIR = false>
__global__ void __launch_bounds__(kThreads, 1)
    attn_fwd_sm100_kernel(const __grid_constant__ CUtensorMap tm_q,
                          const __grid_constant__ CUtensorMap tm_k,
                          const __grid_constant__ CUtensorMap tm_v,
                          const __grid_constant__ CUtensorMap tm_o, const FwdParams p) {
  using C = Cfg<D, F8>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t sQ = sbase + C::kOffQ;
  const uint32_t sKV = sbase + C::kOffKV;
  const uint32_t sStg = sbase + C::kOffStg;
  const uint32_t sP = sbase + C::kOffP;  // e4m3 P buffers (unused otherwise)
  const uint32_t bars = sbase + C::kOffBar;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffBar + 448);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffBar + 452);
  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;

  if (threadIdx.x == 0) {
    for (int t = 0; t < 2; ++t) {
      mbar_init(bars + 8 * (kBarQFull + t), 1);
      mbar_init(bars + 8 * (kBarQEmpty + t), 1);
      mbar_init(bars + 8 * (kBarSFull + t), 1);
      mbar_init(bars + 8 * (kBarPFull + t), kTileRows / 32);
      mbar_init(bars + 8 * (kBarPHalf + t), kTileRows / 32);
      mbar_init(bars + 8 * (kBarTurn + t), kTileRows / 32);
      mbar_init(bars + 8 * (kBarOFull + t), 1);
    }
    mbar_init(bars + 8 * kBarDrain, 1);
    mbar_init(bars + 8 * kBarStgFull, kTileRows / 32);
    mbar_init(bars + 8 * (kBarStgFree + 0), 1);
    mbar_init(bars + 8 * (kBarStgFree + 1), 1);
    mbar_init(bars + 8 * (kBarDrain + 1), 1);
    mbar_init(bars + 8 * (kBarSFree + 0), 1);
    mbar_init(bars + 8 * (kBarSFree + 1), 1);
    mbar_init(bars + 8 * kBarMerge1, kTileRows / 32);
    mbar_init(bars + 8 * kBarMerged, kTileRows / 32);
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(bars + 8 * (kBarKvFull + s), 1);
      // d = 256: a K tile is read by the Q K^T issuer only, a V tile by the P V issuer only
      mbar_init(bars + 8 * (kBarKvEmpty + s), D == 256 ? 1 : 2);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 8 && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
    tma_prefetch_desc(&tm_o);
  }
  if (warp == 9) {
    tmem_alloc(smem_u32(tmem_slot), C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  // Programmatic dependent launch: everything above (barriers, tensor memory,
  // descriptor prefetch) may overlap the previous kernel on this stream; no
  // global memory is touched before that kernel has completed and its writes
  // are visible. The next kernel may then start its own set-up on SMs this
  // grid leaves idle.
  griddep_wait();
  griddep_launch_dependents();

  if constexpr (D == 256) {
    // one query tile: warps 0-3 softmax, warp 8 loads, warp 9 issues Q K^T,
    // warp 10 issues P V
    if (warp < 8) {
      regs_increase<kRegsSoftmax>();
      if (warp < 4)
        softmax_role_single<BF16, CAUSAL, SPLIT, WINDOW, F8>(p, tmem, bars, sP, sbase + C::kOffSk, abort_flag);
    } else {
      regs_decrease<kRegsProducer>();
      if (warp == 8 && lane == 0)
        load_role<D, BF16, CAUSAL, SPLIT, WINDOW, F8>(&tm_q, &tm_k, &tm_v, p, sQ, sKV, bars, abort_flag);
      else if ((warp == 9 || warp == 10) && lane == 0)
        mma_role_single<BF16, CAUSAL, SPLIT, WINDOW, F8>(warp - 9, p, tmem, sQ, sKV, sP, bars, abort_flag);
    }
  } else if (warp < 8) {
    regs_increase<kRegsSoftmax>();
    uint32_t sMl = 0;  // pair split: slot 1's row state for the merge
    if constexpr (PAIR) sMl = sbase + C::kOffMl;
    softmax_role<D, BF16, CAUSAL, SPLIT, WINDOW, F8, PAIR>(warp / 4, p, tmem, bars, sStg, sP,
                                                           sbase + C::kOffSk, sMl, abort_flag);
  } else {
    regs_decrease<kRegsProducer>();
    if (warp == 8) {
      if (lane == 0)
        load_role<D, BF16, CAUSAL, SPLIT, WINDOW, F8, PAIR>(&tm_q, &tm_k, &tm_v, p, sQ, sKV, bars, abort_flag);
    } else if (warp == 9 || warp == 10) {
      if (lane == 0)
        mma_role<D, BF16, CAUSAL, SPLIT, WINDOW, F8, PAIR>(warp - 9, p, tmem, sQ, sKV, sP, bars, abort_flag);
    } else if (!SPLIT) {
      if (lane == 0) store_role<D, BF16, CAUSAL, SPLIT, WINDOW, F8, PAIR>(&tm_o, p, sStg, bars, abort_flag);
    }
  }
  __syncwarp();
  tc_fence_before_sync();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

// ------------------------------------------------------------- key-split merge

// Combines the key splits of attn_fwd_splitkv: for output row (b, i, hq),
// lse = ln sum_g exp(lse_g) and O = sum_g exp(lse_g - lse) O_g (attention over
// disjoint key ranges regrouped: the softmax of the developer guide's "Multi
// Head Attention Definition" with its normaliser summed part by part). One warp
// per output row; lane l holds d / 32 consecutive features. Reads
// n_splits * (d + 1) floats and writes d 16-bit values per row: HBM-bound.
template <int D, bool BF16>
__global__ void __launch_bounds__(256) split_merge_kernel(const float* __restrict__ o_part,
                                                          const float* __restrict__ lse_part, void* o,
                                                          float* lse, int n_splits, int B, int Lq,
                                                          int Hq, int d_out) {
  constexpr int kPer = D / 32;
  const long long w = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) / 32;
  const int lane = threadIdx.x % 32;
  const long long rows = 1LL * B * Hq * Lq;
  if (w >= rows) return;
  // site 10: this lane's columns lie inside the partial rows and the output row
  if (!ATTN_CHECK(lane * kPer + kPer <= D && d_out <= D, 10)) return;
  // w = (b * Hq + hq) * Lq + i: the row index of the partial buffers
  const int i = static_cast<int>(w % Lq);
  const long long bh = w / Lq;
  const int hq = static_cast<int>(bh % Hq);
  const int b = static_cast<int>(bh / Hq);
  const size_t split_rows = static_cast<size_t>(rows);
  float m = -INFINITY;
  for (int g = 0; g < n_splits; ++g) m = fmaxf(m, lse_part[g * split_rows + w]);
  float acc[kPer];
#pragma unroll
  for (int e = 0; e < kPer; ++e) acc[e] = 0.f;
  float tot = 0.f;
  for (int g = 0; g < n_splits; ++g) {
    const float wg = expf(lse_part[g * split_rows + w] - m);
    tot += wg;
    const float* src = o_part + (g * split_rows + w) * D + lane * kPer;
#pragma unroll
    for (int e = 0; e < kPer; ++e) acc[e] = fmaf(wg, src[e], acc[e]);
  }
  const float inv = 1.f / tot;
  uint16_t* out = static_cast<uint16_t*>(o) + ((static_cast<size_t>(b) * Lq + i) * Hq + hq) * d_out + lane * kPer;
  // d_out < D: the partials' columns >= d_out are zero and not stored
  if (lane * kPer < d_out) {
#pragma unroll
    for (int e = 0; e < kPer; e += 2) {
      const uint32_t pk = pack2<BF16>(acc[e] * inv, acc[e + 1] * inv);
      *reinterpret_cast<uint32_t*>(out + e) = pk;
    }
  }
  if (lse != nullptr && lane == 0) lse[w] = m + logf(tot);
}

// ------------------------------------------------------------- diagnostics

// One 128x128 tile: S = Q K^T, then O = round16(S/16) V, through the same
// descriptors and MMA issue code as the forward kernel. 128 threads.
template <bool BF16>
__global__ void __launch_bounds__(128, 1)
    selftest_mma_kernel(const __grid_constant__ CUtensorMap tm_q,
                        const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_v, float* s_out, float* o_out,
                        unsigned long long timeout_ns) {
  constexpr int D = 128;
  using C = Cfg<D>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sQ = smem_u32(smem);
  const uint32_t sK = sQ + C::kTileBytes;
  const uint32_t sV = sK + C::kTileBytes;
  const uint32_t bars = sV + C::kTileBytes;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + 3 * C::kTileBytes + 64);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + 3 * C::kTileBytes + 68);
  const int warp = threadIdx.x / 32;
  if (threadIdx.x == 0) {
    mbar_init(bars, 1);      // TMA
    mbar_init(bars + 8, 1);  // MMA
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  const uint32_t lane_bits = static_cast<uint32_t>(warp * 32) << 16;
  bool ok = true;

  if (threadIdx.x == 0) {
    const uint64_t pol = l2_policy_evict_first();
    mbar_arrive_expect_tx(bars, 3 * C::kTileBytes);
    for (int c = 0; c < 2; ++c) {
      tma_load_4d(sQ + c * C::kChunkBytes, &tm_q, bars, c * 64, 0, 0, 0, pol);
      tma_load_4d(sK + c * C::kChunkBytes, &tm_k, bars, c * 64, 0, 0, 0, pol);
      tma_load_4d(sV + c * C::kChunkBytes, &tm_v, bars, c * 64, 0, 0, 0, pol);
    }
    ok = mbar_wait(bars, 0, abort_flag, kFaultSelftest, timeout_ns);
    if (ok) {
      tc_fence_after_sync();
      issue_qk<D, BF16>(tmem + 0, smem_desc_lo(sQ, 16), smem_desc_lo(sK, 16));
    }
    mma_commit(bars + 8);
  }
  ok = mbar_wait(bars + 8, 0, abort_flag, kFaultSelftest, timeout_ns);
  ok = __all_sync(0xffffffffu, ok);
  tc_fence_after_sync();
  const int row = threadIdx.x;
  if (ok) {
    uint32_t r[128];
    for (int c = 0; c < 4; ++c) tmem_ld_32x32b_x32(tmem + lane_bits + 32 * c, r + 32 * c);
    tmem_wait_ld_x128(r);
    uint32_t pk[64];
    for (int c = 0; c < 128; ++c) s_out[row * 128 + c] = __uint_as_float(r[c]);
    for (int c = 0; c < 64; ++c)
      pk[c] = pack2<BF16>(__uint_as_float(r[2 * c]) * 0.0625f, __uint_as_float(r[2 * c + 1]) * 0.0625f);
    tmem_st_32x32b_x32(tmem + lane_bits, pk);
    tmem_st_32x32b_x32(tmem + lane_bits + 32, pk + 32);
    tmem_wait_st();
  }
  tc_fence_before_sync();
  __syncthreads();
  if (threadIdx.x == 0) {
    tc_fence_after_sync();
    if (!*abort_flag) issue_pv<D, BF16>(tmem + 256, tmem + 0, smem_desc_lo(sV, C::kChunkBytes), 0u);
    mma_commit(bars + 8);
  }
  ok = !*abort_flag && mbar_wait(bars + 8, 1, abort_flag, kFaultSelftest, timeout_ns);
  ok = __all_sync(0xffffffffu, ok);
  tc_fence_after_sync();
  if (ok) {
    for (int c = 0; c < 4; ++c) {
      uint32_t ov[32];
      tmem_ld_32x32b_x32(tmem + lane_bits + 256 + 32 * c, ov);
      tmem_wait_ld_x32(ov);
      for (int e = 0; e < 32; ++e) o_out[row * 128 + 32 * c + e] = __uint_as_float(ov[e]);
    }
  }
  tc_fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, 512);
  }
}

// The FMA-pipe exponential on n inputs (one value per thread pair slot).
__global__ void selftest_exp2_kernel(const float* x, float* y, int n) {
  const int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
  if (i >= n) return;
  const float a = x[i], b = (i + 1 < n) ? x[i + 1] : 0.f;
  float r0, r1;
  f2_unpack(exp2_poly_x2(f2_pack(a, b)), r0, r1);
  y[i] = r0;
  if (i + 1 < n) y[i + 1] = r1;
}

// One thread waits on a barrier nothing completes; the bounded wait must give up.
__global__ void selftest_timeout_kernel(unsigned long long timeout_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    mbar_init(smem_u32(&bar), 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    (void)mbar_wait(smem_u32(&bar), 0, &abort_flag, kFaultSelftest, timeout_ns);
  }
}

// ------------------------------------------------------------------- host

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

std::atomic<unsigned long long> g_timeout_ns{4000000000ull};

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = []() -> EncodeTiledFn {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    return reinterpret_cast<EncodeTiledFn>(f);
  }();
  return fn;
}

struct DeviceInfo {
  bool ok = false;
  bool sm100 = false;
  int num_sms = 0;
};

constexpr int kMaxDevices = 64;

DeviceInfo device_info(int dev) {
  static DeviceInfo infos[kMaxDevices];
  static std::once_flag flags[kMaxDevices];
  if (dev < 0 || dev >= kMaxDevices) return DeviceInfo{};
  std::call_once(flags[dev], [dev]() {
    DeviceInfo di;
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) == cudaSuccess &&
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) == cudaSuccess &&
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess) {
      di.ok = true;
      di.sm100 = (major == 10 && minor == 0);
      di.num_sms = sms;
    }
    infos[dev] = di;
  });
  return infos[dev];
}

// [B, L, H, d] 16-bit tensor as a 4-D TMA map (innermost first: d, H, L, B);
// box = 64 elements of d x 1 head x 128 rows x 1 batch, 128-byte swizzle.
// Consecutive batches are `batch_rows` rows apart (L for a contiguous tensor,
// the capacity S when the rows are the valid prefix of a [B, S, H, d] cache).
bool encode_bl_hd(CUtensorMap* map, const void* ptr, int B, int L, int H, int d, bool bf16,
                  int batch_rows = -1) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t rows = batch_rows < 0 ? (cuuint64_t)L : (cuuint64_t)batch_rows;
  const cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)L, (cuuint64_t)B};
  const cuuint64_t strides[3] = {(cuuint64_t)d * 2, (cuuint64_t)H * d * 2, rows * H * d * 2};
  const cuuint32_t box[4] = {64, 1, (cuuint32_t)kTileRows, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = fn(map, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 4,
                  const_cast<void*>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// [B, L, H, d] e4m3 tensor (d = 128 bytes per head row) as a 4-D TMA map:
// box = the whole 128-byte row of one head x 128 rows, 128-byte swizzle.
bool encode_e4m3_bl_hd(CUtensorMap* map, const void* ptr, int B, int L, int H, int d) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)L, (cuuint64_t)B};
  const cuuint64_t strides[3] = {(cuuint64_t)d, (cuuint64_t)H * d, (cuuint64_t)L * H * d};
  const cuuint32_t box[4] = {128, 1, (cuuint32_t)kTileRows, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, const_cast<void*>(ptr), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Transposed e4m3 V, [B, Hkv, d, pitch] bytes (key index innermost, rows of
// `pitch` >= Lk bytes): box = 128 keys x 128 d-rows, 128-byte swizzle.
bool encode_e4m3_vt(CUtensorMap* map, const void* ptr, int B, int Lk, int pitch, int Hkv, int d) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[4] = {(cuuint64_t)Lk, (cuuint64_t)d, (cuuint64_t)Hkv, (cuuint64_t)B};
  const cuuint64_t strides[3] = {(cuuint64_t)pitch, (cuuint64_t)d * pitch, (cuuint64_t)Hkv * d * pitch};
  const cuuint32_t box[4] = {(cuuint32_t)kTileRows, 128, 1, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, const_cast<void*>(ptr), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D, bool BF16, bool CAUSAL, bool SPLIT = false, bool WINDOW = false, int F8 = 0, bool PAIR = false>
int launch_fwd(const FwdParams& p, const void* q, const void* k, const void* v, int kv_rows, int grid,
               cudaStream_t stream) {
  using C = Cfg<D, F8>;
  CUtensorMap tq, tk, tv, to;
  if constexpr (F8 != 0) {
    // e4m3 Q / K (box: the 128-byte row of a head, 128 rows); V transposed,
    // [B, Hkv, d, kv_rows] bytes with kv_rows a multiple of 16 (box: 128 keys
    // x 128 d-rows); O bf16 as usual
    // d < 128: the 128-byte boxes read the columns (V^T: the rows) past d as
    // zero, and the O chunks past d are clipped or skipped
    const int dt = p.d > 0 ? p.d : D;
    if (dt > D || !encode_e4m3_bl_hd(&tq, q, p.B, p.Lq, p.Hq, dt) ||
        !encode_e4m3_bl_hd(&tk, k, p.B, p.Lk, p.Hkv, dt) ||
        !encode_e4m3_vt(&tv, v, p.B, p.Lk, kv_rows, p.Hkv, dt) ||
        !encode_bl_hd(&to, p.o, p.B, p.Lq, p.Hq, dt, true))
      return ATTN_ERR_CUDA;
  } else {
    const int dt = p.d > 0 ? p.d : D;
    if (dt > D || !encode_bl_hd(&tq, q, p.B, p.Lq, p.Hq, dt, BF16) ||
        !encode_bl_hd(&tk, k, p.B, p.Lk, p.Hkv, dt, BF16, kv_rows) ||
        !encode_bl_hd(&tv, v, p.B, p.Lk, p.Hkv, dt, BF16, kv_rows) ||
        !encode_bl_hd(&to, p.o, p.B, p.Lq, p.Hq, dt, BF16))
      return ATTN_ERR_CUDA;
  }
  auto kern = attn_fwd_sm100_kernel<D, BF16, CAUSAL, SPLIT, WINDOW, F8, PAIR>;
  static std::once_flag attr_flags[kMaxDevices];
  static int attr_status[kMaxDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return ATTN_ERR_CUDA;
  std::call_once(attr_flags[dev], [&]() {
    attr_status[dev] = ATTN_OK;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes) !=
        cudaSuccess) {
      attr_status[dev] = ATTN_ERR_CUDA;
      return;
    }
    // The warpgroup register split must fit the block's launch budget, or the
    // softmax warpgroups' setmaxnreg.inc would wait for registers forever.
    cudaFuncAttributes fa{};
    if (cudaFuncGetAttributes(&fa, kern) != cudaSuccess ||
        fa.numRegs * kThreads < 128 * kRegsProducer + 256 * kRegsSoftmax)
      attr_status[dev] = ATTN_ERR_CUDA;
  });
  if (attr_status[dev] != ATTN_OK) return attr_status[dev];
  (void)cudaGetLastError();  // launch errors below are this launch's own
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = C::kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kern, tq, tk, tv, to, p) != cudaSuccess) return ATTN_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

bool ranges_overlap(const void* a, size_t na, const void* b, size_t nb) {
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return x < y + nb && y < x + na;
}

}  // namespace hasb

using namespace hasb;

extern "C" {

const char* attn_status_string(int status) {
  switch (status) {
    case ATTN_OK: return "ok";
    case ATTN_ERR_INVALID_ARG: return "invalid argument";
    case ATTN_ERR_UNSUPPORTED: return "unsupported configuration (head_dim or device)";
    case ATTN_ERR_CUDA: return "CUDA error";
    case ATTN_ERR_TIMEOUT: return "device-side wait timed out";
    case ATTN_ERR_SCRATCH_LIMIT: return "request exceeds the library's fixed-size scratch";
    default: return "unknown status";
  }
}

int attn_set_wait_timeout_ns(unsigned long long ns) {
  g_timeout_ns.store(ns < 1000000ull ? 1000000ull : ns);
  return ATTN_OK;
}

}  // extern "C"

namespace hasb {

// The argument contract of attn_fwd; makes no CUDA call.
int attn_fwd_validate(const void* q, const void* k, const void* v, const void* o, const float* lse,
                      int B, int Lq, int Lk, int Hq, int Hkv, int d, float scale, int causal,
                      int kv_offset, int dtype, int kv_rows) {
  // ---- argument contract (no CUDA call before this block is passed)
  if (q == nullptr || k == nullptr || v == nullptr || o == nullptr) return ATTN_ERR_INVALID_ARG;
  if (B < 1 || Lq < 1 || Lk < 1 || Hq < 1 || Hkv < 1 || Hq % Hkv != 0) return ATTN_ERR_INVALID_ARG;
  if (d < 16 || d > 256 || (d & (d - 1)) != 0) return ATTN_ERR_INVALID_ARG;
  if (!std::isfinite(scale) || scale < 0.f) return ATTN_ERR_INVALID_ARG;
  if (dtype != ATTN_DTYPE_BF16 && dtype != ATTN_DTYPE_FP16) return ATTN_ERR_INVALID_ARG;
  if (causal != ATTN_MASK_NONE && causal != ATTN_MASK_CAUSAL && causal != ATTN_MASK_CHUNK)
    return ATTN_ERR_INVALID_ARG;
  if (causal == ATTN_MASK_NONE) {
    if (kv_offset != 0) return ATTN_ERR_INVALID_ARG;
  } else if (kv_offset < 0 || static_cast<long long>(kv_offset) + Lq > Lk) {
    return ATTN_ERR_INVALID_ARG;
  }
  const auto aligned16 = [](const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15u) == 0; };
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return ATTN_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(lse) & 3u) != 0) return ATTN_ERR_INVALID_ARG;
  const unsigned long long q_elems = 1ull * B * Lq * Hq * d;
  if (kv_rows < Lk) return ATTN_ERR_INVALID_ARG;
  const unsigned long long kv_elems = 1ull * B * kv_rows * Hkv * d;
  if (q_elems * 2 >= (1ull << 40) || kv_elems * 2 >= (1ull << 40)) return ATTN_ERR_INVALID_ARG;
  const long long n_pairs = (Lq + 2LL * kTileRows - 1) / (2LL * kTileRows);
  const long long n_units = n_pairs * B * Hq;
  if (n_units > 0x7fffffffLL) return ATTN_ERR_INVALID_ARG;
  if (ranges_overlap(o, q_elems * 2, q, q_elems * 2) || ranges_overlap(o, q_elems * 2, k, kv_elems * 2) ||
      ranges_overlap(o, q_elems * 2, v, kv_elems * 2))
    return ATTN_ERR_INVALID_ARG;
  if (d != 16 && d != 32 && d != 64 && d != 128 && d != 256) return ATTN_ERR_UNSUPPORTED;
  return ATTN_OK;
}

// attn_fwd over K/V whose consecutive batches are kv_rows rows apart.
int attn_fwd_impl(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Lq,
                  int Lk, int kv_rows, int Hq, int Hkv, int d, float scale, int causal, int kv_offset,
                  int dtype, void* stream, bool window = false, int win_left = -1,
                  int win_right = -1, int pair = -1) {
  // ---- argument contract (no CUDA call before it passes); a window uses the
  // offset rule of masks 1 and 2 (0 <= kv_offset, kv_offset + Lq <= Lk)
  const int valid = attn_fwd_validate(q, k, v, o, lse, B, Lq, Lk, Hq, Hkv, d, scale,
                                      window ? ATTN_MASK_CHUNK : causal, kv_offset, dtype, kv_rows);
  if (valid != ATTN_OK) return valid;
  if (window && (win_left < -1 || win_right < -1)) return ATTN_ERR_INVALID_ARG;
  // units: pairs of 128-row query tiles; single tiles at d = 256
  const long long rows_per_unit = d == 256 ? kTileRows : 2LL * kTileRows;
  const long long n_pairs = (Lq + rows_per_unit - 1) / rows_per_unit;
  const long long n_units = n_pairs * B * Hq;

  // ---- device
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return ATTN_ERR_CUDA;
  const DeviceInfo di = device_info(dev);
  if (!di.ok) return ATTN_ERR_CUDA;
  if (!di.sm100) return ATTN_ERR_UNSUPPORTED;

  FwdParams p{};
  p.d = d;
  p.o = o;
  p.lse = lse;
  p.B = B; p.Lq = Lq; p.Lk = Lk; p.Hq = Hq; p.Hkv = Hkv; p.group = Hq / Hkv;
  p.kv_offset = kv_offset;
  p.kv_limit = (causal == ATTN_MASK_CHUNK) ? kv_offset + Lq : Lk;
  p.n_pairs = static_cast<int>(n_pairs);
  p.n_units = static_cast<int>(n_units);
  p.sl2 = scale * kLog2e;
  p.timeout_ns = g_timeout_ns.load();
  p.n_splits = 1;
  p.split_tiles = (p.kv_limit + kTileRows - 1) / kTileRows;
  p.o_part = nullptr;
  p.lse_part = nullptr;
  p.win_left = win_left;
  p.win_right = win_right;
  const int grid = static_cast<int>(n_units < di.num_sms ? n_units : di.num_sms);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const bool bf16 = dtype == ATTN_DTYPE_BF16;
  if (window) {
    p.kv_limit = Lk;
    if (d == 256)
      return bf16 ? launch_fwd<256, true, false, false, true>(p, q, k, v, kv_rows, grid, s)
                  : launch_fwd<256, false, false, false, true>(p, q, k, v, kv_rows, grid, s);
    if (d == 128)
      return bf16 ? launch_fwd<128, true, false, false, true>(p, q, k, v, kv_rows, grid, s)
                  : launch_fwd<128, false, false, false, true>(p, q, k, v, kv_rows, grid, s);
    return bf16 ? launch_fwd<64, true, false, false, true>(p, q, k, v, kv_rows, grid, s)
                : launch_fwd<64, false, false, false, true>(p, q, k, v, kv_rows, grid, s);
  }
  const bool cz = causal == ATTN_MASK_CAUSAL;
  // pair < 0: decide from this launch's unit count; 0 / 1: the caller decided
  // (a chunk of a larger call takes the whole call's choice, so its rows are
  // computed exactly as the whole call computes them)
  if (cz && d <= 128 && (pair < 0 ? n_units < di.num_sms : pair != 0)) {
    // pair split: one query tile per unit, its KV tiles shared by the CTA's
    // two slots (causal units of unequal length that do not fill the SMs)
    const long long n_tiles = (Lq + kTileRows - 1) / kTileRows;
    p.n_pairs = static_cast<int>(n_tiles);
    p.n_units = static_cast<int>(n_tiles * B * Hq);
    const int pgrid = static_cast<int>(p.n_units < di.num_sms ? p.n_units : di.num_sms);
    if (d == 128)
      return bf16 ? launch_fwd<128, true, true, false, false, 0, true>(p, q, k, v, kv_rows, pgrid, s)
                  : launch_fwd<128, false, true, false, false, 0, true>(p, q, k, v, kv_rows, pgrid, s);
    return bf16 ? launch_fwd<64, true, true, false, false, 0, true>(p, q, k, v, kv_rows, pgrid, s)
                : launch_fwd<64, false, true, false, false, 0, true>(p, q, k, v, kv_rows, pgrid, s);
  }
  if (d == 256) {
    if (bf16) return cz ? launch_fwd<256, true, true>(p, q, k, v, kv_rows, grid, s) : launch_fwd<256, true, false>(p, q, k, v, kv_rows, grid, s);
    return cz ? launch_fwd<256, false, true>(p, q, k, v, kv_rows, grid, s) : launch_fwd<256, false, false>(p, q, k, v, kv_rows, grid, s);
  }
  if (d == 128) {
    if (bf16) return cz ? launch_fwd<128, true, true>(p, q, k, v, kv_rows, grid, s) : launch_fwd<128, true, false>(p, q, k, v, kv_rows, grid, s);
    return cz ? launch_fwd<128, false, true>(p, q, k, v, kv_rows, grid, s) : launch_fwd<128, false, false>(p, q, k, v, kv_rows, grid, s);
  }
  if (bf16) return cz ? launch_fwd<64, true, true>(p, q, k, v, kv_rows, grid, s) : launch_fwd<64, true, false>(p, q, k, v, kv_rows, grid, s);
  return cz ? launch_fwd<64, false, true>(p, q, k, v, kv_rows, grid, s) : launch_fwd<64, false, false>(p, q, k, v, kv_rows, grid, s);
}

// Key splits for attn_fwd_splitkv: `requested` (0 = choose) split count, the
// KV tile count of the visible range, and the base unit count; returns the
// split count actually used and the tiles per split (no split is empty).
void choose_splits(int requested, int total_tiles, long long base_units, int num_sms, int* n_splits,
                   int* split_tiles, bool causal = false) {
  long long want = requested;
  if (want <= 0 && causal) {
    // causal units differ in length (the diagonal), so splitting only pays
    // while the units do not fill the SMs on their own
    want = base_units >= num_sms ? 1 : num_sms / base_units;
    if (want > 32) want = 32;
  } else if (want <= 0) {
    // fewest waves per unit of work: ceil(units * n / SMs) / n, with 2 % per
    // extra split for the partial outputs and the merge
    double best = 1e300;
    want = 1;
    const int cap = total_tiles < 32 ? total_tiles : 32;
    for (int n = 1; n <= cap; ++n) {
      const long long waves = (base_units * n + num_sms - 1) / num_sms;
      const double cost = static_cast<double>(waves) / n * (1.0 + 0.02 * (n - 1));
      if (cost < best - 1e-12) {
        best = cost;
        want = n;
      }
    }
  }
  if (want > total_tiles) want = total_tiles;
  if (want < 1) want = 1;
  const int per = static_cast<int>((total_tiles + want - 1) / want);
  *split_tiles = per;
  *n_splits = (total_tiles + per - 1) / per;
}


// Scratch of attn_fwd_splitkv_static: float32 partial outputs and LSEs of the
// key ranges, in a file-scope device array (64 MB, reserved on every device
// that loads this library's module, until the process exits); that entry
// point allocates nothing. Calls that use it must not overlap in time (one
// stream, or ordered by the caller): they share the array.
constexpr size_t kStaticScratchFloats = size_t(16) << 20;
__device__ __align__(256) float g_split_scratch[kStaticScratchFloats];

// Device address of g_split_scratch on the current device. In host code the
// array's name is only a host-side stand-in, so the address is asked for once
// per device (with that device current, on the first call there) and kept.
int static_scratch(float** ptr) {
  static std::once_flag flags[kMaxDevices];
  static void* addr[kMaxDevices];
  static int status[kMaxDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return ATTN_ERR_CUDA;
  std::call_once(flags[dev], [dev]() {
    void* a = nullptr;
    status[dev] = cudaGetSymbolAddress(&a, g_split_scratch) == cudaSuccess && a != nullptr ? ATTN_OK
                                                                                        : ATTN_ERR_CUDA;
    addr[dev] = a;
  });
  *ptr = static_cast<float*>(addr[dev]);
  return status[dev];
}

// Argument contract of the key-split entry points (no CUDA call).
int splitkv_validate(const void* q, const void* k, const void* v, const void* o, const float* lse,
                     int n_splits, int B, int Lq, int Lk, int Hq, int Hkv, int d, float scale,
                     int causal, int kv_offset, int dtype) {
  const int valid = attn_fwd_validate(q, k, v, o, lse, B, Lq, Lk, Hq, Hkv, d, scale, causal,
                                      kv_offset, dtype, Lk);
  if (valid != ATTN_OK) return valid;
  if (n_splits < 0) return ATTN_ERR_INVALID_ARG;
  return ATTN_OK;
}

// The key-split forward after validation. fit (the library's fixed scratch):
// an automatic split count (n_splits = 0) is lowered until the partials fit
// (down to one range, i.e. plain attn_fwd); an explicit count that does not
// fit is refused with ATTN_ERR_SCRATCH_LIMIT before anything is launched.
int splitkv_run(const void* q, const void* k, const void* v, void* o, float* lse, float* workspace,
                size_t workspace_bytes, bool fit, int n_splits, int B, int Lq, int Lk, int Hq,
                int Hkv, int d, float scale, int causal, int kv_offset, int dtype, int* splits_used,
                void* stream) {
  // units: pairs of 128-row query tiles; single tiles at d = 256
  const long long rows_per_unit = d == 256 ? kTileRows : 2LL * kTileRows;
  const long long n_pairs = (Lq + rows_per_unit - 1) / rows_per_unit;
  const long long base_units = n_pairs * B * Hq;
  // keys past kv_offset + Lq are invisible to every row under masks 1 and 2
  const int kv_limit = (causal == ATTN_MASK_NONE) ? Lk : kv_offset + Lq;
  const int total_tiles = (kv_limit + kTileRows - 1) / kTileRows;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return ATTN_ERR_CUDA;
  const DeviceInfo di = device_info(dev);
  if (!di.ok) return ATTN_ERR_CUDA;
  if (!di.sm100) return ATTN_ERR_UNSUPPORTED;
  int ns = 1, per = total_tiles;
  choose_splits(n_splits, total_tiles, base_units, di.num_sms, &ns, &per, causal == ATTN_MASK_CAUSAL);
  if (fit) {
    if (n_splits > 0 && ns > 1 && attn_splitkv_workspace_bytes(B, Lq, Hq, d, ns) > workspace_bytes)
      return ATTN_ERR_SCRATCH_LIMIT;
    while (ns > 1 && attn_splitkv_workspace_bytes(B, Lq, Hq, d, ns) > workspace_bytes) {
      per = (total_tiles + ns - 2) / (ns - 1);
      ns = (total_tiles + per - 1) / per;
    }
  }
  if (splits_used != nullptr) *splits_used = ns;
  if (ns == 1)
    return attn_fwd(q, k, v, o, lse, B, Lq, Lk, Hq, Hkv, d, scale, causal, kv_offset, dtype, stream);
  const size_t need = attn_splitkv_workspace_bytes(B, Lq, Hq, d, ns);
  if (workspace == nullptr || workspace_bytes < need) return ATTN_ERR_INVALID_ARG;
  // float32 partial rows of max(d, 64) columns (d = 16, 32 run the 64-wide kernel), then the LSEs
  const size_t o_elems = static_cast<size_t>(ns) * B * Hq * Lq * (d < 64 ? 64 : d);
  if (ranges_overlap(workspace, need, q, 2ull * B * Lq * Hq * d) ||
      ranges_overlap(workspace, need, k, 2ull * B * Lk * Hkv * d) ||
      ranges_overlap(workspace, need, v, 2ull * B * Lk * Hkv * d) ||
      ranges_overlap(workspace, need, o, 2ull * B * Lq * Hq * d) ||
      (lse != nullptr && ranges_overlap(workspace, need, lse, 4ull * B * Hq * Lq)))
    return ATTN_ERR_INVALID_ARG;
  if (base_units * ns > 0x7fffffffLL) return ATTN_ERR_INVALID_ARG;

  FwdParams p{};
  p.d = d;
  p.o = o;
  p.lse = lse;
  p.B = B; p.Lq = Lq; p.Lk = Lk; p.Hq = Hq; p.Hkv = Hkv; p.group = Hq / Hkv;
  p.kv_offset = kv_offset;
  p.kv_limit = kv_limit;
  p.n_pairs = static_cast<int>(n_pairs);
  p.n_units = static_cast<int>(base_units * ns);
  p.sl2 = scale * kLog2e;
  p.timeout_ns = g_timeout_ns.load();
  p.n_splits = ns;
  p.split_tiles = per;
  p.o_part = workspace;
  p.lse_part = workspace + o_elems;
  p.win_left = p.win_right = -1;
  const int grid = static_cast<int>(p.n_units < di.num_sms ? p.n_units : di.num_sms);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const bool bf16 = dtype == ATTN_DTYPE_BF16;
  int st;
  const bool cz = causal == ATTN_MASK_CAUSAL;
  if (d == 256) {
    if (bf16)
      st = cz ? launch_fwd<256, true, true, true>(p, q, k, v, Lk, grid, s)
              : launch_fwd<256, true, false, true>(p, q, k, v, Lk, grid, s);
    else
      st = cz ? launch_fwd<256, false, true, true>(p, q, k, v, Lk, grid, s)
              : launch_fwd<256, false, false, true>(p, q, k, v, Lk, grid, s);
  } else if (d == 128) {
    if (bf16)
      st = cz ? launch_fwd<128, true, true, true>(p, q, k, v, Lk, grid, s)
              : launch_fwd<128, true, false, true>(p, q, k, v, Lk, grid, s);
    else
      st = cz ? launch_fwd<128, false, true, true>(p, q, k, v, Lk, grid, s)
              : launch_fwd<128, false, false, true>(p, q, k, v, Lk, grid, s);
  } else {
    if (bf16)
      st = cz ? launch_fwd<64, true, true, true>(p, q, k, v, Lk, grid, s)
              : launch_fwd<64, true, false, true>(p, q, k, v, Lk, grid, s);
    else
      st = cz ? launch_fwd<64, false, true, true>(p, q, k, v, Lk, grid, s)
              : launch_fwd<64, false, false, true>(p, q, k, v, Lk, grid, s);
  }
  if (st != ATTN_OK) return st;
  const long long rows = 1LL * B * Hq * Lq;
  const unsigned mgrid = static_cast<unsigned>((rows * 32 + 255) / 256);
  if (d == 256) {
    if (bf16) split_merge_kernel<256, true><<<mgrid, 256, 0, s>>>(p.o_part, p.lse_part, o, lse, ns, B, Lq, Hq, d);
    else split_merge_kernel<256, false><<<mgrid, 256, 0, s>>>(p.o_part, p.lse_part, o, lse, ns, B, Lq, Hq, d);
  } else if (d == 128) {
    if (bf16) split_merge_kernel<128, true><<<mgrid, 256, 0, s>>>(p.o_part, p.lse_part, o, lse, ns, B, Lq, Hq, d);
    else split_merge_kernel<128, false><<<mgrid, 256, 0, s>>>(p.o_part, p.lse_part, o, lse, ns, B, Lq, Hq, d);
  } else {
    if (bf16) split_merge_kernel<64, true><<<mgrid, 256, 0, s>>>(p.o_part, p.lse_part, o, lse, ns, B, Lq, Hq, d);
    else split_merge_kernel<64, false><<<mgrid, 256, 0, s>>>(p.o_part, p.lse_part, o, lse, ns, B, Lq, Hq, d);
  }
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}



// ------------------------------------------------------ host-buffer pipeline

// attn_fwd_host's copies overlap the attention. The call is cut into at most
// kHostChunks chunks of at least kHostChunkMinBytes of Q each (a smaller one
// would cost more in launches and copy calls than its overlap saves): whole
// batches per chunk when there are at least as many batches as chunks, else
// every batch cut into row ranges of whole 256-row pairs (the kernel's unit).
// Per chunk the H2D stream copies the K and V of its batches (once per
// batch) and its Q rows; its forward starts on the caller's stream once they
// have landed, and its O (and LSE) go back on the D2H stream while the next
// chunk computes. Events order the three streams, and the caller's stream
// waits for the last copy, so synchronizing it covers the whole call. The
// streams and events are created once per device and reused (calls on one
// device are serialized by a mutex while they are queued).
constexpr int kHostChunks = 16;
constexpr size_t kHostChunkMinBytes = size_t(2) << 20;

struct HostPipe {
  cudaStream_t h2d = nullptr, d2h = nullptr;
  cudaEvent_t start = nullptr, done = nullptr;
  cudaEvent_t q_in[kHostChunks] = {}, fwd_done[kHostChunks] = {};
  std::mutex m;
};

HostPipe* host_pipe(int dev) {
  static HostPipe pipes[kMaxDevices];
  static std::once_flag flags[kMaxDevices];
  static bool ok[kMaxDevices];
  if (dev < 0 || dev >= kMaxDevices) return nullptr;
  std::call_once(flags[dev], [dev]() {
    HostPipe& hp = pipes[dev];
    bool good = cudaStreamCreateWithFlags(&hp.h2d, cudaStreamNonBlocking) == cudaSuccess &&
                cudaStreamCreateWithFlags(&hp.d2h, cudaStreamNonBlocking) == cudaSuccess &&
                cudaEventCreateWithFlags(&hp.start, cudaEventDisableTiming) == cudaSuccess &&
                cudaEventCreateWithFlags(&hp.done, cudaEventDisableTiming) == cudaSuccess;
    for (int c = 0; c < kHostChunks && good; ++c)
      good = cudaEventCreateWithFlags(&hp.q_in[c], cudaEventDisableTiming) == cudaSuccess &&
             cudaEventCreateWithFlags(&hp.fwd_done[c], cudaEventDisableTiming) == cudaSuccess;
    ok[dev] = good;
  });
  return ok[dev] ? &pipes[dev] : nullptr;
}

// One chunk of attn_fwd_host: batches [b0, b0 + nb), query rows [r0, r0 + n)
// of each (nb > 1 only with whole batches: r0 = 0, n = Lq).
struct HostChunk {
  int b0, nb, r0, n;
};

// The chunks of a call (host logic only; exported for tests through
// attn_host_chunks). Returns their number, at most kHostChunks.
int host_chunks(int B, int Lq, int Hq, int d, HostChunk* out) {
  const size_t q_bytes = static_cast<size_t>(B) * Lq * Hq * d * 2;
  const size_t by_size = q_bytes / kHostChunkMinBytes;
  const int target = static_cast<int>(by_size < 1 ? 1 : (by_size > kHostChunks ? kHostChunks : by_size));
  int n = 0;
  if (target <= B) {
    const int per = (B + target - 1) / target;  // whole batches per chunk
    for (int b0 = 0; b0 < B; b0 += per) out[n++] = HostChunk{b0, std::min(per, B - b0), 0, Lq};
  } else {
    const long long per_b = target / B;        // >= 1 row ranges per batch
    const long long want = (Lq + per_b - 1) / per_b;
    const int rows = static_cast<int>(((want + 255) / 256) * 256);
    for (int b = 0; b < B; ++b)
      for (int r0 = 0; r0 < Lq; r0 += rows) out[n++] = HostChunk{b, 1, r0, std::min(rows, Lq - r0)};
  }
  return n;
}

int host_pipeline(HostPipe& hp, const void* q_host, const void* k_host, const void* v_host, void* o_host,
                  float* lse_host, void* q_dev, void* k_dev, void* v_dev, void* o_dev, float* lse_dev, int B,
                  int Lq, int Lk, int Hq, int Hkv, int d, float scale, int causal, int kv_offset, int dtype,
                  cudaStream_t s, int num_sms) {
  const size_t row_bytes = 2ull * Hq * d;      // one query row of Q or O, all heads
  const size_t kv_batch_bytes = 2ull * Lk * Hkv * d;
  HostChunk ch[kHostChunks];
  const int n_chunks = host_chunks(B, Lq, Hq, d, ch);
  // the whole call's pair-split choice, taken by every chunk (bit-identical rows)
  const long long units = static_cast<long long>(B) * Hq * ((Lq + 255) / 256);
  const int pair = causal == ATTN_MASK_CAUSAL && d <= 128 && units < num_sms ? 1 : 0;
  const auto bad = [](cudaError_t e) { return e != cudaSuccess; };
  // streams: the copies wait for everything the caller queued before this call
  if (bad(cudaEventRecord(hp.start, s)) || bad(cudaStreamWaitEvent(hp.h2d, hp.start, 0)) ||
      bad(cudaStreamWaitEvent(hp.d2h, hp.start, 0)))
    return ATTN_ERR_CUDA;
  for (int c = 0; c < n_chunks; ++c) {
    const HostChunk& x = ch[c];
    if (x.r0 == 0) {  // first chunk of its batches: their K and V
      const size_t off = static_cast<size_t>(x.b0) * kv_batch_bytes, len = x.nb * kv_batch_bytes;
      if (bad(cudaMemcpyAsync(static_cast<char*>(k_dev) + off, static_cast<const char*>(k_host) + off, len,
                              cudaMemcpyHostToDevice, hp.h2d)) ||
          bad(cudaMemcpyAsync(static_cast<char*>(v_dev) + off, static_cast<const char*>(v_host) + off, len,
                              cudaMemcpyHostToDevice, hp.h2d)))
        return ATTN_ERR_CUDA;
    }
    const size_t off = (static_cast<size_t>(x.b0) * Lq + x.r0) * row_bytes;
    const size_t len = static_cast<size_t>(x.nb) * x.n * row_bytes;
    if (bad(cudaMemcpyAsync(static_cast<char*>(q_dev) + off, static_cast<const char*>(q_host) + off, len,
                            cudaMemcpyHostToDevice, hp.h2d)) ||
        bad(cudaEventRecord(hp.q_in[c], hp.h2d)))
      return ATTN_ERR_CUDA;
  }
  for (int c = 0; c < n_chunks; ++c) {
    const HostChunk& x = ch[c];
    const size_t qo = (static_cast<size_t>(x.b0) * Lq + x.r0) * Hq * d;     // elements
    const size_t kvo = static_cast<size_t>(x.b0) * Lk * Hkv * d;
    // this chunk's LSE: [nb, Hq, n] floats at the chunk's place in its batches' LSE area
    float* lse_c = lse_dev == nullptr ? nullptr : lse_dev + static_cast<size_t>(x.b0) * Hq * Lq +
                                                      static_cast<size_t>(x.nb) * Hq * x.r0;
    // masks for a row range [r0, r0 + n): causal rows see j <= kv_offset + r (offset moves with r0);
    // chunk rows see every key below kv_offset + Lq (no mask over that key prefix)
    int mask = causal, off = kv_offset, lk = Lk;
    if (causal == ATTN_MASK_CAUSAL) {
      off = kv_offset + x.r0;
    } else if (causal == ATTN_MASK_CHUNK) {
      mask = ATTN_MASK_NONE;
      off = 0;
      lk = kv_offset + Lq;
    }
    if (bad(cudaStreamWaitEvent(s, hp.q_in[c], 0))) return ATTN_ERR_CUDA;
    const int st = attn_fwd_impl(static_cast<const uint16_t*>(q_dev) + qo, static_cast<const uint16_t*>(k_dev) + kvo,
                                 static_cast<const uint16_t*>(v_dev) + kvo, static_cast<uint16_t*>(o_dev) + qo, lse_c,
                                 x.nb, x.n, lk, Lk, Hq, Hkv, d, scale, mask, off, dtype, s, false, -1, -1, pair);
    if (st != ATTN_OK) return st;
    if (bad(cudaEventRecord(hp.fwd_done[c], s)) || bad(cudaStreamWaitEvent(hp.d2h, hp.fwd_done[c], 0)) ||
        bad(cudaMemcpyAsync(static_cast<char*>(o_host) + qo * 2, static_cast<const char*>(o_dev) + qo * 2,
                            static_cast<size_t>(x.nb) * x.n * row_bytes, cudaMemcpyDeviceToHost, hp.d2h)))
      return ATTN_ERR_CUDA;
    if (lse_host != nullptr &&
        bad(cudaMemcpy2DAsync(lse_host + static_cast<size_t>(x.b0) * Hq * Lq + x.r0, static_cast<size_t>(Lq) * 4,
                              lse_c, static_cast<size_t>(x.n) * 4, static_cast<size_t>(x.n) * 4,
                              static_cast<size_t>(x.nb) * Hq, cudaMemcpyDeviceToHost, hp.d2h)))
      return ATTN_ERR_CUDA;
  }
  // the caller's stream covers the whole call
  if (bad(cudaEventRecord(hp.done, hp.d2h)) || bad(cudaStreamWaitEvent(s, hp.done, 0))) return ATTN_ERR_CUDA;
  return ATTN_OK;
}

}  // namespace hasb

extern "C" {

int attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Lq,
             int Lk, int Hq, int Hkv, int d, float scale, int causal, int kv_offset, int dtype,
             void* stream) {
  return attn_fwd_impl(q, k, v, o, lse, B, Lq, Lk, Lk, Hq, Hkv, d, scale, causal, kv_offset, dtype,
                       stream);
}

int attn_fwd_window(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Lq,
                    int Lk, int Hq, int Hkv, int d, float scale, int window_left, int window_right,
                    int kv_offset, int dtype, void* stream) {
  return attn_fwd_impl(q, k, v, o, lse, B, Lq, Lk, Lk, Hq, Hkv, d, scale, ATTN_MASK_NONE, kv_offset,
                       dtype, stream, true, window_left, window_right);
}

}  // extern "C"

namespace hasb {

// Both e4m3 entry points: unscaled (sq == sk == nullptr) and per-token scaled.
int fp8_fwd(const void* q8, const void* k8, const void* vt8, const float* sq, const float* sk,
            const float* sv, int sq_pitch, int sk_pitch, void* o, float* lse, int B, int Lq, int Lk,
            int vt_pitch, int Hq, int Hkv, int d, float scale, int causal, int kv_offset, void* stream,
            bool scaled) {
  // ---- argument contract (no CUDA call before it passes)
  if (q8 == nullptr || k8 == nullptr || vt8 == nullptr || o == nullptr) return ATTN_ERR_INVALID_ARG;
  if (B < 1 || Lq < 1 || Lk < 1 || Hq < 1 || Hkv < 1 || Hq % Hkv != 0) return ATTN_ERR_INVALID_ARG;
  if (d < 16 || d > 256 || (d & (d - 1)) != 0) return ATTN_ERR_INVALID_ARG;
  if (!std::isfinite(scale) || scale < 0.f) return ATTN_ERR_INVALID_ARG;
  if (causal != ATTN_MASK_NONE && causal != ATTN_MASK_CAUSAL && causal != ATTN_MASK_CHUNK)
    return ATTN_ERR_INVALID_ARG;
  if (causal == ATTN_MASK_NONE ? kv_offset != 0
                               : (kv_offset < 0 || static_cast<long long>(kv_offset) + Lq > Lk))
    return ATTN_ERR_INVALID_ARG;
  if (vt_pitch < Lk || vt_pitch % 16 != 0) return ATTN_ERR_INVALID_ARG;
  const auto a16 = [](const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15u) == 0; };
  if (!a16(q8) || !a16(k8) || !a16(vt8) || !a16(o) || (reinterpret_cast<uintptr_t>(lse) & 3u) != 0)
    return ATTN_ERR_INVALID_ARG;
  const unsigned long long q_elems = 1ull * B * Lq * Hq * d, k_elems = 1ull * B * Lk * Hkv * d;
  const unsigned long long vt_bytes = 1ull * B * Hkv * d * vt_pitch;
  if (q_elems * 2 >= (1ull << 40) || k_elems >= (1ull << 40) || vt_bytes >= (1ull << 40))
    return ATTN_ERR_INVALID_ARG;
  const long long rows_per_unit = d == 256 ? kTileRows : 2LL * kTileRows;  // one tile per unit at 256
  const long long n_pairs = (Lq + rows_per_unit - 1) / rows_per_unit;
  const long long n_units = n_pairs * B * Hq;
  if (n_units > 0x7fffffffLL) return ATTN_ERR_INVALID_ARG;
  if (ranges_overlap(o, q_elems * 2, q8, q_elems) || ranges_overlap(o, q_elems * 2, k8, k_elems) ||
      ranges_overlap(o, q_elems * 2, vt8, vt_bytes))
    return ATTN_ERR_INVALID_ARG;
  if (scaled) {
    if (sq == nullptr || sk == nullptr) return ATTN_ERR_INVALID_ARG;
    if (sq_pitch < Lq || sk_pitch < Lk || sk_pitch % 4 != 0) return ATTN_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(sq) & 3u) != 0 || !a16(sk) || (sv != nullptr && !a16(sv)))
      return ATTN_ERR_INVALID_ARG;
    const unsigned long long sq_bytes = 4ull * B * Hq * sq_pitch, sk_bytes = 4ull * B * Hkv * sk_pitch;
    if (sq_bytes >= (1ull << 40) || sk_bytes >= (1ull << 40)) return ATTN_ERR_INVALID_ARG;
    if (ranges_overlap(o, q_elems * 2, sq, sq_bytes) || ranges_overlap(o, q_elems * 2, sk, sk_bytes) ||
        (sv != nullptr && ranges_overlap(o, q_elems * 2, sv, 4ull * B * Hkv * d)))
      return ATTN_ERR_INVALID_ARG;
  }
  // d < 128 runs the 128-wide kernel on zero-filled columns; 256 the one-tile kernel (unscaled only)
  // ---- device
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return ATTN_ERR_CUDA;
  const DeviceInfo di = device_info(dev);
  if (!di.ok) return ATTN_ERR_CUDA;
  if (!di.sm100) return ATTN_ERR_UNSUPPORTED;
  FwdParams p{};
  p.d = d;
  p.o = o;
  p.lse = lse;
  p.B = B; p.Lq = Lq; p.Lk = Lk; p.Hq = Hq; p.Hkv = Hkv; p.group = Hq / Hkv;
  p.kv_offset = kv_offset;
  p.kv_limit = (causal == ATTN_MASK_CHUNK) ? kv_offset + Lq : Lk;
  p.n_pairs = static_cast<int>(n_pairs);
  p.n_units = static_cast<int>(n_units);
  p.sl2 = scale * kLog2e;
  p.timeout_ns = g_timeout_ns.load();
  p.n_splits = 1;
  p.split_tiles = (p.kv_limit + kTileRows - 1) / kTileRows;
  p.o_part = nullptr;
  p.lse_part = nullptr;
  p.win_left = p.win_right = -1;
  p.sq = sq;
  p.sk = sk;
  p.sv = sv;
  p.sq_pitch = sq_pitch;
  p.sk_pitch = sk_pitch;
  const int grid = static_cast<int>(n_units < di.num_sms ? n_units : di.num_sms);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const bool c = causal == ATTN_MASK_CAUSAL;
  if (d == 256 && scaled)
    return c ? launch_fwd<256, true, true, false, false, 2>(p, q8, k8, vt8, vt_pitch, grid, s)
             : launch_fwd<256, true, false, false, false, 2>(p, q8, k8, vt8, vt_pitch, grid, s);
  if (d == 256)
    return c ? launch_fwd<256, true, true, false, false, 1>(p, q8, k8, vt8, vt_pitch, grid, s)
             : launch_fwd<256, true, false, false, false, 1>(p, q8, k8, vt8, vt_pitch, grid, s);
  if (scaled)
    return c ? launch_fwd<128, true, true, false, false, 2>(p, q8, k8, vt8, vt_pitch, grid, s)
             : launch_fwd<128, true, false, false, false, 2>(p, q8, k8, vt8, vt_pitch, grid, s);
  return c ? launch_fwd<128, true, true, false, false, 1>(p, q8, k8, vt8, vt_pitch, grid, s)
           : launch_fwd<128, true, false, false, false, 1>(p, q8, k8, vt8, vt_pitch, grid, s);
}

}  // namespace hasb

extern "C" {

int attn_fwd_fp8(const void* q8, const void* k8, const void* vt8, void* o, float* lse, int B, int Lq,
                 int Lk, int vt_pitch, int Hq, int Hkv, int d, float scale, int causal, int kv_offset,
                 void* stream) {
  return hasb::fp8_fwd(q8, k8, vt8, nullptr, nullptr, nullptr, 0, 0, o, lse, B, Lq, Lk, vt_pitch, Hq,
                       Hkv, d, scale, causal, kv_offset, stream, false);
}

int attn_fwd_fp8_scaled(const void* q8, const void* k8, const void* vt8, const float* sq,
                        const float* sk, const float* sv, void* o, float* lse, int B, int Lq, int Lk,
                        int vt_pitch, int sq_pitch, int sk_pitch, int Hq, int Hkv, int d, float scale,
                        int causal, int kv_offset, void* stream) {
  return hasb::fp8_fwd(q8, k8, vt8, sq, sk, sv, sq_pitch, sk_pitch, o, lse, B, Lq, Lk, vt_pitch, Hq,
                       Hkv, d, scale, causal, kv_offset, stream, true);
}

int attn_fwd_cache(const void* q, const void* k_cache, const void* v_cache, void* o, float* lse,
                   int B, int Lq, int Lk, int S, int Hq, int Hkv, int d, float scale, int causal,
                   int kv_offset, int dtype, void* stream) {
  if (S < 1) return ATTN_ERR_INVALID_ARG;
  return attn_fwd_impl(q, k_cache, v_cache, o, lse, B, Lq, Lk, S, Hq, Hkv, d, scale, causal,
                       kv_offset, dtype, stream);
}

size_t attn_splitkv_workspace_bytes(int B, int Lq, int Hq, int d, int n_splits) {
  if (B < 1 || Lq < 1 || Hq < 1 || d < 1 || n_splits < 1) return 0;
  const size_t dp = d < 64 ? 64 : static_cast<size_t>(d);  // d = 16, 32 run with 64-column partials
  return static_cast<size_t>(n_splits) * B * Hq * Lq * (dp + 1) * sizeof(float);
}

int attn_fwd_splitkv(const void* q, const void* k, const void* v, void* o, float* lse,
                     float* workspace, size_t workspace_bytes, int n_splits, int B, int Lq, int Lk,
                     int Hq, int Hkv, int d, float scale, int causal, int kv_offset, int dtype,
                     int* splits_used, void* stream) {
  const int valid = splitkv_validate(q, k, v, o, lse, n_splits, B, Lq, Lk, Hq, Hkv, d, scale, causal,
                                     kv_offset, dtype);
  if (valid != ATTN_OK) return valid;
  if (workspace != nullptr && (reinterpret_cast<uintptr_t>(workspace) & 15u) != 0)
    return ATTN_ERR_INVALID_ARG;
  return splitkv_run(q, k, v, o, lse, workspace, workspace_bytes, false, n_splits, B, Lq, Lk, Hq, Hkv,
                     d, scale, causal, kv_offset, dtype, splits_used, stream);
}

int attn_fwd_splitkv_static(const void* q, const void* k, const void* v, void* o, float* lse,
                            int n_splits, int B, int Lq, int Lk, int Hq, int Hkv, int d, float scale,
                            int causal, int kv_offset, int dtype, int* splits_used, void* stream) {
  const int valid = splitkv_validate(q, k, v, o, lse, n_splits, B, Lq, Lk, Hq, Hkv, d, scale, causal,
                                     kv_offset, dtype);
  if (valid != ATTN_OK) return valid;
  float* ws = nullptr;
  const int st = static_scratch(&ws);
  if (st != ATTN_OK) return st;
  return splitkv_run(q, k, v, o, lse, ws, sizeof(g_split_scratch), true, n_splits, B, Lq, Lk, Hq, Hkv, d,
                     scale, causal, kv_offset, dtype, splits_used, stream);
}

int attn_fwd_host(const void* q_host, const void* k_host, const void* v_host, void* o_host,
                  float* lse_host, void* q_dev, void* k_dev, void* v_dev, void* o_dev,
                  float* lse_dev, int B, int Lq, int Lk, int Hq, int Hkv, int d, float scale,
                  int causal, int kv_offset, int dtype, void* stream) {
  if (!q_host || !k_host || !v_host || !o_host) return ATTN_ERR_INVALID_ARG;
  if ((lse_host == nullptr) != (lse_dev == nullptr)) return ATTN_ERR_INVALID_ARG;
  if (B < 1 || Lq < 1 || Lk < 1 || Hq < 1 || Hkv < 1 || d < 1) return ATTN_ERR_INVALID_ARG;
  // the device side's contract first: no copy is queued for a call attn_fwd would refuse
  const int pre = attn_fwd_validate(q_dev, k_dev, v_dev, o_dev, lse_dev, B, Lq, Lk, Hq, Hkv, d, scale,
                                    causal, kv_offset, dtype, Lk);
  if (pre != ATTN_OK) return pre;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return ATTN_ERR_CUDA;
  const DeviceInfo di = device_info(dev);
  if (!di.ok) return ATTN_ERR_CUDA;
  HostPipe* hp = host_pipe(dev);
  if (hp == nullptr) return ATTN_ERR_CUDA;
  std::lock_guard<std::mutex> lock(hp->m);
  return host_pipeline(*hp, q_host, k_host, v_host, o_host, lse_host, q_dev, k_dev, v_dev, o_dev, lse_dev, B,
                       Lq, Lk, Hq, Hkv, d, scale, causal, kv_offset, dtype, s, di.num_sms);
}

int attn_host_chunks(int B, int Lq, int Hq, int d, int* plan) {
  if (plan == nullptr || B < 1 || Lq < 1 || Hq < 1 || d < 1) return -ATTN_ERR_INVALID_ARG;
  hasb::HostChunk ch[hasb::kHostChunks];
  const int n = hasb::host_chunks(B, Lq, Hq, d, ch);
  for (int c = 0; c < n; ++c) {
    plan[4 * c] = ch[c].b0;
    plan[4 * c + 1] = ch[c].nb;
    plan[4 * c + 2] = ch[c].r0;
    plan[4 * c + 3] = ch[c].n;
  }
  return n;
}

int attn_device_fault(unsigned int* bits, int clear) {
  if (bits == nullptr) return ATTN_ERR_INVALID_ARG;
  if (cudaDeviceSynchronize() != cudaSuccess) return ATTN_ERR_CUDA;
  unsigned int b = 0;
  if (cudaMemcpyFromSymbol(&b, g_fault_bits, sizeof(b)) != cudaSuccess) return ATTN_ERR_CUDA;
  if (clear) {
    const unsigned int zero = 0;
    if (cudaMemcpyToSymbol(g_fault_bits, &zero, sizeof(zero)) != cudaSuccess) return ATTN_ERR_CUDA;
  }
  *bits = b;
  return b ? ATTN_ERR_TIMEOUT : ATTN_OK;
}

}  // extern "C"

// the debug site words of the other kernel files of the library
namespace hasb_pro {
unsigned int debug_site_read(bool clear);
}
namespace hasb_f8 {
unsigned int debug_site_read(bool clear);
}

extern "C" {

int attn_debug_fault_site(unsigned int* site, int clear) {
  if (site == nullptr) return ATTN_ERR_INVALID_ARG;
  if (cudaDeviceSynchronize() != cudaSuccess) return ATTN_ERR_CUDA;
  unsigned int a = 0;
  if (cudaMemcpyFromSymbol(&a, g_debug_site, sizeof(a)) != cudaSuccess) return ATTN_ERR_CUDA;
  if (clear) {
    const unsigned int zero = 0;
    if (cudaMemcpyToSymbol(g_debug_site, &zero, sizeof(zero)) != cudaSuccess) return ATTN_ERR_CUDA;
  }
  const unsigned int b = hasb_pro::debug_site_read(clear != 0), c = hasb_f8::debug_site_read(clear != 0);
  *site = a != 0 ? a : (b != 0 ? b : c);
  return ATTN_OK;
}

int attn_debug_build(void) {
#ifdef ATTN_DEBUG
  return 1;
#else
  return 0;
#endif
}

int attn_selftest_mma(const void* q, const void* k, const void* v, float* s_out, float* o_out,
                      int dtype, void* stream) {
  if (!q || !k || !v || !s_out || !o_out) return ATTN_ERR_INVALID_ARG;
  if (dtype != ATTN_DTYPE_BF16 && dtype != ATTN_DTYPE_FP16) return ATTN_ERR_INVALID_ARG;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return ATTN_ERR_CUDA;
  const DeviceInfo di = device_info(dev);
  if (!di.ok) return ATTN_ERR_CUDA;
  if (!di.sm100) return ATTN_ERR_UNSUPPORTED;
  const bool bf16 = dtype == ATTN_DTYPE_BF16;
  CUtensorMap tq, tk, tv;
  if (!encode_bl_hd(&tq, q, 1, 128, 1, 128, bf16) || !encode_bl_hd(&tk, k, 1, 128, 1, 128, bf16) ||
      !encode_bl_hd(&tv, v, 1, 128, 1, 128, bf16))
    return ATTN_ERR_CUDA;
  const int smem = 3 * Cfg<128>::kTileBytes + 128 + 1024;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  auto kern = bf16 ? selftest_mma_kernel<true> : selftest_mma_kernel<false>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return ATTN_ERR_CUDA;
  kern<<<1, 128, smem, s>>>(tq, tk, tv, s_out, o_out, g_timeout_ns.load());
  if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return ATTN_ERR_CUDA;
  unsigned int bits = 0;
  return attn_device_fault(&bits, 1);
}

int attn_selftest_exp2(const float* x, float* y, int n, void* stream) {
  if (x == nullptr || y == nullptr || n < 0) return ATTN_ERR_INVALID_ARG;
  if (n == 0) return ATTN_OK;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int pairs = (n + 1) / 2;
  selftest_exp2_kernel<<<(pairs + 255) / 256, 256, 0, s>>>(x, y, n);
  if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
  return cudaStreamSynchronize(s) == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

int attn_selftest_wait_timeout(unsigned long long timeout_ns, void* stream) {
  if (timeout_ns < 1000000ull || timeout_ns > 10000000000ull) return ATTN_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  unsigned int bits = 0;
  int st = attn_device_fault(&bits, 1);  // start from a clear word
  if (st == ATTN_ERR_CUDA) return st;
  selftest_timeout_kernel<<<1, 32, 0, s>>>(timeout_ns);
  if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return ATTN_ERR_CUDA;
  return attn_device_fault(&bits, 1);
}

}  // extern "C"
