// tc_common.cuh -- constants, kernel arguments and small device helpers
// shared by the tensor-core scoring kernels (tc.cu: pass 1, combine, the
// single-CTA second pass; tc_pair.cu: the CTA-pair second pass).
#pragma once

#include <cuda.h>
#include <math.h>

#include "common.cuh"
#include "internal.h"
#include "tc_ptx.cuh"

namespace dropkv {

// Arguments of the tensor-core kernels (one batch slice), passed by value.
struct TcArgs {
  int32_t B, Hq, Hkv, n_max, w, G, nqc, chunks;   // single-CTA pass 2: chunks of nqc <= 128
  int32_t nq;            // query rows per KV head (G * w)
  int32_t chunks1, rows1;  // pass 1: query chunks of rows1 <= 256 rows (two tiles)
  int32_t qbox_rows;     // rows of the pass-1 Q box: min(128, all query rows)
  int32_t L[kMaxB];
  int32_t splits[kMaxB];     // pass 2
  int32_t cta_base[kMaxB + 1];
  int32_t splits1[kMaxB];    // pass 1
  int32_t cta_base1[kMaxB + 1];
  int32_t chunks2, nqc2;     // pair pass 2: query chunks of nqc2 <= 256 rows
  int32_t splits2[kMaxB];    // pair pass 2, in CTA pairs
  int32_t cta_base2[kMaxB + 1];
  float c_log2;          // log2(e) / sqrt(d)
  const __nv_bfloat16* q;  // [rows][128] window queries
  float* partial;        // [pass-1 ctas][rows1][kPartStride]
  int32_t* status;
  __nv_bfloat16* ahi;    // [rows][128]
  __nv_bfloat16* alo;    // [rows][128]
  float4* qstat;         // [rows]: (M, 1/L, L, ||A||^2)
  float* attn_user;      // optional [rows][128]
  float* stats_user;     // optional [rows][2]
  float* parts;          // [chunks][B*Hkv*n_max]
  size_t part_stride;
  float* attn_f32;       // [rows][128] fp32 window outputs a (read back by pass 2)
  const __nv_bfloat16* v;  // [B*Hkv][n_max][128] values (rare direct-distance path)
  float* nvbuf;          // [B*Hkv][ntmax*128] ||v_j||^2 (pass 1 -> pass 2), tile-padded rows
  float* tmin;           // [B*Hkv][ntmax][chunks1] min ||v_j||^2 over a pass-1 chunk's share
  int32_t ntmax;         // ceil(n_max / 128)
};

namespace {

using namespace tc;

constexpr int kTok = 128;          // tokens per tile
constexpr int kHd = 128;           // head dim
constexpr int kBox = 128 * 128;    // bytes of a 128-row x 64-col bf16 box (SW128)
constexpr int kTileBytes = 2 * kBox;
constexpr int kSimtWarps = 16;     // pass-2 score warps: 4 per TMEM lane quarter
constexpr int kWarpTma = kSimtWarps, kWarpMma = kSimtWarps + 1;
constexpr int kThreads2 = (kSimtWarps + 2) * 32;  // pass 2: + TMA warp, MMA warp
constexpr int kMaxRegs2 = 96;      // second passes at launch: 5 warps on a sub-partition (16K registers)
// pass 1: two softmax warpgroups (one per 128-row query tile, one row per
// thread), TMA warps for Q/K and for V, an MMA warp and a ||v||^2 warp
constexpr int kSmWarps1 = 8;
constexpr int kW1Tma = 8, kW1Mma = 9, kW1Nv = 10, kW1TmaV = 11;
constexpr int kThreads1 = 12 * 32;
constexpr int kRegs1 = 168;        // pass 1's registers a thread at launch (65536 / 384, rounded down to 8)
constexpr uint32_t kColO1 = 256;   // pass-1 TMEM: S/P of tile t at 128 t, O of tile t at 256 + 128 t
constexpr uint64_t kWaitNs = 2000000000ull;
constexpr int kPartStride = kTcPartStride;  // floats per partial row: O[128], m, l, pad
constexpr int kMaxCtas = 160;      // split target ceiling (one CTA per SM)
constexpr int kSt1 = 3;            // pass-1 V stages
constexpr int kStK = 2;            // pass-1 K stages
constexpr int kBars1 = 1 + 2 * kStK + 2 * kSt1 + 6;  // pass-1 mbarriers
constexpr int kRing2 = 5;          // attention-only pass 2: ring of 32 KB K slots
constexpr float kLoSkip = 8e-4f;   // pass 2 drops A_lo when ||A||^2 <= kLoSkip ||v||^2 throughout


__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float f32(uint32_t u) { return __uint_as_float(u); }
__device__ __forceinline__ uint32_t u32(float f) { return __float_as_uint(f); }
__device__ __forceinline__ uint32_t pack_bf16_rn(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// (b, h, query chunk, token tiles [t0, t1)) of CTA `cta` for a split plan.
__device__ __forceinline__ void decode_plan(const TcArgs& a, const int32_t* splits,
                                            const int32_t* cta_base, int chunks, int cta, int& b,
                                            int& h, int& chunk, int& t0, int& t1) {
  b = 0;
  while (b + 1 < a.B && cta >= cta_base[b + 1]) ++b;
  const int local = cta - cta_base[b];
  const int sp = local % splits[b];
  const int hc = local / splits[b];
  h = hc / chunks;
  chunk = hc % chunks;
  const int nt = (a.L[b] + kTok - 1) / kTok;
  t0 = (int)((long long)sp * nt / splits[b]);
  t1 = (int)((long long)(sp + 1) * nt / splits[b]);
}
__device__ __forceinline__ void decode_cta(const TcArgs& a, int cta, int& b, int& h, int& chunk,
                                           int& t0, int& t1) {
  decode_plan(a, a.splits, a.cta_base, a.chunks, cta, b, h, chunk, t0, t1);
}

// Records a timeout once and raises the CTA-wide abort flag.
__device__ __forceinline__ void fail(const TcArgs& a, volatile int* abort_flag) {
  *abort_flag = 1;
  atomicMax(a.status, (int)DROPKV_ERR_TIMEOUT);
}
// Bounded wait whose outcome is the same for every lane of the warp, so the
// warp stays converged for the .sync.aligned tcgen05 instructions after it.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity) {
  const bool ok = mbar_wait(bar, parity, kWaitNs);
  return __all_sync(0xffffffffu, ok);
}
__device__ __forceinline__ bool warp_aborted(volatile int* f) {
  return __any_sync(0xffffffffu, *f != 0);
}

// Descriptor-word offset of the 16-wide K slice kk of a K-major SW128 operand
// with `rows` rows (kmajor_desc's address offset >> 4).
__device__ __forceinline__ uint32_t kslice(int kk, uint32_t rows) {
  return (uint32_t)(kk >> 2) * rows * 8u + (uint32_t)(kk & 3) * 2u;
}
// =========================== second-pass scoring ===========================
// ||a - v||^2 taken directly (fp32 a, bf16 v, both from global memory).  Used
// only where the expansion ||a||^2 + ||v||^2 - 2 a.v cancels by more than 32x,
// i.e. a is close to v (a dominant token, p_j near 1).
__device__ __noinline__ float direct_sqdist(const float* A, const __nv_bfloat16* v) {
  float s = 0.f;
  for (int c = 0; c < kHd; c += 4) {
    const float4 a4 = *reinterpret_cast<const float4*>(A + c);
    const uint2 v4 = *reinterpret_cast<const uint2*>(v + c);
    const float d0 = a4.x - __uint_as_float(v4.x << 16);
    const float d1 = a4.y - __uint_as_float(v4.x & 0xFFFF0000u);
    const float d2 = a4.z - __uint_as_float(v4.y << 16);
    const float d3 = a4.w - __uint_as_float(v4.y & 0xFFFF0000u);
    s = fmaf(d0, d0, s);
    s = fmaf(d1, d1, s);
    s = fmaf(d2, d2, s);
    s = fmaf(d3, d3, s);
  }
  return s;
}

// The ratio p / (1 - p) on the fast path's interval 0 <= p < 2^-4 is p t(p),
// t the quadratic closest to 1 / (1 - p) in relative error there (minimax):
// t(p) (1 - p) - 1 is the cubic of least maximum on [0, 2^-4] that takes -1
// at p = 1, i.e. -T3(32 p - 1) / T3(31) (Chebyshev's extremal property of
// T3 outside [-1, 1]), so |p t(p) / (p / (1 - p)) - 1| <= 1 / T3(31) =
// 1 / 119071 = 8.4e-6.  t(p) = (1 - T3(32 p - 1) / T3(31)) / (1 - p) is a
// quadratic (the numerator vanishes at p = 1); kT0, kT1, kT2 are the fp32
// roundings of its coefficients.
constexpr float kT0 = 1.00000834f, kT1 = 0.997589648f, kT2 = 1.10078859f;

// Fast path for 16 query columns of one token (every p < 2^-4, no possible
// cancellation): packed fp32 pairs,
//   p = 2^(x c - M'),  M' = M + log2 L,
//   ratio = p / (1 - p) = p t(p) to 8.4e-6 relative (t above),
//   s += ratio^2 (D' + ||A||^2 + ||v||^2)   with D' = -2 A.v from the MMA.
// kf holds (-M'_t, -M'_t+1, ||A_t||^2, ||A_t+1||^2) per column pair.
// kMask: the causal window mask -- column u is the window query at position
// pbase + (m0 + u) mod w and sees the token only up to that position; a key
// it does not see gets p = 0 (the exponent is -inf).
template <bool kMask>
__device__ __forceinline__ void fast16(const uint32_t (&r)[32], const float4* kf, uint64_t c2,
                                       uint64_t nv2, uint64_t& acc2, float& pmax, int tok = 0,
                                       int pbase = 0, int m0 = 0, int w = 1) {
  int m = m0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float4 k = kf[i];
    float y0, y1;
    upk2(ffma2(pk2(f32(r[2 * i]), f32(r[2 * i + 1])), c2, pk2(k.x, k.y)), y0, y1);
    if constexpr (kMask) {
      if (tok > pbase + m) y0 = -INFINITY;
      m = m + 1 == w ? 0 : m + 1;
      if (tok > pbase + m) y1 = -INFINITY;
      m = m + 1 == w ? 0 : m + 1;
    }
    const float p0 = ex2(y0), p1 = ex2(y1);
    pmax = fmax3(pmax, p0, p1);
    const uint64_t P = pk2(p0, p1);
    const uint64_t ratio =
        fmul2(P, ffma2(P, ffma2(P, pk2(kT2, kT2), pk2(kT1, kT1)), pk2(kT0, kT0)));
    const uint64_t zt = fadd2(fadd2(pk2(f32(r[16 + 2 * i]), f32(r[16 + 2 * i + 1])),
                                    pk2(k.z, k.w)), nv2);
    acc2 = ffma2(fmul2(ratio, ratio), zt, acc2);
  }
}

// Careful path for 16 query columns of one token (r[0..15] = S^T, r[16..31] =
// D): the causal mask, ratio = e / (L - e) with the singular check when
// p >= 2^-8, and the direct squared distance where the expansion cancels by
// more than 32x.
__device__ __noinline__ float careful16(const uint32_t* r, int col0, int tok, bool masked, int L,
                                        int w, int crow0, const float4* qstat_rows, float c,
                                        float nv, const float* arows, const __nv_bfloat16* vrow,
                                        int* sing) {
  float acc = 0.f;
#pragma unroll
  for (int u = 0; u < 16; ++u) {
    const int col = col0 + u;
    const float4 k = qstat_rows[col];  // (M, 1/L, L, ||A||^2)
    const bool vis = !masked || tok <= L - w + (crow0 + col) % w;
    const float e = ex2(fmaf(f32(r[u]), c, -k.x));
    const float p = e * k.y;
    float ratio = fmaf(p, fmaf(p, p, p), p);
    const float base = k.w + nv;
    float zt = base + f32(r[16 + u]);
    if (vis && p >= 0.00390625f) {
      const float den = k.z - e;  // (1 - p) L
      if (!(den > 0.f)) *sing = 1;
      ratio = __fdiv_rn(e, den);
    }
    if (vis && zt < 0.03125f * base) zt = direct_sqdist(arows + (size_t)col * kHd, vrow);
    if (vis) acc += ratio * ratio * zt;
  }
  return acc;
}

}  // namespace
}  // namespace dropkv
