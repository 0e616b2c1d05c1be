// tc.cu -- tensor-core scoring path for bf16 inputs with head dim 128:
// tcgen05 MMAs with accumulators in TMEM, operands staged by TMA.
//
// What is computed (write-up "DropKV：精确单项输出扰动评分组件", section 核心公式):
// for every window query t of a KV head's query group, p = softmax(K q / sqrt d)
// over the causally visible keys, a = sum_j p_j v_j, and for every token j the
// perturbation weight p_j / (1 - p_j) with
//     s_j = sum_t (p_j / (1 - p_j))^2 * (||a||^2 - 2 a.v_j + ||v_j||^2)
// summed over all G*w window queries of the group (the GQA sum; the epilogue
// divides by G).  No n x w matrix is stored: two streaming passes over K/V.
//
// Work split.  The G*w query rows of a KV head are cut into `chunks` chunks of
// nqc <= 128 rows; the tokens of each (b, h, chunk) into `splits` contiguous
// tile ranges so that about one CTA runs per SM.  Tiles are 128 tokens.
//
// k_tc_pass1 (query-major, one CTA per (b, h, chunk, split)):
//   S = Q_chunk K_tile^T      tcgen05 M=128 (queries) N=128 (tokens) K=128
//   online softmax per query row (log2 domain; the reference max only moves up
//   by more than 8, so exp2 stays <= 256 and O rarely rescales).  Sixteen
//   softmax warps share every tile: each owns 32 rows x 32 tokens, posts its
//   row maxima for the other three warps of its rows and, one tile behind,
//   writes P = exp2(S*c - m) back over S in TMEM as two bf16 planes,
//   P_hi = P truncated to bf16 and P_lo = bf16(P - P_hi), so P_hi + P_lo holds
//   P to 2^-16 relative;  O += P_hi V + P_lo V   (A from TMEM, V MN-major).
//   Three S/P buffers let S run two tiles ahead of P V.  Each CTA writes one
//   partial (m, l, O) per row.
// k_tc_combine: merges the partials of a row into the final max M, normaliser
//   L and output A = O / L; writes -2A as bf16 hi/lo planes (same split) plus
//   the per-query constants (M, 1/L, L, ||A||^2) for pass 2.
// k_tc_pass2 (token-major, one CTA per (b, h, chunk, split)):
//   S^T = K_tile Q^T and D = V_tile (-2A_hi)^T [+ V_tile (-2A_lo)^T], tcgen05
//   M=128 (tokens) N=nqc (queries) K=128, into two TMEM buffers; each thread
//   owns one token and sums over its warp's 32 queries:  p = exp2(S*c - M'),
//   M' = M + log2 L; while p < 2^-4 the series p(1 + p(1 + p(1 + p(1 + p))))
//   gives p / (1 - p); otherwise ratio = e / (L - e) with the singular check
//   (L - e not > 0 => rejected); s += ratio^2 * (||A||^2 + ||v_j||^2 + D);
//   where that expansion cancels by more than 32x (A close to v_j: a dominant
//   token) the squared distance is recomputed directly from fp32 A and v_j.
//   A warp hands its TMEM buffer back once its last columns are in registers.
//   The attention-only control score (section 结果与独立对照) is the same
//   kernel instantiated with kAttn: K tiles only, S^T only, s += p.
//
// Warp roles: sixteen score / softmax warps (4 per TMEM lane quarter), one
// warp issuing TMA loads, one allocating TMEM and issuing MMAs (lane 0), and in
// pass 1 one more warp computing ||v_j||^2.  Every wait on an mbarrier is
// bounded (2 s of %globaltimer); on expiry the kernel records
// DROPKV_ERR_TIMEOUT, every role leaves its loop and TMEM is freed.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <math.h>
#include <string.h>

#include <algorithm>

#include "common.cuh"
#include "internal.h"
#include "tc_ptx.cuh"

namespace dropkv {

namespace {

using namespace tc;

constexpr int kTok = 128;          // tokens per tile
constexpr int kHd = 128;           // head dim
constexpr int kBox = 128 * 128;    // bytes of a 128-row x 64-col bf16 box (SW128)
constexpr int kTileBytes = 2 * kBox;
constexpr int kSimtWarps = 16;     // softmax / score warps: 4 per TMEM lane quarter
constexpr int kWarpTma = kSimtWarps, kWarpMma = kSimtWarps + 1, kWarpNv = kSimtWarps + 2;
constexpr int kThreads2 = (kSimtWarps + 2) * 32;  // pass 2: + TMA warp, MMA warp
constexpr int kThreads1 = (kSimtWarps + 3) * 32;  // pass 1: + the ||v||^2 warp
constexpr int kMaxRegs = 96;       // pass 1: 19 warps share the SM's 64K registers
constexpr int kMaxRegs2 = 96;      // pass 2: 18 warps, 5 on a sub-partition (16K registers)
constexpr uint32_t kColO = 384;    // pass-1 TMEM columns: three S/P buffers [0, 384), then O
constexpr uint64_t kWaitNs = 2000000000ull;
constexpr int kPartStride = 136;   // floats per partial row: O[128], m, l (4 parts), pad
constexpr int kMaxCtas = 160;      // split target ceiling (one CTA per SM)
constexpr int kSt1 = 3;            // pass-1 V stages (HBM latency needs > 1 tile in flight)
constexpr int kStK = 2;            // pass-1 K stages (S runs two tiles ahead of P V)
constexpr int kBars1 = 1 + 2 * kStK + 2 * kSt1 + 13;  // pass-1 mbarriers
constexpr int kRing2 = 5;          // pass-2 ring of 32 KB K/V slots (the last one doubles as A_lo)
constexpr float kLoSkip = 8e-4f;   // pass 2 drops A_lo when ||A||^2 <= kLoSkip ||v||^2 throughout

struct TcArgs {
  int32_t B, Hq, Hkv, n_max, w, G, nqc, chunks;
  int32_t qbox_rows;     // rows of the pass-1 Q box: min(128, all query rows)
  int32_t L[kMaxB];
  int32_t splits[kMaxB];
  int32_t cta_base[kMaxB + 1];
  float c_log2;          // log2(e) / sqrt(d)
  const __nv_bfloat16* q;  // [rows][128] window queries
  float* partial;        // [ctas][128][kPartStride]
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
  float* tmin;           // [B*Hkv][ntmax][chunks] min ||v_j||^2 over a chunk's share of a tile
  int32_t ntmax;         // ceil(n_max / 128)
};

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

__device__ __forceinline__ void decode_cta(const TcArgs& a, int cta, int& b, int& h, int& chunk,
                                           int& t0, int& t1) {
  b = 0;
  while (b + 1 < a.B && cta >= a.cta_base[b + 1]) ++b;
  const int local = cta - a.cta_base[b];
  const int sp = local % a.splits[b];
  const int hc = local / a.splits[b];
  h = hc / a.chunks;
  chunk = hc % a.chunks;
  const int nt = (a.L[b] + kTok - 1) / kTok;
  t0 = (int)((long long)sp * nt / a.splits[b]);
  t1 = (int)((long long)(sp + 1) * nt / a.splits[b]);
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
// =========================== pass 1 =========================================
// Writes P = exp2(S c - mu) for one warp's 32 tokens of a query row (S already
// in registers, masked keys at -inf) as hi/lo bf16 planes over the same 32
// TMEM columns: tokens 16k..16k+15 keep hi in columns [16k, 16k+8) and lo in
// [16k+8, 16k+16).  Returns the row's sum of P over the 32 tokens.
// Warp-collective.
__device__ __forceinline__ float p1_exp32(const uint32_t (&sr)[32], uint32_t tS, uint64_t c2,
                                          float mu) {
  const uint64_t nmu2 = pk2(-mu, -mu);
  uint64_t l2 = pk2(0.f, 0.f);
  uint32_t pw[32];  // columns: hi of tokens 0-15, lo of 0-15, hi of 16-31, lo of 16-31
#pragma unroll
  for (int half = 0; half < 2; ++half) {  // 16 tokens -> 8 hi + 8 lo columns
#pragma unroll
    for (int u2 = 0; u2 < 8; ++u2) {
      const int u = half * 16 + 2 * u2;
      float d0, d1;
      upk2(ffma2(pk2(f32(sr[u]), f32(sr[u + 1])), c2, nmu2), d0, d1);
      const float e0 = ex2(d0), e1 = ex2(d1);
      const uint64_t E = pk2(e0, e1);
      l2 = fadd2(l2, E);
      pw[half * 16 + u2] = __byte_perm(u32(e0), u32(e1), 0x7632);  // truncated bf16 pair
      const float nh0 = f32((u32(e0) & 0xFFFF0000u) | 0x80000000u);
      const float nh1 = f32((u32(e1) & 0xFFFF0000u) | 0x80000000u);
      float r0, r1;
      upk2(fadd2(E, pk2(nh0, nh1)), r0, r1);  // exact remainders e - hi
      pw[half * 16 + 8 + u2] = pack_bf16_rn(r0, r1);
    }
  }
  tmem_st32(tS, pw);  // one TMEM store for the warp's 32 columns
  float la, lb;
  upk2(l2, la, lb);
  return la + lb;
}

// Rare path of pass 1, out of line: the reference max moved for some lanes
// (factor fac <= 1 for them, 1 for the others), so this warp's 32 columns of O
// are rescaled once the P V that last accumulated into O has landed (waited on
// through that P V's buffer barrier and parity).  Warp-collective.  Returns
// false on a timeout.
__device__ __noinline__ bool p1_rescale_o(uint32_t tO, float fac, uint32_t pd_bar,
                                          uint32_t parity) {
  if (!warp_wait(pd_bar, parity)) return false;
  tc_fence_after();
  uint32_t o[32];
  tmem_ld32(tO, o);
#pragma unroll
  for (int u = 0; u < 32; ++u) o[u] = u32(f32(o[u]) * fac);
  tmem_st32(tO, o);
  return true;
}

__global__ void __maxnreg__(kMaxRegs)
k_tc_pass1(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
           const __grid_constant__ CUtensorMap tmV, const TcArgs a) {
  extern __shared__ __align__(1024) uint8_t smem[];
  uint8_t* sQ = smem;                              // 128 rows x 2 boxes
  uint8_t* sK = smem + kTileBytes;                 // kStK stages
  uint8_t* sV = sK + kStK * kTileBytes;            // kSt1 stages
  uint64_t* bars = reinterpret_cast<uint64_t*>(sV + kSt1 * kTileBytes);  // kBars1 barriers
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + kBars1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* xmax = reinterpret_cast<float*>(tmem_slot + 2);  // [3 buffers][4 groups][128]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (smem_u32(smem) & 1023u) {  // the swizzled tiles need 1 KB alignment
    if (threadIdx.x == 0) atomicMax(a.status, (int)DROPKV_ERR_CUDA);
    return;
  }
  int b, h, chunk, t0, t1;
  decode_cta(a, blockIdx.x, b, h, chunk, t0, t1);
  const int T = t1 - t0;
  const int L = a.L[b];
  // barriers: Q; K full/empty (kStK stages); V full/empty (kSt1 stages); per
  // TMEM S/P buffer: S ready, P written, tile max exchanged, P V done; O final
  const uint32_t BQ = smem_u32(&bars[0]);
  auto KF = [&](int s) { return smem_u32(&bars[1 + s]); };
  auto KE = [&](int s) { return smem_u32(&bars[1 + kStK + s]); };
  auto VF = [&](int s) { return smem_u32(&bars[1 + 2 * kStK + s]); };
  auto VE = [&](int s) { return smem_u32(&bars[1 + 2 * kStK + kSt1 + s]); };
  constexpr int kB0 = 1 + 2 * kStK + 2 * kSt1;
  auto SF = [&](int s) { return smem_u32(&bars[kB0 + s]); };
  auto PF = [&](int s) { return smem_u32(&bars[kB0 + 3 + s]); };
  auto XB = [&](int s) { return smem_u32(&bars[kB0 + 6 + s]); };
  auto PD = [&](int s) { return smem_u32(&bars[kB0 + 9 + s]); };
  const uint32_t OF = smem_u32(&bars[kB0 + 12]);  // committed once, after the last P V
  if (threadIdx.x == 0) {
    mbar_init(BQ, 1);
    mbar_init(OF, 1);
    for (int s = 0; s < kStK; ++s) {
      mbar_init(KF(s), 1); mbar_init(KE(s), 1);
    }
    for (int s = 0; s < kSt1; ++s) {
      mbar_init(VF(s), 1);
      mbar_init(VE(s), 2);  // P V commit + the ||v||^2 warp's reads
    }
    for (int s = 0; s < 3; ++s) {
      mbar_init(SF(s), 1); mbar_init(PF(s), kSimtWarps); mbar_init(XB(s), kSimtWarps);
      mbar_init(PD(s), 1);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kWarpMma) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;
  const int z = b * a.Hkv + h;
  const int qrow0 = (b * a.Hkv + h) * a.G * a.w + chunk * a.nqc;

  if (warp == kWarpTma) {
    // ---------------- TMA producer ----------------
    // order: Q, K_0, K_1, then K_{j+2} and V_j for each tile j (S runs two
    // tiles ahead of P V)
    if (lane == 0) {
      prefetch_tmap(&tmQ); prefetch_tmap(&tmK); prefetch_tmap(&tmV);
      mbar_expect_tx(BQ, 2u * 128u * (uint32_t)a.qbox_rows);
      tma_load_2d(smem_u32(sQ), &tmQ, BQ, 0, qrow0);
      tma_load_2d(smem_u32(sQ) + kBox, &tmQ, BQ, 64, qrow0);
      auto load = [&](uint8_t* buf, int nst, const CUtensorMap* m, int i, uint32_t full,
                      uint32_t empty) {
        const int ph = (i / nst) & 1;
        if (!mbar_wait(empty, ph ^ 1, kWaitNs)) { fail(a, abort_flag); return false; }
        mbar_expect_tx(full, kTileBytes);
        const uint32_t dst = smem_u32(buf + (i % nst) * kTileBytes);
        tma_load_3d(dst, m, full, 0, (t0 + i) * kTok, z);
        tma_load_3d(dst + kBox, m, full, 64, (t0 + i) * kTok, z);
        return true;
      };
      bool ok = true;
      for (int i = 0; i < 2 && i < T && ok; ++i)
        ok = load(sK, kStK, &tmK, i, KF(i % kStK), KE(i % kStK));
      for (int j = 0; j < T && ok && !*abort_flag; ++j) {
        if (j + 2 < T) ok = load(sK, kStK, &tmK, j + 2, KF((j + 2) % kStK), KE((j + 2) % kStK));
        if (ok) ok = load(sV, kSt1, &tmV, j, VF(j % kSt1), VE(j % kSt1));
      }
    }
  } else if (warp == kWarpMma) {
    // ---------------- MMA issuer ----------------
    constexpr uint32_t IDS = idesc_bf16(128, 128, false, false);   // S = Q K^T
    constexpr uint32_t IDP = idesc_bf16(128, 128, false, true);    // O += P V (V MN-major)
    bool ok = warp_wait(BQ, 0);
    if (!ok) fail(a, abort_flag);
    // operand descriptors of stage 0; a stage or K slice only moves the start
    // address, i.e. adds to the low word
    const SDesc qd = sdesc_split(smem_u32(sQ), 16, 1024);
    const SDesc kd0 = sdesc_split(smem_u32(sK), 16, 1024);
    const SDesc vd0 = sdesc_split(smem_u32(sV), kBox, 1024);
    auto issue_S = [&](int i) {
      const int s = i % kStK, ph = (i / kStK) & 1, bf = i % 3;
      if (!warp_wait(KF(s), ph)) { fail(a, abort_flag); return false; }
      // S(i) overwrites the buffer whose P the (i-3)-th P V reads from TMEM
      if (i >= 3 && !warp_wait(PD(bf), ((i - 3) / 3) & 1)) { fail(a, abort_flag); return false; }
      tc_fence_after();
      if (lane == 0) {
        const uint32_t klo = kd0.lo + (uint32_t)s * (kTileBytes >> 4);
        const uint32_t dS = tbase + (uint32_t)(bf * 128);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ss_w(dS, qd.lo + kslice(kk, 128), qd.hi, klo + kslice(kk, 128), kd0.hi, IDS,
                   kk > 0 ? 1u : 0u);
        mma_commit(KE(s));
        mma_commit(SF(bf));
      }
      __syncwarp();
      return true;
    };
    auto issue_PV = [&](int i) {
      const int s = i % kSt1, ph = (i / kSt1) & 1, bf = i % 3, bph = (i / 3) & 1;
      if (!warp_wait(PF(bf), bph)) { fail(a, abort_flag); return false; }
      if (!warp_wait(VF(s), ph)) { fail(a, abort_flag); return false; }
      uint8_t* vb = sV + s * kTileBytes;
      const int tile0 = (t0 + i) * kTok;
      if (tile0 + kTok > L) {
        // rows at or beyond L hold no data (possibly NaN): zero them so that the
        // P = 0 weights of those rows contribute exactly 0 to O
        const int r0 = L - tile0;
        for (int idx = r0 * 8 + lane; idx < kTok * 8; idx += 32) {
          const int r = idx >> 3, c16 = idx & 7;
          *reinterpret_cast<uint4*>(vb + r * 128 + c16 * 16) = make_uint4(0, 0, 0, 0);
          *reinterpret_cast<uint4*>(vb + kBox + r * 128 + c16 * 16) = make_uint4(0, 0, 0, 0);
        }
        fence_proxy_async_smem();
      }
      __syncwarp();
      tc_fence_after();
      if (lane == 0) {
        const uint32_t vlo = vd0.lo + (uint32_t)s * (kTileBytes >> 4);
        const uint32_t dO = tbase + kColO;
        const uint32_t pS = tbase + (uint32_t)(bf * 128);
        // tokens 16kk..16kk+15: P_hi in columns [16kk, 16kk+8), P_lo in [16kk+8, 16kk+16);
        // V slice kk starts 16 rows (2048 bytes) further
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ts_w(dO, pS + (uint32_t)(16 * kk), vlo + (uint32_t)kk * 128u, vd0.hi, IDP,
                   (i > 0 || kk > 0) ? 1u : 0u);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ts_w(dO, pS + (uint32_t)(16 * kk + 8), vlo + (uint32_t)kk * 128u, vd0.hi, IDP, 1u);
        mma_commit(VE(s));
        mma_commit(PD(bf));
        if (i == T - 1) mma_commit(OF);
      }
      __syncwarp();
      return true;
    };
    // tensor-pipe order: S(0), S(1), then S(j + 2), P V(j) for each j.  S(j + 2)
    // needs only P V(j - 1) done (its buffer) and goes ahead of P V(j), which
    // waits for the softmax warps, so S is ready when they reach tile j + 2.
    for (int i = 0; i < 2 && i < T && ok; ++i) ok = issue_S(i);
    for (int j = 0; j < T && ok && !warp_aborted(abort_flag); ++j) {
      if (j + 2 < T) ok = issue_S(j + 2);
      if (ok) ok = issue_PV(j);
    }
  } else if (warp == kWarpNv) {
    // ---------------- ||v_j||^2 ----------------
    // This CTA's share of every V tile's rows (the query chunks of a KV head
    // cover the same tokens and split the rows), 4 rows per lane; the order of
    // the squares is free, so the 128-byte swizzle only picks a bank-conflict-
    // free order.  Arrives on the V stage's empty barrier when done, and
    // records the share's minimum for pass 2.
    for (int j = 0; j < T; ++j) {
      const int s = j % kSt1, ph = (j / kSt1) & 1;
      if (!warp_wait(VF(s), ph)) { fail(a, abort_flag); break; }
      if (warp_aborted(abort_flag)) break;
      const uint8_t* vb = sV + s * kTileBytes;
      const int tile0 = (t0 + j) * kTok;
      float vmin = INFINITY;
      for (int rr = 0; rr < 4; ++rr) {
        const int row = rr * 32 + lane;
        if ((row * a.chunks) / 128 != chunk || tile0 + row >= L) continue;
        uint64_t acc2 = pk2(0.f, 0.f);
#pragma unroll
        for (int bx = 0; bx < 2; ++bx)
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const uint4 q4 =
                *reinterpret_cast<const uint4*>(vb + bx * kBox + row * 128 + ((q ^ (row & 7)) * 16));
            const uint32_t wv[4] = {q4.x, q4.y, q4.z, q4.w};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const uint64_t pr = pk2(f32(wv[k] << 16), f32(wv[k] & 0xFFFF0000u));
              acc2 = ffma2(pr, pr, acc2);
            }
          }
        float na, nb;
        upk2(acc2, na, nb);
        a.nvbuf[(size_t)z * a.ntmax * kTok + tile0 + row] = na + nb;
        vmin = fminf(vmin, na + nb);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(VE(s));
      vmin = warp_min(vmin);  // pass 2 decides from it whether A needs its low part
      if (lane == 0) a.tmin[((size_t)z * a.ntmax + t0 + j) * a.chunks + chunk] = vmin;
    }
  } else if (warp < kSimtWarps) {
    // ---------------- softmax warps ----------------
    // Sixteen warps work on every tile: warp (g, quarter) owns the query rows
    // [32 quarter, +32) (its TMEM lanes), the tile's tokens [32 g, 32 g + 32)
    // (its S/P columns) and O's head-dim columns [32 g, 32 g + 32).
    // Software pipelined by one tile: step j posts tile j's max for the other
    // three warps of its rows, then writes P of tile j - 1, whose maxes were
    // posted a full step earlier, so the exchange rarely waits.
    const int g = warp >> 2, ql = warp & 3;
    const int row = ql * 32 + lane;  // query row within the chunk
    const bool valid_row = row < a.nqc;
    const int Prow = valid_row ? L - a.w + (chunk * a.nqc + row) % a.w : L - 1;
    const uint32_t lane_off = (uint32_t)(ql * 32) << 16;
    const int c0 = g * 32;
    const uint32_t tO = tbase + kColO + (uint32_t)c0 + lane_off;
    const float c = a.c_log2;
    const uint64_t c2 = pk2(c, c);
    float m_ref = -INFINITY, l = 0.f;
    for (int j = 0; j <= T; ++j) {
      uint32_t sr[32];
      if (j < T) {
        // ---- tile j: row max of this warp's 32 keys, posted to the exchange
        const int bf = j % 3;
        if (!warp_wait(SF(bf), (j / 3) & 1)) { fail(a, abort_flag); break; }
        if (warp_aborted(abort_flag)) break;
        tc_fence_after();
        const int tok0 = (t0 + j) * kTok + c0;
        tmem_ld32(tbase + (uint32_t)(bf * 128) + lane_off + (uint32_t)c0, sr);
        if (tok0 + 31 > L - a.w) {  // only the last tiles: hide keys past P_t
#pragma unroll
          for (int u = 0; u < 32; ++u)
            if (tok0 + u > Prow) sr[u] = 0xFF800000u;  // -inf
        }
        float ya = -INFINITY, yb = -INFINITY;
#pragma unroll
        for (int u = 0; u < 32; u += 4) {
          ya = fmax3(ya, f32(sr[u]), f32(sr[u + 1]));
          yb = fmax3(yb, f32(sr[u + 2]), f32(sr[u + 3]));
        }
        xmax[bf * 512 + g * 128 + row] = fmaxf(ya, yb) * c;  // c > 0: commutes with the max
        __syncwarp();
        if (lane == 0) mbar_arrive(XB(bf));
      }
      if (j >= 1) {
        // ---- tile i = j - 1: the row's reference, then P = 2^(S c - m) over S
        const int i = j - 1, bf = i % 3;
        if (!warp_wait(XB(bf), (i / 3) & 1)) { fail(a, abort_flag); break; }
        const float* xm = xmax + bf * 512;
        const float mt = fmaxf(fmaxf(xm[row], xm[128 + row]), fmaxf(xm[256 + row], xm[384 + row]));
        // the reference max moves only when a tile exceeds it by more than 8
        // (so 2^(S c - m) <= 256); then l and O are rescaled
        float fac = 1.f;
        bool resc = false;
        if (mt > m_ref + 8.f) {
          if (m_ref != -INFINITY) fac = ex2(m_ref - mt);
          resc = m_ref != -INFINITY && i > 0;
          m_ref = mt;
          l *= fac;
        }
        // warp-uniform: every lane votes, and all or none call the rescale; O
        // holds P V up to tile i - 1, which has landed once PD of its buffer
        // completes that tile's phase
        if (__any_sync(0xffffffffu, resc) &&
            !p1_rescale_o(tO, fac, PD((i - 1) % 3), (uint32_t)(((i - 1) / 3) & 1))) {
          fail(a, abort_flag);
          break;
        }
        const uint32_t tS = tbase + (uint32_t)(bf * 128) + lane_off + (uint32_t)c0;
        const int tok0 = (t0 + i) * kTok + c0;
        tmem_ld32(tS, sr);
        if (tok0 + 31 > L - a.w) {
#pragma unroll
          for (int u = 0; u < 32; ++u)
            if (tok0 + u > Prow) sr[u] = 0xFF800000u;
        }
        l += p1_exp32(sr, tS, c2, m_ref == -INFINITY ? 0.f : m_ref);
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(PF(bf));
      }
    }
    // partial row: this warp's 32 columns of O, the shared max, its normaliser part
    float* out = a.partial + ((size_t)blockIdx.x * 128 + row) * kPartStride;
    bool have = T > 0 && !warp_aborted(abort_flag);
    if (have) {
      if (!warp_wait(OF, 0)) {
        fail(a, abort_flag);
        have = false;
      }
      tc_fence_after();
    }
    uint32_t o[32];
    if (have) tmem_ld32(tO, o);
    if (valid_row) {
#pragma unroll
      for (int u = 0; u < 32; u += 4)
        *reinterpret_cast<float4*>(out + c0 + u) =
            have ? make_float4(f32(o[u]), f32(o[u + 1]), f32(o[u + 2]), f32(o[u + 3]))
                 : make_float4(0.f, 0.f, 0.f, 0.f);
      if (g == 0) out[128] = have ? m_ref : -INFINITY;
      out[129 + g] = have ? l : 0.f;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kWarpMma) {
    tc_fence_after();
    tmem_dealloc(tbase, 512);
  }
}

// =========================== combine ========================================
// One warp per query row: merge the 2 * splits partials of its (b, h, chunk).
__global__ void __launch_bounds__(128) k_tc_combine(const TcArgs a) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rows = a.B * a.Hq * a.w;
  const int r = blockIdx.x * 4 + warp;
  if (r >= rows) return;
  const int b = r / (a.Hq * a.w);
  const int hq = (r / a.w) % a.Hq;
  const int t = r % a.w;
  const int h = hq / a.G;
  const int gr = (hq % a.G) * a.w + t;
  const int chunk = gr / a.nqc, rr = gr % a.nqc;
  const int cta0 = a.cta_base[b] + (h * a.chunks + chunk) * a.splits[b];
  const int np = a.splits[b];
  auto P = [&](int i) { return a.partial + ((size_t)(cta0 + i) * 128 + rr) * kPartStride; };
  // lanes take the partials' (max, normaliser) in parallel: M, then the
  // weights 2^(m_i - M) and L = sum_i w_i l_i
  float M = -INFINITY;
  for (int i = lane; i < np; i += 32) M = fmaxf(M, P(i)[128]);
  M = warp_max(M);
  float lpart = 0.f;
  for (int i = lane; i < np; i += 32) {
    const float* p = P(i);
    const float mi = p[128];
    const float wgt = (mi == -INFINITY) ? 0.f : ex2(mi - M);
    lpart = fmaf(wgt, (p[129] + p[130]) + (p[131] + p[132]), lpart);  // four normaliser parts
  }
  const float Lsum = warp_sum(lpart);
  // O = sum_i w_i O_i, four partial rows in flight per step
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int i0 = 0; i0 < np; i0 += 4) {
    float4 o[4];
    float wg[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int i = min(i0 + k, np - 1);
      const float* p = P(i);
      o[k] = *reinterpret_cast<const float4*>(p + lane * 4);
      const float mi = p[128];
      wg[k] = (i0 + k >= np || mi == -INFINITY) ? 0.f : ex2(mi - M);
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      acc.x = fmaf(wg[k], o[k].x, acc.x);
      acc.y = fmaf(wg[k], o[k].y, acc.y);
      acc.z = fmaf(wg[k], o[k].z, acc.z);
      acc.w = fmaf(wg[k], o[k].w, acc.w);
    }
  }
  const float inv = 1.f / Lsum;
  const float A[4] = {acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv};
  const float nA = warp_sum(A[0] * A[0] + A[1] * A[1] + A[2] * A[2] + A[3] * A[3]);
  // pass 2 multiplies V by -2A (exact scaling) so that D = -2 A.v directly
  uint32_t hw[2], lw[2];
  for (int i = 0; i < 2; ++i) {
    const float x0 = -2.f * A[2 * i], x1 = -2.f * A[2 * i + 1];
    const __nv_bfloat162 hv = __floats2bfloat162_rn(x0, x1);
    const float h0 = __bfloat162float(hv.x), h1 = __bfloat162float(hv.y);
    const __nv_bfloat162 lv = __floats2bfloat162_rn(x0 - h0, x1 - h1);
    hw[i] = *reinterpret_cast<const uint32_t*>(&hv);
    lw[i] = *reinterpret_cast<const uint32_t*>(&lv);
  }
  *reinterpret_cast<uint2*>(a.ahi + (size_t)r * kHd + lane * 4) = make_uint2(hw[0], hw[1]);
  *reinterpret_cast<uint2*>(a.alo + (size_t)r * kHd + lane * 4) = make_uint2(lw[0], lw[1]);
  *reinterpret_cast<float4*>(a.attn_f32 + (size_t)r * kHd + lane * 4) =
      make_float4(A[0], A[1], A[2], A[3]);
  if (a.attn_user)
    *reinterpret_cast<float4*>(a.attn_user + (size_t)r * kHd + lane * 4) =
        make_float4(A[0], A[1], A[2], A[3]);
  if (lane == 0) {
    a.qstat[r] = make_float4(M, inv, Lsum, nA);
    if (a.stats_user) {
      a.stats_user[2 * (size_t)r] = M * 0.69314718055994531f;  // log2 units -> natural
      a.stats_user[2 * (size_t)r + 1] = Lsum;
    }
  }
}

// =========================== pass 2 =========================================
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

// Fast path for 16 query columns of one token (every p < 2^-4, no possible
// cancellation, every key visible): packed fp32 pairs,
//   p = 2^(x c - M'),  M' = M + log2 L,
//   ratio = p / (1 - p) = p (1 + p (1 + p (1 + p (1 + p)))) + O(p^6)
//   (relative truncation error p^5 / (1 - p) <= 1.0e-6 for p < 2^-4),
//   s += ratio^2 (D' + ||A||^2 + ||v||^2)   with D' = -2 A.v from the MMA.
// kf holds (-M'_t, -M'_t+1, ||A_t||^2, ||A_t+1||^2) per column pair.
__device__ __forceinline__ void fast16(const uint32_t (&r)[32], const float4* kf, uint64_t c2,
                                       uint64_t nv2, uint64_t& acc2, float& pmax) {
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float4 k = kf[i];
    float y0, y1;
    upk2(ffma2(pk2(f32(r[2 * i]), f32(r[2 * i + 1])), c2, pk2(k.x, k.y)), y0, y1);
    const float p0 = ex2(y0), p1 = ex2(y1);
    pmax = fmax3(pmax, p0, p1);
    const uint64_t P = pk2(p0, p1);
    const uint64_t one = pk2(1.f, 1.f);
    const uint64_t ratio = fmul2(P, ffma2(P, ffma2(P, ffma2(P, fadd2(P, one), one), one), one));
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

// Attention-only score (the write-up's control, section 结果与独立对照) for 16
// query columns of one token: sum of p = 2^(x c - M') over the columns that see
// the token (all of them when `masked` is false).  r[0..15] holds S^T.
__device__ __forceinline__ float attn16(const uint32_t* r, const float4* kf, uint64_t c2,
                                        bool masked, int tok, int L, int w, int crow0, int col0,
                                        float c) {
  if (!masked) {
    uint64_t acc2 = pk2(0.f, 0.f);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float4 k = kf[i];
      float y0, y1;
      upk2(ffma2(pk2(f32(r[2 * i]), f32(r[2 * i + 1])), c2, pk2(k.x, k.y)), y0, y1);
      acc2 = fadd2(acc2, pk2(ex2(y0), ex2(y1)));
    }
    float x0, x1;
    upk2(acc2, x0, x1);
    return x0 + x1;
  }
  float acc = 0.f;
#pragma unroll
  for (int u = 0; u < 16; ++u) {
    const float nM = reinterpret_cast<const float*>(kf)[(u >> 1) * 4 + (u & 1)];
    if (tok <= L - w + (crow0 + col0 + u) % w) acc += ex2(fmaf(f32(r[u]), c, nM));
  }
  return acc;
}

// kAttn = false: the DropKV perturbation score.  kAttn = true: the attention-
// only score; the CTA then streams K alone and issues only the S^T MMA.
template <bool kAttn>
__global__ void __maxnreg__(kMaxRegs2)
k_tc_pass2(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmAhi,
           const __grid_constant__ CUtensorMap tmAlo, const __grid_constant__ CUtensorMap tmK,
           const __grid_constant__ CUtensorMap tmV, const TcArgs a) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const int nqc = a.nqc;
  // A ring of kRing2 32 KB slots takes the K and V tiles in turn (K_0, V_0,
  // K_1, ...).  When A needs its low part, the last slot holds A_lo instead and
  // the ring runs on the first kRing2 - 1 slots.
  uint8_t* sRing = smem;
  uint8_t* sAl = smem + (kRing2 - 1) * kTileBytes;
  uint8_t* sQ = smem + kRing2 * kTileBytes;  // nqc rows x 2 boxes
  uint8_t* sAh = sQ + nqc * 256;
  float4* kf = reinterpret_cast<float4*>(sAh + nqc * 256);   // [nqc/2] fast-path constants
  float* nAmax = reinterpret_cast<float*>(kf + nqc / 2);      // [nqc/16] max ||A||^2 per chunk
  uint64_t* bars = reinterpret_cast<uint64_t*>(nAmax + 8);    // 5 + 2 kRing2 barriers
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 5 + 2 * kRing2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (smem_u32(smem) & 1023u) {
    if (threadIdx.x == 0) atomicMax(a.status, (int)DROPKV_ERR_CUDA);
    return;
  }
  int b, h, chunk, t0, t1;
  decode_cta(a, blockIdx.x, b, h, chunk, t0, t1);
  const int T = t1 - t0;
  const int L = a.L[b];
  const uint32_t BQ = smem_u32(&bars[0]);
  auto MD = [&](int s) { return smem_u32(&bars[1 + s]); };   // MMAs of a tile done
  auto TF = [&](int s) { return smem_u32(&bars[3 + s]); };   // TMEM buffer read out
  auto FULL = [&](int r) { return smem_u32(&bars[5 + r]); };
  auto EMPTY = [&](int r) { return smem_u32(&bars[5 + kRing2 + r]); };
  const int qrow0 = (b * a.Hkv + h) * a.G * a.w + chunk * nqc;
  const int z = b * a.Hkv + h;
  if (threadIdx.x == 0) {
    mbar_init(BQ, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(MD(s), 1); mbar_init(TF(s), kSimtWarps);  // every warp reads every tile
    }
    for (int r = 0; r < kRing2; ++r) {
      mbar_init(FULL(r), 1); mbar_init(EMPTY(r), 1);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (threadIdx.x < nqc) {
    const int i = threadIdx.x;
    const float4 q = a.qstat[qrow0 + i];  // (M, 1/L, L, ||A||^2)
    float* kff = reinterpret_cast<float*>(kf);
    kff[(i >> 1) * 4 + (i & 1)] = -(q.x + log2f(q.z));  // -M' folds 1/L into the exponent
    kff[(i >> 1) * 4 + 2 + (i & 1)] = q.w;
  }
  if (threadIdx.x < 8) nAmax[threadIdx.x] = 0.f;
  if (warp == kWarpMma) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
    tc_fence_before();
  }
  __syncthreads();
  if (threadIdx.x < nqc)  // ||A||^2 >= 0, so the float bits order like ints
    atomicMax(reinterpret_cast<int*>(nAmax) + threadIdx.x / 16,
              __float_as_int(a.qstat[qrow0 + threadIdx.x].w));
  __syncthreads();
  // Does A need its low part on this CTA's tiles?  Dropping A_lo leaves
  // -2A rounded to bf16 (relative error <= 2^-8 per component), which moves
  // -2 A.v by at most 2^-7 ||A|| ||v|| and so the squared distance
  // ||A - v||^2 >= (||v|| - ||A||)^2 by a relative 2^-7 rho / (1 - rho)^2,
  // rho = ||A|| / ||v||.  With ||A||^2 <= kLoSkip ||v||^2 for every query of
  // the chunk and every token of the tiles (rho <= 0.0283) that is <= 2.4e-4.
  bool lo = false;
  if constexpr (!kAttn) {
    float namx = 0.f;
    for (int i = 0; i < (nqc + 15) / 16; ++i) namx = fmaxf(namx, nAmax[i]);
    bool need = false;
    for (int i = threadIdx.x; i < T * a.chunks; i += blockDim.x) {
      const float tm = a.tmin[((size_t)z * a.ntmax + t0) * a.chunks + i];
      if (!(namx <= kLoSkip * tm)) need = true;  // NaN-safe
    }
    lo = __syncthreads_or(need) != 0;
  }
  const int R = lo ? kRing2 - 1 : kRing2;  // ring slots in use
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;

  if (warp == kWarpTma) {
    if (lane == 0) {
      prefetch_tmap(&tmQ); prefetch_tmap(&tmAhi); prefetch_tmap(&tmAlo);
      prefetch_tmap(&tmK); prefetch_tmap(&tmV);
      mbar_expect_tx(BQ, (kAttn ? 1 : lo ? 3 : 2) * nqc * 256);
      tma_load_2d(smem_u32(sQ), &tmQ, BQ, 0, qrow0);
      tma_load_2d(smem_u32(sQ) + nqc * 128, &tmQ, BQ, 64, qrow0);
      if (!kAttn) {
        tma_load_2d(smem_u32(sAh), &tmAhi, BQ, 0, qrow0);
        tma_load_2d(smem_u32(sAh) + nqc * 128, &tmAhi, BQ, 64, qrow0);
      }
      if (lo) {
        tma_load_2d(smem_u32(sAl), &tmAlo, BQ, 0, qrow0);
        tma_load_2d(smem_u32(sAl) + nqc * 128, &tmAlo, BQ, 64, qrow0);
      }
      // single thread: no warp vote needed.  Perturbation: K_j at i = 2j and
      // V_j at 2j + 1; attention-only: K_j at i = j.
      // (slot, phase) of load i kept incrementally: R is a runtime ring size
      const int nload = kAttn ? T : 2 * T;
      int r = 0, ph = 0;
      for (int i = 0; i < nload && !*abort_flag; ++i, r = (r + 1 == R) ? 0 : r + 1, ph ^= (r == 0)) {
        if (!mbar_wait(EMPTY(r), ph ^ 1, kWaitNs)) { fail(a, abort_flag); break; }
        mbar_expect_tx(FULL(r), kTileBytes);
        const uint32_t dst = smem_u32(sRing + r * kTileBytes);
        const CUtensorMap* m = (!kAttn && (i & 1)) ? &tmV : &tmK;
        const int row = (t0 + (kAttn ? i : i >> 1)) * kTok;
        tma_load_3d(dst, m, FULL(r), 0, row, z);
        tma_load_3d(dst + kBox, m, FULL(r), 64, row, z);
      }
    }
  } else if (warp == kWarpMma) {
    const uint32_t IDT = idesc_bf16(128, nqc, false, false);
    bool ok = warp_wait(BQ, 0);
    if (!ok) fail(a, abort_flag);
    const SDesc rd0 = sdesc_split(smem_u32(sRing), 16, 1024);  // ring slot 0
    const SDesc qd = sdesc_split(smem_u32(sQ), 16, 1024), hd = sdesc_split(smem_u32(sAh), 16, 1024),
                ld = sdesc_split(smem_u32(sAl), 16, 1024);
    const uint32_t nq = (uint32_t)nqc;
    // ring (slot, phase) of K_j kept incrementally (R is a runtime ring size):
    // V_j follows K_j, K_{j+1} follows V_j (or K_j for the attention score)
    int pos = 0, pph = 0;
    for (int j = 0; j < T && ok && !warp_aborted(abort_flag); ++j) {
      const int s = j & 1, ph = (j >> 1) & 1;
      const int rk = pos, pk = pph;
      int rv = rk + 1, pv = pk;
      if (rv == R) { rv = 0; pv ^= 1; }
      if (kAttn) {
        pos = rv; pph = pv;
      } else {
        pos = rv + 1; pph = pv;
        if (pos == R) { pos = 0; pph ^= 1; }
      }
      const uint32_t dS = tbase + (uint32_t)(s * 256), dD = dS + 128u;
      if (!warp_wait(TF(s), ph ^ 1) || !warp_wait(FULL(rk), pk)) {
        fail(a, abort_flag);
        break;
      }
      tc_fence_after();
      const uint32_t klo = rd0.lo + (uint32_t)rk * (kTileBytes >> 4);
      const uint32_t vlo = rd0.lo + (uint32_t)rv * (kTileBytes >> 4);
      if (lane == 0) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ss_w(dS, klo + kslice(kk, 128), rd0.hi, qd.lo + kslice(kk, nq), qd.hi, IDT,
                   kk > 0 ? 1u : 0u);
        mma_commit(EMPTY(rk));
        if (kAttn) mma_commit(MD(s));
      }
      __syncwarp();
      if (kAttn) continue;
      if (!warp_wait(FULL(rv), pv)) { fail(a, abort_flag); break; }
      tc_fence_after();
      if (lane == 0) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ss_w(dD, vlo + kslice(kk, 128), rd0.hi, hd.lo + kslice(kk, nq), hd.hi, IDT,
                   kk > 0 ? 1u : 0u);
        if (lo) {
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_ss_w(dD, vlo + kslice(kk, 128), rd0.hi, ld.lo + kslice(kk, nq), ld.hi, IDT, 1u);
        }
        mma_commit(EMPTY(rv));
        mma_commit(MD(s));
      }
      __syncwarp();
    }
  } else if (warp < kSimtWarps) {
    // Sixteen warps work on every tile: warp (g, quarter) owns the tokens
    // [32 quarter, +32) of the tile (its TMEM lanes) and the query columns
    // [32 g, min(nqc, 32 g + 32)), and writes its own partial-score plane.
    const int g = warp >> 2, ql = warp & 3;
    const int row = ql * 32 + lane;  // token within the tile
    const uint32_t lane_off = (uint32_t)(ql * 32) << 16;
    const float c = a.c_log2;
    const uint64_t c2 = pk2(c, c);
    const int ch0 = min(nqc / 16, 2 * g), ch1 = min(nqc / 16, 2 * g + 2);  // 16-column chunks
    const float4* qrows = a.qstat + qrow0;
    const float* arows = a.attn_f32 + (size_t)qrow0 * kHd;
    float* plane = a.parts + (size_t)(chunk * 4 + g) * a.part_stride + (size_t)z * a.n_max;
    const int nch = ch1 - ch0;  // this warp's 16-column chunks: 0, 1 or 2 (warp-uniform)
    // ||v_j||^2 of the next tile is fetched one tile ahead: under the streaming
    // traffic a global load takes of the order of a tile's work to return
    auto nv_at = [&](int jj) -> float {
      const int tk = (t0 + jj) * kTok + row;
      return (!kAttn && jj < T && tk < L) ? a.nvbuf[(size_t)z * a.ntmax * kTok + tk] : 0.f;
    };
    float nv_next = nv_at(0);
    int sing = 0;
    // A warp with no columns (nch = 0) still walks the tiles: it hands every
    // buffer back and writes zeros to its plane.
    for (int j = 0; j < T; ++j) {
      const int s = j & 1, ph = (j >> 1) & 1;
      const int tile0 = (t0 + j) * kTok;
      const int tok = tile0 + row;
      const bool valid = tok < L;
      const float nv = nv_next;
      nv_next = nv_at(j + 1);
      const __nv_bfloat16* vrow_g = a.v + ((size_t)z * a.n_max + (valid ? tok : 0)) * kHd;
      if (!warp_wait(MD(s), ph)) { fail(a, abort_flag); break; }
      if (warp_aborted(abort_flag)) break;
      tc_fence_after();
      const uint32_t tS = tbase + (uint32_t)(s * 256) + lane_off + (uint32_t)(ch0 * 16);
      const uint32_t tD = tS + 128u;
      const bool masked = tile0 + kTok - 1 > L - a.w;
      // The buffer goes back to the MMA warp as soon as its last columns this
      // warp needs are in registers (before the last chunk's arithmetic), so
      // that the MMAs of tile j + 2 overlap the rest of this tile's work.
      auto release = [&]() {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(TF(s));
      };
      // score of 16 columns (chunk ch) from S^T in r[0..15] and D in r[16..31]
      auto chunk_score = [&](const uint32_t(&r)[32], int ch) -> float {
        bool redo = masked;
        uint64_t a2 = pk2(0.f, 0.f);
        if (!masked) {
          float pmax = 0.f;
          fast16(r, kf + ch * 8, c2, pk2(nv, nv), a2, pmax);
          // a large p (>= 2^-4: the series above would be short) or possible
          // cancellation (||A||^2 >= 0.6 ||v||^2): the careful path
          redo = pmax >= 0.0625f || nAmax[ch] >= 0.6f * nv;
        }
        if (__any_sync(0xffffffffu, redo)) {
          uint32_t rc[32];
#pragma unroll
          for (int k = 0; k < 32; ++k) rc[k] = r[k];
          return careful16(rc, ch * 16, tok, masked, L, a.w, chunk * nqc, qrows, c, nv, arows,
                           vrow_g, &sing);
        }
        float x0, x1;
        upk2(a2, x0, x1);
        return x0 + x1;
      };
      float acc = 0.f;
      if (nch == 0) {
        release();
      } else if (kAttn) {
        uint32_t r[32];
        tmem_ld32(tS, r);  // S^T of chunks ch0, ch0 + 1 (the second unused when nch = 1)
        release();
        acc = attn16(r, kf + ch0 * 8, c2, masked, tok, L, a.w, chunk * nqc, ch0 * 16, c);
        if (nch > 1)
          acc += attn16(r + 16, kf + ch0 * 8 + 8, c2, masked, tok, L, a.w, chunk * nqc,
                        ch0 * 16 + 16, c);
      } else {
        uint32_t r[32];
        tmem_ld16x2(tS, tD, r);  // chunk ch0: 16 columns of S^T and of D
        if (nch == 1) release();
        acc = chunk_score(r, ch0);
        if (nch > 1) {
          tmem_ld16x2(tS + 16u, tD + 16u, r);  // chunk ch0 + 1
          release();
          acc += chunk_score(r, ch0 + 1);
        }
      }
      if (valid) plane[tok] = acc;
    }
    if (sing) atomicMax(a.status, (int)DROPKV_ERR_SINGULAR);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kWarpMma) {
    tc_fence_after();
    tmem_dealloc(tbase, 512);
  }
}

// =========================== host side ======================================
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// bf16 [rows][128] row-major, box = 64 columns x box_rows rows, 128B swizzle.
bool map_2d(CUtensorMap* m, const void* base, uint64_t rows, uint32_t box_rows) {
  auto enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)kHd, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)kHd * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t es[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// bf16 [heads][n_max][128], box = 64 columns x 128 tokens x 1 head.
bool map_3d(CUtensorMap* m, const void* base, uint64_t heads, uint64_t n_max) {
  auto enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {(cuuint64_t)kHd, (cuuint64_t)n_max, (cuuint64_t)heads};
  cuuint64_t strides[2] = {(cuuint64_t)kHd * 2, (cuuint64_t)n_max * kHd * 2};
  cuuint32_t box[3] = {64, (cuuint32_t)kTok, 1};
  cuuint32_t es[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

size_t pass1_smem() {
  return (1 + kStK + kSt1) * (size_t)kTileBytes + kBars1 * 8 + 8 + 3 * 4 * 128 * 4;
}
size_t pass2_smem(int nqc) {
  return kRing2 * (size_t)kTileBytes + 2 * (size_t)nqc * 256 + (size_t)nqc / 2 * 16 + 8 * 4 +
         (5 + 2 * kRing2) * 8 + 8;
}

int num_sms() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n;
}

}  // namespace

bool tc_available() { return true; }
int tc_split_target() { return kMaxCtas; }
int tc_launch_count() { return 3; }

// Splits per batch row so that the CTAs (one per SM) carry balanced tile
// counts: greedily give another split to the row whose CTAs are longest.
void tc_splits(const Lens& lens, int units_per_row, int budget, int32_t* splits) {
  int total = 0;
  for (int b = 0; b < lens.B; ++b) {
    splits[b] = 1;
    total += units_per_row;
  }
  for (;;) {
    int best = -1;
    double worst = 0;
    for (int b = 0; b < lens.B; ++b) {
      const int nt = (lens.L[b] + kTok - 1) / kTok;
      const double per = (double)nt / splits[b];
      if (splits[b] < nt && per > worst) {
        worst = per;
        best = b;
      }
    }
    if (best < 0 || total + units_per_row > budget) break;
    splits[best] += 1;
    total += units_per_row;
  }
}

cudaError_t launch_tc_scores(const dropkv_shape& s, const void* q, const void* k, const void* v,
                             const Lens& lens, const ScoresLayout& lay, char* ws, float* attn_out,
                             float* stats_out, int32_t* status, int score, int cta_budget,
                             cudaStream_t st, KernelEvents& kev) {
  const bool attn_only = score == DROPKV_SCORE_ATTENTION;
  auto pass2 = attn_only ? k_tc_pass2<true> : k_tc_pass2<false>;
  const TcPlan plan = tc_plan(s);
  TcArgs a;
  memset(&a, 0, sizeof(a));
  a.B = lens.B;
  a.Hq = s.Hq;
  a.Hkv = s.Hkv;
  a.n_max = s.n_max;
  a.w = s.window;
  a.G = s.Hq / s.Hkv;
  a.nqc = plan.nqc;
  a.chunks = plan.chunks;
  for (int i = 0; i < lens.B; ++i) a.L[i] = lens.L[i];
  const int units = s.Hkv * plan.chunks;
  const int budget = std::min(cta_budget > 0 ? cta_budget : num_sms(), kMaxCtas);
  tc_splits(lens, units, std::max(budget, units * lens.B), a.splits);
  a.cta_base[0] = 0;
  for (int i = 0; i < lens.B; ++i) a.cta_base[i + 1] = a.cta_base[i] + units * a.splits[i];
  const int ctas = a.cta_base[lens.B];
  a.c_log2 = (float)(1.4426950408889634 / sqrt((double)s.d));
  a.q = reinterpret_cast<const __nv_bfloat16*>(q);
  a.partial = reinterpret_cast<float*>(ws + lay.tc_partial);
  a.status = status;
  a.ahi = reinterpret_cast<__nv_bfloat16*>(ws + lay.tc_ahi);
  a.alo = reinterpret_cast<__nv_bfloat16*>(ws + lay.tc_alo);
  a.qstat = reinterpret_cast<float4*>(ws + lay.tc_qstat);
  a.attn_user = attn_out;
  a.stats_user = stats_out;
  a.parts = reinterpret_cast<float*>(ws + lay.parts);
  a.part_stride = (size_t)lens.B * s.Hkv * s.n_max;
  a.attn_f32 = reinterpret_cast<float*>(ws + lay.attn);
  a.v = reinterpret_cast<const __nv_bfloat16*>(v);
  a.nvbuf = reinterpret_cast<float*>(ws + lay.tc_nv);
  a.tmin = reinterpret_cast<float*>(ws + lay.tc_tmin);
  a.ntmax = (s.n_max + kTok - 1) / kTok;

  const uint64_t rows = (uint64_t)lens.B * s.Hq * s.window;
  a.qbox_rows = (int32_t)std::min<uint64_t>(128, rows);
  CUtensorMap mQ1, mQ2, mK, mV, mAh, mAl;
  if (!map_2d(&mQ1, q, rows, (uint32_t)a.qbox_rows) || !map_2d(&mQ2, q, rows, (uint32_t)plan.nqc) ||
      !map_3d(&mK, k, (uint64_t)lens.B * s.Hkv, (uint64_t)s.n_max) ||
      !map_3d(&mV, v, (uint64_t)lens.B * s.Hkv, (uint64_t)s.n_max) ||
      !map_2d(&mAh, a.ahi, rows, (uint32_t)plan.nqc) ||
      !map_2d(&mAl, a.alo, rows, (uint32_t)plan.nqc))
    return cudaErrorNotSupported;

  const size_t sm1 = pass1_smem(), sm2 = pass2_smem(plan.nqc);
  cudaError_t e = cudaFuncSetAttribute(k_tc_pass1, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)sm1);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(pass2, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm2);
  if (e != cudaSuccess) return e;

  kev.begin(st);
  k_tc_pass1<<<ctas, kThreads1, sm1, st>>>(mQ1, mK, mV, a);
  kev.end(st);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  kev.begin(st);
  k_tc_combine<<<(unsigned)((rows + 3) / 4), 128, 0, st>>>(a);
  kev.end(st);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  kev.begin(st);
  pass2<<<ctas, kThreads2, sm2, st>>>(mQ2, mAh, mAl, mK, mV, a);
  kev.end(st);
  return cudaGetLastError();
}

}  // namespace dropkv
