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
// Work split.  The tokens of each (b, h, query chunk) unit are cut into
// `splits` contiguous ranges of 128-token tiles so that about one CTA runs per
// SM.  Pass 1 takes chunks of <= 256 query rows (two tiles of 128); the
// DropKV second pass (tc_pair.cu) runs on CTA pairs; the attention-only
// second pass below takes chunks of nqc <= 128 rows.
//
// k_tc_pass1 (query-major, one CTA per (b, h, chunk, split)):
//   S_t = Q_t K_tile^T for both query tiles t, tcgen05 M=128 (queries) N=128
//   (tokens) K=128; one softmax warpgroup per query tile, one query row per
//   thread: a max pass over the row's 128 logits, then P = exp2(S*c - m)
//   written back over S in TMEM as two bf16 planes, P_hi = P truncated to
//   bf16 and P_lo = bf16(P - P_hi), so P_hi + P_lo holds P to 2^-16 relative;
//   O_t += P_hi V + P_lo V (A from TMEM, V MN-major).  The reference max only
//   moves up by more than 8, so exp2 stays <= 256 and O rarely rescales.
//   While one query tile's softmax runs, the other tile's MMAs keep the
//   tensor pipe busy.  A chunk of at most 128 rows is one query tile: then the
//   two warpgroups take alternate token tiles, each with its own S/P buffer
//   and O, and are folded together at the end.  Each CTA writes one partial
//   (m, l, O) per row.
// k_tc_combine: merges the partials of a row into the final max M, normaliser
//   L and output A = O / L; writes -2A as bf16 hi/lo planes (same split) plus
//   the per-query constants (M, 1/L, L, ||A||^2) for the second pass.
// k_tc_pass2 (token-major, one CTA per (b, h, chunk, split)): the
//   attention-only control score (section 结果与独立对照): S^T = K_tile Q^T,
//   tcgen05 M=128 (tokens) N=nqc (queries) K=128, into two TMEM buffers; each
//   thread owns one token and sums p = exp2(S*c - M') over its warp's
//   queries, M' = M + log2 L.  K tiles only.
//
// Every wait on an mbarrier is bounded (2 s of %globaltimer); on expiry the
// kernel records DROPKV_ERR_TIMEOUT, every role leaves its loop and TMEM is
// freed.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <math.h>
#include <string.h>

#include <algorithm>

#include "tc_common.cuh"

namespace dropkv {

namespace {

// =========================== pass 1 =========================================
// P = exp2(S c - mu) for 16 tokens of one query row (S in s16[0..15], masked
// keys at -inf), written back over s16 as 8 hi + 8 lo bf16 pair words (the
// column layout P V reads: hi of the 16 tokens, then lo).  Returns the sum of
// P over the 16 tokens.
__device__ __forceinline__ float p1_exp16(uint32_t* s16, uint64_t c2, uint64_t nmu2) {
  uint64_t l2 = pk2(0.f, 0.f);
  uint32_t pw[16];
#pragma unroll
  for (int u2 = 0; u2 < 8; ++u2) {
    float d0, d1;
    upk2(ffma2(pk2(f32(s16[2 * u2]), f32(s16[2 * u2 + 1])), c2, nmu2), d0, d1);
    const float e0 = ex2(d0), e1 = ex2(d1);
    const uint64_t E = pk2(e0, e1);
    l2 = fadd2(l2, E);
    pw[u2] = __byte_perm(u32(e0), u32(e1), 0x7632);  // truncated bf16 pair
    const float nh0 = f32((u32(e0) & 0xFFFF0000u) | 0x80000000u);
    const float nh1 = f32((u32(e1) & 0xFFFF0000u) | 0x80000000u);
    float r0, r1;
    upk2(fadd2(E, pk2(nh0, nh1)), r0, r1);  // exact remainders e - hi
    pw[8 + u2] = pack_bf16_rn(r0, r1);
  }
#pragma unroll
  for (int k = 0; k < 16; ++k) s16[k] = pw[k];
  float la, lb;
  upk2(l2, la, lb);
  return la + lb;
}

// Rare path of pass 1, out of line: the reference max of some rows moved
// (factor fac < 1 for them, 1 for the others), so the warp's 32 rows of O
// (128 columns) are rescaled once the P V that last accumulated into O has
// landed (waited on through that P V's barrier and parity).  Warp-collective.
// Returns false on a timeout.
__device__ __noinline__ bool p1_rescale_o(uint32_t tO, float fac, uint32_t pd_bar,
                                          uint32_t parity) {
  if (!warp_wait(pd_bar, parity)) return false;
  tc_fence_after();
  for (int c = 0; c < 4; ++c) {
    uint32_t o[32];
    tmem_ld32(tO + 32u * c, o);
#pragma unroll
    for (int u = 0; u < 32; ++u) o[u] = u32(f32(o[u]) * fac);
    tmem_st32(tO + 32u * c, o);
  }
  tmem_st_wait();
  return true;
}

// One CTA per (b, h, query chunk, token split), two softmax warpgroups, each
// with its own S/P buffer and O accumulator in TMEM (warpgroup u: S/P at
// columns 128 u, O at 256 + 128 u) and its own running max and normaliser.
//  * kAlt = false (chunks of more than 128 rows): the chunk's rows (<= 256)
//    are two query tiles of 128 rows and warpgroup u owns tile u; a K/V tile
//    in shared memory serves both.  Tensor-pipe order per tile j: P V of tile
//    0, S of tile 0 for j + 1, P V of tile 1, S of tile 1 for j + 1.
//  * kAlt = true (chunks of at most 128 rows, one query tile): the warpgroups
//    take the token tiles in turn (warpgroup u the tiles j = u mod 2), so the
//    second warpgroup does not idle.  Tensor-pipe order: S(0), S(1), then per
//    tile j: P V(j), S(j + 2).  At the end warpgroup 0 folds warpgroup 1's
//    (max, normaliser, O) into its own and writes the row's one partial.
// A warpgroup's next S overwrites its P, so it waits for the P V that reads
// it; the other warpgroup's work keeps the tensor pipe busy meanwhile.
template <bool kAlt>
__global__ void __launch_bounds__(kThreads1, 1)
k_tc_pass1(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
           const __grid_constant__ CUtensorMap tmV, const TcArgs a) {
  extern __shared__ __align__(1024) uint8_t smem[];
  uint8_t* sQ = smem;                              // two query tiles
  uint8_t* sK = smem + 2 * kTileBytes;             // kStK stages
  uint8_t* sV = sK + kStK * kTileBytes;            // kSt1 stages
  uint64_t* bars = reinterpret_cast<uint64_t*>(sV + kSt1 * kTileBytes);  // kBars1 barriers
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + kBars1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float2* xml = reinterpret_cast<float2*>(tmem_slot + 2);  // [128] kAlt: warpgroup 1's (m, l)
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (smem_u32(smem) & 1023u) {  // the swizzled tiles need 1 KB alignment
    if (threadIdx.x == 0) atomicMax(a.status, (int)DROPKV_ERR_CUDA);
    return;
  }
  pdl_trigger();  // the combine may launch now; it waits for this grid to finish
  int b, h, chunk, t0, t1;
  decode_plan(a, a.splits1, a.cta_base1, a.chunks1, blockIdx.x, b, h, chunk, t0, t1);
  const int T = t1 - t0;
  const int L = a.L[b];
  const int R = min(a.rows1, a.nq - chunk * a.rows1);  // this chunk's query rows
  const int nt = kAlt ? 1 : (R > 128 ? 2 : 1);          // query tiles
  // barriers: Q; K full/empty (kStK stages); V full/empty (kSt1 stages); per
  // softmax warpgroup: S ready, P written, P V done
  const uint32_t BQ = smem_u32(&bars[0]);
  auto KF = [&](int s) { return smem_u32(&bars[1 + s]); };
  auto KE = [&](int s) { return smem_u32(&bars[1 + kStK + s]); };
  auto VF = [&](int s) { return smem_u32(&bars[1 + 2 * kStK + s]); };
  auto VE = [&](int s) { return smem_u32(&bars[1 + 2 * kStK + kSt1 + s]); };
  constexpr int kB0 = 1 + 2 * kStK + 2 * kSt1;
  auto SF = [&](int t) { return smem_u32(&bars[kB0 + t]); };
  auto PF = [&](int t) { return smem_u32(&bars[kB0 + 2 + t]); };
  auto PD = [&](int t) { return smem_u32(&bars[kB0 + 4 + t]); };
  if (threadIdx.x == 0) {
    mbar_init(BQ, 1);
    for (int s = 0; s < kStK; ++s) {
      mbar_init(KF(s), 1); mbar_init(KE(s), 1);
    }
    for (int s = 0; s < kSt1; ++s) {
      mbar_init(VF(s), 1);
      mbar_init(VE(s), 2);  // the last P V's commit + the ||v||^2 warp's reads
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(SF(t), 1); mbar_init(PF(t), 4); mbar_init(PD(t), 1);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kW1Mma) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;
  const int z = b * a.Hkv + h;
  const int qrow0 = (b * a.Hkv + h) * a.nq + chunk * a.rows1;
  // Two query tiles: the producer warpgroup (TMA, MMA and ||v||^2 warps)
  // hands registers to the softmax warpgroups, whose rows of 128 logits
  // otherwise spill.  The shares add up to the launch's 384 x kRegs1.
  constexpr uint32_t kRegsSm = 224, kRegsPr = 56;
  static_assert(kThreads1 == 384 && kSmWarps1 == 8 &&
                    2 * 128 * kRegsSm + 128 * kRegsPr == kThreads1 * kRegs1,
                "register split of pass 1");

  if (warp >= kSmWarps1) {
    if constexpr (!kAlt) setmaxnreg_dec<kRegsPr>();
    if (warp == kW1Tma || warp == kW1TmaV) {
      // ---------------- TMA producers ----------------
      // warp kW1Tma: the query tiles, then K_0, K_1, ... (K_{i+2} once both
      // query tiles' S have read K_i); warp kW1TmaV: V_0, V_1, ... (kSt1 ahead).
      if (lane == 0) {
        const bool kq = warp == kW1Tma;
        if (kq) {
          prefetch_tmap(&tmQ); prefetch_tmap(&tmK);
          mbar_expect_tx(BQ, (uint32_t)nt * 2u * 128u * (uint32_t)a.qbox_rows);
          for (int t = 0; t < nt; ++t) {  // rows past the tensor read as zeros
            tma_load_2d(smem_u32(sQ) + t * kTileBytes, &tmQ, BQ, 0, qrow0 + 128 * t);
            tma_load_2d(smem_u32(sQ) + t * kTileBytes + kBox, &tmQ, BQ, 64, qrow0 + 128 * t);
          }
        } else {
          prefetch_tmap(&tmV);
        }
        uint8_t* buf = kq ? sK : sV;
        const int nst = kq ? kStK : kSt1;
        const CUtensorMap* m = kq ? &tmK : &tmV;
        for (int i = 0; i < T && !*abort_flag; ++i) {
          const int st = i % nst, ph = (i / nst) & 1;
          const uint32_t full = kq ? KF(st) : VF(st), empty = kq ? KE(st) : VE(st);
          if (!mbar_wait(empty, ph ^ 1, kWaitNs)) { fail(a, abort_flag); break; }
          mbar_expect_tx(full, kTileBytes);
          const uint32_t dst = smem_u32(buf + st * kTileBytes);
          tma_load_3d(dst, m, full, 0, (t0 + i) * kTok, z);
          tma_load_3d(dst + kBox, m, full, 64, (t0 + i) * kTok, z);
        }
      }
    } else if (warp == kW1Mma) {
      // ---------------- MMA issuer ----------------
      constexpr uint32_t IDS = idesc_bf16(128, 128, false, false);   // S = Q K^T
      constexpr uint32_t IDP = idesc_bf16(128, 128, false, true);    // O += P V (V MN-major)
      bool ok = warp_wait(BQ, 0);
      if (!ok) fail(a, abort_flag);
      // operand descriptors of stage 0; a stage, tile or K slice only moves the
      // start address, i.e. adds to the low word
      const SDesc qd = sdesc_split(smem_u32(sQ), 16, 1024);
      const SDesc kd0 = sdesc_split(smem_u32(sK), 16, 1024);
      const SDesc vd0 = sdesc_split(smem_u32(sV), kBox, 1024);
      // S = Q_q K_j^T (query tile q) into warpgroup u's S/P columns, the n-th
      // S of that warpgroup; they hold its previous P until the P V reading it
      // has completed.  K_j's last reader commits the stage free.
      auto issue_S = [&](int u, int q, int j, int n) {
        const int s = j % kStK, ph = (j / kStK) & 1;
        if (!warp_wait(KF(s), ph)) { fail(a, abort_flag); return false; }
        if (n >= 1 && !warp_wait(PD(u), (uint32_t)((n - 1) & 1))) {
          fail(a, abort_flag);
          return false;
        }
        tc_fence_after();
        if (lane == 0) {
          const uint32_t qlo = qd.lo + (uint32_t)q * (kTileBytes >> 4);
          const uint32_t klo = kd0.lo + (uint32_t)s * (kTileBytes >> 4);
          const uint32_t dS = tbase + (uint32_t)(128 * u);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_ss_w(dS, qlo + kslice(kk, 128), qd.hi, klo + kslice(kk, 128), kd0.hi, IDS,
                     kk > 0 ? 1u : 0u);
          mma_commit(SF(u));
          if (kAlt || u == nt - 1) mma_commit(KE(s));
        }
        __syncwarp();
        return true;
      };
      // O_u += P V_j, the n-th P V of warpgroup u; V_j's last reader commits the
      // stage free
      auto issue_PV = [&](int u, int j, int n) {
        const int s = j % kSt1, ph = (j / kSt1) & 1;
        if (!warp_wait(PF(u), (uint32_t)(n & 1))) { fail(a, abort_flag); return false; }
        if (!warp_wait(VF(s), ph)) { fail(a, abort_flag); return false; }
        uint8_t* vb = sV + s * kTileBytes;
        const int tile0 = (t0 + j) * kTok;
        if ((kAlt || u == 0) && tile0 + kTok > L) {
          // rows at or beyond L hold no data (possibly NaN): zero them (once per
          // V tile, before its first P V) so that the P = 0 weights of those
          // rows contribute exactly 0 to O
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
          const uint32_t dO = tbase + kColO1 + (uint32_t)(128 * u);
          const uint32_t pS = tbase + (uint32_t)(128 * u);
          // tokens 16kk..16kk+15: P_hi in columns [16kk, 16kk+8), P_lo in [16kk+8, 16kk+16);
          // V slice kk starts 16 rows (2048 bytes) further
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_ts_w(dO, pS + (uint32_t)(16 * kk), vlo + (uint32_t)kk * 128u, vd0.hi, IDP,
                     (n > 0 || kk > 0) ? 1u : 0u);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_ts_w(dO, pS + (uint32_t)(16 * kk + 8), vlo + (uint32_t)kk * 128u, vd0.hi, IDP, 1u);
          mma_commit(PD(u));
          if (kAlt || u == nt - 1) mma_commit(VE(s));
        }
        __syncwarp();
        return true;
      };
      if (kAlt) {
        for (int j = 0; j < 2 && j < T && ok; ++j) ok = issue_S(j, 0, j, 0);
        for (int j = 0; j < T && ok && !warp_aborted(abort_flag); ++j) {
          ok = issue_PV(j & 1, j, j >> 1);
          if (ok && j + 2 < T) ok = issue_S(j & 1, 0, j + 2, (j >> 1) + 1);
        }
      } else {
        for (int t = 0; t < nt && ok && T > 0; ++t) ok = issue_S(t, t, 0, 0);
        for (int j = 0; j < T && ok && !warp_aborted(abort_flag); ++j)
          for (int t = 0; t < nt && ok; ++t) {
            ok = issue_PV(t, j, j);
            if (ok && j + 1 < T) ok = issue_S(t, t, j + 1, j + 1);
          }
      }
    } else if (warp == kW1Nv) {
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
          if ((row * a.chunks1) / 128 != chunk || tile0 + row >= L) continue;
          uint64_t acc2 = pk2(0.f, 0.f);
#pragma unroll
          for (int bx = 0; bx < 2; ++bx)
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              const uint4 q4 = *reinterpret_cast<const uint4*>(vb + bx * kBox + row * 128 +
                                                               ((q ^ (row & 7)) * 16));
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
        if (lane == 0) a.tmin[((size_t)z * a.ntmax + t0 + j) * a.chunks1 + chunk] = vmin;
      }
    }
  } else {
    if constexpr (!kAlt) setmaxnreg_inc<kRegsSm>();
    // ---------------- softmax warps ----------------
    // Warpgroup u: query tile u and every token tile (kAlt = false), or the
    // query tile and the token tiles j = u, u + 2, ... (kAlt = true).  Thread
    // = one query row (its TMEM lane), all 128 tokens of a tile: a max pass
    // over S, then P = 2^(S c - m) written back over S as hi/lo planes.  The
    // reference max moves only when a tile exceeds it by more than 8 (so
    // 2^(.) <= 256); then l and the row of the warpgroup's O are rescaled,
    // after the P V that last accumulated into it.
    const int u = warp >> 2, ql = warp & 3;
    const int row = ql * 32 + lane;                // row within the query tile
    const int crow = kAlt ? row : 128 * u + row;   // row within the chunk
    const bool valid_row = crow < R;
    const int Prow = L - a.w + (chunk * a.rows1 + crow) % a.w;
    const uint32_t lane_off = (uint32_t)(ql * 32) << 16;
    const uint32_t tS = tbase + (uint32_t)(128 * u) + lane_off;
    const uint32_t tO = tbase + kColO1 + (uint32_t)(128 * u) + lane_off;
    const float c = a.c_log2;
    const uint64_t c2 = pk2(c, c);
    float m_ref = -INFINITY, l = 0.f;
    // this warpgroup's tiles (a second warpgroup without a second query tile
    // has none when kAlt is false)
    const int nmine = kAlt ? (T > u ? (T - u + 1) / 2 : 0) : (u < nt ? T : 0);
    bool live = true;
    for (int n = 0; n < nmine && live; ++n) {
      const int j = kAlt ? u + 2 * n : n;
      if (!warp_wait(SF(u), (uint32_t)(n & 1))) { fail(a, abort_flag); live = false; break; }
      if (warp_aborted(abort_flag)) { live = false; break; }
      tc_fence_after();
      const int tok0 = (t0 + j) * kTok;
      const bool masked = tok0 + kTok - 1 > L - a.w;  // only the last tiles hide keys past P_t
      // the row's 128 logits in one TMEM load (one round trip per tile)
      uint32_t sr[128];
      tmem_ld128(tS, sr);
      if (masked) {
#pragma unroll
        for (int x = 0; x < 128; ++x)
          if (tok0 + x > Prow) sr[x] = 0xFF800000u;  // -inf
      }
      float ya = -INFINITY, yb = -INFINITY;
#pragma unroll
      for (int x = 0; x < 128; x += 4) {
        ya = fmax3(ya, f32(sr[x]), f32(sr[x + 1]));
        yb = fmax3(yb, f32(sr[x + 2]), f32(sr[x + 3]));
      }
      const float mt = fmaxf(ya, yb) * c;  // c > 0: commutes with the max
      float fac = 1.f;
      bool resc = false;
      if (mt > m_ref + 8.f) {
        if (m_ref != -INFINITY) fac = ex2(m_ref - mt);
        resc = m_ref != -INFINITY && n > 0;
        m_ref = mt;
        l *= fac;
      }
      // warp-uniform: every lane votes, and all or none call the rescale; O
      // holds the warpgroup's P V up to its previous tile, which has landed
      // once PD completes that phase
      if (__any_sync(0xffffffffu, resc) &&
          !p1_rescale_o(tO, fac, PD(u), (uint32_t)((n - 1) & 1))) {
        fail(a, abort_flag);
        live = false;
        break;
      }
      const float mu = m_ref == -INFINITY ? 0.f : m_ref;
      const uint64_t nmu2 = pk2(-mu, -mu);
#pragma unroll
      for (int cc = 0; cc < 8; ++cc) l += p1_exp16(sr + 16 * cc, c2, nmu2);
      tmem_st128(tS, sr);  // the whole row of P in one store
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(PF(u));
    }
    // the warpgroup's O is complete once its last P V has landed
    bool have = live && nmine > 0 && !warp_aborted(abort_flag);
    bool own = false;  // O read from this warpgroup's accumulator
    if (have) {
      if (!warp_wait(PD(u), (uint32_t)((nmine - 1) & 1))) {
        fail(a, abort_flag);
        have = false;
      }
      tc_fence_after();
    }
    own = have;
    // kAlt: warpgroup 1 hands (m, l) over through shared memory; warpgroup 0
    // reads its O straight from TMEM (same lanes) and folds it in
    float w0 = 1.f, w1 = 0.f;
    bool have1 = false;
    if (kAlt) {
      if (u == 1) xml[row] = make_float2(have ? m_ref : -INFINITY, have ? l : 0.f);
      tc_fence_before();
      named_barrier_sync(1, kSmWarps1 * 32);  // both softmax warpgroups, unconditionally
      tc_fence_after();
      if (u == 0) {
        const float2 ml1 = xml[row];
        have1 = ml1.x != -INFINITY;
        const float m0 = have ? m_ref : -INFINITY;
        const float M = fmaxf(m0, ml1.x);
        w0 = m0 == -INFINITY ? 0.f : ex2(m0 - M);
        w1 = have1 ? ex2(ml1.x - M) : 0.f;
        l = (have ? w0 * l : 0.f) + (have1 ? w1 * ml1.y : 0.f);
        m_ref = M;
        have = have || have1;
      }
    }
    // the row's partial: O, the reference max, the normaliser
    if (u < nt) {
      float* out = a.partial + ((size_t)blockIdx.x * a.rows1 + crow) * kPartStride;
#pragma unroll 1
      for (int cc = 0; cc < 4; ++cc) {
        uint32_t o[32];
        if (own) {
          tmem_ld32(tO + 32u * cc, o);
        } else {
#pragma unroll
          for (int x = 0; x < 32; ++x) o[x] = 0u;
        }
        if (kAlt && have1) {
          uint32_t o1[32];
          tmem_ld32(tO + 128u + 32u * cc, o1);  // warpgroup 1's O
#pragma unroll
          for (int x = 0; x < 32; ++x) o[x] = u32(fmaf(w1, f32(o1[x]), w0 * f32(o[x])));
        }
        if (valid_row) {
#pragma unroll
          for (int x = 0; x < 32; x += 4)
            *reinterpret_cast<float4*>(out + 32 * cc + x) =
                have ? make_float4(f32(o[x]), f32(o[x + 1]), f32(o[x + 2]), f32(o[x + 3]))
                     : make_float4(0.f, 0.f, 0.f, 0.f);
        }
      }
      if (valid_row) {
        out[128] = have ? m_ref : -INFINITY;
        out[129] = have ? l : 0.f;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kW1Mma) {
    tc_fence_after();
    tmem_dealloc(tbase, 512);
  }
}

// =========================== combine ========================================
// One warp per query row: merge the split partials of its pass-1 (b, h, chunk).
__global__ void __launch_bounds__(128) k_tc_combine(const TcArgs a) {
  pdl_trigger();
  pdl_wait();  // the partials come from pass 1
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rows = a.B * a.Hq * a.w;
  const int r = blockIdx.x * 4 + warp;
  if (r >= rows) return;
  const int b = r / (a.Hq * a.w);
  const int hq = (r / a.w) % a.Hq;
  const int t = r % a.w;
  const int h = hq / a.G;
  const int gr = (hq % a.G) * a.w + t;
  const int chunk = gr / a.rows1, rr = gr % a.rows1;
  const int cta0 = a.cta_base1[b] + (h * a.chunks1 + chunk) * a.splits1[b];
  const int np = a.splits1[b];
  auto P = [&](int i) { return a.partial + ((size_t)(cta0 + i) * a.rows1 + rr) * kPartStride; };
  // The first kFly partial rows of O are requested before anything else, so
  // that they travel with the (max, normaliser) pairs: one round trip for up
  // to kFly partials.  Lanes take the pairs in parallel, 32 at a time: M,
  // then the weights 2^(m_i - M) and L = sum_i w_i l_i; the weights of the
  // first 32 partials stay in the lanes that loaded them.
  constexpr int kFly = 24;
  float4 o[kFly];
#pragma unroll
  for (int k = 0; k < kFly; ++k)
    if (k < np) o[k] = *reinterpret_cast<const float4*>(P(k) + lane * 4);
  float M = -INFINITY, m_own = -INFINITY, l_own = 0.f;
  for (int i = lane; i < np; i += 32) {
    const float2 ml = *reinterpret_cast<const float2*>(P(i) + 128);
    if (i == lane) { m_own = ml.x; l_own = ml.y; }
    M = fmaxf(M, ml.x);
  }
  M = warp_max(M);
  const float w_own = (m_own == -INFINITY) ? 0.f : ex2(m_own - M);
  float lpart = w_own * l_own;
  for (int i = lane + 32; i < np; i += 32) {
    const float2 ml = *reinterpret_cast<const float2*>(P(i) + 128);
    lpart = fmaf((ml.x == -INFINITY) ? 0.f : ex2(ml.x - M), ml.y, lpart);
  }
  const float Lsum = warp_sum(lpart);
  // O = sum_i w_i O_i: the rows in flight, then the rest eight at a time
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  auto add = [&](const float4& v, float wg) {
    acc.x = fmaf(wg, v.x, acc.x);
    acc.y = fmaf(wg, v.y, acc.y);
    acc.z = fmaf(wg, v.z, acc.z);
    acc.w = fmaf(wg, v.w, acc.w);
  };
#pragma unroll
  for (int k = 0; k < kFly; ++k)
    if (k < np) add(o[k], __shfl_sync(0xffffffffu, w_own, k));
  for (int i0 = kFly; i0 < np; i0 += 8) {
    float4 r[8];
#pragma unroll
    for (int k = 0; k < 8; ++k)
      r[k] = *reinterpret_cast<const float4*>(P(min(i0 + k, np - 1)) + lane * 4);
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const int i = i0 + k;
      float wg = __shfl_sync(0xffffffffu, w_own, i & 31);
      if (i >= 32) {  // past the first 32 partials: recompute the weight
        const float mi = P(min(i, np - 1))[128];
        wg = (mi == -INFINITY) ? 0.f : ex2(mi - M);
      }
      if (i >= np) wg = 0.f;
      add(r[k], wg);
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

// The attention-only score: the CTA streams K alone through a ring of kRing2
// 32 KB slots and issues only the S^T MMA, into one of two TMEM buffers.
__global__ void __maxnreg__(kMaxRegs2)
k_tc_pass2(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
           const TcArgs a) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const int nqc = a.nqc;
  uint8_t* sRing = smem;
  uint8_t* sQ = smem + kRing2 * kTileBytes;  // nqc rows x 2 boxes
  float4* kf = reinterpret_cast<float4*>(sQ + nqc * 256);     // [nqc/2] (-M'_t, -M'_t+1, -, -)
  uint64_t* bars = reinterpret_cast<uint64_t*>(kf + nqc / 2);  // 5 + 2 kRing2 barriers
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
  pdl_trigger();
  pdl_wait();  // qstat comes from the combine
  if (threadIdx.x < nqc) {
    const int i = threadIdx.x;
    const float4 q = a.qstat[qrow0 + i];  // (M, 1/L, L, ||A||^2)
    reinterpret_cast<float*>(kf)[(i >> 1) * 4 + (i & 1)] = -(q.x + log2f(q.z));  // -M'
  }
  if (warp == kWarpMma) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;

  if (warp == kWarpTma) {
    if (lane == 0) {
      prefetch_tmap(&tmQ); prefetch_tmap(&tmK);
      mbar_expect_tx(BQ, nqc * 256);
      tma_load_2d(smem_u32(sQ), &tmQ, BQ, 0, qrow0);
      tma_load_2d(smem_u32(sQ) + nqc * 128, &tmQ, BQ, 64, qrow0);
      for (int j = 0; j < T && !*abort_flag; ++j) {  // K_j in slot j % kRing2
        const int r = j % kRing2, ph = (j / kRing2) & 1;
        if (!mbar_wait(EMPTY(r), ph ^ 1, kWaitNs)) { fail(a, abort_flag); break; }
        mbar_expect_tx(FULL(r), kTileBytes);
        const uint32_t dst = smem_u32(sRing + r * kTileBytes);
        tma_load_3d(dst, &tmK, FULL(r), 0, (t0 + j) * kTok, z);
        tma_load_3d(dst + kBox, &tmK, FULL(r), 64, (t0 + j) * kTok, z);
      }
    }
  } else if (warp == kWarpMma) {
    const uint32_t IDT = idesc_bf16(128, nqc, false, false);
    bool ok = warp_wait(BQ, 0);
    if (!ok) fail(a, abort_flag);
    const SDesc rd0 = sdesc_split(smem_u32(sRing), 16, 1024);  // ring slot 0
    const SDesc qd = sdesc_split(smem_u32(sQ), 16, 1024);
    const uint32_t nq = (uint32_t)nqc;
    for (int j = 0; j < T && ok && !warp_aborted(abort_flag); ++j) {
      const int s = j & 1, ph = (j >> 1) & 1;
      const int rk = j % kRing2, pk = (j / kRing2) & 1;
      if (!warp_wait(TF(s), ph ^ 1) || !warp_wait(FULL(rk), pk)) {
        fail(a, abort_flag);
        break;
      }
      tc_fence_after();
      const uint32_t klo = rd0.lo + (uint32_t)rk * (kTileBytes >> 4);
      if (lane == 0) {
        const uint32_t dS = tbase + (uint32_t)(s * 256);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ss_w(dS, klo + kslice(kk, 128), rd0.hi, qd.lo + kslice(kk, nq), qd.hi, IDT,
                   kk > 0 ? 1u : 0u);
        mma_commit(EMPTY(rk));
        mma_commit(MD(s));
      }
      __syncwarp();
    }
  } else if (warp < kSimtWarps) {
    // Sixteen warps work on every tile: warp (g, quarter) owns the tokens
    // [32 quarter, +32) of the tile (its TMEM lanes) and the query columns
    // [32 g, min(nqc, 32 g + 32)), and writes its own partial-score plane.
    // A warp with no columns still walks the tiles, hands every buffer back
    // and writes zeros to its plane.
    const int g = warp >> 2, ql = warp & 3;
    const int row = ql * 32 + lane;  // token within the tile
    const uint32_t lane_off = (uint32_t)(ql * 32) << 16;
    const float c = a.c_log2;
    const uint64_t c2 = pk2(c, c);
    const int ch0 = min(nqc / 16, 2 * g), ch1 = min(nqc / 16, 2 * g + 2);  // 16-column chunks
    const int nch = ch1 - ch0;  // 0, 1 or 2 (warp-uniform)
    float* plane = a.parts + (size_t)(chunk * 4 + g) * a.part_stride + (size_t)z * a.n_max;
    for (int j = 0; j < T; ++j) {
      const int s = j & 1, ph = (j >> 1) & 1;
      const int tile0 = (t0 + j) * kTok;
      const int tok = tile0 + row;
      if (!warp_wait(MD(s), ph)) { fail(a, abort_flag); break; }
      if (warp_aborted(abort_flag)) break;
      tc_fence_after();
      const uint32_t tS = tbase + (uint32_t)(s * 256) + lane_off + (uint32_t)(ch0 * 16);
      const bool masked = tile0 + kTok - 1 > L - a.w;
      float acc = 0.f;
      uint32_t r[32];
      if (nch > 0) tmem_ld32(tS, r);  // S^T of chunks ch0, ch0 + 1 (the second unused when nch = 1)
      // the buffer goes back as soon as the columns are in registers
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(TF(s));
      if (nch > 0) acc = attn16(r, kf + ch0 * 8, c2, masked, tok, L, a.w, chunk * nqc, ch0 * 16, c);
      if (nch > 1)
        acc += attn16(r + 16, kf + ch0 * 8 + 8, c2, masked, tok, L, a.w, chunk * nqc,
                      ch0 * 16 + 16, c);
      if (tok < L) plane[tok] = acc;
    }
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

size_t pass1_smem() { return (2 + kStK + kSt1) * (size_t)kTileBytes + kBars1 * 8 + 8 + 128 * 8; }
size_t pass2_smem(int nqc) {
  return kRing2 * (size_t)kTileBytes + (size_t)nqc * 256 + (size_t)nqc / 2 * 16 +
         (5 + 2 * kRing2) * 8 + 8;
}

int num_sms() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n;
}

}  // namespace

// tc_pair.cu
cudaError_t launch_tc_pass2_pair(const TcArgs& a, const CUtensorMap& mQ, const CUtensorMap& mAh,
                                 const CUtensorMap& mAl, const CUtensorMap& mK,
                                 const CUtensorMap& mV, int pairs, cudaStream_t st);

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
                             cudaStream_t st, KernelEvents& kev, int* nparts_used) {
  const bool attn_only = score == DROPKV_SCORE_ATTENTION;
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
  a.nq = a.G * a.w;
  a.chunks1 = plan.chunks1;
  a.rows1 = plan.rows1;
  for (int i = 0; i < lens.B; ++i) a.L[i] = lens.L[i];
  const int budget = std::min(cta_budget > 0 ? cta_budget : num_sms(), kMaxCtas);
  const int units = s.Hkv * plan.chunks;    // pass 2
  tc_splits(lens, units, std::max(budget, units * lens.B), a.splits);
  a.cta_base[0] = 0;
  for (int i = 0; i < lens.B; ++i) a.cta_base[i + 1] = a.cta_base[i] + units * a.splits[i];
  const int ctas = a.cta_base[lens.B];
  const int units1 = s.Hkv * plan.chunks1;  // pass 1
  tc_splits(lens, units1, std::max(budget, units1 * lens.B), a.splits1);
  a.cta_base1[0] = 0;
  for (int i = 0; i < lens.B; ++i) a.cta_base1[i + 1] = a.cta_base1[i] + units1 * a.splits1[i];
  const int ctas1 = a.cta_base1[lens.B];
  a.chunks2 = plan.chunks2;
  a.nqc2 = plan.nqc2;
  const int units2 = s.Hkv * plan.chunks2;  // pair pass 2, in CTA pairs
  tc_splits(lens, units2, std::max(budget / 2, units2 * lens.B), a.splits2);
  a.cta_base2[0] = 0;
  for (int i = 0; i < lens.B; ++i) a.cta_base2[i + 1] = a.cta_base2[i] + units2 * a.splits2[i];
  const int pairs = a.cta_base2[lens.B];
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
  // the pair pass loads, per query half of nqc2 / nh columns, half the rows per CTA
  const int nh2 = plan.nqc2 > 128 ? 2 : 1;
  const uint32_t box2 = attn_only ? (uint32_t)plan.nqc : (uint32_t)(plan.nqc2 / nh2 / 2);
  if (!map_2d(&mQ1, q, rows, (uint32_t)a.qbox_rows) || !map_2d(&mQ2, q, rows, box2) ||
      !map_3d(&mK, k, (uint64_t)lens.B * s.Hkv, (uint64_t)s.n_max) ||
      !map_3d(&mV, v, (uint64_t)lens.B * s.Hkv, (uint64_t)s.n_max) ||
      !map_2d(&mAh, a.ahi, rows, box2) || !map_2d(&mAl, a.alo, rows, box2))
    return cudaErrorNotSupported;

  const size_t sm1 = pass1_smem(), sm2 = pass2_smem(plan.nqc);
  // one query tile per chunk: the two softmax warpgroups alternate token tiles
  const bool alt1 = plan.rows1 <= 128;
  auto* pass1 = alt1 ? k_tc_pass1<true> : k_tc_pass1<false>;
  cudaError_t e = cudaFuncSetAttribute(pass1, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)sm1);
  if (e == cudaSuccess && !alt1) {
    // the register split of the two-query-tile schedule assumes the launch's
    // kRegs1 registers a thread; any other count would leave its raise waiting
    cudaFuncAttributes fa;
    e = cudaFuncGetAttributes(&fa, pass1);
    if (e == cudaSuccess && fa.numRegs != kRegs1) return cudaErrorInvalidConfiguration;
  }
  if (e == cudaSuccess && attn_only)  // the attention-only control; DropKV runs the pair kernel
    e = cudaFuncSetAttribute(k_tc_pass2, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm2);
  if (e != cudaSuccess) return e;
  *nparts_used = 4 * (attn_only ? plan.chunks : plan.chunks2);

  kev.begin(st);
  pass1<<<ctas1, kThreads1, sm1, st>>>(mQ1, mK, mV, a);
  kev.end(st);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  kev.begin(st);
  e = launch_ex(k_tc_combine, dim3((unsigned)((rows + 3) / 4)), dim3(128), 0, st, true, 1, a);
  kev.end(st);
  if (e != cudaSuccess) return e;
  kev.begin(st);
  if (attn_only) {
    e = launch_ex(k_tc_pass2, dim3(ctas), dim3(kThreads2), sm2, st, true, 1, mQ2, mK, a);
  } else {
    e = launch_tc_pass2_pair(a, mQ2, mAh, mAl, mK, mV, pairs, st);
  }
  kev.end(st);
  return e;
}

}  // namespace dropkv
