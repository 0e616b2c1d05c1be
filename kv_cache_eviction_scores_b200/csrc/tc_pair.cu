// tc_pair.cu -- second scoring pass on CTA pairs (tcgen05 cta_group::2).
//
// What is computed (write-up "DropKV：精确单项输出扰动评分组件", section 核心公式):
// for every token j of a KV head and every window query t of its group, with
// the final max M, normaliser L and output A of query t from the first pass,
//     p = 2^(x c - M') (M' = M + log2 L),  ratio = p / (1 - p),
//     s_j += ratio^2 (||A||^2 - 2 A.v_j + ||v_j||^2),
// summed over all G*w queries of the group (the epilogue divides by G).
//
// Layout.  Two CTAs of a cluster process 256 tokens per step: each CTA owns
// one 128-token tile of its own contiguous token range, taken from its end
// down (the M = 256 MMA takes 128 rows of A from each CTA), and the nqc <= 256 query columns of the chunk
// are split between them (each CTA holds nqc / 2 rows of Q, -2A_hi and -2A_lo,
// the B operand's halves).  Per step the even CTA issues
//     S^T = K Q^T                     into TMEM columns [0, nqc)
//     D   = V (-2A_hi)^T [+ V (-2A_lo)^T]   into TMEM columns [256, 256 + nqc)
// and commits to barriers of both CTAs.  The score warps of each CTA turn S^T
// into ratio^2 (kept in registers) and hand the S columns back, then read D
// and accumulate, and hand the D columns back: S of step i + 1 overlaps the D
// arithmetic of step i, and D of step i + 1 the S arithmetic of step i + 1.
// Halving each CTA's operand reads (compared with one CTA per 128-row MMA)
// keeps the tensor pipe's shared-memory traffic well under the SM's bandwidth.
//
// Every wait is bounded (2 s of %globaltimer); on expiry the kernel records
// DROPKV_ERR_TIMEOUT, every role leaves its loop, and the CTAs meet at the
// hardware cluster barrier before freeing TMEM, so neither leaves while the
// other may still address its shared memory or TMEM.
#include <cuda.h>
#include <string.h>

#include "tc_common.cuh"

namespace dropkv {
namespace {

constexpr int kRingP = 4;          // 32 KB K/V slots per CTA
constexpr int kThreadsP = (kSimtWarps + 2) * 32;
constexpr uint32_t kColD = 256;    // D columns start here

// Fast path of phase A for 16 query columns: ratio^2 for every p < 2^-4 with
// the series p (1 + p (1 + p (1 + p (1 + p)))) of p / (1 - p) (truncation
// error p^5 / (1 - p) <= 1.0e-6 relative).  kf holds (-M'_t, -M'_t+1,
// ||A_t||^2, ||A_t+1||^2) per column pair.
__device__ __forceinline__ void pairA_fast(const uint32_t (&r)[16], const float4* kf, uint64_t c2,
                                           uint64_t (&r2)[8], float& pmax) {
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
    r2[i] = fmul2(ratio, ratio);
  }
}

// Careful path of phase A, out of line: the causal mask (and tokens this CTA
// does not own), ratio = e / (L - e) with the singular check when p >= 2^-8.
// out[u] = ratio^2 of column col0 + u, 0 where the token is not visible.
__device__ __noinline__ void pairA_careful(const uint32_t* r, int col0, int tok, bool valid,
                                           bool masked, int L, int w, int crow0,
                                           const float4* qstat_rows, float c, int* sing,
                                           float* out) {
#pragma unroll 1
  for (int u = 0; u < 16; ++u) {
    const int col = col0 + u;
    const float4 k = qstat_rows[col];  // (M, 1/L, L, ||A||^2)
    const bool vis = valid && (!masked || tok <= L - w + (crow0 + col) % w);
    const float e = ex2(fmaf(f32(r[u]), c, -k.x));
    const float p = e * k.y;
    float ratio = fmaf(p, fmaf(p, p, p), p);
    if (vis && p >= 0.00390625f) {
      const float den = k.z - e;  // (1 - p) L
      if (!(den > 0.f)) *sing = 1;
      ratio = __fdiv_rn(e, den);
    }
    out[u] = vis ? ratio * ratio : 0.f;
  }
}

// ||a - v||^2 taken directly (fp32 a, bf16 v, both from global memory).  Used
// only where the expansion ||a||^2 + ||v||^2 - 2 a.v cancels by more than 32x.
__device__ __noinline__ float pair_direct_sqdist(const float* A, const __nv_bfloat16* v) {
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

// Careful path of phase B, out of line: ratio^2 (r2, 0 where invisible) times
// the squared distance, recomputed directly where the expansion cancels by
// more than 32x.
__device__ __noinline__ float pairB_careful(const uint32_t* d, const float* r2, int col0,
                                            const float4* qstat_rows, float nv, const float* arows,
                                            const __nv_bfloat16* vrow) {
  float acc = 0.f;
#pragma unroll 1
  for (int u = 0; u < 16; ++u) {
    if (!(r2[u] > 0.f)) continue;  // invisible (or an exact zero weight)
    const float base = qstat_rows[col0 + u].w + nv;
    float zt = base + f32(d[u]);
    if (zt < 0.03125f * base) zt = pair_direct_sqdist(arows + (size_t)(col0 + u) * kHd, vrow);
    acc = fmaf(r2[u], zt, acc);
  }
  return acc;
}

__global__ void __maxnreg__(112)
k_tc_pass2_pair(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmAhi,
                const __grid_constant__ CUtensorMap tmAlo, const __grid_constant__ CUtensorMap tmK,
                const __grid_constant__ CUtensorMap tmV, const TcArgs a) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const int nqc = a.nqc2, half = nqc / 2;
  uint8_t* sRing = smem;                          // kRingP slots
  uint8_t* sQ = smem + kRingP * kTileBytes;       // half rows x 2 boxes
  uint8_t* sAh = sQ + half * 256;
  uint8_t* sAl = sAh + half * 256;
  float4* kf = reinterpret_cast<float4*>(sAl + half * 256);  // [nqc/2] fast-path constants
  float* nAmax = reinterpret_cast<float*>(kf + half);           // [16] max ||A||^2 per 16 columns
  uint64_t* bars = reinterpret_cast<uint64_t*>(nAmax + 16);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 6 + 2 * kRingP);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  // the smem layout must sit at the same offsets in both CTAs; a misaligned
  // base is reported and both CTAs still take the cluster barriers below
  const bool aligned = (smem_u32(smem) & 1023u) == 0;
  int b, h, chunk, t0, t1;
  decode_plan(a, a.splits2, a.cta_base2, a.chunks2, blockIdx.x >> 1, b, h, chunk, t0, t1);
  const int T = t1 - t0;
  const int steps = (T + 1) / 2;
  const int my0 = leader ? t0 : t0 + steps;          // this CTA's first tile
  const int my_n = leader ? steps : T - steps;        // and its tile count
  // tiles are taken from the end of the range down: pass 1 walked the same
  // ranges upwards, so the first tiles here are the ones still in L2
  auto tile_at = [&](int st) { return my0 + my_n - 1 - st; };
  const int L = a.L[b];
  const int z = b * a.Hkv + h;
  const int qrow0 = z * a.nq + chunk * nqc;           // the chunk's first query row
  // barriers (leader's copies gather both CTAs): BQ, FULL[r] -- arrivals of
  // both producers; EMPTY[r], S_READY, D_READY -- the leader's commits,
  // multicast to both CTAs; S_FREE, D_FREE -- the 32 score warps of the pair
  const uint32_t BQ = smem_u32(&bars[0]);
  const uint32_t SREADY = smem_u32(&bars[1]), DREADY = smem_u32(&bars[2]);
  const uint32_t SFREE = smem_u32(&bars[3]), DFREE = smem_u32(&bars[4]);
  auto FULL = [&](int r) { return smem_u32(&bars[5 + r]); };
  auto EMPTY = [&](int r) { return smem_u32(&bars[5 + kRingP + r]); };
  const uint32_t FIN = smem_u32(&bars[5 + 2 * kRingP]);  // the leader's MMAs are all done
  if (threadIdx.x == 0) {
    mbar_init(BQ, 2);
    mbar_init(SREADY, 1); mbar_init(DREADY, 1);
    mbar_init(SFREE, 2 * kSimtWarps); mbar_init(DFREE, 2 * kSimtWarps);
    for (int r = 0; r < kRingP; ++r) {
      mbar_init(FULL(r), 2); mbar_init(EMPTY(r), 1);
    }
    mbar_init(FIN, 1);
    *abort_flag = aligned ? 0 : 1;
    if (!aligned) atomicMax(a.status, (int)DROPKV_ERR_CUDA);
    fence_mbar_init();
  }
  pdl_trigger();
  pdl_wait();  // qstat, A and ||v||^2 come from the combine and pass 1
  // per-column constants of the whole chunk (each CTA's score warps see all
  // nqc columns of its tokens)
  for (int i = threadIdx.x; i < nqc; i += blockDim.x) {
    const float4 q = a.qstat[qrow0 + i];  // (M, 1/L, L, ||A||^2)
    float* kff = reinterpret_cast<float*>(kf);
    kff[(i >> 1) * 4 + (i & 1)] = -(q.x + log2f(q.z));  // -M' folds 1/L into the exponent
    kff[(i >> 1) * 4 + 2 + (i & 1)] = q.w;
  }
  if (threadIdx.x < 16) nAmax[threadIdx.x] = 0.f;
  if (warp == kWarpMma) {
    tmem_alloc2(smem_u32(tmem_slot), 512);
    tmem_relinquish2();
    tc_fence_before();
  }
  __syncthreads();
  for (int i = threadIdx.x; i < nqc; i += blockDim.x)  // ||A||^2 >= 0: float bits order as ints
    atomicMax(reinterpret_cast<int*>(nAmax) + i / 16, __float_as_int(a.qstat[qrow0 + i].w));
  // Does A need its low part?  The same decision in both CTAs: the largest
  // ||A||^2 of the chunk against the smallest ||v_j||^2 of the pair's tiles
  // (-2A rounded to bf16 moves ||A - v||^2 >= (||v|| - ||A||)^2 by at most a
  // relative 2^-7 rho / (1 - rho)^2, rho = ||A|| / ||v|| <= 0.0283: 2.4e-4).
  bool need = false;
  __syncthreads();
  {
    float namx = 0.f;
    for (int i = 0; i < (nqc + 15) / 16; ++i) namx = fmaxf(namx, nAmax[i]);
    for (int i = threadIdx.x; i < T * a.chunks1; i += blockDim.x) {
      const float tm = a.tmin[((size_t)z * a.ntmax + t0) * a.chunks1 + i];
      if (!(namx <= kLoSkip * tm)) need = true;  // NaN-safe
    }
  }
  const bool lo = __syncthreads_or(need) != 0;
  // every barrier of both CTAs is initialised before any remote arrival
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;

  if (warp == kWarpTma) {
    if (lane == 0 && !*abort_flag) {
      prefetch_tmap(&tmQ); prefetch_tmap(&tmAhi); prefetch_tmap(&tmAlo);
      prefetch_tmap(&tmK); prefetch_tmap(&tmV);
      // this CTA's half of the query-side operands; completion counted at the leader
      const uint32_t cBQ = mapa_u32(BQ, 0);
      mbar_expect_tx_cluster(cBQ, (uint32_t)((lo ? 3 : 2) * half * 256));
      const int hrow = qrow0 + (int)rank * half;
      tma_load_2d_pair(smem_u32(sQ), &tmQ, cBQ, 0, hrow);
      tma_load_2d_pair(smem_u32(sQ) + half * 128, &tmQ, cBQ, 64, hrow);
      tma_load_2d_pair(smem_u32(sAh), &tmAhi, cBQ, 0, hrow);
      tma_load_2d_pair(smem_u32(sAh) + half * 128, &tmAhi, cBQ, 64, hrow);
      if (lo) {
        tma_load_2d_pair(smem_u32(sAl), &tmAlo, cBQ, 0, hrow);
        tma_load_2d_pair(smem_u32(sAl) + half * 128, &tmAlo, cBQ, 64, hrow);
      }
      // K_i at load 2i, V_i at 2i + 1; a step past this CTA's tiles only arrives
      for (int i = 0; i < 2 * steps && !*abort_flag; ++i) {
        const int r = i % kRingP, ph = (i / kRingP) & 1;
        if (!mbar_wait(EMPTY(r), ph ^ 1, kWaitNs)) { fail(a, abort_flag); break; }
        const uint32_t cF = mapa_u32(FULL(r), 0);
        const int st = i >> 1;
        if (st < my_n) {
          mbar_expect_tx_cluster(cF, kTileBytes);
          const uint32_t dst = smem_u32(sRing + r * kTileBytes);
          const CUtensorMap* m = (i & 1) ? &tmV : &tmK;
          const int row = tile_at(st) * kTok;
          tma_load_3d_pair(dst, m, cF, 0, row, z);
          tma_load_3d_pair(dst + kBox, m, cF, 64, row, z);
        } else {
          mbar_arrive_cluster(cF);
        }
      }
    }
  } else if (warp == kWarpMma) {
    if (leader) {
      const uint32_t IDT = idesc_bf16(256, nqc, false, false);
      bool ok = !warp_aborted(abort_flag);
      if (ok && !(ok = __all_sync(0xffffffffu, mbar_wait_cluster(BQ, 0, kWaitNs))))
        fail(a, abort_flag);
      const SDesc rd0 = sdesc_split(smem_u32(sRing), 16, 1024);
      const SDesc qd = sdesc_split(smem_u32(sQ), 16, 1024), hd = sdesc_split(smem_u32(sAh), 16, 1024),
                  ld = sdesc_split(smem_u32(sAl), 16, 1024);
      const uint32_t hq = (uint32_t)half;
      for (int i = 0; i < steps && ok && !warp_aborted(abort_flag); ++i) {
        const int rk = (2 * i) % kRingP, pk = ((2 * i) / kRingP) & 1;
        const int rv = (2 * i + 1) % kRingP, pv = ((2 * i + 1) / kRingP) & 1;
        const uint32_t pph = (uint32_t)((i - 1) & 1);
        // S^T = K Q^T once both CTAs' K tiles are in and the S columns are free
        if (!__all_sync(0xffffffffu, mbar_wait_cluster(FULL(rk), pk, kWaitNs)) ||
            (i > 0 && !__all_sync(0xffffffffu, mbar_wait_cluster(SFREE, pph, kWaitNs)))) {
          fail(a, abort_flag);
          break;
        }
        tc_fence_after();
        if (lane == 0) {
          const uint32_t klo = rd0.lo + (uint32_t)rk * (kTileBytes >> 4);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma2_ss_w(tbase, klo + kslice(kk, 128), rd0.hi, qd.lo + kslice(kk, hq), qd.hi, IDT,
                      kk > 0 ? 1u : 0u);
          mma2_commit_mc(EMPTY(rk), 3);
          mma2_commit_mc(SREADY, 3);
        }
        __syncwarp();
        // D = V (-2A)^T once both V tiles are in and the D columns are free
        if (!__all_sync(0xffffffffu, mbar_wait_cluster(FULL(rv), pv, kWaitNs)) ||
            (i > 0 && !__all_sync(0xffffffffu, mbar_wait_cluster(DFREE, pph, kWaitNs)))) {
          fail(a, abort_flag);
          break;
        }
        tc_fence_after();
        if (lane == 0) {
          const uint32_t vlo = rd0.lo + (uint32_t)rv * (kTileBytes >> 4);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma2_ss_w(tbase + kColD, vlo + kslice(kk, 128), rd0.hi, hd.lo + kslice(kk, hq), hd.hi,
                      IDT, kk > 0 ? 1u : 0u);
          if (lo) {
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
              mma2_ss_w(tbase + kColD, vlo + kslice(kk, 128), rd0.hi, ld.lo + kslice(kk, hq),
                        ld.hi, IDT, 1u);
          }
          mma2_commit_mc(EMPTY(rv), 3);
          mma2_commit_mc(DREADY, 3);
        }
        __syncwarp();
      }
      // whatever was issued (all of it, or less after a timeout) has completed
      // before either CTA frees its TMEM
      if (lane == 0) mma2_commit_mc(FIN, 1);
      __syncwarp();
      if (!__all_sync(0xffffffffu, mbar_wait(FIN, 0, kWaitNs))) fail(a, abort_flag);
    }
  } else if (warp < kSimtWarps) {
    // Sixteen warps per CTA: warp (g, quarter) owns the tokens [32 quarter,
    // +32) of this CTA's tile (its TMEM lanes) and the 16-column chunks
    // [ch0, ch0 + nch) of the query columns, and writes its own partial-score
    // plane (the epilogue sums the four planes of a chunk).
    const int g = warp >> 2, ql = warp & 3;
    const int row = ql * 32 + lane;
    const uint32_t lane_off = (uint32_t)(ql * 32) << 16;
    const float c = a.c_log2;
    const uint64_t c2 = pk2(c, c);
    const int ncht = nqc / 16;
    const int ch0 = g * ncht / 4, nch = (g + 1) * ncht / 4 - ch0;  // 0..4, warp-uniform
    const float4* qrows = a.qstat + qrow0;
    const float* arows = a.attn_f32 + (size_t)qrow0 * kHd;
    float* plane = a.parts + (size_t)(chunk * 4 + g) * a.part_stride + (size_t)z * a.n_max;
    const uint32_t cSFREE = mapa_u32(SFREE, 0), cDFREE = mapa_u32(DFREE, 0);
    const uint32_t tS = tbase + lane_off + (uint32_t)(ch0 * 16);
    const uint32_t tD = tS + kColD;
    auto nv_at = [&](int st) -> float {
      const int tk = tile_at(st) * kTok + row;
      return (st < my_n && tk < L) ? a.nvbuf[(size_t)z * a.ntmax * kTok + tk] : 0.f;
    };
    float nv_next = nv_at(0);
    int sing = 0;
    bool live = !warp_aborted(abort_flag);
    for (int i = 0; i < steps && live; ++i) {
      const bool valid_tile = i < my_n;
      const int tile0 = (valid_tile ? tile_at(i) : my0) * kTok;
      const int tok = tile0 + row;
      const bool valid = valid_tile && tok < L;
      const bool masked = !valid_tile || tile0 + kTok - 1 > L - a.w;  // warp-uniform
      const float nv = nv_next;
      nv_next = nv_at(i + 1);
      const __nv_bfloat16* vrow = a.v + ((size_t)z * a.n_max + (valid ? tok : 0)) * kHd;
      // ---- phase A: ratio^2 of every owned column, then the S columns go back
      if (!__all_sync(0xffffffffu, mbar_wait_cluster(SREADY, (uint32_t)(i & 1), kWaitNs))) {
        fail(a, abort_flag);
        break;
      }
      if (warp_aborted(abort_flag)) break;
      tc_fence_after();
      uint64_t r2[4][8];
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        if (cc >= nch) break;
        uint32_t r[16];
        tmem_ld16(tS + 16u * cc, r);
        bool redo = masked;
        if (!masked) {
          float pmax = 0.f;
          pairA_fast(r, kf + (ch0 + cc) * 8, c2, r2[cc], pmax);
          redo = pmax >= 0.0625f;  // a large p: the series would be short
        }
        if (__any_sync(0xffffffffu, redo)) {
          float t16[16];
          pairA_careful(r, (ch0 + cc) * 16, tok, valid, masked, L, a.w, chunk * nqc, qrows, c,
                        &sing, t16);
#pragma unroll
          for (int k = 0; k < 8; ++k) r2[cc][k] = pk2(t16[2 * k], t16[2 * k + 1]);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(cSFREE);
      // ---- phase B: D of the owned columns; the D columns go back once read
      if (!__all_sync(0xffffffffu, mbar_wait_cluster(DREADY, (uint32_t)(i & 1), kWaitNs))) {
        fail(a, abort_flag);
        break;
      }
      tc_fence_after();
      float acc = 0.f;
      if (nch == 0) {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(cDFREE);
      }
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        if (cc >= nch) break;
        uint32_t d[16];
        tmem_ld16(tD + 16u * cc, d);
        if (cc == nch - 1) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive_cluster(cDFREE);
        }
        // possible cancellation (||A||^2 >= 0.6 ||v||^2) or masked keys: careful
        const bool cb = masked || nAmax[ch0 + cc] >= 0.6f * nv;
        if (__any_sync(0xffffffffu, cb)) {
          float t16[16];
#pragma unroll
          for (int k = 0; k < 8; ++k) upk2(r2[cc][k], t16[2 * k], t16[2 * k + 1]);
          acc += pairB_careful(d, t16, (ch0 + cc) * 16, qrows, nv, arows, vrow);
        } else {
          const uint64_t nv2 = pk2(nv, nv);
          uint64_t a2 = pk2(0.f, 0.f);
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const float4 kq = kf[(ch0 + cc) * 8 + k];
            const uint64_t zt = fadd2(fadd2(pk2(f32(d[2 * k]), f32(d[2 * k + 1])), pk2(kq.z, kq.w)), nv2);
            a2 = ffma2(r2[cc][k], zt, a2);
          }
          float x0, x1;
          upk2(a2, x0, x1);
          acc += x0 + x1;
        }
      }
      if (valid) plane[tok] = acc;
    }
    if (sing) atomicMax(a.status, (int)DROPKV_ERR_SINGULAR);
  }
  // both CTAs' MMAs, TMEM reads and remote arrivals are over before either
  // CTA frees TMEM or leaves
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();
  if (warp == kWarpMma) {
    tc_fence_after();
    tmem_dealloc2(tbase, 512);
  }
}

}  // namespace

size_t pass2_pair_smem(int nqc) {
  return kRingP * (size_t)kTileBytes + 3 * (size_t)(nqc / 2) * 256 + (size_t)(nqc / 2) * 16 +
         16 * 4 + (6 + 2 * kRingP) * 8 + 8;
}

cudaError_t launch_tc_pass2_pair(const TcArgs& a, const CUtensorMap& mQ, const CUtensorMap& mAh,
                                 const CUtensorMap& mAl, const CUtensorMap& mK,
                                 const CUtensorMap& mV, int pairs, cudaStream_t st) {
  const size_t smem = pass2_pair_smem(a.nqc2);
  cudaError_t e = cudaFuncSetAttribute(k_tc_pass2_pair,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  return launch_ex(k_tc_pass2_pair, dim3(2 * pairs), dim3(kThreadsP), smem, st, true, 2, mQ, mAh,
                   mAl, mK, mV, a);
}

}  // namespace dropkv
