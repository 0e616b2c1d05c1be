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
// down (the M = 256 MMA takes 128 rows of A from each CTA).  The chunk's
// nqc <= 256 query columns are processed as nh halves of nqh <= 128 columns;
// for each half both CTAs hold nqh / 2 rows of Q, -2A_hi and -2A_lo (the B
// operand's halves).  Per (step, half) the even CTA issues
//     S^T = K Q_h^T  and  D = V (-2A_hi,h)^T [+ V (-2A_lo,h)^T]
// into one of two TMEM buffers of 256 columns and commits to barriers of both
// CTAs; the score warps of each CTA read S^T and D of their 32 columns 16 at
// a time and hand the buffer back after the last read, so the MMAs of the
// next half overlap this half's arithmetic.  An M = 256, N = 128 pair MMA
// reads 6 KB of shared memory per CTA per 64-cycle K step (4 KB of its own
// tokens, 2 KB of its query rows), against 8 KB for a single-CTA M = 128,
// N = 128 MMA, which alone is the SM's whole shared-memory bandwidth.
//
// Warps: sixteen score warps (four warpgroups), then a producer warpgroup of
// the TMA warp, the MMA warp and two warps that only hand their registers
// over: the producers drop to 64 registers so that the score warps can hold
// 104 (setmaxnreg), which measured 4 % faster than 96 throughout.
//
// Every wait is bounded (2 s of %globaltimer); on expiry the kernel records
// DROPKV_ERR_TIMEOUT, every role leaves its loop, the issued MMAs are waited
// for, and the CTAs meet at the hardware cluster barrier before freeing TMEM,
// so neither leaves while the other may still address its shared memory or
// TMEM.
#include <cuda.h>
#include <string.h>

#include "tc_common.cuh"

namespace dropkv {
namespace {

constexpr int kRingP = 4;          // 32 KB K/V slots per CTA
// sixteen score warps, then the producer warpgroup: the TMA warp, the MMA
// warp and two warps that only give their registers up
constexpr int kThreadsP = (kSimtWarps + 4) * 32;
// registers: launched at kMaxRegs2 each, the producer warpgroup lowers to 64
// and the four score warpgroups raise to 104 (setmaxnreg)
constexpr uint32_t kRegsScoreP = 104, kRegsProdP = 64;
static_assert(kSimtWarps == 16 &&
                  4 * 128 * kRegsScoreP + 128 * kRegsProdP == kThreadsP * kMaxRegs2,
              "register split of the pair pass");

__global__ void __maxnreg__(kMaxRegs2)
k_tc_pass2_pair(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmAhi,
                const __grid_constant__ CUtensorMap tmAlo, const __grid_constant__ CUtensorMap tmK,
                const __grid_constant__ CUtensorMap tmV, const TcArgs a) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const int nqc = a.nqc2;
  const int nh = nqc > 128 ? 2 : 1;       // query halves per step
  const int nqh = nqc / nh;               // columns per half (multiple of 16, <= 128)
  const int hr = nqh / 2;                 // rows of a half held by each CTA
  const int rows = nqc / 2;               // query rows held by each CTA
  uint8_t* sRing = smem;                          // kRingP slots
  uint8_t* sQ = smem + kRingP * kTileBytes;       // rows x 2 boxes; half h at rows [h hr, +hr)
  uint8_t* sAh = sQ + rows * 256;
  uint8_t* sAl = sAh + rows * 256;
  float4* kf = reinterpret_cast<float4*>(sAl + rows * 256);  // [nqc/2] fast-path constants
  float* nAmax = reinterpret_cast<float*>(kf + nqc / 2);       // [16] max ||A||^2 per 16 columns
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
  // barriers (the leader's copies gather both CTAs): BQ -- both producers
  // announce their query-side bytes; FULL[r] -- the leader announces both
  // CTAs' tile bytes and both CTAs' TMA loads complete on it; TF[2] -- the 32
  // score warps of the pair hand a TMEM buffer back; EMPTY[r], MD[2] -- the
  // leader's commits, multicast to both CTAs; FIN -- the leader's MMAs are done
  const uint32_t BQ = smem_u32(&bars[0]);
  auto MD = [&](int s) { return smem_u32(&bars[1 + s]); };
  auto TF = [&](int s) { return smem_u32(&bars[3 + s]); };
  auto FULL = [&](int r) { return smem_u32(&bars[5 + r]); };
  auto EMPTY = [&](int r) { return smem_u32(&bars[5 + kRingP + r]); };
  const uint32_t FIN = smem_u32(&bars[5 + 2 * kRingP]);
  if (threadIdx.x == 0) {
    mbar_init(BQ, 2);
    for (int s = 0; s < 2; ++s) {
      mbar_init(MD(s), 1); mbar_init(TF(s), 2 * kSimtWarps);
    }
    for (int r = 0; r < kRingP; ++r) {
      mbar_init(FULL(r), 1); mbar_init(EMPTY(r), 1);
    }
    mbar_init(FIN, 1);
    *abort_flag = aligned ? 0 : 1;
    if (!aligned) atomicMax(a.status, (int)DROPKV_ERR_CUDA);
    fence_mbar_init();
  }
  if (warp == kWarpMma) {
    tmem_alloc2(smem_u32(tmem_slot), 512);
    tmem_relinquish2();
    tc_fence_before();
  }
  pdl_trigger();
  pdl_wait();  // qstat, A and ||v||^2 come from the combine and pass 1
  // per-column constants of the whole chunk
  for (int i = threadIdx.x; i < nqc; i += blockDim.x) {
    const float4 q = a.qstat[qrow0 + i];  // (M, 1/L, L, ||A||^2)
    float* kff = reinterpret_cast<float*>(kf);
    kff[(i >> 1) * 4 + (i & 1)] = -(q.x + log2f(q.z));  // -M' folds 1/L into the exponent
    kff[(i >> 1) * 4 + 2 + (i & 1)] = q.w;
  }
  if (threadIdx.x < 16) nAmax[threadIdx.x] = 0.f;
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

  if (warp >= kSimtWarps) {
    setmaxnreg_dec<kRegsProdP>();
    if (warp == kWarpTma) {
      if (lane == 0 && !*abort_flag) {
        prefetch_tmap(&tmQ); prefetch_tmap(&tmAhi); prefetch_tmap(&tmAlo);
        prefetch_tmap(&tmK); prefetch_tmap(&tmV);
        // this CTA's rows of every half of the query-side operands; completion
        // counted at the leader
        const uint32_t cBQ = mapa_u32(BQ, 0);
        mbar_expect_tx_cluster(cBQ, (uint32_t)((lo ? 3 : 2) * rows * 256));
        for (int hh = 0; hh < nh; ++hh) {
          const int grow = qrow0 + hh * nqh + (int)rank * hr;  // global query row
          const uint32_t so = (uint32_t)(hh * hr * 128);       // smem row offset
          tma_load_2d_pair(smem_u32(sQ) + so, &tmQ, cBQ, 0, grow);
          tma_load_2d_pair(smem_u32(sQ) + rows * 128 + so, &tmQ, cBQ, 64, grow);
          tma_load_2d_pair(smem_u32(sAh) + so, &tmAhi, cBQ, 0, grow);
          tma_load_2d_pair(smem_u32(sAh) + rows * 128 + so, &tmAhi, cBQ, 64, grow);
          if (lo) {
            tma_load_2d_pair(smem_u32(sAl) + so, &tmAlo, cBQ, 0, grow);
            tma_load_2d_pair(smem_u32(sAl) + rows * 128 + so, &tmAlo, cBQ, 64, grow);
          }
        }
        // K_i at load 2i, V_i at 2i + 1; the leader announces the bytes of both
        // CTAs' loads of the slot (none for a step past a CTA's tiles)
        for (int i = 0; i < 2 * steps && !*abort_flag; ++i) {
          const int r = i % kRingP, ph = (i / kRingP) & 1;
          if (!mbar_wait(EMPTY(r), ph ^ 1, kWaitNs)) { fail(a, abort_flag); break; }
          const uint32_t cF = mapa_u32(FULL(r), 0);
          const int st = i >> 1;
          if (leader) {
            const int peer_n = T - steps;
            mbar_expect_tx(FULL(r), (uint32_t)kTileBytes *
                                        ((st < my_n ? 1u : 0u) + (st < peer_n ? 1u : 0u)));
          }
          if (st < my_n) {
            const uint32_t dst = smem_u32(sRing + r * kTileBytes);
            const CUtensorMap* m = (i & 1) ? &tmV : &tmK;
            const int row = tile_at(st) * kTok;
            tma_load_3d_pair(dst, m, cF, 0, row, z);
            tma_load_3d_pair(dst + kBox, m, cF, 64, row, z);
          }
        }
      }
    } else if (warp == kWarpMma) {
      if (leader) {
        const uint32_t IDT = idesc_bf16(256, nqh, false, false);
        bool ok = !warp_aborted(abort_flag);
        if (ok && !(ok = __all_sync(0xffffffffu, mbar_wait_cluster(BQ, 0, kWaitNs))))
          fail(a, abort_flag);
        const SDesc rd0 = sdesc_split(smem_u32(sRing), 16, 1024);
        const SDesc qd = sdesc_split(smem_u32(sQ), 16, 1024);
        const SDesc hd = sdesc_split(smem_u32(sAh), 16, 1024);
        const SDesc ld = sdesc_split(smem_u32(sAl), 16, 1024);
        const uint32_t rw = (uint32_t)rows;
        int k = 0;  // (step, half) item: TMEM buffer k & 1
        for (int i = 0; i < steps && ok && !warp_aborted(abort_flag); ++i) {
          const int rk = (2 * i) % kRingP, pk = ((2 * i) / kRingP) & 1;
          const int rv = (2 * i + 1) % kRingP, pv = ((2 * i + 1) / kRingP) & 1;
          // both CTAs' K and V tiles of this step
          if (!__all_sync(0xffffffffu, mbar_wait(FULL(rk), pk, kWaitNs)) ||
              !__all_sync(0xffffffffu, mbar_wait(FULL(rv), pv, kWaitNs))) {
            ok = false;
            break;
          }
          for (int hh = 0; hh < nh; ++hh, ++k) {
            const int s = k & 1;
            // the buffer's previous item has been read by all 32 score warps
            if (k >= 2 &&
                !__all_sync(0xffffffffu, mbar_wait(TF(s), (uint32_t)(((k >> 1) - 1) & 1),
                                                           kWaitNs))) {
              ok = false;
              break;
            }
            tc_fence_after();
            if (lane == 0) {
              const uint32_t dS = tbase + (uint32_t)(s * 256), dD = dS + 128u;
              const uint32_t klo = rd0.lo + (uint32_t)rk * (kTileBytes >> 4);
              const uint32_t vlo = rd0.lo + (uint32_t)rv * (kTileBytes >> 4);
              const uint32_t ho = (uint32_t)(hh * hr * 128) >> 4;  // half's row offset
#pragma unroll
              for (int kk = 0; kk < 8; ++kk)
                mma2_ss_w(dS, klo + kslice(kk, 128), rd0.hi, qd.lo + ho + kslice(kk, rw), qd.hi,
                          IDT, kk > 0 ? 1u : 0u);
              if (hh == nh - 1) mma2_commit_mc(EMPTY(rk), 3);  // the last reader of K_i
#pragma unroll
              for (int kk = 0; kk < 8; ++kk)
                mma2_ss_w(dD, vlo + kslice(kk, 128), rd0.hi, hd.lo + ho + kslice(kk, rw), hd.hi,
                          IDT, kk > 0 ? 1u : 0u);
              if (lo) {
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                  mma2_ss_w(dD, vlo + kslice(kk, 128), rd0.hi, ld.lo + ho + kslice(kk, rw), ld.hi,
                            IDT, 1u);
              }
              if (hh == nh - 1) mma2_commit_mc(EMPTY(rv), 3);  // the last reader of V_i
              mma2_commit_mc(MD(s), 3);
            }
            __syncwarp();
          }
        }
        if (!ok) fail(a, abort_flag);
        // whatever was issued (all of it, or less after a timeout) has completed
        // before either CTA frees its TMEM
        if (lane == 0) mma2_commit_mc(FIN, 1);
        __syncwarp();
        if (!__all_sync(0xffffffffu, mbar_wait(FIN, 0, kWaitNs))) fail(a, abort_flag);
      }
    }
  } else {
    setmaxnreg_inc<kRegsScoreP>();
    // Sixteen warps per CTA: warp (g, quarter) owns the tokens [32 quarter,
    // +32) of this CTA's tile (its TMEM lanes) and the query columns
    // [32 g, min(nqh, 32 g + 32)) of every half, and writes its own
    // partial-score plane (the epilogue sums the four planes of a chunk).
    const int g = warp >> 2, ql = warp & 3;
    const int row = ql * 32 + lane;
    const uint32_t lane_off = (uint32_t)(ql * 32) << 16;
    const float c = a.c_log2;
    const uint64_t c2 = pk2(c, c);
    const int ch0 = min(nqh / 16, 2 * g), ch1 = min(nqh / 16, 2 * g + 2);  // 16-column chunks
    const int nch = ch1 - ch0;  // 0, 1 or 2 (warp-uniform)
    const float4* qrows = a.qstat + qrow0;
    const float* arows = a.attn_f32 + (size_t)qrow0 * kHd;
    float* plane = a.parts + (size_t)(chunk * 4 + g) * a.part_stride + (size_t)z * a.n_max;
    const uint32_t cTF0 = mapa_u32(TF(0), 0), cTF1 = mapa_u32(TF(1), 0);
    auto nv_at = [&](int st) -> float {
      const int tk = tile_at(st) * kTok + row;
      return (st < my_n && tk < L) ? a.nvbuf[(size_t)z * a.ntmax * kTok + tk] : 0.f;
    };
    float nv_next = nv_at(0);
    int sing = 0;
    int k = 0;
    bool live = !warp_aborted(abort_flag);
    for (int i = 0; i < steps && live; ++i) {
      const bool valid_tile = i < my_n;  // warp-uniform
      const int tile0 = (valid_tile ? tile_at(i) : my0) * kTok;
      const int tok = tile0 + row;
      const bool valid = valid_tile && tok < L;
      // only the window's last w keys can be hidden from a window query: the
      // warp's 32 tokens need the mask when they reach past L - w (warp-uniform)
      const bool masked = tile0 + 32 * ql + 31 > L - a.w;
      const float nv = nv_next;
      nv_next = nv_at(i + 1);
      const __nv_bfloat16* vrow = a.v + ((size_t)z * a.n_max + (valid ? tok : 0)) * kHd;
      float acc = 0.f;
      for (int hh = 0; hh < nh; ++hh, ++k) {
        const int s = k & 1;
        if (!__all_sync(0xffffffffu, mbar_wait(MD(s), (uint32_t)((k >> 1) & 1), kWaitNs))) {
          fail(a, abort_flag);
          live = false;
          break;
        }
        if (warp_aborted(abort_flag)) { live = false; break; }
        tc_fence_after();
        const uint32_t tS = tbase + (uint32_t)(s * 256) + lane_off + (uint32_t)(ch0 * 16);
        const uint32_t tD = tS + 128u;
        const int hc0 = hh * nqh;  // the half's first column within the chunk
        auto release = [&]() {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive_remote(s ? cTF1 : cTF0);
        };
        // score of 16 columns (chunk ch of the half) from S^T in r[0..15] and D
        // in r[16..31]
        auto chunk_score = [&](const uint32_t(&r)[32], int ch) -> float {
          uint64_t a2 = pk2(0.f, 0.f);
          float pmax = 0.f;
          const float4* kfc = kf + (hc0 / 2) + ch * 8;
          if (!masked) {
            fast16<false>(r, kfc, c2, pk2(nv, nv), a2, pmax);
          } else {
            // the window's causal mask: column u is the window query at
            // position L - w + (chunk * nqc + hc0 + 16 ch + u) mod w
            fast16<true>(r, kfc, c2, pk2(nv, nv), a2, pmax, tok, L - a.w,
                         (chunk * nqc + hc0 + ch * 16) % a.w, a.w);
          }
          // a large p (>= 2^-4: outside the fast ratio's interval) or possible
          // cancellation (||A||^2 >= 0.6 ||v||^2): the careful path (lanes past
          // L write nothing and do not vote)
          const bool redo = valid && (pmax >= 0.0625f || nAmax[hc0 / 16 + ch] >= 0.6f * nv);
          if (__any_sync(0xffffffffu, redo)) {
            uint32_t rc[32];
#pragma unroll
            for (int q = 0; q < 32; ++q) rc[q] = r[q];
            return careful16(rc, hc0 + ch * 16, tok, masked, L, a.w, chunk * nqc, qrows, c, nv,
                             arows, vrow, &sing);
          }
          float x0, x1;
          upk2(a2, x0, x1);
          return x0 + x1;
        };
        if (nch == 0 || !valid_tile) {
          // no columns, or a step past this CTA's tiles: only hand the buffer back
          release();
          continue;
        }
        uint32_t r[32];
        tmem_ld16x2(tS, tD, r);  // chunk ch0: 16 columns of S^T and of D
        if (nch == 1) release();
        acc += chunk_score(r, ch0);
        if (nch > 1) {
          tmem_ld16x2(tS + 16u, tD + 16u, r);  // chunk ch0 + 1
          release();
          acc += chunk_score(r, ch0 + 1);
        }
      }
      if (live && valid) plane[tok] = acc;
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
  // the register split assumes the launch's kMaxRegs2 registers a thread; any
  // other count would leave the score warps' raise waiting
  cudaFuncAttributes fa;
  e = cudaFuncGetAttributes(&fa, k_tc_pass2_pair);
  if (e != cudaSuccess) return e;
  if (fa.numRegs != kMaxRegs2) return cudaErrorInvalidConfiguration;
  return launch_ex(k_tc_pass2_pair, dim3(2 * pairs), dim3(kThreadsP), smem, st, true, 2, mQ, mAh,
                   mAl, mK, mV, a);
}

}  // namespace dropkv
