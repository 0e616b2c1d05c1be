// select.cu -- exact lowest-score eviction per (b, KV head): thread-block
// clusters of 1 to 8 CTAs run a radix select over a segment's keys and an
// order-preserving compaction, in a single launch.
//
// Write-up "DropKV：精确单项输出扰动评分组件", Algorithm 1 paragraph: after
// pooling and window protection, the lowest-scoring tokens are evicted.  The
// order used is (score ascending, position ascending); NaN sorts above +inf.
//
// Scores map to 32-bit keys whose unsigned order is the float order.  A
// segment (b, h) of L keys is split into kC contiguous ranges, one per CTA of
// a kC-CTA cluster, kC the smallest power of two (<= 8) that leaves every
// range within one 16384-key shared-memory cache; with one CTA the phases
// below are block barriers.  Cluster i takes the i-th longest segment, so
// that when not all clusters fit on the device at once the ones the hardware
// starts later are the short ones.
// The histogram rounds take a range in sub-ranges of 16384 keys, 32
// consecutive keys per thread (one sub-range when it fits the shared-memory
// cache, which then holds it for every phase, and the thread's 32 keys stay
// in registers).
//   rounds 0, 1: every CTA histograms an 11-bit digit of its keys that match
//       the prefix found so far and adds its non-zero bins into the round's
//       histogram of every CTA of the cluster (distributed shared memory
//       atomics; all histograms zeroed before a hardware cluster barrier);
//       after one cluster-wide
//       phase every CTA finds the digit holding the E-th smallest key itself,
//       and counts its own keys below that digit.
//   round 2: the same for the last 10 bits, except that every CTA stores its
//       histogram into its own slot of every CTA, together with its counts
//       below the round-0 and round-1 digits.  After the phase the prefix is
//       the threshold key T, `rem` is how many keys equal to T are evicted
//       (the lowest positions among them), and every CTA knows how many keys
//       below / at T every lower rank holds, without another pass.
//   write: each warp counts the keys < T and == T of its contiguous part of
//       the CTA's range (from the registers when the range is cached); the
//       lower warps' counts order the warps; the warp then walks its part 32
//       consecutive keys at a time (lane = key): ballots give every lane its
//       evicted rank and an == T key's rank among the == T keys, and each lane
//       writes its position straight to its slot of the keep or evict list.
// The rounds are separated by cluster-wide phases.  In the product build they
// are the hardware cluster barrier: the rounds are uniform over a cluster and
// every thread of every CTA reaches every phase, as it reaches the barriers
// after the set-up and at the end (measured 1.6 us per phase faster than
// mbarrier phases).  The self-test build keeps bounded mbarrier phases: a
// wait that gives up records DROPKV_ERR_TIMEOUT in the status word and the
// CTA keeps taking the remaining phase barriers (without the work).  The
// kernel ends on the hardware cluster barrier, so no CTA leaves while another
// may still address its shared memory.  Before that barrier every CTA stores
// whether it gave up into every CTA; after it, if any CTA of the cluster gave
// up, each CTA writes -1 over its share of the segment's keep and evict slots.
// Every data write precedes the barrier, so no stale index survives a timeout.
#include "common.cuh"
#include "internal.h"

namespace dropkv {
namespace {

constexpr int kMaxC = 8;             // the largest cluster (CTAs taking one segment)
constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kBins = 2048;          // rounds 0, 1: 11-bit digits
constexpr int kBins2 = 1024;         // round 2: the last 10 bits
// keys per thread in one sub-range: kPer = 32 (16384-key sub-ranges), or 64
// (32768) where that saves a second wave of clusters
constexpr int kCopies = 4;           // histogram copies (warp % 4), padded apart by one bank
constexpr int kCopyStride = kBins + 1;
constexpr uint64_t kWaitNs = 2000000000ull;

struct SelParams {
  int32_t B, Hkv, n_max;
  int32_t max_keep, max_evict;
  int32_t L[kMaxB];
  int32_t E[kMaxB];                  // evictions per row
  int32_t* status;                   // device status word (0 = OK), or NULL: not reported
  int32_t stall_rank;                // self-test only: this rank withholds its arrivals
                                     // of the first round (-1: none, the product path)
  uint8_t row_order[kMaxB];          // batch rows by decreasing length
  uint64_t wait_ns;                  // limit of every bounded wait
};

__device__ __forceinline__ uint32_t key_of(float s) {
  const uint32_t u = __float_as_uint(s);
  if (s != s) return 0xFFFFFFFFu;  // NaN above everything
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// ---- cluster / distributed shared memory -----------------------------------
__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// address of the same shared-memory variable in CTA `rank` of the cluster
__device__ __forceinline__ uint32_t mapa(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}
__device__ __forceinline__ void dsm_add(uint32_t raddr, uint32_t v) {
  asm volatile("red.shared::cluster.add.u32 [%0], %1;" ::"r"(raddr), "r"(v) : "memory");
}
__device__ __forceinline__ void dsm_st(uint32_t raddr, uint32_t v) {
  asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(raddr), "r"(v) : "memory");
}
__device__ __forceinline__ uint64_t gtimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Block-wide exclusive prefix sum of one int per thread (kThreads threads);
// also returns the block total.  Contains __syncthreads.
__device__ __forceinline__ int block_excl_scan(int v, int& total, int* warp_tot) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_tot[wid] = x;
  __syncthreads();
  int before = 0;
  total = 0;
  for (int i = 0; i < kWarps; ++i) {
    const int t = warp_tot[i];
    if (i < wid) before += t;
    total += t;
  }
  __syncthreads();
  return before + x - v;
}

// One cluster-wide phase: after a block barrier (which orders every thread's
// prior shared / distributed shared memory writes before thread 0), thread 0
// fences at cluster scope and arrives on the phase barrier of every CTA of the
// cluster, then waits (bounded, acquire at cluster scope) for all kC arrivals
// on its own; a second block barrier releases the other threads.  Returns
// false once any wait of this CTA has given up.  `withhold` (self-test only)
// skips the arrivals.
template <int kC>
__device__ bool cluster_phase(uint32_t bar, int& phase, volatile int* fail, int32_t* status,
                              uint64_t limit_ns, bool withhold = false) {
  __syncthreads();
  if (threadIdx.x == 0) {
    asm volatile("fence.acq_rel.cluster;" ::: "memory");
    for (uint32_t r = 0; r < (uint32_t)kC && !withhold; ++r)
      asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(mapa(bar, r))
                   : "memory");
    const uint32_t parity = (uint32_t)(phase & 1);
    const uint64_t t0 = gtimer();
    for (;;) {
      uint32_t done;
      asm volatile(
          "{\n\t.reg .pred p;\n\t"
          "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
          "selp.u32 %0, 1, 0, p;\n\t}"
          : "=r"(done)
          : "r"(bar), "r"(parity)
          : "memory");
      if (done) break;
      if (gtimer() - t0 > limit_ns) {
        *fail = 1;
        if (status) atomicMax(status, (int)DROPKV_ERR_TIMEOUT);
        break;
      }
    }
  }
  __syncthreads();
  ++phase;
  return *fail == 0;
}

// kC: CTAs per cluster (1, 2, 4 or 8); a cluster takes one segment.
// kHw: the rounds' phases are hardware cluster barriers (the product); false
// for the self-test, whose phases are bounded mbarrier waits that one rank's
// withheld arrivals make run out.
// kPer: consecutive keys per thread in one sub-range of kThreads * kPer keys.
// kCached: every CTA's range fits one sub-range and is read from the
// shared-memory key cache in every phase (no global loads after the fill).
template <int kC, int kPer, bool kCached, bool kHw = true>
__global__ void __launch_bounds__(kThreads, 1)
k_select(SelParams p, const float* __restrict__ scores, int32_t* __restrict__ keep_idx,
         int32_t* __restrict__ evict_idx) {
  constexpr int kSub = kThreads * kPer;
  constexpr int kSh = kPer == 64 ? 6 : 5;   // log2(kPer): the cache swizzle's row
  extern __shared__ uint32_t smem_dyn[];     // key cache, histogram copies, round-2 slots
  uint32_t* cached_keys = smem_dyn;          // [kSub] this CTA's range when it fits one sub-range
  uint32_t* loc = smem_dyn + kSub;           // [kCopies][kCopyStride] this CTA's histograms;
                                             // copy 0 then holds this CTA's round totals
  uint32_t* H2 = loc + kCopies * kCopyStride;  // [kC][kBins2] every rank's round-2 histogram
  __shared__ uint32_t H[2][kBins];           // the cluster histograms of rounds 0 and 1
  __shared__ uint32_t bel[kC][2];            // per rank: its keys below the round-0 / -1 digits
  __shared__ uint32_t below[2];              // this CTA's counts below the round-0 / -1 digits
  __shared__ uint32_t cross[2];              // keys < T / == T held by the lower ranks
  __shared__ int32_t warp_tot[kWarps];
  __shared__ uint32_t ctl[2];                // (prefix, rem) after a round
  __shared__ int32_t wsum[2][kWarps];
  __shared__ __align__(8) uint64_t bar;     // the rounds' all-to-all phases: kC arrivals
  __shared__ uint32_t fails[kC];             // per rank: 1 if a wait of that CTA gave up
  __shared__ int fail;
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  const uint32_t rank = kC > 1 ? cluster_rank() : 0u;
  const int cl = blockIdx.x / kC;            // this cluster
  const uint32_t barA = smem_addr(&bar);
  // cluster i takes the i-th longest segment: the hardware starts clusters in
  // order, so when not all fit at once the ones left for later are short
  const int seg = p.row_order[cl / p.Hkv] * p.Hkv + cl % p.Hkv;

  if (tid == 0) {
    if constexpr (kC > 1) {
      asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(barA), "r"(kC) : "memory");
      asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    fail = 0;
  }
  if (tid < kC) fails[tid] = 0;
  for (int i = tid; i < kCopies * kCopyStride; i += kThreads) loc[i] = 0;
  // the set-up above overlaps the previous kernel's tail; the scores may come
  // from that kernel
  pdl_wait();
  int phase = 0;
  bool ok = true;

  {  // the segment's select
    const int b = seg / p.Hkv;
    const int L = p.L[b], E = p.E[b];
    const long long span_ll = (((long long)L + kC - 1) / kC + 31) & ~31ll;
    const int lo = (int)min((long long)L, (long long)rank * span_ll);
    const int hi = (int)min((long long)L, (long long)lo + span_ll);
    const float* s = scores + (size_t)seg * p.n_max;
    if (tid == 0) {
      ctl[0] = 0;
      ctl[1] = (uint32_t)E;
    }
    for (int i = tid; i < 2 * kBins; i += kThreads) (&H[0][0])[i] = 0;
    for (int i = tid; i < kC * kBins2; i += kThreads) H2[i] = 0;
    if (tid < 2 * kC) bel[tid >> 1][tid & 1] = 0;
    if (tid < 2) below[tid] = cross[tid] = 0;
    // cache layout: key r of the range at r ^ ((r / kPer) & 31), so that both
    // the coalesced fill (consecutive r across a warp) and the per-thread runs
    // (lane t reads r = kPer t + u) touch 32 distinct banks.  16-byte loads,
    // eight in flight per thread, when the range starts 16-byte aligned.
    if (kCached) {
      const int n = hi - lo;
      auto put = [&](int r, float v) { cached_keys[r ^ ((r >> kSh) & 31)] = key_of(v); };
      int done = 0;
      if ((reinterpret_cast<uintptr_t>(s + lo) & 15u) == 0) {
        const int n4 = n >> 2;
        const float4* s4 = reinterpret_cast<const float4*>(s + lo);
        for (int q0 = tid; q0 < n4; q0 += 8 * kThreads) {
          float4 v[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const int q = q0 + u * kThreads;
            v[u] = q < n4 ? __ldg(s4 + q) : make_float4(0.f, 0.f, 0.f, 0.f);
          }
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const int q = q0 + u * kThreads;
            if (q < n4) {
              put(4 * q, v[u].x); put(4 * q + 1, v[u].y); put(4 * q + 2, v[u].z); put(4 * q + 3, v[u].w);
            }
          }
        }
        done = 4 * n4;
      }
      for (int r = done + tid; r < n; r += kThreads) put(r, __ldg(s + lo + r));
    }
    __syncthreads();
    // every CTA's barrier and cleared state are in place before any remote
    // access (the hardware cluster barrier; all threads of all CTAs reach it)
    if constexpr (kC > 1)
      asm volatile(
          "barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" :::
              "memory");
    auto key_at = [&](int j) {
      const int r = j - lo;
      if constexpr (kCached) return cached_keys[r ^ ((r >> kSh) & 31)];
      else return key_of(__ldg(s + j));
    };
    // this thread's kPer consecutive keys of the sub-range starting at sub0
    // (slots past hi read as the NaN key; every use masks them by position)
    auto load_run = [&](int sub0, uint32_t (&kk)[kPer]) {
      const int j0 = sub0 + tid * kPer;
#pragma unroll
      for (int u = 0; u < kPer; ++u) kk[u] = (j0 + u < hi) ? key_at(j0 + u) : 0xFFFFFFFFu;
    };
    // kCached: this thread's run of the range, held in registers for every round
    uint32_t kr[kPer];
    if constexpr (kCached) load_run(lo, kr);
    uint32_t prefix = 0, rem = (uint32_t)E;

    // ---- radix select: three digit rounds (E is uniform over the cluster) ----
    if (E > 0) {
      for (int round = 0; round < 3; ++round) {
        const int shift = (round == 0) ? 21 : (round == 1) ? 10 : 0;
        const int width = (round == 2) ? 10 : 11;
        const int nb = 1 << width;
        const uint32_t mask = (uint32_t)nb - 1u;
        if (ok) {
          // (the copies are zero: cleared at the start and by each round's owners)
          // scores concentrate in few bins: four copies (by warp), one bank
          // apart, spread the colliding atomics
          uint32_t* myloc = loc + (wid & (kCopies - 1)) * kCopyStride;
          auto hist_run = [&](const uint32_t(&kk)[kPer], int j0) {
#pragma unroll
            for (int u = 0; u < kPer; ++u)
              if (j0 + u < hi && (round == 0 || (kk[u] >> (shift + width)) == prefix))
                atomicAdd(&myloc[(kk[u] >> shift) & mask], 1u);
          };
          if constexpr (kCached) {
            hist_run(kr, lo + tid * kPer);
          } else {
            for (int sub0 = lo; sub0 < hi; sub0 += kSub) {
              uint32_t kk[kPer];
              load_run(sub0, kk);
              hist_run(kk, sub0 + tid * kPer);
            }
          }
          __syncthreads();
          // this CTA's totals (kept in copy 0) go into every CTA: added into the
          // round's cluster histogram, or (round 2) stored into this rank's slot
          uint32_t* dst = round < 2 ? &H[round][0] : H2 + rank * kBins2;
          for (int i = tid; i < nb; i += kThreads) {
            uint32_t v = loc[i];
#pragma unroll
            for (int c = 1; c < kCopies; ++c) {
              v += loc[c * kCopyStride + i];
              loc[c * kCopyStride + i] = 0;  // ready for the next round
            }
            loc[i] = v;
            if (v) {
              if constexpr (kC == 1) {
                dst[i] = v;
              } else {
                const uint32_t a0 = smem_addr(dst + i);
                for (uint32_t d = 0; d < (uint32_t)kC; ++d) {
                  const uint32_t ra = mapa(a0, d);
                  if (round < 2) dsm_add(ra, v);
                  else dsm_st(ra, v);
                }
              }
            }
          }
          if (round == 2 && tid < kC) {  // and the counts below the earlier digits
            if constexpr (kC == 1) {
              bel[0][0] = below[0];
              bel[0][1] = below[1];
            } else {
              const uint32_t ra = mapa(smem_addr(&bel[rank][0]), (uint32_t)tid);
              dsm_st(ra, below[0]);
              dsm_st(ra + 4u, below[1]);
            }
          }
        }
        if constexpr (kC == 1) {
          __syncthreads();
        } else if constexpr (kHw) {
          // every thread of every CTA takes every round's phase, so the
          // hardware cluster barrier needs no limit (release / acquire at
          // cluster scope orders the pushes before the reads)
          asm volatile(
              "barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" :::
                  "memory");
        } else {
          ok = cluster_phase<kC>(barA, phase, &fail, p.status, p.wait_ns,
                             round == 0 && (int)rank == p.stall_rank) && ok;
        }
        if (ok) {
          // the digit holding rank `rem` (1-based) of the keys with this
          // prefix, found by every CTA from the same histogram
          const int per = nb / kThreads;  // 4 or 2 bins per thread
          uint32_t v[kBins / kThreads], tot = 0;
#pragma unroll
          for (int i = 0; i < kBins / kThreads; ++i) {
            v[i] = 0;
            if (i < per) {
              const int bin = tid * per + i;
              if (round < 2) {
                v[i] = H[round][bin];
              } else {
#pragma unroll
                for (int r = 0; r < kC; ++r) v[i] += H2[r * kBins2 + bin];
              }
            }
            tot += v[i];
          }
          int total;
          uint32_t before = (uint32_t)block_excl_scan((int)tot, total, warp_tot);
          if (before < rem && rem <= before + tot) {
            for (int i = 0; i < per; ++i) {
              if (before + v[i] >= rem) {
                const uint32_t digit = (uint32_t)(tid * per + i);
                ctl[0] = (round == 0) ? digit : ((prefix << width) | digit);
                ctl[1] = rem - before;
                break;
              }
              before += v[i];
            }
          }
          __syncthreads();
          prefix = ctl[0];
          rem = ctl[1];
          const int digit = (int)(prefix & mask);
          if (round < 2) {
            // this CTA's keys below the digit (those with the prefix, for round
            // 1); each thread clears the totals it owns for the next round
            uint32_t part = 0;
            for (int i = tid; i < nb; i += kThreads) {
              if (i < digit) part += loc[i];
              loc[i] = 0;
            }
            if (part) atomicAdd(&below[round], part);
          } else {
            // keys below / at T held by the lower ranks; copy 0 cleared for the
            // next segment
            uint32_t lt = 0;
            for (int i = tid; i < nb; i += kThreads) {
              if (i < digit)
                for (int r = 0; r < (int)rank; ++r) lt += H2[r * kBins2 + i];
              loc[i] = 0;
            }
            if (tid == 0)
              for (int r = 0; r < (int)rank; ++r) {
                lt += bel[r][0] + bel[r][1];
                atomicAdd(&cross[1], H2[r * kBins2 + digit]);
              }
            if (lt) atomicAdd(&cross[0], lt);
          }
          __syncthreads();  // ctl and copy 0 are read before the next round rewrites them
        }
      }
    }
    const uint32_t T = prefix;
    const int quota = E > 0 ? (int)rem : 0;  // keys == T that are evicted

    // ---- counts below / at the threshold per warp ---------------------------
    // Each warp takes a contiguous, 32-aligned part of the CTA's range: with the
    // range cached, the 1024 keys its lanes hold in registers (counted there);
    // otherwise an equal share, walked 32 consecutive keys at a time (lane =
    // key) with ballots.  The compaction below walks the same parts.
    const int wlen = kCached ? kPer * 32 : ((hi - lo + kWarps * 32 - 1) / (kWarps * 32)) * 32;
    const int w_lo = min(hi, lo + wid * wlen), w_hi = min(hi, w_lo + wlen);
    const uint32_t lanelt = (1u << lane) - 1u;
    int nlt = 0, neq = 0;
    if (ok && E > 0) {
      if constexpr (kCached) {
        const int j0 = lo + tid * kPer;
        uint32_t a = 0, e = 0;
#pragma unroll
        for (int u = 0; u < kPer; ++u)
          if (j0 + u < hi) {
            a += kr[u] < T ? 1u : 0u;
            e += kr[u] == T ? 1u : 0u;
          }
        nlt = (int)__reduce_add_sync(0xffffffffu, a);
        neq = (int)__reduce_add_sync(0xffffffffu, e);
      } else {
        for (int c0 = w_lo; c0 < w_hi; c0 += 32) {
          const int j = c0 + lane;
          const bool in = j < w_hi;
          const uint32_t kk = in ? key_at(j) : 0xFFFFFFFFu;
          nlt += __popc(__ballot_sync(0xffffffffu, in && kk < T));
          neq += __popc(__ballot_sync(0xffffffffu, in && kk == T));
        }
      }
    }
    if (lane == 0) {
      wsum[0][wid] = nlt;
      wsum[1][wid] = neq;
    }
    __syncthreads();

    // ---- order-preserving compaction of this CTA's range --------------------
    // Per warp, in position order: the keys below / at T before its part (lower
    // ranks, from the round-2 phase, then lower warps of this CTA), then per 32
    // keys the ballots give every lane its evicted rank (those before it) and
    // an == T key's rank among the == T keys (evicted while below the quota); a
    // kept key's rank is its position minus the evicted keys before it.  Lanes
    // write their positions straight to the lists (consecutive lanes,
    // consecutive slots).
    if (ok) {
      int32_t* kout = keep_idx + (size_t)seg * p.max_keep;
      int32_t* eout = evict_idx + (size_t)seg * p.max_evict;
      int lt_run = (int)cross[0], eq_run = (int)cross[1];  // the lower ranks: lower positions
      for (int i = 0; i < wid; ++i) {
        lt_run += wsum[0][i];
        eq_run += wsum[1][i];
      }
      int ev_run = lt_run + min(eq_run, quota);  // evicted before this warp's part
      const bool any = E > 0;
      if constexpr (kCached) {
        // the warp's kPer groups, 32 at a time: every ballot first
        // (independent), then the running ranks group by group, one predicated
        // store per lane
#pragma unroll 1
        for (int g0 = 0; g0 < kPer; g0 += 32) {
          uint32_t ltm[32], eqm[32];
#pragma unroll
          for (int g = 0; g < 32; ++g) {
            const int j = w_lo + 32 * (g0 + g) + lane;
            const bool in = any && j < w_hi;
            const uint32_t kk = j < w_hi ? key_at(j) : 0xFFFFFFFFu;
            ltm[g] = __ballot_sync(0xffffffffu, in && kk < T);
            eqm[g] = __ballot_sync(0xffffffffu, in && kk == T);
          }
#pragma unroll
          for (int g = 0; g < 32; ++g) {
            const int j = w_lo + 32 * (g0 + g) + lane;
            uint32_t evm = ltm[g];
            if (eqm[g]) {  // keys == T: evicted while their rank among them is below the quota
              const bool e =
                  ((eqm[g] >> lane) & 1u) && eq_run + __popc(eqm[g] & lanelt) < quota;
              evm |= __ballot_sync(0xffffffffu, e);
            }
            const bool ev = (evm >> lane) & 1u;
            const int ev_before = ev_run + __popc(evm & lanelt);
            const int r = j - ev_before;
            int32_t* dst = ev ? eout + ev_before : kout + r;
            // the guards only matter after a wait gave up (inconsistent counts)
            const bool okw =
                ev ? (ev_before >= 0 && ev_before < p.max_evict) : (r >= 0 && r < p.max_keep);
            if (j < w_hi && okw) *dst = j;
            ev_run += __popc(evm);
            eq_run += __popc(eqm[g]);
          }
        }
      } else {
        // uncached ranges: four groups of 32 keys per step
        for (int c0 = w_lo; c0 < w_hi; c0 += 4 * 32) {
          uint32_t ltm[4], eqm[4];
#pragma unroll
          for (int g = 0; g < 4; ++g) {
            const int j = c0 + 32 * g + lane;
            const bool in = any && j < w_hi;
            const uint32_t kk = j < w_hi ? key_at(j) : 0xFFFFFFFFu;
            ltm[g] = __ballot_sync(0xffffffffu, in && kk < T);
            eqm[g] = __ballot_sync(0xffffffffu, in && kk == T);
          }
#pragma unroll
          for (int g = 0; g < 4; ++g) {
            const int j = c0 + 32 * g + lane;
            uint32_t evm = ltm[g];
            if (eqm[g]) {
              const bool e =
                  ((eqm[g] >> lane) & 1u) && eq_run + __popc(eqm[g] & lanelt) < quota;
              evm |= __ballot_sync(0xffffffffu, e);
            }
            const bool ev = (evm >> lane) & 1u;
            const int ev_before = ev_run + __popc(evm & lanelt);
            const int r = j - ev_before;
            int32_t* dst = ev ? eout + ev_before : kout + r;
            const bool okw =
                ev ? (ev_before >= 0 && ev_before < p.max_evict) : (r >= 0 && r < p.max_keep);
            if (j < w_hi && okw) *dst = j;
            ev_run += __popc(evm);
            eq_run += __popc(eqm[g]);
          }
        }
      }
      // slots past this row's own counts (rows shorter than the maxima): -1,
      // each CTA of the cluster taking an equal share
      {
        const int k_lo = L - E, e_lo = E;
        const int kn = max(0, p.max_keep - k_lo), en = max(0, p.max_evict - e_lo);
        const int ks = (kn + kC - 1) / kC, es = (en + kC - 1) / kC;
        const int k0 = k_lo + (int)rank * ks, k1 = min(p.max_keep, k0 + ks);
        const int e0 = e_lo + (int)rank * es, e1 = min(p.max_evict, e0 + es);
        for (int i = k0 + tid; i < k1; i += kThreads) kout[i] = -1;
        for (int i = e0 + tid; i < e1; i += kThreads) eout[i] = -1;
      }
    }
  }

  // every CTA learns whether any CTA of the cluster gave up a wait
  if constexpr (kC > 1) {
    if (tid < kC) dsm_st(mapa(smem_addr(&fails[rank]), (uint32_t)tid), fail != 0 ? 1u : 0u);
    // The hardware cluster barrier, not a bounded phase: no CTA may exit while
    // another can still address its shared memory, even after a wait gave up
    // (the waits' limits can expire at different times).  Every thread of
    // every CTA reaches it after finitely many bounded waits.
    asm volatile(
        "barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" :::
            "memory");
  }
  bool any = fail != 0;
  for (int r = 0; r < kC; ++r) any = any || fails[r] != 0;
  if (any) {
    // this CTA's share of the slots; the shares of the kC CTAs cover them all
    int32_t* kout = keep_idx + (size_t)seg * p.max_keep;
    int32_t* eout = evict_idx + (size_t)seg * p.max_evict;
    const int kc = (p.max_keep + kC - 1) / kC, ec = (p.max_evict + kC - 1) / kC;
    const int k0 = min(p.max_keep, (int)rank * kc), k1 = min(p.max_keep, k0 + kc);
    const int e0 = min(p.max_evict, (int)rank * ec), e1 = min(p.max_evict, e0 + ec);
    for (int i = k0 + tid; i < k1; i += kThreads) kout[i] = -1;
    for (int i = e0 + tid; i < e1; i += kThreads) eout[i] = -1;
  }
}

SelParams make_params(int B, int Hkv, int n_max, const int32_t* L, const int32_t* keep,
                      int max_keep, int max_evict, int32_t* status) {
  SelParams p;
  p.stall_rank = -1;
  p.wait_ns = kWaitNs;
  p.B = B;
  p.Hkv = Hkv;
  p.n_max = n_max;
  p.max_keep = max_keep;
  p.max_evict = max_evict;
  p.status = status;
  for (int b = 0; b < B; ++b) {
    p.L[b] = L[b];
    p.E[b] = L[b] - keep[b];
  }
  return p;
}

}  // namespace

// The select path keeps its state in shared memory; the workspace holds only
// the device status word.
size_t select_workspace_bytes(int, int, int) { return 256; }

int select_launch_count() { return 1; }

namespace {
// Clusters of kC CTAs of this kernel that fit on the device at once (queried
// once per kernel); 0 when the query fails.
template <int kC, int kPer, bool kCached>
int max_active_clusters(size_t smem) {
  static int cached = -1;
  if (cached < 0) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(kC * 256);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeClusterDimension;
    attr.val.clusterDim.x = (unsigned)kC;
    attr.val.clusterDim.y = 1;
    attr.val.clusterDim.z = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    int n = 0;
    cached = cudaOccupancyMaxActiveClusters(&n, k_select<kC, kPer, kCached>, &cfg) == cudaSuccess
                 ? n
                 : 0;
    (void)cudaGetLastError();
  }
  return cached;
}

template <int kC, int kPer, bool kCached>
size_t select_smem() {
  // [key cache][histogram copies][round-2 slots]; the copies start at kSub words
  return ((size_t)kThreads * kPer + kCopies * (size_t)kCopyStride + (size_t)kC * kBins2) *
         sizeof(uint32_t);
}

template <int kC, int kPer, bool kCached>
cudaError_t prepare(int* waves, int nseg) {
  const size_t smem = select_smem<kC, kPer, kCached>();
  cudaError_t e = cudaFuncSetAttribute(k_select<kC, kPer, kCached>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int cap = max_active_clusters<kC, kPer, kCached>(smem);
  *waves = cap > 0 ? (nseg + cap - 1) / cap : 1;
  return cudaSuccess;
}

template <int kC, int kPer, bool kCached>
cudaError_t launch_kc(const SelParams& p, const float* scores, int32_t* keep_idx,
                      int32_t* evict_idx, cudaStream_t st) {
  const size_t smem = select_smem<kC, kPer, kCached>();
  // the self-test (a rank that withholds its arrivals) needs the bounded phases
  auto* kern = p.stall_rank >= 0 ? k_select<kC, kPer, kCached, false>
                                 : k_select<kC, kPer, kCached, true>;
  cudaError_t e =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  return launch_ex(kern, dim3(p.B * p.Hkv * kC), dim3(kThreads), smem, st, true, kC, p, scores,
                   keep_idx, evict_idx);
}

cudaError_t launch_impl(int B, int Hkv, int n_max, const float* scores, const int32_t* L,
                        const int32_t* keep, int32_t* keep_idx, int32_t max_keep,
                        int32_t* evict_idx, int32_t max_evict, int32_t* status, int stall_rank,
                        uint64_t wait_ns, cudaStream_t st) {
  SelParams p = make_params(B, Hkv, n_max, L, keep, max_keep, max_evict, status);
  p.wait_ns = wait_ns;
  int max_L = 0;
  for (int b = 0; b < B; ++b) max_L = L[b] > max_L ? L[b] : max_L;
  // rows by decreasing length (stable)
  for (int b = 0; b < B; ++b) p.row_order[b] = (uint8_t)b;
  for (int i = 1; i < B; ++i)
    for (int j = i; j > 0 && L[p.row_order[j - 1]] < L[p.row_order[j]]; --j) {
      const uint8_t t = p.row_order[j];
      p.row_order[j] = p.row_order[j - 1];
      p.row_order[j - 1] = t;
    }
  auto span = [&](int kc) { return ((long long)max_L + kc - 1) / kc; };
  // the smallest cluster whose CTAs' ranges fit one cached 16384-key sub-range
  // (the self-test needs cross-CTA waits: at least two CTAs)
  int kc = stall_rank >= 0 ? 2 : 1;
  while (kc < kMaxC && span(kc) > kThreads * 32) kc *= 2;
  bool cached = span(kc) <= kThreads * 32;
  p.stall_rank = stall_rank < kc ? stall_rank : kc - 1;
  const int nseg = B * Hkv;
  // 32768-key sub-ranges on 4- or 8-CTA clusters, where they save a wave of
  // clusters or keep a longer range cached
  int kc64 = 4;
  while (kc64 < kMaxC && span(kc64) > kThreads * 64) kc64 *= 2;
  if (stall_rank < 0 && span(kc64) <= kThreads * 64 && kc >= 4) {
    int w32 = 2, w64 = 1;
    cudaError_t e = cudaSuccess;
    if (cached) {
      e = kc == 4 ? prepare<4, 32, true>(&w32, nseg) : prepare<8, 32, true>(&w32, nseg);
      if (e != cudaSuccess) return e;
    }
    e = kc64 == 4 ? prepare<4, 64, true>(&w64, nseg) : prepare<8, 64, true>(&w64, nseg);
    if (e != cudaSuccess) return e;
    if (!cached || w64 < w32)
      return kc64 == 4 ? launch_kc<4, 64, true>(p, scores, keep_idx, evict_idx, st)
                       : launch_kc<8, 64, true>(p, scores, keep_idx, evict_idx, st);
  }
  switch (kc) {
    case 1: return cached ? launch_kc<1, 32, true>(p, scores, keep_idx, evict_idx, st)
                          : launch_kc<1, 32, false>(p, scores, keep_idx, evict_idx, st);
    case 2: return cached ? launch_kc<2, 32, true>(p, scores, keep_idx, evict_idx, st)
                          : launch_kc<2, 32, false>(p, scores, keep_idx, evict_idx, st);
    case 4: return cached ? launch_kc<4, 32, true>(p, scores, keep_idx, evict_idx, st)
                          : launch_kc<4, 32, false>(p, scores, keep_idx, evict_idx, st);
    default: return cached ? launch_kc<8, 32, true>(p, scores, keep_idx, evict_idx, st)
                           : launch_kc<8, 32, false>(p, scores, keep_idx, evict_idx, st);
  }
}
}  // namespace

// L, keep: host arrays of B <= kMaxB rows.
cudaError_t launch_select(int B, int Hkv, int n_max, const float* scores, const int32_t* L,
                          const int32_t* keep, int32_t* keep_idx, int32_t max_keep,
                          int32_t* evict_idx, int32_t max_evict, int32_t* status,
                          cudaStream_t st) {
  return launch_impl(B, Hkv, n_max, scores, L, keep, keep_idx, max_keep, evict_idx, max_evict,
                     status, -1, kWaitNs, st);
}

// Self-test: CTA rank 1 of every cluster withholds its arrivals of round 0, so
// every CTA's wait for them runs out after wait_ns (and later waits of the
// segment may too); the kernel then reports the timeout and fills -1.
cudaError_t launch_select_stalled(int B, int Hkv, int n_max, const float* scores,
                                  const int32_t* L, const int32_t* keep, int32_t* keep_idx,
                                  int32_t max_keep, int32_t* evict_idx, int32_t max_evict,
                                  int32_t* status, uint64_t wait_ns, cudaStream_t st) {
  return launch_impl(B, Hkv, n_max, scores, L, keep, keep_idx, max_keep, evict_idx, max_evict,
                     status, 1, wait_ns, st);
}

}  // namespace dropkv
