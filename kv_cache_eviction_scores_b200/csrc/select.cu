// select.cu -- exact lowest-score eviction per (b, KV head): multi-CTA radix
// select plus an order-preserving compaction.
//
// Write-up "DropKV：精确单项输出扰动评分组件", Algorithm 1 paragraph: after
// pooling and window protection, the lowest-scoring tokens are evicted.  The
// order used is (score ascending, position ascending); NaN sorts above +inf.
//
// Scores map to 32-bit keys whose unsigned order is the float order.  Every
// segment (b, h) is cut into 4096-key chunks, one CTA each, so the work spreads
// over the whole GPU even when B * Hkv is small.
//   round 0..2: histogram of an 11/11/10-bit digit of the keys that match the
//       prefix found so far; the last CTA of a segment to finish (an atomic
//       arrival counter, no waiting) picks the digit holding the E-th smallest
//       key.  After round 2 the prefix is the threshold key T and `rem` is how
//       many keys equal to T are evicted (the lowest positions among them).
//   count: per chunk, #keys < T and #keys == T; the last CTA of the segment
//       turns them into exclusive prefixes.
//   write: each chunk walks its keys in position order with block scans and
//       writes kept / evicted positions to their final slots.
// Outputs are pre-filled with -1 by the init kernel.
#include "common.cuh"
#include "internal.h"

namespace dropkv {
namespace {

constexpr int kChunk = 4096;
constexpr int kThreads = 256;
constexpr int kBins = 2048;

struct SegState {
  uint32_t prefix;  // digits found so far; after round 2 the threshold key T
  int32_t rem;      // rank still to place; after round 2 the quota among keys == T
  uint32_t arrive;  // arrival counter for the last-CTA step
  int32_t done;     // 1: nothing to select (no eviction)
};

struct SelParams {
  int32_t B, Hkv, n_max;
  int32_t max_keep, max_evict;
  int32_t L[kMaxB];
  int32_t E[kMaxB];            // evictions per row
  int32_t nchunk[kMaxB];       // chunks per segment of row b
  int32_t chunk_base[kMaxB + 1];  // first CTA of row b (Hkv segments each)
};

__device__ __forceinline__ uint32_t key_of(float s) {
  const uint32_t u = __float_as_uint(s);
  if (s != s) return 0xFFFFFFFFu;  // NaN above everything
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// CTA -> (b, h, chunk)
__device__ __forceinline__ void locate(const SelParams& p, int blk, int& b, int& h, int& c) {
  b = 0;
  while (b + 1 < p.B && blk >= p.chunk_base[b + 1]) ++b;
  const int local = blk - p.chunk_base[b];
  h = local / p.nchunk[b];
  c = local % p.nchunk[b];
}

struct Workspace {
  SegState* seg;
  uint32_t* hist;   // [segments][kBins]
  int32_t* cnt;     // [chunks][2]: #< T, #== T
  int32_t* off;     // [chunks][2]: exclusive prefixes within the segment
};

__device__ __forceinline__ Workspace carve(void* ws, const SelParams& p) {
  const int segs = p.B * p.Hkv;
  const int chunks = p.chunk_base[p.B];
  char* base = reinterpret_cast<char*>(ws);
  Workspace w;
  w.seg = reinterpret_cast<SegState*>(base);
  size_t o = align_up(sizeof(SegState) * segs, 256);
  w.hist = reinterpret_cast<uint32_t*>(base + o);
  o += align_up(sizeof(uint32_t) * kBins * (size_t)segs, 256);
  w.cnt = reinterpret_cast<int32_t*>(base + o);
  o += align_up(sizeof(int32_t) * 2 * (size_t)chunks, 256);
  w.off = reinterpret_cast<int32_t*>(base + o);
  return w;
}

__global__ void k_sel_init(SelParams p, void* ws, int32_t* keep_idx, int32_t* evict_idx) {
  Workspace w = carve(ws, p);
  const int segs = p.B * p.Hkv;
  const size_t tid = blockIdx.x * (size_t)blockDim.x + threadIdx.x;
  const size_t nthr = (size_t)gridDim.x * blockDim.x;
  for (size_t i = tid; i < (size_t)segs; i += nthr) {
    const int b = (int)(i / p.Hkv);
    SegState s;
    s.prefix = 0;
    s.rem = p.E[b];
    s.arrive = 0;
    s.done = (p.E[b] == 0) ? 1 : 0;
    w.seg[i] = s;
  }
  for (size_t i = tid; i < (size_t)segs * kBins; i += nthr) w.hist[i] = 0;
  for (size_t i = tid; i < (size_t)segs * p.max_keep; i += nthr) keep_idx[i] = -1;
  for (size_t i = tid; i < (size_t)segs * p.max_evict; i += nthr) evict_idx[i] = -1;
}

__global__ void __launch_bounds__(kThreads)
k_sel_hist(SelParams p, const float* __restrict__ scores, void* ws, int round) {
  __shared__ uint32_t sh[kBins];
  __shared__ int last;
  __shared__ uint32_t part[kThreads];
  Workspace w = carve(ws, p);
  int b, h, c;
  locate(p, blockIdx.x, b, h, c);
  const int seg = b * p.Hkv + h;
  if (w.seg[seg].done) return;  // uniform for the whole segment
  const int shift = (round == 0) ? 21 : (round == 1) ? 10 : 0;
  const int width = (round == 2) ? 10 : 11;
  const uint32_t mask = (1u << width) - 1u;
  const uint32_t prefix = w.seg[seg].prefix;
  for (int i = threadIdx.x; i < kBins; i += kThreads) sh[i] = 0;
  __syncthreads();
  const int L = p.L[b];
  const float* s = scores + (size_t)seg * p.n_max;
  const int beg = c * kChunk, end = min(L, beg + kChunk);
  for (int j = beg + threadIdx.x; j < end; j += kThreads) {
    const uint32_t key = key_of(s[j]);
    if (round == 0 || (key >> (shift + width)) == prefix) atomicAdd(&sh[(key >> shift) & mask], 1u);
  }
  __syncthreads();
  uint32_t* gh = w.hist + (size_t)seg * kBins;
  for (int i = threadIdx.x; i < kBins; i += kThreads)
    if (sh[i]) atomicAdd(&gh[i], sh[i]);
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) last = (atomicAdd(&w.seg[seg].arrive, 1u) == (uint32_t)p.nchunk[b] - 1);
  __syncthreads();
  if (!last) return;
  __threadfence();
  // Last CTA of the segment: find the digit that holds rank `rem` (1-based).
  const int per = kBins / kThreads;  // 8 bins per thread
  uint32_t local[kBins / kThreads];
  uint32_t tot = 0;
  for (int i = 0; i < per; ++i) {
    local[i] = __ldcg(&gh[threadIdx.x * per + i]);
    tot += local[i];
  }
  part[threadIdx.x] = tot;
  __syncthreads();
  // inclusive scan of the per-thread totals (Hillis-Steele in shared memory)
  for (int o = 1; o < kThreads; o <<= 1) {
    const uint32_t add = (threadIdx.x >= o) ? part[threadIdx.x - o] : 0u;
    __syncthreads();
    part[threadIdx.x] += add;
    __syncthreads();
  }
  const uint32_t rem = (uint32_t)w.seg[seg].rem;
  uint32_t before = part[threadIdx.x] - tot;  // exclusive prefix
  if (before < rem && rem <= part[threadIdx.x]) {
    for (int i = 0; i < per; ++i) {
      if (before + local[i] >= rem) {
        SegState st = w.seg[seg];
        st.prefix = (round == 0) ? (uint32_t)(threadIdx.x * per + i)
                                 : ((prefix << width) | (uint32_t)(threadIdx.x * per + i));
        st.rem = (int32_t)(rem - before);
        st.arrive = 0;
        w.seg[seg] = st;
        break;
      }
      before += local[i];
    }
  }
  for (int i = threadIdx.x; i < kBins; i += kThreads) gh[i] = 0;
}

__global__ void __launch_bounds__(kThreads)
k_sel_count(SelParams p, const float* __restrict__ scores, void* ws) {
  __shared__ int32_t red[2][kThreads / 32];
  __shared__ int last;
  Workspace w = carve(ws, p);
  int b, h, c;
  locate(p, blockIdx.x, b, h, c);
  const int seg = b * p.Hkv + h;
  const SegState st = w.seg[seg];
  const uint32_t T = st.done ? 0u : st.prefix;
  const int L = p.L[b];
  const float* s = scores + (size_t)seg * p.n_max;
  const int beg = c * kChunk, end = min(L, beg + kChunk);
  int nlt = 0, neq = 0;
  if (!st.done)
    for (int j = beg + threadIdx.x; j < end; j += kThreads) {
      const uint32_t key = key_of(s[j]);
      nlt += key < T;
      neq += key == T;
    }
  for (int o = 16; o > 0; o >>= 1) {
    nlt += __shfl_xor_sync(0xffffffffu, nlt, o);
    neq += __shfl_xor_sync(0xffffffffu, neq, o);
  }
  if ((threadIdx.x & 31) == 0) {
    red[0][threadIdx.x >> 5] = nlt;
    red[1][threadIdx.x >> 5] = neq;
  }
  __syncthreads();
  const int blk = blockIdx.x;
  if (threadIdx.x == 0) {
    int a = 0, e = 0;
    for (int i = 0; i < kThreads / 32; ++i) { a += red[0][i]; e += red[1][i]; }
    w.cnt[2 * blk] = a;
    w.cnt[2 * blk + 1] = e;
    __threadfence();
    last = (atomicAdd(&w.seg[seg].arrive, 1u) == (uint32_t)p.nchunk[b] - 1);
  }
  __syncthreads();
  if (!last || threadIdx.x != 0) return;
  __threadfence();
  // exclusive prefixes over the segment's chunks, in position order
  const int first = blk - c;
  int a = 0, e = 0;
  for (int i = 0; i < p.nchunk[b]; ++i) {
    w.off[2 * (first + i)] = a;
    w.off[2 * (first + i) + 1] = e;
    a += __ldcg(&w.cnt[2 * (first + i)]);
    e += __ldcg(&w.cnt[2 * (first + i) + 1]);
  }
}

__global__ void __launch_bounds__(kThreads)
k_sel_write(SelParams p, const float* __restrict__ scores, const void* ws,
            int32_t* __restrict__ keep_idx, int32_t* __restrict__ evict_idx) {
  __shared__ int32_t wsum[2][kThreads / 32];
  Workspace w = carve(const_cast<void*>(ws), p);
  int b, h, c;
  locate(p, blockIdx.x, b, h, c);
  const int seg = b * p.Hkv + h;
  const SegState st = w.seg[seg];
  const uint32_t T = st.prefix;
  const int quota = st.done ? 0 : st.rem;  // keys == T that are evicted
  const bool any = !st.done;
  const int L = p.L[b];
  const float* s = scores + (size_t)seg * p.n_max;
  int32_t* kout = keep_idx + (size_t)seg * p.max_keep;
  int32_t* eout = evict_idx + (size_t)seg * p.max_evict;
  const int blk = blockIdx.x;
  const int lt_before = w.off[2 * blk];
  int eq_seen = w.off[2 * blk + 1];                      // keys == T before this point
  int ev_seen = lt_before + min(eq_seen, quota);         // evicted before this point
  const int beg = c * kChunk, end = min(L, beg + kChunk);
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  for (int t0 = beg; t0 < end; t0 += kThreads) {
    const int j = t0 + threadIdx.x;
    const bool in = j < end;
    uint32_t key = in ? key_of(s[j]) : 0xFFFFFFFFu;
    const bool lt = in && any && key < T;
    const bool eq = in && any && key == T;
    // exclusive rank of eq among this tile's eq, in position order
    const unsigned beq = __ballot_sync(0xffffffffu, eq);
    if (lane == 0) wsum[1][wid] = __popc(beq);
    __syncthreads();
    int eq_rank = eq_seen + __popc(beq & ((1u << lane) - 1u));
    int eq_tile = 0;
    for (int i = 0; i < kThreads / 32; ++i) {
      if (i < wid) eq_rank += wsum[1][i];
      eq_tile += wsum[1][i];
    }
    const bool ev = in && (lt || (eq && eq_rank < quota));
    const unsigned bev = __ballot_sync(0xffffffffu, ev);
    if (lane == 0) wsum[0][wid] = __popc(bev);
    __syncthreads();
    int ev_rank = ev_seen + __popc(bev & ((1u << lane) - 1u));
    int ev_tile = 0;
    for (int i = 0; i < kThreads / 32; ++i) {
      if (i < wid) ev_rank += wsum[0][i];
      ev_tile += wsum[0][i];
    }
    if (in) {  // the guards only matter if the ranks were inconsistent
      if (ev) {
        if (ev_rank < p.max_evict) eout[ev_rank] = j;
      } else if (j - ev_rank < p.max_keep) {
        kout[j - ev_rank] = j;
      }
    }
    eq_seen += eq_tile;
    ev_seen += ev_tile;
    __syncthreads();
  }
}

SelParams make_params(int B, int Hkv, int n_max, const int32_t* L, const int32_t* keep,
                      int max_keep, int max_evict) {
  SelParams p;
  p.B = B;
  p.Hkv = Hkv;
  p.n_max = n_max;
  p.max_keep = max_keep;
  p.max_evict = max_evict;
  p.chunk_base[0] = 0;
  for (int b = 0; b < B; ++b) {
    p.L[b] = L[b];
    p.E[b] = L[b] - keep[b];
    p.nchunk[b] = (L[b] + kChunk - 1) / kChunk;
    if (p.nchunk[b] == 0) p.nchunk[b] = 1;  // an empty row still gets one (idle) CTA
    p.chunk_base[b + 1] = p.chunk_base[b] + Hkv * p.nchunk[b];
  }
  return p;
}

}  // namespace

size_t select_workspace_bytes(int B, int Hkv, int n_max) {
  const size_t segs = (size_t)B * Hkv;
  const size_t nchunk = (size_t)(n_max + kChunk - 1) / kChunk + 1;
  return align_up(sizeof(SegState) * segs, 256) + align_up(sizeof(uint32_t) * kBins * segs, 256) +
         2 * align_up(sizeof(int32_t) * 2 * segs * nchunk, 256);
}

int select_launch_count() { return 6; }

// L, keep: host arrays of B <= kMaxB rows.  Workspace carve-up depends only on
// (B, Hkv, chunk counts), all of which are bounded by select_workspace_bytes.
cudaError_t launch_select(int B, int Hkv, int n_max, const float* scores, const int32_t* L,
                          const int32_t* keep, int32_t* keep_idx, int32_t max_keep,
                          int32_t* evict_idx, int32_t max_evict, void* ws, cudaStream_t st) {
  const SelParams p = make_params(B, Hkv, n_max, L, keep, max_keep, max_evict);
  const int chunks = p.chunk_base[B];
  k_sel_init<<<148, 256, 0, st>>>(p, ws, keep_idx, evict_idx);
  for (int r = 0; r < 3; ++r) k_sel_hist<<<chunks, kThreads, 0, st>>>(p, scores, ws, r);
  k_sel_count<<<chunks, kThreads, 0, st>>>(p, scores, ws);
  k_sel_write<<<chunks, kThreads, 0, st>>>(p, scores, ws, keep_idx, evict_idx);
  return cudaGetLastError();
}

}  // namespace dropkv
