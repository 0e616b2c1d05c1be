// simt.cu -- CUDA-core scoring path: any head dim up to 256, bf16 or fp32
// inputs.  It is the path for fp32 inputs and for shapes the tensor-core path
// does not cover.
//
// Pass 1 (one CTA per window query): streams the visible keys 0..P_t in
// 128-token chunks staged through shared memory, keeping the running max, the
// softmax normaliser and the unnormalised output a (write-up
// "DropKV：精确单项输出扰动评分组件", section 核心公式: p = softmax(K q /
// sqrt d), a = sum_j p_j v_j).
// Pass 2 (one thread per cached token): recomputes each logit with the same
// evaluation order as pass 1, forms p_j / (1 - p_j) as e_j / (l - e_j), and
// accumulates ratio^2 * ||a - v_j||^2 over the G*w window queries of the KV
// head (the s_j sum and the GQA sum in one register).  The squared distance is
// taken directly, not expanded.
//
// Arithmetic type: fp32 for bf16 inputs; fp64 for fp32 inputs.  With fp32
// inputs the scores are held to 1e-6 relative, which fp32 arithmetic cannot
// guarantee: the complement l - e_j cancels when p_j is large and the sums over
// the window and the group add O(log n) roundings.
#include <type_traits>

#include "common.cuh"
#include "internal.h"

namespace dropkv {
namespace {

template <typename T>
using acc_t = typename std::conditional<std::is_same<T, float>::value, double, float>::type;

__device__ __forceinline__ float exp_acc(float x) { return expf(x); }
__device__ __forceinline__ double exp_acc(double x) { return exp(x); }
__device__ __forceinline__ float fma_acc(float a, float b, float c) { return __fmaf_rn(a, b, c); }
__device__ __forceinline__ double fma_acc(double a, double b, double c) { return __fma_rn(a, b, c); }
__device__ __forceinline__ float mul_acc(float a, float b) { return __fmul_rn(a, b); }
__device__ __forceinline__ double mul_acc(double a, double b) { return __dmul_rn(a, b); }
__device__ __forceinline__ double to_acc(double, float x) { return (double)x; }
__device__ __forceinline__ float to_acc(float, __nv_bfloat16 x) { return __bfloat162float(x); }

// Logit q . k / sqrt(d) in one fixed order; both passes call it with keys held
// transposed in shared memory ([d][stride]), so pass 2's recomputed logit is
// bit-identical to pass 1's.
template <typename T, typename A>
__device__ __forceinline__ A logit(const A* qs, const T* kp, int stride, int d, A inv_sqrt_d) {
  A acc = A(0);
  for (int c = 0; c < d; ++c) acc = fma_acc(qs[c], to_acc(A(0), kp[(size_t)c * stride]), acc);
  return mul_acc(acc, inv_sqrt_d);  // not contracted into a later add
}

template <typename A>
__device__ __forceinline__ A block_max_acc(A x, A* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x = fmax(x, __shfl_xor_sync(0xffffffffu, x, o));
  __syncthreads();
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = x;
  __syncthreads();
  return fmax(fmax(red[0], red[1]), fmax(red[2], red[3]));
}
template <typename A>
__device__ __forceinline__ A block_sum_acc(A x, A* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  __syncthreads();
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = x;
  __syncthreads();
  return (red[0] + red[1]) + (red[2] + red[3]);
}

constexpr int kP1 = 128;  // pass-1 threads = keys per chunk

// Pass 1.  Internal outputs (read by pass 2): stats_ws [rows][2] fp64 (max,
// normaliser), attn_ws [rows][d] in the arithmetic type.  Optional fp32 copies
// for the caller: stats_user [rows][2], attn_user [rows][d].
template <typename T>
__global__ void __launch_bounds__(kP1)
k_simt_pass1(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v, Lens lens,
             int Hq, int Hkv, int n_max, int d, int w, double* __restrict__ stats_ws,
             acc_t<T>* __restrict__ attn_ws, float* __restrict__ stats_user,
             float* __restrict__ attn_user) {
  using A = acc_t<T>;
  extern __shared__ __align__(16) unsigned char smem_raw[];
  T* ks = reinterpret_cast<T*>(smem_raw);  // [d][kP1] keys of the chunk, transposed
  __shared__ A qs[256];
  __shared__ A es[kP1];
  __shared__ A red[4];
  const int row = blockIdx.x;  // (b, hq, t) flattened like q
  const int t = row % w;
  const int hq = (row / w) % Hq;
  const int b = row / (w * Hq);
  const int h = hq / (Hq / Hkv);
  const int L = lens.L[b];
  const int P = L - w + t;  // causal tail alignment: query t sees keys 0..P
  const int tid = threadIdx.x;
  const A isd = A(1) / sqrt(A(d));
  for (int c = tid; c < d; c += kP1) qs[c] = to_acc(A(0), q[(size_t)row * d + c]);
  const T* K = k + ((size_t)b * Hkv + h) * (size_t)n_max * d;
  const T* V = v + ((size_t)b * Hkv + h) * (size_t)n_max * d;
  A m = -CUDART_INF, l = A(0), a0 = A(0), a1 = A(0);
  for (int j0 = 0; j0 <= P; j0 += kP1) {
    const int cnt = min(kP1, P + 1 - j0);
    __syncthreads();  // previous chunk's ks / es fully consumed
    for (int idx = tid; idx < cnt * d; idx += kP1) {  // coalesced rows -> transposed tile
      const int r = idx / d, c = idx % d;
      ks[c * kP1 + r] = K[(size_t)(j0 + r) * d + c];
    }
    __syncthreads();
    A x = -CUDART_INF;
    if (tid < cnt) x = logit(qs, ks + tid, kP1, d, isd);
    const A mt = block_max_acc(x, red);
    const A m_new = fmax(m, mt);
    const A scale = (m == -CUDART_INF) ? A(0) : exp_acc(m - m_new);
    const A e = (tid < cnt) ? exp_acc(x - m_new) : A(0);
    es[tid] = e;
    const A lt = block_sum_acc(e, red);  // its barriers also publish es[]
    l = l * scale + lt;
    a0 *= scale;
    a1 *= scale;
    for (int jj = 0; jj < cnt; ++jj) {
      const A ej = es[jj];
      const T* vr = V + (size_t)(j0 + jj) * d;
      if (tid < d) a0 = fma_acc(ej, to_acc(A(0), vr[tid]), a0);
      if (tid + kP1 < d) a1 = fma_acc(ej, to_acc(A(0), vr[tid + kP1]), a1);
    }
    m = m_new;
  }
  if (tid == 0) {
    stats_ws[2 * (size_t)row] = (double)m;
    stats_ws[2 * (size_t)row + 1] = (double)l;
    if (stats_user) {
      stats_user[2 * (size_t)row] = (float)m;
      stats_user[2 * (size_t)row + 1] = (float)l;
    }
  }
  if (tid < d) {
    const A o = a0 / l;
    attn_ws[(size_t)row * d + tid] = o;
    if (attn_user) attn_user[(size_t)row * d + tid] = (float)o;
  }
  if (tid + kP1 < d) {
    const A o = a1 / l;
    attn_ws[(size_t)row * d + tid + kP1] = o;
    if (attn_user) attn_user[(size_t)row * d + tid + kP1] = (float)o;
  }
}

constexpr int kQB = 8;  // window queries staged in shared memory at a time

template <typename T, int TPB>
__global__ void __launch_bounds__(TPB)
k_simt_pass2(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v, Lens lens,
             int Hq, int Hkv, int n_max, int d, int w, const double* __restrict__ stats,
             const acc_t<T>* __restrict__ attn, float* __restrict__ part,
             int32_t* __restrict__ status, int attn_only) {
  using A = acc_t<T>;
  extern __shared__ __align__(16) unsigned char smem_raw[];
  A* qa = reinterpret_cast<A*>(smem_raw);                    // [kQB][2][d]
  T* ks = reinterpret_cast<T*>(qa + (size_t)kQB * 2 * d);    // [d][TPB] keys, transposed
  T* vs = ks + (size_t)d * TPB;                               // [d][TPB] values, transposed
  const int bh = blockIdx.y, b = bh / Hkv, h = bh % Hkv;
  const int L = lens.L[b];
  const int j0 = blockIdx.x * TPB;
  if (j0 >= L) return;
  const int tid = threadIdx.x, j = j0 + tid;
  const bool valid = j < L;
  const A isd = A(1) / sqrt(A(d));
  const T* K = k + ((size_t)b * Hkv + h) * (size_t)n_max * d;
  const T* V = v + ((size_t)b * Hkv + h) * (size_t)n_max * d;
  for (int idx = tid; idx < TPB * d; idx += TPB) {
    const int r = idx / d, c = idx % d;
    T kv = T(0.f), vv = T(0.f);  // rows >= L are never read as data
    if (j0 + r < L) {
      kv = K[(size_t)(j0 + r) * d + c];
      vv = V[(size_t)(j0 + r) * d + c];
    }
    ks[c * TPB + r] = kv;
    vs[c * TPB + r] = vv;
  }
  __syncthreads();
  const int G = Hq / Hkv, NQ = G * w;
  const size_t qrow0 = ((size_t)b * Hq + (size_t)h * G) * w;  // the group's first query row
  A s = A(0);
  for (int i0 = 0; i0 < NQ; i0 += kQB) {
    const int nb = min(kQB, NQ - i0);
    for (int idx = tid; idx < nb * d; idx += TPB) {
      const int i = idx / d, c = idx % d;
      qa[(2 * i) * d + c] = to_acc(A(0), q[(qrow0 + i0 + i) * d + c]);
      qa[(2 * i + 1) * d + c] = attn[(qrow0 + i0 + i) * d + c];
    }
    __syncthreads();
    for (int i = 0; i < nb; ++i) {
      const int r = i0 + i;
      const int P = L - w + r % w;
      if (valid && j <= P) {
        const A m = (A)stats[2 * (qrow0 + r)], l = (A)stats[2 * (qrow0 + r) + 1];
        const A x = logit(qa + 2 * i * d, ks + tid, TPB, d, isd);
        const A e = exp_acc(x - m);
        if (attn_only) {  // attention-only score: the probability itself
          s += e / l;
          continue;
        }
        const A den = l - e;  // (1 - p_j) * l
        // p_j rounds to 1 (in fp32, the precision of the stored inputs, also
        // when the arithmetic is fp64) or its complement is not positive:
        // removal is singular
        if (!(den > A(0)) || (float)(e / l) == 1.0f) {
          atomicMax(status, kStatusSingular);
          continue;
        }
        const A ratio = e / den;  // p_j / (1 - p_j)
        const A* a = qa + (2 * i + 1) * d;
        A sq = A(0);
        for (int c = 0; c < d; ++c) {
          const A df = a[c] - to_acc(A(0), vs[c * TPB + tid]);
          sq = fma_acc(df, df, sq);
        }
        s = fma_acc(ratio * ratio, sq, s);
      }
    }
    __syncthreads();
  }
  if (valid) part[((size_t)b * Hkv + h) * n_max + j] = (float)s;
}

template <typename T>
cudaError_t pass1_launch(const dropkv_shape& s, const void* q, const void* k, const void* v,
                         const Lens& lens, double* stats_ws, void* attn_ws, float* stats_user,
                         float* attn_user, cudaStream_t st) {
  const size_t smem = (size_t)s.d * kP1 * sizeof(T);
  auto fn = k_simt_pass1<T>;
  cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int rows = lens.B * s.Hq * s.window;
  fn<<<rows, kP1, smem, st>>>((const T*)q, (const T*)k, (const T*)v, lens, s.Hq, s.Hkv, s.n_max,
                              s.d, s.window, stats_ws, (acc_t<T>*)attn_ws, stats_user, attn_user);
  return cudaGetLastError();
}

template <typename T, int TPB>
cudaError_t pass2_launch(const dropkv_shape& s, const void* q, const void* k, const void* v,
                         const Lens& lens, const double* stats, const void* attn, float* part,
                         int32_t* status, int attn_only, cudaStream_t st) {
  const size_t smem = 2 * (size_t)s.d * TPB * sizeof(T) + (size_t)kQB * 2 * s.d * sizeof(acc_t<T>);
  auto fn = k_simt_pass2<T, TPB>;
  cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((s.n_max + TPB - 1) / TPB, lens.B * s.Hkv);
  fn<<<grid, TPB, smem, st>>>((const T*)q, (const T*)k, (const T*)v, lens, s.Hq, s.Hkv, s.n_max,
                              s.d, s.window, stats, (const acc_t<T>*)attn, part, status,
                              attn_only);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_simt_pass1(const dropkv_shape& s, const void* q, const void* k,
                              const void* v, const Lens& lens, double* stats_ws, void* attn_ws,
                              float* stats_user, float* attn_user, cudaStream_t st) {
  if (s.dtype == DROPKV_BF16)
    return pass1_launch<__nv_bfloat16>(s, q, k, v, lens, stats_ws, attn_ws, stats_user,
                                       attn_user, st);
  return pass1_launch<float>(s, q, k, v, lens, stats_ws, attn_ws, stats_user, attn_user, st);
}

cudaError_t launch_simt_pass2(const dropkv_shape& s, const void* q, const void* k,
                              const void* v, const Lens& lens, const double* stats_ws,
                              const void* attn_ws, float* part, int32_t* status, int score,
                              cudaStream_t st) {
  const int ao = score == DROPKV_SCORE_ATTENTION ? 1 : 0;
  if (s.dtype == DROPKV_BF16)
    return pass2_launch<__nv_bfloat16, 128>(s, q, k, v, lens, stats_ws, attn_ws, part, status,
                                            ao, st);
  if (s.d <= 128)
    return pass2_launch<float, 128>(s, q, k, v, lens, stats_ws, attn_ws, part, status, ao, st);
  return pass2_launch<float, 64>(s, q, k, v, lens, stats_ws, attn_ws, part, status, ao, st);
}

}  // namespace dropkv
