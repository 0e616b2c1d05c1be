// simt.cu -- fp32 CUDA-core scoring path: any head dim up to 256, bf16 or fp32
// inputs.  It is the path for fp32 inputs (tight 1e-6 tolerance) and for
// shapes the tensor-core path does not cover.
//
// Pass 1 (one CTA per window query): streams the visible keys 0..P_t in
// 128-token chunks, keeping the running max, the softmax normaliser and the
// unnormalised output a (write-up "DropKV：精确单项输出扰动评分组件", section
// 核心公式: p = softmax(K q / sqrt d), a = sum_j p_j v_j).
// Pass 2 (one thread per cached token): recomputes each logit with the same
// evaluation order as pass 1, forms p_j / (1 - p_j) as e_j / (l - e_j), and
// accumulates ratio^2 * ||a - v_j||^2 over the G*w window queries of the KV
// head (the s_j sum and the GQA sum in one register).  The squared distance is
// taken directly, not expanded, so fp32 inputs keep full relative accuracy.
#include "common.cuh"
#include "internal.h"

namespace dropkv {
namespace {

// Logit q . k / sqrt(d) in one fixed order (both passes call this, so the
// recomputed logit in pass 2 is bit-identical to pass 1's).
template <typename T>
__device__ __forceinline__ float logit(const float* qs, const T* kp, int kstride, int d,
                                       float inv_sqrt_d) {
  float acc = 0.f;
  for (int c = 0; c < d; ++c) acc = __fmaf_rn(qs[c], to_f(kp[(size_t)c * kstride]), acc);
  return __fmul_rn(acc, inv_sqrt_d);
}

template <typename T>
__global__ void __launch_bounds__(128)
k_simt_pass1(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v, Lens lens,
             int Hq, int Hkv, int n_max, int d, int w, float inv_sqrt_d,
             float* __restrict__ stats, float* __restrict__ attn) {
  __shared__ float qs[256];
  __shared__ float es[128];
  __shared__ float red[4];
  const int row = blockIdx.x;  // (b, hq, t) flattened like q
  const int t = row % w;
  const int hq = (row / w) % Hq;
  const int b = row / (w * Hq);
  const int h = hq / (Hq / Hkv);
  const int L = lens.L[b];
  const int P = L - w + t;  // causal tail alignment: query t sees keys 0..P
  const int tid = threadIdx.x;
  for (int c = tid; c < d; c += 128) qs[c] = to_f(q[(size_t)row * d + c]);
  __syncthreads();
  const T* K = k + ((size_t)b * Hkv + h) * (size_t)n_max * d;
  const T* V = v + ((size_t)b * Hkv + h) * (size_t)n_max * d;
  float m = -CUDART_INF_F, l = 0.f, a0 = 0.f, a1 = 0.f;
  for (int j0 = 0; j0 <= P; j0 += 128) {
    const int j = j0 + tid;
    float x = -CUDART_INF_F;
    if (j <= P) x = logit(qs, K + (size_t)j * d, 1, d, inv_sqrt_d);
    const float mt = block_max<128>(x, red);
    const float m_new = fmaxf(m, mt);
    const float scale = (m == -CUDART_INF_F) ? 0.f : expf(m - m_new);
    const float e = (j <= P) ? expf(x - m_new) : 0.f;
    es[tid] = e;
    const float lt = block_sum<128>(e, red);  // its barriers also publish es[]
    l = l * scale + lt;
    a0 *= scale;
    a1 *= scale;
    const int cnt = min(128, P + 1 - j0);
    for (int jj = 0; jj < cnt; ++jj) {
      const float ej = es[jj];
      const T* vr = V + (size_t)(j0 + jj) * d;
      if (tid < d) a0 = fmaf(ej, to_f(vr[tid]), a0);
      if (tid + 128 < d) a1 = fmaf(ej, to_f(vr[tid + 128]), a1);
    }
    m = m_new;
    __syncthreads();
  }
  if (tid == 0) {
    stats[2 * (size_t)row] = m;
    stats[2 * (size_t)row + 1] = l;
  }
  if (tid < d) attn[(size_t)row * d + tid] = a0 / l;
  if (tid + 128 < d) attn[(size_t)row * d + tid + 128] = a1 / l;
}

constexpr int kQB = 8;  // window queries staged in shared memory at a time

template <typename T, int TPB>
__global__ void __launch_bounds__(TPB)
k_simt_pass2(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v, Lens lens,
             int Hq, int Hkv, int n_max, int d, int w, float inv_sqrt_d,
             const float* __restrict__ stats, const float* __restrict__ attn,
             float* __restrict__ part, int32_t* __restrict__ status) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  T* ks = reinterpret_cast<T*>(smem_raw);  // [d][TPB] keys, transposed
  T* vs = ks + (size_t)d * TPB;             // [d][TPB] values, transposed
  float* qa = reinterpret_cast<float*>(vs + (size_t)d * TPB);  // [kQB][2][d]
  const int bh = blockIdx.y, b = bh / Hkv, h = bh % Hkv;
  const int L = lens.L[b];
  const int j0 = blockIdx.x * TPB;
  if (j0 >= L) return;
  const int tid = threadIdx.x, j = j0 + tid;
  const bool valid = j < L;
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
  float s = 0.f;
  for (int i0 = 0; i0 < NQ; i0 += kQB) {
    const int nb = min(kQB, NQ - i0);
    for (int idx = tid; idx < nb * d; idx += TPB) {
      const int i = idx / d, c = idx % d;
      qa[(2 * i) * d + c] = to_f(q[(qrow0 + i0 + i) * d + c]);
      qa[(2 * i + 1) * d + c] = attn[(qrow0 + i0 + i) * d + c];
    }
    __syncthreads();
    for (int i = 0; i < nb; ++i) {
      const int r = i0 + i;
      const int P = L - w + r % w;
      if (valid && j <= P) {
        const float m = stats[2 * (qrow0 + r)], l = stats[2 * (qrow0 + r) + 1];
        const float x = logit(qa + 2 * i * d, ks + tid, TPB, d, inv_sqrt_d);
        const float e = expf(x - m);
        const float den = l - e;  // (1 - p_j) * l
        if (!(den > 0.f)) {       // p_j rounds to 1: removal is singular
          atomicOr(status, kStatusSingular);
          continue;
        }
        const float ratio = e / den;  // p_j / (1 - p_j)
        const float* A = qa + (2 * i + 1) * d;
        float sq = 0.f;
        for (int c = 0; c < d; ++c) {
          const float df = A[c] - to_f(vs[c * TPB + tid]);
          sq = fmaf(df, df, sq);
        }
        s = fmaf(ratio * ratio, sq, s);
      }
    }
    __syncthreads();
  }
  if (valid) part[((size_t)b * Hkv + h) * n_max + j] = s;
}

template <typename T, int TPB>
cudaError_t pass2_launch(const dropkv_shape& s, const void* q, const void* k, const void* v,
                         const Lens& lens, const float* stats, const float* attn, float* part,
                         int32_t* status, cudaStream_t st) {
  const size_t smem = 2 * (size_t)s.d * TPB * sizeof(T) + (size_t)kQB * 2 * s.d * sizeof(float);
  auto fn = k_simt_pass2<T, TPB>;
  cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((s.n_max + TPB - 1) / TPB, lens.B * s.Hkv);
  fn<<<grid, TPB, smem, st>>>((const T*)q, (const T*)k, (const T*)v, lens, s.Hq, s.Hkv, s.n_max,
                              s.d, s.window, 1.0f / sqrtf((float)s.d), stats, attn, part, status);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_simt_pass1(const dropkv_shape& s, const void* q, const void* k,
                              const void* v, const Lens& lens, float* stats, float* attn,
                              cudaStream_t st) {
  const int rows = lens.B * s.Hq * s.window;
  const float isd = 1.0f / sqrtf((float)s.d);
  if (s.dtype == DROPKV_BF16)
    k_simt_pass1<__nv_bfloat16><<<rows, 128, 0, st>>>(
        (const __nv_bfloat16*)q, (const __nv_bfloat16*)k, (const __nv_bfloat16*)v, lens, s.Hq,
        s.Hkv, s.n_max, s.d, s.window, isd, stats, attn);
  else
    k_simt_pass1<float><<<rows, 128, 0, st>>>((const float*)q, (const float*)k, (const float*)v,
                                               lens, s.Hq, s.Hkv, s.n_max, s.d, s.window, isd,
                                               stats, attn);
  return cudaGetLastError();
}

cudaError_t launch_simt_pass2(const dropkv_shape& s, const void* q, const void* k,
                              const void* v, const Lens& lens, const float* stats,
                              const float* attn, float* part, int32_t* status,
                              cudaStream_t st) {
  if (s.dtype == DROPKV_BF16)
    return pass2_launch<__nv_bfloat16, 128>(s, q, k, v, lens, stats, attn, part, status, st);
  if (s.d <= 128)
    return pass2_launch<float, 128>(s, q, k, v, lens, stats, attn, part, status, st);
  return pass2_launch<float, 64>(s, q, k, v, lens, stats, attn, part, status, st);
}

}  // namespace dropkv
