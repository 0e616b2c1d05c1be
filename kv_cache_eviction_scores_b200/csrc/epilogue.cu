// epilogue.cu -- GQA mean-merge + MaxPool1D + window protection, fused.
//
// Write-up "DropKV：精确单项输出扰动评分组件", Algorithm 1 paragraph after the
// core formula: the query heads sharing a physical KV head are averaged, the
// merged scores are max-pooled along the tokens, and the final observation
// window is set to +inf.  Pooling: odd kernel, stride 1, window clipped to
// [0, L) (out-of-range taps ignored), applied to the merged scores of every
// position before the window is overwritten.  Positions >= L are written NaN.
//
// The scoring passes leave `nparts` partial sums per token (one per query
// chunk and column group); merged[j] = (sum over parts, in part order) / G.
// One CTA handles 1024 positions of one (b, h), four per thread with 16-byte
// loads, and stages the merged values of its tile plus the pooling halo in
// shared memory, so every merged value is formed with the same operation order
// wherever it is read.
#include "common.cuh"
#include "internal.h"

namespace dropkv {
namespace {

constexpr int kThreads = 256;
constexpr int kVec = 4;                      // positions per thread
constexpr int kTile = kThreads * kVec;       // positions per CTA

// merged value of position jj: (sum over parts, in part order) / G, or -inf
// outside [0, L) so that out-of-range pooling taps never win
__device__ __forceinline__ float merged_at(const float* __restrict__ parts, int nparts,
                                           size_t part_stride, size_t base, int jj, int L,
                                           float G) {
  if (jj < 0 || jj >= L) return -CUDART_INF_F;
  float sum = 0.f;
  for (int p = 0; p < nparts; ++p) sum += __ldg(parts + p * part_stride + base + jj);
  return sum / G;
}

__global__ void __launch_bounds__(kThreads)
k_epilogue(const float* __restrict__ parts, int nparts, size_t part_stride, Lens lens, int Hkv,
           int n_max, int w, int radius, float G, float* __restrict__ scores) {
  extern __shared__ float merged[];  // radius + kTile + radius
  pdl_trigger();
  pdl_wait();  // the partial planes come from the previous kernel
  const int bh = blockIdx.y, b = bh / Hkv;
  const int L = lens.L[b];
  const int j0 = blockIdx.x * kTile;
  const size_t base = (size_t)bh * n_max;
  // the tile body: 4 consecutive positions per thread with 16-byte loads when
  // the rows allow it (n_max % 4 == 0 keeps every part row 16-byte aligned)
  const int jt = j0 + threadIdx.x * kVec;
  if ((n_max & 3) == 0 && jt + kVec <= L) {
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int p = 0; p < nparts; ++p) {
      const float4 v = __ldg(reinterpret_cast<const float4*>(parts + p * part_stride + base + jt));
      acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
    }
    float* m = merged + radius + threadIdx.x * kVec;
    m[0] = acc.x / G; m[1] = acc.y / G; m[2] = acc.z / G; m[3] = acc.w / G;
  } else {
    for (int u = 0; u < kVec; ++u)
      merged[radius + threadIdx.x * kVec + u] =
          merged_at(parts, nparts, part_stride, base, jt + u, L, G);
  }
  // the pooling halo on both sides
  for (int i = threadIdx.x; i < 2 * radius; i += kThreads) {
    const int off = i < radius ? i : kTile + i;  // index into merged
    merged[off] = merged_at(parts, nparts, part_stride, base, j0 - radius + off, L, G);
  }
  __syncthreads();
#pragma unroll
  for (int u = 0; u < kVec; ++u) {
    const int t = threadIdx.x + u * kThreads;  // coalesced output positions
    const int j = j0 + t;
    if (j >= n_max) break;
    float out;
    if (j >= L) {
      out = CUDART_NAN_F;
    } else if (j >= L - w) {
      out = CUDART_INF_F;
    } else {
      out = merged[t];
      for (int k = 1; k <= 2 * radius; ++k) out = fmaxf(out, merged[t + k]);
    }
    scores[base + j] = out;
  }
}

}  // namespace

cudaError_t launch_epilogue(const dropkv_shape& s, const Lens& lens, const float* parts,
                            int nparts, size_t part_stride, float* scores, cudaStream_t st) {
  const int radius = s.pool_kernel / 2;
  const size_t smem = (size_t)(kTile + 2 * radius) * sizeof(float);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(k_epilogue, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
  }
  dim3 grid((s.n_max + kTile - 1) / kTile, lens.B * s.Hkv);
  return launch_ex(k_epilogue, grid, dim3(kThreads), smem, st, true, 1, parts, nparts, part_stride,
                   lens, s.Hkv, s.n_max, s.window, radius, (float)(s.Hq / s.Hkv), scores);
}

}  // namespace dropkv
