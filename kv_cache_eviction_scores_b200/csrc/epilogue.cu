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
// chunk); merged[j] = (sum over parts) / G.  One CTA handles 256 positions of
// one (b, h) and stages the merged values of its tile plus the pooling halo in
// shared memory, so every merged value is formed with the same operation order
// wherever it is read.
#include "common.cuh"
#include "internal.h"

namespace dropkv {
namespace {

constexpr int kTile = 256;

__global__ void __launch_bounds__(kTile)
k_epilogue(const float* __restrict__ parts, int nparts, size_t part_stride, Lens lens, int Hkv,
           int n_max, int w, int radius, float G, float* __restrict__ scores) {
  extern __shared__ float merged[];  // kTile + 2 * radius
  const int bh = blockIdx.y, b = bh / Hkv;
  const int L = lens.L[b];
  const int j0 = blockIdx.x * kTile;
  const size_t base = (size_t)bh * n_max;
  for (int i = threadIdx.x; i < kTile + 2 * radius; i += kTile) {
    const int jj = j0 - radius + i;
    float val = -CUDART_INF_F;
    if (jj >= 0 && jj < L) {
      float sum = 0.f;
      for (int p = 0; p < nparts; ++p) sum += parts[p * part_stride + base + jj];
      val = sum / G;
    }
    merged[i] = val;
  }
  __syncthreads();
  const int j = j0 + threadIdx.x;
  if (j >= n_max) return;
  float out;
  if (j >= L) {
    out = CUDART_NAN_F;
  } else if (j >= L - w) {
    out = CUDART_INF_F;
  } else {
    out = merged[threadIdx.x];
    for (int u = 1; u <= 2 * radius; ++u) out = fmaxf(out, merged[threadIdx.x + u]);
  }
  scores[base + j] = out;
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
  k_epilogue<<<grid, kTile, smem, st>>>(parts, nparts, part_stride, lens, s.Hkv, s.n_max,
                                        s.window, radius, (float)(s.Hq / s.Hkv), scores);
  return cudaGetLastError();
}

}  // namespace dropkv
