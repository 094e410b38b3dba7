// Selection-quality metrics (LatentIndex summary, Sec. 4.1, Sec. C.2,
// Sec. C.3, Sec. D.3): the attention mass a selection captures, relative to
// the best set of the same size, per head and for the head average.  The
// best sets come from the library's own exact top-k; these kernels only
// average heads and add up masses.
#include <cuda_runtime.h>

#include <algorithm>

#include "internal.h"
#include "sm100.cuh"

namespace li {
namespace {

__device__ __forceinline__ float warp_sum_f(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

__device__ __forceinline__ int valid_len(const int32_t* lengths, int r, int N) {
  int n = lengths ? lengths[r] : N;
  return n < 0 ? 0 : (n > N ? N : n);
}

// pbar[r][s] = (sum over h in ascending order of probs[r][h][s]) / H for
// s < n_r; 0 past the prefix.  Consecutive threads take consecutive s.
__global__ void __launch_bounds__(256) head_mean_kernel(const float* __restrict__ probs, int rows, int H, int N,
                                                        const int32_t* __restrict__ lengths, float* __restrict__ pbar) {
  pdl_begin();
  const int64_t total = static_cast<int64_t>(rows) * N;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int r = static_cast<int>(i / N), s = static_cast<int>(i - static_cast<int64_t>(r) * N);
    float acc = 0.f;
    if (s < valid_len(lengths, r, N)) {
      const float* p = probs + static_cast<int64_t>(r) * H * N + s;
      for (int h = 0; h < H; ++h) acc += p[static_cast<int64_t>(h) * N];
      acc = __fdiv_rn(acc, static_cast<float>(H));
    }
    pbar[i] = acc;
  }
}

// One warp per (query row r, head h): the selected mass sum_j vals[r, h,
// sel[r][j]] over valid selected positions, the best mass sum of the row's
// top-K values, and their ratio (0 when the best mass is 0).
__global__ void __launch_bounds__(256) recall_kernel(const float* __restrict__ vals, int rows, int Hh, int N,
                                                     const int32_t* __restrict__ lengths,
                                                     const int32_t* __restrict__ sel, int k,
                                                     const int32_t* __restrict__ top_idx,
                                                     const float* __restrict__ top_val, int K,
                                                     float* __restrict__ out) {
  pdl_begin();
  const int w = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (w >= rows * Hh) return;
  const int r = w / Hh;
  const int n = valid_len(lengths, r, N);
  const float* row = vals + static_cast<int64_t>(w) * N;
  float got = 0.f, best = 0.f;
  for (int j = lane; j < k; j += 32) {
    const int s = sel[static_cast<int64_t>(r) * k + j];
    if (s >= 0 && s < n) got += row[s];
  }
  for (int j = lane; j < K; j += 32) {
    const int64_t o = static_cast<int64_t>(w) * K + j;
    if (top_idx[o] >= 0) best += top_val[o];
  }
  got = warp_sum_f(got);
  best = warp_sum_f(best);
  if (lane == 0) out[w] = best > 0.f ? __fdiv_rn(got, best) : 0.f;
}

}  // namespace

cudaError_t launch_head_mean(const float* probs, int rows, int H, int N, const int32_t* lengths, float* pbar,
                             int num_sms, cudaStream_t st) {
  const int64_t total = static_cast<int64_t>(rows) * N;
  const int64_t want = (total + 255) / 256;
  const int grid = static_cast<int>(std::min<int64_t>(want, static_cast<int64_t>(num_sms) * 8));
  return launch_pdl(head_mean_kernel, dim3(grid > 0 ? grid : 1), dim3(256), 0, st, 1, probs, rows, H, N, lengths,
                    pbar);
}

cudaError_t launch_recall(const float* vals, int rows, int Hh, int N, const int32_t* lengths, const int32_t* sel,
                          int k, const int32_t* top_idx, const float* top_val, int K, float* out, cudaStream_t st) {
  const int warps = rows * Hh;
  return launch_pdl(recall_kernel, dim3((warps + 7) / 8), dim3(256), 0, st, 1, vals, rows, Hh, N, lengths, sel, k,
                    top_idx, top_val, K, out);
}

}  // namespace li
