// construct.cu -- the two small steps on either side of the scan:
//
//  * latent (or key) construction and append (LatentIndex summary, Sec. 3.1:
//    the anchor builds the shared latent c = W_down h once per token; the
//    DSA-style path builds one key per layer the same way), quantised to the
//    cache dtype and written at row lengths[b] + t;
//  * query-side decoder absorption (Sec. 3.1, Sec. A.2, Sec. B.2):
//    qt_h = W_K^T q_h (+ beta_h = q_h . b_K), quantised to the scan's dtype.
//
// Both accumulate in fp32 in a fixed order, so a result is identical whichever
// output dtype is requested.
#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include "internal.h"
#include "sm100.cuh"

namespace li {

namespace {

__device__ __forceinline__ float load_elt(const void* p, int64_t i, int dtype) {
  return dtype == LI_BF16 ? __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(p)[i])
                          : reinterpret_cast<const float*>(p)[i];
}

__device__ __forceinline__ uint8_t to_e4m3(float x) {
  return static_cast<uint8_t>(__nv_cvt_float_to_fp8(x, __NV_SATFINITE, __NV_E4M3));
}

constexpr int kGemvTok = 8;    // tokens per warp task
constexpr int kGemvWarps = 8;

// out[m][j] = sum_i W[j][i] * h[m][i]; one warp per output j and 8 tokens.
// Lanes stride the reduction dimension by 8 elements (16 B of bf16), then a
// fixed butterfly sums the lanes.
template <typename T>
__global__ void __launch_bounds__(kGemvWarps * 32) gemv_kernel(const T* __restrict__ h,
                                                               const T* __restrict__ W, int d_model,
                                                               int dim, int n_tok, float* __restrict__ out) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int j = blockIdx.x * kGemvWarps + warp;
  const int m0 = blockIdx.y * kGemvTok;
  if (j >= dim) return;
  const int nm = min(kGemvTok, n_tok - m0);
  float acc[kGemvTok];
#pragma unroll
  for (int t = 0; t < kGemvTok; ++t) acc[t] = 0.f;
  const T* wrow = W + static_cast<int64_t>(j) * d_model;
  for (int i = lane * 8; i < d_model; i += 256) {
    float wv[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) wv[e] = static_cast<float>(wrow[i + e]);
#pragma unroll
    for (int t = 0; t < kGemvTok; ++t) {
      if (t < nm) {
        const T* hr = h + static_cast<int64_t>(m0 + t) * d_model + i;
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[t] = fmaf(wv[e], static_cast<float>(hr[e]), acc[t]);
      }
    }
  }
#pragma unroll
  for (int t = 0; t < kGemvTok; ++t) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc[t] += __shfl_xor_sync(0xffffffffu, acc[t], o);
  }
  if (lane == 0)
    for (int t = 0; t < nm; ++t) out[static_cast<int64_t>(m0 + t) * dim + j] = acc[t];
}

// One warp per new token: write c (fp32 rows) into the cache at row
// lengths[b] + t0 + t in the cache dtype.  The last block to finish advances
// lengths[b] by T_total when `bump` is set (all blocks read lengths first).
__global__ void __launch_bounds__(256) store_kernel(const float* __restrict__ c, int64_t c_tok_stride,
                                                    int batch, int T_chunk, int t0, int T_total, int bump,
                                                    void* data, float* scale, int32_t* lengths,
                                                    int capacity, int dim, int dtype,
                                                    unsigned int* done, int* status) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tok = blockIdx.x * 8 + warp;
  if (tok < batch * T_chunk) {
    const int b = tok / T_chunk, t = tok % T_chunk;
    const int len = lengths[b];
    if (len < 0 || len + T_total > capacity) {
      if (lane == 0) record_status(status, kStatusCapacity);
    } else {
      const int64_t row = static_cast<int64_t>(b) * capacity + len + t0 + t;
      const float* src = c + static_cast<int64_t>(tok) * c_tok_stride;
      float v[8];
      float amax = 0.f;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const int i = lane + 32 * e;
        v[e] = i < dim ? src[i] : 0.f;
        amax = fmaxf(amax, fabsf(v[e]));
      }
      if (dtype == LI_F32) {
        float* dst = reinterpret_cast<float*>(data) + row * dim;
#pragma unroll
        for (int e = 0; e < 8; ++e)
          if (lane + 32 * e < dim) dst[lane + 32 * e] = v[e];
      } else if (dtype == LI_BF16) {
        __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(data) + row * dim;
#pragma unroll
        for (int e = 0; e < 8; ++e)
          if (lane + 32 * e < dim) dst[lane + 32 * e] = __float2bfloat16_rn(v[e]);
      } else {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        const float sc = amax > 0.f ? __fdiv_rn(amax, 448.f) : 1.f;
        uint8_t* dst = reinterpret_cast<uint8_t*>(data) + row * dim;
#pragma unroll
        for (int e = 0; e < 8; ++e)
          if (lane + 32 * e < dim) dst[lane + 32 * e] = to_e4m3(__fdiv_rn(v[e], sc));
        if (lane == 0) scale[row] = sc;
      }
    }
  }
  if (!bump) return;
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    const unsigned prev = atomicAdd(done, 1u);
    if (prev == gridDim.x - 1) {
      __threadfence();
      for (int b = 0; b < batch; ++b) {
        const int len = lengths[b];
        if (len >= 0 && len + T_total <= capacity) lengths[b] = len + T_total;
      }
      *done = 0;
      __threadfence();
    }
  }
}

constexpr int kAbsorbHeads = 8;

// Block per (token, 8 heads); thread i computes output element i of the 8
// absorbed heads: qt[h][i] = sum_j W[h][j][i] q[h][j] (j ascending, fp32).
__global__ void __launch_bounds__(256) absorb_kernel(const void* __restrict__ q, int q_dtype, int H, int d_k,
                                                     const void* __restrict__ W, int64_t W_hs,
                                                     const float* __restrict__ bK, int64_t b_hs, int d_c,
                                                     int out_dtype, void* q_abs, float* q_abs_scale,
                                                     float* beta) {
  __shared__ float qs[kAbsorbHeads][256];
  __shared__ float red[8][kAbsorbHeads];
  const int t = blockIdx.y, h0 = blockIdx.x * kAbsorbHeads;
  const int nh = min(kAbsorbHeads, H - h0);
  for (int x = threadIdx.x; x < kAbsorbHeads * d_k; x += blockDim.x) {
    const int hh = x / d_k, jj = x % d_k;
    qs[hh][jj] = hh < nh ? load_elt(q, (static_cast<int64_t>(t) * H + h0 + hh) * d_k + jj, q_dtype) : 0.f;
  }
  __syncthreads();
  const int i = threadIdx.x;
  float acc[kAbsorbHeads];
#pragma unroll
  for (int hh = 0; hh < kAbsorbHeads; ++hh) acc[hh] = 0.f;
  if (i < d_c) {
    if (W == nullptr) {
#pragma unroll
      for (int hh = 0; hh < kAbsorbHeads; ++hh) acc[hh] = qs[hh][i];
    } else if (W_hs == 0) {
      for (int j = 0; j < d_k; ++j) {
        const float wv = load_elt(W, static_cast<int64_t>(j) * d_c + i, q_dtype);
#pragma unroll
        for (int hh = 0; hh < kAbsorbHeads; ++hh) acc[hh] = fmaf(wv, qs[hh][j], acc[hh]);
      }
    } else {
      for (int j = 0; j < d_k; ++j) {
#pragma unroll
        for (int hh = 0; hh < kAbsorbHeads; ++hh) {
          if (hh < nh) {
            const float wv = load_elt(W, (h0 + hh) * W_hs + static_cast<int64_t>(j) * d_c + i, q_dtype);
            acc[hh] = fmaf(wv, qs[hh][j], acc[hh]);
          }
        }
      }
    }
  }
  if (beta && i < nh) {
    float bsum = 0.f;
    for (int j = 0; j < d_k; ++j) bsum = fmaf(qs[i][j], bK[(h0 + i) * b_hs + j], bsum);
    beta[static_cast<int64_t>(t) * H + h0 + i] = bsum;
  }
  const int64_t obase = (static_cast<int64_t>(t) * H + h0) * d_c;
  if (out_dtype == LI_F32) {
    if (i < d_c)
      for (int hh = 0; hh < nh; ++hh) reinterpret_cast<float*>(q_abs)[obase + hh * d_c + i] = acc[hh];
  } else if (out_dtype == LI_BF16) {
    if (i < d_c)
      for (int hh = 0; hh < nh; ++hh)
        reinterpret_cast<__nv_bfloat16*>(q_abs)[obase + hh * d_c + i] = __float2bfloat16_rn(acc[hh]);
  } else {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
#pragma unroll
    for (int hh = 0; hh < kAbsorbHeads; ++hh) {
      float m = i < d_c ? fabsf(acc[hh]) : 0.f;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      if (lane == 0) red[warp][hh] = m;
    }
    __syncthreads();
    if (i < d_c) {
      for (int hh = 0; hh < nh; ++hh) {
        float amax = 0.f;
        for (int w = 0; w < 8; ++w) amax = fmaxf(amax, red[w][hh]);
        const float sc = amax > 0.f ? __fdiv_rn(amax, 448.f) : 1.f;
        reinterpret_cast<uint8_t*>(q_abs)[obase + hh * d_c + i] = to_e4m3(__fdiv_rn(acc[hh], sc));
        if (i == 0) q_abs_scale[static_cast<int64_t>(t) * H + h0 + hh] = sc;
      }
    }
  }
}

}  // namespace

cudaError_t launch_append_gemv(const void* h, int h_dtype, const void* W, int d_model, int dim, int n_tok,
                               float* out, cudaStream_t st) {
  const dim3 grid((dim + kGemvWarps - 1) / kGemvWarps, (n_tok + kGemvTok - 1) / kGemvTok);
  if (h_dtype == LI_BF16)
    gemv_kernel<__nv_bfloat16><<<grid, kGemvWarps * 32, 0, st>>>(
        reinterpret_cast<const __nv_bfloat16*>(h), reinterpret_cast<const __nv_bfloat16*>(W), d_model, dim,
        n_tok, out);
  else
    gemv_kernel<float><<<grid, kGemvWarps * 32, 0, st>>>(reinterpret_cast<const float*>(h),
                                                          reinterpret_cast<const float*>(W), d_model, dim,
                                                          n_tok, out);
  return cudaGetLastError();
}

cudaError_t launch_append_store(const float* c, int64_t c_tok_stride, int batch, int T_chunk, int t0,
                                int T_total, bool bump, void* data, float* scale, int32_t* lengths,
                                int capacity, int dim, int dtype, unsigned int* done_counter, int* status,
                                cudaStream_t st) {
  const int n_tok = batch * T_chunk;
  const int grid = (n_tok + 7) / 8;
  store_kernel<<<grid, 256, 0, st>>>(c, c_tok_stride, batch, T_chunk, t0, T_total, bump ? 1 : 0, data, scale,
                                     lengths, capacity, dim, dtype, done_counter, status);
  return cudaGetLastError();
}

cudaError_t launch_absorb(const void* q, int q_dtype, int n_tok, int H, int d_k, const void* W,
                          int64_t W_head_stride, const float* b, int64_t b_head_stride, int d_c,
                          int out_dtype, void* q_abs, float* q_abs_scale, float* beta, cudaStream_t st) {
  const dim3 grid((H + kAbsorbHeads - 1) / kAbsorbHeads, n_tok);
  absorb_kernel<<<grid, 256, 0, st>>>(q, q_dtype, H, d_k, W, W_head_stride, b, b_head_stride, d_c, out_dtype,
                                      q_abs, q_abs_scale, beta);
  return cudaGetLastError();
}

}  // namespace li
