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
#include <algorithm>

#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include "internal.h"
#include "sm100.cuh"

namespace li {

namespace {

__device__ __forceinline__ uint8_t to_e4m3(float x) {
  return static_cast<uint8_t>(__nv_cvt_float_to_fp8(x, __NV_SATFINITE, __NV_E4M3));
}

constexpr int kGemvTok = 8;    // tokens per warp task
constexpr int kMaxSplits = 32; // reduction splits of the construction GEMV
constexpr int kGemvWarps = 8;

template <typename T>
__device__ __forceinline__ void load8(const T* p, float (&v)[8]);
template <>
__device__ __forceinline__ void load8<__nv_bfloat16>(const __nv_bfloat16* p, float (&v)[8]) {
  const uint4 u = *reinterpret_cast<const uint4*>(p);
  const __nv_bfloat162* b = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float2 f = __bfloat1622float2(b[e]);
    v[2 * e] = f.x;
    v[2 * e + 1] = f.y;
  }
}
template <>
__device__ __forceinline__ void load8<float>(const float* p, float (&v)[8]) {
  const float4 a = *reinterpret_cast<const float4*>(p);
  const float4 b = *reinterpret_cast<const float4*>(p + 4);
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

// Split-K GEMV: partial[s][m][j] = sum_{i in split s} W[j][i] * h[m][i].  One
// warp per (output j, split s, 8 tokens); lanes take 8 consecutive elements
// (16-byte loads) at a stride of 256, then a fixed butterfly sums the lanes.
// The store kernel adds the splits in order, so results are deterministic.
template <typename T>
__global__ void __launch_bounds__(kGemvWarps * 32) gemv_kernel(const T* __restrict__ h,
                                                               const T* __restrict__ W, int d_model,
                                                               int dim, int n_tok, int splits,
                                                               float* __restrict__ out) {
  pdl_begin();
  pdl_release();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int task = blockIdx.x * kGemvWarps + warp;
  if (task >= dim * splits) return;
  const int j = task / splits, sp = task % splits;
  const int m0 = blockIdx.y * kGemvTok;
  const int nm = min(kGemvTok, n_tok - m0);
  const int len = d_model / splits;
  const int i0 = sp * len, i1 = i0 + len;
  float acc[kGemvTok];
#pragma unroll
  for (int t = 0; t < kGemvTok; ++t) acc[t] = 0.f;
  const T* wrow = W + static_cast<int64_t>(j) * d_model;
  for (int i = i0 + lane * 8; i < i1; i += 256) {
    float wv[8];
    load8<T>(wrow + i, wv);
#pragma unroll
    for (int t = 0; t < kGemvTok; ++t) {
      if (t < nm) {
        float hv[8];
        load8<T>(h + static_cast<int64_t>(m0 + t) * d_model + i, hv);
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[t] = fmaf(wv[e], hv[e], acc[t]);
      }
    }
  }
#pragma unroll
  for (int t = 0; t < kGemvTok; ++t) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc[t] += __shfl_xor_sync(0xffffffffu, acc[t], o);
  }
  if (lane == 0)
    for (int t = 0; t < nm; ++t)
      out[(static_cast<int64_t>(sp) * n_tok + m0 + t) * dim + j] = acc[t];
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
  return x;
}

// Per-lane constants of the row transforms (the same for every row): the
// LayerNorm affine terms and the rotary frequency of each element the lane
// holds.  Loaded once per warp, before the rows are ready, so that no global
// read sits between a row's reduction and its store.
struct TfLane {
  float g[8], b[8], f[8];
};

__device__ __forceinline__ TfLane load_tf_lane(const RowTransform& tf, int lane) {
  TfLane t;
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const int i = lane + 32 * e;
    const bool in_norm = tf.norm_dim > 0 && i >= tf.norm_offset && i < tf.norm_offset + tf.norm_dim;
    const bool in_rope = tf.rope_dim > 0 && i >= tf.rope_offset && i < tf.rope_offset + tf.rope_dim;
    t.g[e] = in_norm && tf.gamma ? __ldg(tf.gamma + (i - tf.norm_offset)) : 1.f;
    t.b[e] = in_norm && tf.beta ? __ldg(tf.beta + (i - tf.norm_offset)) : 0.f;
    t.f[e] = in_rope ? __ldg(tf.inv_freq + ((i - tf.rope_offset) >> 1) / tf.rope_sources) : 0.f;
  }
  return t;
}

// The two-branch latent's row transforms (LatentIndex summary, Sec. 3.1,
// Sec. A.2, Sec. D.2) on one fp32 row held by a warp (lane holds elements
// lane + 32 e): LayerNorm of the NoPE range (biased variance, correctly
// rounded division and square root), and rotation of the rotary range at
// position `pos`: slot p = (x[2p], x[2p+1]) of the range turns by
// pos * inv_freq[p / sources], the angle formed exactly and its cosine and
// sine taken in double precision, then rounded to fp32.  Slot partners are
// adjacent lanes (the range starts on an even element).
__device__ __forceinline__ void transform_row(float (&v)[8], int lane, int64_t pos, const RowTransform& tf,
                                              const TfLane& c) {
  if (tf.norm_dim > 0) {
    const int a = tf.norm_offset, b = tf.norm_offset + tf.norm_dim;
    float s = 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const int i = lane + 32 * e;
      if (i >= a && i < b) s += v[e];
    }
    const float mean = __fdiv_rn(warp_sum(s), static_cast<float>(tf.norm_dim));
    float ss = 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const int i = lane + 32 * e;
      if (i >= a && i < b) {
        const float d = v[e] - mean;
        ss = fmaf(d, d, ss);
      }
    }
    const float sd = __fsqrt_rn(__fdiv_rn(warp_sum(ss), static_cast<float>(tf.norm_dim)) + tf.eps);
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const int i = lane + 32 * e;
      if (i >= a && i < b) v[e] = __fdiv_rn(v[e] - mean, sd) * c.g[e] + c.b[e];
    }
  }
  if (tf.rope_dim > 0) {
    const int a = tf.rope_offset, b = tf.rope_offset + tf.rope_dim;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const int i = lane + 32 * e;
      const float partner = __shfl_xor_sync(0xffffffffu, v[e], 1);
      if (i >= a && i < b) {
        double sn, cs;
        sincos(static_cast<double>(pos) * static_cast<double>(c.f[e]), &sn, &cs);
        const float co = static_cast<float>(cs), si = static_cast<float>(sn);
        v[e] = ((i - a) & 1) == 0 ? v[e] * co - partner * si : partner * si + v[e] * co;
      }
    }
  }
}

// Write one fp32 row (lane holds elements lane + 32 e) into the cache at
// `row` (sequence position `pos`) in the cache dtype, after the row
// transforms.  E4M3 rows get scale amax / 448 per row, or, with
// scale_split > 0, one per segment: elements [0, scale_split) and
// [scale_split, dim), stored as scale[2 row] and scale[2 row + 1].
template <bool TF>
__device__ __forceinline__ void write_row(float (&v)[8], int lane, int64_t row, int64_t pos, int dim, int dtype,
                                          int scale_split, const RowTransform& tf, const TfLane& tc, void* data,
                                          float* scale) {
  if constexpr (TF) transform_row(v, lane, pos, tf, tc);
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
    float am0 = 0.f, am1 = 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const int i = lane + 32 * e;
      if (i < dim) {
        if (scale_split > 0 && i >= scale_split) am1 = fmaxf(am1, fabsf(v[e]));
        else am0 = fmaxf(am0, fabsf(v[e]));
      }
    }
    am0 = warp_max(am0);
    am1 = warp_max(am1);
    const float sc0 = am0 > 0.f ? __fdiv_rn(am0, 448.f) : 1.f;
    const float sc1 = am1 > 0.f ? __fdiv_rn(am1, 448.f) : 1.f;
    uint8_t* dst = reinterpret_cast<uint8_t*>(data) + row * dim;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const int i = lane + 32 * e;
      if (i < dim) dst[i] = to_e4m3(__fdiv_rn(v[e], scale_split > 0 && i >= scale_split ? sc1 : sc0));
    }
    if (lane == 0) {
      if (scale_split > 0) {
        scale[2 * row] = sc0;
        scale[2 * row + 1] = sc1;
      } else {
        scale[row] = sc0;
      }
    }
  }
}

// Decode append in one launch: the split-K GEMV above, after which the last
// block to finish (a counter in the workspace) adds every token's splits in
// split order, quantises the rows, writes them at lengths[b] + t, advances
// lengths[b] by T and resets the counter.  The last block first copies all
// partial sums to shared memory with many loads in flight, then sums each
// output over the splits in order.  Used when the partials fit in the
// block's shared memory.
constexpr int kFuseMaxPartials = 16384;   // floats of partial sums (64 KB)
constexpr int kAppendWarps = 16;          // 512-thread blocks: few arrivals on the completion counter
constexpr int kStagePer = kFuseMaxPartials / (kAppendWarps * 32);   // partial sums each thread stages

template <typename T, bool TF>
__global__ void __launch_bounds__(kAppendWarps * 32) gemv_append_kernel(const T* __restrict__ h,
                                                                      const T* __restrict__ W, int d_model,
                                                                      int dim, int n_tok, int splits,
                                                                      float* __restrict__ part, int batch, int T_tok,
                                                                      void* data, float* scale, int32_t* lengths,
                                                                      int capacity, int dtype, int scale_split,
                                                                      RowTransform tf, unsigned int* done,
                                                                      int* status) {
  pdl_begin();
  pdl_release();
  extern __shared__ __align__(16) float ps[];       // [splits][n_tok * dim], then cs [n_tok * dim]
  __shared__ unsigned last;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // block b takes split b % splits for kAppendWarps consecutive outputs, so
  // its warps share one slice of the hidden states (read once, then from L1)
  const int sp = static_cast<int>(blockIdx.x) % splits;
  const int j = (static_cast<int>(blockIdx.x) / splits) * kAppendWarps + warp;
  const int len = d_model / splits;   // a multiple of 256 (append_fused_splits)
  const int i0 = sp * len;
  // The block's slice of every token's hidden state goes to shared memory
  // once (all 16-byte pieces in flight), while each warp requests all of its
  // decoder row slice at once: the GEMV waits one memory round trip, not one
  // per 256-element step.  (The last block reuses this memory for the
  // partial sums afterwards.)
  T* hs = reinterpret_cast<T*>(ps);   // [n_tok][len]
  {
    const int per_tok = len * static_cast<int>(sizeof(T)) / 16;
    const uint32_t dst = static_cast<uint32_t>(__cvta_generic_to_shared(hs));
    for (int x = threadIdx.x; x < n_tok * per_tok; x += blockDim.x) {
      const int t = x / per_tok, c = x - t * per_tok;
      cp_async_16(dst + 16u * x, h + static_cast<int64_t>(t) * d_model + i0 + c * (16 / static_cast<int>(sizeof(T))));
    }
    cp_async_commit();
  }
  float acc[kGemvTok];
#pragma unroll
  for (int t = 0; t < kGemvTok; ++t) acc[t] = 0.f;
  constexpr int kSteps = 8;           // 256-element steps held in registers at once
  for (int ib = 0; ib < len; ib += kSteps * 256) {
    float wv[kSteps][8];
    if (j < dim) {
      const T* wrow = W + static_cast<int64_t>(j) * d_model + i0;
#pragma unroll
      for (int u = 0; u < kSteps; ++u)
        if (ib + u * 256 < len) load8<T>(wrow + ib + u * 256 + lane * 8, wv[u]);
    }
    if (ib == 0) {
      cp_async_wait_all();
      __syncthreads();
    }
    if (j < dim) {
#pragma unroll
      for (int u = 0; u < kSteps; ++u) {
        const int i = ib + u * 256 + lane * 8;
        if (ib + u * 256 < len) {
#pragma unroll
          for (int t = 0; t < kGemvTok; ++t) {
            if (t < n_tok) {
              float hv[8];
              load8<T>(hs + t * len + i, hv);
#pragma unroll
              for (int e = 0; e < 8; ++e) acc[t] = fmaf(wv[u][e], hv[e], acc[t]);
            }
          }
        }
      }
    }
  }
  if (j < dim) {
#pragma unroll
    for (int t = 0; t < kGemvTok; ++t) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) acc[t] += __shfl_xor_sync(0xffffffffu, acc[t], o);
    }
    if (lane == 0)
      for (int t = 0; t < n_tok; ++t) part[(static_cast<int64_t>(sp) * n_tok + t) * dim + j] = acc[t];
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    // acquire-release at GPU scope: publishes this block's partial sums
    // (ordered before it by the barrier) and, in the last block, makes
    // every other block's visible to the reads below
    unsigned prev;
    asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], 1;" : "=r"(prev) : "l"(done) : "memory");
    last = prev == gridDim.x - 1 ? 1u : 0u;
  }
  __syncthreads();
  if (!last) return;
  TfLane tc;
  if constexpr (TF) tc = load_tf_lane(tf, threadIdx.x & 31);
  const int nx = n_tok * dim, np = splits * nx;   // np <= kStagePer * blockDim.x
  {
    // every partial sum in flight at once
    float v[kStagePer];
#pragma unroll
    for (int m = 0; m < kStagePer; ++m) {
      const int idx = static_cast<int>(threadIdx.x) + m * kAppendWarps * 32;
      v[m] = idx < np ? __ldcg(part + idx) : 0.f;
    }
#pragma unroll
    for (int m = 0; m < kStagePer; ++m) {
      const int idx = static_cast<int>(threadIdx.x) + m * kAppendWarps * 32;
      if (idx < np) ps[idx] = v[m];
    }
  }
  __syncthreads();
  float* cs = ps + np;
  for (int x = threadIdx.x; x < nx; x += blockDim.x) {
    float sum = ps[x];
    for (int sp = 1; sp < splits; ++sp) sum += ps[sp * nx + x];
    cs[x] = sum;
  }
  __syncthreads();
  for (int m = warp; m < n_tok; m += kAppendWarps) {
    const int b = m / T_tok, t = m % T_tok;
    const int len = lengths[b];
    if (len < 0 || len + T_tok > capacity) {
      if (lane == 0) record_status(status, kStatusCapacity);
      continue;
    }
    float v[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const int i = lane + 32 * e;
      v[e] = i < dim ? cs[m * dim + i] : 0.f;
    }
    write_row<TF>(v, lane, static_cast<int64_t>(b) * capacity + len + t, len + t, dim, dtype, scale_split, tf, tc,
                  data, scale);
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int b = 0; b < batch; ++b) {
      const int len = lengths[b];
      if (len >= 0 && len + T_tok <= capacity) lengths[b] = len + T_tok;
    }
    *done = 0;
    __threadfence();
  }
}

// One warp per new token: write c (fp32 rows) into the cache at row
// lengths[b] + t0 + t in the cache dtype.  The last block to finish advances
// lengths[b] by T_total when `bump` is set (all blocks read lengths first).
template <bool TF>
__global__ void __launch_bounds__(256) store_kernel(const float* __restrict__ c, int64_t c_tok_stride,
                                                    int64_t split_stride, int splits,
                                                    int batch, int T_chunk, int t0, int T_total, int bump,
                                                    void* data, float* scale, int32_t* lengths,
                                                    int capacity, int dim, int dtype, int scale_split,
                                                    RowTransform tf, unsigned int* done, int* status) {
  pdl_begin();
  pdl_release();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  TfLane tc;
  if constexpr (TF) tc = load_tf_lane(tf, lane);
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
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const int i = lane + 32 * e;
        float x = 0.f;
        if (i < dim) {
          // all partial sums in flight at once, then added in split order
          float part[kMaxSplits];
#pragma unroll
          for (int sp = 0; sp < kMaxSplits; ++sp) part[sp] = sp < splits ? src[sp * split_stride + i] : 0.f;
          x = part[0];
#pragma unroll
          for (int sp = 1; sp < kMaxSplits; ++sp)
            if (sp < splits) x += part[sp];
        }
        v[e] = x;
      }
      write_row<TF>(v, lane, row, len + t0 + t, dim, dtype, scale_split, tf, tc, data, scale);
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

constexpr int kAbsorbHeads = 2;

template <typename T>
__device__ __forceinline__ float to_f(T x) { return static_cast<float>(x); }
template <>
__device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }

// Block per (token, 2 heads); thread i computes output element i of both
// absorbed heads: qt[h][i] = sum_j W[h][j][i] q[h][j] (j ascending, fp32).
// The decoder is read in column order (coalesced over i), 8 rows per step.
template <typename T>
__global__ void __launch_bounds__(256) absorb_kernel(const T* __restrict__ q, int H, int d_k,
                                                     const T* __restrict__ W, int64_t W_hs,
                                                     const float* __restrict__ bK, int64_t b_hs, int d_c,
                                                     int out_dtype, void* q_abs, float* q_abs_scale,
                                                     float* beta) {
  pdl_begin();
  pdl_release();
  __shared__ float qs[kAbsorbHeads][256];
  __shared__ float red[8][kAbsorbHeads];
  const int t = blockIdx.y, h0 = blockIdx.x * kAbsorbHeads;
  const int nh = min(kAbsorbHeads, H - h0);
  for (int x = threadIdx.x; x < kAbsorbHeads * d_k; x += blockDim.x) {
    const int hh = x / d_k, jj = x % d_k;
    qs[hh][jj] = hh < nh ? to_f(q[(static_cast<int64_t>(t) * H + h0 + hh) * d_k + jj]) : 0.f;
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
    } else {
#pragma unroll
      for (int hh = 0; hh < kAbsorbHeads; ++hh) {
        if (hh >= nh) break;
        if (hh > 0 && W_hs == 0) break;      // shared decoder: handled below with one read
        const T* Wh = W + (h0 + hh) * W_hs + i;
        int j = 0;
        for (; j + 8 <= d_k; j += 8) {
          float wv[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) wv[u] = to_f(Wh[static_cast<int64_t>(j + u) * d_c]);
          if (W_hs == 0) {
#pragma unroll
            for (int u = 0; u < 8; ++u)
#pragma unroll
              for (int h2 = 0; h2 < kAbsorbHeads; ++h2) acc[h2] = fmaf(wv[u], qs[h2][j + u], acc[h2]);
          } else {
#pragma unroll
            for (int u = 0; u < 8; ++u) acc[hh] = fmaf(wv[u], qs[hh][j + u], acc[hh]);
          }
        }
        for (; j < d_k; ++j) {
          const float wv = to_f(Wh[static_cast<int64_t>(j) * d_c]);
          if (W_hs == 0) {
#pragma unroll
            for (int h2 = 0; h2 < kAbsorbHeads; ++h2) acc[h2] = fmaf(wv, qs[h2][j], acc[h2]);
          } else {
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

__device__ __forceinline__ float2 load2(const __nv_bfloat16* p) {
  return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(p));
}
__device__ __forceinline__ float2 load2(const float* p) { return *reinterpret_cast<const float2*>(p); }

// Decoders of the layers one absorb launch serves (one, or a group's layers).
struct AbsorbLayers {
  const void* W[kMaxAbsorbLayers];
  int G, H;
};

// Shared decoder (one W_K for every head): rows (token, head) are taken R at a
// time per block. The decoder is staged once in shared memory with 16-byte
// loads, the R query rows as fp32; each thread then owns column pairs of a row
// and accumulates j = 0..d_k-1 in order with fp32 fma (the same order as the
// per-head kernel above, so both give identical results). A warp per row
// finally converts the fp32 row to the output dtype.
// With several layers (grid y = layer l, decoder L.W[l]), the rows of
// token b and head h of layer l sit at row (b * G + l) * H + h of q and of
// the outputs (the layers of a token stacked), and M counts the rows of one
// layer; with one layer, row m is m.
template <typename T>
__global__ void __launch_bounds__(256) absorb_shared_kernel(const T* __restrict__ q, int M, int d_k, AbsorbLayers L,
                                                            const float* __restrict__ bK, int d_c, int R,
                                                            int out_dtype, void* q_abs, float* q_abs_scale,
                                                            float* beta) {
  pdl_begin();
  pdl_release();
  const int layer = blockIdx.y;
  const T* __restrict__ W = static_cast<const T*>(L.W[layer]);
  auto grow = [&](int m) -> int64_t {
    return L.G == 1 ? static_cast<int64_t>(m)
                    : (static_cast<int64_t>(m / L.H) * L.G + layer) * L.H + (m % L.H);
  };
  extern __shared__ __align__(16) unsigned char absorb_smem[];
  T* Ws = reinterpret_cast<T*>(absorb_smem);                                   // [d_k][d_c]
  float* qs = reinterpret_cast<float*>(absorb_smem + (static_cast<size_t>(d_k) * d_c * sizeof(T) + 15) / 16 * 16);
  float* os = qs + R * d_k;                                                    // [R][d_c]
  const int r0 = blockIdx.x * R;
  const int nr = min(R, M - r0);
  {
    // every 16-byte piece of the decoder in flight at once (cp.async), the
    // query rows meanwhile through registers
    const int n16 = static_cast<int>(static_cast<size_t>(d_k) * d_c * sizeof(T) / 16);
    const uint4* src = reinterpret_cast<const uint4*>(W);
    const uint32_t dst = static_cast<uint32_t>(__cvta_generic_to_shared(Ws));
    for (int x = threadIdx.x; x < n16; x += blockDim.x) cp_async_16(dst + 16u * x, src + x);
    cp_async_commit();
    const int nq = nr * d_k;
    if (L.G == 1) {
      for (int x = threadIdx.x; x < R * d_k; x += blockDim.x)
        qs[x] = x < nq ? to_f(q[static_cast<int64_t>(r0) * d_k + x]) : 0.f;
    } else {
      for (int x = threadIdx.x; x < R * d_k; x += blockDim.x) {
        const int rr = x / d_k;
        qs[x] = x < nq ? to_f(q[grow(r0 + rr) * d_k + (x - rr * d_k)]) : 0.f;
      }
    }
    cp_async_wait_all();
  }
  __syncthreads();
  const int npairs = d_c >> 1;
  for (int u = threadIdx.x; u < nr * npairs; u += blockDim.x) {
    const int rr = u / npairs, p = u - rr * npairs;
    const float* qr = qs + rr * d_k;
    const T* wc = Ws + 2 * p;
    float a0 = 0.f, a1 = 0.f;
#pragma unroll 8
    for (int j = 0; j < d_k; ++j) {
      const float qv = qr[j];
      const float2 w2 = load2(wc + static_cast<size_t>(j) * d_c);
      a0 = fmaf(w2.x, qv, a0);
      a1 = fmaf(w2.y, qv, a1);
    }
    os[rr * d_c + 2 * p] = a0;
    os[rr * d_c + 2 * p + 1] = a1;
  }
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int rr = warp; rr < nr; rr += blockDim.x >> 5) {
    const int64_t row = grow(r0 + rr);
    const float* orow = os + rr * d_c;
    if (beta) {
      float bsum = 0.f;
      for (int j = lane; j < d_k; j += 32) bsum = fmaf(qs[rr * d_k + j], bK[j], bsum);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) bsum += __shfl_xor_sync(0xffffffffu, bsum, o);
      if (lane == 0) beta[row] = bsum;
    }
    if (out_dtype == LI_F32) {
      for (int i = lane; i < d_c; i += 32) reinterpret_cast<float*>(q_abs)[row * d_c + i] = orow[i];
    } else if (out_dtype == LI_BF16) {
      for (int i = lane; i < d_c; i += 32)
        reinterpret_cast<__nv_bfloat16*>(q_abs)[row * d_c + i] = __float2bfloat16_rn(orow[i]);
    } else {
      float m = 0.f;
      for (int i = lane; i < d_c; i += 32) m = fmaxf(m, fabsf(orow[i]));
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      const float sc = m > 0.f ? __fdiv_rn(m, 448.f) : 1.f;
      for (int i = lane; i < d_c; i += 32)
        reinterpret_cast<uint8_t*>(q_abs)[row * d_c + i] = to_e4m3(__fdiv_rn(orow[i], sc));
      if (lane == 0) q_abs_scale[row] = sc;
    }
  }
}

size_t absorb_shared_smem(int d_k, int d_c, int R, size_t elt) {
  return (static_cast<size_t>(d_k) * d_c * elt + 15) / 16 * 16 + static_cast<size_t>(R) * (d_k + d_c) * 4;
}

// Shared decoder at decode sizes, split by output columns, for fp32 and bf16
// output: CTA (s, g) computes the columns [s kSplitCols, (s + 1) kSplitCols)
// of the U * 4 rows (token, head) of row group g, from its slice of the
// decoder (d_k x kSplitCols) staged in shared memory; thread t takes column
// t % kSplitCols of rows t / kSplitCols + 4 u.  The slice is a weight, not
// a result of the step, so it is requested before the kernel waits for the
// previous one in the stream; only the query rows wait.  Each output
// accumulates j = 0..d_k-1 in order with fp32 fma, as the other absorb
// kernels do (identical results).
constexpr int kSplitCols = 64;   // 4 rows x kSplitCols columns per pass of 256 threads

template <typename T, int U>
__global__ void __launch_bounds__(256) absorb_split_kernel(const T* __restrict__ q, int M, int d_k,
                                                           const T* __restrict__ W, int d_c, int out_dtype,
                                                           void* q_abs) {
  constexpr int kRows = 4 * U;
  const int r0 = blockIdx.y * kRows;
  const int c0 = blockIdx.x * kSplitCols;
  extern __shared__ __align__(16) unsigned char split_smem[];
  T* Ws = reinterpret_cast<T*>(split_smem);                                        // [d_k][kSplitCols]
  float* qs = reinterpret_cast<float*>(split_smem + static_cast<size_t>(d_k) * kSplitCols * sizeof(T));  // [kRows][d_k]
  {
    // the decoder slice, every 16-byte piece in flight at once
    constexpr int kPieces = kSplitCols * static_cast<int>(sizeof(T)) / 16;   // per decoder row
    const uint32_t dst = static_cast<uint32_t>(__cvta_generic_to_shared(Ws));
    for (int x = threadIdx.x; x < d_k * kPieces; x += blockDim.x) {
      const int j = x / kPieces, pc = x - j * kPieces;
      cp_async_16(dst + 16u * x, reinterpret_cast<const uint4*>(W + static_cast<int64_t>(j) * d_c + c0) + pc);
    }
    cp_async_commit();
  }
  pdl_begin();
  pdl_release();
  for (int x = threadIdx.x; x < kRows * d_k; x += blockDim.x) {
    const int rr = x / d_k;
    qs[x] = r0 + rr < M ? to_f(q[static_cast<int64_t>(r0) * d_k + x]) : 0.f;
  }
  cp_async_wait_all();
  __syncthreads();
  const int rs = threadIdx.x / kSplitCols, cc = threadIdx.x - rs * kSplitCols;
  const T* wc = Ws + cc;
  float acc[U];
#pragma unroll
  for (int u = 0; u < U; ++u) acc[u] = 0.f;
#pragma unroll 4
  for (int j = 0; j < d_k; ++j) {
    const float w = to_f(wc[j * kSplitCols]);
#pragma unroll
    for (int u = 0; u < U; ++u) acc[u] = fmaf(w, qs[(rs + 4 * u) * d_k + j], acc[u]);
  }
#pragma unroll
  for (int u = 0; u < U; ++u) {
    const int row = r0 + rs + 4 * u;
    if (row >= M) continue;
    const int64_t o = static_cast<int64_t>(row) * d_c + c0 + cc;
    if (out_dtype == LI_F32) reinterpret_cast<float*>(q_abs)[o] = acc[u];
    else reinterpret_cast<__nv_bfloat16*>(q_abs)[o] = __float2bfloat16_rn(acc[u]);
  }
}

template <typename T>
cudaError_t launch_absorb_split(const T* q, int M, int d_k, const T* W, int d_c, int out_dtype, void* q_abs,
                                int num_sms, cudaStream_t st) {
  // rows a thread takes: enough CTAs to cover about the SMs once, no more
  const int S = d_c / kSplitCols;
  int U = 1;
  while (U < 8 && static_cast<int64_t>((M + 8 * U - 1) / (8 * U)) * S >= num_sms) U *= 2;
  const size_t smem = static_cast<size_t>(d_k) * kSplitCols * sizeof(T) + static_cast<size_t>(4 * U) * d_k * 4;
  const dim3 grid(S, (M + 4 * U - 1) / (4 * U));
  auto go = [&](auto kernel) -> cudaError_t {
    const cudaError_t e = raise_smem_limit(reinterpret_cast<const void*>(kernel), static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    return launch_pdl(kernel, grid, dim3(256), smem, st, 1, q, M, d_k, W, d_c, out_dtype, q_abs);
  };
  switch (U) {
    case 1: return go(absorb_split_kernel<T, 1>);
    case 2: return go(absorb_split_kernel<T, 2>);
    case 4: return go(absorb_split_kernel<T, 4>);
    default: return go(absorb_split_kernel<T, 8>);
  }
}

}  // namespace

int gemv_splits(int d_model, int n_tok) {
  // decode: enough warps that each reads one 256-element slice of a W row
  if (n_tok > 64) return 1;
  for (int sp = kMaxSplits; sp > 1; --sp)
    if (d_model % (8 * sp) == 0 && d_model / sp >= 256 && (d_model / sp) % 256 == 0) return sp;
  for (int sp = kMaxSplits; sp > 1; --sp)
    if (d_model % (8 * sp) == 0 && d_model / sp >= 256) return sp;
  return 1;
}

cudaError_t launch_append_gemv(const void* h, int h_dtype, const void* W, int d_model, int dim, int n_tok,
                               int splits, float* out, cudaStream_t st) {
  const dim3 grid((dim * splits + kGemvWarps - 1) / kGemvWarps, (n_tok + kGemvTok - 1) / kGemvTok);
  if (h_dtype == LI_BF16)
    return launch_pdl(gemv_kernel<__nv_bfloat16>, grid, dim3(kGemvWarps * 32), 0, st, 1,
                      reinterpret_cast<const __nv_bfloat16*>(h), reinterpret_cast<const __nv_bfloat16*>(W), d_model,
                      dim, n_tok, splits, out);
  return launch_pdl(gemv_kernel<float>, grid, dim3(kGemvWarps * 32), 0, st, 1, reinterpret_cast<const float*>(h),
                    reinterpret_cast<const float*>(W), d_model, dim, n_tok, splits, out);
}

int append_fused_splits(int d_model, int dim) {
  // enough (output, split) warp tasks for a wave of 8 warps on every SM, with
  // slices of whole 256-element steps
  if (d_model % 256) return 0;
  const int steps = d_model / 256;
  for (int sp = 1; sp <= steps && sp <= kMaxSplits; ++sp)
    if (steps % sp == 0 && dim * sp >= 148 * kGemvWarps) return sp;
  for (int sp = std::min(steps, kMaxSplits); sp >= 1; --sp)
    if (steps % sp == 0) return sp;
  return 1;
}

// Shared memory of the one-launch append: the hidden-state slices during the
// GEMV, then (last block) the partial sums.
size_t append_fused_smem(int n_tok, int dim, int splits, int d_model, size_t h_elt) {
  const size_t partials = static_cast<size_t>(splits + 1) * n_tok * dim * sizeof(float);
  const size_t slices = static_cast<size_t>(n_tok) * (d_model / splits) * h_elt;
  return partials > slices ? partials : slices;
}

bool append_fusable(int n_tok, int dim, int splits) {
  return splits >= 1 && n_tok <= kGemvTok && dim <= 256 && (splits + 1) * n_tok * dim <= kFuseMaxPartials;
}

template <bool TF>
cudaError_t launch_append_fused_tf(const void* h, int h_dtype, const void* W, int d_model, int dim, int batch, int T,
                                   int splits, float* part, void* data, float* scale, int32_t* lengths, int capacity,
                                   int dtype, int scale_split, const RowTransform& tf, unsigned int* done,
                                   int* status, cudaStream_t st) {
  const int n_tok = batch * T;
  const int grid = splits * ((dim + kAppendWarps - 1) / kAppendWarps);
  const size_t smem = append_fused_smem(n_tok, dim, splits, d_model, h_dtype == LI_BF16 ? 2 : 4);
  cudaError_t e;
  if (h_dtype == LI_BF16) {
    auto k = gemv_append_kernel<__nv_bfloat16, TF>;
    if ((e = raise_smem_limit(reinterpret_cast<const void*>(k), static_cast<int>(smem))) != cudaSuccess) return e;
    return launch_pdl(k, dim3(grid), dim3(kAppendWarps * 32), smem, st, 1, reinterpret_cast<const __nv_bfloat16*>(h),
                      reinterpret_cast<const __nv_bfloat16*>(W), d_model, dim, n_tok, splits, part, batch, T, data,
                      scale, lengths, capacity, dtype, scale_split, tf, done, status);
  } else {
    auto k = gemv_append_kernel<float, TF>;
    if ((e = raise_smem_limit(reinterpret_cast<const void*>(k), static_cast<int>(smem))) != cudaSuccess) return e;
    return launch_pdl(k, dim3(grid), dim3(kAppendWarps * 32), smem, st, 1, reinterpret_cast<const float*>(h),
                      reinterpret_cast<const float*>(W), d_model, dim, n_tok, splits, part, batch, T, data, scale,
                      lengths, capacity, dtype, scale_split, tf, done, status);
  }
}

bool has_transform(const RowTransform& tf) { return tf.rope_dim > 0 || tf.norm_dim > 0; }

cudaError_t launch_append_fused(const void* h, int h_dtype, const void* W, int d_model, int dim, int batch, int T,
                                int splits, float* part, void* data, float* scale, int32_t* lengths, int capacity,
                                int dtype, int scale_split, const RowTransform& tf, unsigned int* done, int* status,
                                cudaStream_t st) {
  return has_transform(tf)
             ? launch_append_fused_tf<true>(h, h_dtype, W, d_model, dim, batch, T, splits, part, data, scale, lengths,
                                            capacity, dtype, scale_split, tf, done, status, st)
             : launch_append_fused_tf<false>(h, h_dtype, W, d_model, dim, batch, T, splits, part, data, scale, lengths,
                                             capacity, dtype, scale_split, tf, done, status, st);
}

cudaError_t launch_append_store(const float* c, int64_t c_tok_stride, int64_t split_stride, int splits, int batch,
                                int T_chunk, int t0, int T_total, bool bump, void* data, float* scale,
                                int32_t* lengths, int capacity, int dim, int dtype, int scale_split,
                                const RowTransform& tf, unsigned int* done_counter, int* status, cudaStream_t st) {
  const int n_tok = batch * T_chunk;
  const int grid = (n_tok + 7) / 8;
  return launch_pdl(has_transform(tf) ? store_kernel<true> : store_kernel<false>, dim3(grid), dim3(256), 0, st, 1, c,
                    c_tok_stride, split_stride, splits, batch, T_chunk, t0, T_total, bump ? 1 : 0, data, scale, lengths,
                    capacity, dim, dtype, scale_split, tf, done_counter, status);
}

static cudaError_t launch_absorb_shared(const void* q, int q_dtype, int M, int d_k, const AbsorbLayers& L, int layers,
                                 const float* b, int d_c, int R, size_t smem, int out_dtype, void* q_abs,
                                 float* q_abs_scale, float* beta, cudaStream_t st) {
  const dim3 grid((M + R - 1) / R, layers);
  cudaError_t e;
  if (q_dtype == LI_BF16) {
    auto k = absorb_shared_kernel<__nv_bfloat16>;
    e = raise_smem_limit(reinterpret_cast<const void*>(k), static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    return launch_pdl(k, grid, dim3(256), smem, st, 1, reinterpret_cast<const __nv_bfloat16*>(q), M, d_k, L, b, d_c,
                      R, out_dtype, q_abs, q_abs_scale, beta);
  }
  auto k = absorb_shared_kernel<float>;
  e = raise_smem_limit(reinterpret_cast<const void*>(k), static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  return launch_pdl(k, grid, dim3(256), smem, st, 1, reinterpret_cast<const float*>(q), M, d_k, L, b, d_c, R,
                    out_dtype, q_abs, q_abs_scale, beta);
}

cudaError_t launch_absorb_group(const void* q, int q_dtype, int batch, int G, int H, int d_k, const void* const* W,
                                int d_c, int out_dtype, void* q_abs, float* q_abs_scale, cudaStream_t st) {
  const size_t elt = q_dtype == LI_BF16 ? 2 : 4;
  const int M = batch * H;                       // rows of one layer
  const int R = M <= 4096 ? 2 : 32;
  const size_t smem = absorb_shared_smem(d_k, d_c, R, elt);
  if (G < 1 || G > kMaxAbsorbLayers || (d_c & 1) || smem > 200 * 1024 || (static_cast<size_t>(d_k) * d_c * elt) % 16)
    return cudaErrorInvalidValue;
  AbsorbLayers L{};
  for (int l = 0; l < G; ++l) {
    if (!W[l] || (reinterpret_cast<uintptr_t>(W[l]) & 15)) return cudaErrorInvalidValue;
    L.W[l] = W[l];
  }
  L.G = G;
  L.H = H;
  return launch_absorb_shared(q, q_dtype, M, d_k, L, G, nullptr, d_c, R, smem, out_dtype, q_abs, q_abs_scale,
                              nullptr, st);
}

cudaError_t launch_absorb(const void* q, int q_dtype, int n_tok, int H, int d_k, const void* W,
                          int64_t W_head_stride, const float* b, int64_t b_head_stride, int d_c,
                          int out_dtype, void* q_abs, float* q_abs_scale, float* beta, int num_sms,
                          cudaStream_t st) {
  const size_t elt = q_dtype == LI_BF16 ? 2 : 4;
  const int M = n_tok * H;
  // shared decoder: rows of R (token, head) pairs; two rows per block at
  // decode sizes (more blocks stage the decoder in parallel: 5.4 -> 4.0 us
  // at 4 x 64 heads against 4 rows), more when there are many queries
  const int R = M <= 4096 ? 2 : 32;
  const size_t smem = absorb_shared_smem(d_k, d_c, R, elt);
  const bool aligned = (reinterpret_cast<uintptr_t>(W) & 15) == 0 && (static_cast<size_t>(d_k) * d_c * elt) % 16 == 0;
  if (W != nullptr && W_head_stride == 0 && b == nullptr && beta == nullptr && M <= 4096 && aligned &&
      d_c % kSplitCols == 0 && out_dtype != LI_E4M3) {
    // decode, fp32 or bf16 output: the column-split kernel (its decoder
    // slices stage before the wait).  E4M3 output needs each row's amax over
    // all columns and stays with the whole-row kernel below.
    if (q_dtype == LI_BF16)
      return launch_absorb_split(reinterpret_cast<const __nv_bfloat16*>(q), M, d_k,
                                 reinterpret_cast<const __nv_bfloat16*>(W), d_c, out_dtype, q_abs, num_sms, st);
    return launch_absorb_split(reinterpret_cast<const float*>(q), M, d_k, reinterpret_cast<const float*>(W), d_c,
                               out_dtype, q_abs, num_sms, st);
  }
  if (W != nullptr && W_head_stride == 0 && b_head_stride == 0 && (d_c & 1) == 0 && aligned &&
      smem <= 200 * 1024) {
    AbsorbLayers L{};
    L.W[0] = W;
    L.G = 1;
    L.H = H;
    return launch_absorb_shared(q, q_dtype, M, d_k, L, 1, b, d_c, R, smem, out_dtype, q_abs, q_abs_scale, beta, st);
  }
  const dim3 grid((H + kAbsorbHeads - 1) / kAbsorbHeads, n_tok);
  if (q_dtype == LI_BF16)
    return launch_pdl(absorb_kernel<__nv_bfloat16>, grid, dim3(256), 0, st, 1,
                      reinterpret_cast<const __nv_bfloat16*>(q), H, d_k, reinterpret_cast<const __nv_bfloat16*>(W),
                      W_head_stride, b, b_head_stride, d_c, out_dtype, q_abs, q_abs_scale, beta);
  return launch_pdl(absorb_kernel<float>, grid, dim3(256), 0, st, 1, reinterpret_cast<const float*>(q), H, d_k,
                    reinterpret_cast<const float*>(W), W_head_stride, b, b_head_stride, d_c, out_dtype, q_abs,
                    q_abs_scale, beta);
}

}  // namespace li
