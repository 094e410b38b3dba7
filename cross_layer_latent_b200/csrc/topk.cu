// topk.cu -- exact per-row top-k selection by radix select (LatentIndex
// summary, Sec. 3.1 / Sec. 4.1: every layer keeps its own top-k tokens, up to
// 2048 per query; Sec. C.4: budgets are capped by the valid prefix length).
//
// Selection rule: the k_eff = min(k, n) positions with the largest scores,
// ties broken toward the lower position, written in ascending position order
// and padded with -1.  Scores are compared through an order-preserving uint32
// key (-0.0 == +0.0).  With T the k_eff-th largest key and idx_T the
// position of the last tied element that still fits, position i is selected
// iff key_i > T or (key_i == T and i <= idx_T); this predicate is local, so
// the ordered output is written by independent chunks.
//
// Stages (one stream, in order):
//   0 hist   : per-row histogram of the key's top 11 bits (fused into the
//              scoring kernel when the scores come from it)
//   1 filter : finds the boundary bucket b1, counts per chunk the elements in
//              higher buckets and appends the boundary bucket's (key, pos)
//              pairs to a per-row candidate list
//   2 select : one CTA per row resolves the remaining 21 key bits on the
//              candidates (two more radix digits), the tie cut idx_T, and
//              each chunk's output offset
//   3 emit   : each chunk writes its selected positions in order
#include <climits>

#include "internal.h"
#include "sm100.cuh"

namespace li {

namespace {

enum { kInfoKeff = 0, kInfoB1, kInfoAbove1, kInfoT, kInfoIdxT, kInfoCandCount };

__device__ __forceinline__ int row_len(const TopkArgs& a, int r) {
  int n = a.n;
  if (a.lengths) {
    const int v = a.lengths[r / a.len_div];
    n = min(n, max(v, 0));
  }
  if (a.q_pos) {
    const int v = a.q_pos[r] + 1;
    n = min(n, max(v, 0));
  }
  return n;
}

// Exclusive prefix sum over the block (blockDim.x a multiple of 32, <= 1024).
__device__ __forceinline__ int block_excl_scan(int v, int* scratch, int* total) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = blockDim.x >> 5;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int u = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += u;
  }
  if (lane == 31) scratch[wid] = incl;
  __syncthreads();
  if (wid == 0) {
    int s = lane < nw ? scratch[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int u = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += u;
    }
    scratch[lane] = s;
  }
  __syncthreads();
  const int res = (wid > 0 ? scratch[wid - 1] : 0) + incl - v;
  if (total) *total = scratch[nw - 1];
  __syncthreads();
  return res;
}

// Find the bucket holding the need-th element counted from the top (largest
// bin first) of a histogram h[nbins] in shared memory; *above = elements in
// higher bins.  nbins must be a multiple of blockDim.x.  Result in out[0..1].
__device__ void find_bucket_desc(const unsigned* h, int nbins, int need, int* scratch, int* out) {
  const int per = nbins / blockDim.x;
  const int hi = nbins - threadIdx.x * per;          // this thread covers [hi - per, hi)
  int sum = 0;
  for (int i = 1; i <= per; ++i) sum += h[hi - i];
  if (threadIdx.x == 0) { out[0] = 0; out[1] = 0; }
  const int before = block_excl_scan(sum, scratch, nullptr);
  if (before < need && need <= before + sum) {
    int cum = before;
    for (int i = 1; i <= per; ++i) {
      const int bin = hi - i;
      if (cum + static_cast<int>(h[bin]) >= need) { out[0] = bin; out[1] = cum; break; }
      cum += h[bin];
    }
  }
  __syncthreads();
}

// Same from the bottom (smallest bin first); *below = elements in lower bins.
__device__ void find_bucket_asc(const unsigned* h, int nbins, int need, int* scratch, int* out) {
  const int per = nbins / blockDim.x;
  const int lo = threadIdx.x * per;
  int sum = 0;
  for (int i = 0; i < per; ++i) sum += h[lo + i];
  if (threadIdx.x == 0) { out[0] = 0; out[1] = 0; }
  const int before = block_excl_scan(sum, scratch, nullptr);
  if (before < need && need <= before + sum) {
    int cum = before;
    for (int i = 0; i < per; ++i) {
      const int bin = lo + i;
      if (cum + static_cast<int>(h[bin]) >= need) { out[0] = bin; out[1] = cum; break; }
      cum += h[bin];
    }
  }
  __syncthreads();
}

__global__ void __launch_bounds__(kTopkThreads) topk_hist_kernel(const TopkArgs a) {
  __shared__ unsigned h[kHistBins];
  const int r = blockIdx.y, c = blockIdx.x;
  const int n = row_len(a, r);
  const int lo = c * kTopkChunk;
  if (lo >= n) return;
  const int hi = min(n, lo + kTopkChunk);
  for (int i = threadIdx.x; i < kHistBins; i += blockDim.x) h[i] = 0;
  __syncthreads();
  const float* row = a.scores + static_cast<int64_t>(r) * a.row_stride;
  for (int i = lo + threadIdx.x; i < hi; i += blockDim.x) atomicAdd(&h[radix_key(row[i]) >> 21], 1u);
  __syncthreads();
  for (int i = threadIdx.x; i < kHistBins; i += blockDim.x)
    if (h[i]) atomicAdd(&a.hist[static_cast<int64_t>(r) * kHistBins + i], h[i]);
}

__global__ void __launch_bounds__(kTopkThreads) topk_filter_kernel(const TopkArgs a) {
  __shared__ unsigned h[kHistBins];
  __shared__ int scratch[32];
  __shared__ int res[2];
  __shared__ int gt_sum;
  const int r = blockIdx.y, c = blockIdx.x;
  const int n = row_len(a, r);
  const int keff = min(a.k, n);
  int* info = a.rowinfo + static_cast<int64_t>(r) * 16;
  int* cgt = a.chunk_gt + static_cast<int64_t>(r) * a.n_chunks;
  if (keff <= 0) {
    if (threadIdx.x == 0) {
      cgt[c] = 0;
      if (c == 0) info[kInfoKeff] = 0;
    }
    return;
  }
  for (int i = threadIdx.x; i < kHistBins; i += blockDim.x) h[i] = a.hist[static_cast<int64_t>(r) * kHistBins + i];
  if (threadIdx.x == 0) gt_sum = 0;
  __syncthreads();
  find_bucket_desc(h, kHistBins, keff, scratch, res);
  const unsigned b1 = static_cast<unsigned>(res[0]);
  const int lo = c * kTopkChunk;
  const int hi = min(n, lo + kTopkChunk);
  const float* row = a.scores + static_cast<int64_t>(r) * a.row_stride;
  uint2* cand = a.cand + static_cast<int64_t>(r) * a.n;
  int gt = 0;
  const int lane = threadIdx.x & 31;
  for (int base = lo; base < hi; base += blockDim.x) {
    const int i = base + threadIdx.x;
    unsigned key = 0;
    bool is_cand = false;
    if (i < hi) {
      key = radix_key(row[i]);
      const unsigned d = key >> 21;
      gt += d > b1 ? 1 : 0;
      is_cand = d == b1;
    }
    const unsigned m = __ballot_sync(0xffffffffu, is_cand);
    if (m) {
      int slot = 0;
      if (lane == 0) slot = atomicAdd(&info[kInfoCandCount], __popc(m));
      slot = __shfl_sync(0xffffffffu, slot, 0);
      if (is_cand) cand[slot + __popc(m & ((1u << lane) - 1u))] = make_uint2(key, static_cast<unsigned>(i));
    }
  }
  for (int o = 16; o > 0; o >>= 1) gt += __shfl_xor_sync(0xffffffffu, gt, o);
  if (lane == 0 && gt) atomicAdd(&gt_sum, gt);
  __syncthreads();
  if (threadIdx.x == 0) {
    cgt[c] = lo < n ? gt_sum : 0;
    if (c == 0) {
      info[kInfoKeff] = keff;
      info[kInfoB1] = res[0];
      info[kInfoAbove1] = res[1];
    }
  }
}

constexpr int kSelectThreads = 1024;

__global__ void __launch_bounds__(kSelectThreads) topk_select_kernel(const TopkArgs a) {
  __shared__ unsigned h[kHistBins];
  __shared__ int scratch[32];
  __shared__ int res[2];
  __shared__ int cc[kMaxTopkChunks];
  const int r = blockIdx.x;
  int* info = a.rowinfo + static_cast<int64_t>(r) * 16;
  const int keff = info[kInfoKeff];
  int32_t* oidx = a.out_idx + static_cast<int64_t>(r) * a.k;
  float* oscore = a.out_score ? a.out_score + static_cast<int64_t>(r) * a.k : nullptr;
  for (int j = max(keff, 0) + threadIdx.x; j < a.k; j += blockDim.x) {
    oidx[j] = -1;
    if (oscore) oscore[j] = -INFINITY;
  }
  if (a.out_count && threadIdx.x == 0) a.out_count[r] = max(keff, 0);
  if (keff <= 0) return;
  const unsigned b1 = static_cast<unsigned>(info[kInfoB1]);
  const int above1 = info[kInfoAbove1];
  const int nc = info[kInfoCandCount];
  const uint2* cand = a.cand + static_cast<int64_t>(r) * a.n;
  const int need = keff - above1;

  // digit 2: key bits 20..10
  for (int i = threadIdx.x; i < kHistBins; i += blockDim.x) h[i] = 0;
  __syncthreads();
  for (int i = threadIdx.x; i < nc; i += blockDim.x) atomicAdd(&h[(cand[i].x >> 10) & 2047u], 1u);
  __syncthreads();
  find_bucket_desc(h, kHistBins, need, scratch, res);
  const unsigned b2 = static_cast<unsigned>(res[0]);
  const int need2 = need - res[1];
  // digit 3: key bits 9..0
  for (int i = threadIdx.x; i < kHistBins; i += blockDim.x) h[i] = 0;
  __syncthreads();
  for (int i = threadIdx.x; i < nc; i += blockDim.x) {
    const unsigned key = cand[i].x;
    if (((key >> 10) & 2047u) == b2) atomicAdd(&h[key & 1023u], 1u);
  }
  __syncthreads();
  find_bucket_desc(h, 1024, need2, scratch, res);
  const unsigned b3 = static_cast<unsigned>(res[0]);
  const int need3 = need2 - res[1];
  const int eq_count = static_cast<int>(h[b3]);
  __syncthreads();
  const unsigned T = (b1 << 21) | (b2 << 10) | b3;

  // Tie cut: the need3-th smallest position among the elements equal to T
  // (positions < 2^31; digits of bits 30..20, 19..10 and 9..0).
  int idx_T = INT_MAX;
  if (need3 < eq_count) {
    int needp = need3;
    unsigned d0 = 0, d1 = 0, d2 = 0;
    for (int pass = 0; pass < 3; ++pass) {
      for (int i = threadIdx.x; i < kHistBins; i += blockDim.x) h[i] = 0;
      __syncthreads();
      for (int i = threadIdx.x; i < nc; i += blockDim.x) {
        const uint2 e = cand[i];
        if (e.x != T) continue;
        const unsigned p = e.y;
        if (pass == 0) atomicAdd(&h[p >> 20], 1u);
        else if (pass == 1) { if ((p >> 20) == d0) atomicAdd(&h[(p >> 10) & 1023u], 1u); }
        else if ((p >> 10) == ((d0 << 10) | d1)) atomicAdd(&h[p & 1023u], 1u);
      }
      __syncthreads();
      find_bucket_asc(h, pass == 0 ? kHistBins : 1024, needp, scratch, res);
      const unsigned d = static_cast<unsigned>(res[0]);
      needp -= res[1];
      if (pass == 0) d0 = d; else if (pass == 1) d1 = d; else d2 = d;
      __syncthreads();
    }
    idx_T = static_cast<int>((d0 << 20) | (d1 << 10) | d2);
  }

  // Output offset of every chunk: elements of higher buckets (counted by the
  // filter) plus the selected candidates that fall in the chunk.
  const int nchunks = a.n_chunks;
  for (int i = threadIdx.x; i < nchunks; i += blockDim.x) cc[i] = 0;
  __syncthreads();
  for (int i = threadIdx.x; i < nc; i += blockDim.x) {
    const uint2 e = cand[i];
    if (e.x > T || (e.x == T && static_cast<int>(e.y) <= idx_T)) atomicAdd(&cc[e.y / kTopkChunk], 1);
  }
  __syncthreads();
  const int* cgt = a.chunk_gt + static_cast<int64_t>(r) * nchunks;
  int* coff = a.chunk_off + static_cast<int64_t>(r) * nchunks;
  const int per = (nchunks + blockDim.x - 1) / blockDim.x;
  const int c0 = threadIdx.x * per;
  int local = 0;
  for (int i = 0; i < per; ++i)
    if (c0 + i < nchunks) local += cc[c0 + i] + cgt[c0 + i];
  int run = block_excl_scan(local, scratch, nullptr);
  for (int i = 0; i < per; ++i) {
    if (c0 + i < nchunks) {
      coff[c0 + i] = run;
      run += cc[c0 + i] + cgt[c0 + i];
    }
  }
  if (threadIdx.x == 0) {
    info[kInfoT] = static_cast<int>(T);
    info[kInfoIdxT] = idx_T;
  }
}

constexpr int kEmitPerThread = kTopkChunk / kTopkThreads;   // 16

__global__ void __launch_bounds__(kTopkThreads) topk_emit_kernel(const TopkArgs a) {
  __shared__ int scratch[32];
  const int r = blockIdx.y, c = blockIdx.x;
  const int* info = a.rowinfo + static_cast<int64_t>(r) * 16;
  const int keff = info[kInfoKeff];
  if (keff <= 0) return;
  const int n = row_len(a, r);
  const int lo = c * kTopkChunk;
  if (lo >= n) return;
  const int hi = min(n, lo + kTopkChunk);
  const unsigned T = static_cast<unsigned>(info[kInfoT]);
  const int idx_T = info[kInfoIdxT];
  const int off = a.chunk_off[static_cast<int64_t>(r) * a.n_chunks + c];
  const float* row = a.scores + static_cast<int64_t>(r) * a.row_stride;
  const int i0 = lo + threadIdx.x * kEmitPerThread;
  float v[kEmitPerThread];
  unsigned sel = 0;
#pragma unroll
  for (int e = 0; e < kEmitPerThread; ++e) {
    const int i = i0 + e;
    v[e] = i < hi ? row[i] : 0.f;
    if (i < hi) {
      const unsigned key = radix_key(v[e]);
      if (key > T || (key == T && i <= idx_T)) sel |= 1u << e;
    }
  }
  int pos = off + block_excl_scan(__popc(sel), scratch, nullptr);
  int32_t* oidx = a.out_idx + static_cast<int64_t>(r) * a.k;
  float* oscore = a.out_score ? a.out_score + static_cast<int64_t>(r) * a.k : nullptr;
  const int* map = a.idx_map ? a.idx_map + static_cast<int64_t>(r) * a.map_stride : nullptr;
#pragma unroll
  for (int e = 0; e < kEmitPerThread; ++e) {
    if (sel & (1u << e)) {
      if (pos < a.k) {
        const int i = i0 + e;
        oidx[pos] = map ? map[i] : i;
        if (oscore) oscore[pos] = v[e];
      }
      ++pos;
    }
  }
}

}  // namespace

cudaError_t launch_topk_stage(int stage, const TopkArgs& a, cudaStream_t st) {
  const dim3 grid_chunks(a.n_chunks, a.rows);
  switch (stage) {
    case 0: topk_hist_kernel<<<grid_chunks, kTopkThreads, 0, st>>>(a); break;
    case 1: topk_filter_kernel<<<grid_chunks, kTopkThreads, 0, st>>>(a); break;
    case 2: topk_select_kernel<<<a.rows, kSelectThreads, 0, st>>>(a); break;
    case 3: topk_emit_kernel<<<grid_chunks, kTopkThreads, 0, st>>>(a); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace li
