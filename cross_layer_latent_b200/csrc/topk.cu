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

// ============================================================================
// Single-launch cluster selection.
//
// One thread-block cluster (CS <= 8 CTAs of 512 threads) per row; CTA c owns
// positions [c*E, (c+1)*E), E = 512 * PT, as register-resident keys (warp w
// holds a contiguous run of 32*PT positions, lane l position j*32 + l).  Four
// cluster barriers:
//   1. first-digit (top 11 bits) histograms are complete; every CTA sums the
//      cluster's histograms through distributed shared memory and finds the
//      boundary bucket b1 of each budget;
//   2. each CTA has compacted the keys of its elements in the boundary
//      bucket(s) to its own region of the workspace; every CTA then resolves
//      the two remaining digits (11 + 10 bits) over all of them, redundantly,
//      giving the exact k-th key T and how many elements equal to T are taken;
//   3. per-CTA counts of (key > T, key == T) are published; an element's
//      output rank is #greater before it + min(#equal before it, taken);
//   4. no CTA leaves while another may still read its counts.
// Up to two budgets (k and k2 <= k) are selected from the same keys.
// ============================================================================
#include <cooperative_groups.h>

namespace li {
namespace {

namespace cg = cooperative_groups;

struct SelState {
  int keff;          // min(k, n)
  unsigned b1;       // boundary bucket of the first digit
  int above1;        // elements in higher first-digit buckets
  unsigned T;        // exact key of the keff-th element
  int n_gt;          // elements with key > T
  int need_eq;       // elements equal to T that are taken (lowest positions first)
};

constexpr int kCandCap = 16384;   // boundary-bucket keys a CTA stages in shared memory

// Find the boundary bucket of `need` counting from the top in a 2048-bin
// histogram whose per-thread bins are held in loc[0..3] (bins hi-1..hi-4).
__device__ __forceinline__ void find_from_loc(const unsigned (&loc)[4], int hi, int need, int* scratch,
                                              int* out) {
  const int sum = static_cast<int>(loc[0] + loc[1] + loc[2] + loc[3]);
  if (threadIdx.x == 0) { out[0] = 0; out[1] = 0; }
  const int before = block_excl_scan(sum, scratch, nullptr);
  if (before < need && need <= before + sum) {
    int cum = before;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      if (cum + static_cast<int>(loc[i]) >= need) { out[0] = hi - 1 - i; out[1] = cum; break; }
      cum += static_cast<int>(loc[i]);
    }
  }
  __syncthreads();
}

// Remaining two digits over `m` candidate keys (shared memory).
__device__ __forceinline__ void resolve_low_digits(SelState& st, const unsigned* cand, int m, unsigned* hist,
                                                   int* scratch, int* res) {
  int need = st.keff - st.above1;
  unsigned prefix2 = 0;
#pragma unroll
  for (int d = 0; d < 2; ++d) {
    const int nb = d == 0 ? 2048 : 1024;
    for (int i = threadIdx.x; i < nb; i += blockDim.x) hist[i] = 0;
    __syncthreads();
    for (int i = threadIdx.x; i < m; i += blockDim.x) {
      const unsigned key = cand[i];
      if (d == 0) atomicAdd(&hist[(key >> 10) & 2047u], 1u);
      else if (((key >> 10) & 2047u) == prefix2) atomicAdd(&hist[key & 1023u], 1u);
    }
    __syncthreads();
    find_bucket_desc(hist, nb, need, scratch, res);
    const unsigned bin = static_cast<unsigned>(res[0]);
    const int above = res[1];
    __syncthreads();
    need -= above;
    st.n_gt += above;
    if (d == 0) prefix2 = bin;
    else st.T = (st.b1 << 21) | (prefix2 << 10) | bin;
  }
  st.need_eq = need;
}

// Thread t of CTA c owns positions [c*E + t*PT, +PT), E = 512 * PT, as
// register keys; NSEL budgets (k, and k2 <= k) are selected from them.
template <int PT, int NSEL>
__global__ void __launch_bounds__(kClusterThreads, 1) topk_cluster_kernel(const TopkArgs a, const TopkOut2 o2) {
  extern __shared__ __align__(16) unsigned cand_smem[];   // kCandCap keys
  __shared__ __align__(16) unsigned hist[kHistBins];
  __shared__ int scratch[32];
  __shared__ int res[2];
  __shared__ int cnt_local[2];                  // candidates of this CTA per bucket
  __shared__ int ctot[2 * NSEL];                // (gt, eq) per budget of this CTA
  cg::cluster_group cluster = cg::this_cluster();
  const int CS = static_cast<int>(cluster.num_blocks());
  const int c = static_cast<int>(cluster.block_rank());
  const int r = blockIdx.y;
  const int n = row_len(a, r);
  SelState sel[NSEL];
  sel[0].keff = min(a.k, n);
  if (NSEL == 2) sel[NSEL - 1].keff = min(o2.k2, n);
  if (c == 0) {
#pragma unroll
    for (int si = 0; si < NSEL; ++si) {
      const int kk = si == 0 ? a.k : o2.k2;
      int32_t* oi = (si == 0 ? a.out_idx : o2.out_idx2) + static_cast<int64_t>(r) * kk;
      float* osv = si == 0 ? a.out_score : o2.out_score2;
      for (int j = max(sel[si].keff, 0) + threadIdx.x; j < kk; j += blockDim.x) {
        oi[j] = -1;
        if (osv) osv[static_cast<int64_t>(r) * kk + j] = -INFINITY;
      }
    }
    if (a.out_count && threadIdx.x == 0) a.out_count[r] = max(sel[0].keff, 0);
  }
  if (sel[0].keff <= 0) return;   // uniform over the cluster (depends on the row only)

  const int64_t E = static_cast<int64_t>(kClusterThreads) * PT;
  const int64_t p0 = static_cast<int64_t>(c) * E + static_cast<int64_t>(threadIdx.x) * PT;
  const float* row = a.scores + static_cast<int64_t>(r) * a.row_stride;
  unsigned key[PT];
  unsigned vmask = 0;
  if ((a.row_stride & 3) == 0 && (reinterpret_cast<uintptr_t>(a.scores) & 15) == 0 && p0 + PT <= n) {
#pragma unroll
    for (int j = 0; j < PT; j += 4) {
      const float4 f = *reinterpret_cast<const float4*>(row + p0 + j);
      key[j] = radix_key(f.x);
      key[j + 1] = radix_key(f.y);
      key[j + 2] = radix_key(f.z);
      key[j + 3] = radix_key(f.w);
    }
    vmask = PT == 32 ? 0xffffffffu : ((1u << PT) - 1u);
  } else {
#pragma unroll
    for (int j = 0; j < PT; ++j) {
      key[j] = 0;
      if (p0 + j < n) {
        key[j] = radix_key(row[p0 + j]);
        vmask |= 1u << j;
      }
    }
  }

  // ---- 1. first digit: histograms summed over the cluster
  for (int i = threadIdx.x; i < kHistBins; i += blockDim.x) hist[i] = 0;
  __syncthreads();
#pragma unroll
  for (int j = 0; j < PT; ++j)
    if ((vmask >> j) & 1u) atomicAdd(&hist[key[j] >> 21], 1u);
  cluster.sync();
  const int hi = kHistBins - static_cast<int>(threadIdx.x) * 4;
  unsigned loc[4] = {0, 0, 0, 0};
  {
    uint4 parts[kClusterMaxSize];
#pragma unroll
    for (int rk = 0; rk < kClusterMaxSize; ++rk)
      if (rk < CS) parts[rk] = *reinterpret_cast<const uint4*>(cluster.map_shared_rank(hist, rk) + hi - 4);
#pragma unroll
    for (int rk = 0; rk < kClusterMaxSize; ++rk)
      if (rk < CS) { loc[3] += parts[rk].x; loc[2] += parts[rk].y; loc[1] += parts[rk].z; loc[0] += parts[rk].w; }
  }
#pragma unroll
  for (int si = 0; si < NSEL; ++si) {
    find_from_loc(loc, hi, sel[si].keff, scratch, res);
    sel[si].b1 = static_cast<unsigned>(res[0]);
    sel[si].above1 = res[1];
    sel[si].n_gt = res[1];
    __syncthreads();
  }

  // ---- 2. this CTA's boundary-bucket keys -> its workspace region
  //         (bucket of budget 0, then budget 1's if it differs)
  const bool two = NSEL == 2 && sel[NSEL - 1].b1 != sel[0].b1;
  unsigned* rowcand = reinterpret_cast<unsigned*>(a.cand) + static_cast<int64_t>(r) * a.n;
  {
    int m0 = 0, m1 = 0;
#pragma unroll
    for (int j = 0; j < PT; ++j) {
      const bool v = (vmask >> j) & 1u;
      const unsigned d = key[j] >> 21;
      m0 += (v && d == sel[0].b1) ? 1 : 0;
      m1 += (v && two && d == sel[NSEL - 1].b1) ? 1 : 0;
    }
    int tot = 0;
    const int off = block_excl_scan(m0 | (m1 << 16), scratch, &tot);   // both counts < 2^15
    int o0 = off & 0xFFFF, o1 = (off >> 16) + (tot & 0xFFFF);
    unsigned* region = rowcand + static_cast<int64_t>(c) * E;
#pragma unroll
    for (int j = 0; j < PT; ++j) {
      const bool v = (vmask >> j) & 1u;
      const unsigned d = key[j] >> 21;
      if (v && d == sel[0].b1) region[o0++] = key[j];
      else if (v && two && d == sel[NSEL - 1].b1) region[o1++] = key[j];
    }
    if (threadIdx.x == 0) { cnt_local[0] = tot & 0xFFFF; cnt_local[1] = tot >> 16; }
  }
  cluster.sync();
  // stage every CTA's keys of one bucket in shared memory, resolve the two
  // remaining digits there (each CTA redundantly: no broadcast needed)
#pragma unroll
  for (int si = 0; si < NSEL; ++si) {
    const int bk = (si == 1 && two) ? 1 : 0;
    int m = 0;
    for (int rk = 0; rk < CS; ++rk) {
      const int* rc = cluster.map_shared_rank(cnt_local, rk);
      const int cnt = rc[bk];
      const unsigned* src = rowcand + static_cast<int64_t>(rk) * E + (bk ? rc[0] : 0);
      for (int i = threadIdx.x; i < cnt; i += blockDim.x)
        if (m + i < kCandCap) cand_smem[m + i] = src[i];
      m += cnt;
    }
    __syncthreads();
    if (m <= kCandCap) {
      resolve_low_digits(sel[si], cand_smem, m, hist, scratch, res);
    } else {
      // more boundary keys than shared memory holds (heavy ties): resolve from
      // the workspace copies, one CTA region after the other
      int need = sel[si].keff - sel[si].above1;
      unsigned prefix2 = 0;
#pragma unroll 1
      for (int d = 0; d < 2; ++d) {
        const int nb = d == 0 ? 2048 : 1024;
        for (int i = threadIdx.x; i < nb; i += blockDim.x) hist[i] = 0;
        __syncthreads();
        for (int rk = 0; rk < CS; ++rk) {
          const int* rc = cluster.map_shared_rank(cnt_local, rk);
          const int cnt = rc[bk];
          const unsigned* src = rowcand + static_cast<int64_t>(rk) * E + (bk ? rc[0] : 0);
          for (int i = threadIdx.x; i < cnt; i += blockDim.x) {
            const unsigned kq = src[i];
            if (d == 0) atomicAdd(&hist[(kq >> 10) & 2047u], 1u);
            else if (((kq >> 10) & 2047u) == prefix2) atomicAdd(&hist[kq & 1023u], 1u);
          }
        }
        __syncthreads();
        find_bucket_desc(hist, nb, need, scratch, res);
        const unsigned bin = static_cast<unsigned>(res[0]);
        const int above = res[1];
        __syncthreads();
        need -= above;
        sel[si].n_gt += above;
        if (d == 0) prefix2 = bin;
        else sel[si].T = (sel[si].b1 << 21) | (prefix2 << 10) | bin;
      }
      sel[si].need_eq = need;
    }
    __syncthreads();
  }

  // ---- 3. ordered output: rank = #greater before + min(#equal before, need_eq)
  int off_gt[NSEL], off_eq[NSEL];
#pragma unroll
  for (int si = 0; si < NSEL; ++si) {
    int g = 0, e = 0;
#pragma unroll
    for (int j = 0; j < PT; ++j) {
      const bool v = (vmask >> j) & 1u;
      g += (v && key[j] > sel[si].T) ? 1 : 0;
      e += (v && key[j] == sel[si].T) ? 1 : 0;
    }
    int tot = 0;
    const int off = block_excl_scan(g | (e << 16), scratch, &tot);
    off_gt[si] = off & 0xFFFF;
    off_eq[si] = off >> 16;
    if (threadIdx.x == 0) { ctot[2 * si] = tot & 0xFFFF; ctot[2 * si + 1] = tot >> 16; }
  }
  cluster.sync();
  for (int rk = 0; rk < c; ++rk) {
    const int* rt = cluster.map_shared_rank(ctot, rk);
#pragma unroll
    for (int si = 0; si < NSEL; ++si) { off_gt[si] += rt[2 * si]; off_eq[si] += rt[2 * si + 1]; }
  }
  const int* map = a.idx_map ? a.idx_map + static_cast<int64_t>(r) * a.map_stride : nullptr;
#pragma unroll
  for (int si = 0; si < NSEL; ++si) {
    const int kk = si == 0 ? a.k : o2.k2;
    int32_t* oi = (si == 0 ? a.out_idx : o2.out_idx2) + static_cast<int64_t>(r) * kk;
    float* osv = si == 0 ? a.out_score : o2.out_score2;
    if (osv) osv += static_cast<int64_t>(r) * kk;
    int gb = off_gt[si], eb = off_eq[si];
    const unsigned T = sel[si].T;
    const int need_eq = sel[si].need_eq;
#pragma unroll
    for (int j = 0; j < PT; ++j) {
      const bool v = (vmask >> j) & 1u;
      const bool gt = v && key[j] > T;
      const bool eq = v && key[j] == T;
      if (gt || (eq && eb < need_eq)) {
        const int rank = gb + min(eb, need_eq);
        if (rank < kk) {
          const int64_t pos = p0 + j;
          oi[rank] = map ? map[pos] : static_cast<int32_t>(pos);
          if (osv) osv[rank] = row[pos];
        }
      }
      gb += gt ? 1 : 0;
      eb += eq ? 1 : 0;
    }
  }
  cluster.sync();   // the counts of this CTA may be read until everyone is past here
}

template <int PT, int NSEL>
cudaError_t launch_cluster_pt(const TopkArgs& a, const TopkOut2& o2, int cs, cudaStream_t st) {
  auto k = topk_cluster_kernel<PT, NSEL>;
  const int dyn = kCandCap * 4;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, dyn);
  if (e != cudaSuccess) {
    (void)cudaGetLastError();
    return e;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(cs, a.rows, 1);
  cfg.blockDim = dim3(kClusterThreads, 1, 1);
  cfg.dynamicSmemBytes = dyn;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = cs;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, k, a, o2);
}

template <int PT>
cudaError_t launch_cluster_sel(const TopkArgs& a, const TopkOut2& o2, int cs, cudaStream_t st) {
  return o2.k2 > 0 ? launch_cluster_pt<PT, 2>(a, o2, cs, st) : launch_cluster_pt<PT, 1>(a, o2, cs, st);
}

}  // namespace

cudaError_t launch_topk_cluster(const TopkArgs& a, const TopkOut2& o2, cudaStream_t st, int* cluster_size) {
  const int64_t n = a.n;
  int cs = static_cast<int>((n + kClusterThreads * 16 - 1) / (kClusterThreads * 16));
  cs = cs < 1 ? 1 : (cs > kClusterMaxSize ? kClusterMaxSize : cs);
  const int64_t per_thread = (n + static_cast<int64_t>(cs) * kClusterThreads - 1) / (static_cast<int64_t>(cs) * kClusterThreads);
  if (cluster_size) *cluster_size = cs;
  if (per_thread <= 4) return launch_cluster_sel<4>(a, o2, cs, st);
  if (per_thread <= 8) return launch_cluster_sel<8>(a, o2, cs, st);
  if (per_thread <= 16) return launch_cluster_sel<16>(a, o2, cs, st);
  if (per_thread <= 32) return launch_cluster_sel<32>(a, o2, cs, st);
  return cudaErrorInvalidValue;
}

}  // namespace li
