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
//   0 hist   : per-row histogram of the key's top 11 bits
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
  pdl_begin();
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
  pdl_begin();
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
  pdl_begin();
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
  pdl_begin();
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
    case 0: return launch_pdl(topk_hist_kernel, grid_chunks, dim3(kTopkThreads), 0, st, 1, a);
    case 1: return launch_pdl(topk_filter_kernel, grid_chunks, dim3(kTopkThreads), 0, st, 1, a);
    case 2: return launch_pdl(topk_select_kernel, dim3(a.rows), dim3(kSelectThreads), 0, st, 1, a);
    case 3: return launch_pdl(topk_emit_kernel, grid_chunks, dim3(kTopkThreads), 0, st, 1, a);
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace li

// ============================================================================
// Single-launch selection for rows of up to 131072 positions.
//
// A row is taken by CS <= 16 CTAs of 512 threads (a thread-block cluster when
// CS > 1).  Warp w of CTA c owns the contiguous run of 32 * PT positions
// starting at (c * 16 + w) * 32 * PT, and lane l the PT positions from
// l * PT on within it (PT / 4 16-byte loads), held as order-preserving
// uint32 keys in registers for the whole kernel.  The exact k-th key T is
// found digit by digit (11 + 11 + 10 bits): each pass histograms, in its own
// shared-memory array, the keys matching the digits found so far.  The CTAs then exchange counts by one-way pushes: each
// sends its group counts (32 bins a group) into a slot of every other CTA's
// shared memory; every CTA sums the same slots, so all find the same
// boundary group, and each then sends that group's 32 bins the same way and
// finds the boundary bin.  A push lands against an mbarrier of the receiving
// CTA that expects exactly the bytes its peers send (one mbarrier per
// exchange, each completed once), so a CTA waits only for its own data: there
// is no cluster-wide barrier or remote read on the way to T.  The output rank
// of a selected element is #greater before it + min(#equal before it, #equal
// taken), from a scan over the lanes, warp totals within the CTA and
// per-CTA totals pushed to the later CTAs; each lane then writes its own
// selected keys in position order.  One relaxed cluster barrier opens
// the exchanges (every CTA's mbarriers are initialised) and one closes the
// kernel (no CTA exits while a peer may still push to it).  Every wait is
// bounded; a CTA whose wait ran out records the timeout, keeps sending what
// its peers expect, writes no output, and waits for what is still in flight
// to it before exiting.
// ============================================================================
#include <cooperative_groups.h>

namespace li {
namespace {

namespace cg = cooperative_groups;

// Exchanges of one selection, each an mbarrier completed once (parity 0).
enum { kXGroups1 = 0, kXBins1, kXGroups2, kXBins2, kXGroups3, kXBins3, kXTotals, kNumExchanges };

// One radix digit.  hist[NG * 32] is this CTA's complete histogram (the block
// has synchronised).  Group counts go into slot c of gcnt[CS][NG] of every CTA
// (bars[0] of the receiver), the boundary group's bins into slot c of
// gbins[CS][32] (bars[1]).  Warp 0 finds the bin holding the need-th element
// counted from the top (1 <= need <= the row's total) and the elements in
// higher bins: res = {bin, above}.  The caller synchronises the block
// afterwards.
template <int NG, bool CL, int CMAX>
__device__ __forceinline__ void select_digit(int CS, int c, const unsigned* hist, unsigned* gcnt, unsigned* gbins,
                                             uint64_t* bars, int need, int (*res)[2], const WaitCtl& w) {
  constexpr int GPW = NG / (kClusterThreads / 32);    // groups per warp: 4 (NG 64) or 2 (NG 32)
  static_assert(GPW == 2 || GPW == 4, "one 8- or 16-byte push per warp and receiver");
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  {
    unsigned v[GPW];
#pragma unroll
    for (int e = 0; e < GPW; ++e) v[e] = __reduce_add_sync(0xffffffffu, hist[(warp * GPW + e) * 32 + lane]);
    unsigned* mine = gcnt + c * NG + warp * GPW;
    if (lane == c) {
#pragma unroll
      for (int e = 0; e < GPW; ++e) mine[e] = v[e];
    } else if (CL && lane < CS) {
      const uint32_t dst = cluster_addr(mine, lane), bar = cluster_addr(&bars[0], lane);
      if constexpr (GPW == 4) st_async_v4(dst, make_uint4(v[0], v[1], v[2], v[3]), bar);
      else st_async_v2(dst, v[0], v[1], bar);
    }
  }
  __syncthreads();                                     // own slot visible to warp 0
  if (warp != 0) return;
  if (CL) bounded_wait(&bars[0], 0, w);

  // boundary group: lane l owns groups (descending) NG-1-GPL*l ...
  constexpr int GPL = NG / 32;
  unsigned gc[GPL];
#pragma unroll
  for (int e = 0; e < GPL; ++e) gc[e] = 0;
  {
    const int g_lo = NG - GPL * (lane + 1);            // lowest group of this lane
#pragma unroll
    for (int rk = 0; rk < CMAX; ++rk) {
      if (rk < CS) {
        const unsigned* src = gcnt + rk * NG + g_lo;
        if constexpr (GPL == 2) {
          const uint2 u = *reinterpret_cast<const uint2*>(src);
          gc[0] += u.y;                                // higher group first
          gc[1] += u.x;
        } else {
          gc[0] += src[0];
        }
      }
    }
  }
  unsigned tot = 0;
#pragma unroll
  for (int e = 0; e < GPL; ++e) tot += gc[e];
  unsigned incl = tot;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned u = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += u;
  }
  const unsigned nd = static_cast<unsigned>(need);
  const unsigned hit = __ballot_sync(0xffffffffu, incl - tot < nd && nd <= incl);
  const int src_lane = hit ? __ffs(hit) - 1 : 0;
  int grp_sel = 0;
  unsigned above = 0;
  if (lane == src_lane) {
    unsigned cum = incl - tot;
    grp_sel = NG - 1 - GPL * lane;
#pragma unroll
    for (int e = 0; e < GPL; ++e) {
      if (cum + gc[e] >= nd) { grp_sel = NG - 1 - GPL * lane - e; break; }
      cum += gc[e];
    }
    above = cum;
  }
  grp_sel = __shfl_sync(0xffffffffu, grp_sel, src_lane);
  above = __shfl_sync(0xffffffffu, above, src_lane);

  // this CTA's bins of the boundary group to every other CTA (8 x 16 B each)
  if (CL) {
    const uint4* src = reinterpret_cast<const uint4*>(hist + grp_sel * 32);
    for (int o = lane; o < 8 * CS; o += 32) {
      const int rk = o >> 3, ch = o & 7;
      if (rk != c) st_async_v4(cluster_addr(gbins + c * 32 + ch * 4, rk), src[ch], cluster_addr(&bars[1], rk));
    }
    bounded_wait(&bars[1], 0, w);
  }
  // the group's 32 bins summed over the CTAs, descending: lane l takes bin 32 g + 31 - l
  const int bin = grp_sel * 32 + 31 - lane;
  unsigned bc = hist[bin];
  if (CL) {
#pragma unroll
    for (int rk = 0; rk < CMAX; ++rk)
      if (rk < CS && rk != c) bc += gbins[rk * 32 + 31 - lane];
  }
  unsigned bincl = bc;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned u = __shfl_up_sync(0xffffffffu, bincl, o);
    if (lane >= o) bincl += u;
  }
  const unsigned nd2 = nd - above;
  const unsigned bexcl = bincl - bc;
  if (bexcl < nd2 && nd2 <= bincl) {
    res[0][0] = bin;
    res[0][1] = static_cast<int>(above + bexcl);
  }
}

// CMAX: the largest cluster this instantiation serves (8, portable; 16 for
// the longest decode rows, non-portable).
template <int PT, bool CL, int CMAX = 8>
__global__ void __launch_bounds__(kClusterThreads, 1) topk_radix_kernel(const TopkArgs a) {
  pdl_begin();
  constexpr int NW = kClusterThreads / 32;
  constexpr int NSLAB = PT / 4;
  __shared__ __align__(16) unsigned H1[2048];                       // top 11 bits
  __shared__ __align__(16) unsigned H2[2048];                       // next 11 bits (boundary bin)
  __shared__ __align__(16) unsigned H3[1024];                       // last 10 bits (boundary prefix)
  __shared__ __align__(16) unsigned G1[CMAX * 64];                  // group counts of every CTA
  __shared__ __align__(16) unsigned G2[CMAX * 64];
  __shared__ __align__(16) unsigned G3[CMAX * 32];
  __shared__ __align__(16) unsigned B1[CL ? CMAX * 32 : 1];         // boundary-group bins of every CTA
  __shared__ __align__(16) unsigned B2[CL ? CMAX * 32 : 1];
  __shared__ __align__(16) unsigned B3[CL ? CMAX * 32 : 1];
  __shared__ __align__(8) uint64_t xbar[kNumExchanges];
  __shared__ __align__(8) int cin[CMAX][2];                         // (gt, eq) totals of earlier CTAs
  __shared__ int res[1][2];
  __shared__ int wtot[NW];                                          // packed (gt, eq) per warp
  __shared__ int abort_flag;
  cg::cluster_group cluster = cg::this_cluster();
  const int CS = CL ? static_cast<int>(cluster.num_blocks()) : 1;
  const int c = CL ? static_cast<int>(cluster.block_rank()) : 0;
  // rows past a.rows select the second budget of the same score rows
  const bool second = a.k2 > 0 && static_cast<int>(blockIdx.y) >= a.rows;
  const int r = second ? static_cast<int>(blockIdx.y) - a.rows : static_cast<int>(blockIdx.y);
  const int kk = second ? a.k2 : a.k;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n = row_len(a, r);
  const int keff = min(kk, n);
  int32_t* oi = (second ? a.out_idx2 : a.out_idx) + static_cast<int64_t>(r) * kk;
  float* const os_base = second ? a.out_score2 : a.out_score;
  float* osv = os_base ? os_base + static_cast<int64_t>(r) * kk : nullptr;
  if (c == 0) {
    for (int j = max(keff, 0) + threadIdx.x; j < kk; j += blockDim.x) {
      oi[j] = -1;
      if (osv) osv[j] = -INFINITY;
    }
    if (!second && a.out_count && threadIdx.x == 0) a.out_count[r] = max(keff, 0);
  }
  if (keff <= 0) return;   // the same for every CTA of the row

  const WaitCtl wctl{&abort_flag, a.status, a.wait_ns};
  if (threadIdx.x == 0) {
    abort_flag = 0;
    if (CL) {
      for (int i = 0; i < kNumExchanges; ++i) mbar_init(&xbar[i], 1);
      // the bytes every other CTA pushes: group counts (NG x 4 B), boundary
      // bins (128 B), and the totals of the earlier CTAs (8 B each)
      const uint32_t peers = static_cast<uint32_t>(CS - 1);
      mbar_arrive_expect_tx(&xbar[kXGroups1], peers * 64 * 4);
      mbar_arrive_expect_tx(&xbar[kXBins1], peers * 128);
      mbar_arrive_expect_tx(&xbar[kXGroups2], peers * 64 * 4);
      mbar_arrive_expect_tx(&xbar[kXBins2], peers * 128);
      mbar_arrive_expect_tx(&xbar[kXGroups3], peers * 32 * 4);
      mbar_arrive_expect_tx(&xbar[kXBins3], peers * 128);
      mbar_arrive_expect_tx(&xbar[kXTotals], static_cast<uint32_t>(c) * 8);
      fence_barrier_init();
    }
  }
  if (CL) cluster_arrive_relaxed();
  {
    uint4* z = reinterpret_cast<uint4*>(H1);
    for (int i = threadIdx.x; i < 512; i += blockDim.x) z[i] = make_uint4(0, 0, 0, 0);
    z = reinterpret_cast<uint4*>(H2);
    for (int i = threadIdx.x; i < 512; i += blockDim.x) z[i] = make_uint4(0, 0, 0, 0);
    z = reinterpret_cast<uint4*>(H3);
    for (int i = threadIdx.x; i < 256; i += blockDim.x) z[i] = make_uint4(0, 0, 0, 0);
  }

  const int64_t run = (static_cast<int64_t>(c) * NW + warp) * 32 * PT;   // first position of this warp
  const int64_t first = run + static_cast<int64_t>(lane) * PT;          // first position of this lane
  const float* row = a.scores + static_cast<int64_t>(r) * a.row_stride;
  unsigned key[PT];
  unsigned vmask = 0;
  if ((a.row_stride & 3) == 0 && (reinterpret_cast<uintptr_t>(a.scores) & 15) == 0 && run + 32 * PT <= n) {
#pragma unroll
    for (int j = 0; j < NSLAB; ++j) {
      const float4 f = *reinterpret_cast<const float4*>(row + first + 4 * j);
      key[4 * j] = radix_key(f.x);
      key[4 * j + 1] = radix_key(f.y);
      key[4 * j + 2] = radix_key(f.z);
      key[4 * j + 3] = radix_key(f.w);
    }
    vmask = PT == 32 ? 0xffffffffu : ((1u << PT) - 1u);
  } else {
#pragma unroll
    for (int i = 0; i < PT; ++i) {
      key[i] = 0;
      if (first + i < n) {
        key[i] = radix_key(row[first + i]);
        vmask |= 1u << i;
      }
    }
  }
  __syncthreads();   // histograms cleared

  // ---- pass 1: top 11 bits
#pragma unroll
  for (int j = 0; j < PT; ++j)
    if ((vmask >> j) & 1u) atomicAdd(&H1[key[j] >> 21], 1u);
  __syncthreads();
  if (CL) cluster_wait();                              // every CTA's mbarriers are initialised
  select_digit<64, CL, CMAX>(CS, c, H1, G1, B1, &xbar[kXGroups1], keff, res, wctl);
  __syncthreads();
  unsigned pre = static_cast<unsigned>(res[0][0]);
  int above = res[0][1];
  int need = keff - above;

  // ---- pass 2: bits 20..10 of the keys in the boundary bin
#pragma unroll
  for (int j = 0; j < PT; ++j)
    if (((vmask >> j) & 1u) && (key[j] >> 21) == pre) atomicAdd(&H2[(key[j] >> 10) & 2047u], 1u);
  __syncthreads();
  select_digit<64, CL, CMAX>(CS, c, H2, G2, B2, &xbar[kXGroups2], need, res, wctl);
  __syncthreads();
  pre = (pre << 11) | static_cast<unsigned>(res[0][0]);
  above += res[0][1];
  need -= res[0][1];

  // ---- pass 3: bits 9..0 of the keys matching the 22-bit prefix
#pragma unroll
  for (int j = 0; j < PT; ++j)
    if (((vmask >> j) & 1u) && (key[j] >> 10) == pre) atomicAdd(&H3[key[j] & 1023u], 1u);
  __syncthreads();
  select_digit<32, CL, CMAX>(CS, c, H3, G3, B3, &xbar[kXGroups3], need, res, wctl);
  __syncthreads();
  const unsigned T = (pre << 10) | static_cast<unsigned>(res[0][0]);
  above += res[0][1];
  const int need_eq = keff - above;     // elements equal to T that are taken

  // ---- ordered output: lane scan, warp totals, CTA totals, then each lane's keys
  int lane_before = 0;                  // packed (gt, eq) of the lower lanes of this warp
  {
    int x = 0;
#pragma unroll
    for (int j = 0; j < PT; ++j) {
      const bool v = (vmask >> j) & 1u;
      x += (v && key[j] > T) ? 1 : 0;
      x += (v && key[j] == T) ? 0x10000 : 0;
    }
    int incl = x;                       // <= 32 * PT each field
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int u = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += u;
    }
    lane_before = incl - x;
    if (lane == 31) wtot[warp] = incl;
  }
  __syncthreads();
  int gb = 0, eb = 0;                   // elements before this lane's positions
  {
    int before = lane_before, total = 0;
#pragma unroll
    for (int w = 0; w < NW; ++w) {
      const int v = wtot[w];
      before += w < warp ? v : 0;
      total += v;
    }
    gb = before & 0xFFFF;               // <= 16384 each field within a CTA
    eb = before >> 16;
    // per-CTA totals (<= 16384 each) to every later CTA
    if (CL && threadIdx.x < CS && static_cast<int>(threadIdx.x) > c)
      st_async_v2(cluster_addr(&cin[c][0], threadIdx.x), static_cast<uint32_t>(total & 0xFFFF),
                  static_cast<uint32_t>(total >> 16), cluster_addr(&xbar[kXTotals], threadIdx.x));
  }
  if (CL) {
    cluster_arrive_relaxed();           // this CTA has sent everything it sends
    if (warp == 0) bounded_wait(&xbar[kXTotals], 0, wctl);
    __syncthreads();
    for (int rk = 0; rk < c; ++rk) {
      gb += cin[rk][0];
      eb += cin[rk][1];
    }
  }
  const bool aborted = abort_flag != 0;   // uniform: set before the last block barrier
  if (!aborted) {
    const int* map = a.idx_map ? a.idx_map + static_cast<int64_t>(r) * a.map_stride : nullptr;
    int g = gb, q = eb;
#pragma unroll
    for (int i = 0; i < PT; ++i) {
      const bool v = (vmask >> i) & 1u;
      const bool gt = v && key[i] > T;
      const bool eq = v && key[i] == T;
      if (gt || (eq && q < need_eq)) {
        const int rank = g + min(q, need_eq);
        if (rank < kk) {
          const int64_t pos = first + i;
          oi[rank] = map ? map[pos] : static_cast<int32_t>(pos);
          if (osv) osv[rank] = radix_value(key[i]);   // no reload: the key is the score
        }
      }
      g += gt ? 1 : 0;
      q += eq ? 1 : 0;
    }
  }
  if (CL) {
    cluster_wait();                     // every CTA has sent everything it sends
    if (aborted && warp == 0)           // let what is still in flight to this CTA land
      for (int i = 0; i < kNumExchanges; ++i) drain_wait(&xbar[i], 0, 1000000);
  }
}

template <int PT>
cudaError_t launch_radix_pt(const TopkArgs& a, int cs, cudaStream_t st) {
  const unsigned rows = static_cast<unsigned>(a.rows) * (a.k2 > 0 ? 2u : 1u);
  if (cs == 1) return launch_pdl(topk_radix_kernel<PT, false>, dim3(1, rows, 1), dim3(kClusterThreads), 0, st, 1, a);
  if constexpr (PT == 16) {
    if (cs > 8) {
      // a 16-CTA cluster is non-portable: allowed once per process
      static cudaError_t allowed = cudaFuncSetAttribute(topk_radix_kernel<16, true, 16>,
                                                         cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
      if (allowed != cudaSuccess) return allowed;
      return launch_pdl(topk_radix_kernel<16, true, 16>, dim3(cs, rows, 1), dim3(kClusterThreads), 0, st, cs, a);
    }
  }
  if (cs > kClusterMaxSize) return cudaErrorInvalidValue;   // only 16 keys a thread comes in clusters past 8
  return launch_pdl(topk_radix_kernel<PT, true>, dim3(cs, rows, 1), dim3(kClusterThreads), 0, st, cs, a);
}

}  // namespace

int topk_cluster_size(int64_t n, int keys_per_thread, int rows) {
  // A few rows (at most 4) past 65536 positions at the latency target
  // (decode's full-prefix selections) take clusters of up to 16 CTAs (16
  // keys a thread at 131072), measured faster than 8 CTAs at 32 keys a
  // thread.  A 16-CTA cluster needs most of a GPC, so more rows would not
  // run in one wave; everything else stays within portable clusters of 8.
  if (keys_per_thread == kTopkKeysLatency && n > 65536 && rows <= 4) {
    const int64_t cs16 = (n + static_cast<int64_t>(kClusterThreads) * 16 - 1) / (static_cast<int64_t>(kClusterThreads) * 16);
    return static_cast<int>(cs16 > 16 ? 16 : cs16);
  }
  // As many CTAs as keep `keys_per_thread` keys a thread, up to a cluster of
  // 8.  A few rows (decode) are latency-bound: 4 keys a thread spreads them
  // over more CTAs and shortens every pass.  Many rows (a prefill chunk)
  // fill the GPU many times over: 32 keys a thread means fewer CTAs, each
  // paying the per-pass overhead once for more keys.
  int64_t cs = (n + static_cast<int64_t>(kClusterThreads) * keys_per_thread - 1) /
               (static_cast<int64_t>(kClusterThreads) * keys_per_thread);
  return static_cast<int>(cs < 1 ? 1 : (cs > kClusterMaxSize ? kClusterMaxSize : cs));
}

int topk_cluster_capacity(int cs, int num_sms) {
  if (cs < 1 || cs > 16) return -1;
  cudaError_t e;
  if (cs == 1) {
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, topk_radix_kernel<4, false>, kClusterThreads, 0);
    return e == cudaSuccess ? per_sm * num_sms : -1;
  }
  // every instantiation of the clustered kernel is resident one CTA an SM
  // (512 threads above 64 registers each), so one stands for all
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = static_cast<unsigned>(cs);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.gridDim = dim3(static_cast<unsigned>(cs), 1, 1);
  cfg.blockDim = dim3(kClusterThreads, 1, 1);
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cs > kClusterMaxSize) {
    e = cudaFuncSetAttribute(topk_radix_kernel<16, true, 16>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e == cudaSuccess) e = cudaOccupancyMaxActiveClusters(&n, topk_radix_kernel<16, true, 16>, &cfg);
  } else {
    e = cudaOccupancyMaxActiveClusters(&n, topk_radix_kernel<4, true>, &cfg);
  }
  return e == cudaSuccess ? n : -1;
}

int topk_keys_per_thread(int64_t n, int rows, const int* cap) {
  // A few rows are latency-bound: more CTAs a row shorten every pass, as
  // long as all the rows' clusters run in one wave (a second wave costs a
  // whole selection).  Measured: 16 rows of 32768 (the HS anchor's two
  // budgets over 8 sequences) took 30.7 us with the anchor scan at 4 keys a
  // thread (8-CTA clusters, more than are resident at once) against 25.3 us
  // at 16 (4-CTA clusters).  Many rows fill the GPU many times over: 32 keys
  // a thread means fewer CTAs, each paying the per-pass overhead once for
  // more keys (1024 x 65536: 467 us at 32 keys a thread against 788 us at 4).
  for (int kpt = kTopkKeysLatency; kpt <= 16; kpt *= 2) {
    const int cs = topk_cluster_size(n, kpt, rows);
    if (cap[cs] >= rows) return kpt;
  }
  return kTopkKeysThroughput;
}

cudaError_t launch_topk_cluster(const TopkArgs& a, cudaStream_t st, int* cluster_size, int keys_per_thread) {
  const int64_t n = a.n;
  const int cs = topk_cluster_size(n, keys_per_thread, a.rows * (a.k2 > 0 ? 2 : 1));
  const int64_t per_thread = (n + static_cast<int64_t>(cs) * kClusterThreads - 1) / (static_cast<int64_t>(cs) * kClusterThreads);
  if (cluster_size) *cluster_size = cs;
  if (per_thread <= 4) return launch_radix_pt<4>(a, cs, st);
  if (per_thread <= 8) return launch_radix_pt<8>(a, cs, st);
  if (per_thread <= 16) return launch_radix_pt<16>(a, cs, st);
  if (per_thread <= 32) return launch_radix_pt<32>(a, cs, st);
  return cudaErrorInvalidValue;
}

}  // namespace li
