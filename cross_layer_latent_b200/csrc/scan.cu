// scan.cu -- the latent-scan scoring kernel (full prefix) and its HS gather
// variant (candidate rows only), on 5th-generation tensor cores.
//
// Computes, for every valid (query t, cached position s),
//     score(t, s) = sum_h w_{t,h} * max(0, qt_{t,h} . c_s + beta_{t,h})
// (LatentIndex summary, Sec. 3.1: absorbed queries score the shared latent
// directly; Sec. 3.2 / C.4: HS followers rescore only the anchor's
// candidates).  The per-head dot products are one tensor-core contraction
// per 128-row tile: A = 128 cache rows x dim (K-major, swizzled smem, loaded
// by TMA or gathered by cp.async), B = Qg queries x H_pad heads x dim, D =
// 128 x N fp32 in tensor memory.  An epilogue warpgroup reads D lane by lane
// (one cached row per thread), applies ReLU, the head weights and the
// per-token / per-head fp8 scales, reduces over heads and writes one fp32
// score per (query, row); per-head scores never leave the SM.
//
// Warp roles (192 threads): warp 0 loads (TMA, or 32-lane cp.async gather),
// warp 1 allocates tensor memory and issues the MMAs, warps 2..5 run the
// epilogue.  Each CTA is persistent over a contiguous range of work items
// (segment, tile); a segment is one (sequence, query group) of the scan or
// one (sequence, query) of the gather.  All waits are bounded.
#include "internal.h"
#include "sm100.cuh"

namespace li {

namespace {

constexpr uint64_t kDrainNs = 200ull * 1000ull * 1000ull;   // 0.2 s

struct ScanSmem {
  uint8_t* a_stages;
  uint8_t* b_slots;
  uint64_t* full;
  uint64_t* empty;
  uint64_t* bfull;
  uint64_t* bempty;
  uint64_t* accfull;
  uint64_t* accempty;
  uint64_t* drain;
  uint32_t* tmem_base;
  int* abort_flag;
  int* prefix;          // [kMaxSegments + 1]
  float* ep;            // 4 warps x (3 * N + 16) floats
};

__device__ __forceinline__ ScanSmem carve(uint8_t* base, const ScanArgs& a) {
  ScanSmem s;
  s.a_stages = base;
  s.b_slots = base + static_cast<size_t>(a.n_stages) * a.a_stage_bytes;
  uint8_t* p = base + a.misc_offset;
  s.full = reinterpret_cast<uint64_t*>(p);
  s.empty = s.full + kMaxStages;
  s.bfull = s.empty + kMaxStages;
  s.bempty = s.bfull + 2;
  s.accfull = s.bempty + 2;
  s.accempty = s.accfull + 4;
  s.drain = s.accempty + 4;
  s.tmem_base = reinterpret_cast<uint32_t*>(s.drain + 1);
  s.abort_flag = reinterpret_cast<int*>(s.tmem_base + 1);
  s.prefix = s.abort_flag + 3;
  s.ep = reinterpret_cast<float*>(s.prefix + kMaxSegments + 1);
  return s;
}

// Number of 128-row tiles a segment needs.
template <bool GATHER>
__device__ __forceinline__ int segment_tiles(const ScanArgs& a, int seg) {
  if (GATHER) {
    int n = a.cand_n[seg];
    n = n < 0 ? 0 : (n > a.cand_stride ? a.cand_stride : n);
    return (n + kTileM - 1) / kTileM;
  }
  const int b = seg / a.n_groups, g = seg % a.n_groups;
  int len = a.lengths[b];
  len = len < 0 ? 0 : (len > a.capacity ? a.capacity : len);
  int L = len;
  if (a.q_pos) {
    L = 0;
    for (int qi = 0; qi < a.Qg; ++qi) {
      const int t = g * a.Qg + qi;
      if (t >= a.T) break;
      int v = a.q_pos[b * a.T + t] + 1;
      v = v < 0 ? 0 : (v > len ? len : v);
      L = v > L ? v : L;
    }
  }
  return (L + kTileM - 1) / kTileM;
}

struct ItemCursor {
  const int* prefix;
  int seg;
  __device__ __forceinline__ void seek(int item) {
    while (prefix[seg + 1] <= item) ++seg;
  }
};

// Swizzled byte offset inside a K-major tile whose rows are `swz` bytes.
__device__ __forceinline__ uint32_t swizzle(uint32_t off, uint32_t swz) {
  return off ^ (((off >> 7) & ((swz >> 4) - 1u)) << 4);
}

template <int KIND, bool GATHER>
__global__ void __launch_bounds__(kScanThreads, 1) scan_kernel(const __grid_constant__ ScanArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  ScanSmem s = carve(base, a);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (tid == 0) {
    for (int i = 0; i < a.n_stages; ++i) { mbar_init(&s.full[i], GATHER ? 32 : 1); mbar_init(&s.empty[i], 1); }
    for (int i = 0; i < a.n_bslots; ++i) { mbar_init(&s.bfull[i], 1); mbar_init(&s.bempty[i], 1); }
    for (int i = 0; i < a.n_acc; ++i) { mbar_init(&s.accfull[i], 1); mbar_init(&s.accempty[i], 4); }
    mbar_init(s.drain, 1);
    *s.abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(s.tmem_base, a.tmem_cols);
    tmem_relinquish();
  }
  // Tiles per segment, then an exclusive prefix over segments.
  for (int i = tid; i < a.n_segments; i += blockDim.x) s.prefix[i + 1] = segment_tiles<GATHER>(a, i);
  __syncthreads();
  if (warp == 0) {
    int carry = 0;
    for (int c = 0; c < a.n_segments; c += 32) {
      const int i = c + lane;
      int v = i < a.n_segments ? s.prefix[i + 1] : 0;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += u;
      }
      if (i < a.n_segments) s.prefix[i + 1] = v + carry;
      carry += __shfl_sync(0xffffffffu, v, 31);
    }
    if (lane == 0) s.prefix[0] = 0;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  const int total = s.prefix[a.n_segments];
  const int begin = static_cast<int>((static_cast<int64_t>(total) * blockIdx.x) / gridDim.x);
  const int end = static_cast<int>((static_cast<int64_t>(total) * (blockIdx.x + 1)) / gridDim.x);
  const WaitCtl wc{s.abort_flag, a.status, a.wait_ns};
  const uint32_t tmem = *s.tmem_base;
  const int S = a.n_stages;
  const int elt_per_chunk = a.swz / a.elt_bytes;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    uint32_t kcount = 0, b_use = 0;
    int cur_seg = -1;
    ItemCursor cur{s.prefix, 0};
    if (!GATHER) {
      if (lane == 0) {
        tma_prefetch_desc(&a.map_a);
        tma_prefetch_desc(&a.map_b);
        for (int item = begin; item < end && !*s.abort_flag; ++item) {
          cur.seek(item);
          const int seg = cur.seg, tile = item - s.prefix[seg];
          if (seg != cur_seg) {
            const int slot = b_use % a.n_bslots;
            if (!bounded_wait(&s.bempty[slot], ((b_use / a.n_bslots) & 1u) ^ 1u, wc)) break;
            mbar_arrive_expect_tx(&s.bfull[slot], a.b_slot_bytes);
            const int b = seg / a.n_groups, g = seg % a.n_groups;
            uint8_t* dst = s.b_slots + static_cast<size_t>(slot) * a.b_slot_bytes;
            for (int kc = 0; kc < a.n_kchunks; ++kc)
              tma_load_3d(dst + static_cast<size_t>(kc) * a.N * a.swz, &a.map_b, &s.bfull[slot],
                          kc * elt_per_chunk, 0, b * a.T + g * a.Qg);
            ++b_use;
            cur_seg = seg;
          }
          const int b = seg / a.n_groups;
          const int row0 = b * a.capacity + tile * kTileM;
          bool ok = true;
          for (int kc = 0; kc < a.n_kchunks; ++kc) {
            const int st = kcount % S;
            if (!bounded_wait(&s.empty[st], ((kcount / S) & 1u) ^ 1u, wc)) { ok = false; break; }
            mbar_arrive_expect_tx(&s.full[st], a.a_stage_bytes);
            tma_load_2d(s.a_stages + static_cast<size_t>(st) * a.a_stage_bytes, &a.map_a, &s.full[st],
                        kc * elt_per_chunk, row0);
            ++kcount;
          }
          if (!ok) break;
        }
        if (*s.abort_flag) {
          // Let every copy already issued land before the CTA exits.
          const uint32_t nst = kcount < static_cast<uint32_t>(S) ? kcount : S;
          for (uint32_t i = 0; i < nst; ++i) {
            const uint32_t last = kcount - 1 - ((kcount - 1 - i) % S);   // last use of stage i
            drain_wait(&s.full[i], (last / S) & 1u, kDrainNs);
          }
          const uint32_t nb = b_use < static_cast<uint32_t>(a.n_bslots) ? b_use : a.n_bslots;
          for (uint32_t i = 0; i < nb; ++i) {
            const uint32_t last = b_use - 1 - ((b_use - 1 - i) % a.n_bslots);
            drain_wait(&s.bfull[i], (last / a.n_bslots) & 1u, kDrainNs);
          }
        }
      }
    } else {
      // Gather: 32 lanes copy candidate rows with 16-byte cp.async into the
      // same swizzled layout TMA would produce; a stage is signalled full
      // once every lane's copies for it have landed (4 stages in flight).
      constexpr int kDepth = 4;
      uint32_t pend[kDepth];
      int inflight = 0;
      const int chunks16 = a.swz >> 4;
      for (int item = begin; item < end && !*s.abort_flag; ++item) {
        cur.seek(item);
        const int seg = cur.seg, tile = item - s.prefix[seg];
        if (seg != cur_seg) {
          bool ok = true;
          if (lane == 0) {
            const int slot = b_use % a.n_bslots;
            ok = bounded_wait(&s.bempty[slot], ((b_use / a.n_bslots) & 1u) ^ 1u, wc);
            if (ok) {
              mbar_arrive_expect_tx(&s.bfull[slot], a.b_slot_bytes);
              uint8_t* dst = s.b_slots + static_cast<size_t>(slot) * a.b_slot_bytes;
              for (int kc = 0; kc < a.n_kchunks; ++kc)
                tma_load_3d(dst + static_cast<size_t>(kc) * a.N * a.swz, &a.map_b, &s.bfull[slot],
                            kc * elt_per_chunk, 0, seg);
            }
          }
          ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
          if (!ok) break;
          ++b_use;
          cur_seg = seg;
        }
        const int b = seg / a.T;
        int len = a.lengths[b];
        len = len < 0 ? 0 : (len > a.capacity ? a.capacity : len);
        int cn = a.cand_n[seg];
        cn = cn < 0 ? 0 : (cn > a.cand_stride ? a.cand_stride : cn);
        int tok[kTileM / 32];
#pragma unroll
        for (int i = 0; i < kTileM / 32; ++i) {
          const int j = tile * kTileM + lane + 32 * i;
          const int t = j < cn ? a.cand[static_cast<int64_t>(seg) * a.cand_stride + j] : -1;
          tok[i] = (t >= 0 && t < len) ? t : -1;
        }
        bool ok = true;
        for (int kc = 0; kc < a.n_kchunks; ++kc) {
          const int st = kcount % S;
          // One lane waits; the whole warp follows its verdict so the lanes
          // never diverge around the warp-synchronous calls.
          int got = 1;
          if (lane == 0) got = bounded_wait(&s.empty[st], ((kcount / S) & 1u) ^ 1u, wc) ? 1 : 0;
          got = __shfl_sync(0xffffffffu, got, 0);
          if (!got) { ok = false; break; }
          const uint32_t dst = smem_addr(s.a_stages + static_cast<size_t>(st) * a.a_stage_bytes);
#pragma unroll
          for (int i = 0; i < kTileM / 32; ++i) {
            if (tok[i] < 0) continue;
            const int r = lane + 32 * i;
            const uint8_t* src = a.cache + (static_cast<int64_t>(b) * a.capacity + tok[i]) * a.row_bytes +
                                 static_cast<int64_t>(kc) * a.swz;
            for (int c = 0; c < chunks16; ++c)
              cp_async_16(dst + swizzle(static_cast<uint32_t>(r * a.swz + c * 16), a.swz), src + c * 16);
          }
          cp_async_commit();
          pend[kcount % kDepth] = st;
          ++kcount;
          if (++inflight == kDepth) {
            cp_async_wait_group<kDepth - 1>();
            fence_proxy_async_smem();
            mbar_arrive(&s.full[pend[(kcount - kDepth) % kDepth]]);
            --inflight;
          }
        }
        if (!ok) break;
      }
      cp_async_wait_all();
      fence_proxy_async_smem();
      if (!*s.abort_flag) {
        for (; inflight > 0; --inflight) mbar_arrive(&s.full[pend[(kcount - inflight) % kDepth]]);
      } else if (lane == 0) {
        const uint32_t nb = b_use < static_cast<uint32_t>(a.n_bslots) ? b_use : a.n_bslots;
        for (uint32_t i = 0; i < nb; ++i) {
          const uint32_t last = b_use - 1 - ((b_use - 1 - i) % a.n_bslots);
          drain_wait(&s.bfull[i], (last / a.n_bslots) & 1u, kDrainNs);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      uint32_t kcount = 0, b_use = 0, acc_use = 0;
      int cur_seg = -1, slot = -1;
      ItemCursor cur{s.prefix, 0};
      for (int item = begin; item < end && !*s.abort_flag; ++item) {
        cur.seek(item);
        const int seg = cur.seg;
        if (seg != cur_seg) {
          if (slot >= 0) umma_commit(&s.bempty[slot]);
          slot = b_use % a.n_bslots;
          if (!bounded_wait(&s.bfull[slot], (b_use / a.n_bslots) & 1u, wc)) break;
          tc_fence_after();
          ++b_use;
          cur_seg = seg;
        }
        const int acc = acc_use % a.n_acc;
        if (!bounded_wait(&s.accempty[acc], ((acc_use / a.n_acc) & 1u) ^ 1u, wc)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem + static_cast<uint32_t>(acc * a.N);
        const uint32_t b_base = smem_addr(s.b_slots + static_cast<size_t>(slot) * a.b_slot_bytes);
        bool ok = true;
        for (int kc = 0; kc < a.n_kchunks; ++kc) {
          const int st = kcount % S;
          if (!bounded_wait(&s.full[st], (kcount / S) & 1u, wc)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_base = smem_addr(s.a_stages + static_cast<size_t>(st) * a.a_stage_bytes);
          const uint32_t bk = b_base + static_cast<uint32_t>(kc * a.N * a.swz);
          for (int ks = 0; ks < (a.swz >> 5); ++ks) {
            umma<KIND>(d_tmem, make_smem_desc(a_base + ks * 32, a.swz), make_smem_desc(bk + ks * 32, a.swz),
                       a.idesc, (kc | ks) != 0 ? 1u : 0u);
          }
          umma_commit(&s.empty[st]);
          ++kcount;
        }
        if (!ok) break;
        umma_commit(&s.accfull[acc]);
        ++acc_use;
      }
      if (*s.abort_flag) {
        umma_commit(s.drain);
        drain_wait(s.drain, 0, kDrainNs);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int ew = warp - 2;                 // 0..3
    const int quad = warp & 3;               // TMEM lane quadrant this warp may access
    const int r = quad * 32 + lane;          // row of the tile = TMEM lane
    float* ep_w = s.ep + ew * (3 * a.N + 16);
    float* ep_qs = ep_w + a.N;
    float* ep_beta = ep_qs + a.N;
    int* ep_len = reinterpret_cast<int*>(ep_beta + a.N);
    uint32_t acc_use = 0;
    int cur_seg = -1;
    ItemCursor cur{s.prefix, 0};
    const bool has_beta = a.beta != nullptr;
    for (int item = begin; item < end && !*s.abort_flag; ++item) {
      cur.seek(item);
      const int seg = cur.seg, tile = item - s.prefix[seg];
      const int b = GATHER ? seg / a.T : seg / a.n_groups;
      const int g = GATHER ? seg % a.T : seg % a.n_groups;
      int len = a.lengths[b];
      len = len < 0 ? 0 : (len > a.capacity ? a.capacity : len);
      if (seg != cur_seg) {
        __syncwarp();
        for (int i = lane; i < a.N; i += 32) {
          const int qi = i / a.H_pad, h = i % a.H_pad;
          const int t = g * a.Qg + qi;
          float wv = 0.f, qs = 1.f, be = 0.f;
          if (h < a.H && t < a.T) {
            const int64_t o = (static_cast<int64_t>(b) * a.T + t) * a.H + h;
            wv = a.w[o];
            if (a.q_scale) qs = a.q_scale[o];
            if (has_beta) be = a.beta[o];
          }
          // Without a bias, fold the query scale into the weight (ReLU is
          // positively homogeneous and the scales are positive).
          ep_w[i] = has_beta ? wv : wv * qs;
          ep_qs[i] = qs;
          ep_beta[i] = be;
        }
        if (lane < 16) {
          const int t = g * a.Qg + lane;
          int v = 0;
          if (lane < a.Qg && t < a.T) {
            if (GATHER) {
              v = a.cand_n[seg];
              v = v < 0 ? 0 : (v > a.cand_stride ? a.cand_stride : v);
            } else {
              v = len;
              if (a.q_pos) {
                int p = a.q_pos[b * a.T + t] + 1;
                v = p < 0 ? 0 : (p > len ? len : p);
              }
            }
          }
          ep_len[lane] = v;
        }
        __syncwarp();
        cur_seg = seg;
      }
      const int acc = acc_use % a.n_acc;
      if (!bounded_wait(&s.accfull[acc], (acc_use / a.n_acc) & 1u, wc)) break;
      tc_fence_after();

      const int j = tile * kTileM + r;      // position (scan) or candidate slot (gather)
      int tok = j;
      bool tok_ok = true;
      if (GATHER) {
        tok = j < ep_len[0] ? a.cand[static_cast<int64_t>(seg) * a.cand_stride + j] : -1;
        tok_ok = tok >= 0 && tok < len;
      }
      float cs = 1.f;
      if (a.cache_scale && tok_ok && j < (GATHER ? ep_len[0] : len))
        cs = a.cache_scale[static_cast<int64_t>(b) * a.capacity + tok];
      const uint32_t tbase = tmem + (static_cast<uint32_t>(quad * 32) << 16) + static_cast<uint32_t>(acc * a.N);
      for (int qi = 0; qi < a.Qg; ++qi) {
        const int t = g * a.Qg + qi;
        if (t >= a.T) break;
        float sc = 0.f;
        const float* wq = ep_w + qi * a.H_pad;
        const float* qs = ep_qs + qi * a.H_pad;
        const float* be = ep_beta + qi * a.H_pad;
        int h0 = 0;
        for (; h0 + 32 <= a.H_pad; h0 += 32) {
          float v[32];
          tmem_load32_sync(tbase + static_cast<uint32_t>(qi * a.H_pad + h0), v);
          if (!has_beta) {
#pragma unroll
            for (int e = 0; e < 32; ++e) sc = fmaf(wq[h0 + e], fmaxf(v[e], 0.f), sc);
          } else {
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              const float x = fmaf(v[e], qs[h0 + e] * cs, be[h0 + e]);
              sc = fmaf(wq[h0 + e], fmaxf(x, 0.f), sc);
            }
          }
        }
        if (h0 < a.H_pad) {   // H_pad % 32 == 16
          float v[16];
          tmem_load16_sync(tbase + static_cast<uint32_t>(qi * a.H_pad + h0), v);
          if (!has_beta) {
#pragma unroll
            for (int e = 0; e < 16; ++e) sc = fmaf(wq[h0 + e], fmaxf(v[e], 0.f), sc);
          } else {
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              const float x = fmaf(v[e], qs[h0 + e] * cs, be[h0 + e]);
              sc = fmaf(wq[h0 + e], fmaxf(x, 0.f), sc);
            }
          }
        }
        if (!has_beta && a.cache_scale) sc *= cs;
        if (j < ep_len[qi]) {
          if (!tok_ok) {
            sc = -INFINITY;
            record_status(a.status, kStatusIndex);
          }
          const int64_t row = static_cast<int64_t>(b) * a.T + t;
          a.scores[row * a.score_stride + j] = sc;
          if (a.hist) atomicAdd(&a.hist[row * kHistBins + (radix_key(sc) >> 21)], 1u);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s.accempty[acc]);
      ++acc_use;
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, a.tmem_cols);
}

template <int KIND, bool GATHER>
cudaError_t launch_one(const ScanArgs& a, int grid, cudaStream_t st) {
  auto k = scan_kernel<KIND, GATHER>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, a.smem_bytes);
  if (e != cudaSuccess) return e;
  k<<<grid, kScanThreads, a.smem_bytes, st>>>(a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_scan_kernel(int kind, bool gather, const ScanArgs& a, int grid, cudaStream_t st) {
  switch (kind * 2 + (gather ? 1 : 0)) {
    case kKindTF32 * 2: return launch_one<kKindTF32, false>(a, grid, st);
    case kKindTF32 * 2 + 1: return launch_one<kKindTF32, true>(a, grid, st);
    case kKindBF16 * 2: return launch_one<kKindBF16, false>(a, grid, st);
    case kKindBF16 * 2 + 1: return launch_one<kKindBF16, true>(a, grid, st);
    case kKindE4M3 * 2: return launch_one<kKindE4M3, false>(a, grid, st);
    case kKindE4M3 * 2 + 1: return launch_one<kKindE4M3, true>(a, grid, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace li
