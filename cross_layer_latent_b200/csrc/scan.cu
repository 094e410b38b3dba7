// scan.cu -- the latent-scan scoring kernel (full prefix) and its HS gather
// variant (candidate rows only), on 5th-generation tensor cores.
//
// Computes, for every valid (query t, cached position s),
//     score(t, s) = sum_h w_{t,h} * max(0, qt_{t,h} . c_s + beta_{t,h})
// (LatentIndex summary, Sec. 3.1: absorbed queries score the shared latent
// directly; Sec. 3.2 / C.4: HS followers rescore only the anchor's
// candidates).  The per-head dot products are tensor-core contractions:
// A = 128 cache rows x dim (K-major, swizzled smem), B = Qg queries x H_pad
// heads x dim, D = 128 x N fp32 in tensor memory.  Epilogue warps read D lane
// by lane (one cached row per thread), apply ReLU, the head weights and the
// per-token / per-head fp8 scales, reduce over heads and write one fp32 score
// per (query, row); per-head scores never leave the SM.
//
// Work is cut into items of R = 128 or 256 rows (one or two M=128 MMA
// blocks).  A pipeline stage holds KS K-chunks of an item's R rows, loaded by
// ONE 3-D TMA box ({chunk bytes, rows, chunks}, smem order [chunk][row]) or
// gathered by cp.async; decode items use one stage per item.  The control
// paths are single-lane dependency chains whose every step (mbarrier wait,
// MMA issue, shared load) costs on the order of 100 cycles, so each step is
// made to move as many bytes as the shared-memory budget allows.
//
// Warp roles (64 + 32 * kEpiWarps threads): warp 0 loads (one lane issues
// TMA; all 32 lanes gather), warp 1 allocates tensor memory and one lane
// issues the MMAs, and two epilogue warpgroups take the two M blocks of an
// item (R = 256) or alternate items (R = 128).  Per-item row metadata (fp8
// per-token scales, gathered token ids) travels through its own ring.  Each
// CTA is persistent over a contiguous range of items; a segment is one
// (sequence, query group) of the scan or one (sequence, query) of the gather.
// Every wait is bounded; ring positions advance without integer division.
#include <type_traits>

#include "internal.h"
#include "sm100.cuh"

namespace li {

namespace {

constexpr uint64_t kDrainNs = 200ull * 1000ull * 1000ull;   // 0.2 s

struct ScanSmem {
  uint8_t* a_stages;
  uint8_t* b_slots;
  uint8_t* meta;        // n_meta x meta_bytes: scale[R x scales per row] (then tok[R] when gathering)
  uint64_t* full;
  uint64_t* empty;
  uint64_t* bfull;
  uint64_t* bempty;
  uint64_t* accfull;
  uint64_t* accempty;
  uint64_t* mfull;
  uint64_t* mempty;
  uint64_t* drain;
  uint64_t* ready;      // gather: [stage] the first loader has armed the stage and published its rows
  uint32_t* tmem_base;
  int* abort_flag;
  int* prefix;          // [n_segments + 1]
  float* ep;            // kEpiWarps x ep_stride floats
  int* seg_n;           // gather: [n_segments] candidates of each segment (clamped)
  int* seg_len;         // gather: [n_segments] valid length of the segment's sequence
};

// Shared-memory layout; scan_misc_bytes() on the host sizes the part after
// misc_offset the same way.
__device__ __forceinline__ ScanSmem carve(uint8_t* base, const ScanArgs& a) {
  ScanSmem s;
  s.a_stages = base;
  s.b_slots = base + static_cast<size_t>(a.n_stages) * a.a_stage_bytes;
  s.meta = s.b_slots + static_cast<size_t>(a.n_bslots) * a.b_slot_bytes;
  uint8_t* p = base + a.misc_offset;
  s.full = reinterpret_cast<uint64_t*>(p);
  s.empty = s.full + kMaxStages;
  s.bfull = s.empty + kMaxStages;
  s.bempty = s.bfull + 2;
  s.accfull = s.bempty + 2;               // [accumulator slot][M block]
  s.accempty = s.accfull + 8;
  s.mfull = s.accempty + 8;
  s.mempty = s.mfull + kMetaSlots;
  s.drain = s.mempty + kMetaSlots;        // one per MMA issuer
  s.ready = s.drain + 2;
  s.tmem_base = reinterpret_cast<uint32_t*>(s.ready + kMaxStages);
  s.abort_flag = reinterpret_cast<int*>(s.tmem_base + 1);
  s.prefix = s.abort_flag + 2;
  // 16-byte aligned parameter arrays (read four at a time)
  s.ep = reinterpret_cast<float*>((reinterpret_cast<uintptr_t>(s.prefix + a.n_segments + 1) + 15) & ~uintptr_t(15));
  s.seg_n = reinterpret_cast<int*>(s.ep + kEpiWarps * a.ep_stride);
  s.seg_len = s.seg_n + a.n_segments;
  return s;
}

// Number of R-row items a segment needs.
template <bool GATHER>
__device__ __forceinline__ int segment_items(const ScanArgs& a, int seg) {
  if (GATHER) {
    int n = a.cand_n[seg];
    n = n < 0 ? 0 : (n > a.cand_stride ? a.cand_stride : n);
    return (n + a.RI - 1) / a.RI;
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
  return (L + a.R - 1) / a.R;
}

// Position in a ring of n barriers/buffers: index and the parity of the
// current pass.  Advancing never divides (integer division costs ~50 cycles
// on the issuing warp, and these loops run once per item).
struct Ring {
  uint32_t i = 0, ph = 0;
  __device__ __forceinline__ void step(uint32_t n) {
    if (++i == n) { i = 0; ph ^= 1u; }
  }
  __device__ __forceinline__ void step_by(uint32_t k, uint32_t n) {   // k <= n
    i += k;
    if (i >= n) { i -= n; ph ^= 1u; }
  }
};

// Walks the segments of an item range in order, keeping (b, g) without
// division: segment seg = b * n_groups + g.
struct SegWalk {
  const int* prefix;
  int n_groups;
  int seg = 0, b = 0, g = 0;
  __device__ __forceinline__ bool to(int item) {
    bool moved = false;
    while (prefix[seg + 1] <= item) {
      ++seg;
      if (++g == n_groups) { g = 0; ++b; }
      moved = true;
    }
    return moved;
  }
};

// 4-byte cp.async reading src_bytes (0 or 4).
__device__ __forceinline__ void cp_async_4_zfill(uint32_t dst_smem, const void* src, int src_bytes) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(dst_smem), "l"(src), "r"(src_bytes)
               : "memory");
}

__device__ __forceinline__ void cp_async_8_zfill(uint32_t dst_smem, const void* src, int src_bytes) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 8, %2;" ::"r"(dst_smem), "l"(src), "r"(src_bytes)
               : "memory");
}

// Bulk (non-tensor) global -> shared copy completing on an mbarrier;
// addresses and size must be multiples of 16 bytes.
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_addr(dst)),
      "l"(src), "r"(bytes), "r"(smem_addr(bar))
      : "memory");
}

// sum_h wq_h * max(v_h, 0) over 16 columns, in 4 interleaved partial sums;
// the weights are read four at a time.
__device__ __forceinline__ void relu_dot16(const float* v, const float* wq, float (&acc)[4]) {
#pragma unroll
  for (int e = 0; e < 16; e += 4) {
    const float4 w4 = *reinterpret_cast<const float4*>(wq + e);
    acc[0] = fmaf(w4.x, fmaxf(v[e], 0.f), acc[0]);
    acc[1] = fmaf(w4.y, fmaxf(v[e + 1], 0.f), acc[1]);
    acc[2] = fmaf(w4.z, fmaxf(v[e + 2], 0.f), acc[2]);
    acc[3] = fmaf(w4.w, fmaxf(v[e + 3], 0.f), acc[3]);
  }
}

// c0 += a0 * b0 and c1 += a1 * b1 as one paired fp32 FMA (sm_100's
// fma.rn.f32x2): each lane is an IEEE fma, so the results equal two fmaf.
__device__ __forceinline__ void ffma2(float& c0, float& c1, float a0, float a1, float b0, float b1) {
  asm("{\n\t.reg .b64 ra, rb, rc;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%0, %1};\n\t"
      "fma.rn.f32x2 rc, ra, rb, rc;\n\tmov.b64 {%0, %1}, rc;\n\t}"
      : "+f"(c0), "+f"(c1)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}

// relu_dot16 with paired FMAs (same arithmetic, same order): the epilogue of
// several query rows per item is bound by its arithmetic and tensor-memory
// loads, and this takes 4% off the prefill scan; the decode epilogue is not
// bound by it and keeps the scalar form.
__device__ __forceinline__ void relu_dot16_pk(const float* v, const float* wq, float (&acc)[4]) {
#pragma unroll
  for (int e = 0; e < 16; e += 4) {
    const float4 w4 = *reinterpret_cast<const float4*>(wq + e);
    ffma2(acc[0], acc[1], w4.x, w4.y, fmaxf(v[e], 0.f), fmaxf(v[e + 1], 0.f));
    ffma2(acc[2], acc[3], w4.z, w4.w, fmaxf(v[e + 2], 0.f), fmaxf(v[e + 3], 0.f));
  }
}

__device__ __forceinline__ void relu_dot16_beta(const float* v, const float* w, const float* qs,
                                                const float* be, float cs, float (&acc)[4]) {
#pragma unroll
  for (int e = 0; e < 16; ++e) {
    const float x = fmaf(v[e], qs[e] * cs, be[e]);
    acc[e & 3] = fmaf(w[e], fmaxf(x, 0.f), acc[e & 3]);
  }
}

// The MMAs of one K-chunk of a stage: KSTEPS steps of 32 bytes along K, each
// for MB row blocks (separate accumulators N columns apart).  Unrolled: the
// issuing thread is a single dependency chain, so loop control and address
// arithmetic per MMA would otherwise cost as much as the MMA itself.
template <int KIND, int KSTEPS, int MB>
__device__ __forceinline__ void issue_chunk(uint32_t d0, uint32_t a_c, uint32_t b_c, uint64_t adesc_hi, uint64_t desc_hi,
                                            uint32_t m_stride, uint32_t n_cols, uint32_t idesc, bool first_chunk) {
#pragma unroll
  for (int ks = 0; ks < KSTEPS; ++ks) {
    const uint64_t bdesc = desc_hi | ((b_c + ks * 32u) >> 4);
#pragma unroll
    for (int mb = 0; mb < MB; ++mb) {
      const uint64_t adesc = adesc_hi | ((a_c + mb * m_stride + ks * 32u) >> 4);
      umma<KIND>(d0 + mb * n_cols, adesc, bdesc, idesc, (first_chunk && ks == 0) ? 0u : 1u);
    }
  }
}

template <int KIND>
__device__ __forceinline__ void issue_chunk_rt(int ksteps, int mbs, uint32_t d0, uint32_t a_c, uint32_t b_c,
                                               uint64_t adesc_hi, uint64_t desc_hi, uint32_t m_stride,
                                               uint32_t n_cols, uint32_t idesc,
                                               bool first_chunk) {
  switch (ksteps * 4 + mbs) {
    case 1 * 4 + 1: issue_chunk<KIND, 1, 1>(d0, a_c, b_c, adesc_hi, desc_hi, m_stride, n_cols, idesc, first_chunk); break;
    case 1 * 4 + 2: issue_chunk<KIND, 1, 2>(d0, a_c, b_c, adesc_hi, desc_hi, m_stride, n_cols, idesc, first_chunk); break;
    case 2 * 4 + 1: issue_chunk<KIND, 2, 1>(d0, a_c, b_c, adesc_hi, desc_hi, m_stride, n_cols, idesc, first_chunk); break;
    case 2 * 4 + 2: issue_chunk<KIND, 2, 2>(d0, a_c, b_c, adesc_hi, desc_hi, m_stride, n_cols, idesc, first_chunk); break;
    case 3 * 4 + 1: issue_chunk<KIND, 3, 1>(d0, a_c, b_c, adesc_hi, desc_hi, m_stride, n_cols, idesc, first_chunk); break;
    case 3 * 4 + 2: issue_chunk<KIND, 3, 2>(d0, a_c, b_c, adesc_hi, desc_hi, m_stride, n_cols, idesc, first_chunk); break;
    case 4 * 4 + 1: issue_chunk<KIND, 4, 1>(d0, a_c, b_c, adesc_hi, desc_hi, m_stride, n_cols, idesc, first_chunk); break;
    default: issue_chunk<KIND, 4, 2>(d0, a_c, b_c, adesc_hi, desc_hi, m_stride, n_cols, idesc, first_chunk); break;
  }
}

__device__ __forceinline__ void trace_event(uint64_t* trace, uint32_t lt, int ev) {
  if (trace && blockIdx.x < kTraceCtas && lt < kTraceTiles)
    trace[(static_cast<size_t>(blockIdx.x) * kTraceTiles + lt) * kTraceEvents + ev] = cycles();
}

// Wait for the last pass of every slot of a ring used `uses` times (only
// after an abort; divisions are fine here).
__device__ __forceinline__ void drain_ring(uint64_t* bars, uint32_t n, uint32_t uses) {
  const uint32_t m = uses < n ? uses : n;
  for (uint32_t i = 0; i < m; ++i) {
    const uint32_t last = uses - 1 - ((uses - 1 - i) % n);
    drain_wait(&bars[i], (last / n) & 1u, kDrainNs);
  }
}

template <int KIND, bool GATHER, bool SEG, bool MQ>
__global__ void __launch_bounds__(kScanThreads, 1) scan_kernel(const __grid_constant__ ScanArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  ScanSmem s = carve(base, a);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const bool e4 = a.cache_scale != nullptr;
  const bool has_meta = GATHER || e4;

  if (tid == 0) {
    // every MMA issuer (one per M block) releases stages and query slots
    for (int i = 0; i < a.n_stages; ++i) {
      mbar_init(&s.full[i], 1);
      mbar_init(&s.empty[i], a.MB);
      mbar_init(&s.ready[i], 1);
    }
    for (int i = 0; i < a.n_bslots; ++i) { mbar_init(&s.bfull[i], 1); mbar_init(&s.bempty[i], a.MB); }
    // accumulator (slot, M block): one issuer fills it, one warpgroup drains it
    for (int i = 0; i < 2 * a.n_acc; ++i) { mbar_init(&s.accfull[i], 1); mbar_init(&s.accempty[i], 4); }
    for (int i = 0; i < kMetaSlots; ++i) {
      // gather: every loader lane arrives once after storing its token ids
      // and once (asynchronously) when its scale copies have landed
      mbar_init(&s.mfull[i], GATHER ? 64 : 1);
      mbar_init(&s.mempty[i], 4 * a.MB);
    }
    mbar_init(&s.drain[0], 1);
    mbar_init(&s.drain[1], 1);
    *s.abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_desc(&a.map_a);
    tma_prefetch_desc(&a.map_b);
    if (GATHER && a.tail64) tma_prefetch_desc(&a.map_a2);
  }
  if (warp == 1) {
    tmem_alloc(s.tmem_base, a.tmem_cols);
    tmem_relinquish();
  }
  if (!GATHER && warp == kGatherWarp2 && lane == 0 && a.q_pos == nullptr) {
    // Until the lengths are visible the CTA cannot know its first items; it
    // guesses them from full-capacity segments (exact when every sequence
    // is full) and prefetches their rows and scales into L2, so that the
    // first tile loads after the prologue hit L2 instead of HBM.  The warp
    // that issues them has no other role in the scan and stays out of the
    // prologue's barriers (issuing the prefetches takes about a microsecond).
    const int ips = (a.capacity + a.R - 1) / a.R;
    const int64_t total = static_cast<int64_t>(a.n_segments) * ips;
    const int64_t b0 = total * blockIdx.x / gridDim.x, b1 = total * (blockIdx.x + 1) / gridDim.x;
    const int nsc = SEG ? 2 : 1;
    for (int64_t item = b0; item < b1 && item < b0 + 2; ++item) {
      const int seg = static_cast<int>(item / ips), it = static_cast<int>(item % ips);
      const int64_t row0 = static_cast<int64_t>(seg / a.n_groups) * a.capacity + static_cast<int64_t>(it) * a.R;
      const int rows = min(a.R, a.capacity - it * a.R);
      prefetch_l2_bulk(a.cache_data + row0 * a.row_bytes, static_cast<uint32_t>(rows * a.row_bytes));
      if (a.cache_scale) prefetch_l2_bulk(a.cache_scale + row0 * nsc, static_cast<uint32_t>(rows * 4 * nsc));
    }
  }
  // everything above touches only this CTA's own resources; the lengths,
  // queries and cache rows below may come from the previous kernel
  pdl_begin();
  // Items per segment, then an exclusive prefix over segments (the scan:
  // every warp but the prefetching one; the gather: all of them).
  constexpr int kPrologueThreads = GATHER ? kScanThreads : kScanThreads - 32;
  const bool in_prologue = GATHER || warp != kGatherWarp2;
  auto prologue_sync = [in_prologue] {
    if constexpr (GATHER) {
      __syncthreads();
    } else {
      if (in_prologue) named_bar_sync(1, kPrologueThreads);   // the prefetching warp does not take part
    }
  };
  for (int i = tid; i < a.n_segments && tid < kPrologueThreads; i += kPrologueThreads) {
    s.prefix[i + 1] = segment_items<GATHER>(a, i);
    if (GATHER) {
      int n = a.cand_n[i];
      s.seg_n[i] = n < 0 ? 0 : (n > a.cand_stride ? a.cand_stride : n);
      int len = a.lengths[i / a.T];
      s.seg_len[i] = len < 0 ? 0 : (len > a.capacity ? a.capacity : len);
    }
  }
  prologue_sync();
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
  prologue_sync();
  tc_fence_after();

  // Every scalar argument is copied into registers once: the argument block
  // is addressable (the tensor maps are read through their addresses), so a
  // field read after an asm statement with a memory clobber would otherwise
  // be reloaded from parameter memory.
  const int k_capacity = a.capacity, k_T = a.T, k_H = a.H, k_H_pad = a.H_pad, k_Qg = a.Qg, k_N = a.N;
  const int k_cand_stride = a.cand_stride, k_swz = a.swz, k_n_kchunks = a.n_kchunks;
  const int k_R = a.R, k_MB = a.MB, k_KS = a.KS, k_spi = a.stages_per_item;
  const int k_RI = GATHER ? a.RI : a.R;      // rows an item covers (gather: fewer than the M block)
  const bool k_tail64 = GATHER && a.tail64;   // gathered rows end in a 64-byte chunk (map_a2)
  const uint32_t k_a_stage_bytes = a.a_stage_bytes, k_b_slot_bytes = a.b_slot_bytes, k_idesc = a.idesc;
  const uint32_t k_meta_bytes = a.meta_bytes;
  const int64_t k_score_stride = a.score_stride;
  const float* const k_cache_scale = a.cache_scale;
  // SEG: two scales per row (segmented fp8), two accumulators per (slot, M block)
  const int k_SK = SEG ? a.seg_kstep : 0;
  constexpr int k_nsc = SEG ? 2 : 1;
  const int* const k_lengths = a.lengths;
  const int* const k_q_pos = a.q_pos;
  const float* const k_w = a.w;
  const float* const k_q_scale = a.q_scale;
  const float* const k_beta = a.beta;
  const int* const k_cand = a.cand;
  const int* const k_cand_n = a.cand_n;
  float* const k_scores = a.scores;
  int* const k_status = a.status;
  uint64_t* const k_trace = a.trace;

  const int total = s.prefix[a.n_segments];
  const int begin = static_cast<int>((static_cast<int64_t>(total) * blockIdx.x) / gridDim.x);
  const int end = static_cast<int>((static_cast<int64_t>(total) * (blockIdx.x + 1)) / gridDim.x);
  const WaitCtl wc{s.abort_flag, k_status, a.wait_ns};
  const uint32_t tmem = *s.tmem_base;
  const uint32_t S = static_cast<uint32_t>(a.n_stages);
  const uint32_t NB = static_cast<uint32_t>(a.n_bslots);
  const uint32_t NA = static_cast<uint32_t>(a.n_acc);
  const uint32_t NM = static_cast<uint32_t>(a.n_meta);
  const int elt_per_chunk = k_swz / a.elt_bytes;
  const int n_groups = GATHER ? k_T : a.n_groups;
  const uint32_t chunk_region = static_cast<uint32_t>(k_R * k_swz);   // one K-chunk of a stage

  if (warp == 0 && !GATHER) {
    // ------------------------------------------------------------ loader (TMA), one lane
    if (lane == 0) {
      Ring st, bs, ms;
      uint32_t n_st = 0, n_bs = 0, n_ms = 0;
      SegWalk w{s.prefix, n_groups};
      bool first = true;
      uint32_t lt = 0;
      for (int item = begin; item < end; ++item, ++lt) {
        if (*s.abort_flag) break;
        const bool moved = w.to(item) || first;
        first = false;
        const int it = item - s.prefix[w.seg];   // item index within the segment
        // The item's first stage of rows goes first (the long HBM round
        // trip), then its queries and scales, then its other stages.  The
        // queries must precede the second stage: the MMA issuer cannot free
        // a stage of this item before it has them, and the ring may hold
        // fewer stages than an item has.
        const int row0 = w.b * k_capacity + it * k_R;
        auto load_stage = [&](int sp) -> bool {
          if (!bounded_wait(&s.empty[st.i], st.ph ^ 1u, wc)) return false;
          if (sp == 0) trace_event(k_trace, lt, 0);
          mbar_arrive_expect_tx(&s.full[st.i], k_a_stage_bytes);
          tma_load_3d(s.a_stages + static_cast<size_t>(st.i) * k_a_stage_bytes, &a.map_a, &s.full[st.i], 0, row0,
                      sp * k_KS);
          st.step(S);
          ++n_st;
          return true;
        };
        if (!load_stage(0)) break;
        if (moved) {
          if (!bounded_wait(&s.bempty[bs.i], bs.ph ^ 1u, wc)) break;
          mbar_arrive_expect_tx(&s.bfull[bs.i], k_b_slot_bytes);
          uint8_t* dst = s.b_slots + static_cast<size_t>(bs.i) * k_b_slot_bytes;
          const int z = w.b * k_T + w.g * k_Qg;
          for (int kc = 0; kc < k_n_kchunks; ++kc)
            tma_load_3d(dst + static_cast<size_t>(kc) * k_N * k_swz, &a.map_b, &s.bfull[bs.i],
                        kc * elt_per_chunk, 0, z);
          bs.step(NB);
          ++n_bs;
        }
        if (e4) {
          // the item's per-token scales, one bulk copy (rows past the
          // capacity are not read: the epilogue ignores them)
          if (!bounded_wait(&s.mempty[ms.i], ms.ph ^ 1u, wc)) break;
          const int rows = min(k_R, k_capacity - it * k_R);
          const uint32_t bytes = static_cast<uint32_t>(rows * k_nsc) * 4u;
          mbar_arrive_expect_tx(&s.mfull[ms.i], bytes);
          bulk_load(s.meta + static_cast<size_t>(ms.i) * k_meta_bytes,
                    k_cache_scale + (static_cast<int64_t>(w.b) * k_capacity + it * k_R) * k_nsc, bytes,
                    &s.mfull[ms.i]);
          ms.step(NM);
          ++n_ms;
        }
        bool ok = true;
        for (int sp = 1; sp < k_spi && ok; ++sp) ok = load_stage(sp);
        if (!ok) break;
        trace_event(k_trace, lt, 1);
      }
      if (*s.abort_flag) {
        // let every copy already issued land before the CTA exits
        drain_ring(s.full, S, n_st);
        drain_ring(s.bfull, NB, n_bs);
        drain_ring(s.mfull, NM, n_ms);
      }
    }
  } else if (warp == 0) {
    // ------------------------------------------------------------ loader (gather), 32 lanes
    // Per item: the lanes read the item's candidate ids (prefetched one item
    // ahead, coalesced), validate them against the segment's limits cached
    // in the prologue and publish token ids (and, with fp8, the rows' scales
    // by 4-byte cp.async) in the item's metadata slot.  The rows themselves
    // move by TMA row gathers, four rows of one K-chunk per instruction,
    // spread over the 32 lanes, into the [chunk][row] swizzled layout the
    // tiled load produces; a stage completes by its transaction count.
    // Invalid or padding candidates gather row 0 of the sequence; the
    // epilogue masks them.  All waits are warp-uniform.
    constexpr int kIdsPerLane = kMaxItemRows / 32;
    uint32_t n_st = 0, n_bs = 0;
    const int rows_per_lane = k_R >> 5;
    const int groups = k_RI >> 2;                  // 4-row gathers per K-chunk
    // bytes gathered per stage (the stage holding a 64-byte last chunk: 64 B less a row)
    const uint32_t stage_tx_full = static_cast<uint32_t>(k_RI * k_swz * k_KS);
    const uint32_t stage_tx_last = stage_tx_full - (k_tail64 ? static_cast<uint32_t>(k_RI * 64) : 0u);
    Ring st, bs, ms;
    SegWalk w{s.prefix, n_groups};
    SegWalk wn{s.prefix, n_groups};                // one item ahead
    bool first = true;
    int ids[kIdsPerLane];
    auto fetch_ids = [&](int item, SegWalk& ww, int (&out)[kIdsPerLane]) {
      ww.to(item);
      const int sg = ww.seg, itn = item - s.prefix[sg];
#pragma unroll
      for (int i = 0; i < kIdsPerLane; ++i) {
        out[i] = -1;
        const int r = lane + 32 * i;
        const int j = itn * k_RI + r;
        if (i < rows_per_lane && r < k_RI && j < k_cand_stride)
          out[i] = k_cand[static_cast<int64_t>(sg) * k_cand_stride + j];
      }
    };
    if (begin < end) fetch_ids(begin, wn, ids);
    for (int item = begin; item < end; ++item) {
      if (*s.abort_flag) break;
      const bool moved = w.to(item) || first;
      first = false;
      const int seg = w.seg, it = item - s.prefix[seg];
      if (moved) {
        if (!bounded_wait(&s.bempty[bs.i], bs.ph ^ 1u, wc)) break;
        if (lane == 0) {
          mbar_arrive_expect_tx(&s.bfull[bs.i], k_b_slot_bytes);
          uint8_t* dst = s.b_slots + static_cast<size_t>(bs.i) * k_b_slot_bytes;
          for (int kc = 0; kc < k_n_kchunks; ++kc)
            tma_load_3d(dst + static_cast<size_t>(kc) * k_N * k_swz, &a.map_b, &s.bfull[bs.i],
                        kc * elt_per_chunk, 0, seg);
        }
        bs.step(NB);
        ++n_bs;
      }
      int cur[kIdsPerLane];
#pragma unroll
      for (int i = 0; i < kIdsPerLane; ++i) cur[i] = ids[i];
      if (item + 1 < end) fetch_ids(item + 1, wn, ids);   // in flight while this item is issued
      const int len = s.seg_len[seg], cn = s.seg_n[seg];
      if (!bounded_wait(&s.mempty[ms.i], ms.ph ^ 1u, wc)) break;
      float* mscale = reinterpret_cast<float*>(s.meta + static_cast<size_t>(ms.i) * k_meta_bytes);
      int* mtok = reinterpret_cast<int*>(mscale + k_R * k_nsc);
      const int seq_row = w.b * k_capacity;
#pragma unroll
      for (int i = 0; i < kIdsPerLane; ++i) {
        if (i < rows_per_lane) {
          const int r = lane + 32 * i;
          const int j = it * k_RI + r;
          int t = (r < k_RI && j < cn) ? cur[i] : -1;
          if (j < cn && (t < 0 || t >= len)) t = -2;     // invalid candidate
          mtok[r] = t;
          if (e4) {
            const int64_t srow = seq_row + (t >= 0 ? t : 0);
            if constexpr (SEG) cp_async_8_zfill(smem_addr(mscale + 2 * r), k_cache_scale + 2 * srow, t >= 0 ? 8 : 0);
            else cp_async_4_zfill(smem_addr(mscale + r), k_cache_scale + srow, t >= 0 ? 4 : 0);
          }
        }
      }
      cp_async_arrive_noinc(&s.mfull[ms.i]);
      mbar_arrive(&s.mfull[ms.i]);
      __threadfence_block();                       // the token ids, for the second loader warp
      __syncwarp();
      ms.step(NM);
      bool ok = true;
      for (int sp = 0; sp < k_spi; ++sp) {
        if (!bounded_wait(&s.empty[st.i], st.ph ^ 1u, wc)) { ok = false; break; }
        if (lane == 0) {
          // both warps' copies land on it
          mbar_arrive_expect_tx(&s.full[st.i], sp == k_spi - 1 ? stage_tx_last : stage_tx_full);
          mbar_arrive(&s.ready[st.i]);
        }
        __syncwarp();
        const uint32_t stage = smem_addr(s.a_stages + static_cast<size_t>(st.i) * k_a_stage_bytes);
        // one TMA operation costs its issuing warp ~74 cycles: the second
        // loader warp issues the upper half of the stage's gathers
        for (int u = lane; u < (groups * k_KS + 1) / 2; u += 32) {
          const int c = u / groups, r0 = 4 * (u - c * groups);
          const int t0 = mtok[r0], t1 = mtok[r0 + 1], t2 = mtok[r0 + 2], t3 = mtok[r0 + 3];
          const bool tail = k_tail64 && sp * k_KS + c == k_n_kchunks - 1;
          tma_gather4(stage + static_cast<uint32_t>(c) * chunk_region + static_cast<uint32_t>(r0 * (tail ? 64 : k_swz)),
                      tail ? &a.map_a2 : &a.map_a, &s.full[st.i], (sp * k_KS + c) * elt_per_chunk,
                      seq_row + (t0 >= 0 ? t0 : 0), seq_row + (t1 >= 0 ? t1 : 0), seq_row + (t2 >= 0 ? t2 : 0),
                      seq_row + (t3 >= 0 ? t3 : 0));
        }
        st.step(S);
        ++n_st;
      }
      if (!ok) break;
    }
    if (*s.abort_flag) {
      // let every copy already issued land before the CTA exits
      cp_async_wait_all();
      if (lane == 0) {
        drain_ring(s.full, S, n_st);
        drain_ring(s.bfull, NB, n_bs);
      }
    }
  } else if (warp == kGatherWarp2) {
    // ------------------------------------------------------------ second gather loader, 32 lanes
    // Follows the first loader item by item and stage by stage: once a stage
    // is armed and the item's token ids are published (ready), it issues the
    // upper half of the stage's row gathers onto the same barrier.
    if constexpr (GATHER) {
      Ring st, ms;
      SegWalk w{s.prefix, n_groups};
      const int groups = k_RI >> 2;
      const int nops = groups * k_KS, half = (nops + 1) / 2;
      for (int item = begin; item < end; ++item) {
        if (*s.abort_flag) break;
        w.to(item);
        const int* mtok = reinterpret_cast<const int*>(
            reinterpret_cast<const float*>(s.meta + static_cast<size_t>(ms.i) * k_meta_bytes) + k_R * k_nsc);
        const int seq_row = w.b * k_capacity;
        bool ok = true;
        for (int sp = 0; sp < k_spi; ++sp) {
          if (!bounded_wait(&s.ready[st.i], st.ph, wc)) { ok = false; break; }
          const uint32_t stage = smem_addr(s.a_stages + static_cast<size_t>(st.i) * k_a_stage_bytes);
          for (int u = half + lane; u < nops; u += 32) {
            const int c = u / groups, r0 = 4 * (u - c * groups);
            const int t0 = mtok[r0], t1 = mtok[r0 + 1], t2 = mtok[r0 + 2], t3 = mtok[r0 + 3];
            const bool tail = k_tail64 && sp * k_KS + c == k_n_kchunks - 1;
            tma_gather4(stage + static_cast<uint32_t>(c) * chunk_region + static_cast<uint32_t>(r0 * (tail ? 64 : k_swz)),
                        tail ? &a.map_a2 : &a.map_a, &s.full[st.i], (sp * k_KS + c) * elt_per_chunk,
                        seq_row + (t0 >= 0 ? t0 : 0), seq_row + (t1 >= 0 ? t1 : 0), seq_row + (t2 >= 0 ? t2 : 0),
                        seq_row + (t3 >= 0 ? t3 : 0));
          }
          st.step(S);
        }
        if (!ok) break;
        ms.step(NM);
      }
    }
  } else if (warp == 1 || warp == kMmaWarp2) {
    // ------------------------------------------------------------ MMA issuers, one lane each
    // Issuer mi issues the MMAs of M block mi of every item (with one M
    // block per item only warp 1 works): each waits for the stage and for its
    // accumulator, issues and commits on its own, so the per-item waits and
    // the MMA issue of the two blocks overlap.
    const int mi = warp == 1 ? 0 : 1;
    if (lane == 0 && mi < k_MB) {
      Ring st, bs, acc;
      SegWalk w{s.prefix, n_groups};
      bool first = true;
      int slot = -1;
      uint32_t lt = 0;
      // K-major swizzled descriptors: everything but the start address is
      // fixed, so only the address field is added per MMA.
      const uint64_t desc_hi = make_smem_desc(0, static_cast<uint32_t>(k_swz));
      // a gathered row's 64-byte last chunk sits in a 64-byte-swizzled tile
      const uint64_t desc_hi64 = make_smem_desc(0, 64u);
      const uint32_t m_off = static_cast<uint32_t>(mi * 128 * k_swz);   // this M block within a chunk
      const uint32_t ksteps = static_cast<uint32_t>(k_swz >> 5);
      for (int item = begin; item < end; ++item, ++lt) {
        if (*s.abort_flag) break;
        const bool moved = w.to(item) || first;
        first = false;
        if (moved) {
          if (slot >= 0) umma_commit(&s.bempty[slot]);
          if (!bounded_wait(&s.bfull[bs.i], bs.ph, wc)) break;
          tc_fence_after();
          slot = static_cast<int>(bs.i);
          bs.step(NB);
        }
        uint64_t* accf = &s.accfull[2 * acc.i + mi];
        if (!bounded_wait(&s.accempty[2 * acc.i + mi], acc.ph ^ 1u, wc)) break;
        tc_fence_after();
        const uint32_t d0 = tmem + (acc.i * static_cast<uint32_t>(k_MB) + static_cast<uint32_t>(mi)) *
                                       static_cast<uint32_t>(k_N * k_nsc);
        const uint32_t b_base = smem_addr(s.b_slots + static_cast<size_t>(slot) * k_b_slot_bytes);
        bool ok = true;
        for (int sp = 0; sp < k_spi; ++sp) {
          if (sp == 0 && mi == 0) trace_event(k_trace, lt, 6);
          if (!bounded_wait(&s.full[st.i], st.ph, wc)) { ok = false; break; }
          if (sp == 0 && mi == 0) trace_event(k_trace, lt, 2);
          tc_fence_after();
          const uint32_t a_base = smem_addr(s.a_stages + static_cast<size_t>(st.i) * k_a_stage_bytes) + m_off;
          for (int c = 0; c < k_KS; ++c) {
            const int kc = sp * k_KS + c;
            const uint32_t a_c = a_base + static_cast<uint32_t>(c) * chunk_region;
            const uint32_t b_c = b_base + static_cast<uint32_t>(kc * k_N * k_swz);
            const bool tail = k_tail64 && kc == k_n_kchunks - 1;
            const int kst = tail ? 2 : static_cast<int>(ksteps);
            const uint64_t adh = tail ? desc_hi64 : desc_hi;
            if constexpr (!SEG) {
              issue_chunk_rt<KIND>(kst, 1, d0, a_c, b_c, adh, desc_hi, 0u, static_cast<uint32_t>(k_N), k_idesc, kc == 0);
            } else {
              // segmented scales: K steps before k_SK accumulate into the
              // first accumulator, the rest into the second (N columns on)
              const int g0 = kc * static_cast<int>(ksteps);
              const int n0 = max(0, min(kst, k_SK - g0));
              if (n0 > 0)
                issue_chunk_rt<KIND>(n0, 1, d0, a_c, b_c, adh, desc_hi, 0u, static_cast<uint32_t>(k_N), k_idesc,
                                     kc == 0);
              if (n0 < kst)
                issue_chunk_rt<KIND>(kst - n0, 1, d0 + static_cast<uint32_t>(k_N),
                                     a_c + static_cast<uint32_t>(n0) * 32u, b_c + static_cast<uint32_t>(n0) * 32u,
                                     adh, desc_hi, 0u, static_cast<uint32_t>(k_N), k_idesc, g0 + n0 == k_SK);
            }
          }
          umma_commit(&s.empty[st.i]);
          st.step(S);
        }
        if (!ok) break;
        umma_commit(accf);
        if (mi == 0) trace_event(k_trace, lt, 3);
        acc.step(NA);
      }
      if (*s.abort_flag) {
        umma_commit(&s.drain[mi]);
        drain_wait(&s.drain[mi], 0, kDrainNs);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    // Two warpgroups.  With two M blocks per item (R = 256) warpgroup g takes
    // block g of every item; with one (R = 128) they take alternate items.
    const int ew = warp - 2;                 // 0 .. kEpiWarps-1
    const int wg = ew >> 2;
    const int quad = warp & 3;               // TMEM lane quadrant this warp may access
    const int mb = k_MB == 2 ? wg : 0;
    const int istep = k_MB == 2 ? 1 : 2;
    const int r = mb * 128 + quad * 32 + lane;   // row of the item
    const bool has_beta = k_beta != nullptr;
    // per-warp parameters: folded weights; with a bias also the query scales
    // and the bias terms; then the valid lengths of the group's queries
    float* ep_w = s.ep + ew * a.ep_stride;
    float* ep_qs = ep_w + k_N;
    float* ep_beta = ep_qs + k_N;
    int* ep_len = reinterpret_cast<int*>(ep_w + (has_beta ? 3 * k_N : k_N));
    Ring acc, ms;
    const uint32_t first_item = k_MB == 2 ? 0u : static_cast<uint32_t>(wg);
    acc.i = first_item;                      // n_acc, n_meta >= 2
    ms.i = first_item;
    SegWalk w{s.prefix, n_groups};
    bool first = true;
    uint32_t lt = first_item;
    for (int item = begin + static_cast<int>(first_item); item < end; item += istep, lt += istep) {
      if (*s.abort_flag) break;
      const bool moved = w.to(item) || first;
      first = false;
      const int seg = w.seg, it = item - s.prefix[seg];
      const int b = w.b, g = w.g;
      if (moved) {
        int len = k_lengths[b];
        len = len < 0 ? 0 : (len > k_capacity ? k_capacity : len);
        __syncwarp();
        for (int qi = 0, i0 = 0; qi < k_Qg; ++qi, i0 += k_H_pad) {
          const int t = g * k_Qg + qi;
          for (int h = lane; h < k_H_pad; h += 32) {
            float wv = 0.f, qs = 1.f, be = 0.f;
            if (h < k_H && t < k_T) {
              const int64_t o = (static_cast<int64_t>(b) * k_T + t) * k_H + h;
              wv = k_w[o];
              if (k_q_scale) qs = k_q_scale[o];
              if (has_beta) be = k_beta[o];
            }
            // Without a bias, fold the query scale into the weight (ReLU is
            // positively homogeneous and the scales are positive).
            ep_w[i0 + h] = has_beta ? wv : wv * qs;
            if (has_beta) {
              ep_qs[i0 + h] = qs;
              ep_beta[i0 + h] = be;
            }
          }
        }
        if (lane < 16) {
          const int t = g * k_Qg + lane;
          int v = 0;
          if (lane < k_Qg && t < k_T) {
            if (GATHER) {
              v = k_cand_n[seg];
              v = v < 0 ? 0 : (v > k_cand_stride ? k_cand_stride : v);
            } else {
              v = len;
              if (k_q_pos) {
                int p = k_q_pos[b * k_T + t] + 1;
                v = p < 0 ? 0 : (p > len ? len : p);
              }
            }
          }
          ep_len[lane] = v;
        }
        __syncwarp();
      }
      const int j = it * k_RI + r;          // position (scan) or candidate slot (gather)
      const bool row_in_item = !GATHER || r < k_RI;
      int tok = j;
      float cs = 1.f, cs1 = 0.f;
      if (has_meta) {
        if (!bounded_wait(&s.mfull[ms.i], ms.ph, wc)) break;
        const float* mscale = reinterpret_cast<const float*>(s.meta + static_cast<size_t>(ms.i) * k_meta_bytes);
        if (GATHER) tok = reinterpret_cast<const int*>(mscale + k_R * k_nsc)[r];
        // rows past the valid prefix read stale values, unused
        if (e4 && tok >= 0) {
          if constexpr (SEG) {
            cs = mscale[2 * r];
            cs1 = mscale[2 * r + 1];
          } else {
            cs = mscale[r];
          }
        }
      }
      if (!bounded_wait(&s.accfull[2 * acc.i + mb], acc.ph, wc)) break;
      if (lane == 0 && (ew & 3) == 0) trace_event(k_trace, lt, 4);
      tc_fence_after();

      const uint32_t tbase = tmem + (static_cast<uint32_t>(quad * 32) << 16) +
                             (acc.i * static_cast<uint32_t>(k_MB) + static_cast<uint32_t>(mb)) *
                                 static_cast<uint32_t>(k_N * k_nsc);
      // segmented scales: head h's product is cs * D0_h + cs1 * D1_h, formed
      // per head before the ReLU (no division: a zero scale stays finite);
      // with one scale per row it is taken outside the head sum instead
      const bool scale_after = !has_beta && e4 && !SEG;
      // One score: the head sums of query row qi from its HP columns at vq,
      // in the same order as the per-query loop below (so results agree bit
      // for bit whichever path runs), then the store.
      auto finish = [&](int qi, const float* vq, auto hp) {
        constexpr int HP = decltype(hp)::value;
        const int t = g * k_Qg + qi;
        float part[4] = {0.f, 0.f, 0.f, 0.f};
        const float* wq = ep_w + qi * k_H_pad;
        const float* qs = ep_qs + qi * k_H_pad;
        const float* be = ep_beta + qi * k_H_pad;
#pragma unroll
        for (int h0 = 0; h0 < HP; h0 += 16) {
          if (!has_beta) relu_dot16_pk(vq + h0, wq + h0, part);
          else relu_dot16_beta(vq + h0, wq + h0, qs + h0, be + h0, cs, part);
        }
        float sc = (part[0] + part[1]) + (part[2] + part[3]);
        if (scale_after) sc *= cs;
        if (row_in_item && j < ep_len[qi]) {
          if (GATHER && tok < 0) {
            sc = -INFINITY;
            record_status(k_status, kStatusIndex);
          }
          const int64_t row = static_cast<int64_t>(b) * k_T + t;
          k_scores[row * k_score_stride + j] = sc;
        }
      };
      // Several query rows per item (prefill, a stacked group): their columns
      // come 64 at a time under one wait, since the epilogue is then bound by
      // the latency of tensor-memory loads rather than by arithmetic.
      // (MQ: Qg > 1, H_pad of 16, 32 or 64, N a multiple of 64, no segments)
      if constexpr (MQ) {
        {
          for (int q0 = 0; q0 < k_Qg && g * k_Qg + q0 < k_T; q0 += 64 / k_H_pad) {
            float v[64];
            tmem_load64_sync(tbase + static_cast<uint32_t>(q0 * k_H_pad), v);
            const int nq = min(64 / k_H_pad, k_T - (g * k_Qg + q0));
            if (k_H_pad == 64) {
              finish(q0, v, std::integral_constant<int, 64>{});
            } else if (k_H_pad == 32) {
              finish(q0, v, std::integral_constant<int, 32>{});
              if (nq > 1) finish(q0 + 1, v + 32, std::integral_constant<int, 32>{});
            } else {
#pragma unroll
              for (int u = 0; u < 4; ++u)
                if (u < nq) finish(q0 + u, v + 16 * u, std::integral_constant<int, 16>{});
            }
          }
        }
      }
      for (int qi = 0; qi < k_Qg && !MQ; ++qi) {
        const int t = g * k_Qg + qi;
        if (t >= k_T) break;
        float part[4] = {0.f, 0.f, 0.f, 0.f};
        const float* wq = ep_w + qi * k_H_pad;
        const float* qs = ep_qs + qi * k_H_pad;
        const float* be = ep_beta + qi * k_H_pad;
        int h0 = 0;
        if constexpr (SEG) {
          for (; h0 + 16 <= k_H_pad; h0 += 16) {
            float v[16], v1[16];
            tmem_load16x2_sync(tbase + static_cast<uint32_t>(qi * k_H_pad + h0),
                               tbase + static_cast<uint32_t>(k_N + qi * k_H_pad + h0), v, v1);
            if (!has_beta) {
#pragma unroll
              for (int e = 0; e < 16; ++e) v[e] = fmaf(cs1, v1[e], cs * v[e]);
              relu_dot16(v, wq + h0, part);
            } else {
#pragma unroll
              for (int e = 0; e < 16; ++e) v[e] = fmaf(cs1, v1[e], cs * v[e]);
              relu_dot16_beta(v, wq + h0, qs + h0, be + h0, 1.f, part);
            }
          }
        }
        for (; h0 + 32 <= k_H_pad; h0 += 32) {
          float v[32];
          tmem_load32_sync(tbase + static_cast<uint32_t>(qi * k_H_pad + h0), v);
          if (!has_beta) {
            relu_dot16(v, wq + h0, part);
            relu_dot16(v + 16, wq + h0 + 16, part);
          } else {
            relu_dot16_beta(v, wq + h0, qs + h0, be + h0, cs, part);
            relu_dot16_beta(v + 16, wq + h0 + 16, qs + h0 + 16, be + h0 + 16, cs, part);
          }
        }
        if (h0 < k_H_pad) {   // H_pad % 32 == 16
          float v[16];
          tmem_load16_sync(tbase + static_cast<uint32_t>(qi * k_H_pad + h0), v);
          if (!has_beta) relu_dot16(v, wq + h0, part);
          else relu_dot16_beta(v, wq + h0, qs + h0, be + h0, cs, part);
        }
        if (qi == 0 && lane == 0 && (ew & 3) == 0) trace_event(k_trace, lt, 7);
        float sc = (part[0] + part[1]) + (part[2] + part[3]);
        if (scale_after) sc *= cs;
        if (row_in_item && j < ep_len[qi]) {
          if (GATHER && tok < 0) {
            sc = -INFINITY;
            record_status(k_status, kStatusIndex);
          }
          const int64_t row = static_cast<int64_t>(b) * k_T + t;
          k_scores[row * k_score_stride + j] = sc;
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if ((ew & 3) == 0) trace_event(k_trace, lt, 5);
        mbar_arrive(&s.accempty[2 * acc.i + mb]);
        if (has_meta) mbar_arrive(&s.mempty[ms.i]);
      }
      acc.step_by(static_cast<uint32_t>(istep), NA);
      if (has_meta) ms.step_by(static_cast<uint32_t>(istep), NM);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, a.tmem_cols);
}

template <int KIND, bool GATHER, bool SEG = false>
cudaError_t launch_one(const ScanArgs& a, int grid, cudaStream_t st) {
  // several query rows per item with head groups of 16, 32 or 64: the
  // epilogue variant that reads 64 columns per tensor-memory wait
  if constexpr (!GATHER && !SEG) {
    if (a.Qg > 1 && (a.H_pad == 16 || a.H_pad == 32 || a.H_pad == 64) && a.N % 64 == 0) {
      auto k = scan_kernel<KIND, false, false, true>;
      const cudaError_t e = raise_smem_limit(reinterpret_cast<const void*>(k), a.smem_bytes);
      if (e != cudaSuccess) return e;
      return launch_pdl(k, dim3(grid), dim3(kScanThreads), a.smem_bytes, st, 1, a);
    }
  }
  auto k = scan_kernel<KIND, GATHER, SEG, false>;
  const cudaError_t e = raise_smem_limit(reinterpret_cast<const void*>(k), a.smem_bytes);
  if (e != cudaSuccess) return e;
  return launch_pdl(k, dim3(grid), dim3(kScanThreads), a.smem_bytes, st, 1, a);
}

}  // namespace

cudaError_t launch_scan_kernel(int kind, bool gather, const ScanArgs& a, int grid, cudaStream_t st) {
  switch (kind * 2 + (gather ? 1 : 0)) {
    case kKindTF32 * 2: return launch_one<kKindTF32, false>(a, grid, st);
    case kKindTF32 * 2 + 1: return launch_one<kKindTF32, true>(a, grid, st);
    case kKindBF16 * 2: return launch_one<kKindBF16, false>(a, grid, st);
    case kKindBF16 * 2 + 1: return launch_one<kKindBF16, true>(a, grid, st);
    case kKindE4M3 * 2:
      return a.seg_kstep > 0 ? launch_one<kKindE4M3, false, true>(a, grid, st) : launch_one<kKindE4M3, false>(a, grid, st);
    case kKindE4M3 * 2 + 1:
      return a.seg_kstep > 0 ? launch_one<kKindE4M3, true, true>(a, grid, st) : launch_one<kKindE4M3, true>(a, grid, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace li
