// api.cu -- the extern "C" entry points declared in include/li.h: argument
// validation, workspace layout, TMA descriptor encoding and the launch
// sequence of every operation.  Host state lives in li_ctx; the library
// allocates no device memory.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#include "internal.h"
#include "sm100.cuh"

using namespace li;

namespace li {

cudaError_t raise_smem_limit(const void* fn, int bytes) {
  struct Entry {
    const void* fn;
    int device;
    int bytes;
  };
  static std::mutex mu;
  static std::vector<Entry> done;
  int device = 0;
  cudaError_t e = cudaGetDevice(&device);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  for (const Entry& x : done)
    if (x.fn == fn && x.device == device && x.bytes >= bytes) return cudaSuccess;
  e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e != cudaSuccess) {
    (void)cudaGetLastError();
    return e;
  }
  for (Entry& x : done)
    if (x.fn == fn && x.device == device) {
      x.bytes = bytes;
      return cudaSuccess;
    }
  done.push_back({fn, device, bytes});
  return cudaSuccess;
}

}  // namespace li

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

struct ProfRec {
  std::string name;
  cudaEvent_t beg, end;
  int grid, block, smem;
};

struct ScanPlan {
  ScanArgs a;
  int kind;
  int grid;
};

// Everything a scan plan depends on (zero-filled, compared bytewise).
struct PlanKey {
  const void* data;
  const float* scale;
  const int32_t* lengths;
  const void* q;
  const float* q_scale;
  const float* beta;
  const float* w;
  const int32_t* q_pos;
  const uint64_t* trace;
  uint64_t wait_ns;
  int32_t batch, capacity, dim, dtype;
  int32_t q_dtype, T, H, gather;
  int32_t cand_stride, scale_split;
};

struct li_ctx {
  int device = 0;
  int num_sms = 0;
  int max_smem_optin = 0;
  // resident clusters of the single-launch selection, by cluster size 1..16
  int cluster_cap[17] = {};
  EncodeTiledFn encode = nullptr;
  std::string last_error;
  uint64_t wait_ns = 2000000000ull;
  bool profile = false;
  uint64_t* trace = nullptr;
  std::vector<ProfRec> prof;
  std::vector<cudaEvent_t> free_events;
  // Recently built scan plans (tensor maps included): a decode loop calls
  // the same entry points on the same buffers every step.
  static constexpr int kPlanCache = 16;
  PlanKey plan_key[kPlanCache] = {};
  ScanPlan plan_val[kPlanCache];
  bool plan_used[kPlanCache] = {};
  int plan_next = 0;
};

namespace {

li_status fail(li_ctx* ctx, li_status s, const char* fmt, ...) {
  if (ctx) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof(buf), fmt, ap);
    va_end(ap);
    ctx->last_error = buf;
  }
  return s;
}

li_status cuda_fail(li_ctx* ctx, cudaError_t e, const char* what) {
  return fail(ctx, LI_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int elt_bytes(li_dtype d) { return d == LI_F32 ? 4 : (d == LI_BF16 ? 2 : 1); }

size_t up256(size_t x) { return (x + 255) & ~size_t(255); }

// ------------------------------------------------------------------ workspace

struct WsLayout {
  size_t status = 0, done = 64, hist, rowinfo, chunk_gt, chunk_off, cand, scores, cand_scores, tmp, total;
  int n_chunks;
};

constexpr int kAppendChunkTok = 8192;

WsLayout ws_layout(int64_t rows, int64_t n, int64_t B) {
  WsLayout L;
  size_t off = 256;
  auto take = [&](size_t bytes) { size_t o = off; off += up256(bytes); return o; };
  const int64_t nn = std::max<int64_t>(std::max<int64_t>(n, B), 1);
  L.n_chunks = static_cast<int>((nn + kTopkChunk - 1) / kTopkChunk);
  L.hist = take(rows * kHistBins * 4);
  L.rowinfo = take(rows * 16 * 4);
  L.chunk_gt = take(rows * L.n_chunks * 4);
  L.chunk_off = take(rows * L.n_chunks * 4);
  L.cand = take(rows * nn * 8);
  L.scores = take(rows * nn * 4);
  L.cand_scores = take(rows * std::max<int64_t>(B, 1) * 4);
  L.tmp = take(static_cast<size_t>(kAppendChunkTok) * 256 * 4);
  L.total = off;
  return L;
}

template <typename T>
T* at(void* ws, size_t off) { return reinterpret_cast<T*>(static_cast<uint8_t*>(ws) + off); }

// ------------------------------------------------------------------ profiling

cudaEvent_t get_event(li_ctx* c) {
  if (!c->free_events.empty()) {
    cudaEvent_t e = c->free_events.back();
    c->free_events.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  cudaEventCreate(&e);
  return e;
}

struct Launch {
  li_ctx* c;
  cudaStream_t st;
  const char* name;
  int grid, block, smem;
  cudaEvent_t beg = nullptr;
  Launch(li_ctx* c_, cudaStream_t st_, const char* name_, int grid_, int block_, int smem_)
      : c(c_), st(st_), name(name_), grid(grid_), block(block_), smem(smem_) {
    if (c->profile) {
      beg = get_event(c);
      cudaEventRecord(beg, st);
    }
  }
  void done() {
    if (c->profile && beg) {
      cudaEvent_t end = get_event(c);
      cudaEventRecord(end, st);
      c->prof.push_back(ProfRec{name, beg, end, grid, block, smem});
    }
  }
};

// ------------------------------------------------------------------ validation

li_status check_cache(li_ctx* ctx, const li_cache* c, const char* what) {
  if (!c) return fail(ctx, LI_ERR_ARG, "%s: cache is NULL", what);
  if (!c->data || !c->lengths) return fail(ctx, LI_ERR_ARG, "%s: cache data/lengths is NULL", what);
  if (c->dtype != LI_F32 && c->dtype != LI_BF16 && c->dtype != LI_E4M3)
    return fail(ctx, LI_ERR_DTYPE, "%s: unknown cache dtype %d", what, static_cast<int>(c->dtype));
  if (c->dtype == LI_E4M3 && !c->scale) return fail(ctx, LI_ERR_ARG, "%s: E4M3 cache needs a scale array", what);
  if (c->batch < 1 || c->capacity < 1) return fail(ctx, LI_ERR_SHAPE, "%s: batch and capacity must be >= 1", what);
  if (static_cast<int64_t>(c->batch) * c->capacity >= (int64_t(1) << 31))
    return fail(ctx, LI_ERR_SHAPE, "%s: batch * capacity must be < 2^31", what);
  const int kmul = c->dtype == LI_F32 ? 8 : (c->dtype == LI_BF16 ? 16 : 32);
  if (c->dim < kmul || c->dim > 256 || c->dim % kmul)
    return fail(ctx, LI_ERR_SHAPE, "%s: dim %d must be a multiple of %d in [%d, 256]", what, c->dim, kmul, kmul);
  if (!aligned(c->data, 16)) return fail(ctx, LI_ERR_ALIGN, "%s: cache data not 16-byte aligned", what);
  if (c->scale && !aligned(c->scale, 16)) return fail(ctx, LI_ERR_ALIGN, "%s: scale not 16-byte aligned", what);
  if (c->scale_split != 0) {
    if (c->dtype != LI_E4M3)
      return fail(ctx, LI_ERR_ARG, "%s: scale_split is only for E4M3 caches (got %d)", what, c->scale_split);
    if (c->scale_split < 0 || c->scale_split >= c->dim || c->scale_split % 32)
      return fail(ctx, LI_ERR_SHAPE, "%s: scale_split %d must be a multiple of 32 in (0, dim = %d)", what,
                  c->scale_split, c->dim);
  }

  return LI_OK;
}

li_status check_query(li_ctx* ctx, const li_cache* c, const li_query* q, const char* what) {
  if (!q) return fail(ctx, LI_ERR_ARG, "%s: query is NULL", what);
  if (!q->q || !q->w) return fail(ctx, LI_ERR_ARG, "%s: q and w must be non-NULL", what);
  if (q->dtype != c->dtype)
    return fail(ctx, LI_ERR_DTYPE, "%s: query dtype %d must match the cache dtype %d", what,
                static_cast<int>(q->dtype), static_cast<int>(c->dtype));
  if (q->dtype == LI_E4M3 && !q->q_scale) return fail(ctx, LI_ERR_ARG, "%s: E4M3 query needs q_scale", what);
  if (q->H < 1 || q->H > 256) return fail(ctx, LI_ERR_SHAPE, "%s: H = %d must be in [1, 256]", what, q->H);
  if (q->T < 1) return fail(ctx, LI_ERR_SHAPE, "%s: T must be >= 1", what);
  if (static_cast<int64_t>(c->batch) * q->T >= (int64_t(1) << 31))
    return fail(ctx, LI_ERR_SHAPE, "%s: batch * T too large", what);
  if (!aligned(q->q, 16)) return fail(ctx, LI_ERR_ALIGN, "%s: q not 16-byte aligned", what);
  return LI_OK;
}

li_status check_ws(li_ctx* ctx, void* ws, size_t ws_bytes, const WsLayout& L, const char* what) {
  if (!ws) return fail(ctx, LI_ERR_WORKSPACE, "%s: workspace is NULL", what);
  if (!aligned(ws, 256)) return fail(ctx, LI_ERR_WORKSPACE, "%s: workspace not 256-byte aligned", what);
  if (ws_bytes < L.total)
    return fail(ctx, LI_ERR_WORKSPACE, "%s: workspace of %zu bytes, %zu needed", what, ws_bytes, L.total);
  return LI_OK;
}

// ------------------------------------------------------------------ tensor maps

// Tiled loads stream whole rows and use 256-byte L2 promotion; row gathers
// read scattered rows and ask for none (promotion would pull in neighbouring
// sectors of every gathered row).
li_status encode_map(li_ctx* ctx, CUtensorMap* m, li_dtype dt, int rank, void* base, const cuuint64_t* dims,
                     const cuuint64_t* strides, const cuuint32_t* box, int swz, bool promote = true) {
  const CUtensorMapDataType t = dt == LI_F32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
                                : dt == LI_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                                : CU_TENSOR_MAP_DATA_TYPE_UINT8;
  const CUtensorMapSwizzle sw = swz == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                                : swz == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                            : CU_TENSOR_MAP_SWIZZLE_32B;
  const cuuint32_t es[3] = {1, 1, 1};
  const CUresult r = ctx->encode(m, t, rank, base, dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                                 promote ? CU_TENSOR_MAP_L2_PROMOTION_L2_256B : CU_TENSOR_MAP_L2_PROMOTION_NONE,
                                 CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(ctx, LI_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
  return LI_OK;
}

// ------------------------------------------------------------------ scan plan


li_status plan_scan_build(li_ctx* ctx, const li_cache* c, const li_query* q, bool gather, int cand_stride,
                          ScanPlan* P, const char* what);

// The plan of a scan launch, from the context's cache when the same buffers
// and shapes were planned before (the tensor maps hold the buffer addresses).
li_status plan_scan(li_ctx* ctx, const li_cache* c, const li_query* q, bool gather, int cand_stride,
                    ScanPlan* P, const char* what) {
  PlanKey k;
  memset(&k, 0, sizeof(k));
  k.data = c->data;
  k.scale = c->scale;
  k.lengths = c->lengths;
  k.q = q->q;
  k.q_scale = q->q_scale;
  k.beta = q->beta;
  k.w = q->w;
  k.q_pos = q->q_pos;
  k.trace = ctx->trace;
  k.wait_ns = ctx->wait_ns;
  k.batch = c->batch;
  k.capacity = c->capacity;
  k.dim = c->dim;
  k.dtype = static_cast<int32_t>(c->dtype);
  k.q_dtype = static_cast<int32_t>(q->dtype);
  k.T = q->T;
  k.H = q->H;
  k.gather = gather ? 1 : 0;
  k.cand_stride = cand_stride;
  k.scale_split = c->scale_split;
  for (int i = 0; i < li_ctx::kPlanCache; ++i)
    if (ctx->plan_used[i] && memcmp(&ctx->plan_key[i], &k, sizeof(k)) == 0) {
      *P = ctx->plan_val[i];
      return LI_OK;
    }
  li_status s = plan_scan_build(ctx, c, q, gather, cand_stride, P, what);
  if (s != LI_OK) return s;
  const int slot = ctx->plan_next;
  ctx->plan_next = (slot + 1) % li_ctx::kPlanCache;
  ctx->plan_key[slot] = k;
  ctx->plan_val[slot] = *P;
  ctx->plan_used[slot] = true;
  return LI_OK;
}

li_status plan_scan_build(li_ctx* ctx, const li_cache* c, const li_query* q, bool gather, int cand_stride,
                          ScanPlan* P, const char* what) {
  ScanArgs& a = P->a;
  memset(&a, 0, sizeof(a));
  const int eb = elt_bytes(c->dtype);
  const int64_t row_bytes = static_cast<int64_t>(c->dim) * eb;
  int swz = row_bytes % 128 == 0 ? 128 : (row_bytes % 64 == 0 ? 64 : 32);
  int n_kchunks = static_cast<int>(row_bytes / swz);
  bool tail64 = false;
  if (gather && swz < 128 && row_bytes > 128) {
    // Row gathers are bound by the number of TMA operations, so gather whole
    // 128-byte chunks: K is padded to a multiple of 128 bytes, and the bytes
    // past the row's end lie outside both tensor maps and arrive as zeros
    // (cache and queries alike), which adds exact zeros to every product.
    // A row of 128 m + 64 bytes (the e4m3 latent: 192) gathers its last 64
    // bytes by a second map with a 64-byte box, into a 64-byte-swizzled tile:
    // as many operations, and no bytes read past the row.
    swz = 128;
    n_kchunks = static_cast<int>((row_bytes + 127) / 128);
    tail64 = row_bytes % 128 == 64;
  }
  // segmented fp8: two scales per row and two accumulators per item, so at
  // most 128 MMA columns per accumulator
  const int nsc = c->dtype == LI_E4M3 && c->scale_split > 0 ? 2 : 1;
  const int H_pad = (q->H + 15) / 16 * 16;
  if (H_pad * nsc > 256)
    return fail(ctx, LI_ERR_UNSUPPORTED, "%s: H = %d exceeds %d heads with segmented scales", what, q->H, 256 / nsc);
  const int Qg = gather ? 1 : std::max(1, std::min(256 / nsc / H_pad, q->T));
  const int N = Qg * H_pad;
  const int n_groups = (q->T + Qg - 1) / Qg;
  const int n_seg = gather ? c->batch * q->T : c->batch * n_groups;
  if (n_seg > kMaxSegments)
    return fail(ctx, LI_ERR_UNSUPPORTED, "%s: %d segments (batch x query groups) exceed %d", what, n_seg,
                kMaxSegments);
  a.batch = c->batch;
  a.capacity = c->capacity;
  a.T = q->T;
  a.H = q->H;
  a.H_pad = H_pad;
  a.Qg = Qg;
  a.n_groups = n_groups;
  a.N = N;
  a.n_segments = n_seg;
  a.swz = swz;
  a.elt_bytes = eb;
  a.n_kchunks = n_kchunks;
  a.row_bytes = row_bytes;
  a.cand_stride = cand_stride;
  const int kind = c->dtype == LI_F32 ? kKindTF32 : (c->dtype == LI_BF16 ? kKindBF16 : kKindE4M3);
  const uint32_t fmt = c->dtype == LI_F32 ? 2u : (c->dtype == LI_BF16 ? 1u : 0u);
  a.idesc = make_instr_desc(fmt, 128, N);
  a.b_slot_bytes = static_cast<uint32_t>(a.n_kchunks) * N * swz;
  // Work item of R rows (two M=128 blocks when both accumulators of every
  // in-flight item fit tensor memory), stage of KS K-chunks.  Among the
  // layouts that fit, the one with the deepest pipeline wins: items in
  // flight = min(stages / stages_per_item, metadata slots - 2), so the
  // metadata ring never throttles the stage ring; then more query slots.
  const bool has_meta = gather || c->dtype == LI_E4M3;
  const int ep_stride = (q->beta ? 3 * N : N) + 16;
  // barriers (3 x kMaxStages + 2 + 2 + 8 + 8 + 2 x kMetaSlots + 2) x 8 B,
  // tensor-memory base, abort flag, prefix, epilogue parameters, gather limits
  const size_t fixed_misc = static_cast<size_t>(3 * kMaxStages + 22 + 2 * kMetaSlots) * 8 + 16 +
                            static_cast<size_t>(n_seg + 1) * 4 + 16 + static_cast<size_t>(kEpiWarps) * ep_stride * 4 +
                            (gather ? static_cast<size_t>(2 * n_seg) * 4 : 0) + 64;
  const size_t budget = static_cast<size_t>(ctx->max_smem_optin) - 1024;
  const size_t kStageCap = 48 * 1024;
  bool planned = false;
  for (int R = (2 * N * nsc <= 256 && !gather) ? 256 : 128; R >= 128 && !planned; R -= 128) {
    // metadata slot: R x nsc scales, then (gather) R token ids
    const uint32_t meta_bytes = has_meta ? static_cast<uint32_t>((4 * nsc + (gather ? 4 : 0)) * R) : 0u;
    for (int KS = a.n_kchunks; KS >= 1 && !planned; --KS) {
      if (a.n_kchunks % KS) continue;
      const size_t stage = static_cast<size_t>(R) * swz * KS;
      if (stage > kStageCap && KS > 1) continue;
      const int spi = a.n_kchunks / KS;
      const int need = KS < a.n_kchunks ? 4 : 3;
      // Two query slots let a CTA whose items cross into the next segment
      // load its queries ahead; one slot is taken only with a single segment
      // (or when two leave no room for the minimum ring).
      int best_depth = -1, best_stages = 0, best_bslots = 0, best_meta = 0;
      for (int bslots = 2; bslots >= 1; --bslots) {
        if (bslots == 1 && n_seg > 1 && best_stages >= need) break;
        for (int nm = has_meta ? kMetaSlots : 0; nm >= (has_meta ? 4 : 0); --nm) {
          const int64_t room = static_cast<int64_t>(budget) - static_cast<int64_t>(bslots) * a.b_slot_bytes -
                               static_cast<int64_t>(nm) * meta_bytes - static_cast<int64_t>(fixed_misc);
          const int stages = room > 0 ? static_cast<int>(std::min<int64_t>(kMaxStages, room / stage)) : 0;
          // stages the metadata ring lets the loader run ahead
          const int depth = has_meta ? std::min(stages, (nm - 2) * spi) : stages;
          if (depth > best_depth) {
            best_depth = depth;
            best_stages = stages;
            best_bslots = bslots;
            best_meta = nm;
          }
          if (!has_meta) break;
        }
      }
      if (best_stages < need) continue;
      a.R = R;
      a.MB = R / 128;
      a.KS = KS;
      a.stages_per_item = spi;
      a.n_stages = best_stages;
      a.n_bslots = best_bslots;
      a.n_meta = best_meta;
      a.ep_stride = ep_stride;
      a.a_stage_bytes = static_cast<uint32_t>(stage);
      a.meta_bytes = meta_bytes;
      a.misc_offset = static_cast<uint32_t>(best_stages * stage + best_bslots * a.b_slot_bytes +
                                            static_cast<size_t>(best_meta) * meta_bytes);
      a.smem_bytes = static_cast<uint32_t>(std::max<size_t>(1024 + a.misc_offset + fixed_misc, 120 * 1024));
      planned = true;
    }
  }
  if (!planned || a.smem_bytes > static_cast<uint32_t>(ctx->max_smem_optin))
    return fail(ctx, LI_ERR_UNSUPPORTED, "%s: operands too large for shared memory (N=%d, dim=%d)", what, N, c->dim);
  a.n_acc = std::min(4, 512 / (a.MB * N * nsc));
  a.seg_kstep = nsc == 2 ? c->scale_split / 32 : 0;
  uint32_t cols = 32;
  while (cols < static_cast<uint32_t>(a.n_acc * a.MB * N * nsc)) cols <<= 1;
  a.tmem_cols = cols;
  a.wait_ns = ctx->wait_ns;
  a.trace = ctx->trace;

  // Tensor maps: cache rows as {chunk elements, rows, chunks} so that one
  // box carries all KS chunks of R rows in [chunk][row] order, and queries.
  if (gather) {
    // rows gathered four at a time: a 2-D map whose box is one row high
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(c->dim), static_cast<cuuint64_t>(c->batch) * c->capacity};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(row_bytes)};
    const cuuint32_t box[2] = {static_cast<cuuint32_t>(swz / eb), 1};
    li_status s = encode_map(ctx, &a.map_a, c->dtype, 2, c->data, dims, strides, box, swz, false);
    if (s != LI_OK) return s;
    if (tail64) {
      const cuuint32_t box2[2] = {static_cast<cuuint32_t>(64 / eb), 1};
      s = encode_map(ctx, &a.map_a2, c->dtype, 2, c->data, dims, strides, box2, 64, false);
      if (s != LI_OK) return s;
      a.tail64 = 1;
    }
  } else {
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(swz / eb), static_cast<cuuint64_t>(c->batch) * c->capacity,
                                static_cast<cuuint64_t>(a.n_kchunks)};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(row_bytes), static_cast<cuuint64_t>(swz)};
    const cuuint32_t box[3] = {static_cast<cuuint32_t>(swz / eb), static_cast<cuuint32_t>(a.R),
                               static_cast<cuuint32_t>(a.KS)};
    li_status s = encode_map(ctx, &a.map_a, c->dtype, 3, c->data, dims, strides, box, swz);
    if (s != LI_OK) return s;
  }
  {
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(c->dim), static_cast<cuuint64_t>(q->H),
                                static_cast<cuuint64_t>(c->batch) * q->T};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(row_bytes),
                                   static_cast<cuuint64_t>(row_bytes) * q->H};
    const cuuint32_t box[3] = {static_cast<cuuint32_t>(swz / eb), static_cast<cuuint32_t>(H_pad),
                               static_cast<cuuint32_t>(Qg)};
    li_status s = encode_map(ctx, &a.map_b, c->dtype, 3, const_cast<void*>(q->q), dims, strides, box, swz);
    if (s != LI_OK) return s;
  }
  if (c->dtype == LI_E4M3 && !gather && c->capacity % 4)
    // the loader copies each tile's 128 scales in 16-byte pieces
    return fail(ctx, LI_ERR_SHAPE, "%s: scanning an E4M3 cache needs capacity %% 4 == 0 (got %d)", what,
                c->capacity);
  a.cache_scale = c->dtype == LI_E4M3 ? c->scale : nullptr;
  a.cache_data = static_cast<const uint8_t*>(c->data);
  a.lengths = c->lengths;
  a.q_pos = q->q_pos;
  a.w = q->w;
  a.q_scale = q->dtype == LI_E4M3 ? q->q_scale : nullptr;
  a.beta = q->beta;
  P->kind = kind;
  a.RI = a.R;
  if (gather) {
    // gathered rows per item: the largest of 128 / 64 / 32 that still gives
    // every SM an item (the gather is bound by TMA operations per SM; the
    // MMA block stays 128 rows, the rows past RI are neither gathered nor
    // stored)
    a.RI = 32;
    for (int ri = a.R; ri >= 32; ri >>= 1)
      if (static_cast<int64_t>(n_seg) * ((cand_stride + ri - 1) / ri) >= ctx->num_sms) { a.RI = ri; break; }
  }
  const int64_t tiles_per_seg = (static_cast<int64_t>(gather ? cand_stride : c->capacity) + a.RI - 1) / a.RI;
  P->grid = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(ctx->num_sms, n_seg * tiles_per_seg)));
  return LI_OK;
}

li_status run_scan(li_ctx* ctx, ScanPlan& P, bool gather, cudaStream_t st) {
  (void)cudaGetLastError();   // do not blame this launch for an earlier, unrelated error
  Launch L(ctx, st, gather ? "gather" : "scan", P.grid, kScanThreads, static_cast<int>(P.a.smem_bytes));
  const cudaError_t e = launch_scan_kernel(P.kind, gather, P.a, P.grid, st);
  L.done();
  if (e != cudaSuccess) return cuda_fail(ctx, e, gather ? "gather kernel launch" : "scan kernel launch");
  return LI_OK;
}

// ------------------------------------------------------------------ selection

li_status memset_async(li_ctx* ctx, void* p, size_t bytes, cudaStream_t st) {
  Launch L(ctx, st, "memset", 0, 0, 0);
  const cudaError_t e = cudaMemsetAsync(p, 0, bytes, st);
  L.done();
  if (e != cudaSuccess) return cuda_fail(ctx, e, "cudaMemsetAsync");
  return LI_OK;
}

// Clears the histogram and per-row info of `rows` rows.
li_status clear_select_state(li_ctx* ctx, void* ws, const WsLayout& L, int64_t rows, cudaStream_t st) {
  li_status s = memset_async(ctx, at<uint8_t>(ws, L.hist), rows * kHistBins * 4, st);
  if (s != LI_OK) return s;
  return memset_async(ctx, at<uint8_t>(ws, L.rowinfo), rows * 16 * 4, st);
}

li_status run_topk_chunked(li_ctx* ctx, TopkArgs& t, void* ws, const WsLayout& L, cudaStream_t st) {
  t.hist = at<unsigned int>(ws, L.hist);
  t.rowinfo = at<int>(ws, L.rowinfo);
  t.chunk_gt = at<int>(ws, L.chunk_gt);
  t.chunk_off = at<int>(ws, L.chunk_off);
  t.cand = at<uint2>(ws, L.cand);
  t.n_chunks = (t.n + kTopkChunk - 1) / kTopkChunk;
  if (t.n_chunks < 1) t.n_chunks = 1;
  if (t.n_chunks > kMaxTopkChunks)
    return fail(ctx, LI_ERR_UNSUPPORTED, "selection rows longer than %d", kMaxTopkChunks * kTopkChunk);
  if (t.rows > 65535) return fail(ctx, LI_ERR_UNSUPPORTED, "more than 65535 selection rows");
  static const char* names[4] = {"topk_hist", "topk_filter", "topk_select", "topk_emit"};
  for (int stage = 0; stage < 4; ++stage) {
    const int grid = stage == 2 ? t.rows : t.rows * t.n_chunks;
    Launch Lc(ctx, st, names[stage], grid, stage == 2 ? 1024 : kTopkThreads, 0);
    const cudaError_t e = launch_topk_stage(stage, t, st);
    Lc.done();
    if (e != cudaSuccess) return cuda_fail(ctx, e, names[stage]);
  }
  return LI_OK;
}

// One selection: the single-launch cluster kernel when the rows fit it, else
// the chunked multi-kernel path (which needs its histogram and row state
// cleared).
li_status run_topk(li_ctx* ctx, TopkArgs& t, void* ws, const WsLayout& L, cudaStream_t st) {
  // workspace regions used by either path (the cluster kernel compacts its
  // boundary-bucket keys into `cand`)
  t.hist = at<unsigned int>(ws, L.hist);
  t.rowinfo = at<int>(ws, L.rowinfo);
  t.chunk_gt = at<int>(ws, L.chunk_gt);
  t.chunk_off = at<int>(ws, L.chunk_off);
  t.cand = at<uint2>(ws, L.cand);
  t.status = at<int>(ws, L.status);
  t.wait_ns = ctx->wait_ns;
  if (static_cast<int64_t>(t.rows) * t.n > static_cast<int64_t>((L.scores - L.cand) / 8))
    return fail(ctx, LI_ERR_WORKSPACE, "selection of %d x %d exceeds the workspace candidate buffer", t.rows, t.n);
  // Rows of up to kClusterMaxN positions take the single-launch cluster
  // kernel: sized for latency while every row's cluster can be resident at
  // once, for throughput beyond (measured on 1024 x 65536: 467 us, against
  // 566 us for the chunked multi-kernel path).
  if (t.rows > 65535) return fail(ctx, LI_ERR_UNSUPPORTED, "more than 65535 selection rows");
  if (t.n <= kClusterMaxN) {
    const int rows_all = t.rows * (t.k2 > 0 ? 2 : 1);   // a second budget doubles the clusters
    const int kpt = topk_keys_per_thread(t.n, rows_all, ctx->cluster_cap);
    int cs = 0;
    Launch Lc(ctx, st, "topk_cluster", 0, kClusterThreads, 0);
    const cudaError_t e = launch_topk_cluster(t, st, &cs, kpt);
    Lc.grid = cs * rows_all;
    Lc.done();
    if (e != cudaSuccess) return cuda_fail(ctx, e, "topk_cluster");
    return LI_OK;
  }
  if (t.k2 > 0) return fail(ctx, LI_ERR_UNSUPPORTED, "two budgets in one selection need rows of at most %d",
                            kClusterMaxN);
  li_status s = clear_select_state(ctx, ws, L, t.rows, st);
  if (s != LI_OK) return s;
  return run_topk_chunked(ctx, t, ws, L, st);
}

TopkArgs topk_args(const float* scores, int64_t stride, int rows, int n, int k) {
  TopkArgs t;
  memset(&t, 0, sizeof(t));
  t.scores = scores;
  t.row_stride = stride;
  t.rows = rows;
  t.n = n;
  t.k = k;
  t.len_div = 1;
  t.wait_ns = 2000000000ull;
  return t;
}

// Full-prefix scan + selection shared by li_score_topk and li_dsa_score_topk.
li_status score_topk_impl(li_ctx* ctx, const li_cache* c, const li_query* q, int k, int32_t* out_idx,
                          float* out_score, float* dump, void* ws, size_t ws_bytes, cudaStream_t st,
                          const char* what) {
  if (!ctx) return LI_ERR_ARG;
  li_status s = check_cache(ctx, c, what);
  if (s != LI_OK) return s;
  if ((s = check_query(ctx, c, q, what)) != LI_OK) return s;
  if (!out_idx) return fail(ctx, LI_ERR_ARG, "%s: out_idx is NULL", what);
  if (k < 1 || k > c->capacity) return fail(ctx, LI_ERR_ARG, "%s: k = %d must be in [1, capacity]", what, k);
  const int64_t rows = static_cast<int64_t>(c->batch) * q->T;
  const WsLayout L = ws_layout(rows, c->capacity, 0);
  if ((s = check_ws(ctx, ws, ws_bytes, L, what)) != LI_OK) return s;
  ScanPlan P;
  if ((s = plan_scan(ctx, c, q, false, 0, &P, what)) != LI_OK) return s;
  float* scores = dump ? dump : at<float>(ws, L.scores);
  P.a.scores = scores;
  P.a.score_stride = c->capacity;
  P.a.status = at<int>(ws, L.status);
  if ((s = run_scan(ctx, P, false, st)) != LI_OK) return s;
  TopkArgs t = topk_args(scores, c->capacity, static_cast<int>(rows), c->capacity, k);
  t.lengths = c->lengths;
  t.len_div = q->T;
  t.q_pos = q->q_pos;
  t.out_idx = out_idx;
  t.out_score = out_score;
  return run_topk(ctx, t, ws, L, st);
}

}  // namespace

// ======================================================================== C ABI

extern "C" {

const char* li_status_string(li_status s) {
  switch (s) {
    case LI_OK: return "ok";
    case LI_ERR_ARG: return "invalid argument";
    case LI_ERR_SHAPE: return "unsupported or inconsistent shape";
    case LI_ERR_DTYPE: return "unsupported dtype";
    case LI_ERR_ALIGN: return "misaligned pointer or row";
    case LI_ERR_WORKSPACE: return "workspace missing, short or misaligned";
    case LI_ERR_CAPACITY: return "append past the cache capacity";
    case LI_ERR_CUDA: return "CUDA error";
    case LI_ERR_DEVICE_TIMEOUT: return "a bounded device wait ran out";
    case LI_ERR_UNSUPPORTED: return "unsupported request";
    case LI_ERR_INDEX: return "candidate index outside the valid prefix";
  }
  return "unknown status";
}

li_status li_create(li_ctx** out, int device) {
  if (!out) return LI_ERR_ARG;
  *out = nullptr;
  li_ctx* c = new (std::nothrow) li_ctx();
  if (!c) return LI_ERR_ARG;
  int major = 0, minor = 0;
  cudaError_t e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, device);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, device);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&c->num_sms, cudaDevAttrMultiProcessorCount, device);
  if (e == cudaSuccess)
    e = cudaDeviceGetAttribute(&c->max_smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, device);
  if (e != cudaSuccess) {
    delete c;
    return LI_ERR_CUDA;
  }
  if (major != 10 || minor != 0) {
    delete c;
    return LI_ERR_UNSUPPORTED;
  }
  c->device = device;
  {
    // The occupancy queries read the current device: select ours for them.
    // A cluster size whose query fails counts as never resident, so the
    // selection sizes around it (the throughput form needs no residency).
    int prev = 0;
    e = cudaGetDevice(&prev);
    if (e == cudaSuccess) e = cudaSetDevice(device);
    if (e != cudaSuccess) {
      delete c;
      return LI_ERR_CUDA;
    }
    for (int cs = 1; cs <= 16; ++cs) {
      const int cap = topk_cluster_capacity(cs, c->num_sms);
      c->cluster_cap[cs] = cap > 0 ? cap : 0;
    }
    (void)cudaGetLastError();   // a failed query leaves no sticky error behind
    if (cudaSetDevice(prev) != cudaSuccess) {
      delete c;
      return LI_ERR_CUDA;
    }
  }
  void* fn = nullptr;
  cudaDriverEntryPointQueryResult q;
  e = cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault, &q);
  if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || !fn) {
    delete c;
    return LI_ERR_CUDA;
  }
  c->encode = reinterpret_cast<EncodeTiledFn>(fn);
  *out = c;
  return LI_OK;
}

li_status li_destroy(li_ctx* c) {
  if (!c) return LI_ERR_ARG;
  for (auto& r : c->prof) {
    cudaEventDestroy(r.beg);
    cudaEventDestroy(r.end);
  }
  for (auto e : c->free_events) cudaEventDestroy(e);
  delete c;
  return LI_OK;
}

const char* li_last_error(const li_ctx* c) { return c ? c->last_error.c_str() : "null context"; }

size_t li_workspace_bytes(const li_ctx* c, int batch, int T, int capacity, int H, int k, int B) {
  (void)c;
  (void)H;
  (void)k;
  const int64_t rows = static_cast<int64_t>(std::max(batch, 1)) * std::max(T, 1);
  return ws_layout(rows, std::max(capacity, 1), std::max(B, 0)).total;
}

li_status li_device_status(li_ctx* c, const void* ws, void* stream, li_status* out) {
  if (!c || !ws || !out) return LI_ERR_ARG;
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  int v = 0;
  cudaError_t e = cudaMemcpyAsync(&v, ws, sizeof(int), cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(c, e, "li_device_status read");
  e = cudaMemsetAsync(const_cast<void*>(ws), 0, sizeof(int), st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(c, e, "li_device_status clear");
  *out = static_cast<li_status>(v);
  return LI_OK;
}

li_status li_set_wait_limit(li_ctx* c, uint64_t ns) {
  if (!c) return LI_ERR_ARG;
  c->wait_ns = ns;
  return LI_OK;
}

li_status li_append_latent(li_ctx* c, const li_cache* cache, const void* h, li_dtype h_dtype, int d_model,
                           const void* W_down, int T, void* ws, size_t ws_bytes, void* stream) {
  return li_append_latent_ex(c, cache, h, h_dtype, d_model, W_down, T, nullptr, ws, ws_bytes, stream);
}

li_status li_append_latent_ex(li_ctx* c, const li_cache* cache, const void* h, li_dtype h_dtype, int d_model,
                              const void* W_down, int T, const li_latent_transform* tfp, void* ws, size_t ws_bytes,
                              void* stream) {
  const char* what = tfp ? "li_append_latent_ex" : "li_append_latent";
  if (!c) return LI_ERR_ARG;
  li_status s = check_cache(c, cache, what);
  if (s != LI_OK) return s;
  RowTransform tf;
  memset(&tf, 0, sizeof(tf));
  if (tfp) {
    const int dim = cache->dim;
    if (tfp->rope_dim < 0 || tfp->norm_dim < 0) return fail(c, LI_ERR_SHAPE, "%s: negative branch width", what);
    if (tfp->rope_dim > 0) {
      if (tfp->rope_sources < 1) return fail(c, LI_ERR_ARG, "%s: rope_sources must be >= 1", what);
      if (tfp->rope_offset < 0 || tfp->rope_offset % 2 || tfp->rope_dim % (2 * tfp->rope_sources) ||
          tfp->rope_offset + tfp->rope_dim > dim)
        return fail(c, LI_ERR_SHAPE,
                    "%s: rotary range [%d, %d) must start even, lie in the row of %d and hold whole frequencies "
                    "of %d sources", what, tfp->rope_offset, tfp->rope_offset + tfp->rope_dim, dim,
                    tfp->rope_sources);
      if (!tfp->inv_freq) return fail(c, LI_ERR_ARG, "%s: inv_freq is NULL", what);
      tf.rope_offset = tfp->rope_offset;
      tf.rope_dim = tfp->rope_dim;
      tf.rope_sources = tfp->rope_sources;
      tf.inv_freq = tfp->inv_freq;
    }
    if (tfp->norm_dim > 0) {
      if (tfp->norm_offset < 0 || tfp->norm_offset + tfp->norm_dim > dim)
        return fail(c, LI_ERR_SHAPE, "%s: NoPE range [%d, %d) outside the row of %d", what, tfp->norm_offset,
                    tfp->norm_offset + tfp->norm_dim, dim);
      if (!(tfp->norm_eps >= 0.f) || !std::isfinite(tfp->norm_eps))
        return fail(c, LI_ERR_ARG, "%s: norm_eps must be finite and >= 0", what);
      tf.norm_offset = tfp->norm_offset;
      tf.norm_dim = tfp->norm_dim;
      tf.gamma = tfp->norm_gamma;
      tf.beta = tfp->norm_beta;
      tf.eps = tfp->norm_eps;
    }
    if (tf.rope_dim > 0 && tf.norm_dim > 0 && tf.rope_offset < tf.norm_offset + tf.norm_dim &&
        tf.norm_offset < tf.rope_offset + tf.rope_dim)
      return fail(c, LI_ERR_SHAPE, "%s: the rotary and NoPE ranges overlap", what);
  }
  if (!h) return fail(c, LI_ERR_ARG, "%s: h is NULL", what);
  if (T < 1) return fail(c, LI_ERR_SHAPE, "%s: T must be >= 1", what);
  if (T > cache->capacity) return fail(c, LI_ERR_SHAPE, "%s: T = %d exceeds the capacity", what, T);
  if (W_down) {
    if (h_dtype != LI_F32 && h_dtype != LI_BF16) return fail(c, LI_ERR_DTYPE, "%s: h must be F32 or BF16", what);
    if (d_model < 8 || d_model % 8) return fail(c, LI_ERR_SHAPE, "%s: d_model must be a multiple of 8", what);
    if (!aligned(h, 16) || !aligned(W_down, 16)) return fail(c, LI_ERR_ALIGN, "%s: h and W_down must be 16-byte aligned", what);
  } else if (h_dtype != LI_F32) {
    return fail(c, LI_ERR_DTYPE, "%s: without W_down, h must be the F32 latent", what);
  }
  const WsLayout L = ws_layout(1, 1, 0);
  if ((s = check_ws(c, ws, ws_bytes, L, what)) != LI_OK) return s;
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int dim = cache->dim;
  unsigned int* done = at<unsigned int>(ws, L.done);
  int* status = at<int>(ws, L.status);
  if (!W_down) {
    // h already holds the fp32 rows [batch][T][dim]: quantise and store.
    Launch Ls(c, st, "append_store", 0, 256, 0);
    const cudaError_t e = launch_append_store(static_cast<const float*>(h), dim, 0, 1, cache->batch, T, 0, T, true,
                                              cache->data, cache->scale, cache->lengths, cache->capacity, dim,
                                              cache->dtype, cache->scale_split, tf, done, status, st);
    Ls.done();
    return e == cudaSuccess ? LI_OK : cuda_fail(c, e, "append store launch");
  }
  // c = W_down h in chunks of tokens, staged as fp32 in the workspace.
  float* tmp = at<float>(ws, L.tmp);
  const int eb = elt_bytes(h_dtype);
  const int tchunk = std::max(1, std::min(T, kAppendChunkTok / cache->batch));
  {
    const int n_tok = cache->batch * T;
    const int splits = append_fused_splits(d_model, dim);
    if (append_fusable(n_tok, dim, splits) &&
        append_fused_smem(n_tok, dim, splits, d_model, static_cast<size_t>(eb)) <= 96 * 1024) {
      Launch Lg(c, st, "append", 0, 256, 0);
      const cudaError_t e = launch_append_fused(h, h_dtype, W_down, d_model, dim, cache->batch, T, splits, tmp,
                                                cache->data, cache->scale, cache->lengths, cache->capacity,
                                                cache->dtype, cache->scale_split, tf, done, status, st);
      Lg.done();
      return e == cudaSuccess ? LI_OK : cuda_fail(c, e, "append launch");
    }
  }
  for (int t0 = 0; t0 < T; t0 += tchunk) {
    const int tn = std::min(tchunk, T - t0);
    int splits = 1;
    if (tn == T) {
      // every token of the batch at once: h rows are contiguous
      Launch Lg(c, st, "append_gemv", 0, 256, 0);
      splits = gemv_splits(d_model, cache->batch * T);
      const cudaError_t e = launch_append_gemv(h, h_dtype, W_down, d_model, dim, cache->batch * T, splits, tmp, st);
      Lg.done();
      if (e != cudaSuccess) return cuda_fail(c, e, "append gemv launch");
    } else {
      for (int b = 0; b < cache->batch; ++b) {
        const uint8_t* hb = static_cast<const uint8_t*>(h) + (static_cast<int64_t>(b) * T + t0) * d_model * eb;
        Launch Lg(c, st, "append_gemv", 0, 256, 0);
        splits = 1;
        const cudaError_t e = launch_append_gemv(hb, h_dtype, W_down, d_model, dim, tn, 1,
                                                 tmp + static_cast<int64_t>(b) * tn * dim, st);
        Lg.done();
        if (e != cudaSuccess) return cuda_fail(c, e, "append gemv launch");
      }
    }
    Launch Ls(c, st, "append_store", 0, 256, 0);
    const cudaError_t e = launch_append_store(tmp, dim, static_cast<int64_t>(cache->batch) * tn * dim, splits,
                                              cache->batch, tn, t0, T, t0 + tn >= T, cache->data,
                                              cache->scale, cache->lengths, cache->capacity, dim, cache->dtype,
                                              cache->scale_split, tf, done, status, st);
    Ls.done();
    if (e != cudaSuccess) return cuda_fail(c, e, "append store launch");
  }
  return LI_OK;
}

li_status li_absorb_query_group(li_ctx* c, const void* q, li_dtype q_dtype, int batch, int G, int H, int d_k,
                                const void* const* W_K, int d_c, li_dtype out_dtype, void* q_abs, float* q_abs_scale,
                                void* stream) {
  const char* what = "li_absorb_query_group";
  if (!c) return LI_ERR_ARG;
  if (!q || !q_abs || !W_K) return fail(c, LI_ERR_ARG, "%s: q, q_abs and W_K must be non-NULL", what);
  if (q_dtype != LI_F32 && q_dtype != LI_BF16) return fail(c, LI_ERR_DTYPE, "%s: q must be F32 or BF16", what);
  if (out_dtype != LI_F32 && out_dtype != LI_BF16 && out_dtype != LI_E4M3)
    return fail(c, LI_ERR_DTYPE, "%s: unknown out dtype", what);
  if (out_dtype == LI_E4M3 && !q_abs_scale) return fail(c, LI_ERR_ARG, "%s: E4M3 output needs q_abs_scale", what);
  if (G < 1 || G > kMaxAbsorbLayers) return fail(c, LI_ERR_SHAPE, "%s: G = %d must be in [1, %d]", what, G,
                                                 kMaxAbsorbLayers);
  if (batch < 1 || H < 1 || d_k < 1 || d_k > 256 || d_c < 2 || d_c > 256 || (d_c & 1))
    return fail(c, LI_ERR_SHAPE, "%s: need batch, H >= 1, d_k in [1, 256] and an even d_c in [2, 256]", what);
  if (static_cast<int64_t>(batch) * H > 2 * 65535)
    return fail(c, LI_ERR_SHAPE, "%s: batch * H must be <= %d", what, 2 * 65535);
  const size_t elt = q_dtype == LI_BF16 ? 2 : 4;
  if ((static_cast<size_t>(d_k) * d_c * elt) % 16)
    return fail(c, LI_ERR_SHAPE, "%s: d_k * d_c * element size must be a multiple of 16", what);
  for (int l = 0; l < G; ++l)
    if (!W_K[l] || !aligned(W_K[l], 16)) return fail(c, LI_ERR_ALIGN, "%s: W_K[%d] NULL or not 16-byte aligned", what, l);
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  Launch L(c, st, "absorb", 0, 256, 0);
  const cudaError_t e = launch_absorb_group(q, q_dtype, batch, G, H, d_k, W_K, d_c, out_dtype, q_abs, q_abs_scale, st);
  L.done();
  if (e != cudaSuccess) return cuda_fail(c, e, "group absorb launch");
  return LI_OK;
}

li_status li_absorb_query(li_ctx* c, const void* q, li_dtype q_dtype, int n_tok, int H, int d_k, const void* W_K,
                          int64_t W_K_head_stride, const float* b_K, int64_t b_K_head_stride, int d_c,
                          li_dtype out_dtype, void* q_abs, float* q_abs_scale, float* beta, void* stream) {
  const char* what = "li_absorb_query";
  if (!c) return LI_ERR_ARG;
  if (!q || !q_abs) return fail(c, LI_ERR_ARG, "%s: q and q_abs must be non-NULL", what);
  if (q_dtype != LI_F32 && q_dtype != LI_BF16) return fail(c, LI_ERR_DTYPE, "%s: q must be F32 or BF16", what);
  if (out_dtype != LI_F32 && out_dtype != LI_BF16 && out_dtype != LI_E4M3)
    return fail(c, LI_ERR_DTYPE, "%s: unknown out dtype", what);
  if (out_dtype == LI_E4M3 && !q_abs_scale) return fail(c, LI_ERR_ARG, "%s: E4M3 output needs q_abs_scale", what);
  if (n_tok < 1 || H < 1 || d_k < 1 || d_k > 256 || d_c < 1 || d_c > 256)
    return fail(c, LI_ERR_SHAPE, "%s: need n_tok, H >= 1 and d_k, d_c in [1, 256]", what);
  if (n_tok > 65535) return fail(c, LI_ERR_SHAPE, "%s: n_tok must be <= 65535 per call", what);
  if (!W_K && d_c != d_k) return fail(c, LI_ERR_SHAPE, "%s: identity decoder needs d_c == d_k", what);
  if (beta && !b_K) return fail(c, LI_ERR_ARG, "%s: beta requested without b_K", what);
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  Launch L(c, st, "absorb", 0, 256, 0);
  const cudaError_t e = launch_absorb(q, q_dtype, n_tok, H, d_k, W_K, W_K_head_stride, b_K, b_K_head_stride, d_c,
                                      out_dtype, q_abs, q_abs_scale, beta, c->num_sms, st);
  L.done();
  if (e != cudaSuccess) return cuda_fail(c, e, "absorb launch");
  return LI_OK;
}

li_status li_score_topk(li_ctx* c, const li_cache* cache, const li_query* q, int k, int32_t* out_idx,
                        float* out_score, float* scores_dump, void* ws, size_t ws_bytes, void* stream) {
  return score_topk_impl(c, cache, q, k, out_idx, out_score, scores_dump, ws, ws_bytes,
                         static_cast<cudaStream_t>(stream), "li_score_topk");
}

li_status li_dsa_score_topk(li_ctx* c, const li_cache* key_cache, const li_query* q, int k, int32_t* out_idx,
                            float* out_score, float* scores_dump, void* ws, size_t ws_bytes, void* stream) {
  return score_topk_impl(c, key_cache, q, k, out_idx, out_score, scores_dump, ws, ws_bytes,
                         static_cast<cudaStream_t>(stream), "li_dsa_score_topk");
}

li_status li_hs_anchor_candidates(li_ctx* c, const li_cache* cache, const li_query* q, int B, int k,
                                  int32_t* cand, int32_t* cand_n, int32_t* anchor_idx, float* anchor_score,
                                  float* scores_dump, void* ws, size_t ws_bytes, void* stream) {
  const char* what = "li_hs_anchor_candidates";
  if (!c) return LI_ERR_ARG;
  li_status s = check_cache(c, cache, what);
  if (s != LI_OK) return s;
  if ((s = check_query(c, cache, q, what)) != LI_OK) return s;
  if (!cand || !cand_n || !anchor_idx) return fail(c, LI_ERR_ARG, "%s: cand, cand_n, anchor_idx required", what);
  if (k < 1 || B < k || k > cache->capacity)
    return fail(c, LI_ERR_ARG, "%s: need 1 <= k <= B and k <= capacity (k=%d, B=%d)", what, k, B);
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int64_t rows = static_cast<int64_t>(cache->batch) * q->T;
  const WsLayout L = ws_layout(rows, cache->capacity, B);
  if ((s = check_ws(c, ws, ws_bytes, L, what)) != LI_OK) return s;
  ScanPlan P;
  if ((s = plan_scan(c, cache, q, false, 0, &P, what)) != LI_OK) return s;
  float* scores = scores_dump ? scores_dump : at<float>(ws, L.scores);
  P.a.scores = scores;
  P.a.score_stride = cache->capacity;
  P.a.status = at<int>(ws, L.status);
  if ((s = run_scan(c, P, false, st)) != LI_OK) return s;
  // candidates = top-B of the full prefix, with their scores
  float* cand_scores = at<float>(ws, L.cand_scores);
  TopkArgs t = topk_args(scores, cache->capacity, static_cast<int>(rows), cache->capacity, B);
  t.lengths = cache->lengths;
  t.len_div = q->T;
  t.q_pos = q->q_pos;
  t.out_idx = cand;
  t.out_score = cand_scores;
  t.out_count = cand_n;
  if (cache->capacity <= kClusterMaxN) {
    // the anchor's own top-k is the top-k of the full prefix: it is selected
    // from the same scores by clusters of their own in the same launch as
    // the candidates, rather than after them from the candidates' scores
    t.out_score = nullptr;
    t.k2 = k;
    t.out_idx2 = anchor_idx;
    t.out_score2 = anchor_score;
    return run_topk(c, t, ws, L, st);
  }
  if ((s = run_topk(c, t, ws, L, st)) != LI_OK) return s;
  // the anchor's own top-k: under the same order (score desc, position asc)
  // the top-k of the prefix is the top-k of its top-B, whose positions are
  // ascending, so it is selected from the candidates' scores alone
  TopkArgs t2 = topk_args(cand_scores, B, static_cast<int>(rows), B, k);
  t2.lengths = cand_n;
  t2.len_div = 1;
  t2.idx_map = cand;
  t2.map_stride = B;
  t2.out_idx = anchor_idx;
  t2.out_score = anchor_score;
  return run_topk(c, t2, ws, L, st);
}

li_status li_hs_follower_refine(li_ctx* c, const li_cache* cache, const li_query* q, const int32_t* cand,
                                const int32_t* cand_n, int B, int k, int32_t* out_idx, float* out_score,
                                float* scores_dump, void* ws, size_t ws_bytes, void* stream) {
  const char* what = "li_hs_follower_refine";
  if (!c) return LI_ERR_ARG;
  li_status s = check_cache(c, cache, what);
  if (s != LI_OK) return s;
  if ((s = check_query(c, cache, q, what)) != LI_OK) return s;
  if (!cand || !cand_n || !out_idx) return fail(c, LI_ERR_ARG, "%s: cand, cand_n, out_idx required", what);
  if (k < 1 || B < k) return fail(c, LI_ERR_ARG, "%s: need 1 <= k <= B (k=%d, B=%d)", what, k, B);
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int64_t rows = static_cast<int64_t>(cache->batch) * q->T;
  const WsLayout L = ws_layout(rows, B, B);
  if ((s = check_ws(c, ws, ws_bytes, L, what)) != LI_OK) return s;
  ScanPlan P;
  if ((s = plan_scan(c, cache, q, true, B, &P, what)) != LI_OK) return s;
  float* scores = scores_dump ? scores_dump : at<float>(ws, L.scores);
  P.a.scores = scores;
  P.a.score_stride = B;
  P.a.status = at<int>(ws, L.status);
  P.a.cand = cand;
  P.a.cand_n = cand_n;
  if ((s = run_scan(c, P, true, st)) != LI_OK) return s;
  TopkArgs t = topk_args(scores, B, static_cast<int>(rows), B, k);
  t.lengths = cand_n;
  t.len_div = 1;
  t.idx_map = cand;
  t.map_stride = B;
  t.out_idx = out_idx;
  t.out_score = out_score;
  return run_topk(c, t, ws, L, st);
}

li_status li_topk(li_ctx* c, const float* scores, int rows, int n, int64_t row_stride, const int32_t* lengths,
                  int k, int32_t* out_idx, float* out_score, void* ws, size_t ws_bytes, void* stream) {
  const char* what = "li_topk";
  if (!c) return LI_ERR_ARG;
  if (!scores || !out_idx) return fail(c, LI_ERR_ARG, "%s: scores and out_idx must be non-NULL", what);
  if (rows < 1 || n < 1 || k < 1 || row_stride < n)
    return fail(c, LI_ERR_SHAPE, "%s: need rows, n, k >= 1 and row_stride >= n", what);
  const WsLayout L = ws_layout(rows, n, 0);
  li_status s = check_ws(c, ws, ws_bytes, L, what);
  if (s != LI_OK) return s;
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  TopkArgs t = topk_args(scores, row_stride, rows, n, k);
  t.lengths = lengths;
  t.out_idx = out_idx;
  t.out_score = out_score;
  return run_topk(c, t, ws, L, st);
}

// ------------------------------------------------------------------ selection quality

namespace {
struct RecallLayout {
  WsLayout L;
  size_t top_idx, top_val, pbar, total;
};
RecallLayout recall_layout(int64_t rows, int64_t H, int64_t N, int64_t K) {
  RecallLayout R;
  R.L = ws_layout(rows * H, N, 0);
  size_t off = R.L.total;
  auto take = [&](size_t bytes) { size_t o = off; off += up256(bytes); return o; };
  R.top_idx = take(rows * H * K * 4);
  R.top_val = take(rows * H * K * 4);
  R.pbar = take(rows * N * 4);
  R.total = off;
  return R;
}
}  // namespace

size_t li_recall_workspace_bytes(const li_ctx*, int rows, int H, int N, int K) {
  if (rows < 1 || H < 1 || N < 1 || K < 1) return 0;
  return recall_layout(rows, H, N, std::min(K, N)).total;
}

li_status li_attention_recall(li_ctx* c, const float* probs, int rows, int H, int N, const int32_t* lengths,
                              const int32_t* sel, int k, int K, float* recall, float* mean_recall, void* ws,
                              size_t ws_bytes, void* stream) {
  const char* what = "li_attention_recall";
  if (!c) return LI_ERR_ARG;
  if (!probs || !sel || !recall) return fail(c, LI_ERR_ARG, "%s: probs, sel and recall must be non-NULL", what);
  if (rows < 1 || H < 1 || N < 1 || k < 1 || K < 1)
    return fail(c, LI_ERR_SHAPE, "%s: rows, H, N, k and K must be >= 1", what);
  if (static_cast<int64_t>(rows) * H > 65535)
    return fail(c, LI_ERR_UNSUPPORTED, "%s: rows x H = %lld exceeds 65535", what,
                static_cast<long long>(rows) * H);
  const int KK = std::min(K, N);
  const RecallLayout R = recall_layout(rows, H, N, KK);
  if (!ws || ws_bytes < R.total)
    return fail(c, LI_ERR_WORKSPACE, "%s: workspace of %zu bytes, %zu needed", what, ws_bytes, R.total);
  if (!aligned(ws, 256)) return fail(c, LI_ERR_ALIGN, "%s: workspace must be 256-byte aligned", what);
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  int32_t* top_idx = at<int32_t>(ws, R.top_idx);
  float* top_val = at<float>(ws, R.top_val);
  // each head's best size-K mass: the exact top-K of its row
  TopkArgs t = topk_args(probs, N, rows * H, N, KK);
  t.lengths = lengths;
  t.len_div = H;
  t.out_idx = top_idx;
  t.out_score = top_val;
  li_status s = run_topk(c, t, ws, R.L, st);
  if (s != LI_OK) return s;
  {
    Launch Lr(c, st, "recall", 0, 256, 0);
    const cudaError_t e = launch_recall(probs, rows, H, N, lengths, sel, k, top_idx, top_val, KK, recall, st);
    Lr.done();
    if (e != cudaSuccess) return cuda_fail(c, e, "recall launch");
  }
  if (!mean_recall) return LI_OK;
  float* pbar = at<float>(ws, R.pbar);
  {
    Launch Lm(c, st, "head_mean", 0, 256, 0);
    const cudaError_t e = launch_head_mean(probs, rows, H, N, lengths, pbar, c->num_sms, st);
    Lm.done();
    if (e != cudaSuccess) return cuda_fail(c, e, "head mean launch");
  }
  TopkArgs t2 = topk_args(pbar, N, rows, N, KK);
  t2.lengths = lengths;
  t2.out_idx = top_idx;
  t2.out_score = top_val;
  if ((s = run_topk(c, t2, ws, R.L, st)) != LI_OK) return s;
  Launch Lr(c, st, "recall", 0, 256, 0);
  const cudaError_t e = launch_recall(pbar, rows, 1, N, lengths, sel, k, top_idx, top_val, KK, mean_recall, st);
  Lr.done();
  return e == cudaSuccess ? LI_OK : cuda_fail(c, e, "recall launch");
}

li_status li_set_trace(li_ctx* c, void* buf, size_t bytes) {
  if (!c) return LI_ERR_ARG;
  if (buf && bytes < static_cast<size_t>(kTraceCtas) * kTraceTiles * kTraceEvents * 8)
    return fail(c, LI_ERR_WORKSPACE, "li_set_trace: buffer of %zu bytes, %zu needed", bytes,
                static_cast<size_t>(kTraceCtas) * kTraceTiles * kTraceEvents * 8);
  c->trace = static_cast<uint64_t*>(buf);
  return LI_OK;
}

li_status li_profile_enable(li_ctx* c, int enable) {
  if (!c) return LI_ERR_ARG;
  c->profile = enable != 0;
  return LI_OK;
}

li_status li_profile_read(li_ctx* c, li_profile_record* out, int max, int* count) {
  if (!c || !count) return LI_ERR_ARG;
  *count = static_cast<int>(c->prof.size());
  for (int i = 0; i < *count && i < max && out; ++i) {
    const ProfRec& r = c->prof[i];
    cudaError_t e = cudaEventSynchronize(r.end);
    if (e != cudaSuccess) return cuda_fail(c, e, "li_profile_read");
    float ms = 0.f;
    cudaEventElapsedTime(&ms, r.beg, r.end);
    memset(&out[i], 0, sizeof(out[i]));
    snprintf(out[i].kernel, sizeof(out[i].kernel), "%s", r.name.c_str());
    out[i].ms = ms;
    out[i].grid = r.grid;
    out[i].block = r.block;
    out[i].smem = r.smem;
  }
  return LI_OK;
}

li_status li_profile_reset(li_ctx* c) {
  if (!c) return LI_ERR_ARG;
  for (auto& r : c->prof) {
    c->free_events.push_back(r.beg);
    c->free_events.push_back(r.end);
  }
  c->prof.clear();
  return LI_OK;
}

}  // extern "C"

// ======================================================================== allocation-free selection

namespace {

// Scratch of li_score_topk_static, part of the library image (no allocation
// at any time): a 256-byte header holding the device status word, then the
// fp32 scores of every query row.  The module loader zero-fills it; the
// entry point clears the status word itself before every call.
constexpr size_t kStaticScratchBytes = size_t(8) << 20;   // 8 MiB
constexpr size_t kStaticScoresOffset = 256;
__device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

constexpr int kStaticMaxDevices = 64;
std::mutex g_static_mu;
// Per device: the scratch's device address and the CUDA context it was
// looked up in (a device reset replaces the context and unmaps the old one).
void* g_static_addr[kStaticMaxDevices] = {};
CUcontext g_static_cuctx[kStaticMaxDevices] = {};

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);

// Device address of the scratch on the current device, looked up once per
// device and context (the lookup is the only setup this entry point needs).
li_status static_scratch(li_ctx* c, void** out, const char* what) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(c, e, what);
  if (dev != c->device)
    return fail(c, LI_ERR_ARG, "%s: the context's device (%d) must be the current device (%d)", what, c->device,
                dev);
  if (dev < 0 || dev >= kStaticMaxDevices)
    return fail(c, LI_ERR_UNSUPPORTED, "%s: device ordinal %d above %d", what, dev, kStaticMaxDevices - 1);
  static CtxGetCurrentFn ctx_current = [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    const cudaError_t r = cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &fn, 12000, cudaEnableDefault, &q);
    return (r == cudaSuccess && q == cudaDriverEntryPointSuccess) ? reinterpret_cast<CtxGetCurrentFn>(fn) : nullptr;
  }();
  if (!ctx_current) return fail(c, LI_ERR_CUDA, "%s: cuCtxGetCurrent is unavailable", what);
  CUcontext cur = nullptr;
  if (ctx_current(&cur) == CUDA_SUCCESS && !cur) {
    // nothing has made the primary context current in this thread yet
    if ((e = cudaSetDevice(dev)) != cudaSuccess) return cuda_fail(c, e, what);
    (void)ctx_current(&cur);
  }
  if (!cur) return fail(c, LI_ERR_CUDA, "%s: no current CUDA context", what);
  std::lock_guard<std::mutex> lock(g_static_mu);
  if (!g_static_addr[dev] || g_static_cuctx[dev] != cur) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_static_scratch);
    if (e != cudaSuccess || !p) {
      (void)cudaGetLastError();
      return cuda_fail(c, e != cudaSuccess ? e : cudaErrorInvalidSymbol, "cudaGetSymbolAddress (static scratch)");
    }
    g_static_addr[dev] = p;
    g_static_cuctx[dev] = cur;
  }
  *out = g_static_addr[dev];
  return LI_OK;
}

}  // namespace

extern "C" li_status li_score_topk_static(li_ctx* c, const li_cache* cache, const li_query* q, int k,
                                          int32_t* out_idx, float* out_score, int32_t* device_status,
                                          void* stream) {
  const char* what = "li_score_topk_static";
  if (!c) return LI_ERR_ARG;
  li_status s = check_cache(c, cache, what);
  if (s != LI_OK) return s;
  if ((s = check_query(c, cache, q, what)) != LI_OK) return s;
  if (!out_idx) return fail(c, LI_ERR_ARG, "%s: out_idx is NULL", what);
  if (k < 1 || k > cache->capacity) return fail(c, LI_ERR_ARG, "%s: k = %d must be in [1, capacity]", what, k);
  const int64_t rows = static_cast<int64_t>(cache->batch) * q->T;
  if (cache->capacity > kClusterMaxN || rows > 65535)
    return fail(c, LI_ERR_UNSUPPORTED, "%s: rows of at most %d positions and at most 65535 query rows (got %d, %lld)",
                what, kClusterMaxN, cache->capacity, static_cast<long long>(rows));
  const size_t need = kStaticScoresOffset + static_cast<size_t>(rows) * cache->capacity * sizeof(float);
  if (need > kStaticScratchBytes)
    return fail(c, LI_ERR_WORKSPACE, "%s: %lld query rows x %d positions need %zu bytes of scratch; the static "
                "scratch holds %zu (use li_score_topk with a caller-owned workspace)", what,
                static_cast<long long>(rows), cache->capacity, need, kStaticScratchBytes);
  void* base = nullptr;
  if ((s = static_scratch(c, &base, what)) != LI_OK) return s;
  int* status = static_cast<int*>(base);
  float* scores = reinterpret_cast<float*>(static_cast<uint8_t*>(base) + kStaticScoresOffset);
  ScanPlan P;
  if ((s = plan_scan(c, cache, q, false, 0, &P, what)) != LI_OK) return s;
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemsetAsync(status, 0, sizeof(int), st);
  if (e != cudaSuccess) return cuda_fail(c, e, "static scratch status clear");
  P.a.scores = scores;
  P.a.score_stride = cache->capacity;
  P.a.status = status;
  if ((s = run_scan(c, P, false, st)) != LI_OK) return s;
  TopkArgs t = topk_args(scores, cache->capacity, static_cast<int>(rows), cache->capacity, k);
  t.lengths = cache->lengths;
  t.len_div = q->T;
  t.q_pos = q->q_pos;
  t.out_idx = out_idx;
  t.out_score = out_score;
  t.status = status;
  t.wait_ns = c->wait_ns;
  {
    int cs = 0;
    Launch Lc(c, st, "topk_cluster", 0, kClusterThreads, 0);
    e = launch_topk_cluster(t, st, &cs, topk_keys_per_thread(t.n, t.rows, c->cluster_cap));
    Lc.grid = cs * t.rows;
    Lc.done();
    if (e != cudaSuccess) return cuda_fail(c, e, "topk_cluster");
  }
  if (device_status) {
    e = cudaMemcpyAsync(device_status, status, sizeof(int), cudaMemcpyDeviceToDevice, st);
    if (e != cudaSuccess) return cuda_fail(c, e, "static scratch status copy");
  }
  return LI_OK;
}
