// internal.h -- declarations shared by the library's translation units.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/li.h"

namespace li {

constexpr int kTileM = 128;          // cache rows per MMA tile (UMMA M)
constexpr int kEpiWarps = 8;         // two epilogue warpgroups, alternating tiles
// warp 0 loads, warps 1 and 2 + kEpiWarps issue the MMAs of the two M blocks,
// warps 2 .. 1 + kEpiWarps run the epilogue, warp 3 + kEpiWarps issues half
// of the row gathers (gather variant; idle in the scan)
constexpr int kScanThreads = 128 + 32 * kEpiWarps;
constexpr int kMmaWarp2 = 2 + kEpiWarps;
constexpr int kGatherWarp2 = 3 + kEpiWarps;
constexpr int kMetaSlots = 8;        // ring of per-item row metadata (fp8 scales, gathered rows)
constexpr int kMaxItemRows = 256;    // rows of one work item (two M=128 MMA blocks)
constexpr int kMaxSegments = 1024;   // (sequence, query group) segments per scan launch
constexpr int kMaxStages = 32;
constexpr int kHistBins = 2048;      // first radix digit: key bits 31..21

// Arguments of the scoring kernel (scan of whole prefixes, or gather of
// candidate rows).  Tensor maps first: they must stay 64-byte aligned.
struct alignas(64) ScanArgs {
  CUtensorMap map_a;          // cache rows: dims {swz/elt, batch*capacity, n_kchunks}, box {swz/elt, R, KS};
                              // gather: dims {dim, batch*capacity}, box {swz/elt, 1}
  CUtensorMap map_b;          // queries: dims {dim, H, batch*T}, box {swz/elt, H_pad, Qg}
  CUtensorMap map_a2;         // gather with tail64: dims {dim, batch*capacity}, box {64 B / elt, 1}, 64-B swizzle
  const uint8_t* cache_data;  // [batch*capacity][row_bytes] (the rows the cache map covers)
  const float* cache_scale;   // [batch*capacity] (segmented: [batch*capacity][2]) or null
  const int* lengths;         // [batch]
  const int* q_pos;           // [batch*T] or null
  const float* w;             // [batch*T*H]
  const float* q_scale;       // [batch*T*H] or null
  const float* beta;          // [batch*T*H] or null
  const int* cand;            // gather: [batch*T][cand_stride]
  const int* cand_n;          // gather: [batch*T]
  float* scores;              // [batch*T][score_stride]
  int* status;
  int64_t score_stride;
  int64_t row_bytes;
  uint64_t wait_ns;
  int batch, capacity, T, H, H_pad, Qg, n_groups, N;
  int cand_stride;
  int swz, n_kchunks, elt_bytes;
  int R, MB;                  // rows per work item (128 or 256) and M=128 blocks per item
  int RI;                     // gather: candidate rows gathered per item (32, 64 or 128 <= R)
  int tail64;                 // gather: rows of 128 m + 64 bytes; the last 64-byte chunk comes by map_a2
  int KS, stages_per_item;    // K-chunks per stage, stages per item
  int n_stages, n_bslots, n_acc, n_meta;
  int ep_stride;              // floats of epilogue parameters per epilogue warp
  uint32_t tmem_cols, idesc;
  uint32_t a_stage_bytes, b_slot_bytes, meta_bytes, misc_offset, smem_bytes;
  int n_segments;
  int seg_kstep;              // segmented fp8: first K step (32 bytes) of the second scale's segment; 0: one scale
  uint64_t* trace;            // per-tile event times of the first kTraceCtas CTAs, or null
};

// Diagnostic tile trace: [kTraceCtas][kTraceTiles][kTraceEvents] SM clock
// cycles (comparable within one CTA).  Events: 0 producer has the first stage of the tile, 1 producer issued
// the last stage, 2 MMA saw the first stage full, 3 MMA committed the tile,
// 4 epilogue saw the accumulator full, 5 epilogue released it, 6 MMA issuer
// started waiting for the first stage, 7 epilogue finished its head sums.
constexpr int kTraceCtas = 8, kTraceTiles = 64, kTraceEvents = 8;

// Kernel families (for the launch profile).
enum KernelKind { kKScan = 0, kKGather, kKTopkHist, kKTopkFilter, kKTopkSelect, kKTopkEmit,
                  kKAppendGemv, kKAppendStore, kKAbsorb, kKMemset };

// Launch `kernel` with programmatic stream serialisation (it may begin while
// the previous kernel on the stream finishes; the kernel itself waits for it
// in pdl_begin() before touching global memory), as a cluster of cluster_x
// CTAs along x when cluster_x > 1.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, int cluster_x,
                       Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  int n = 0;
  attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[n].val.programmaticStreamSerializationAllowed = 1;
  ++n;
  if (cluster_x > 1) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = cluster_x;
    attr[n].val.clusterDim.y = 1;
    attr[n].val.clusterDim.z = 1;
    ++n;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// Raise a kernel's dynamic shared-memory limit to at least `bytes` on the
// current device. The attribute is set once per (kernel, device) and
// remembered, so later calls make no runtime call at all (and so are safe
// while a stream is being captured into a graph).
cudaError_t raise_smem_limit(const void* fn, int bytes);

cudaError_t launch_scan_kernel(int kind, bool gather, const ScanArgs& a, int grid, cudaStream_t st);

// ---- top-k

struct TopkArgs {
  const float* scores;
  int64_t row_stride;
  int rows, n, k;
  // per-row valid length: n_r = min(n, lengths ? lengths[r / len_div] : n),
  // further capped by q_pos[r] + 1 when q_pos is given; negatives -> 0.
  const int* lengths;
  int len_div;
  const int* q_pos;
  const int* idx_map;         // output index = idx_map[r * map_stride + pos], or pos
  int64_t map_stride;
  int32_t* out_idx;
  float* out_score;
  int32_t* out_count;         // k_eff per row, or null
  // A second budget over the same rows in the same launch (cluster kernel
  // only): with k2 > 0 the grid holds 2 x rows rows of clusters, and row
  // rows + r selects the top-k2 of score row r into out_idx2 / out_score2
  // (same lengths and index map, no count), independently of row r.
  int k2;
  int32_t* out_idx2;
  float* out_score2;
  // workspace
  unsigned int* hist;         // [rows][2048]
  int* rowinfo;               // [rows][16]
  int* chunk_gt;              // [rows][n_chunks]
  int* chunk_off;             // [rows][n_chunks]
  uint2* cand;                // [rows][n]
  int n_chunks;
  // bounded waits of the cluster kernel's exchanges: a wait that runs out
  // records LI_ERR_DEVICE_TIMEOUT in *status (may be null)
  int* status;
  uint64_t wait_ns;
};

// Single-launch selection for rows of up to kClusterMaxN positions: one
// thread-block cluster per row, keys held in registers, digit histograms
// summed across the cluster in distributed shared memory.
constexpr int kClusterThreads = 512;
constexpr int kClusterMaxSize = 8;
constexpr int kClusterMaxN = kClusterThreads * 32 * kClusterMaxSize;   // 131072
// CTAs per row of the single-launch selection at a target of keys per thread
// (kTopkKeysLatency for a few rows, kTopkKeysThroughput for many).
constexpr int kTopkKeysLatency = 4, kTopkKeysThroughput = 32;
int topk_cluster_size(int64_t n, int keys_per_thread, int rows);
// How many clusters of cs CTAs (1..16) of the single-launch selection can be
// resident at once on the current device; -1 if the query fails.
int topk_cluster_capacity(int cs, int num_sms);
// The keys-per-thread target of a selection of `rows` rows of n positions:
// the latency target (4 keys a thread) when every row's cluster can be
// resident at once, else 8 or 16 keys a thread (smaller clusters) when
// those fit, else the throughput target.  cap[cs] is the residency for
// cluster size cs (1..16), from topk_cluster_capacity.
int topk_keys_per_thread(int64_t n, int rows, const int* cap);
cudaError_t launch_topk_cluster(const TopkArgs& a, cudaStream_t st, int* cluster_size,
                                int keys_per_thread = kTopkKeysLatency);

constexpr int kTopkChunk = 4096;
constexpr int kTopkThreads = 256;
constexpr int kMaxTopkChunks = 8192;

// The four stages of a selection, launched in order on one stream:
// 0 first-digit histogram, 1 filter (boundary
// bucket candidates and per-chunk counts), 2 select (exact threshold, tie
// cut and output offsets, one CTA per row), 3 emit (ordered output).
cudaError_t launch_topk_stage(int stage, const TopkArgs& a, cudaStream_t st);

// ---- construction

// Split count of the construction GEMV for n_tok tokens of width d_model.
int gemv_splits(int d_model, int n_tok);
// Per-row transforms of the two-branch latent, applied after c = W_down h
// and before quantisation (see li_latent_transform).  All zero: none.
struct RowTransform {
  int rope_offset, rope_dim, rope_sources;
  const float* inv_freq;
  int norm_offset, norm_dim;
  const float* gamma;
  const float* beta;
  float eps;
};

cudaError_t launch_append_gemv(const void* h, int h_dtype, const void* W, int d_model, int dim,
                               int n_tok, int splits, float* out, cudaStream_t st);
// Decode-sized appends (at most 8 tokens whose partial sums fit one block's
// shared memory) run as one launch: split-K GEMV, then the last block
// reduces the splits in order and stores the rows.
int append_fused_splits(int d_model, int dim);
bool append_fusable(int n_tok, int dim, int splits);
size_t append_fused_smem(int n_tok, int dim, int splits, int d_model, size_t h_elt);
cudaError_t launch_append_fused(const void* h, int h_dtype, const void* W, int d_model, int dim, int batch, int T,
                                int splits, float* part, void* data, float* scale, int32_t* lengths, int capacity,
                                int dtype, int scale_split, const RowTransform& tf, unsigned int* done, int* status,
                                cudaStream_t st);
cudaError_t launch_append_store(const float* c, int64_t c_tok_stride, int64_t split_stride, int splits,
                                int batch, int T_chunk, int t0, int T_total, bool bump, void* data,
                                float* scale, int32_t* lengths, int capacity, int dim, int dtype, int scale_split,
                                const RowTransform& tf, unsigned int* done_counter, int* status, cudaStream_t st);
// G layers' decoders (G <= kMaxAbsorbLayers, 16-byte aligned, shared by the
// heads) absorbed into queries stacked [batch][G][H][.] in one launch.
constexpr int kMaxAbsorbLayers = 8;
cudaError_t launch_absorb_group(const void* q, int q_dtype, int batch, int G, int H, int d_k, const void* const* W,
                                int d_c, int out_dtype, void* q_abs, float* q_abs_scale, cudaStream_t st);
cudaError_t launch_absorb(const void* q, int q_dtype, int n_tok, int H, int d_k, const void* W,
                          int64_t W_head_stride, const float* b, int64_t b_head_stride, int d_c,
                          int out_dtype, void* q_abs, float* q_abs_scale, float* beta, int num_sms,
                          cudaStream_t st);

// ---- selection quality
cudaError_t launch_head_mean(const float* probs, int rows, int H, int N, const int32_t* lengths, float* pbar,
                             int num_sms, cudaStream_t st);
cudaError_t launch_recall(const float* vals, int rows, int Hh, int N, const int32_t* lengths, const int32_t* sel,
                          int k, const int32_t* top_idx, const float* top_val, int K, float* out, cudaStream_t st);

}  // namespace li
