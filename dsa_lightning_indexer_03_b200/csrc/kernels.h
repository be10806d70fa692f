// kernels.h -- launchers of the library's CUDA kernels (internal to the .so).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"

namespace dsa {

// ---------------------------------------------------------------- projections
struct ProjKwEpilogue {
  int M;                          // tokens
  __nv_bfloat16* key_cache;       // [cache_rows, 128]
  int64_t cache_rows;
  float* w_out;                   // [M, 32]
  const int32_t* positions;       // [M]
  const int32_t* q_seq_offsets;   // [B+1]
  int B;
  const int64_t* cache_offsets;   // [B+1]
  uint8_t* key8;                  // FP8 cache instead of key_cache when set: e4m3 codes [cache_rows, 128]
  float* key_scale;               // FP8 cache: [cache_rows] scale of each row
  int n_heads;                    // 32 or 64: head-weight columns after the 128 key columns
  int rope_dim;                   // rotated dims at the start of the key (0: none)
  const double* inv_freq;         // rotary frequencies, rope_dim / 2 of them
  const float* gamma;             // [128]
  const float* beta;              // [128]
  float eps;
  int* err;
  uint64_t timeout_ns;
};

// q_out[M, N] = bf16(RoPE(A[M,K] * Bt[N,K]^T)); tmA box {64,128}, tmB box {64,256}; with
// rope_dim > 0 the first rope_dim dims of every 128-dim head turn by positions[m] * inv_freq[i]
cudaError_t launch_proj_q(const CUtensorMap& tmA, const CUtensorMap& tmB, int M, int K, int N,
                          __nv_bfloat16* q_out, int* err, uint64_t timeout_ns, cudaStream_t s,
                          const int32_t* positions = nullptr, const double* inv_freq = nullptr, int rope_dim = 0);

// [k~ | w] = A[M,K] * Bt[128+H,K]^T with the key LayerNorm (+ RoPE) / scatter epilogue;
// tmB box {64, 128+H}
cudaError_t launch_proj_kw(const CUtensorMap& tmA, const CUtensorMap& tmB, int K, const ProjKwEpilogue& e,
                           cudaStream_t s);

// q8_out[M, N] = e4m3 codes of bf16(A * Bt^T) per 128-column head, q_scale[M, N/128]
cudaError_t launch_proj_q8(const CUtensorMap& tmA, const CUtensorMap& tmB, int M, int K, int N, uint8_t* q8_out,
                           float* q_scale, int* err, uint64_t timeout_ns, cudaStream_t s);

// FP8 e4m3 codes and scales of n bf16 key rows (one scale per row)
cudaError_t launch_quantize_keys_fp8(int64_t n, const __nv_bfloat16* keys, uint8_t* out, float* scale,
                                     cudaStream_t s);

cudaError_t launch_key_norm(int64_t n, const float* raw, __nv_bfloat16* out, const float* gamma,
                            const float* beta, float eps, cudaStream_t s);

// dst[N, K] = src[K, N]^T (bf16), dst row stride K, written at row offset dst_row0
cudaError_t launch_transpose_bf16(const __nv_bfloat16* src, int K, int N, __nv_bfloat16* dst, int dst_row0,
                                  cudaStream_t s);

// ---------------------------------------------------------------- score + top-k
// Candidate storage of one query, in (ordered score key, position) pairs: two keep
// sets of kTopK entries (the current best list and the target of the next
// compaction) and one append area per epilogue warp of the query's lane quadrants.
constexpr int kWarpApp = 2048;                         // append slots of one warp, per query
constexpr int kCandStride = 2 * kTopK + 4 * kWarpApp;  // keep 0 | keep 1 | areas 0..3
constexpr int kMaxChunks = 16;                 // key chunks per query on the split-key path
constexpr int kMinChunk = 4096;                // shortest key chunk on the split-key path
constexpr int kSplitMaxTokens = 256;           // split-key path is offered up to this many queries
constexpr int kPrefillQ = 8;                   // queries per work item on the prefill path (32 heads)

struct WorkItem {
  int32_t t0;       // first query token
  int32_t nq;       // queries in the item
  int32_t b;        // sequence
  int32_t k_begin;  // first key position scored (multiple of 128)
  int32_t k_end;    // one past the last key position any query of the item scores
  int32_t chunk;    // -1: writes the output rows; >= 0: key chunk of a split query (writes partials)
  int32_t pad0, pad1;
};

struct TopkWorkspace {
  WorkItem* items;
  int max_items;
  int* n_items;
  int* work_counter;
  int* seq_base;     // [max(B, T) + 2]
  int* pos_eff;      // [T] validated positions, -1 for an invalid query
  int* tok_nchunks;  // [T] key chunks of each query on the split-key path
  uint2* cand;       // [cand_slots][kPrefillQ][kCandStride]
  int cand_slots;    // CTA slots (x kPrefillQ queries each)
  uint32_t* part_keys;
  int32_t* part_idx;
  uint32_t* part_hist;  // [part_tokens][2048] bin counts of the partial lists; zero between calls
  int part_tokens;
  int* err;
};

struct TopkArgs {
  int T, B;
  int64_t cache_rows;
  const __nv_bfloat16* q;
  const float* w;
  const int32_t* positions;
  const int32_t* q_seq_offsets;
  const __nv_bfloat16* key_cache;
  const int64_t* cache_offsets;
  int32_t* idx_out;
  float* score_out;
  bool split;
  bool sorted;       // order each row by (score desc, position asc); short rows stay [0..p, -1...]
  int heads;         // 32, or 64 (bf16 only)
  bool fp8;          // q and key_cache hold FP8 e4m3 codes with the scales below
  const float* q_scale;    // FP8: [T, 32] per query head
  const float* key_scale;  // FP8: [cache_rows] per key row
  uint64_t timeout_ns;
};

cudaError_t launch_topk(const TopkArgs& a, const TopkWorkspace& ws, const CUtensorMap& tmQ1, const CUtensorMap& tmQ8,
                        const CUtensorMap& tmK, int num_sms, cudaStream_t s);

// dst rows d = 0..n-1 := src row anchor[d] (indices, and scores when both score pointers are
// given; an anchor outside [0, n_src) gives a padding row and sets kErrBounds)
cudaError_t launch_reuse_rows(int n, const int32_t* anchor, int n_src, const int32_t* src_idx, const float* src_score,
                              int32_t* dst_idx, float* dst_score, int* err, int num_sms, cudaStream_t s);

// ---------------------------------------------------------------- sparse MLA
// Attention of T queries (H <= 96 heads of 576 values) over the k_sel cache rows each query's
// idx row selects (positions inside its sequence, -1 = none); out bf16 [T, H, 512], lse
// fp32 [T, H] (natural log; -inf and zeros for a query with no token).
struct SparseMlaArgs {
  int T, B, H, k_sel;
  int64_t cache_rows;
  const void* q;                  // bf16 [T, H, 576]
  const void* kv_cache;           // bf16 [cache_rows, 576]
  const int64_t* cache_offsets;   // [B+1]
  const int32_t* q_seq_offsets;   // [B+1]
  const int32_t* idx;             // [T, k_sel]
  float scale;
  void* out;                      // bf16 [T, H, 512]
  float* lse;                     // [T, H]
  int* err;
  uint64_t timeout_ns;
};

cudaError_t launch_sparse_mla(const SparseMlaArgs& a, cudaStream_t s);

cudaError_t launch_wait_timeout_selftest(int* status, uint64_t timeout_ns, cudaStream_t s);

// Limit of every bounded pipeline wait in the library's kernels: 2 s, or
// DSA_INDEXER_WAIT_TIMEOUT_MS milliseconds when that variable is set (read once).
uint64_t wait_timeout_ns();

}  // namespace dsa
