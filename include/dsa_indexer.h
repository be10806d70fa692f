/*
 * dsa_indexer.h -- C ABI of the B200 (sm_100a) DSA lightning indexer.
 *
 * The operation (archdiff.com compare pages on Kimi K3.1 Pro, component table,
 * 'Sparse / compressed attn' row, Kimi K3.1 Pro column): every MLA layer owns an
 * indexer with 32 heads x 128 dims.  Per token t it forms
 *     q_t = q_latent_t W_q           (1,536 -> 4,096 = 32 heads x 128),
 *     k_t = LayerNorm(hidden_t W_k)  (7,168 -> 128, one key shared by all heads),
 *     w_t = hidden_t W_w             (7,168 -> 32 per-head weights),
 * scores every causal prior token s of its sequence with
 *     I[t,s] = sum_h w_t[h] * ReLU(q_t[h] . k_s)
 * and keeps the 2,048 highest-scoring tokens.  The key norm is a LayerNorm
 * ('QK-Clip and normalized latents; LayerNorm on the indexer key' row), no
 * rotary step is applied ('Partial RoPE / NoPE' row: index_rope_dim = 0), the
 * weights are BF16 ('FP8 -> FP4 training' row) and the whole prefix is scored
 * ('Long-context extension' row).
 *
 * Conventions for every entry point:
 *   - All tensor arguments are DEVICE pointers to caller-owned memory, 16-byte
 *     aligned, densely packed row-major.  bf16 tensors are passed as void*.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream).  Calls are
 *     asynchronous on that stream; the library never synchronises the host,
 *     except dsa_indexer_create / _destroy / _device_error.
 *   - Host-detectable argument errors return a status and launch nothing.
 *     Problems only the device can see set bits in the handle's device error
 *     word, which dsa_indexer_device_error() reports and clears: a position
 *     outside its sequence's key cache or malformed offsets (the affected
 *     output rows are written as padding), or a pipeline wait that ran out (the
 *     kernel leaves early; rows of unfinished work items are left unwritten).
 *   - A handle may be used from one stream and one host thread at a time (its
 *     workspace is shared by consecutive calls and ordered by that stream, and
 *     dsa_indexer_project forks part of its work onto a stream the handle owns
 *     and joins it back with two events the handle owns).
 */
#ifndef DSA_INDEXER_H
#define DSA_INDEXER_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define DSA_INDEXER_ABI_VERSION 2

typedef enum {
  DSA_OK = 0,
  DSA_ERR_INVALID_ARG = 1,    /* NULL/misaligned pointer, bad size, bad config */
  DSA_ERR_UNSUPPORTED = 2,    /* a valid request this library does not implement */
  DSA_ERR_CUDA = 3,           /* a CUDA runtime/driver call or a launch failed */
  DSA_ERR_OOM = 4,            /* device allocation failed at create */
  DSA_ERR_WORKSPACE = 5,      /* T exceeds the handle's max_tokens */
  DSA_ERR_DEVICE_TIMEOUT = 6, /* a bounded device-side wait ran out (kernel exited early) */
  DSA_ERR_DEVICE_BOUNDS = 7   /* a position / offset was outside its sequence's cache rows */
} dsa_status_t;

/* flags of dsa_indexer_topk */
#define DSA_TOPK_SORTED   1u  /* rows ordered by (score desc, position asc), padding last */
#define DSA_TOPK_SPLIT    2u  /* force the split-key path (one query per work item, key chunks merged) */
#define DSA_TOPK_NO_SPLIT 4u  /* never use the split-key path */

typedef struct dsa_indexer* dsa_indexer_t;

/* Create-time configuration.  head_dim = 128 and top_k = 2048; n_heads = 32
 * (Kimi K3.1 Pro) or 64 (the DeepSeek-V3.2 form: 'Sparse / compressed attn'
 * row, "DeepSeek-V3.2's indexer has 64 heads"); rope_dim = 0 (Kimi K3.1 Pro:
 * index_rope_dim = 0) or 64 ('Partial RoPE / NoPE' row of the page "Kimi K3.1
 * Pro vs Gemma 4 31B": DeepSeek-V3.2's indexer rotates 64 of its 128 dims).
 * Other values: DSA_ERR_UNSUPPORTED.  hidden_dim and q_latent_dim must be
 * positive multiples of 64 (hidden_dim >= 128 for n_heads = 64 or rope_dim > 0). */
typedef struct {
  int32_t hidden_dim;    /* 7168: width of the hidden state feeding W_k and W_w */
  int32_t q_latent_dim;  /* 1536: width of the MLA query latent feeding W_q */
  int32_t n_heads;       /* 32 (64: DeepSeek-V3.2 form) */
  int32_t head_dim;      /* 128 */
  int32_t top_k;         /* 2048 */
  float ln_eps;          /* LayerNorm epsilon of the key norm; 1e-6 by default */
  int64_t max_tokens;    /* largest T passed to _topk; sizes the handle's workspace */
  int32_t rope_dim;      /* 0, or 64: rotated dims at the start of q's heads and of k */
  float rope_theta;      /* rotary base: pair i of a token at position p turns by
                            p * rope_theta^(-2i / rope_dim); 10000 by default */
} dsa_indexer_config_t;

/* Fills *cfg with the Kimi K3.1 Pro indexer dimensions (above), rope_dim = 0,
 * rope_theta = 10000 and max_tokens = 131072. */
void dsa_indexer_default_config(dsa_indexer_config_t* cfg);

/* Creates a handle for one layer's indexer on the current CUDA device.
 * Weight pointers are device bf16 tensors stored (in x out), row-major:
 *   W_q [q_latent_dim, n_heads*head_dim]   (head h = columns h*128 .. h*128+127)
 *   (n_heads = 64: W_q [q_latent_dim, 8192], W_w [hidden_dim, 64])
 *   W_k [hidden_dim, head_dim], W_w [hidden_dim, n_heads],
 *   ln_gamma [head_dim], ln_beta [head_dim].
 * The weights are copied (re-laid out for the tensor cores) into memory the
 * handle owns; the caller may free its copies on return.  Synchronous.
 * Returns DSA_ERR_INVALID_ARG / _UNSUPPORTED / _OOM / _CUDA on failure, in
 * which case *out is left NULL. */
dsa_status_t dsa_indexer_create(const dsa_indexer_config_t* cfg, const void* W_q, const void* W_k,
                                const void* W_w, const void* ln_gamma, const void* ln_beta,
                                dsa_indexer_t* out);

/* Frees the handle and its device memory (synchronises the device first). */
dsa_status_t dsa_indexer_destroy(dsa_indexer_t h);

/* Projections of T tokens belonging to B sequences ('Sparse / compressed attn'
 * row: query latent 1,536 -> 4,096, hidden -> one LayerNorm'd 128-dim key,
 * hidden 7,168 -> 32 head weights).
 *   hidden        bf16 [T, hidden_dim]
 *   q_latent      bf16 [T, q_latent_dim]
 *   positions     int32 [T], position of token t inside its sequence
 *   q_seq_offsets int32 [B+1], tokens of sequence b are q_seq_offsets[b] .. [b+1]-1
 *   key_cache     bf16 [cache_rows, head_dim]; k_t is written to row
 *                 cache_offsets[b] + positions[t] (one 256-byte row per token)
 *   cache_rows    number of rows the key_cache allocation holds
 *   cache_offsets int64 [B+1], key-cache rows of sequence b are
 *                 cache_offsets[b] .. cache_offsets[b+1]-1, with
 *                 0 <= cache_offsets[b] <= cache_offsets[b+1] <= cache_rows
 *   q_out         bf16 [T, n_heads*head_dim] = bf16(q_latent W_q), fp32 accumulate
 *   w_out         fp32 [T, n_heads]          = hidden W_w, fp32 accumulate
 * The key is k = bf16(gamma * (x - mean) / sqrt(var + eps) + beta) with
 * x = hidden W_k kept in fp32 and the biased variance.  With rope_dim > 0 the
 * first rope_dim dims of every query head and of the normalised key turn, pair
 * (2i, 2i+1) by the angle positions[t] * rope_theta^(-2i / rope_dim), before
 * the bf16 rounding.  A token whose position
 * lies outside [0, rows of its sequence) gets no key row and sets
 * DSA_ERR_DEVICE_BOUNDS.  T = 0 is a no-op.  One call covers at most
 * 8,388,480 tokens (65,535 tiles of 128 rows): a larger T is refused at launch
 * and returns DSA_ERR_CUDA, so project longer inputs in several calls. */
dsa_status_t dsa_indexer_project(dsa_indexer_t h, int64_t T, const void* hidden, const void* q_latent,
                                 const int32_t* positions, const int32_t* q_seq_offsets, int32_t B,
                                 void* key_cache, int64_t cache_rows, const int64_t* cache_offsets, void* q_out,
                                 float* w_out, void* stream);

/* LayerNorm + bf16 cast of n pre-norm key rows (the key-norm step of the
 * projection on its own, for callers that compute hidden W_k elsewhere or fill
 * a cache from stored pre-norm keys).
 *   raw_keys fp32 [n, head_dim] -> keys_out bf16 [n, head_dim]. */
dsa_status_t dsa_indexer_key_norm(dsa_indexer_t h, int64_t n, const float* raw_keys, void* keys_out,
                                  void* stream);

/* Score + top-k of T query tokens ('Sparse / compressed attn' row: I = sum_h
 * w_h ReLU(q_h . k), top 2,048 per query; 'Long-context extension' row: the
 * whole causal prefix is scored).
 *   q          bf16 [T, n_heads, head_dim]   (as written by _project)
 *   w          fp32 [T, n_heads]
 *   positions, q_seq_offsets, B, cache_rows, cache_offsets: as for _project
 *   key_cache  bf16 [cache_rows, head_dim]
 *   idx_out    int32 [T, top_k]
 *   score_out  fp32 [T, top_k] or NULL
 * Query t at position p of sequence b scores keys s = 0..p (inclusive) read
 * from row cache_offsets[b] + s.  Indices are positions inside the sequence.
 * If p + 1 <= top_k the row is exactly [0, 1, ..., p, -1, ...] (scores in
 * the same order, -inf in the padding), with or without DSA_TOPK_SORTED.
 * Otherwise the row holds the top_k positions of highest score: in
 * unspecified order, or with DSA_TOPK_SORTED by score descending, then
 * position ascending.  Among exactly equal scores at the cut any subset may be
 * kept.  The T x S score matrix is never written to memory.
 * Flags: DSA_TOPK_SORTED, DSA_TOPK_SPLIT, DSA_TOPK_NO_SPLIT (default: the
 * split-key path when T <= 256).  A query whose position is outside its
 * sequence's cache rows gets an all-padding row and sets
 * DSA_ERR_DEVICE_BOUNDS; malformed offsets set it too, and then every output
 * row is padding.  Returns DSA_ERR_WORKSPACE if T or B exceeds max_tokens,
 * and DSA_ERR_UNSUPPORTED for DSA_TOPK_SPLIT with T > 256. */
dsa_status_t dsa_indexer_topk(dsa_indexer_t h, int64_t T, const void* q, const float* w,
                              const int32_t* positions, const int32_t* q_seq_offsets, int32_t B,
                              const void* key_cache, int64_t cache_rows, const int64_t* cache_offsets,
                              int32_t* idx_out,
                              float* score_out, uint32_t flags, void* stream);

/* ---- FP8 indexer-key cache ('FP8 -> FP4 training' row of the page "Kimi K3.1
 * Pro vs GLM-5": vLLM and SGLang cache the indexer keys in FP8 by default).
 * The key cache holds FP8 e4m3 codes [cache_rows, head_dim] (one byte each,
 * 128-byte rows) and one fp32 scale per row; queries hold e4m3 codes
 * [T, n_heads, head_dim] and one fp32 scale per (token, head).  A row x of
 * float values is stored as scale = amax / 448 (0 for an all-zero row) and
 * codes e4m3(x * (448 / amax)), rounded to nearest even with saturation; the
 * value represented is code * scale.  x is the bf16 key (after the LayerNorm)
 * or the bf16 query head, so the FP8 cache stores what the bf16 path would,
 * rounded once more.  Scores become
 *     I[t,s] = key_scale[s] * sum_h (w[t,h] * q_scale[t,h]) * ReLU(q8[t,h] . k8[s])
 * (the positive scales factor out of the ReLU), computed on the tensor cores
 * with kind::f8f6f4 MMAs; decode reads 132 bytes per cached key instead of 256.
 * Requires hidden_dim >= 128, n_heads = 32 and rope_dim = 0 (the Kimi K3.1 form;
 * DSA_ERR_UNSUPPORTED otherwise). */

/* dsa_indexer_project with FP8 outputs: key_cache_fp8 uint8 [cache_rows, head_dim]
 * and key_scale fp32 [cache_rows] receive the token's key row; q_fp8 uint8
 * [T, n_heads*head_dim] and q_scale fp32 [T, n_heads] the query; w_out as for
 * dsa_indexer_project.  Other arguments and rules as for dsa_indexer_project. */
dsa_status_t dsa_indexer_project_fp8(dsa_indexer_t h, int64_t T, const void* hidden, const void* q_latent,
                                     const int32_t* positions, const int32_t* q_seq_offsets, int32_t B,
                                     void* key_cache_fp8, float* key_scale, int64_t cache_rows,
                                     const int64_t* cache_offsets, void* q_fp8, float* q_scale, float* w_out,
                                     void* stream);

/* FP8 codes and scales of n bf16 key rows keys [n, head_dim] (e.g. an existing
 * bf16 cache, or the output of dsa_indexer_key_norm): key_cache_fp8 uint8
 * [n, head_dim], key_scale fp32 [n]. */
dsa_status_t dsa_indexer_quantize_keys_fp8(dsa_indexer_t h, int64_t n, const void* keys, void* key_cache_fp8,
                                           float* key_scale, void* stream);

/* dsa_indexer_topk over an FP8 cache: q_fp8 uint8 [T, n_heads, head_dim] with
 * q_scale fp32 [T, n_heads], key_cache_fp8 uint8 [cache_rows, head_dim] with
 * key_scale fp32 [cache_rows]; scores as above.  Every other argument, flag,
 * output rule and error as for dsa_indexer_topk. */
dsa_status_t dsa_indexer_topk_fp8(dsa_indexer_t h, int64_t T, const void* q_fp8, const float* q_scale, const float* w,
                                  const int32_t* positions, const int32_t* q_seq_offsets, int32_t B,
                                  const void* key_cache_fp8, const float* key_scale, int64_t cache_rows,
                                  const int64_t* cache_offsets, int32_t* idx_out, float* score_out, uint32_t flags,
                                  void* stream);

/* Index reuse across speculative draft steps ('MTP' row of the page "Kimi K3.1
 * Pro vs GLM-5": GLM-5.2 reuses the first step's top-k indices in its later
 * draft steps).  Draft token d takes the selection of its anchor: row
 * anchor_rows[d] of a [n_src, top_k] result of dsa_indexer_topk (the first
 * step's queries), copied bit for bit.
 *   anchor_rows int32 [n_draft], each in [0, n_src)
 *   src_idx     int32 [n_src, top_k];  src_score fp32 [n_src, top_k] or NULL
 *   idx_out     int32 [n_draft, top_k]; score_out fp32 [n_draft, top_k] or NULL
 *               (scores are copied when both score pointers are given; giving
 *               only one of them is DSA_ERR_INVALID_ARG)
 * The output must not overlap the source.  An anchor outside [0, n_src) gives
 * an all-padding row (-1, -inf) and sets DSA_ERR_DEVICE_BOUNDS.  Asynchronous on
 * `stream`; n_draft = 0 is a no-op. */
dsa_status_t dsa_indexer_topk_reuse(dsa_indexer_t h, int64_t n_draft, const int32_t* anchor_rows, int64_t n_src,
                                    const int32_t* src_idx, const float* src_score, int32_t* idx_out,
                                    float* score_out, void* stream);

/* Allocation-free score + top-k (no counterpart on the pages; it exists for the
 * library's users).  Some callers cannot let a library allocate device memory:
 * a framework whose memory pool already holds the device's whole budget, or a
 * latency-critical loop that must never pay for cudaMalloc / cudaFree and the
 * device synchronisation they can imply.  This entry point needs no handle and
 * calls no allocator: its scratch is a fixed array in the library's static
 * device memory, 6,473,216 bytes (6.2 MiB), which every GPU that loads the library holds until the
 * process exits.  The caller still passes every input and output, as for
 * dsa_indexer_topk (same arguments without handle and flags; same output rules;
 * the prefill path of dsa_indexer_topk with DSA_TOPK_NO_SPLIT).
 * Limits: T <= 4096 and B <= 4096 (otherwise DSA_ERR_WORKSPACE); the kernels run
 * on at most 8 SMs (the scratch holds 8 per-SM candidate areas), so this is
 * slower than dsa_indexer_topk.  Device-side problems follow dsa_indexer_topk's
 * rules (bad positions or offsets: padded rows; a wait that ran out: unfinished
 * rows unwritten) and are recorded in an error word inside the scratch, which
 * dsa_indexer_noalloc_device_error() reads.
 * Every call looks up the scratch's device address with the caller's device
 * current; the first call on a device also loads the library's device code there,
 * so make that first call before any stream capture.  All calls on a device share
 * the one scratch array, which keeps the previous call's contents (each call clears
 * what must start at zero, its error word included): calls whose kernels can
 * overlap on the GPU (e.g. on unordered streams) race and corrupt each other's
 * results; order them on one stream. */
dsa_status_t dsa_indexer_topk_noalloc(int64_t T, const void* q, const float* w, const int32_t* positions,
                                      const int32_t* q_seq_offsets, int32_t B, const void* key_cache,
                                      int64_t cache_rows, const int64_t* cache_offsets, int32_t* idx_out,
                                      float* score_out, void* stream);

/* Synchronises `stream`, then returns the device-side status recorded by the
 * last dsa_indexer_topk_noalloc call on the current device: DSA_OK,
 * DSA_ERR_DEVICE_BOUNDS or DSA_ERR_DEVICE_TIMEOUT (allocates nothing; no
 * counterpart on the pages, as for dsa_indexer_topk_noalloc). */
dsa_status_t dsa_indexer_noalloc_device_error(void* stream);

/* Sparse MLA attention over the indexer's selection ('Latent attention (MLA)' row of
 * the pages "Qwen3.5-397B-A17B vs Kimi K3.1 Pro" and "Kimi K3.1 Pro vs Gemma 4 31B":
 * 96 heads; keys and values come from a 512-dim latent plus a 64-dim shared key slot, 576
 * cached values per token; each query attends only to the 2,048 tokens the indexer
 * selects).  It runs in the latent ("absorbed") form: a head's query is 576 values (its
 * no-rope part already taken into the latent space), the score of a selected token s is
 *     x[h,s] = scale * (q[t,h] . kv[s])          over all 576 values,
 * and the value is the row's first 512 values (the latent):
 *     out[t,h] = sum_s softmax_s(x[h,.]) * kv[s][0..511],   lse[t,h] = ln sum_s exp(x[h,s]).
 *   q             bf16 [T, n_heads, 576], n_heads in 1..96
 *   kv_cache      bf16 [cache_rows, 576]; token s of sequence b is row cache_offsets[b] + s
 *   cache_offsets int64 [B+1], q_seq_offsets int32 [B+1]: as for dsa_indexer_project
 *   idx           int32 [T, k_sel]: positions inside the query's sequence, -1 = no token
 *                 (the idx_out of dsa_indexer_topk, k_sel = top_k); a position may repeat
 *                 and then counts once per entry; k_sel <= 2,048 (larger:
 *                 DSA_ERR_UNSUPPORTED); k_sel = 0 (idx may be NULL) gives every query no token
 *   scale         > 0 (e.g. 1/sqrt(192) for 128 + 64-dim query/key heads)
 *   out           bf16 [T, n_heads, 512];  lse fp32 [T, n_heads]
 * A query with no valid entry gets out = 0 and lse = -inf.  An entry at or past its
 * sequence's row count is skipped and sets DSA_ERR_DEVICE_BOUNDS; malformed offsets set it
 * too and give the affected queries no token.  Scores and the softmax weights' sum are
 * fp32; the weights multiply the latent as bf16 (fp32 accumulate).  T = 0 is a no-op;
 * asynchronous on `stream`. */
dsa_status_t dsa_indexer_sparse_mla(dsa_indexer_t h, int64_t T, const void* q, int32_t n_heads, const void* kv_cache,
                                    int64_t cache_rows, const int64_t* cache_offsets, const int32_t* q_seq_offsets,
                                    int32_t B, const int32_t* idx, int32_t k_sel, float scale, void* out, float* lse,
                                    void* stream);

/* Synchronises the device, then returns DSA_OK or the first device-side error
 * recorded since the last call (DSA_ERR_DEVICE_BOUNDS, DSA_ERR_DEVICE_TIMEOUT)
 * and clears the error word. */
dsa_status_t dsa_indexer_device_error(dsa_indexer_t h);

/* Launches one kernel that waits on a barrier nothing will ever signal, with a
 * device-side limit of timeout_ns nanoseconds, synchronises the stream and
 * returns the status the kernel reported: DSA_ERR_DEVICE_TIMEOUT when the
 * bounded wait works.  Used to test the failure path without hanging a GPU. */
dsa_status_t dsa_indexer_selftest_wait_timeout(int64_t timeout_ns, void* stream);

/* Human-readable name of a status code (static storage). */
const char* dsa_indexer_status_string(dsa_status_t s);

/* DSA_INDEXER_ABI_VERSION of the loaded library. */
int32_t dsa_indexer_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* DSA_INDEXER_H */
