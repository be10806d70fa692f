// api.cu -- the C ABI declared in include/dsa_indexer.h: handle life cycle,
// argument validation, TMA descriptor encoding, and the kernel launches.

#include <cudaTypedefs.h>

#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <vector>

#include "../../include/dsa_indexer.h"
#include "kernels.h"

using namespace dsa;

uint64_t dsa::wait_timeout_ns() {
  static const uint64_t t = [] {
    const char* s = std::getenv("DSA_INDEXER_WAIT_TIMEOUT_MS");
    if (s && *s) {
      const long long v = std::atoll(s);
      if (v > 0) return static_cast<uint64_t>(v) * uint64_t(1000000);
    }
    return static_cast<uint64_t>(2000ull * 1000 * 1000);
  }();
  return t;
}

namespace {

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

bool load_encode() {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  return g_encode != nullptr;
}

// 2-D bf16 (or, with `bytes`, 1-byte FP8) tensor [rows, inner] (row-major, dense rows),
// 128-byte swizzled boxes of box_inner x box_rows elements.
bool make_tmap(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint32_t box_inner,
               uint32_t box_rows, bool bytes = false) {
  if (!load_encode()) return false;
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {inner * (bytes ? 1 : 2)};
  cuuint32_t box[2] = {box_inner, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = g_encode(m, bytes ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                        const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

uint64_t timeout_ns() { return dsa::wait_timeout_ns(); }

}  // namespace

struct dsa_indexer {
  dsa_indexer_config_t cfg;
  int device = 0;
  int num_sms = 0;
  __nv_bfloat16* WqT = nullptr;   // [n_heads*head_dim, q_latent_dim]
  __nv_bfloat16* WkwT = nullptr;  // [head_dim + n_heads, hidden_dim]
  float* gamma = nullptr;         // [head_dim]
  float* beta = nullptr;
  double* inv_freq = nullptr;     // [32] rotary frequencies (rope_dim > 0)
  CUtensorMap tm_WqT, tm_WkwT;
  TopkWorkspace ws{};
  std::vector<void*> allocs;
  // dsa_indexer_project runs the k|w GEMM (HBM-bound) on `side` next to the q GEMM
  // (tensor-bound) on the caller's stream, forked and joined with the two events
  cudaStream_t side = nullptr;
  cudaEvent_t ev_fork = nullptr, ev_join = nullptr;

  template <class T>
  bool alloc(T** p, size_t count) {
    void* q = nullptr;
    if (cudaMalloc(&q, count * sizeof(T) + 16) != cudaSuccess) return false;
    allocs.push_back(q);
    *p = static_cast<T*>(q);
    return true;
  }
  ~dsa_indexer() {
    if (ev_fork) cudaEventDestroy(ev_fork);
    if (ev_join) cudaEventDestroy(ev_join);
    if (side) cudaStreamDestroy(side);
    for (void* p : allocs) cudaFree(p);
  }
};

extern "C" {

void dsa_indexer_default_config(dsa_indexer_config_t* cfg) {
  if (!cfg) return;
  cfg->hidden_dim = 7168;
  cfg->q_latent_dim = 1536;
  cfg->n_heads = 32;
  cfg->head_dim = 128;
  cfg->top_k = 2048;
  cfg->ln_eps = 1e-6f;
  cfg->max_tokens = 131072;
  cfg->rope_dim = 0;
  cfg->rope_theta = 10000.f;
}

int32_t dsa_indexer_abi_version(void) { return DSA_INDEXER_ABI_VERSION; }

const char* dsa_indexer_status_string(dsa_status_t s) {
  switch (s) {
    case DSA_OK: return "DSA_OK";
    case DSA_ERR_INVALID_ARG: return "DSA_ERR_INVALID_ARG";
    case DSA_ERR_UNSUPPORTED: return "DSA_ERR_UNSUPPORTED";
    case DSA_ERR_CUDA: return "DSA_ERR_CUDA";
    case DSA_ERR_OOM: return "DSA_ERR_OOM";
    case DSA_ERR_WORKSPACE: return "DSA_ERR_WORKSPACE";
    case DSA_ERR_DEVICE_TIMEOUT: return "DSA_ERR_DEVICE_TIMEOUT";
    case DSA_ERR_DEVICE_BOUNDS: return "DSA_ERR_DEVICE_BOUNDS";
  }
  return "DSA_ERR_UNKNOWN";
}

dsa_status_t dsa_indexer_create(const dsa_indexer_config_t* cfg, const void* W_q, const void* W_k, const void* W_w,
                                const void* ln_gamma, const void* ln_beta, dsa_indexer_t* out) {
  if (!out) return DSA_ERR_INVALID_ARG;
  *out = nullptr;
  if (!cfg || !W_q || !W_k || !W_w || !ln_gamma || !ln_beta) return DSA_ERR_INVALID_ARG;
  if (cfg->hidden_dim <= 0 || cfg->q_latent_dim <= 0 || cfg->max_tokens <= 0 || !(cfg->ln_eps >= 0.f) ||
      !std::isfinite(cfg->ln_eps))
    return DSA_ERR_INVALID_ARG;
  if (cfg->hidden_dim % 64 || cfg->q_latent_dim % 64) return DSA_ERR_INVALID_ARG;
  if (cfg->max_tokens > (int64_t(1) << 26)) return DSA_ERR_INVALID_ARG;
  if ((cfg->n_heads != 32 && cfg->n_heads != 64) || cfg->head_dim != kHeadDim || cfg->top_k != kTopK ||
      (cfg->rope_dim != 0 && cfg->rope_dim != 64))
    return DSA_ERR_UNSUPPORTED;
  if (cfg->rope_dim > 0 && !(cfg->rope_theta > 1.f && std::isfinite(cfg->rope_theta))) return DSA_ERR_INVALID_ARG;
  if ((cfg->n_heads == 64 || cfg->rope_dim > 0) && cfg->hidden_dim < 128) return DSA_ERR_UNSUPPORTED;
  if (!aligned16(W_q) || !aligned16(W_k) || !aligned16(W_w) || !aligned16(ln_gamma) || !aligned16(ln_beta))
    return DSA_ERR_INVALID_ARG;
  if (!load_encode()) return DSA_ERR_CUDA;

  dsa_indexer* h = new dsa_indexer();
  h->cfg = *cfg;
  if (cudaGetDevice(&h->device) != cudaSuccess ||
      cudaDeviceGetAttribute(&h->num_sms, cudaDevAttrMultiProcessorCount, h->device) != cudaSuccess) {
    delete h;
    return DSA_ERR_CUDA;
  }
  const int H = cfg->n_heads, D = kHeadDim, HD = cfg->hidden_dim, QL = cfg->q_latent_dim;
  const int64_t T = cfg->max_tokens;
  bool ok = h->alloc(&h->WqT, size_t(H) * D * QL) && h->alloc(&h->WkwT, size_t(D + H) * HD) &&
            h->alloc(&h->gamma, D) && h->alloc(&h->beta, D) && h->alloc(&h->inv_freq, 32);
  TopkWorkspace& ws = h->ws;
  ws.part_tokens = static_cast<int>(T < kSplitMaxTokens ? T : kSplitMaxTokens);
  ws.max_items = static_cast<int>(T > ws.part_tokens * kMaxChunks ? T : ws.part_tokens * kMaxChunks) + 16;
  ws.cand_slots = h->num_sms;
  ok = ok && h->alloc(&ws.items, ws.max_items) && h->alloc(&ws.n_items, 4) && h->alloc(&ws.work_counter, 4) &&
       h->alloc(&ws.seq_base, size_t(T) + 2) && h->alloc(&ws.pos_eff, size_t(T)) &&
       h->alloc(&ws.tok_nchunks, size_t(T)) &&
       h->alloc(&ws.cand, size_t(ws.cand_slots) * kPrefillQ * kCandStride) &&
       h->alloc(&ws.part_keys, size_t(ws.part_tokens) * kMaxChunks * kTopK) &&
       h->alloc(&ws.part_idx, size_t(ws.part_tokens) * kMaxChunks * kTopK) &&
       h->alloc(&ws.part_hist, size_t(ws.part_tokens) * 2048) && h->alloc(&ws.err, 4);
  if (!ok) {
    delete h;
    return DSA_ERR_OOM;
  }
  if (cudaStreamCreateWithFlags(&h->side, cudaStreamNonBlocking) != cudaSuccess ||
      cudaEventCreateWithFlags(&h->ev_fork, cudaEventDisableTiming) != cudaSuccess ||
      cudaEventCreateWithFlags(&h->ev_join, cudaEventDisableTiming) != cudaSuccess) {
    delete h;
    return DSA_ERR_CUDA;
  }
  cudaStream_t s = nullptr;
  cudaError_t e = cudaMemset(ws.err, 0, sizeof(int));
  // the merge of the split-key path clears the counts it used; they start at zero
  if (e == cudaSuccess) e = cudaMemset(ws.part_hist, 0, size_t(ws.part_tokens) * 2048 * sizeof(uint32_t));
  // tensor-core layouts: W_q^T [4096, QL]; [W_k | W_w]^T [160, HD]
  if (e == cudaSuccess) e = launch_transpose_bf16(static_cast<const __nv_bfloat16*>(W_q), QL, H * D, h->WqT, 0, s);
  if (e == cudaSuccess) e = launch_transpose_bf16(static_cast<const __nv_bfloat16*>(W_k), HD, D, h->WkwT, 0, s);
  if (e == cudaSuccess) e = launch_transpose_bf16(static_cast<const __nv_bfloat16*>(W_w), HD, H, h->WkwT, D, s);
  if (e == cudaSuccess) e = cudaDeviceSynchronize();
  if (e == cudaSuccess) {
    uint16_t gb[2 * kHeadDim];
    e = cudaMemcpy(gb, ln_gamma, D * 2, cudaMemcpyDeviceToHost);
    if (e == cudaSuccess) e = cudaMemcpy(gb + D, ln_beta, D * 2, cudaMemcpyDeviceToHost);
    if (e == cudaSuccess) {
      float gf[2 * kHeadDim];
      for (int i = 0; i < 2 * D; ++i) {
        const uint32_t u = static_cast<uint32_t>(gb[i]) << 16;
        std::memcpy(&gf[i], &u, 4);
      }
      e = cudaMemcpy(h->gamma, gf, D * 4, cudaMemcpyHostToDevice);
      if (e == cudaSuccess) e = cudaMemcpy(h->beta, gf + D, D * 4, cudaMemcpyHostToDevice);
    }
  }
  if (e == cudaSuccess) {
    // rotary frequencies theta^(-2i / rope_dim), in double precision
    double f[32] = {};
    for (int i = 0; i < 32 && cfg->rope_dim > 0; ++i)
      f[i] = std::pow(static_cast<double>(cfg->rope_theta), -2.0 * i / cfg->rope_dim);
    e = cudaMemcpy(h->inv_freq, f, sizeof(f), cudaMemcpyHostToDevice);
  }
  if (e != cudaSuccess) {
    delete h;
    return DSA_ERR_CUDA;
  }
  if (!make_tmap(&h->tm_WqT, h->WqT, QL, uint64_t(H) * D, 64, 256) ||
      !make_tmap(&h->tm_WkwT, h->WkwT, HD, uint64_t(D + H), 64, D + H)) {
    delete h;
    return DSA_ERR_CUDA;
  }
  *out = h;
  return DSA_OK;
}

dsa_status_t dsa_indexer_destroy(dsa_indexer_t h) {
  if (!h) return DSA_ERR_INVALID_ARG;
  cudaDeviceSynchronize();
  delete h;
  return DSA_OK;
}

}  // extern "C"

namespace {

// Shared body of dsa_indexer_project and dsa_indexer_project_fp8: key_cache / q_out are bf16
// for the former; key8 + key_scale and q8 + q_scale for the latter.
dsa_status_t project_impl(dsa_indexer_t h, int64_t T, const void* hidden, const void* q_latent,
                          const int32_t* positions, const int32_t* q_seq_offsets, int32_t B, void* key_cache,
                          float* key_scale, int64_t cache_rows, const int64_t* cache_offsets, void* q_out,
                          float* q_scale, float* w_out, void* stream, bool fp8) {
  if (!h) return DSA_ERR_INVALID_ARG;
  if (T < 0 || T > (int64_t(1) << 26) || B < 1) return DSA_ERR_INVALID_ARG;
  if (T == 0) return DSA_OK;
  if (!hidden || !q_latent || !positions || !q_seq_offsets || !key_cache || !cache_offsets || !q_out || !w_out)
    return DSA_ERR_INVALID_ARG;
  if (fp8 && (!key_scale || !q_scale || (reinterpret_cast<uintptr_t>(key_scale) & 3) ||
              (reinterpret_cast<uintptr_t>(q_scale) & 3)))
    return DSA_ERR_INVALID_ARG;
  if (!aligned16(hidden) || !aligned16(q_latent) || !aligned16(key_cache) || !aligned16(q_out) ||
      !aligned16(w_out) || (reinterpret_cast<uintptr_t>(positions) & 3) ||
      (reinterpret_cast<uintptr_t>(q_seq_offsets) & 3) || (reinterpret_cast<uintptr_t>(cache_offsets) & 7))
    return DSA_ERR_INVALID_ARG;
  if (cache_rows < 1 || cache_rows > (int64_t(1) << 31) - (int64_t(1) << 20)) return DSA_ERR_INVALID_ARG;
  const dsa_indexer_config_t& c = h->cfg;
  // FP8: the K3.1 form (32 heads, no rotary step), whose key epilogue is the split-K one
  if (fp8 && (c.hidden_dim < 128 || c.n_heads != 32 || c.rope_dim != 0)) return DSA_ERR_UNSUPPORTED;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  CUtensorMap tmX, tmQL;
  if (!make_tmap(&tmX, hidden, c.hidden_dim, uint64_t(T), 64, 128) ||
      !make_tmap(&tmQL, q_latent, c.q_latent_dim, uint64_t(T), 64, 128))
    return DSA_ERR_INVALID_ARG;
  ProjKwEpilogue e{};
  e.M = static_cast<int>(T);
  e.key_cache = fp8 ? nullptr : static_cast<__nv_bfloat16*>(key_cache);
  e.key8 = fp8 ? static_cast<uint8_t*>(key_cache) : nullptr;
  e.key_scale = fp8 ? key_scale : nullptr;
  e.cache_rows = cache_rows;
  e.w_out = w_out;
  e.positions = positions;
  e.q_seq_offsets = q_seq_offsets;
  e.B = B;
  e.cache_offsets = cache_offsets;
  e.n_heads = c.n_heads;
  e.rope_dim = c.rope_dim;
  e.inv_freq = h->inv_freq;
  e.gamma = h->gamma;
  e.beta = h->beta;
  e.eps = c.ln_eps;
  e.err = h->ws.err;
  e.timeout_ns = timeout_ns();
  // k|w on the handle's side stream, q on the caller's; both ordered after the caller's
  // earlier work, and the caller's later work after both
  if (cudaEventRecord(h->ev_fork, s) != cudaSuccess || cudaStreamWaitEvent(h->side, h->ev_fork, 0) != cudaSuccess)
    return DSA_ERR_CUDA;
  const cudaError_t ekw = launch_proj_kw(tmX, h->tm_WkwT, c.hidden_dim, e, h->side);
  const cudaError_t eq =
      fp8 ? launch_proj_q8(tmQL, h->tm_WqT, static_cast<int>(T), c.q_latent_dim, kHeads * kHeadDim,
                           static_cast<uint8_t*>(q_out), q_scale, h->ws.err, timeout_ns(), s)
          : launch_proj_q(tmQL, h->tm_WqT, static_cast<int>(T), c.q_latent_dim, c.n_heads * kHeadDim,
                          static_cast<__nv_bfloat16*>(q_out), h->ws.err, timeout_ns(), s, positions, h->inv_freq,
                          c.rope_dim);
  // join even if a launch failed, so that the side stream never runs ahead unordered
  if (cudaEventRecord(h->ev_join, h->side) != cudaSuccess || cudaStreamWaitEvent(s, h->ev_join, 0) != cudaSuccess)
    return DSA_ERR_CUDA;
  if (ekw != cudaSuccess || eq != cudaSuccess) return DSA_ERR_CUDA;
  return DSA_OK;
}

// Shared body of dsa_indexer_topk and dsa_indexer_topk_fp8.
dsa_status_t topk_impl(dsa_indexer_t h, int64_t T, const void* q, const float* q_scale, const float* w,
                       const int32_t* positions, const int32_t* q_seq_offsets, int32_t B, const void* key_cache,
                       const float* key_scale, int64_t cache_rows, const int64_t* cache_offsets, int32_t* idx_out,
                       float* score_out, uint32_t flags, void* stream, bool fp8) {
  if (!h) return DSA_ERR_INVALID_ARG;
  if (T < 0 || B < 1) return DSA_ERR_INVALID_ARG;
  if ((flags & DSA_TOPK_SPLIT) && (flags & DSA_TOPK_NO_SPLIT)) return DSA_ERR_INVALID_ARG;
  if (flags & ~(DSA_TOPK_SORTED | DSA_TOPK_SPLIT | DSA_TOPK_NO_SPLIT)) return DSA_ERR_INVALID_ARG;
  if (T == 0) return DSA_OK;
  if (T > h->cfg.max_tokens || B > h->cfg.max_tokens) return DSA_ERR_WORKSPACE;
  if (!q || !w || !positions || !q_seq_offsets || !key_cache || !cache_offsets || !idx_out) return DSA_ERR_INVALID_ARG;
  if (fp8 && (!q_scale || !key_scale || (reinterpret_cast<uintptr_t>(q_scale) & 3) ||
              (reinterpret_cast<uintptr_t>(key_scale) & 3)))
    return DSA_ERR_INVALID_ARG;
  const int H = h->cfg.n_heads;
  if (fp8 && H != 32) return DSA_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(w) || !aligned16(key_cache) || !aligned16(idx_out) ||
      (score_out && !aligned16(score_out)) || (reinterpret_cast<uintptr_t>(positions) & 3) ||
      (reinterpret_cast<uintptr_t>(q_seq_offsets) & 3) || (reinterpret_cast<uintptr_t>(cache_offsets) & 7))
    return DSA_ERR_INVALID_ARG;
  if (cache_rows < 1 || cache_rows > (int64_t(1) << 31) - (int64_t(1) << 20)) return DSA_ERR_INVALID_ARG;
  bool split = (T <= kSplitMaxTokens);
  if (flags & DSA_TOPK_SPLIT) {
    if (T > h->ws.part_tokens) return DSA_ERR_UNSUPPORTED;
    split = true;
  }
  if (flags & DSA_TOPK_NO_SPLIT) split = false;
  if (split && T > h->ws.part_tokens) split = false;
  // a box row is 128 bytes: 64 bf16 (two boxes per 128-dim row) or 128 FP8 codes (one)
  const uint32_t bi = fp8 ? 128 : 64;
  CUtensorMap tmQ1, tmQ8, tmK;
  // an item of the prefill path holds 256 (query, head) rows: 8 queries of 32 heads or 4 of 64
  if (!make_tmap(&tmQ1, q, kHeadDim, uint64_t(T) * H, bi, H, fp8) ||
      !make_tmap(&tmQ8, q, kHeadDim, uint64_t(T) * H, bi, 256, fp8) ||
      !make_tmap(&tmK, key_cache, kHeadDim, uint64_t(cache_rows), bi, kKeyTile, fp8))
    return DSA_ERR_INVALID_ARG;
  TopkArgs a{};
  a.T = static_cast<int>(T);
  a.B = B;
  a.cache_rows = cache_rows;
  a.q = static_cast<const __nv_bfloat16*>(q);
  a.w = w;
  a.positions = positions;
  a.q_seq_offsets = q_seq_offsets;
  a.key_cache = static_cast<const __nv_bfloat16*>(key_cache);
  a.cache_offsets = cache_offsets;
  a.idx_out = idx_out;
  a.score_out = score_out;
  a.split = split;
  a.sorted = (flags & DSA_TOPK_SORTED) != 0;
  a.fp8 = fp8;
  a.heads = H;
  a.q_scale = fp8 ? q_scale : nullptr;
  a.key_scale = fp8 ? key_scale : nullptr;
  a.timeout_ns = timeout_ns();
  if (launch_topk(a, h->ws, tmQ1, tmQ8, tmK, h->num_sms, static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return DSA_ERR_CUDA;
  return DSA_OK;
}

}  // namespace

extern "C" {

dsa_status_t dsa_indexer_project(dsa_indexer_t h, int64_t T, const void* hidden, const void* q_latent,
                                 const int32_t* positions, const int32_t* q_seq_offsets, int32_t B, void* key_cache,
                                 int64_t cache_rows, const int64_t* cache_offsets, void* q_out, float* w_out,
                                 void* stream) {
  return project_impl(h, T, hidden, q_latent, positions, q_seq_offsets, B, key_cache, nullptr, cache_rows,
                      cache_offsets, q_out, nullptr, w_out, stream, false);
}

dsa_status_t dsa_indexer_project_fp8(dsa_indexer_t h, int64_t T, const void* hidden, const void* q_latent,
                                     const int32_t* positions, const int32_t* q_seq_offsets, int32_t B,
                                     void* key_cache_fp8, float* key_scale, int64_t cache_rows,
                                     const int64_t* cache_offsets, void* q_fp8, float* q_scale, float* w_out,
                                     void* stream) {
  return project_impl(h, T, hidden, q_latent, positions, q_seq_offsets, B, key_cache_fp8, key_scale, cache_rows,
                      cache_offsets, q_fp8, q_scale, w_out, stream, true);
}

dsa_status_t dsa_indexer_quantize_keys_fp8(dsa_indexer_t h, int64_t n, const void* keys, void* key_cache_fp8,
                                           float* key_scale, void* stream) {
  if (!h || n < 0) return DSA_ERR_INVALID_ARG;
  if (n == 0) return DSA_OK;
  if (!keys || !key_cache_fp8 || !key_scale || !aligned16(keys) || !aligned16(key_cache_fp8) ||
      (reinterpret_cast<uintptr_t>(key_scale) & 3) || n > (int64_t(1) << 34))
    return DSA_ERR_INVALID_ARG;
  if (launch_quantize_keys_fp8(n, static_cast<const __nv_bfloat16*>(keys), static_cast<uint8_t*>(key_cache_fp8),
                               key_scale, static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return DSA_ERR_CUDA;
  return DSA_OK;
}

dsa_status_t dsa_indexer_key_norm(dsa_indexer_t h, int64_t n, const float* raw_keys, void* keys_out, void* stream) {
  if (!h || n < 0) return DSA_ERR_INVALID_ARG;
  if (n == 0) return DSA_OK;
  if (!raw_keys || !keys_out || !aligned16(raw_keys) || !aligned16(keys_out)) return DSA_ERR_INVALID_ARG;
  if (n > (int64_t(1) << 34)) return DSA_ERR_INVALID_ARG;
  if (launch_key_norm(n, raw_keys, static_cast<__nv_bfloat16*>(keys_out), h->gamma, h->beta, h->cfg.ln_eps,
                      static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return DSA_ERR_CUDA;
  return DSA_OK;
}

dsa_status_t dsa_indexer_topk(dsa_indexer_t h, int64_t T, const void* q, const float* w, const int32_t* positions,
                              const int32_t* q_seq_offsets, int32_t B, const void* key_cache, int64_t cache_rows,
                              const int64_t* cache_offsets, int32_t* idx_out, float* score_out, uint32_t flags,
                              void* stream) {
  return topk_impl(h, T, q, nullptr, w, positions, q_seq_offsets, B, key_cache, nullptr, cache_rows, cache_offsets,
                   idx_out, score_out, flags, stream, false);
}

dsa_status_t dsa_indexer_topk_fp8(dsa_indexer_t h, int64_t T, const void* q_fp8, const float* q_scale, const float* w,
                                  const int32_t* positions, const int32_t* q_seq_offsets, int32_t B,
                                  const void* key_cache_fp8, const float* key_scale, int64_t cache_rows,
                                  const int64_t* cache_offsets, int32_t* idx_out, float* score_out, uint32_t flags,
                                  void* stream) {
  return topk_impl(h, T, q_fp8, q_scale, w, positions, q_seq_offsets, B, key_cache_fp8, key_scale, cache_rows,
                   cache_offsets, idx_out, score_out, flags, stream, true);
}

dsa_status_t dsa_indexer_topk_reuse(dsa_indexer_t h, int64_t n_draft, const int32_t* anchor_rows, int64_t n_src,
                                    const int32_t* src_idx, const float* src_score, int32_t* idx_out,
                                    float* score_out, void* stream) {
  if (!h || n_draft < 0 || n_src < 0) return DSA_ERR_INVALID_ARG;
  if (n_draft == 0) return DSA_OK;
  if (n_draft > (int64_t(1) << 30) || n_src > (int64_t(1) << 30)) return DSA_ERR_INVALID_ARG;
  if (!anchor_rows || !src_idx || !idx_out || n_src == 0) return DSA_ERR_INVALID_ARG;
  if ((score_out != nullptr) != (src_score != nullptr)) return DSA_ERR_INVALID_ARG;
  if (!aligned16(src_idx) || !aligned16(idx_out) || (src_score && !aligned16(src_score)) ||
      (score_out && !aligned16(score_out)) || (reinterpret_cast<uintptr_t>(anchor_rows) & 3))
    return DSA_ERR_INVALID_ARG;
  if (launch_reuse_rows(static_cast<int>(n_draft), anchor_rows, static_cast<int>(n_src), src_idx, src_score, idx_out,
                        score_out, h->ws.err, h->num_sms, static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return DSA_ERR_CUDA;
  return DSA_OK;
}

dsa_status_t dsa_indexer_sparse_mla(dsa_indexer_t h, int64_t T, const void* q, int32_t n_heads, const void* kv_cache,
                                    int64_t cache_rows, const int64_t* cache_offsets, const int32_t* q_seq_offsets,
                                    int32_t B, const int32_t* idx, int32_t k_sel, float scale, void* out, float* lse,
                                    void* stream) {
  if (!h || T < 0 || B < 1 || k_sel < 0) return DSA_ERR_INVALID_ARG;
  if (n_heads < 1 || n_heads > 96 || !(scale > 0.f) || !std::isfinite(scale)) return DSA_ERR_INVALID_ARG;
  if (k_sel > 2048) return DSA_ERR_UNSUPPORTED;
  if (T == 0) return DSA_OK;
  if (T > (int64_t(1) << 31) - 1 || cache_rows < 1 || cache_rows > (int64_t(1) << 40)) return DSA_ERR_INVALID_ARG;
  if (!q || !kv_cache || !cache_offsets || !q_seq_offsets || (!idx && k_sel > 0) || !out || !lse)
    return DSA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(kv_cache) || !aligned16(out) || (reinterpret_cast<uintptr_t>(idx) & 3) ||
      (reinterpret_cast<uintptr_t>(lse) & 3) || (reinterpret_cast<uintptr_t>(cache_offsets) & 7) ||
      (reinterpret_cast<uintptr_t>(q_seq_offsets) & 3))
    return DSA_ERR_INVALID_ARG;
  SparseMlaArgs a;
  a.T = static_cast<int>(T);
  a.B = B;
  a.H = n_heads;
  a.k_sel = k_sel;
  a.cache_rows = cache_rows;
  a.q = q;
  a.kv_cache = kv_cache;
  a.cache_offsets = cache_offsets;
  a.q_seq_offsets = q_seq_offsets;
  a.idx = idx;
  a.scale = scale;
  a.out = out;
  a.lse = lse;
  a.err = h->ws.err;
  a.timeout_ns = timeout_ns();
  if (launch_sparse_mla(a, static_cast<cudaStream_t>(stream)) != cudaSuccess) return DSA_ERR_CUDA;
  return DSA_OK;
}

dsa_status_t dsa_indexer_device_error(dsa_indexer_t h) {
  if (!h) return DSA_ERR_INVALID_ARG;
  if (cudaDeviceSynchronize() != cudaSuccess) return DSA_ERR_CUDA;
  int v = 0;
  if (cudaMemcpy(&v, h->ws.err, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return DSA_ERR_CUDA;
  if (cudaMemset(h->ws.err, 0, sizeof(int)) != cudaSuccess) return DSA_ERR_CUDA;
  if (v & kErrTimeout) return DSA_ERR_DEVICE_TIMEOUT;
  if (v & (kErrBounds | kErrOffsets)) return DSA_ERR_DEVICE_BOUNDS;
  return DSA_OK;
}

dsa_status_t dsa_indexer_selftest_wait_timeout(int64_t timeout_ns_arg, void* stream) {
  if (timeout_ns_arg <= 0 || timeout_ns_arg > int64_t(10) * 1000 * 1000 * 1000) return DSA_ERR_INVALID_ARG;
  int* d = nullptr;
  if (cudaMalloc(&d, sizeof(int)) != cudaSuccess) return DSA_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int v = -1;
  cudaError_t e = cudaMemsetAsync(d, 0xFF, sizeof(int), s);
  if (e == cudaSuccess) e = launch_wait_timeout_selftest(d, static_cast<uint64_t>(timeout_ns_arg), s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e == cudaSuccess) e = cudaMemcpy(&v, d, sizeof(int), cudaMemcpyDeviceToHost);
  cudaFree(d);
  if (e != cudaSuccess) return DSA_ERR_CUDA;
  if (v == 2) return DSA_ERR_DEVICE_TIMEOUT;
  return v == 0 ? DSA_OK : DSA_ERR_CUDA;
}

}  // extern "C"
