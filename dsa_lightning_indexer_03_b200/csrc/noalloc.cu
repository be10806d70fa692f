// noalloc.cu -- dsa_indexer_topk_noalloc: the score + top-k entry point for callers that
// cannot allocate device memory.
//
// dsa_indexer_topk needs a handle, and a handle owns a workspace that dsa_indexer_create
// obtains with cudaMalloc (work list, validated positions, per-SM candidate lists).  Some
// callers cannot do that: a framework whose memory pool already holds the whole device
// budget, or a latency-critical loop that must never pay for cudaMalloc / cudaFree and
// the device synchronisation they can imply.  This entry point needs no handle and
// allocates nothing: its scratch is a fixed array in the library's own static device
// memory (kScratchBytes = 6,473,216 bytes, held on every GPU that loads the library until the
// process exits).  It runs the same kernels as dsa_indexer_topk's prefill path, on at most
// kStaticCtas SMs (the array holds that many per-SM candidate areas), so it is slower.

#include <cudaTypedefs.h>

#include <mutex>

#include "../../include/dsa_indexer.h"
#include "kernels.h"

using namespace dsa;

namespace {

constexpr int kStaticCtas = 8;           // persistent CTAs (candidate areas) the scratch holds
constexpr int kStaticMaxTokens = 4096;   // largest T (and B) this entry point accepts
constexpr int kStaticMaxItems = kStaticMaxTokens + 16;

constexpr size_t align256(size_t x) { return (x + 255) / 256 * 256; }
constexpr size_t kOffErr = 0;
constexpr size_t kOffNItems = 256;
constexpr size_t kOffCounter = 512;
constexpr size_t kOffItems = 768;
constexpr size_t kOffSeqBase = kOffItems + align256(size_t(kStaticMaxItems) * sizeof(WorkItem));
constexpr size_t kOffPos = kOffSeqBase + align256(size_t(kStaticMaxTokens + 2) * 4);
constexpr size_t kOffNch = kOffPos + align256(size_t(kStaticMaxTokens) * 4);
constexpr size_t kCandEntries = size_t(kStaticCtas) * kPrefillQ * kCandStride;
constexpr size_t kOffCand = kOffNch + align256(size_t(kStaticMaxTokens) * 4);
constexpr size_t kScratchBytes = kOffCand + align256(kCandEntries * sizeof(uint2));
static_assert(kScratchBytes == 6473216, "the scratch size is stated in include/dsa_indexer.h");


}  // namespace

// The scratch.  In host code this name is only a host-side stand-in: its device address
// comes from cudaGetSymbolAddress, looked up once per device below.
static __device__ __align__(256) unsigned char g_topk_scratch[kScratchBytes];

namespace {

PFN_cuTensorMapEncodeTiled_v12000 g_encode_fn = nullptr;
std::once_flag g_encode_flag;

bool tmap_bf16(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint32_t box_inner,
               uint32_t box_rows) {
  std::call_once(g_encode_flag, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode_fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  if (!g_encode_fn) return false;
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {inner * 2};
  cuuint32_t box[2] = {box_inner, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return g_encode_fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Device address of the scratch on the current device.  Looked up on every call, with the
// caller's device current: the lookup costs far less than the launches, and an address kept
// from an earlier call could belong to a context that no longer exists (after a device reset).
unsigned char* scratch_on_current_device(int* num_sms) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return nullptr;
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_topk_scratch) != cudaSuccess || p == nullptr) return nullptr;
  if (cudaDeviceGetAttribute(num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return nullptr;
  return static_cast<unsigned char*>(p);
}

bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" dsa_status_t dsa_indexer_topk_noalloc(int64_t T, const void* q, const float* w, const int32_t* positions,
                                                 const int32_t* q_seq_offsets, int32_t B, const void* key_cache,
                                                 int64_t cache_rows, const int64_t* cache_offsets, int32_t* idx_out,
                                                 float* score_out, void* stream) {
  if (T < 0 || B < 1) return DSA_ERR_INVALID_ARG;
  if (T == 0) return DSA_OK;
  if (T > kStaticMaxTokens || B > kStaticMaxTokens) return DSA_ERR_WORKSPACE;
  if (!q || !w || !positions || !q_seq_offsets || !key_cache || !cache_offsets || !idx_out) return DSA_ERR_INVALID_ARG;
  if (!al16(q) || !al16(w) || !al16(key_cache) || !al16(idx_out) || (score_out && !al16(score_out)) ||
      (reinterpret_cast<uintptr_t>(positions) & 3) || (reinterpret_cast<uintptr_t>(q_seq_offsets) & 3) ||
      (reinterpret_cast<uintptr_t>(cache_offsets) & 7))
    return DSA_ERR_INVALID_ARG;
  if (cache_rows < 1 || cache_rows > (int64_t(1) << 31) - (int64_t(1) << 20)) return DSA_ERR_INVALID_ARG;

  int sms = 0;
  unsigned char* base = scratch_on_current_device(&sms);
  if (!base) return DSA_ERR_CUDA;

  CUtensorMap tmQ8, tmK;
  if (!tmap_bf16(&tmQ8, q, kHeadDim, uint64_t(T) * kHeads, 64, kHeads * kPrefillQ) ||
      !tmap_bf16(&tmK, key_cache, kHeadDim, uint64_t(cache_rows), 64, kKeyTile))
    return DSA_ERR_INVALID_ARG;

  TopkWorkspace ws{};
  ws.err = reinterpret_cast<int*>(base + kOffErr);
  ws.n_items = reinterpret_cast<int*>(base + kOffNItems);
  ws.work_counter = reinterpret_cast<int*>(base + kOffCounter);
  ws.items = reinterpret_cast<WorkItem*>(base + kOffItems);
  ws.max_items = kStaticMaxItems;
  ws.seq_base = reinterpret_cast<int*>(base + kOffSeqBase);
  ws.pos_eff = reinterpret_cast<int*>(base + kOffPos);
  ws.tok_nchunks = reinterpret_cast<int*>(base + kOffNch);
  ws.cand = reinterpret_cast<uint2*>(base + kOffCand);
  ws.cand_slots = kStaticCtas;
  ws.part_keys = nullptr;
  ws.part_idx = nullptr;
  ws.part_hist = nullptr;
  ws.part_tokens = 0;

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
  a.split = false;
  a.sorted = false;
  a.fp8 = false;
  a.heads = kHeads;
  a.timeout_ns = wait_timeout_ns();
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // the error word keeps the previous call's bits: start each call from zero
  if (cudaMemsetAsync(ws.err, 0, sizeof(int), s) != cudaSuccess) return DSA_ERR_CUDA;
  // the prep kernel rewrites the work list and resets the work counter on every call
  if (launch_topk(a, ws, tmQ8, tmQ8, tmK, sms < kStaticCtas ? sms : kStaticCtas, s) != cudaSuccess)
    return DSA_ERR_CUDA;
  return DSA_OK;
}

extern "C" dsa_status_t dsa_indexer_noalloc_device_error(void* stream) {
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return DSA_ERR_CUDA;
  int v = 0;
  // the error word sits at the start of the scratch; the copy allocates nothing
  if (cudaMemcpyFromSymbol(&v, g_topk_scratch, sizeof(int), kOffErr, cudaMemcpyDeviceToHost) != cudaSuccess)
    return DSA_ERR_CUDA;
  if (v & kErrTimeout) return DSA_ERR_DEVICE_TIMEOUT;
  if (v & (kErrBounds | kErrOffsets)) return DSA_ERR_DEVICE_BOUNDS;
  return DSA_OK;
}
