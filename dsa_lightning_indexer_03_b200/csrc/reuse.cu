// reuse.cu -- index reuse across speculative (multi-token-prediction) draft steps.
//
// 'MTP' row of the page "Kimi K3.1 Pro vs GLM-5" (GLM-5.2): the later draft steps reuse the
// top-k indices of the first step instead of running the indexer again.  Here a draft token
// d names its anchor row a(d) (the first step's query, already selected by
// dsa_indexer_topk); its output row is an exact copy of the anchor's row, indices and (if
// requested) scores.  The copy is HBM-bound (8 KB in, 8 KB out per row): each CTA copies
// rows with 16-byte loads and stores, one warp per row, grid sized to the SMs.

#include "kernels.h"

namespace dsa {
namespace {

constexpr int kReuseWarps = 8;

__global__ void __launch_bounds__(kReuseWarps * 32) reuse_rows_kernel(int n, const int32_t* __restrict__ anchor,
                                                                      int n_src, const int32_t* __restrict__ src_idx,
                                                                      const float* __restrict__ src_score,
                                                                      int32_t* __restrict__ dst_idx,
                                                                      float* __restrict__ dst_score, int* err) {
  const int lane = threadIdx.x & 31;
  const int gw = blockIdx.x * kReuseWarps + (threadIdx.x >> 5);
  const int nw = gridDim.x * kReuseWarps;
  for (int d = gw; d < n; d += nw) {
    const int a = anchor[d];
    const bool ok = a >= 0 && a < n_src;
    if (!ok && lane == 0) atomicOr(err, kErrBounds);
    const int4* si = reinterpret_cast<const int4*>(src_idx + static_cast<size_t>(ok ? a : 0) * kTopK);
    int4* di = reinterpret_cast<int4*>(dst_idx + static_cast<size_t>(d) * kTopK);
    const float4* ss = src_score ? reinterpret_cast<const float4*>(src_score + static_cast<size_t>(ok ? a : 0) * kTopK)
                                 : nullptr;
    float4* ds = dst_score ? reinterpret_cast<float4*>(dst_score + static_cast<size_t>(d) * kTopK) : nullptr;
#pragma unroll 4
    for (int v = lane; v < kTopK / 4; v += 32) {
      // an anchor outside the source rows gives an all-padding row
      __stcs(di + v, ok ? __ldcs(si + v) : make_int4(-1, -1, -1, -1));
      if (ds) __stcs(ds + v, (ok && ss) ? __ldcs(ss + v) : make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY));
    }
  }
}

}  // namespace

cudaError_t launch_reuse_rows(int n, const int32_t* anchor, int n_src, const int32_t* src_idx, const float* src_score,
                              int32_t* dst_idx, float* dst_score, int* err, int num_sms, cudaStream_t s) {
  if (n <= 0) return cudaSuccess;
  const int want = (n + kReuseWarps - 1) / kReuseWarps;
  const int grid = want < 4 * num_sms ? want : 4 * num_sms;
  reuse_rows_kernel<<<grid, kReuseWarps * 32, 0, s>>>(n, anchor, n_src, src_idx, src_score, dst_idx, dst_score, err);
  return cudaGetLastError();
}

}  // namespace dsa
