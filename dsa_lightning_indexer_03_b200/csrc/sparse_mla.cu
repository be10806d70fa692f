// sparse_mla.cu -- attention of each query over the tokens its indexer selected, in the
// latent form of multi-head latent attention.
//
// 'Latent attention (MLA)' row (Kimi K3.1 Pro): 96 heads; keys and values come from a
// 512-dim latent plus a 64-dim shared key slot (576 cached values per token); each query
// attends only to the 2,048 tokens its layer's indexer selects.  In the latent form a head's
// query is 576 values (its no-rope part already taken into the latent space), the score of a
// selected token is scale * (q . row) over the 576 cached values, and the value is the row's
// 512-dim latent: o = softmax(scores) . latent, lse = log sum exp(scores).
//
// sparse_mla_kernel: one CTA per (query, half of the 512 output dims), 288 threads.
//   warps 0-3  gather: the selected rows of each 32-token tile (cp.async, 16 bytes a copy)
//              into a 3-stage ring, laid out as the MMA's 128-byte-swizzled tiles.
//   warp 8     MMA issuer: S = Q . K^T (M = 128 head rows of which the first H are real,
//              N = 32 tokens, K = 576 as 36 tcgen05.mma of K = 16) into one of two TMEM
//              score buffers, and O += P . V of the previous tile (A = P, bf16 in TMEM;
//              B = that tile's latent half read in place as an MN-major operand), issued
//              between those MMAs as soon as its P is ready.
//   warps 4-7  softmax, one thread per head row (the warp's TMEM lane quadrant): masks the
//              tile's missing tokens, keeps the running maximum m (in log2 units) and sum l,
//              writes P = 2^(s - m) as bf16 into TMEM, and rescales O in TMEM only when the
//              maximum rises by more than 8 (log2 units, so P stays below 256); at the end
//              O / l is written out in bf16 and the half-0 CTA writes lse.

#include "kernels.h"

namespace dsa {
namespace {

constexpr int kMlaDim = 576;                 // cached values per token
constexpr int kMlaLatent = 512;              // value part
constexpr int kMlaHalf = 256;                // output dims per CTA
constexpr int kMlaMaxHeads = 96;             // head rows held in shared memory
constexpr int kMlaChunks = kMlaDim / 64;     // 64-value (128-byte) chunks of a row
constexpr int kMlaTok = 32;                  // tokens per tile
constexpr int kMlaStages = 3;
constexpr int kMlaQChunk = kMlaMaxHeads * 128;          // one chunk of Q: 96 rows x 128 B
constexpr int kMlaKvChunk = kMlaTok * 128;              // one chunk of a tile: 32 rows x 128 B
constexpr int kMlaStage = kMlaChunks * kMlaKvChunk;     // 36 KB
constexpr int kMlaQBytes = kMlaChunks * kMlaQChunk;     // 108 KB
constexpr int kMlaThreads = 288;
constexpr int kMlaMmaWarp = 8;
// TMEM columns: O (256 fp32), two score buffers (32 each), two P buffers (16 each)
constexpr uint32_t kMlaTmemO = 0, kMlaTmemS = 256, kMlaTmemP = 320;
constexpr int kMlaNumBars = 3 * 2 + 2 * 4 + 1;          // kv_full/empty[3], s_full/empty, p_full, pv_done [2], mma_done
constexpr uint64_t kMlaDrainNs = 200ull * 1000 * 1000;   // limit of the final wait for this CTA's MMAs
constexpr int kMlaMaxSel = 2048;                         // selected entries per query held in shared memory
constexpr int kMlaSmem = kMlaQBytes + kMlaStages * kMlaStage + 4 * kMlaMaxSel + 8 * kMlaNumBars + 64 + 1024;
static_assert(kMlaQChunk % 1024 == 0 && kMlaKvChunk % 1024 == 0, "swizzle atoms stay 1024-byte aligned");
static_assert(kMlaSmem <= 232448, "shared memory per CTA");

struct MlaParams {
  const __nv_bfloat16* q;        // [T, H, 576]
  const __nv_bfloat16* kv;       // [cache_rows, 576]
  const int64_t* cache_offsets;  // [B+1]
  const int32_t* q_seq_offsets;  // [B+1]
  const int32_t* idx;            // [T, k_sel]
  __nv_bfloat16* out;            // [T, H, 512]
  float* lse;                    // [T, H]
  int B, H, k_sel;
  int64_t cache_rows;
  float scale_log2;              // scale * log2(e)
  int* err;
  uint64_t timeout_ns;
};

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t d;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
  return d;
}

// Shared-memory descriptor of an MN-major operand with 128-byte swizzling: 64 values along
// N per 128-byte row, rows (the K direction) 128 B apart; the next 64 values along N start
// `lbo` bytes on, the next 8 rows along K `sbo` bytes on.
__device__ __forceinline__ uint64_t umma_desc_sw128_mn(uint32_t addr, uint32_t lbo, uint32_t sbo) {
  return static_cast<uint64_t>((addr >> 4) & 0x3FFFu) | (static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16) |
         (static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32) | (static_cast<uint64_t>(1) << 46) |
         (static_cast<uint64_t>(2) << 61);
}

// D (+)= A[tmem] * B[smem] (kind::f16)
__device__ __forceinline__ void umma_bf16_ta(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                             uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void tmem_st_16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};\n\t"
      "tcgen05.wait::st.sync.aligned;"
      ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}

__device__ __forceinline__ void tmem_st_32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
      "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};\n\t"
      "tcgen05.wait::st.sync.aligned;"
      ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]),
        "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]),
        "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}

// 2^x by the hardware's approximate base-2 exponential (relative error near 2^-22, far below
// the bf16 rounding the weights then get); 2^-inf = 0.
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__global__ void __launch_bounds__(kMlaThreads, 1) sparse_mla_kernel(MlaParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sKV = smem + kMlaQBytes;
  int32_t* sIdx = reinterpret_cast<int32_t*>(sKV + kMlaStages * kMlaStage);   // the query's idx row
  uint64_t* bars = reinterpret_cast<uint64_t*>(sIdx + kMlaMaxSel);
  uint64_t* kv_full = bars;
  uint64_t* kv_empty = kv_full + kMlaStages;
  uint64_t* s_full = kv_empty + kMlaStages;
  uint64_t* s_empty = s_full + 2;
  uint64_t* p_full = s_empty + 2;
  uint64_t* pv_done = p_full + 2;
  uint64_t* mma_done = pv_done + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + kMlaNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x, half = blockIdx.y;
  const int H = p.H;
  const int ntiles = (p.k_sel + kMlaTok - 1) / kMlaTok;

  // the query's sequence (the last b with q_seq_offsets[b] <= t) and its cache rows
  int lo = 0, hi = p.B - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (p.q_seq_offsets[mid] <= t) lo = mid;
    else hi = mid - 1;
  }
  int64_t row0 = p.cache_offsets[lo];
  int64_t len = p.cache_offsets[lo + 1] - row0;
  // malformed offsets: the query attends to nothing (o = 0, lse = -inf) and the error is set
  if (t < p.q_seq_offsets[0] || t >= p.q_seq_offsets[p.B] || row0 < 0 || len < 0 || row0 + len > p.cache_rows) {
    if (threadIdx.x == 0 && half == 0) atomicOr(p.err, kErrOffsets);
    row0 = 0;
    len = 0;
  }

  if (threadIdx.x == 0) {
    for (int s = 0; s < kMlaStages; ++s) {
      mbar_init(&kv_full[s], 128);   // one arrive per gather thread
      mbar_init(&kv_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&s_full[b], 1);
      mbar_init(&s_empty[b], 4);
      mbar_init(&p_full[b], 4);
      mbar_init(&pv_done[b], 1);
    }
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kMlaMmaWarp) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  // Q: rows 0..H-1 of this query, rows H..95 zero, as 9 chunks of 96 x 128 B with the
  // 128-byte swizzle (16-byte unit u of row r at unit u ^ (r & 7)).  The MMA reads 128 rows
  // per chunk: rows 96..127 fall on the next chunk (or the ring) and only feed score rows
  // that nothing reads.
  {
    const __nv_bfloat16* qsrc = p.q + static_cast<size_t>(t) * H * kMlaDim;
    for (int u = threadIdx.x; u < kMlaMaxHeads * (kMlaDim / 8); u += kMlaThreads) {
      const int r = u / (kMlaDim / 8), w = u % (kMlaDim / 8), c = w >> 3, cu = w & 7;
      const uint32_t dst = smem_u32(sQ + c * kMlaQChunk + r * 128 + ((cu ^ (r & 7)) * 16));
      const __nv_bfloat16* src = qsrc + (r < H ? static_cast<size_t>(r) * kMlaDim + w * 8 : 0);
      asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(r < H ? 16 : 0)
                   : "memory");
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
    // the idx row, padded with -1 to whole tiles
    const int32_t* isrc = p.idx + static_cast<size_t>(t) * p.k_sel;
    for (int k = threadIdx.x; k < ntiles * kMlaTok; k += kMlaThreads) sIdx[k] = k < p.k_sel ? isrc[k] : -1;
    asm volatile("cp.async.wait_group 0;" ::: "memory");
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const WaitCtl wc{p.err, abort_flag, p.timeout_ns};

  if (warp < 4) {
    // ============================================================ gather
    // Each thread copies 18 of a tile's 32 x 72 16-byte units (cp.async) into the ring stage,
    // 128-byte swizzled as the MMA reads it; a missing token's row is zero-filled (no global
    // read).  A tile is published once this thread's copies of it have landed: wait for the
    // previous tile's group, fence it over to the async proxy the MMA reads through, then
    // arrive on its barrier.
    const int pt = threadIdx.x;   // 0..127
    bool ok = true;
    for (int tile = 0; tile < ntiles; ++tile) {
      const int s = tile % kMlaStages;
      if (tile >= kMlaStages && !mbar_wait(&kv_empty[s], ((tile / kMlaStages) - 1) & 1, wc)) {
        ok = false;
        break;
      }
      const int my_pos = sIdx[tile * kMlaTok + lane];
      uint8_t* const st = sKV + s * kMlaStage;
#pragma unroll 6
      for (int i = 0; i < kMlaTok * (kMlaDim / 8) / 128; ++i) {
        const int u = pt + 128 * i;
        const int j = u / (kMlaDim / 8), w = u % (kMlaDim / 8), c = w >> 3, cu = w & 7;
        const int pos = __shfl_sync(0xffffffffu, my_pos, j);
        const bool valid = pos >= 0 && pos < len;
        const __nv_bfloat16* src = p.kv + (valid ? (row0 + pos) * kMlaDim + w * 8 : 0);
        const uint32_t dst = smem_u32(st + c * kMlaKvChunk + j * 128 + ((cu ^ (j & 7)) * 16));
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(valid ? 16 : 0)
                     : "memory");
      }
      asm volatile("cp.async.commit_group;" ::: "memory");
      if (tile >= 1) {
        asm volatile("cp.async.wait_group 1;" ::: "memory");
        fence_proxy_async_smem();
        mbar_arrive(&kv_full[(tile - 1) % kMlaStages]);
      }
    }
    asm volatile("cp.async.wait_group 0;" ::: "memory");
    if (ok && ntiles > 0) {
      fence_proxy_async_smem();
      mbar_arrive(&kv_full[(ntiles - 1) % kMlaStages]);
    }
  } else if (warp < kMlaMmaWarp) {
    // ============================================================ softmax
    const int qd = warp & 3;
    const int r = qd * 32 + lane;                             // head row
    const uint32_t trow = tmem + (static_cast<uint32_t>(qd * 32) << 16);
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    for (int tile = 0; tile < ntiles && ok; ++tile) {
      const int b = tile & 1;
      // the tile's tokens that exist (one per lane, then shared by ballot)
      const int pos = sIdx[tile * kMlaTok + lane];
      const uint32_t valid = __ballot_sync(0xffffffffu, pos >= 0 && pos < len);
      // an index past the sequence's rows is reported once (by one softmax warp)
      const uint32_t past = __ballot_sync(0xffffffffu, pos >= len);
      if (warp == 4 && lane == 0 && past != 0u) atomicOr(p.err, kErrBounds);
      ok = __all_sync(0xffffffffu, mbar_wait(&s_full[b], (tile >> 1) & 1, wc));
      if (!ok) break;
      tc_fence_after();
      uint32_t x[32];
      tmem_ld_32cols(trow + kMlaTmemS + 32 * b, x);
      tmem_ld_wait(x);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_empty[b]);
      float v[32];
      float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        v[j] = ((valid >> j) & 1u) ? __uint_as_float(x[j]) * p.scale_log2 : -INFINITY;
        mx4[j & 3] = fmaxf(mx4[j & 3], v[j]);
      }
      const float tmax = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3]));
      // running maximum: set by the first tile with a token; raised (with O and l scaled
      // down) only when a tile's maximum exceeds it by more than 8, so 2^(s - m) < 256
      float f = 1.f;
      bool rescale = false;
      if (m == -INFINITY) {
        m = tmax;
      } else if (tmax > m + 8.f) {
        f = ex2_approx(m - tmax);
        m = tmax;
        rescale = true;
      }
      if (__any_sync(0xffffffffu, rescale)) {
        // every earlier P . V has landed in O before it is scaled
        ok = __all_sync(0xffffffffu, mbar_wait(&pv_done[(tile - 1) & 1], ((tile - 1) >> 1) & 1, wc));
        if (!ok) break;
        tc_fence_after();
#pragma unroll 1
        for (int c = 0; c < kMlaHalf / 32; ++c) {
          uint32_t o[32];
          tmem_ld_32cols(trow + kMlaTmemO + 32 * c, o);
          tmem_ld_wait(o);
#pragma unroll
          for (int j = 0; j < 32; ++j) o[j] = __float_as_uint(__uint_as_float(o[j]) * f);
          tmem_st_32(trow + kMlaTmemO + 32 * c, o);
        }
        l *= f;
      }
      uint32_t pk[16];
      float ps4[4] = {0.f, 0.f, 0.f, 0.f};
      // with no token seen yet (m = -inf) every weight is 0; a masked token's is 2^-inf = 0
      const float mm = m == -INFINITY ? INFINITY : m;
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        pk[j] = pack_bf16x2(ex2_approx(v[2 * j] - mm), ex2_approx(v[2 * j + 1] - mm));
        // the sum uses the bf16 values the MMA multiplies
        ps4[j & 3] += __uint_as_float(pk[j] << 16) + __uint_as_float(pk[j] & 0xFFFF0000u);
      }
      l += (ps4[0] + ps4[1]) + (ps4[2] + ps4[3]);
      // P buffer b was last read by the P . V of tile - 2
      if (tile >= 2) {
        ok = __all_sync(0xffffffffu, mbar_wait(&pv_done[b], ((tile >> 1) - 1) & 1, wc));
        if (!ok) break;
        tc_fence_after();
      }
      tmem_st_16(trow + kMlaTmemP + 16 * b, pk);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[b]);
    }
    if (ok && ntiles > 0)
      ok = __all_sync(0xffffffffu, mbar_wait(&pv_done[(ntiles - 1) & 1], ((ntiles - 1) >> 1) & 1, wc));
    if (ok) {
      tc_fence_after();
      const float inv = l > 0.f ? 1.f / l : 0.f;
      const bool none = !(l > 0.f);   // no token: O holds no product, write zeros
      __nv_bfloat16* const orow = p.out + (static_cast<size_t>(t) * H + r) * kMlaLatent + half * kMlaHalf;
#pragma unroll 1
      for (int c = 0; c < kMlaHalf / 32; ++c) {
        uint32_t o[32];
        tmem_ld_32cols(trow + kMlaTmemO + 32 * c, o);
        tmem_ld_wait(o);
        if (r < H) {
          uint4 w[4];
          uint32_t* const wp = reinterpret_cast<uint32_t*>(w);
#pragma unroll
          for (int j = 0; j < 16; ++j)
            wp[j] = none ? 0u : pack_bf16x2(__uint_as_float(o[2 * j]) * inv, __uint_as_float(o[2 * j + 1]) * inv);
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) reinterpret_cast<uint4*>(orow + 32 * c)[q4] = w[q4];
        }
      }
      if (half == 0 && r < H)
        p.lse[static_cast<size_t>(t) * H + r] = l > 0.f ? m * 0.69314718055994531f + logf(l) : -INFINITY;
    }
  } else if (lane == 0) {
    // ============================================================ MMA issuer (warp 8)
    constexpr uint32_t idesc_s = umma_idesc_bf16(128, kMlaTok);
    constexpr uint32_t idesc_pv = umma_idesc_bf16(128, kMlaHalf) | (1u << 16);   // B (V) MN-major
    const uint32_t qa = smem_u32(sQ);
    // O += P . V of tile u: V is this CTA's four 64-value chunks of the tile's latent, 16
    // tokens (two 8-row groups, 1 KB apart) per MMA
    auto issue_pv = [&](int u) {
      const int su = u % kMlaStages, bu = u & 1;
      tc_fence_after();
      const uint32_t vb = smem_u32(sKV + su * kMlaStage + half * 4 * kMlaKvChunk);
#pragma unroll
      for (int ks = 0; ks < 2; ++ks)
        umma_bf16_ta(tmem + kMlaTmemO, tmem + kMlaTmemP + 16 * bu + 8 * ks,
                     umma_desc_sw128_mn(vb + ks * 16 * 128, kMlaKvChunk, 1024), idesc_pv, (u > 0 || ks > 0) ? 1u : 0u);
      umma_commit(&pv_done[bu]);
      umma_commit(&kv_empty[su]);
    };
    // The P . V of a tile is issued as soon as its P is ready, between the score MMAs of the
    // next tile (the tensor pipe runs them in issue order), and at the latest before the wait
    // for tile + 2: the gather threads publish tile + 2 only after they have passed the wait
    // for the ring stage of tile + 3, which this P . V frees.
    int pv_next = 0;
    bool ok = true;
    for (int tile = 0; tile < ntiles && ok; ++tile) {
      const int s = tile % kMlaStages, b = tile & 1;
      for (; pv_next < tile - 1; ++pv_next)
        if (!(ok = mbar_wait(&p_full[pv_next & 1], (pv_next >> 1) & 1, wc))) break; else issue_pv(pv_next);
      if (!ok) break;
      if (!mbar_wait(&kv_full[s], (tile / kMlaStages) & 1, wc)) break;
      if (tile >= 2 && !mbar_wait(&s_empty[b], ((tile >> 1) - 1) & 1, wc)) break;
      tc_fence_after();
      const uint32_t ka = smem_u32(sKV + s * kMlaStage);
#pragma unroll 1
      for (int c = 0; c < kMlaChunks; ++c) {
        const uint64_t ad = umma_desc_sw128(qa + c * kMlaQChunk), bd = umma_desc_sw128(ka + c * kMlaKvChunk);
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
          umma_bf16(tmem + kMlaTmemS + 32 * b, ad + 2 * ks, bd + 2 * ks, idesc_s, (c > 0 || ks > 0) ? 1u : 0u);
        if (pv_next < tile && mbar_try_wait(smem_u32(&p_full[pv_next & 1]), (pv_next >> 1) & 1)) {
          issue_pv(pv_next);
          ++pv_next;
        }
      }
      umma_commit(&s_full[b]);
    }
    for (; ok && pv_next < ntiles; ++pv_next)
      if ((ok = mbar_wait(&p_full[pv_next & 1], (pv_next >> 1) & 1, wc))) issue_pv(pv_next);
    // every MMA this thread issued has finished before TMEM is freed (on an early exit too);
    // the wait is bounded
    umma_commit(mma_done);
    const uint64_t t0 = global_timer_ns();
    while (!mbar_try_wait(smem_u32(mma_done), 0) && global_timer_ns() - t0 <= kMlaDrainNs) {
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kMlaMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace

cudaError_t launch_sparse_mla(const SparseMlaArgs& a, cudaStream_t s) {
  if (a.T == 0) return cudaSuccess;
  MlaParams p;
  p.q = static_cast<const __nv_bfloat16*>(a.q);
  p.kv = static_cast<const __nv_bfloat16*>(a.kv_cache);
  p.cache_offsets = a.cache_offsets;
  p.q_seq_offsets = a.q_seq_offsets;
  p.idx = a.idx;
  p.out = static_cast<__nv_bfloat16*>(a.out);
  p.lse = a.lse;
  p.B = a.B;
  p.H = a.H;
  p.k_sel = a.k_sel;
  p.cache_rows = a.cache_rows;
  p.scale_log2 = a.scale * 1.4426950408889634f;
  p.err = a.err;
  p.timeout_ns = a.timeout_ns;
  cudaError_t e = cudaFuncSetAttribute(sparse_mla_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kMlaSmem);
  if (e != cudaSuccess) return e;
  sparse_mla_kernel<<<dim3(a.T, 2), kMlaThreads, kMlaSmem, s>>>(p);
  return cudaGetLastError();
}

}  // namespace dsa
