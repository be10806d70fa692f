// proj.cu -- the indexer's three projections on the tcgen05 tensor cores.
//
// 'Sparse / compressed attn' row (Kimi K3.1 Pro): queries from the 1,536-dim
// query latent (1,536 -> 4,096 = 32 heads x 128), one shared 128-dim key from
// the hidden state with a LayerNorm, per-head weights from a 7,168 -> 32
// projection.  The key and weight projections read the same hidden row, so
// they run as one GEMM with N = 128 + 32 = 160 whose epilogue applies the
// LayerNorm to columns 0..127 (one TMEM lane = one token, so each epilogue
// thread owns its whole 128-wide row), casts to bf16 and scatters the row to
// its key-cache slot, and stores columns 128..159 as fp32 head weights.
//
// Kernel shape: one 128-row output tile per CTA; warp 0 issues TMA loads of
// 64-wide K slices of A and B into a STAGES-deep ring (128-byte swizzle),
// warp 1 issues tcgen05.mma (M=128, N=BN, K=16) into a TMEM accumulator,
// warps 2..5 drain TMEM (tcgen05.ld 32x32b) in the epilogue.  The k|w GEMM
// (proj_kw_cluster_kernel) splits its 7,168-deep contraction over a cluster of
// CTAs that reduce their partial tiles through distributed shared memory before
// the LayerNorm epilogue, so that every token count keeps many SMs streaming.

#include <cuda_fp8.h>

#include "kernels.h"

namespace dsa {
namespace {

constexpr int kBM = 128;
constexpr int kBK = 64;
constexpr int kABytes = kBM * kBK * 2;  // 16 KB per stage
constexpr uint64_t kDrainNs = 200ull * 1000 * 1000;

enum { EPI_Q = 0, EPI_KW = 1, EPI_Q8 = 2 };

struct ProjParams {
  int M, K;
  __nv_bfloat16* q_out;  // EPI_Q
  int ldq;
  uint8_t* q8_out;       // EPI_Q8: FP8 e4m3 codes [M, ldq]
  float* q_scale;        // EPI_Q8: [M, ldq / 128], one scale per query head
  const int32_t* positions;   // EPI_Q with rope_dim > 0: token positions [M]
  const double* inv_freq;     // rotary frequencies theta^(-2i / rope_dim), i < rope_dim / 2
  int rope_dim;               // rotated dims at the start of each 128-dim head (0: none)
  ProjKwEpilogue kw;     // EPI_KW
  int* err;
  uint64_t timeout_ns;
};

template <int BN, int STAGES>
struct ProjSmem {
  static constexpr int kBBytes = BN * kBK * 2;
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kBarOff = STAGES * kStageBytes;
  static constexpr int kMiscOff = kBarOff + 8 * (2 * STAGES + 2);
  static constexpr int kGammaOff = (kMiscOff + 16 + 15) / 16 * 16;
  static constexpr int kTotal = kGammaOff + 2 * 128 * 4 + 1024;  // + alignment slack
};

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ float round_bf16(float x) { return __bfloat162float(__float2bfloat16_rn(x)); }

// cos and sin of the rotary angle pos * inv_freq: the angle is formed and reduced to
// [-pi, pi] in double precision (positions reach 10^6 radians), then sincosf.
__device__ __forceinline__ void rope_cos_sin(int pos, double inv_freq, float* c, float* s) {
  const double ang = static_cast<double>(pos) * inv_freq;
  const double r = ang - 6.283185307179586 * rint(ang * 0.15915494309189535);
  sincosf(static_cast<float>(r), s, c);
}

// Rotates the pairs (x[2m], x[2m+1]) of a run of N values that starts at dim d0 of a head:
// pair i = d0/2 + m turns by pos * inv_freq[i] when 2i < rope_dim.
template <int N>
__device__ __forceinline__ void rope_rotate(float (&x)[N], int d0, int pos, const double* inv_freq, int rope_dim) {
#pragma unroll
  for (int m = 0; m < N / 2; ++m) {
    const int i = d0 / 2 + m;
    if (2 * i < rope_dim) {
      float c, sn;
      rope_cos_sin(pos, inv_freq[i], &c, &sn);
      const float a = x[2 * m], b = x[2 * m + 1];
      x[2 * m] = a * c - b * sn;
      x[2 * m + 1] = a * sn + b * c;
    }
  }
}

// FP8 e4m3 codes of four values (round to nearest even, saturating at +-448), first value
// in the lowest byte.
__device__ __forceinline__ uint32_t pack_e4m3x4(float a, float b, float c, float d) {
  const uint32_t lo = __nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3);
  const uint32_t hi = __nv_cvt_float2_to_fp8x2(make_float2(c, d), __NV_SATFINITE, __NV_E4M3);
  return (lo & 0xFFFFu) | (hi << 16);
}

// Scale and inverse scale of a row whose largest magnitude is amax: amax / 448 and
// 448 / amax (both 0 for an all-zero row); codes are e4m3(x * inv), values code * scale.
__device__ __forceinline__ void fp8_row_scale(float amax, float* scale, float* inv) {
  *scale = amax > 0.f ? __fdiv_rn(amax, 448.f) : 0.f;
  *inv = amax > 0.f ? __fdiv_rn(448.f, amax) : 0.f;
}

// waits without looking at the abort flag (used only to drain in-flight work)
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) {
  const uint32_t a = smem_u32(bar);
  const uint64_t t0 = global_timer_ns();
  while (!mbar_try_wait(a, parity)) {
    if (global_timer_ns() - t0 > kDrainNs) break;
  }
}

template <int BN, int STAGES, int EPI>
__global__ void __launch_bounds__(192, 1)
    proj_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                     ProjParams p) {
  using L = ProjSmem<BN, STAGES>;
  constexpr uint32_t kTmemCols = BN <= 32 ? 32 : BN <= 64 ? 64 : BN <= 128 ? 128 : 256;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * kABytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
  uint64_t* empty = full + STAGES;
  uint64_t* acc_full = empty + STAGES;
  uint64_t* mma_done = acc_full + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMiscOff + 4);
  float* s_gamma = reinterpret_cast<float*>(smem + L::kGammaOff);
  float* s_beta = s_gamma + 128;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.y * kBM;
  const int n0 = blockIdx.x * BN;
  const int nk = p.K / kBK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  if (EPI == EPI_KW && threadIdx.x >= 64) {
    const int i = threadIdx.x - 64;
    s_gamma[i] = p.kw.gamma[i];
    s_beta[i] = p.kw.beta[i];
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const WaitCtl wc{p.err, abort_flag, p.timeout_ns};

  if (warp == 0) {
    if (lane == 0) {
      int issued = 0;
      for (int kb = 0; kb < nk; ++kb) {
        const int s = kb % STAGES;
        if (kb >= STAGES && !mbar_wait(&empty[s], ((kb / STAGES) - 1) & 1, wc)) break;
        mbar_arrive_expect_tx(&full[s], L::kStageBytes);
        tma_load_2d(sA + s * kABytes, &tmA, &full[s], kb * kBK, m0);
        tma_load_2d(sB + s * L::kBBytes, &tmB, &full[s], kb * kBK, n0);
        issued = kb + 1;
      }
      if (*abort_flag) {  // let the loads still in flight land before the CTA exits
        for (int kb = (issued > STAGES ? issued - STAGES : 0); kb < issued; ++kb)
          drain_wait(&full[kb % STAGES], (kb / STAGES) & 1);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = umma_idesc_bf16(kBM, BN);
      for (int kb = 0; kb < nk; ++kb) {
        const int s = kb % STAGES;
        if (!mbar_wait(&full[s], (kb / STAGES) & 1, wc)) break;
        tc_fence_after();
        const uint32_t a = smem_u32(sA + s * kABytes);
        const uint32_t b = smem_u32(sB + s * L::kBBytes);
#pragma unroll
        for (int kk = 0; kk < kBK / 16; ++kk)
          umma_bf16(tmem, umma_desc_sw128(a + kk * 32), umma_desc_sw128(b + kk * 32), idesc, (kb | kk) != 0);
        umma_commit(&empty[s]);
      }
      umma_commit(acc_full);
      umma_commit(mma_done);
      drain_wait(mma_done, 0);
    }
  } else {
    // epilogue: warps 2..5; TMEM lane quadrant = warp % 4
    const int qd = warp & 3;
    const int row = m0 + qd * 32 + lane;
    const bool ok = __all_sync(0xffffffffu, mbar_wait(acc_full, 0, wc));
    tc_fence_after();
    const uint32_t tbase = tmem + (static_cast<uint32_t>(qd * 32) << 16);
    if (ok) {
      if constexpr (EPI == EPI_Q) {
        __nv_bfloat16* dst = p.q_out + static_cast<size_t>(row) * p.ldq + n0;
#pragma unroll 1
        for (int c = 0; c < BN / 32; ++c) {
          uint32_t r[32];
          tmem_ld_32cols(tbase + c * 32, r);
          tmem_ld_wait(r);
          const int hd0 = (n0 + c * 32) & 127;   // first dim of this chunk inside its head
          if (p.rope_dim > 0 && hd0 < p.rope_dim && row < p.M) {
            float x[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) x[i] = __uint_as_float(r[i]);
            rope_rotate<32>(x, hd0, p.positions[row], p.inv_freq, p.rope_dim);
#pragma unroll
            for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(x[i]);
          }
          if (row < p.M) {
            uint4* d4 = reinterpret_cast<uint4*>(dst + c * 32);
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              uint4 pk;
              pk.x = pack_bf16x2(__uint_as_float(r[8 * v + 0]), __uint_as_float(r[8 * v + 1]));
              pk.y = pack_bf16x2(__uint_as_float(r[8 * v + 2]), __uint_as_float(r[8 * v + 3]));
              pk.z = pack_bf16x2(__uint_as_float(r[8 * v + 4]), __uint_as_float(r[8 * v + 5]));
              pk.w = pack_bf16x2(__uint_as_float(r[8 * v + 6]), __uint_as_float(r[8 * v + 7]));
              d4[v] = pk;
            }
          }
        }
      } else if constexpr (EPI == EPI_Q8) {
        // per head (128 columns): q = bf16(acc), then FP8 codes with the head's scale
#pragma unroll 1
        for (int hh = 0; hh < BN / 128; ++hh) {
          float amax = 0.f;
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {
            uint32_t r[32];
            tmem_ld_32cols(tbase + hh * 128 + c * 32, r);
            tmem_ld_wait(r);
#pragma unroll
            for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(round_bf16(__uint_as_float(r[i]))));
          }
          float scale, inv;
          fp8_row_scale(amax, &scale, &inv);
          const int head = (n0 >> 7) + hh;
          uint8_t* dst = p.q8_out + static_cast<size_t>(row) * p.ldq + head * 128;
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {
            uint32_t r[32];
            tmem_ld_32cols(tbase + hh * 128 + c * 32, r);
            tmem_ld_wait(r);
            if (row < p.M) {
              uint32_t w8[8];
#pragma unroll
              for (int v = 0; v < 8; ++v)
                w8[v] = pack_e4m3x4(__fmul_rn(round_bf16(__uint_as_float(r[4 * v])), inv),
                                    __fmul_rn(round_bf16(__uint_as_float(r[4 * v + 1])), inv),
                                    __fmul_rn(round_bf16(__uint_as_float(r[4 * v + 2])), inv),
                                    __fmul_rn(round_bf16(__uint_as_float(r[4 * v + 3])), inv));
              uint4* d4 = reinterpret_cast<uint4*>(dst + c * 32);
              d4[0] = make_uint4(w8[0], w8[1], w8[2], w8[3]);
              d4[1] = make_uint4(w8[4], w8[5], w8[6], w8[7]);
            }
          }
          if (row < p.M) p.q_scale[static_cast<size_t>(row) * (p.ldq >> 7) + head] = scale;
        }
      } else {
        // key: LayerNorm over columns 0..127 of this token's row, fp32 math
        float x[128];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t r[32];
          tmem_ld_32cols(tbase + c * 32, r);
          tmem_ld_wait(r);
#pragma unroll
          for (int i = 0; i < 32; ++i) x[c * 32 + i] = __uint_as_float(r[i]);
        }
        float sum = 0.f;
#pragma unroll
        for (int i = 0; i < 128; ++i) sum += x[i];
        const float mean = sum * (1.0f / 128.0f);
        float ss = 0.f;
#pragma unroll
        for (int i = 0; i < 128; ++i) {
          const float d = x[i] - mean;
          ss = fmaf(d, d, ss);
        }
        const float rstd = rsqrtf(ss * (1.0f / 128.0f) + p.kw.eps);
        uint32_t wr[32];
        tmem_ld_32cols(tbase + 128, wr);
        tmem_ld_wait(wr);
        if (row < p.M) {
          const int t = row;
          const int pos = p.kw.positions[t];
          // sequence of token t: the last b with q_seq_offsets[b] <= t
          int lo = 0, hi = p.kw.B - 1;
          while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (p.kw.q_seq_offsets[mid] <= t) lo = mid;
            else hi = mid - 1;
          }
          const int64_t base = p.kw.cache_offsets[lo];
          const int64_t len = p.kw.cache_offsets[lo + 1] - base;
          if (pos >= 0 && pos < len && base >= 0 && base + pos < p.kw.cache_rows) {
            uint4* d4 = reinterpret_cast<uint4*>(p.kw.key_cache + static_cast<size_t>(base + pos) * kHeadDim);
#pragma unroll
            for (int v = 0; v < 16; ++v) {
              float y[8];
#pragma unroll
              for (int i = 0; i < 8; ++i) {
                const int d = 8 * v + i;
                y[i] = fmaf((x[d] - mean) * rstd, s_gamma[d], s_beta[d]);
              }
              uint4 pk;
              pk.x = pack_bf16x2(y[0], y[1]);
              pk.y = pack_bf16x2(y[2], y[3]);
              pk.z = pack_bf16x2(y[4], y[5]);
              pk.w = pack_bf16x2(y[6], y[7]);
              d4[v] = pk;
            }
          } else {
            atomicOr(p.err, kErrBounds);
          }
          float4* w4 = reinterpret_cast<float4*>(p.kw.w_out + static_cast<size_t>(t) * kHeads);
#pragma unroll
          for (int v = 0; v < 8; ++v)
            w4[v] = make_float4(__uint_as_float(wr[4 * v]), __uint_as_float(wr[4 * v + 1]),
                                __uint_as_float(wr[4 * v + 2]), __uint_as_float(wr[4 * v + 3]));
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ---------------------------------------------------------------- k|w projection, split over a cluster
// The k|w GEMM is bound by reading `hidden` (14,336 bytes per token): one CTA per 128-token
// tile streams the whole 7,168-wide contraction through one SM.  Here a cluster of CS CTAs
// shares each 128-token tile: CTA r accumulates k-blocks [r*nk/CS, (r+1)*nk/CS) in its TMEM,
// stores its partial [128 x 160] fp32 tile in its shared memory, and after a cluster barrier
// reduces 128/CS of the tile's rows over all CS partials through distributed shared memory
// (ld.shared::cluster), then applies the key LayerNorm, the bf16 cast and the key-cache
// scatter to those rows and stores their head weights.  Each row is handled by CS threads
// (128/CS key columns and 32/CS weight columns each); the LayerNorm's sums over the row are
// shuffles inside those CS lanes.

__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ uint32_t map_shared_rank(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}
__device__ __forceinline__ float4 ld_dsmem_f4(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(addr)
               : "memory");
  return v;
}

template <int CS, int STAGES, int H>
__global__ void __launch_bounds__(192, 1)
    proj_kw_cluster_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                           ProjParams p) {
  constexpr int BN = 128 + H;              // key columns, then the H head-weight columns
  constexpr int kPartStride = BN + 4;      // floats per row of the partial tile (conflict-free float4 stores)
  constexpr int kRows = kBM / CS;        // rows of the tile this CTA finishes
  constexpr int kKeyCols = 128 / CS;     // key columns per thread
  constexpr int kWCols = H / CS;         // weight columns per thread
  static_assert(CS == 2 || CS == 4 || CS == 8, "cluster of 2, 4 or 8");
  static_assert(kBM * kPartStride * 4 <= STAGES * ProjSmem<BN, STAGES>::kStageBytes, "partial fits the ring");
  using L = ProjSmem<BN, STAGES>;
  constexpr uint32_t kTmemCols = 256;
  static_assert(BN <= 256 && BN % 16 == 0, "one MMA covers the key and weight columns");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * kABytes;
  float* part = reinterpret_cast<float*>(smem);   // [kBM][kPartStride], over the ring once it is drained
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
  uint64_t* empty = full + STAGES;
  uint64_t* acc_full = empty + STAGES;
  uint64_t* mma_done = acc_full + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMiscOff + 4);
  float* s_gamma = reinterpret_cast<float*>(smem + L::kGammaOff);
  float* s_beta = s_gamma + 128;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int m0 = blockIdx.y * kBM;
  const int nk_all = p.K / kBK;
  const int kb0 = static_cast<int>(rank) * nk_all / CS, kb1 = (static_cast<int>(rank) + 1) * nk_all / CS;
  const int nk = kb1 - kb0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  if (threadIdx.x >= 64) {
    const int i = threadIdx.x - 64;
    s_gamma[i] = p.kw.gamma[i];
    s_beta[i] = p.kw.beta[i];
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const WaitCtl wc{p.err, abort_flag, p.timeout_ns};

  if (warp == 0) {
    if (lane == 0) {
      int issued = 0;
      for (int i = 0; i < nk; ++i) {
        const int s = i % STAGES;
        if (i >= STAGES && !mbar_wait(&empty[s], ((i / STAGES) - 1) & 1, wc)) break;
        mbar_arrive_expect_tx(&full[s], L::kStageBytes);
        tma_load_2d(sA + s * kABytes, &tmA, &full[s], (kb0 + i) * kBK, m0);
        tma_load_2d(sB + s * L::kBBytes, &tmB, &full[s], (kb0 + i) * kBK, 0);
        issued = i + 1;
      }
      if (*abort_flag) {
        for (int i = (issued > STAGES ? issued - STAGES : 0); i < issued; ++i)
          drain_wait(&full[i % STAGES], (i / STAGES) & 1);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = umma_idesc_bf16(kBM, BN);
      for (int i = 0; i < nk; ++i) {
        const int s = i % STAGES;
        if (!mbar_wait(&full[s], (i / STAGES) & 1, wc)) break;
        tc_fence_after();
        const uint32_t a = smem_u32(sA + s * kABytes);
        const uint32_t b = smem_u32(sB + s * L::kBBytes);
#pragma unroll
        for (int kk = 0; kk < kBK / 16; ++kk)
          umma_bf16(tmem, umma_desc_sw128(a + kk * 32), umma_desc_sw128(b + kk * 32), idesc, (i | kk) != 0);
        umma_commit(&empty[s]);
      }
      umma_commit(acc_full);
      umma_commit(mma_done);
      drain_wait(mma_done, 0);
    }
  } else {
    // this CTA's partial tile: TMEM lane = row, into shared memory (the ring is free: every
    // load issued was consumed by an MMA, and acc_full follows every MMA)
    const int qd = warp & 3;
    const int row = qd * 32 + lane;
    const bool ok = __all_sync(0xffffffffu, mbar_wait(acc_full, 0, wc));
    tc_fence_after();
    float4* prow = reinterpret_cast<float4*>(part + row * kPartStride);
    if (ok && nk > 0) {
      const uint32_t tbase = tmem + (static_cast<uint32_t>(qd * 32) << 16);
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        uint32_t r[32];
        tmem_ld_32cols(tbase + c * 32, r);
        tmem_ld_wait(r);
#pragma unroll
        for (int v = 0; v < 8; ++v)
          prow[c * 8 + v] = make_float4(__uint_as_float(r[4 * v]), __uint_as_float(r[4 * v + 1]),
                                        __uint_as_float(r[4 * v + 2]), __uint_as_float(r[4 * v + 3]));
      }
    } else {
      for (int v = 0; v < BN / 4; ++v) prow[v] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }
  __syncwarp();
  cluster_sync_all();   // every partial of the cluster is in place
  if (warp >= 2) {
    const int e = threadIdx.x - 64;
    const int rl = e / CS, t = e % CS;                 // row of this CTA's share, thread within the row
    const int trow = static_cast<int>(rank) * kRows + rl;  // row inside the tile
    float xk[kKeyCols], xw[kWCols];
#pragma unroll
    for (int i = 0; i < kKeyCols; ++i) xk[i] = 0.f;
#pragma unroll
    for (int i = 0; i < kWCols; ++i) xw[i] = 0.f;
    const uint32_t base = smem_u32(part + trow * kPartStride);
#pragma unroll 1
    for (int src = 0; src < CS; ++src) {
      const uint32_t rb = map_shared_rank(base, static_cast<uint32_t>(src));
#pragma unroll
      for (int v = 0; v < kKeyCols / 4; ++v) {
        const float4 f = ld_dsmem_f4(rb + (t * kKeyCols + 4 * v) * 4);
        xk[4 * v] += f.x;
        xk[4 * v + 1] += f.y;
        xk[4 * v + 2] += f.z;
        xk[4 * v + 3] += f.w;
      }
#pragma unroll
      for (int v = 0; v < kWCols / 4; ++v) {
        const float4 f = ld_dsmem_f4(rb + (128 + t * kWCols + 4 * v) * 4);
        xw[4 * v] += f.x;
        xw[4 * v + 1] += f.y;
        xw[4 * v + 2] += f.z;
        xw[4 * v + 3] += f.w;
      }
    }
    // LayerNorm over the 128 key columns of the row, spread over its CS threads
    float sum = 0.f;
#pragma unroll
    for (int i = 0; i < kKeyCols; ++i) sum += xk[i];
#pragma unroll
    for (int o = 1; o < CS; o <<= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    const float mean = sum * (1.0f / 128.0f);
    float ss = 0.f;
#pragma unroll
    for (int i = 0; i < kKeyCols; ++i) {
      const float d = xk[i] - mean;
      ss = fmaf(d, d, ss);
    }
#pragma unroll
    for (int o = 1; o < CS; o <<= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    const float rstd = rsqrtf(ss * (1.0f / 128.0f) + p.kw.eps);
    // the key: y = LayerNorm (fp32), rotary step on its first rope_dim dims, then bf16; the
    // FP8 cache stores e4m3 codes of the bf16 key with the row's scale (the shuffles run on
    // every lane, before the per-token branch)
    const int tok = m0 + trow;
    float y[kKeyCols];
#pragma unroll
    for (int i = 0; i < kKeyCols; ++i) {
      const int d = t * kKeyCols + i;
      y[i] = fmaf((xk[i] - mean) * rstd, s_gamma[d], s_beta[d]);
    }
    if (p.kw.rope_dim > 0 && tok < p.M)
      rope_rotate<kKeyCols>(y, t * kKeyCols, p.kw.positions[tok], p.kw.inv_freq, p.kw.rope_dim);
#pragma unroll
    for (int i = 0; i < kKeyCols; ++i) y[i] = round_bf16(y[i]);
    const bool fp8 = p.kw.key8 != nullptr;
    float scale8 = 0.f, inv8 = 0.f;
    if (fp8) {
      float amax = 0.f;
#pragma unroll
      for (int i = 0; i < kKeyCols; ++i) amax = fmaxf(amax, fabsf(y[i]));
#pragma unroll
      for (int o = 1; o < CS; o <<= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
      fp8_row_scale(amax, &scale8, &inv8);
    }
    if (tok < p.M) {
      const int pos = p.kw.positions[tok];
      int lo = 0, hi = p.kw.B - 1;   // sequence of the token: the last b with q_seq_offsets[b] <= tok
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (p.kw.q_seq_offsets[mid] <= tok) lo = mid;
        else hi = mid - 1;
      }
      const int64_t cb = p.kw.cache_offsets[lo];
      const int64_t len = p.kw.cache_offsets[lo + 1] - cb;
      const bool in_cache = pos >= 0 && pos < len && cb >= 0 && cb + pos < p.kw.cache_rows;
      if (!in_cache) {
        if (t == 0) atomicOr(p.err, kErrBounds);
      } else if (fp8) {
        uint32_t* d32 = reinterpret_cast<uint32_t*>(p.kw.key8 + static_cast<size_t>(cb + pos) * kHeadDim +
                                                    t * kKeyCols);
#pragma unroll
        for (int v = 0; v < kKeyCols / 4; ++v)
          d32[v] = pack_e4m3x4(__fmul_rn(y[4 * v], inv8), __fmul_rn(y[4 * v + 1], inv8),
                               __fmul_rn(y[4 * v + 2], inv8), __fmul_rn(y[4 * v + 3], inv8));
        if (t == 0) p.kw.key_scale[cb + pos] = scale8;
      } else {
        uint4* d4 = reinterpret_cast<uint4*>(p.kw.key_cache + static_cast<size_t>(cb + pos) * kHeadDim +
                                             t * kKeyCols);
#pragma unroll
        for (int v = 0; v < kKeyCols / 8; ++v) {
          uint4 pk;
          pk.x = pack_bf16x2(y[8 * v], y[8 * v + 1]);
          pk.y = pack_bf16x2(y[8 * v + 2], y[8 * v + 3]);
          pk.z = pack_bf16x2(y[8 * v + 4], y[8 * v + 5]);
          pk.w = pack_bf16x2(y[8 * v + 6], y[8 * v + 7]);
          d4[v] = pk;
        }
      }
      float4* w4 = reinterpret_cast<float4*>(p.kw.w_out + static_cast<size_t>(tok) * H + t * kWCols);
#pragma unroll
      for (int v = 0; v < kWCols / 4; ++v)
        w4[v] = make_float4(xw[4 * v], xw[4 * v + 1], xw[4 * v + 2], xw[4 * v + 3]);
    }
  }
  __syncwarp();
  cluster_sync_all();   // no CTA leaves while a peer may still read its partial
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ---------------------------------------------------------------- key LayerNorm on its own
__global__ void __launch_bounds__(256) key_norm_kernel(int64_t n, const float* __restrict__ raw,
                                                       __nv_bfloat16* __restrict__ out, const float* __restrict__ gamma,
                                                       const float* __restrict__ beta, float eps) {
  const int64_t row = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= n) return;
  const float4 v = reinterpret_cast<const float4*>(raw + row * kHeadDim)[lane];
  float s = v.x + v.y + v.z + v.w;
#pragma unroll
  for (int o = 16; o; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  const float mean = s * (1.0f / 128.0f);
  const float d0 = v.x - mean, d1 = v.y - mean, d2 = v.z - mean, d3 = v.w - mean;
  float ss = d0 * d0 + d1 * d1 + d2 * d2 + d3 * d3;
#pragma unroll
  for (int o = 16; o; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  const float rstd = rsqrtf(ss * (1.0f / 128.0f) + eps);
  const float4 g = reinterpret_cast<const float4*>(gamma)[lane];
  const float4 b = reinterpret_cast<const float4*>(beta)[lane];
  uint2 pk;
  pk.x = pack_bf16x2(fmaf(d0 * rstd, g.x, b.x), fmaf(d1 * rstd, g.y, b.y));
  pk.y = pack_bf16x2(fmaf(d2 * rstd, g.z, b.z), fmaf(d3 * rstd, g.w, b.w));
  reinterpret_cast<uint2*>(out + row * kHeadDim)[lane] = pk;
}

// ---------------------------------------------------------------- bf16 key rows -> FP8 cache rows
// One warp per 128-value row: each lane converts 4 values; the row's largest magnitude comes
// from a warp reduction.
__global__ void __launch_bounds__(256) quantize_keys_fp8_kernel(int64_t n, const __nv_bfloat16* __restrict__ keys,
                                                                uint8_t* __restrict__ out, float* __restrict__ scale) {
  const int64_t row = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= n) return;
  const uint2 raw = reinterpret_cast<const uint2*>(keys + row * kHeadDim)[lane];
  const __nv_bfloat162 b0 = *reinterpret_cast<const __nv_bfloat162*>(&raw.x);
  const __nv_bfloat162 b1 = *reinterpret_cast<const __nv_bfloat162*>(&raw.y);
  const float v0 = __low2float(b0), v1 = __high2float(b0), v2 = __low2float(b1), v3 = __high2float(b1);
  float amax = fmaxf(fmaxf(fabsf(v0), fabsf(v1)), fmaxf(fabsf(v2), fabsf(v3)));
#pragma unroll
  for (int o = 16; o; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  float sc, inv;
  fp8_row_scale(amax, &sc, &inv);
  reinterpret_cast<uint32_t*>(out + row * kHeadDim)[lane] =
      pack_e4m3x4(__fmul_rn(v0, inv), __fmul_rn(v1, inv), __fmul_rn(v2, inv), __fmul_rn(v3, inv));
  if (lane == 0) scale[row] = sc;
}

// ---------------------------------------------------------------- weight re-layout at create
__global__ void transpose_bf16_kernel(const __nv_bfloat16* __restrict__ src, int K, int N,
                                      __nv_bfloat16* __restrict__ dst, int dst_row0) {
  __shared__ __nv_bfloat16 tile[32][33];
  const int k0 = blockIdx.y * 32, n0 = blockIdx.x * 32;
  for (int i = threadIdx.y; i < 32; i += 8) {
    const int k = k0 + i, nn = n0 + threadIdx.x;
    if (k < K && nn < N) tile[i][threadIdx.x] = src[static_cast<size_t>(k) * N + nn];
  }
  __syncthreads();
  for (int i = threadIdx.y; i < 32; i += 8) {
    const int nn = n0 + i, k = k0 + threadIdx.x;
    if (k < K && nn < N) dst[static_cast<size_t>(dst_row0 + nn) * K + k] = tile[threadIdx.x][i];
  }
}

template <int BN, int STAGES, int EPI>
cudaError_t launch_proj(const CUtensorMap& tmA, const CUtensorMap& tmB, const ProjParams& p, int n_tiles,
                        cudaStream_t s) {
  using L = ProjSmem<BN, STAGES>;
  auto kern = proj_gemm_kernel<BN, STAGES, EPI>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kTotal);
  if (e != cudaSuccess) return e;
  dim3 grid(n_tiles, (p.M + kBM - 1) / kBM);
  kern<<<grid, 192, L::kTotal, s>>>(tmA, tmB, p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_proj_q(const CUtensorMap& tmA, const CUtensorMap& tmB, int M, int K, int N,
                          __nv_bfloat16* q_out, int* err, uint64_t timeout_ns, cudaStream_t s,
                          const int32_t* positions, const double* inv_freq, int rope_dim) {
  ProjParams p{};
  p.positions = positions;
  p.inv_freq = inv_freq;
  p.rope_dim = rope_dim;
  p.M = M;
  p.K = K;
  p.q_out = q_out;
  p.ldq = N;
  p.err = err;
  p.timeout_ns = timeout_ns;
  return launch_proj<256, 4, EPI_Q>(tmA, tmB, p, N / 256, s);
}

template <int CS, int H>
cudaError_t launch_kw_cluster(const CUtensorMap& tmA, const CUtensorMap& tmB, const ProjParams& p, cudaStream_t s) {
  using L = ProjSmem<128 + H, 5>;
  auto kern = proj_kw_cluster_kernel<CS, 5, H>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kTotal);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(CS, (p.M + kBM - 1) / kBM);
  cfg.blockDim = dim3(192);
  cfg.dynamicSmemBytes = L::kTotal;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = CS;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, tmA, tmB, p);
}

cudaError_t launch_proj_kw(const CUtensorMap& tmA, const CUtensorMap& tmB, int K, const ProjKwEpilogue& e,
                           cudaStream_t s) {
  ProjParams p{};
  p.M = e.M;
  p.K = K;
  p.kw = e;
  p.err = e.err;
  p.timeout_ns = e.timeout_ns;
  const int nk = K / kBK;
  const int tiles = (e.M + kBM - 1) / kBM;
  // Few token tiles (decode): split the contraction over a cluster so that more SMs stream
  // `hidden`.  Many tiles: the q GEMM runs next to this kernel, and one CTA per tile leaves it
  // the most SMs (measured: 0.149 ms for both GEMMs at 8,192 tokens with one CTA per tile,
  // 0.155 / 0.172 / 0.207 ms with clusters of 2 / 4 / 8).  The single-CTA kernel has the bf16,
  // 32-head, no-rotary epilogue; the other forms use clusters of at least 2.
  const bool plain = e.key8 == nullptr && e.rope_dim == 0 && e.n_heads == 32;
  int cs = tiles <= 2 ? 8 : tiles <= 4 ? 4 : tiles <= 8 ? 2 : 1;
  if (cs == 1 && !plain) cs = 2;
  while (cs > 1 && nk < cs) cs >>= 1;   // at least one k-block per CTA of the cluster
  if (cs == 1) {
    if (!plain) return cudaErrorInvalidValue;
    return launch_proj<160, 5, EPI_KW>(tmA, tmB, p, 1, s);
  }
  if (e.n_heads == 64) {
    if (cs == 8) return launch_kw_cluster<8, 64>(tmA, tmB, p, s);
    if (cs == 4) return launch_kw_cluster<4, 64>(tmA, tmB, p, s);
    return launch_kw_cluster<2, 64>(tmA, tmB, p, s);
  }
  if (cs == 8) return launch_kw_cluster<8, 32>(tmA, tmB, p, s);
  if (cs == 4) return launch_kw_cluster<4, 32>(tmA, tmB, p, s);
  return launch_kw_cluster<2, 32>(tmA, tmB, p, s);
}

cudaError_t launch_proj_q8(const CUtensorMap& tmA, const CUtensorMap& tmB, int M, int K, int N, uint8_t* q8_out,
                           float* q_scale, int* err, uint64_t timeout_ns, cudaStream_t s) {
  ProjParams p{};
  p.M = M;
  p.K = K;
  p.q8_out = q8_out;
  p.q_scale = q_scale;
  p.ldq = N;
  p.err = err;
  p.timeout_ns = timeout_ns;
  return launch_proj<256, 4, EPI_Q8>(tmA, tmB, p, N / 256, s);
}

cudaError_t launch_quantize_keys_fp8(int64_t n, const __nv_bfloat16* keys, uint8_t* out, float* scale,
                                     cudaStream_t s) {
  if (n <= 0) return cudaSuccess;
  const int64_t blocks = (n + 7) / 8;
  quantize_keys_fp8_kernel<<<static_cast<unsigned>(blocks), 256, 0, s>>>(n, keys, out, scale);
  return cudaGetLastError();
}

cudaError_t launch_key_norm(int64_t n, const float* raw, __nv_bfloat16* out, const float* gamma,
                            const float* beta, float eps, cudaStream_t s) {
  if (n <= 0) return cudaSuccess;
  const int64_t blocks = (n + 7) / 8;
  key_norm_kernel<<<static_cast<unsigned>(blocks), 256, 0, s>>>(n, raw, out, gamma, beta, eps);
  return cudaGetLastError();
}

cudaError_t launch_transpose_bf16(const __nv_bfloat16* src, int K, int N, __nv_bfloat16* dst, int dst_row0,
                                  cudaStream_t s) {
  dim3 grid((N + 31) / 32, (K + 31) / 32);
  transpose_bf16_kernel<<<grid, dim3(32, 8), 0, s>>>(src, K, N, dst, dst_row0);
  return cudaGetLastError();
}

}  // namespace dsa
