// score_topk.cu -- indexer score I[t,s] = sum_h w[t,h] * ReLU(q[t,h] . k[s]) over the
// causal prefix of every query, and the streaming top-2,048 selection.
//
// 'Sparse / compressed attn' row (Kimi K3.1 Pro): scores I = sum_h w_h ReLU(q_h . k)
// pick the top 2,048 tokens per query; 'Long-context extension' row: the indexer
// scores the whole prefix.  Nothing of size T x S is ever written to memory.
//
// Work items.  prep_kernel (one CTA) validates the offsets/positions and writes a
// list of work items: on the prefill path an item is up to 8 consecutive queries
// of one sequence scored against every key up to the last query's position; on
// the split-key path (few queries, long prefixes: decode) an item is one query
// against one key chunk, and merge_kernel combines the chunks' partial lists.
// Items are listed longest first and handed out by an atomic counter.
//
// score_topk_kernel (persistent, one CTA per SM):
//   warp 0     TMA producer: the item's Q tile (nq*32 rows of [T*32, 128] bf16,
//              K-major) once, then 128-key tiles of the key cache into a ring.
//   warp 1     MMA issuer: D[key, (query, head)] = K_tile (M=128) x Q^T (N=nq*32),
//              K=128 as 8 tcgen05.mma of K=16, into one of ACC_BUFS TMEM buffers.
//   warps 2..  epilogue warpgroups (4 warps = the 4 TMEM lane quadrants).  Thread
//              (quadrant, lane) owns one key; per query it loads that query's 32
//              head columns (tcgen05.ld 32x32b.x32), applies ReLU and the fp32
//              head weights in registers, masks s > pos, and appends (score, s)
//              to the query's candidate list if the score reaches the query's
//              running threshold (warp ballot + one shared atomic per warp).
//              A list that nears its capacity is compacted to its best 2,048
//              (radix select in shared memory), which raises the threshold.
//              At the end of the item each list is reduced to exactly the top
//              2,048 and written out.

#include "kernels.h"

namespace dsa {
namespace {

constexpr uint64_t kDrainNs = 200ull * 1000 * 1000;

struct ScoreParams {
  const WorkItem* items;
  const int* n_items;
  int* work_counter;
  const float* w;               // [T, 32]
  const int* pos_eff;           // [T]
  const int64_t* cache_offsets; // [B+1]
  int32_t* idx_out;             // [T, 2048]
  float* score_out;             // [T, 2048] or null
  uint32_t* cand_keys;          // [slots][QMAX][kCandStride]
  int32_t* cand_idx;
  uint32_t* part_keys;          // [T][kMaxChunks][kTopK]
  int32_t* part_idx;
  int* err;
  uint64_t timeout_ns;
};

__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) {
  const uint32_t a = smem_u32(bar);
  const uint64_t t0 = global_timer_ns();
  while (!mbar_try_wait(a, parity)) {
    if (global_timer_ns() - t0 > kDrainNs) break;
  }
}

// ------------------------------------------------------------------------------------------
// Radix select over `n` order-preserving keys held in shared memory by a group of NT
// threads (tid = 0..NT-1, named barrier `bar`).  Returns the k-th largest key K*
// (1 <= k <= n); *n_above receives the number of keys strictly greater than K*.
// Four passes of 8 bits, most significant first; each pass histograms the keys that
// match the prefix found so far (warp-aggregated shared atomics).
template <int NT>
__device__ uint32_t radix_kth(const uint32_t* skeys, int n, int k, uint32_t* hist, int* sh, int tid, int bar,
                              int* n_above) {
  const int lane = tid & 31;
  uint32_t prefix = 0, mask = 0;
  int need = k;
#pragma unroll 1
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int i = tid; i < 256; i += NT) hist[i] = 0;
    named_bar_sync(bar, NT);
    for (int base = 0; base < n; base += NT) {
      const int e = base + tid;
      const uint32_t key = (e < n) ? skeys[e] : 0u;
      const bool act = (e < n) && ((key & mask) == prefix);
      const uint32_t bin = act ? ((key >> shift) & 255u) : 256u;
      const uint32_t peers = __match_any_sync(0xffffffffu, bin);
      if (act && lane == __ffs(peers) - 1) atomicAdd(&hist[bin], static_cast<uint32_t>(__popc(peers)));
    }
    named_bar_sync(bar, NT);
    if (tid < 32) {
      // lane l owns bins 255-8l .. 248-8l (from the top)
      uint32_t c[8], tot = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        c[i] = hist[255 - 8 * lane - i];
        tot += c[i];
      }
      uint32_t incl = tot;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += y;
      }
      const uint32_t excl = incl - tot;
      if (excl < static_cast<uint32_t>(need) && static_cast<uint32_t>(need) <= incl) {
        uint32_t cum = excl;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          if (cum + c[i] >= static_cast<uint32_t>(need)) {
            sh[0] = 255 - 8 * lane - i;
            sh[1] = static_cast<int>(cum);
            break;
          }
          cum += c[i];
        }
      }
    }
    named_bar_sync(bar, NT);
    const uint32_t bin = static_cast<uint32_t>(sh[0]);
    need -= sh[1];
    prefix |= bin << shift;
    mask |= 255u << shift;
    named_bar_sync(bar, NT);
  }
  *n_above = k - need;
  return prefix;
}

// Emits the top k of n candidate (key, idx) pairs: every key > kth and the first
// (k - n_above) keys equal to kth.  sink(slot, key, e) is called once per kept
// entry with a distinct slot in [0, k).  ctr[0..1] are zeroed shared counters.
template <int NT, class Sink>
__device__ void emit_topk(const uint32_t* skeys, int n, int k, uint32_t kth, int n_above, int* ctr, int tid,
                          Sink sink) {
  const int lane = tid & 31;
  const int ties = k - n_above;
  for (int base = 0; base < n; base += NT) {
    const int e = base + tid;
    const uint32_t key = (e < n) ? skeys[e] : 0u;
    const bool gt = (e < n) && key > kth;
    const bool eq = (e < n) && key == kth;
    const uint32_t bg = __ballot_sync(0xffffffffu, gt);
    const uint32_t be = __ballot_sync(0xffffffffu, eq);
    int b0 = 0, b1 = 0;
    if (lane == 0) {
      if (bg) b0 = atomicAdd(&ctr[0], __popc(bg));
      if (be) b1 = atomicAdd(&ctr[1], __popc(be));
    }
    b0 = __shfl_sync(0xffffffffu, b0, 0);
    b1 = __shfl_sync(0xffffffffu, b1, 0);
    if (gt) sink(b0 + __popc(bg & lanemask_lt()), key, e);
    if (eq) {
      const int r = b1 + __popc(be & lanemask_lt());
      if (r < ties) sink(n_above + r, key, e);
    }
  }
}

// ------------------------------------------------------------------------------------------
template <int QPW>
struct WGState {
  uint32_t skeys[kCandCap];   // staged candidate keys for a selection
  uint32_t hist[256];
  float w[QPW][kHeads];
  int cnt[QPW];
  uint32_t thr[QPW];
  int pos[QPW];
  int sh[4];
  int ctr[2];
};

template <int QMAX, int STAGES, int ACC_BUFS, int NWG>
struct ScoreCfg {
  static constexpr int kQPW = QMAX / NWG;
  static constexpr int kThreads = 64 + NWG * 128;
  static constexpr int kAccCols = QMAX * kHeads;
  static constexpr int kTmemNeed = ACC_BUFS * kAccCols;
  static constexpr int kTmemCols = kTmemNeed <= 32 ? 32 : kTmemNeed <= 64 ? 64 : kTmemNeed <= 128 ? 128
                                   : kTmemNeed <= 256 ? 256 : 512;
  static constexpr int kQHalf = QMAX * kHeads * 128;  // bytes of one 64-column half of the Q tile
  static constexpr int kKHalf = kKeyTile * 128;       // 16 KB
  static constexpr int kKStage = 2 * kKHalf;
  static constexpr int kQOff = 0;
  static constexpr int kKOff = 2 * kQHalf;
  static constexpr int kWGOff = kKOff + STAGES * kKStage;
  static constexpr int kWGBytes = (static_cast<int>(sizeof(WGState<kQPW>)) + 15) / 16 * 16;
  static constexpr int kBarOff = kWGOff + NWG * kWGBytes;
  static constexpr int kNumBars = 2 * STAGES + 2 * ACC_BUFS + 2 + 4 + 1;
  static constexpr int kMiscOff = kBarOff + 8 * kNumBars;
  static constexpr int kSmemBytes = kMiscOff + 64 + 1024;
  static_assert(kTmemNeed <= 512, "TMEM holds 512 columns");
  static_assert(kQHalf % 1024 == 0, "Q halves must stay 1024-byte aligned");
};

template <int QMAX, int STAGES, int ACC_BUFS, int NWG>
__global__ void __launch_bounds__(ScoreCfg<QMAX, STAGES, ACC_BUFS, NWG>::kThreads, 1)
    score_topk_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                      ScoreParams p) {
  using C = ScoreCfg<QMAX, STAGES, ACC_BUFS, NWG>;
  constexpr int QPW = C::kQPW;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem + C::kQOff;
  uint8_t* sK = smem + C::kKOff;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
  uint64_t* full = bars;
  uint64_t* empty = full + STAGES;
  uint64_t* acc_full = empty + STAGES;
  uint64_t* acc_empty = acc_full + ACC_BUFS;
  uint64_t* q_full = acc_empty + ACC_BUFS;
  uint64_t* q_empty = q_full + 1;
  uint64_t* sched_full = q_empty + 1;
  uint64_t* sched_empty = sched_full + 2;
  uint64_t* mma_done = sched_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kMiscOff + 4);
  volatile int* sched_item = reinterpret_cast<volatile int*>(smem + C::kMiscOff + 8);  // [2]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < ACC_BUFS; ++a) {
      mbar_init(&acc_full[a], 1);
      mbar_init(&acc_empty[a], NWG * 4);
    }
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sched_full[i], 1);
      mbar_init(&sched_empty[i], 1 + NWG * 4);
    }
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int n_items = *p.n_items;
  const WaitCtl wc{p.err, abort_flag, p.timeout_ns};

  if (warp == 0) {
    // ===================================================== TMA producer
    if (lane == 0) {
      int kstage = 0, qloads = 0;
      for (int local = 0;; ++local) {
        const int slot = local & 1;
        if (local >= 2 && !mbar_wait(&sched_empty[slot], ((local >> 1) - 1) & 1, wc)) break;
        int it = atomicAdd(p.work_counter, 1);
        if (it >= n_items) it = -1;
        sched_item[slot] = it;
        mbar_arrive(&sched_full[slot]);
        if (it < 0) break;
        const WorkItem wi = p.items[it];
        const int kt0 = wi.k_begin / kKeyTile, kt1 = (wi.k_end + kKeyTile - 1) / kKeyTile;
        if (kt1 <= kt0) continue;
        if (qloads > 0 && !mbar_wait(q_empty, (qloads - 1) & 1, wc)) break;
        mbar_arrive_expect_tx(q_full, 2 * C::kQHalf);
        tma_load_2d(sQ, &tmQ, q_full, 0, wi.t0 * kHeads);
        tma_load_2d(sQ + C::kQHalf, &tmQ, q_full, 64, wi.t0 * kHeads);
        ++qloads;
        const int row0 = static_cast<int>(p.cache_offsets[wi.b]);
        bool ok = true;
        for (int kt = kt0; kt < kt1; ++kt, ++kstage) {
          const int s = kstage % STAGES;
          if (kstage >= STAGES && !mbar_wait(&empty[s], ((kstage / STAGES) - 1) & 1, wc)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[s], C::kKStage);
          uint8_t* dst = sK + s * C::kKStage;
          tma_load_2d(dst, &tmK, &full[s], 0, row0 + kt * kKeyTile);
          tma_load_2d(dst + C::kKHalf, &tmK, &full[s], 64, row0 + kt * kKeyTile);
        }
        if (!ok) break;
      }
      if (*abort_flag) {
        for (int ks = (kstage > STAGES ? kstage - STAGES : 0); ks < kstage; ++ks)
          drain_wait(&full[ks % STAGES], (ks / STAGES) & 1);
        if (qloads > 0) drain_wait(q_full, (qloads - 1) & 1);
      }
    }
  } else if (warp == 1) {
    // ===================================================== MMA issuer
    if (lane == 0) {
      int kstage = 0, acc_ctr = 0, qloads = 0;
      const uint32_t qa = smem_u32(sQ);
      for (int local = 0;; ++local) {
        const int slot = local & 1;
        if (!mbar_wait(&sched_full[slot], (local >> 1) & 1, wc)) break;
        const int it = sched_item[slot];
        mbar_arrive(&sched_empty[slot]);
        if (it < 0) break;
        const WorkItem wi = p.items[it];
        const int kt0 = wi.k_begin / kKeyTile, kt1 = (wi.k_end + kKeyTile - 1) / kKeyTile;
        if (kt1 <= kt0) continue;
        if (!mbar_wait(q_full, qloads & 1, wc)) break;
        ++qloads;
        tc_fence_after();
        const uint32_t idesc = umma_idesc_bf16(kKeyTile, wi.nq * kHeads);
        bool ok = true;
        for (int kt = kt0; kt < kt1; ++kt, ++kstage, ++acc_ctr) {
          const int s = kstage % STAGES;
          const int ab = acc_ctr % ACC_BUFS;
          if (!mbar_wait(&full[s], (kstage / STAGES) & 1, wc)) { ok = false; break; }
          if (acc_ctr >= ACC_BUFS && !mbar_wait(&acc_empty[ab], ((acc_ctr / ACC_BUFS) - 1) & 1, wc)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t d = tmem + ab * C::kAccCols;
          const uint32_t ka = smem_u32(sK + s * C::kKStage);
#pragma unroll
          for (int kb = 0; kb < 2; ++kb)
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              umma_bf16(d, umma_desc_sw128(ka + kb * C::kKHalf + kk * 32),
                        umma_desc_sw128(qa + kb * C::kQHalf + kk * 32), idesc, (kb | kk) != 0);
          umma_commit(&empty[s]);
          umma_commit(&acc_full[ab]);
        }
        umma_commit(q_empty);
        if (!ok) break;
      }
      umma_commit(mma_done);
      drain_wait(mma_done, 0);
    }
  } else {
    // ===================================================== epilogue warpgroups
    const int ew = warp - 2;
    const int g = ew >> 2;                 // warpgroup
    const int qd = warp & 3;               // TMEM lane quadrant of this warp
    const int gtid = threadIdx.x - 64 - g * 128;
    const int bar = 1 + g;
    const int r = qd * 32 + lane;          // key row of this thread inside a tile
    WGState<QPW>& st = *reinterpret_cast<WGState<QPW>*>(smem + C::kWGOff + g * C::kWGBytes);
    const uint32_t tlane = tmem + (static_cast<uint32_t>(qd * 32) << 16);
    int acc_ctr = 0;

    for (int local = 0;; ++local) {
      const int slot = local & 1;
      const bool got = __all_sync(0xffffffffu, mbar_wait(&sched_full[slot], (local >> 1) & 1, wc));
      const int it = got ? sched_item[slot] : -1;
      __syncwarp();
      if (lane == 0 && got) mbar_arrive(&sched_empty[slot]);
      WorkItem wi;
      if (it >= 0) wi = p.items[it];
      if (gtid < QPW && it >= 0) {
        const int j = g * QPW + gtid;
        st.cnt[gtid] = 0;
        st.thr[gtid] = 0u;
        st.pos[gtid] = (j < wi.nq) ? p.pos_eff[wi.t0 + j] : -2;
      }
      if (it >= 0) {
        for (int i = gtid; i < QPW * kHeads; i += 128) {
          const int jj = i / kHeads, j = g * QPW + jj;
          st.w[jj][i % kHeads] = (j < wi.nq) ? p.w[static_cast<size_t>(wi.t0 + j) * kHeads + (i % kHeads)] : 0.f;
        }
      }
      if (named_bar_or(bar, 128, it < 0)) break;   // every thread of the group leaves together

      const int nloc = min(QPW, wi.nq - g * QPW);
      const int kt0 = wi.k_begin / kKeyTile, kt1 = (wi.k_end + kKeyTile - 1) / kKeyTile;
      bool failed = false;
      for (int kt = kt0; kt < kt1; ++kt, ++acc_ctr) {
        const int ab = acc_ctr % ACC_BUFS;
        const bool ok = __all_sync(0xffffffffu, mbar_wait(&acc_full[ab], (acc_ctr / ACC_BUFS) & 1, wc));
        tc_fence_after();
        bool need = false;
        const int s_pos = kt * kKeyTile + r;
        if (ok) {
#pragma unroll 1
          for (int jj = 0; jj < nloc; ++jj) {
            uint32_t v[32];
            tmem_ld_32cols(tlane + ab * C::kAccCols + (g * QPW + jj) * kHeads, v);
            tmem_ld_wait(v);
            const float4* w4 = reinterpret_cast<const float4*>(st.w[jj]);
            float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll
            for (int h4 = 0; h4 < 8; ++h4) {
              const float4 ww = w4[h4];
              a0 = fmaf(ww.x, fmaxf(__uint_as_float(v[4 * h4 + 0]), 0.f), a0);
              a1 = fmaf(ww.y, fmaxf(__uint_as_float(v[4 * h4 + 1]), 0.f), a1);
              a2 = fmaf(ww.z, fmaxf(__uint_as_float(v[4 * h4 + 2]), 0.f), a2);
              a3 = fmaf(ww.w, fmaxf(__uint_as_float(v[4 * h4 + 3]), 0.f), a3);
            }
            const float score = (a0 + a1) + (a2 + a3);
            const uint32_t u = float_to_ordered(score);
            const bool pass = (s_pos < wi.k_end) && (s_pos <= st.pos[jj]) && (u >= st.thr[jj]);
            const uint32_t bal = __ballot_sync(0xffffffffu, pass);
            if (bal) {
              int base = 0;
              if (lane == 0) {
                base = atomicAdd(&st.cnt[jj], __popc(bal));
                if (base + __popc(bal) > kCandCap - kKeyTile) need = true;
              }
              base = __shfl_sync(0xffffffffu, base, 0);
              if (pass) {
                const size_t q = (static_cast<size_t>(blockIdx.x) * QMAX + g * QPW + jj) * kCandStride;
                const int o = base + __popc(bal & lanemask_lt());
                p.cand_keys[q + o] = u;
                p.cand_idx[q + o] = s_pos;
              }
            }
          }
        } else {
          failed = true;
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0 && ok) mbar_arrive(&acc_empty[ab]);
        if (named_bar_or(bar, 128, need || failed)) {
          if (named_bar_or(bar, 128, failed)) { failed = true; break; }
          int cnts[QPW];
#pragma unroll
          for (int jj = 0; jj < QPW; ++jj) cnts[jj] = st.cnt[jj];
#pragma unroll 1
          for (int jj = 0; jj < QPW; ++jj) {
            if (jj >= nloc || cnts[jj] <= kCandCap - kKeyTile) continue;
            // ---- compaction: keep the best kTopK candidates, raise the threshold
            const size_t q = (static_cast<size_t>(blockIdx.x) * QMAX + g * QPW + jj) * kCandStride;
            uint32_t* ck = p.cand_keys + q;
            int32_t* ci = p.cand_idx + q;
            const int n = cnts[jj];
            for (int e = gtid; e < n; e += 128) st.skeys[e] = ck[e];
            if (gtid == 0) { st.ctr[0] = 0; st.ctr[1] = 0; }
            named_bar_sync(bar, 128);
            int above;
            const uint32_t kth = radix_kth<128>(st.skeys, n, kTopK, st.hist, st.sh, gtid, bar, &above);
            emit_topk<128>(st.skeys, n, kTopK, kth, above, st.ctr, gtid, [&](int slot2, uint32_t key, int e) {
              ck[kCandCap + slot2] = key;
              ci[kCandCap + slot2] = ci[e];
            });
            named_bar_sync(bar, 128);
            for (int e = gtid; e < kTopK; e += 128) {
              ck[e] = ck[kCandCap + e];
              ci[e] = ci[kCandCap + e];
            }
            if (gtid == 0) {
              st.cnt[jj] = kTopK;
              st.thr[jj] = (kth == 0xFFFFFFFFu) ? kth : kth + 1u;
            }
            named_bar_sync(bar, 128);
          }
        }
      }
      if (failed) break;

      // ---- end of item: exact top-k of each query's list
#pragma unroll 1
      for (int jj = 0; jj < nloc; ++jj) {
        const int t = wi.t0 + g * QPW + jj;
        const size_t q = (static_cast<size_t>(blockIdx.x) * QMAX + g * QPW + jj) * kCandStride;
        const uint32_t* ck = p.cand_keys + q;
        const int32_t* ci = p.cand_idx + q;
        const int n = st.cnt[jj];
        if (wi.chunk < 0) {
          int32_t* oi = p.idx_out + static_cast<size_t>(t) * kTopK;
          float* os = p.score_out ? p.score_out + static_cast<size_t>(t) * kTopK : nullptr;
          const int prefix = st.pos[jj] + 1;   // keys this query scores (0 if invalid)
          if (prefix <= kTopK) {
            for (int e = gtid; e < n; e += 128) {
              const int s = ci[e];
              oi[s] = s;
              if (os) os[s] = ordered_to_float(ck[e]);
            }
            for (int s = max(prefix, 0) + gtid; s < kTopK; s += 128) {
              oi[s] = -1;
              if (os) os[s] = -INFINITY;
            }
          } else {
            for (int e = gtid; e < n; e += 128) st.skeys[e] = ck[e];
            if (gtid == 0) { st.ctr[0] = 0; st.ctr[1] = 0; }
            named_bar_sync(bar, 128);
            int above;
            const uint32_t kth = radix_kth<128>(st.skeys, n, kTopK, st.hist, st.sh, gtid, bar, &above);
            emit_topk<128>(st.skeys, n, kTopK, kth, above, st.ctr, gtid, [&](int slot2, uint32_t key, int e) {
              oi[slot2] = ci[e];
              if (os) os[slot2] = ordered_to_float(key);
            });
          }
        } else {
          uint32_t* pk = p.part_keys + (static_cast<size_t>(t) * kMaxChunks + wi.chunk) * kTopK;
          int32_t* pi = p.part_idx + (static_cast<size_t>(t) * kMaxChunks + wi.chunk) * kTopK;
          if (n <= kTopK) {
            for (int e = gtid; e < kTopK; e += 128) {
              pk[e] = (e < n) ? ck[e] : 0u;
              pi[e] = (e < n) ? ci[e] : -1;
            }
          } else {
            for (int e = gtid; e < n; e += 128) st.skeys[e] = ck[e];
            if (gtid == 0) { st.ctr[0] = 0; st.ctr[1] = 0; }
            named_bar_sync(bar, 128);
            int above;
            const uint32_t kth = radix_kth<128>(st.skeys, n, kTopK, st.hist, st.sh, gtid, bar, &above);
            emit_topk<128>(st.skeys, n, kTopK, kth, above, st.ctr, gtid, [&](int slot2, uint32_t key, int e) {
              pk[slot2] = key;
              pi[slot2] = ci[e];
            });
          }
        }
        named_bar_sync(bar, 128);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

// ------------------------------------------------------------------------------------------
// merge of the split-key path: top-k over the kMaxChunks partial lists of one query
constexpr int kMergeThreads = 512;

__global__ void __launch_bounds__(kMergeThreads) merge_kernel(const uint32_t* __restrict__ part_keys,
                                                              const int32_t* __restrict__ part_idx,
                                                              const int* __restrict__ tok_nchunks,
                                                              int32_t* __restrict__ idx_out,
                                                              float* __restrict__ score_out) {
  extern __shared__ uint32_t mkeys[];  // [kMaxChunks * kTopK]
  __shared__ uint32_t hist[256];
  __shared__ int sh[4];
  __shared__ int ctr[2];
  const int t = blockIdx.x;
  const int nch = tok_nchunks[t];
  if (nch < 2) return;
  const int n = nch * kTopK;
  const uint32_t* pk = part_keys + static_cast<size_t>(t) * kMaxChunks * kTopK;
  const int32_t* pi = part_idx + static_cast<size_t>(t) * kMaxChunks * kTopK;
  for (int e = threadIdx.x * 4; e < n; e += kMergeThreads * 4)
    *reinterpret_cast<uint4*>(mkeys + e) = *reinterpret_cast<const uint4*>(pk + e);
  if (threadIdx.x == 0) { ctr[0] = 0; ctr[1] = 0; }
  __syncthreads();
  int above;
  const uint32_t kth = radix_kth<kMergeThreads>(mkeys, n, kTopK, hist, sh, threadIdx.x, 1, &above);
  int32_t* oi = idx_out + static_cast<size_t>(t) * kTopK;
  float* os = score_out ? score_out + static_cast<size_t>(t) * kTopK : nullptr;
  emit_topk<kMergeThreads>(mkeys, n, kTopK, kth, above, ctr, threadIdx.x, [&](int slot, uint32_t key, int e) {
    oi[slot] = pi[e];
    if (os) os[slot] = ordered_to_float(key);
  });
}

// ------------------------------------------------------------------------------------------
// prep: validate, build the work list (one CTA)
constexpr int kPrepThreads = 1024;

struct PrepParams {
  int T, B;
  int64_t cache_rows;
  const int32_t* positions;
  const int32_t* q_seq_offsets;
  const int64_t* cache_offsets;
  int split;
  TopkWorkspace ws;
};

__device__ int block_exclusive_scan(int* a, int n, int* warp_sums) {
  // in-place exclusive scan of a[0..n) by kPrepThreads threads; returns the total
  __shared__ int carry;
  if (threadIdx.x == 0) carry = 0;
  __syncthreads();
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  for (int base = 0; base < n; base += kPrepThreads) {
    const int i = base + threadIdx.x;
    const int v = (i < n) ? a[i] : 0;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) warp_sums[wid] = x;
    __syncthreads();
    if (wid == 0) {
      int s = warp_sums[lane];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, s, o);
        if (lane >= o) s += y;
      }
      warp_sums[lane] = s;  // inclusive
    }
    __syncthreads();
    const int before = carry + (wid > 0 ? warp_sums[wid - 1] : 0) + x - v;
    if (i < n) a[i] = before;
    __syncthreads();
    if (threadIdx.x == 0) carry += warp_sums[31];
    __syncthreads();
  }
  return carry;
}

__device__ __forceinline__ int owner_of(const int* base, int n_owners, int i) {
  // the last o with base[o] <= i
  int lo = 0, hi = n_owners - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (base[mid] <= i) lo = mid;
    else hi = mid - 1;
  }
  return lo;
}

__device__ __forceinline__ int chunk_len_for(int n) {
  // shortest multiple of 128 that is >= kMinChunk and covers n in kMaxChunks chunks
  int c = (n + kMaxChunks - 1) / kMaxChunks;
  c = (c + kKeyTile - 1) / kKeyTile * kKeyTile;
  return c < kMinChunk ? kMinChunk : c;
}

__global__ void __launch_bounds__(kPrepThreads) prep_kernel(PrepParams p) {
  __shared__ int warp_sums[32];
  __shared__ int bad;
  const TopkWorkspace& ws = p.ws;
  if (threadIdx.x == 0) bad = 0;
  __syncthreads();
  // 1. offsets
  for (int b = threadIdx.x; b <= p.B; b += kPrepThreads) {
    const int qo = p.q_seq_offsets[b];
    const int64_t co = p.cache_offsets[b];
    bool ok = qo >= 0 && qo <= p.T && co >= 0 && co <= p.cache_rows;
    if (b == 0) ok = ok && qo == 0;
    if (b == p.B) ok = ok && qo == p.T;
    if (b > 0) ok = ok && p.q_seq_offsets[b - 1] <= qo && p.cache_offsets[b - 1] <= co;
    if (!ok) bad = 1;
  }
  __syncthreads();
  if (bad) {
    if (threadIdx.x == 0) {
      atomicOr(ws.err, kErrBounds | kErrOffsets);
      *ws.n_items = 0;
      *ws.work_counter = 0;
    }
    for (int t = threadIdx.x; t < p.T; t += kPrepThreads) ws.tok_nchunks[t] = 0;
    return;
  }
  // 2. validated positions
  for (int t = threadIdx.x; t < p.T; t += kPrepThreads) {
    int lo = 0, hi = p.B - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (p.q_seq_offsets[mid] <= t) lo = mid;
      else hi = mid - 1;
    }
    const int64_t len = p.cache_offsets[lo + 1] - p.cache_offsets[lo];
    const int pos = p.positions[t];
    const bool ok = pos >= 0 && pos < len;
    if (!ok) atomicOr(ws.err, kErrBounds);
    ws.pos_eff[t] = ok ? pos : -1;
    ws.tok_nchunks[t] = 0;
  }
  __syncthreads();
  // 3. items per owner (sequence on the prefill path, query on the split path)
  const int n_owners = p.split ? p.T : p.B;
  for (int o = threadIdx.x; o < n_owners; o += kPrepThreads) {
    int c;
    if (p.split) {
      const int n = ws.pos_eff[o] + 1;
      const int cl = chunk_len_for(n);
      c = n > cl ? (n + cl - 1) / cl : 1;
      ws.tok_nchunks[o] = c;
    } else {
      const int nq = p.q_seq_offsets[o + 1] - p.q_seq_offsets[o];
      c = (nq + kPrefillQ - 1) / kPrefillQ;
    }
    ws.seq_base[o] = c;
  }
  __syncthreads();
  const int total = block_exclusive_scan(ws.seq_base, n_owners, warp_sums);
  if (threadIdx.x == 0) {
    ws.seq_base[n_owners] = total;
    *ws.n_items = total;
    *ws.work_counter = 0;
  }
  __syncthreads();
  // 4. items, written in reverse order of (owner, tile) so the longest prefixes come first
  for (int i = threadIdx.x; i < total; i += kPrepThreads) {
    const int o = owner_of(ws.seq_base, n_owners, i);
    const int local = i - ws.seq_base[o];
    WorkItem wi;
    wi.pad0 = wi.pad1 = 0;
    if (p.split) {
      const int t = o;
      const int n = ws.pos_eff[t] + 1;
      const int nch = ws.tok_nchunks[t];
      const int cl = chunk_len_for(n);
      int lo = 0, hi = p.B - 1;
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (p.q_seq_offsets[mid] <= t) lo = mid;
        else hi = mid - 1;
      }
      wi.t0 = t;
      wi.nq = 1;
      wi.b = lo;
      wi.k_begin = (nch > 1) ? local * cl : 0;
      wi.k_end = (nch > 1) ? min(n, (local + 1) * cl) : n;
      wi.chunk = (nch > 1) ? local : -1;
    } else {
      const int b = o;
      const int t0 = p.q_seq_offsets[b] + local * kPrefillQ;
      const int nq = min(kPrefillQ, p.q_seq_offsets[b + 1] - t0);
      int kend = 0;
      for (int j = 0; j < nq; ++j) kend = max(kend, ws.pos_eff[t0 + j] + 1);
      wi.t0 = t0;
      wi.nq = nq;
      wi.b = b;
      wi.k_begin = 0;
      wi.k_end = kend;
      wi.chunk = -1;
    }
    ws.items[total - 1 - i] = wi;
  }
}

// ------------------------------------------------------------------------------------------
__global__ void wait_timeout_selftest_kernel(int* status, uint64_t timeout_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  __shared__ int err;
  if (threadIdx.x != 0) return;
  mbar_init(&bar, 1);
  abort_flag = 0;
  err = 0;
  fence_mbar_init();
  const WaitCtl wc{&err, &abort_flag, timeout_ns};
  const bool ok = mbar_wait(&bar, 0, wc);   // nothing ever arrives on `bar`
  *status = ok ? 0 : ((err & kErrTimeout) ? 2 : 1);
}

template <int QMAX, int STAGES, int ACC_BUFS, int NWG>
cudaError_t launch_score(const CUtensorMap& tmQ, const CUtensorMap& tmK, const ScoreParams& p, int grid,
                         cudaStream_t s) {
  using C = ScoreCfg<QMAX, STAGES, ACC_BUFS, NWG>;
  auto kern = score_topk_kernel<QMAX, STAGES, ACC_BUFS, NWG>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
  if (e != cudaSuccess) return e;
  kern<<<grid, C::kThreads, C::kSmemBytes, s>>>(tmQ, tmK, p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_topk(const TopkArgs& a, const TopkWorkspace& ws, const CUtensorMap& tmQ1, const CUtensorMap& tmQ8,
                        const CUtensorMap& tmK, int num_sms, cudaStream_t s) {
  PrepParams pp;
  pp.T = a.T;
  pp.B = a.B;
  pp.cache_rows = a.cache_rows;
  pp.positions = a.positions;
  pp.q_seq_offsets = a.q_seq_offsets;
  pp.cache_offsets = a.cache_offsets;
  pp.split = a.split ? 1 : 0;
  pp.ws = ws;
  prep_kernel<<<1, kPrepThreads, 0, s>>>(pp);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;

  ScoreParams sp;
  sp.items = ws.items;
  sp.n_items = ws.n_items;
  sp.work_counter = ws.work_counter;
  sp.w = a.w;
  sp.pos_eff = ws.pos_eff;
  sp.cache_offsets = a.cache_offsets;
  sp.idx_out = a.idx_out;
  sp.score_out = a.score_out;
  sp.cand_keys = ws.cand_keys;
  sp.cand_idx = ws.cand_idx;
  sp.part_keys = ws.part_keys;
  sp.part_idx = ws.part_idx;
  sp.err = ws.err;
  sp.timeout_ns = a.timeout_ns;
  const int grid = num_sms < ws.cand_slots ? num_sms : ws.cand_slots;
  if (a.split) {
    e = launch_score<1, 5, 4, 1>(tmQ1, tmK, sp, grid, s);
    if (e != cudaSuccess) return e;
    const int msmem = kMaxChunks * kTopK * 4;
    e = cudaFuncSetAttribute(merge_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, msmem);
    if (e != cudaSuccess) return e;
    merge_kernel<<<a.T, kMergeThreads, msmem, s>>>(ws.part_keys, ws.part_idx, ws.tok_nchunks, a.idx_out,
                                                    a.score_out);
    return cudaGetLastError();
  }
  return launch_score<kPrefillQ, 3, 2, 2>(tmQ8, tmK, sp, grid, s);
}

cudaError_t launch_wait_timeout_selftest(int* status, uint64_t timeout_ns, cudaStream_t s) {
  wait_timeout_selftest_kernel<<<1, 32, 0, s>>>(status, timeout_ns);
  return cudaGetLastError();
}

}  // namespace dsa
