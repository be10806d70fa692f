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
//   epilogue   warpgroups of 4 warps (the 4 TMEM lane quadrants); a warp covers its
//              quadrant's 32 keys for one or two queries.  It reads its columns with
//              tcgen05.ld 16x256b, in which each thread holds a fixed set of 8 heads, so
//              the fp32 head weights stay in registers; ReLU and the weights give partial
//              sums that two shuffle steps across 4 threads turn into one score per thread
//              and query.  A key is masked if s > pos, and (key, s) is admitted when the
//              key reaches the query's admission threshold: the pair goes to the warp's own
//              append area (warp ballot, warp-uniform counts in registers, no atomics) and
//              the key is counted in the query's first-level histogram in shared memory.
//              Every 16 tiles (24 in items of more than 512 tiles) the threshold rises to
//              the lowest bin that still holds the query's best 2,048 counted keys (a warp
//              scan of the histogram);
//              in long items a nearly full append area is compacted to the exact best
//              2,048.  At the end of the item each query's candidates are reduced to
//              exactly the top 2,048 in one pass (resolve_topk) and written out.

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
  uint2* cand;                  // [slots][QMAX][kCandStride] (key, position) pairs
  uint32_t* part_keys;          // [T][kMaxChunks][kTopK]
  int32_t* part_idx;
  uint32_t* part_hist;          // [T][kBins1]: first-level bin counts of each query's partial lists
  const float* q_scale;         // FP8: [T, 32] scale of each query head (folded into its weight)
  const float* key_scale;       // FP8: [cache_rows] scale of each key row (multiplies the score)
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
// Group-wide helpers for a group of NT threads (tid = 0..NT-1) that synchronise on the
// named barrier `bar`.

// Sum of v over the threads of the group with a larger tid.
template <int NT>
__device__ __forceinline__ uint32_t group_suffix_excl(uint32_t v, int tid, uint32_t* scratch, int bar) {
  const int lane = tid & 31, wid = tid >> 5;
  uint32_t x = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const uint32_t y = __shfl_down_sync(0xffffffffu, x, off);
    if (lane + off < 32) x += y;
  }
  if (lane == 0) scratch[wid] = x;  // warp total
  named_bar_sync(bar, NT);
  uint32_t wa = 0;
#pragma unroll
  for (int w = 0; w < NT / 32; ++w)
    if (w > wid) wa += scratch[w];
  named_bar_sync(bar, NT);
  return wa + x - v;
}

constexpr int kHistBins = 1024;   // histogram bins of one selection round

// k-th largest of the order-preserving keys that a group of NT threads visits, among those
// inside the window [lo, hi] (1 <= k <= their number; keys outside are ignored).
// keys(f) calls f(key) for every key the calling thread owns; each key has one owner, and
// keys may be called once per round.  Each round histograms the window into at most
// kHistBins bins of width 2^shift, locates the bin that holds the k-th largest and narrows
// the window to it; a round of width-1 bins ends it (at most three rounds for 32-bit keys).
// *n_above receives the number of keys in the window strictly greater than the result.
template <int NT, class Keys>
__device__ uint32_t kth_window(const Keys& keys, int k, uint32_t lo, uint32_t hi, uint32_t* hist,
                               uint32_t* scratch, int* sh, int tid, int bar, int* n_above) {
  constexpr int kBPT = kHistBins / NT;  // bins owned by one thread when locating the k-th
  uint32_t base = lo, span = hi - lo;
  int need = k, above_total = 0;
#pragma unroll 1
  while (true) {
    const int shift = (span >> 10) ? 32 - __clz(static_cast<int>(span >> 10)) : 0;
    for (int i = tid; i < kHistBins; i += NT) hist[i] = 0;
    named_bar_sync(bar, NT);
    keys([&](uint32_t key) {
      const uint32_t d = key - base;
      if (d <= span) atomicAdd(&hist[d >> shift], 1u);
    });
    named_bar_sync(bar, NT);
    const int b0 = tid * kBPT;
    uint32_t c[kBPT];
    uint32_t s = 0;
#pragma unroll
    for (int i = 0; i < kBPT; ++i) {
      c[i] = hist[b0 + i];
      s += c[i];
    }
    const uint32_t above_t = group_suffix_excl<NT>(s, tid, scratch, bar);
    if (above_t < static_cast<uint32_t>(need) && static_cast<uint32_t>(need) <= above_t + s) {
      uint32_t cum = above_t;
#pragma unroll
      for (int i = kBPT - 1; i >= 0; --i) {
        if (cum + c[i] >= static_cast<uint32_t>(need)) {
          sh[0] = b0 + i;
          sh[1] = static_cast<int>(cum);
          break;
        }
        cum += c[i];
      }
    }
    named_bar_sync(bar, NT);
    const int bstar = sh[0];
    const int above = sh[1];
    named_bar_sync(bar, NT);
    need -= above;
    above_total += above;
    if (shift == 0) {
      *n_above = above_total;
      return base + static_cast<uint32_t>(bstar);
    }
    base += static_cast<uint32_t>(bstar) << shift;
    span = (1u << shift) - 1u;
  }
}

// kth_window over n keys held in shared memory.
template <int NT>
__device__ uint32_t kth_largest(const uint32_t* keys, int n, int k, uint32_t lo, uint32_t hi, uint32_t* hist,
                                uint32_t* scratch, int* sh, int tid, int bar, int* n_above) {
  auto visit = [&](auto f) {
    for (int e = tid; e < n; e += NT) f(keys[e]);
  };
  return kth_window<NT>(visit, k, lo, hi, hist, scratch, sh, tid, bar, n_above);
}

// ------------------------------------------------------------------------------------------
__device__ __forceinline__ uint32_t u4_get(const uint4& v, int j) {
  return j == 0 ? v.x : j == 1 ? v.y : j == 2 ? v.z : v.w;
}
__device__ __forceinline__ int i4_get(const int4& v, int j) {
  return j == 0 ? v.x : j == 1 ? v.y : j == 2 ? v.z : v.w;
}

// ------------------------------------------------------------------------------------------
// Candidates of the score kernel.  A query's candidates are (ordered key, position) pairs:
// its current keep set and the append areas of the four epilogue warps that own its key
// rows.  Beside them, in shared memory, the query keeps the count of its candidates in
// each of kBins1 first-level bins (bin = the key's top 11 bits: sign, exponent and two
// mantissa bits of the score), two 16-bit counts per word.  The counts drive both the
// admission threshold while scores stream in and the exact selection at the end.
constexpr int kBinShift = 21;                  // first-level bin = key >> kBinShift
constexpr int kBins1 = 1 << (32 - kBinShift);  // 2,048 bins
constexpr int kSubShift = kBinShift - 11;      // second-level bin = next 11 bits
constexpr int kListCap = 1024;                 // boundary-bin candidates gathered in shared memory
constexpr int kCheckTiles = 16;                // key tiles between threshold updates (and capacity checks)
// items of more than kLongCheckItem tiles space their check points kLongCheckTiles apart: late in
// a long prefix the threshold moves slowly, and the check points (a scan of the counts, a group
// barrier, the capacity test) cost more than the extra admissions they save (measured on 96 K to
// 128 K-key items: 3-5 % faster; on 32 K to 64 K-key items 1-2 % slower, so those keep 16)
constexpr int kLongCheckItem = 512;
constexpr int kLongCheckTiles = 24;
constexpr int kSmallRank = 32;                 // boundary sub-bins up to this size are ranked by one warp

// An admission threshold held as a float, raised to the order-preserving key t if that is
// higher.  Keys at or below that of -inf admit every finite score (-inf).
__device__ __forceinline__ float raise_threshold(float thr, uint32_t t) {
  const uint32_t u = max(float_to_ordered(thr), t);
  return u <= float_to_ordered(-INFINITY) ? -INFINITY : ordered_to_float(u);
}

// h is shared memory: a fire-and-forget shared-memory reduction (the barrier that precedes
// every read of the counts orders it)
__device__ __forceinline__ void count_key(uint32_t* h, uint32_t bin) {
  asm volatile("red.shared.add.u32 [%0], %1;" ::"r"(smem_u32(&h[bin >> 1])), "r"((bin & 1u) ? 0x10000u : 1u)
               : "memory");
}

constexpr int kRoundU = 4;   // 16-byte loads (two candidates each) per thread and round

// Entry e (0..2 U - 1) of a round: entries 2i and 2i+1 sit in x[i].
template <int U>
__device__ __forceinline__ uint2 round_entry(const uint4 (&x)[U], int e) {
  return (e & 1) ? make_uint2(x[e >> 1].z, x[e >> 1].w) : make_uint2(x[e >> 1].x, x[e >> 1].y);
}

struct CandView {
  const uint2* keep;   // the current keep set
  const uint2* area;   // warp w's append area starts at area + w * kWarpApp
  int nk, n0, n1, n2, n3;
  __device__ __forceinline__ int total() const { return nk + n0 + n1 + n2 + n3; }

  // Calls f(x, lim) once per round.  A round gives each thread up to 2 kRoundU candidates,
  // all requested before any is used, read in pairs with 16-byte loads: x[i] holds entries
  // 2i and 2i+1, lim[i] how many of the two are valid.  Every thread of the group makes
  // the same calls, so f may use warp-collective operations.
  template <int NT, int U = kRoundU, class F>
  __device__ __forceinline__ void for_rounds(int tid, F&& f) const {
    const int u0 = (nk + 1) >> 1;
    const int u1 = u0 + ((n0 + 1) >> 1);
    const int u2 = u1 + ((n1 + 1) >> 1);
    const int u3 = u2 + ((n2 + 1) >> 1);
    const int u4 = u3 + ((n3 + 1) >> 1);
#pragma unroll 1
    for (int base = 0; base < u4; base += U * NT) {
      uint4 x[U];
      int lim[U];
#pragma unroll
      for (int i = 0; i < U; ++i) {
        const int u = base + i * NT + tid;
        const uint2* p;
        int off, cnt;
        if (u < u0) { p = keep; off = u; cnt = nk; }
        else if (u < u1) { p = area; off = u - u0; cnt = n0; }
        else if (u < u2) { p = area + kWarpApp; off = u - u1; cnt = n1; }
        else if (u < u3) { p = area + 2 * kWarpApp; off = u - u2; cnt = n2; }
        else { p = area + 3 * kWarpApp; off = u - u3; cnt = n3; }
        lim[i] = u < u4 ? min(2, cnt - 2 * off) : 0;
        x[i] = lim[i] > 0 ? *reinterpret_cast<const uint4*>(p + 2 * off) : make_uint4(0u, 0u, 0u, 0u);
      }
      f(x, lim);
    }
  }
};

// Calls f(rank, entry) for every candidate, ranks 0..total-1 (order unspecified);
// *ctr is a shared counter zeroed beforehand.
template <int NT, class F>
__device__ __forceinline__ void collect(const CandView& v, int* ctr, int tid, F&& f) {
  const int lane = tid & 31;
  const uint32_t lt = lanemask_lt();
  v.for_rounds<NT>(tid, [&](const uint4 (&x)[kRoundU], const int (&lim)[kRoundU]) {
    int c = 0;
#pragma unroll
    for (int i = 0; i < kRoundU; ++i) c += lim[i] > 0 ? lim[i] : 0;
    int sc = c;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, sc, off);
      if (lane >= off) sc += y;
    }
    const int tot = __shfl_sync(0xffffffffu, sc, 31);
    if (tot) {
      int o = 0;
      if (lane == 0) o = atomicAdd(ctr, tot);
      o = __shfl_sync(0xffffffffu, o, 0) + sc - c;
#pragma unroll
      for (int e = 0; e < 2 * kRoundU; ++e)
        if (lim[e >> 1] > (e & 1)) f(o++, round_entry(x, e));
    }
  });
}

// Bin b of kBins1 bins, counted two per word in hw, that holds the need-th largest counted
// key: count(bins > b) < need <= count(bins >= b) (need <= the total count).  Returns b and
// sets *above = count(bins > b); sh[0..1] carry the result.  With `clear` each thread
// zeroes the words it read.
template <int NT>
__device__ int locate_packed(uint32_t* hw, uint32_t need, bool clear, uint32_t* scratch, int* sh, int tid, int bar,
                             uint32_t* above) {
  constexpr int kWPT = (kBins1 / 2) / NT;  // words per thread
  const int w0 = tid * kWPT;
  uint32_t c[2 * kWPT];
  uint32_t s = 0;
#pragma unroll
  for (int i = 0; i < kWPT; ++i) {
    const uint32_t word = hw[w0 + i];
    c[2 * i] = word & 0xFFFFu;
    c[2 * i + 1] = word >> 16;
    s += c[2 * i] + c[2 * i + 1];
  }
  if (clear) {
#pragma unroll
    for (int i = 0; i < kWPT; ++i) hw[w0 + i] = 0u;
  }
  if (tid == 0) {   // defaults in case no bin qualifies (the barrier below orders them first)
    sh[0] = 0;
    sh[1] = 0;
  }
  const uint32_t above_t = group_suffix_excl<NT>(s, tid, scratch, bar);
  if (above_t < need && need <= above_t + s) {
    uint32_t cum = above_t;
#pragma unroll
    for (int i = 2 * kWPT - 1; i >= 0; --i) {
      if (cum + c[i] >= need) {
        sh[0] = 2 * w0 + i;
        sh[1] = static_cast<int>(cum);
        break;
      }
      cum += c[i];
    }
  }
  named_bar_sync(bar, NT);
  const int b = min(max(sh[0], 0), kBins1 - 1);
  *above = static_cast<uint32_t>(max(sh[1], 0));
  return b;
}

// One warp: the highest bin b with count(bins >= b) >= need in a packed kBins1-bin
// histogram, or 0 if the histogram holds fewer than need keys.  Lane l first sums bins
// 64l..64l+63 (the total of all counts stays below 2^16, so the two halves of a word sum
// can be added without carries), then the lanes scan the 64 bins of the crossing.  Counts
// may be growing meanwhile: the result is then a lower bound of the exact one.
__device__ __forceinline__ int scan_bins_warp(const uint32_t* hw, uint32_t need, int lane) {
  const uint4* q = reinterpret_cast<const uint4*>(hw) + lane * 8;
  uint32_t s = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint4 x = q[(i + lane) & 7];   // rotated: the lanes of one load cover every bank
    s += x.x + x.y + x.z + x.w;
  }
  const uint32_t cnt = (s & 0xFFFFu) + (s >> 16);
  uint32_t x = cnt;   // inclusive suffix over lanes >= lane
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const uint32_t y = __shfl_down_sync(0xffffffffu, x, off);
    if (lane + off < 32) x += y;
  }
  const uint32_t m = __ballot_sync(0xffffffffu, x >= need);
  if (!m) return 0;
  const int ls = 31 - __clz(m);
  const uint32_t run = __shfl_sync(0xffffffffu, x - cnt, ls);   // count above lane ls's bins
  const uint32_t word = hw[ls * 32 + lane];
  const uint32_t lo = word & 0xFFFFu;
  uint32_t z = lo + (word >> 16);
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const uint32_t y = __shfl_down_sync(0xffffffffu, z, off);
    if (lane + off < 32) z += y;
  }
  const uint32_t cum_even = run + z;        // count(bins >= 64 ls + 2 lane)
  const uint32_t cum_odd = cum_even - lo;   // count(bins >= 64 ls + 2 lane + 1)
  const uint32_t m2 = __ballot_sync(0xffffffffu, cum_even >= need);
  const int l = 31 - __clz(m2);             // m2 holds lane 0 at least
  const uint32_t co = __shfl_sync(0xffffffffu, cum_odd, l);
  return 64 * ls + 2 * l + (co >= need ? 1 : 0);
}

struct ResolveSmem {
  uint32_t* rh;      // kBins1 / 2 words: second-level counts, then kth_window's bins
  uint2* list;       // list_cap boundary-bin candidates
  int list_cap;
  uint32_t* small;   // kSmallRank keys of the boundary sub-bin
  uint32_t* scratch;
  int* sh;
  int* ctr;          // four shared counters
};

// Exact top kTopK of a query's candidates (at least kTopK of them), given h1, the packed
// first-level counts of exactly those candidates:
// 1. locate the bin b1 that holds the kTopK-th largest key; `above` keys lie above it;
// 2. one pass over the candidates: keys above b1 go to slots [0, above); keys in b1 are
//    gathered into the list and counted by their next 11 bits;
// 3. locate the boundary's second-level bin b2 and find the exact kTopK-th largest key K*
//    inside it: one warp ranks a small sub-bin, else a histogram round runs over the list
//    (or over the candidates again when the list overflowed);
// 4. emit the keys of b1 greater than K* and the first kTopK - n_above keys equal to K*.
// sink(slot, key, pos) is called once for each slot 0..kTopK-1.  With clear_h1 the words
// of h1 are zeroed before the first sink call.  Returns K*.
// With rs.rh == h1 the first-level counts are consumed (and cleared) by step 1 and their
// words then hold the second-level counts (clear_h1 must be set).
template <int NT, class Sink>
__device__ uint32_t resolve_topk(const CandView& v, uint32_t* h1, bool clear_h1, const ResolveSmem& rs, int tid,
                                 int bar, Sink&& sink) {
  const int lane = tid & 31;
  const uint32_t lt = lanemask_lt();
  if (rs.rh != h1)
    for (int i = tid; i < kBins1 / 2; i += NT) rs.rh[i] = 0u;
  if (tid == 0) {
    rs.ctr[0] = 0;
    rs.ctr[1] = 0;
    rs.ctr[2] = 0;
    rs.ctr[3] = 0;
  }
  // 1. (its barriers also publish the zeroed scratch)
  uint32_t above;
  const int b1 = locate_packed<NT>(h1, kTopK, clear_h1, rs.scratch, rs.sh, tid, bar, &above);
  const uint32_t ub1 = static_cast<uint32_t>(b1);
  // 2.
  constexpr int kPassU = kRoundU;
  v.for_rounds<NT, kPassU>(tid, [&](const uint4 (&x)[kPassU], const int (&lim)[kPassU]) {
    // above-b1 entries: one ballot per entry position and one shared counter update per warp
    // and round, so that each store instruction writes warp-contiguous slots; the few entries
    // of the boundary bin take a slot each from their own counter
    uint32_t bu[2 * kPassU];
    int tu = 0, ca = 0;
#pragma unroll
    for (int e = 0; e < 2 * kPassU; ++e) {
      const uint32_t b = round_entry(x, e).x >> kBinShift;
      const bool ok = lim[e >> 1] > (e & 1);
      bu[e] = __ballot_sync(0xffffffffu, ok && b > ub1);
      tu += __popc(bu[e]);
      ca += (ok && b == ub1) ? 1 : 0;
    }
    int ou = 0;
    if (tu) {
      if (lane == 0) ou = atomicAdd(&rs.ctr[0], tu);
      ou = __shfl_sync(0xffffffffu, ou, 0);
    }
    int oa = ca ? atomicAdd(&rs.ctr[1], ca) : 0;
#pragma unroll
    for (int e = 0; e < 2 * kPassU; ++e) {
      const uint2 c = round_entry(x, e);
      if ((bu[e] >> lane) & 1u) {
        const int o = ou + __popc(bu[e] & lt);
        if (o < kTopK) sink(o, c.x, c.y);
      }
      ou += __popc(bu[e]);
      if (lim[e >> 1] > (e & 1) && (c.x >> kBinShift) == ub1) {
        if (oa < rs.list_cap) rs.list[oa] = c;
        count_key(rs.rh, (c.x >> kSubShift) & (kBins1 - 1));
        ++oa;
      }
    }
  });
  named_bar_sync(bar, NT);
  const int m = rs.ctr[1];
  // 3.
  const uint32_t need2 = kTopK - above;
  uint32_t above2;
  const int b2 = locate_packed<NT>(rs.rh, need2, false, rs.scratch, rs.sh + 2, tid, bar, &above2);
  const uint32_t lo = (ub1 << kBinShift) | (static_cast<uint32_t>(b2) << kSubShift);
  const uint32_t hi = lo + ((1u << kSubShift) - 1u);
  const int need3 = static_cast<int>(need2 - above2);
  const int m2 = static_cast<int>((rs.rh[b2 >> 1] >> ((b2 & 1) * 16)) & 0xFFFFu);
  const bool in_list = m <= rs.list_cap;
  int n3;
  uint32_t kth;
  if (in_list && m2 <= kSmallRank) {
    // gather the sub-bin's keys; one warp ranks them
    if (tid == 0) {   // defaults in case no key qualifies (ordered first by the barrier below)
      rs.sh[4] = static_cast<int>(lo);
      rs.sh[5] = 0;
    }
    for (int e = tid; e < m; e += NT) {
      const uint32_t key = rs.list[e].x;
      if (key - lo <= hi - lo) {
        const int o = atomicAdd(&rs.ctr[3], 1);
        if (o < kSmallRank) rs.small[o] = key;
      }
    }
    named_bar_sync(bar, NT);
    if (tid < 32) {
      const uint32_t mine = lane < m2 ? rs.small[lane] : 0u;
      int gt = 0, eq = 0;
      for (int j = 0; j < m2; ++j) {
        const uint32_t y = __shfl_sync(0xffffffffu, mine, j);
        gt += y > mine;
        eq += y == mine;
      }
      if (lane < m2 && gt < need3 && need3 <= gt + eq) {   // every finder writes the same values
        rs.sh[4] = static_cast<int>(mine);
        rs.sh[5] = gt;
      }
    }
    named_bar_sync(bar, NT);
    kth = static_cast<uint32_t>(rs.sh[4]);
    n3 = min(max(rs.sh[5], 0), kTopK);
  } else if (in_list) {
    auto keys = [&](auto f) {
      for (int e = tid; e < m; e += NT) f(rs.list[e].x);
    };
    kth = kth_window<NT>(keys, need3, lo, hi, rs.rh, rs.scratch, rs.sh, tid, bar, &n3);
  } else {
    auto keys = [&](auto f) {
      v.for_rounds<NT>(tid, [&](const uint4 (&x)[kRoundU], const int (&lim)[kRoundU]) {
#pragma unroll
        for (int e = 0; e < 2 * kRoundU; ++e)
          if (lim[e >> 1] > (e & 1)) f(round_entry(x, e).x);
      });
    };
    kth = kth_window<NT>(keys, need3, lo, hi, rs.rh, rs.scratch, rs.sh, tid, bar, &n3);
  }
  const int n_above = min(static_cast<int>(min(above + above2, static_cast<uint32_t>(kTopK))) + n3, kTopK);
  const int ties = kTopK - n_above;
  // 4. slots below n_above continue rs.ctr[0] (== above after step 2); ties count in ctr[2]
  auto fin = [&](uint2 c, bool ok) {
    const bool in = ok && (c.x >> kBinShift) == ub1;
    const bool gt = in && c.x > kth, eq = in && c.x == kth;
    const uint32_t bg = __ballot_sync(0xffffffffu, gt), be = __ballot_sync(0xffffffffu, eq);
    if (bg | be) {
      int og = 0, oe = 0;
      if (lane == 0) {
        if (bg) og = atomicAdd(&rs.ctr[0], __popc(bg));
        if (be) oe = atomicAdd(&rs.ctr[2], __popc(be));
      }
      og = __shfl_sync(0xffffffffu, og, 0) + __popc(bg & lt);
      oe = __shfl_sync(0xffffffffu, oe, 0) + __popc(be & lt);
      if (gt && og < kTopK) sink(og, c.x, c.y);
      if (eq && oe < ties && n_above + oe >= 0) sink(n_above + oe, c.x, c.y);
    }
  };
  if (in_list) {
    for (int base = 0; base < m; base += NT) {
      const int e = base + tid;
      const bool ok = e < m;
      fin(ok ? rs.list[e] : make_uint2(0u, 0u), ok);
    }
  } else {
    v.for_rounds<NT>(tid, [&](const uint4 (&x)[kRoundU], const int (&lim)[kRoundU]) {
#pragma unroll
      for (int e = 0; e < 2 * kRoundU; ++e) fin(round_entry(x, e), lim[e >> 1] > (e & 1));
    });
  }
  return kth;
}

// ------------------------------------------------------------------------------------------
// DSA_TOPK_SORTED: orders one row of kTopK selected (ordered score key, position) pairs by
// score descending, then position ascending, and writes it out.  A group of NT threads
// (tid = 0..NT-1, named barrier `bar`) runs a bitonic sorting network over 64-bit words
// (key << 32 | ~position), descending; thread tid holds elements tid*E .. tid*E + E - 1.
// Compare-exchange steps between elements of one thread run in registers, between threads
// of one warp through shuffles, and between warps through `stage` (kTopK pairs, global or
// shared memory), which also holds the input.
__device__ __forceinline__ uint64_t sort_word(uint2 c) {
  return (static_cast<uint64_t>(c.x) << 32) | static_cast<uint64_t>(0xFFFFFFFFu - c.y);
}

// One compare-exchange step (distance J inside bitonic blocks of K elements).
template <int NT, int K, int J>
__device__ __forceinline__ void bitonic_step(uint64_t (&v)[kTopK / NT], int tid, uint64_t* s64, int bar) {
  constexpr int E = kTopK / NT;
  if constexpr (J < E) {
#pragma unroll
    for (int r = 0; r < E; ++r) {
      const int l = r ^ J;
      if (l > r) {
        const bool desc = ((tid * E + r) & K) == 0;   // the lower index keeps the larger word
        const uint64_t a = v[r], b = v[l];
        if (desc ? (a < b) : (a > b)) {
          v[r] = b;
          v[l] = a;
        }
      }
    }
  } else {
    if constexpr (J >= 32 * E) {
#pragma unroll
      for (int r = 0; r < E; ++r) s64[tid * E + r] = v[r];
      named_bar_sync(bar, NT);
    }
#pragma unroll
    for (int r = 0; r < E; ++r) {
      const int i = tid * E + r;
      uint64_t o;
      if constexpr (J < 32 * E) {
        const uint32_t hi = __shfl_xor_sync(0xffffffffu, static_cast<uint32_t>(v[r] >> 32), J / E);
        const uint32_t lo = __shfl_xor_sync(0xffffffffu, static_cast<uint32_t>(v[r]), J / E);
        o = (static_cast<uint64_t>(hi) << 32) | lo;
      } else {
        o = s64[i ^ J];
      }
      const bool desc = (i & K) == 0;
      const bool keep_max = ((i & J) == 0) == desc;   // lower index of a descending pair
      v[r] = keep_max ? (v[r] > o ? v[r] : o) : (v[r] < o ? v[r] : o);
    }
    if constexpr (J >= 32 * E) named_bar_sync(bar, NT);
  }
}

template <int NT, int K, int J>
__device__ __forceinline__ void bitonic_merge(uint64_t (&v)[kTopK / NT], int tid, uint64_t* s64, int bar) {
  bitonic_step<NT, K, J>(v, tid, s64, bar);
  if constexpr (J > 1) bitonic_merge<NT, K, J / 2>(v, tid, s64, bar);
}

template <int NT, int K>
__device__ __forceinline__ void bitonic_sort(uint64_t (&v)[kTopK / NT], int tid, uint64_t* s64, int bar) {
  bitonic_merge<NT, K, K / 2>(v, tid, s64, bar);
  if constexpr (K < kTopK) bitonic_sort<NT, 2 * K>(v, tid, s64, bar);
}

// not inlined: its 2,048 / NT 64-bit words per thread stay out of its callers' register allocation
template <int NT>
__device__ __noinline__ void sort_stage_and_emit(uint2* stage, int tid, int bar, int32_t* oi, float* os) {
  constexpr int E = kTopK / NT;
  static_assert(E >= 1 && (E & (E - 1)) == 0 && E * NT == kTopK, "power-of-two elements per thread");
  uint64_t* const s64 = reinterpret_cast<uint64_t*>(stage);
  uint64_t v[E];
#pragma unroll
  for (int r = 0; r < E; ++r) v[r] = sort_word(stage[tid * E + r]);
  named_bar_sync(bar, NT);   // every entry is in registers before the stage is rewritten
  bitonic_sort<NT, 2>(v, tid, s64, bar);
#pragma unroll
  for (int r = 0; r < E; ++r) {
    const int i = tid * E + r;
    __stcs(oi + i, static_cast<int>(0xFFFFFFFFu - static_cast<uint32_t>(v[r])));
    if (os) __stcs(os + i, ordered_to_float(static_cast<uint32_t>(v[r] >> 32)));
  }
}

// ------------------------------------------------------------------------------------------
template <int QPW, int H>
struct WGState {
  uint32_t hist[QPW][kBins1 / 2];  // per query: first-level counts of its candidates (packed)
  uint32_t rhist[kBins1 / 2];      // resolution scratch
  uint2 list[kListCap];            // boundary-bin candidates of one resolution
  uint32_t small[2 * kSmallRank];  // keys of the boundary sub-bin (per sub-group)
  float w[QPW][H];
  int cnt_w[QPW][4];               // per-warp append counts, published at check points
  int cnt_k[QPW];                  // entries in the current keep set
  int kcur[QPW];                   // which keep set is current
  uint32_t thr[QPW];               // exact admission threshold left by a compaction
  uint32_t thr_bin[QPW];           // admission threshold found by the query's scanning warp
  int pos[QPW];
  uint32_t scratch[64];
  int sh[16];                      // 8 per sub-group
  int ctr[8];                      // 4 per sub-group
};

// Thread layout of the score kernel.  EW = epilogue warps per group: 4 (one warp per
// TMEM lane quadrant, each warp handles every query of the group) or 8 (two warps per
// quadrant, each handles half of the group's queries).  With EW = 8 the two control
// warps sit in a warpgroup of their own (warps 0-3) so that registers can be moved
// from it to the epilogue warpgroups (setmaxnreg).  NWG groups either split each item's
// queries (ALT = false) or, with ALT, take whole items in turn (group g takes the items
// the CTA receives at positions g, g + 2, ...): one group's end-of-item selection then
// overlaps the other group's tiles.
template <int QMAX, int STAGES, int ACC_BUFS, int NWG, int EW, bool ALT, int EB = 2, int H = kHeads>
struct ScoreCfg {
  // H = indexer heads (32, or 64 for the DeepSeek-V3.2 form); a query's H columns of the
  // accumulator are H / 32 blocks of 32.
  static constexpr int kHB = H / 32;
  // EB = bytes per element of q and of the keys: 2 (bf16, kind::f16 MMA) or 1 (FP8 e4m3,
  // kind::f8f6f4 MMA).  A 128-dim row is EB 128-byte swizzle rows ("halves") wide.
  static constexpr int kHalves = EB;
  static constexpr int kQPW = ALT ? QMAX : QMAX / NWG;  // queries of one epilogue group
  static constexpr int kConsumers = ALT ? EW : NWG * EW; // warps that consume each tile
  static constexpr int kQPH = kQPW / (EW / 4);        // queries of one epilogue warp
  static constexpr int kEpiWarp0 = EW == 8 ? 4 : 2;   // first epilogue warp
  static constexpr int kGroupThreads = EW * 32;
  static constexpr int kThreads = kEpiWarp0 * 32 + NWG * kGroupThreads;
  static constexpr bool kRegSplit = EW == 8;
  static constexpr int kCtrlRegs = 32;                // per thread of warps 0-3 after the split
  static constexpr int kEpiRegs = 112;                // per epilogue thread after the split
  static constexpr int kAccCols = QMAX * H;
  static constexpr int kTotalBufs = ALT ? NWG * ACC_BUFS : ACC_BUFS;  // with ALT each group has its own
  static constexpr int kTmemNeed = kTotalBufs * kAccCols;
  static constexpr int kTmemCols = kTmemNeed <= 32 ? 32 : kTmemNeed <= 64 ? 64 : kTmemNeed <= 128 ? 128
                                   : kTmemNeed <= 256 ? 256 : 512;
  static constexpr int kQHalf = QMAX * H * 128;       // bytes of one 128-byte-wide half of the Q tile
  static constexpr int kKHalf = kKeyTile * 128;       // 16 KB
  static constexpr int kKStage = kHalves * kKHalf;
  static constexpr int kQBytes = kHalves * kQHalf;   // one item's Q tile
  static constexpr int kWGBytes = (static_cast<int>(sizeof(WGState<kQPW, H>)) + 15) / 16 * 16;
  // small Q tiles (the split path: one query per item) are double-buffered where shared memory
  // allows, so that the next item's tile loads while this item's last key tiles are scored
  static constexpr int kQBufs =
      (kQBytes <= 16384 &&
       2 * kQBytes + STAGES * kKStage + NWG * kWGBytes + 8 * (2 * STAGES + 2 * kTotalBufs + 9) + 1088 <= 232448)
          ? 2 : 1;
  static constexpr int kQOff = 0;
  static constexpr int kKOff = kQBufs * kQBytes;
  static constexpr int kWGOff = kKOff + STAGES * kKStage;
  static constexpr int kBarOff = kWGOff + NWG * kWGBytes;
  static constexpr int kNumBars = 2 * STAGES + 2 * kTotalBufs + 2 * kQBufs + 4 + 1;
  static constexpr int kMiscOff = kBarOff + 8 * kNumBars;
  static constexpr int kSmemBytes = kMiscOff + 64 + 1024;
  static_assert(kTmemNeed <= 512, "TMEM holds 512 columns");
  static_assert(kQHalf % 1024 == 0, "Q halves must stay 1024-byte aligned");
  static_assert(kSmemBytes <= 232448, "shared memory per CTA");
  static_assert(kQPH >= 1 && kQPH * (EW / 4) == kQPW, "queries split evenly over a quadrant's warps");
  static_assert(kCtrlRegs % 8 == 0 && kEpiRegs % 8 == 0, "setmaxnreg takes multiples of 8");
  static_assert(!ALT || NWG == 2, "alternating items need two epilogue groups");
  static_assert(H % 32 == 0 && QMAX * H <= 256, "an item's (query, head) columns fit one MMA");
};

// The four threads t, t^1, t^2, t^3 hold partial sums over disjoint head sets for the same
// 2 x 2 rows (lane half h = 0/1, row t/4 or t/4 + 8) of each of QPH queries.  Two butterfly
// steps, each sending half of the remaining values to the partner, leave every thread
// with the full sums of one row for each query: the row of lane half (t & 1), offset
// 8 ((t >> 1) & 1).
template <int QPH>
__device__ __forceinline__ void sum_over_quad(const float (&part)[4 * QPH], float (&s)[QPH], int lane) {
  const bool b0 = lane & 1, b1 = (lane >> 1) & 1;
  float q[2 * QPH];
#pragma unroll
  for (int i = 0; i < 2 * QPH; ++i) {
    const float send = b0 ? part[i] : part[2 * QPH + i];
    const float keep = b0 ? part[2 * QPH + i] : part[i];
    q[i] = keep + __shfl_xor_sync(0xffffffffu, send, 1);
  }
#pragma unroll
  for (int i = 0; i < QPH; ++i) {
    const float send = b1 ? q[i] : q[QPH + i];
    const float keep = b1 ? q[QPH + i] : q[i];
    s[i] = keep + __shfl_xor_sync(0xffffffffu, send, 2);
  }
}

template <int QMAX, int STAGES, int ACC_BUFS, int NWG, int EW, bool ALT, bool SORTED, int EB, int H>
__global__ void __launch_bounds__(ScoreCfg<QMAX, STAGES, ACC_BUFS, NWG, EW, ALT, EB, H>::kThreads, 1)
    score_topk_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                      ScoreParams p) {
  using C = ScoreCfg<QMAX, STAGES, ACC_BUFS, NWG, EW, ALT, EB, H>;
  constexpr int HB = C::kHB;
  constexpr bool kFp8 = EB == 1;
  constexpr int QPW = C::kQPW;
  constexpr int QPH = C::kQPH;
  constexpr int NTG = C::kGroupThreads;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem + C::kQOff;
  uint8_t* sK = smem + C::kKOff;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
  uint64_t* full = bars;
  uint64_t* empty = full + STAGES;
  uint64_t* acc_full = empty + STAGES;
  uint64_t* acc_empty = acc_full + C::kTotalBufs;
  uint64_t* q_full = acc_empty + C::kTotalBufs;   // [kQBufs]
  uint64_t* q_empty = q_full + C::kQBufs;         // [kQBufs]
  uint64_t* sched_full = q_empty + C::kQBufs;
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
    for (int a = 0; a < C::kTotalBufs; ++a) {
      mbar_init(&acc_full[a], 1);
      mbar_init(&acc_empty[a], C::kConsumers);
    }
    for (int b = 0; b < C::kQBufs; ++b) {
      mbar_init(&q_full[b], 1);
      mbar_init(&q_empty[b], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sched_full[i], 1);
      mbar_init(&sched_empty[i], 1 + C::kConsumers);
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
  // everything above overlaps the prep kernel; its work list is read only after it completed
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int n_items = *p.n_items;
  const WaitCtl wc{p.err, abort_flag, p.timeout_ns};

  if (warp < C::kEpiWarp0) {
    // ===================================================== control warps
    if constexpr (C::kRegSplit) {
      asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;\n" ::"n"(C::kCtrlRegs));
    }
  if (warp == 0) {
    // ===================================================== TMA producer
    if (lane == 0) {
      int kstage = 0, qloads = 0;
      const uint64_t pol_q = l2_policy_evict_first();   // each Q tile is read once
      // prefill: key tiles are read by every item of a sequence; split path (decode): each key
      // is read once, and should not push the partial lists out of L2
      const uint64_t pol_k = ALT ? l2_policy_evict_first() : l2_policy_evict_last();
      for (int local = 0;; ++local) {
        const int slot = local & 1;
        if (local >= 2 && !mbar_wait(&sched_empty[slot], ((local >> 1) - 1) & 1, wc)) break;
        int it = atomicAdd(p.work_counter, 1);
        if (it >= n_items) it = -1;
        sched_item[slot] = it;
        mbar_arrive(&sched_full[slot]);
        if (it < 0) {
          // no work left for this CTA: a programmatic dependent (the merge of the split-key
          // path) may be scheduled once every CTA got here; it still waits for this grid's end
          asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
          if constexpr (ALT) {
            // the other group waits on the next slot: end it as well
            const int l2 = local + 1, s2 = l2 & 1;
            if (l2 >= 2 && !mbar_wait(&sched_empty[s2], ((l2 >> 1) - 1) & 1, wc)) break;
            sched_item[s2] = -1;
            mbar_arrive(&sched_full[s2]);
          }
          break;
        }
        const WorkItem wi = p.items[it];
        const int kt0 = wi.k_begin / kKeyTile, kt1 = (wi.k_end + kKeyTile - 1) / kKeyTile;
        if (kt1 <= kt0) continue;
        const int qb = qloads % C::kQBufs;
        if (qloads >= C::kQBufs && !mbar_wait(&q_empty[qb], ((qloads / C::kQBufs) - 1) & 1, wc)) break;
        uint8_t* const dq = sQ + qb * C::kQBytes;
        mbar_arrive_expect_tx(&q_full[qb], C::kQBytes);
        tma_load_2d_hint(dq, &tmQ, &q_full[qb], 0, wi.t0 * H, pol_q);
        if constexpr (!kFp8) tma_load_2d_hint(dq + C::kQHalf, &tmQ, &q_full[qb], 64, wi.t0 * H, pol_q);
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
          tma_load_2d_hint(dst, &tmK, &full[s], 0, row0 + kt * kKeyTile, pol_k);
          if constexpr (!kFp8) tma_load_2d_hint(dst + C::kKHalf, &tmK, &full[s], 64, row0 + kt * kKeyTile, pol_k);
          if constexpr (kFp8) {
            // the tile's key scales, read by the epilogue threads once the tile is scored:
            // bring their lines into L2 now (every prefetched address is a scale of the item)
            const int nrows = min(kKeyTile, wi.k_end - kt * kKeyTile);
            const float* sp = p.key_scale + row0 + kt * kKeyTile;
            for (int i = 0; i < nrows; i += 32) asm volatile("prefetch.global.L2 [%0];" ::"l"(sp + i));
            asm volatile("prefetch.global.L2 [%0];" ::"l"(sp + nrows - 1));
          }
        }
        if (!ok) break;
      }
      if (*abort_flag) {
        for (int ks = (kstage > STAGES ? kstage - STAGES : 0); ks < kstage; ++ks)
          drain_wait(&full[ks % STAGES], (ks / STAGES) & 1);
        for (int ql = (qloads > C::kQBufs ? qloads - C::kQBufs : 0); ql < qloads; ++ql)
          drain_wait(&q_full[ql % C::kQBufs], (ql / C::kQBufs) & 1);
      }
    }
  } else if (warp == 1) {
    // ===================================================== MMA issuer
    if (lane == 0) {
      int kstage = 0, qloads = 0;
      int acc0 = 0, acc1 = 0;   // tiles given to group 0 / group 1 (one shared ring without ALT)
      for (int local = 0;; ++local) {
        const int slot = local & 1;
        if (!mbar_wait(&sched_full[slot], (local >> 1) & 1, wc)) break;
        const int it = sched_item[slot];
        mbar_arrive(&sched_empty[slot]);
        if (it < 0) break;
        const WorkItem wi = p.items[it];
        const int kt0 = wi.k_begin / kKeyTile, kt1 = (wi.k_end + kKeyTile - 1) / kKeyTile;
        if (kt1 <= kt0) continue;
        const int qb = qloads % C::kQBufs;
        if (!mbar_wait(&q_full[qb], (qloads / C::kQBufs) & 1, wc)) break;
        ++qloads;
        const uint32_t qa = smem_u32(sQ + qb * C::kQBytes);
        tc_fence_after();
        const uint32_t idesc = kFp8 ? umma_idesc_e4m3(kKeyTile, wi.nq * H) : umma_idesc_bf16(kKeyTile, wi.nq * H);
        const bool second = ALT && (local & 1);   // with ALT, the CTA's odd items go to group 1
        bool ok = true;
        for (int kt = kt0; kt < kt1; ++kt, ++kstage) {
          const int s = kstage % STAGES;
          const int acc_ctr = second ? acc1 : acc0;
          const int ab = (second ? ACC_BUFS : 0) + acc_ctr % ACC_BUFS;
          if (second) ++acc1;
          else ++acc0;
          if (!mbar_wait(&full[s], (kstage / STAGES) & 1, wc)) { ok = false; break; }
          if (acc_ctr >= ACC_BUFS && !mbar_wait(&acc_empty[ab], ((acc_ctr / ACC_BUFS) - 1) & 1, wc)) {
            ok = false;
            break;
          }
          tc_fence_after();
          if constexpr (kFp8)
            umma_tile_k128_e4m3(tmem + ab * C::kAccCols, smem_u32(sK + s * C::kKStage), qa, idesc, &empty[s],
                                &acc_full[ab]);
          else
            umma_tile_k128<C::kKHalf, C::kQHalf>(tmem + ab * C::kAccCols, smem_u32(sK + s * C::kKStage), qa, idesc,
                                                &empty[s], &acc_full[ab]);
        }
        umma_commit(&q_empty[qb]);
        if (!ok) break;
      }
      umma_commit(mma_done);
      drain_wait(mma_done, 0);
    }
  }
  } else {
    // ===================================================== epilogue groups
    if constexpr (C::kRegSplit) {
      asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;\n" ::"n"(C::kEpiRegs));
    }
    const int ew = warp - C::kEpiWarp0;
    const int g = ew / EW;                   // epilogue group = a set of QPW queries of the item
    const int hq = (ew % EW) / 4;            // which part of the group's queries this warp scores
    const int qd = warp & 3;                 // TMEM lane quadrant of this warp (also its append area)
    const int gtid = threadIdx.x - C::kEpiWarp0 * 32 - g * NTG;
    const int bar = 1 + g;
    // key row of this thread inside a tile (the row whose scores it holds after sum_over_quad)
    const int r = qd * 32 + (lane >> 2) + 8 * ((lane >> 1) & 1) + 16 * (lane & 1);
    const uint32_t lt = lanemask_lt();
    WGState<QPW, H>& st = *reinterpret_cast<WGState<QPW, H>*>(smem + C::kWGOff + g * C::kWGBytes);
    const uint32_t tlane = tmem + (static_cast<uint32_t>(qd * 32) << 16);
    const int j0 = hq * QPH;                 // first of this warp's queries inside the group
    // candidates of query jj of this group start at qcand + jj * kCandStride
    const int qbase = ALT ? 0 : g * QPW;    // first query of the item this group scores
    uint2* const qcand =
        p.cand + (static_cast<size_t>(blockIdx.x) * (ALT ? QMAX * NWG : QMAX) + g * QPW) * kCandStride;
    uint2* const my_area = qcand + static_cast<size_t>(j0) * kCandStride + 2 * kTopK + qd * kWarpApp;
    const ResolveSmem rs{st.rhist, st.list, kListCap, st.small, st.scratch, st.sh, st.ctr};
    // the prefill path's end-of-item selections run in sub-groups of NTS threads, one query
    // each at a time, so that the latency of one query's passes overlaps another's; each
    // sub-group has its own named barrier and its own share of the selection scratch, and
    // the query's own first-level counts serve as its second-level counts
    constexpr int kSub = (!ALT && QPW >= 2) ? 2 : 1;
    constexpr int NTS = NTG / kSub;
    const int sg = gtid / NTS, stid = gtid % NTS;
    const int sbar = kSub == 1 ? bar : 3 + kSub * g + sg;
    const ResolveSmem rsub{st.rhist, st.list + sg * (kListCap / kSub), kListCap / kSub, st.small + sg * kSmallRank,
                           st.scratch + sg * 32, st.sh + sg * 8, st.ctr + sg * 4};
    const uint64_t pol_cand = l2_policy_evict_last();   // candidates are read back at the item's end
    int acc_ctr = 0;

    // the candidates of query jj of this group, with the published counts
    auto cands = [&](int jj) {
      const uint2* q = qcand + static_cast<size_t>(jj) * kCandStride;
      CandView v;
      v.keep = q + st.kcur[jj] * kTopK;
      v.area = q + 2 * kTopK;
      v.nk = st.cnt_k[jj];
      v.n0 = st.cnt_w[jj][0];
      v.n1 = st.cnt_w[jj][1];
      v.n2 = st.cnt_w[jj][2];
      v.n3 = st.cnt_w[jj][3];
      return v;
    };

    // the histograms start empty (ordered before any count by the item barrier)
    for (int i = gtid; i < QPW * (kBins1 / 2); i += NTG) (&st.hist[0][0])[i] = 0u;

    for (int n = 0;; ++n) {
      const int local = ALT ? 2 * n + g : n;
      const int slot = local & 1;
      const bool got = __all_sync(0xffffffffu, mbar_wait(&sched_full[slot], (local >> 1) & 1, wc));
      const int it = got ? sched_item[slot] : -1;
      __syncwarp();
      if (lane == 0 && got) mbar_arrive(&sched_empty[slot]);
      WorkItem wi;
      if (it >= 0) wi = p.items[it];
      if (gtid < QPW && it >= 0) {
        const int j = qbase + gtid;
        st.cnt_k[gtid] = 0;
        st.kcur[gtid] = 0;
        st.thr[gtid] = 0u;
        st.thr_bin[gtid] = 0u;
        st.pos[gtid] = (j < wi.nq) ? p.pos_eff[wi.t0 + j] : -2;
#pragma unroll
        for (int w = 0; w < 4; ++w) st.cnt_w[gtid][w] = 0;
      }
      if (it >= 0) {
        for (int i = gtid; i < QPW * H; i += NTG) {
          const int jj = i / H, j = qbase + jj;
          const size_t wix = static_cast<size_t>(wi.t0 + j) * H + (i % H);
          // FP8: the query head's scale joins its weight (sum_h w_h s_h ReLU(q8_h . k8))
          st.w[jj][i % H] = (j < wi.nq) ? (kFp8 ? p.w[wix] * p.q_scale[wix] : p.w[wix]) : 0.f;
        }
      }
      if (named_bar_or(bar, NTG, it < 0)) break;   // every thread of the group leaves together

      const int nloc = min(QPW, wi.nq - qbase);    // queries of the group present in this item
      const int nmine = min(QPH, nloc - j0);        // ... and scored by this warp (may be <= 0)
      const int kt0 = wi.k_begin / kKeyTile, kt1 = (wi.k_end + kKeyTile - 1) / kKeyTile;
      const int64_t kbase = kFp8 ? p.cache_offsets[wi.b] : 0;   // first key-cache row of the sequence
      // an item of at most kWarpApp / 32 tiles cannot fill an append area: no capacity checks
      const bool long_item = (kt1 - kt0) * 32 > kWarpApp;
      int cnt_r[QPH], pos_r[QPH];
#pragma unroll
      for (int j = 0; j < QPH; ++j) {
        cnt_r[j] = 0;
        pos_r[j] = (j < nmine) ? min(st.pos[j0 + j], wi.k_end - 1) : -2;   // last key position scored
      }
      // this thread's head weights: heads 32 hb + 8 blk + 2 (lane % 4) + {0, 1} of each of its
      // queries (hb = head block)
      float2 w2[QPH * HB][4];
#pragma unroll
      for (int j = 0; j < QPH; ++j)
#pragma unroll
        for (int hb = 0; hb < HB; ++hb)
#pragma unroll
          for (int blk = 0; blk < 4; ++blk)
            w2[j * HB + hb][blk] = *reinterpret_cast<const float2*>(&st.w[j0 + j][32 * hb + 8 * blk + 2 * (lane & 3)]);
      bool failed = false;
      // per-tile state kept incrementally: the group's accumulator slot and its phase, the
      // TMEM column of this warp's first block in slot 0, this thread's key position, the
      // admission thresholds as floats, and the tiles left until the next check point
      int aslot = acc_ctr % ACC_BUFS;
      uint32_t phase = static_cast<uint32_t>(acc_ctr / ACC_BUFS) & 1u;
      const int slot0 = ALT ? g * ACC_BUFS : 0;
      const uint32_t tcol0 = tlane + slot0 * C::kAccCols + (qbase + j0) * H;
      const uint32_t afull0 = smem_u32(&acc_full[slot0]), aempty0 = smem_u32(&acc_empty[slot0]);
      int s_pos = kt0 * kKeyTile + r;
      const int check_tiles = (kt1 - kt0 > kLongCheckItem) ? kLongCheckTiles : kCheckTiles;
      const int check_margin = check_tiles * 32;   // appends one warp can make per query between checks
      int to_check = check_tiles;
      float thr_f[QPH];
#pragma unroll
      for (int j = 0; j < QPH; ++j) thr_f[j] = -INFINITY;
      acc_ctr += kt1 - kt0;
      // a warp that holds one 32-column block per tile (one query of 32 heads: the split path)
      // takes two tiles per iteration, so that the two tiles' loads and arithmetic overlap
      constexpr int CB = QPH * HB;
      constexpr int TPI = CB == 1 ? 2 : 1;
      for (int kt = kt0; kt < kt1; kt += TPI, s_pos += TPI * kKeyTile) {
        const int ntile = (TPI == 2 && kt + 1 < kt1) ? 2 : 1;
        // FP8: this thread's key scales, requested before the accumulator waits (the producer
        // brought their lines into L2 when it loaded the tiles); rows past the item's last
        // scored key read as 0
        float sk[TPI];
        uint32_t tcol[TPI], aoff[TPI];
        bool ok = true;
#pragma unroll
        for (int u = 0; u < TPI; ++u) {
          if (u < ntile) {
            const int sp = s_pos + u * kKeyTile;
            sk[u] = (kFp8 && sp < wi.k_end) ? __ldg(p.key_scale + kbase + sp) : 0.f;
            aoff[u] = static_cast<uint32_t>(aslot) * 8u;
            ok = ok && __all_sync(0xffffffffu, mbar_wait_addr(afull0 + aoff[u], phase, wc));
            tcol[u] = tcol0 + aslot * C::kAccCols;
            if (++aslot == ACC_BUFS) {
              aslot = 0;
              phase ^= 1u;
            }
          }
        }
        tc_fence_after();
        if (ok) {
          // this warp's columns of the tiles, as 16x256b blocks of 32 columns (CB per tile: its
          // queries' head blocks, contiguous): one TMEM round trip per iteration
          uint32_t v[TPI][2 * CB][16];   // [tile][lane half h][column block cb] at [u][h * CB + cb]
          constexpr uint32_t kHalf16 = 16u << 16;   // lane offset of the quadrant's upper half
          if constexpr (CB == 2) {
            tmem_ld4_16x256b_x4_wait(tcol[0], tcol[0] + 32, tcol[0] + kHalf16, tcol[0] + kHalf16 + 32, v[0]);
          } else {
            static_assert(CB == 1, "one or two column blocks per epilogue warp");
            if (ntile == 2)
              tmem_ld4_16x256b_x4_wait(tcol[0], tcol[0] + kHalf16, tcol[1], tcol[1] + kHalf16,
                                       reinterpret_cast<uint32_t(&)[4][16]>(v));
            else
              tmem_ld2_16x256b_x4_wait(tcol[0], tcol[0] + kHalf16, v[0]);
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) {   // TMEM buffers free for the next MMAs
#pragma unroll
            for (int u = 0; u < TPI; ++u)
              if (u < ntile) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(aempty0 + aoff[u]) : "memory");
          }
#pragma unroll
          for (int u = 0; u < TPI; ++u) {
            if (u >= ntile) break;
            const int sp = s_pos + u * kKeyTile;   // this thread's key position in tile u
            // partial sums over this thread's 8 heads of each head block, for its two rows of
            // each lane half
            float part[4 * QPH];   // [2 h + row][query j] at (2 h + row) * QPH + j
#pragma unroll
            for (int h = 0; h < 2; ++h)
#pragma unroll
              for (int j = 0; j < QPH; ++j) {
                float2 a = make_float2(0.f, 0.f), b = make_float2(0.f, 0.f);
#pragma unroll
                for (int hb = 0; hb < HB; ++hb) {
                  const uint32_t(&x)[16] = v[u][h * CB + j * HB + hb];
#pragma unroll
                  for (int blk = 0; blk < 4; ++blk) {
                    a = ffma2(w2[j * HB + hb][blk], make_float2(fmaxf(__uint_as_float(x[4 * blk]), 0.f),
                                                                fmaxf(__uint_as_float(x[4 * blk + 1]), 0.f)), a);
                    b = ffma2(w2[j * HB + hb][blk], make_float2(fmaxf(__uint_as_float(x[4 * blk + 2]), 0.f),
                                                                fmaxf(__uint_as_float(x[4 * blk + 3]), 0.f)), b);
                  }
                }
                part[(2 * h) * QPH + j] = a.x + a.y;
                part[(2 * h + 1) * QPH + j] = b.x + b.y;
              }
            float score[QPH];
            sum_over_quad<QPH>(part, score, lane);
            if constexpr (kFp8) {
              // the key row's scale (positive) multiplies every head's ReLU term
#pragma unroll
              for (int j = 0; j < QPH; ++j) score[j] *= sk[u];
            }
            // admit (key, position) into this warp's area of each of its queries and count it;
            // the append counts stay warp-uniform in registers.  The float comparison with the
            // threshold admits what the order-preserving key comparison admits (and -0 against
            // a threshold of +0, a harmless extra candidate)
#pragma unroll
            for (int j = 0; j < QPH; ++j) {
              if (j >= nmine) break;
              const bool pass = (sp <= pos_r[j]) && (score[j] >= thr_f[j]);
              const uint32_t bal = __ballot_sync(0xffffffffu, pass);
              if (bal) {
                if (pass) {
                  const uint32_t uk = float_to_ordered(score[j]);
                  st_global_u2_hint(&my_area[static_cast<size_t>(j) * kCandStride + cnt_r[j] + __popc(bal & lt)],
                                    make_uint2(uk, static_cast<uint32_t>(sp)), pol_cand);
                  count_key(st.hist[j0 + j], uk >> kBinShift);
                }
                cnt_r[j] += __popc(bal);
              }
            }
          }
        } else {
          failed = true;
        }
        // check point every check_tiles tiles (the same tiles for every warp of the group); in
        // a long item every check point also checks the append areas' capacity
        to_check -= ntile;
        if (to_check <= 0 && kt + ntile < kt1) {
          to_check = check_tiles;
          bool need = false;
          const bool cap_check = long_item;
          if (cap_check) {
#pragma unroll
            for (int j = 0; j < QPH; ++j) {
              if (j < nmine) {
                need |= cnt_r[j] > kWarpApp - check_margin;
                if (lane == 0) st.cnt_w[j0 + j][qd] = cnt_r[j];
              }
            }
          }
          if (cap_check && named_bar_or(bar, NTG, need || failed)) {
            if (named_bar_or(bar, NTG, failed)) { failed = true; break; }
#pragma unroll 1
            for (int jj = 0; jj < nloc; ++jj) {
              // st.*[jj] is read by every thread here and written only after the barriers below
              const CandView v = cands(jj);
              if (max(max(v.n0, v.n1), max(v.n2, v.n3)) <= kWarpApp - check_margin) continue;
              uint2* const q = qcand + static_cast<size_t>(jj) * kCandStride;
              const int kc = st.kcur[jj];
              const int n_valid = v.total();
              if (n_valid <= kTopK) {
                // fewer than kTopK so far: move the append areas behind the keep set
                uint2* const kk = q + kc * kTopK + v.nk;
                if (gtid == 0) st.ctr[0] = 0;
                named_bar_sync(bar, NTG);
                CandView a = v;
                a.nk = 0;
                collect<NTG>(a, st.ctr, gtid, [&](int rank, uint2 x) { kk[rank] = x; });
                named_bar_sync(bar, NTG);
                if (gtid == 0) {
                  st.cnt_k[jj] = n_valid;
#pragma unroll
                  for (int w = 0; w < 4; ++w) st.cnt_w[jj][w] = 0;
                }
              } else {
                // keep exactly the best kTopK (in the other keep set) and count them afresh
                uint2* const kn = q + (kc ^ 1) * kTopK;
                uint32_t* const h = st.hist[jj];
                const uint32_t kth = resolve_topk<NTG>(v, h, true, rs, gtid, bar, [&](int s2, uint32_t key, uint32_t pos) {
                  kn[s2] = make_uint2(key, pos);
                  count_key(h, key >> kBinShift);
                });
                named_bar_sync(bar, NTG);
                if (gtid == 0) {
                  st.cnt_k[jj] = kTopK;
                  st.kcur[jj] = kc ^ 1;
                  st.thr[jj] = (kth == 0xFFFFFFFFu) ? kth : kth + 1u;
#pragma unroll
                  for (int w = 0; w < 4; ++w) st.cnt_w[jj][w] = 0;
                }
              }
              named_bar_sync(bar, NTG);
            }
#pragma unroll
            for (int j = 0; j < QPH; ++j) {
              if (j < nmine) {
                cnt_r[j] = st.cnt_w[j0 + j][qd];
                thr_f[j] = raise_threshold(thr_f[j], st.thr[j0 + j]);
              }
            }
          }
          // raise each query's admission threshold to the lowest bin of its best kTopK.  Query
          // jl of the group is scanned by the warp of lane quadrant jl % 4 among those that score
          // it, which publishes the bin; the others pick it up here, possibly one check point
          // late.  Neither needs a barrier: a count read early only lowers the bin found, and
          // the published thresholds only rise.
#pragma unroll
          for (int j = 0; j < QPH; ++j) {
            if (j < nmine) {
              const int jl = j0 + j;
              if ((jl & 3) == qd) {
                const uint32_t t = static_cast<uint32_t>(scan_bins_warp(st.hist[jl], kTopK, lane)) << kBinShift;
                thr_f[j] = raise_threshold(thr_f[j], t);
                __syncwarp();
                if (lane == 0) st.thr_bin[jl] = max(st.thr_bin[jl], t);
              } else {
                thr_f[j] = raise_threshold(thr_f[j], st.thr_bin[jl]);
              }
            }
          }
        }
      }
      // ---- end of item: exact top-k of each query's candidates
      if (lane == 0) {
#pragma unroll
        for (int j = 0; j < QPH; ++j)
          if (j < nmine) st.cnt_w[j0 + j][qd] = cnt_r[j];
      }
      if (named_bar_or(bar, NTG, failed)) break;   // a failed wait ends every warp of the group
      if (wi.chunk < 0) {
        // output rows: query jj of the group is resolved by sub-group jj % kSub
#pragma unroll 1
        for (int jj = sg; jj < nloc; jj += kSub) {
          const int t = wi.t0 + qbase + jj;
          const CandView v = cands(jj);
          int32_t* oi = p.idx_out + static_cast<size_t>(t) * kTopK;
          float* os = p.score_out ? p.score_out + static_cast<size_t>(t) * kTopK : nullptr;
          const int prefix = st.pos[jj] + 1;   // keys this query scores (<= 0 if invalid)
          ResolveSmem rq = rsub;
          if (kSub > 1) rq.rh = st.hist[jj];
          if (prefix <= kTopK) {
            // every position 0..prefix-1 is a candidate: place each at its own index
            v.for_rounds<NTS>(stid, [&](const uint4 (&x)[kRoundU], const int (&lim)[kRoundU]) {
#pragma unroll
              for (int e = 0; e < 2 * kRoundU; ++e) {
                const uint2 c = round_entry(x, e);
                if (lim[e >> 1] > (e & 1) && c.y < static_cast<uint32_t>(kTopK)) {
                  __stcs(oi + c.y, static_cast<int>(c.y));
                  if (os) __stcs(os + c.y, ordered_to_float(c.x));
                }
              }
            });
            for (int s2 = max(prefix, 0) + stid; s2 < kTopK; s2 += NTS) {
              __stcs(oi + s2, -1);
              if (os) __stcs(os + s2, -INFINITY);
            }
          } else if constexpr (SORTED) {
            // the query's other keep set is not read by this selection: it stages the row
            uint2* const stage = qcand + static_cast<size_t>(jj) * kCandStride + (st.kcur[jj] ^ 1) * kTopK;
            resolve_topk<NTS>(v, st.hist[jj], kSub > 1, rq, stid, sbar, [&](int s2, uint32_t key, uint32_t pos) {
              stage[s2] = make_uint2(key, pos);
            });
            named_bar_sync(sbar, NTS);
            sort_stage_and_emit<NTS>(stage, stid, sbar, oi, os);
          } else {
            resolve_topk<NTS>(v, st.hist[jj], kSub > 1, rq, stid, sbar, [&](int s2, uint32_t key, uint32_t pos) {
              __stcs(oi + s2, static_cast<int>(pos));
              if (os) __stcs(os + s2, ordered_to_float(key));
            });
          }
          named_bar_sync(sbar, NTS);
        }
        if (kSub > 1) named_bar_sync(bar, NTG);   // every sub-group is done with the counts
      } else {
#pragma unroll 1
        for (int jj = 0; jj < nloc; ++jj) {
          const int t = wi.t0 + qbase + jj;
          const CandView v = cands(jj);
          const int n_valid = v.total();
          uint32_t* pk = p.part_keys + (static_cast<size_t>(t) * kMaxChunks + wi.chunk) * kTopK;
          int32_t* pi = p.part_idx + (static_cast<size_t>(t) * kMaxChunks + wi.chunk) * kTopK;
          uint32_t* const h = st.hist[jj];
          if (n_valid <= kTopK) {
            // every candidate is kept; h already counts exactly these
            if (gtid == 0) st.ctr[0] = 0;
            named_bar_sync(bar, NTG);
            collect<NTG>(v, st.ctr, gtid, [&](int rank, uint2 x) {
              pk[rank] = x.x;
              pi[rank] = static_cast<int>(x.y);
            });
            for (int e = n_valid + gtid; e < kTopK; e += NTG) {
              pk[e] = 0u;
              pi[e] = -1;
            }
          } else {
            // h is cleared before the first kept entry is emitted and counts the kept entries
            resolve_topk<NTG>(v, h, true, rs, gtid, bar, [&](int s2, uint32_t key, uint32_t pos) {
              pk[s2] = key;
              pi[s2] = static_cast<int>(pos);
              count_key(h, key >> kBinShift);
            });
          }
          named_bar_sync(bar, NTG);
          // add the partial list's bin counts to the query's totals, which the merge reads
          uint32_t* const qh = p.part_hist + static_cast<size_t>(t) * kBins1;
          for (int i = gtid; i < kBins1 / 2; i += NTG) {
            const uint32_t wd = h[i];
            if (wd & 0xFFFFu) atomicAdd(&qh[2 * i], wd & 0xFFFFu);
            if (wd >> 16) atomicAdd(&qh[2 * i + 1], wd >> 16);
          }
          named_bar_sync(bar, NTG);
        }
      }
      // empty histograms for the next item
      for (int i = gtid; i < QPW * (kBins1 / 2); i += NTG) (&st.hist[0][0])[i] = 0u;
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
// merge of the split-key path: top-k over the partial lists of one query's key chunks.
// Every chunk added the first-level bin counts of the entries it kept to the query's
// histogram, so the bin b1 holding the kTopK-th largest entry is found from those counts
// alone.  A first pass over the partial lists counts b1's entries by their next 11 bits; the
// sub-bin b2 holding the kTopK-th largest follows.  A second pass writes every entry above
// (b1, b2) to its output slot and gathers the entries of (b1, b2) -- a range of 2^10 keys --
// into shared memory, where the exact kTopK-th largest key K* is found (kth_largest) and the
// entries above K*, then the first ties, are written.  The histogram is cleared after use,
// ready for the next call.
constexpr int kMergeThreads = 1024;
constexpr int kMergeList = 8192;   // entries of the boundary sub-bin held in shared memory

__global__ void __launch_bounds__(kMergeThreads) merge_kernel(const uint32_t* __restrict__ part_keys,
                                                              const int32_t* __restrict__ part_idx,
                                                              const int* __restrict__ tok_nchunks,
                                                              uint32_t* __restrict__ part_hist,
                                                              int32_t* __restrict__ idx_out,
                                                              float* __restrict__ score_out, int sorted) {
  // dynamic: list keys [kMergeList], list positions [kMergeList], stage [kTopK] pairs,
  // second-level counts [kBins1]
  extern __shared__ uint32_t msm[];
  uint32_t* const lkeys = msm;
  int32_t* const lidx = reinterpret_cast<int32_t*>(msm + kMergeList);
  uint2* const stage = reinterpret_cast<uint2*>(msm + 2 * kMergeList);
  uint32_t* const hist2 = msm + 2 * kMergeList + 2 * kTopK;
  __shared__ uint32_t hist[kHistBins];
  __shared__ uint32_t scratch[kMergeThreads / 32];
  __shared__ int sh[8];
  __shared__ int ctr[4];
  // launched as a programmatic dependent of the score kernel: the partial lists and the
  // counts are read only after that grid completed and its writes are visible
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int t = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31;
  const int nch = tok_nchunks[t];
  if (nch < 2) return;   // written by the score kernel itself; no counts were added
  const int n = nch * kTopK;
  const uint32_t* const keys = part_keys + static_cast<size_t>(t) * kMaxChunks * kTopK;
  const int32_t* const pos = part_idx + static_cast<size_t>(t) * kMaxChunks * kTopK;
  uint32_t* const qh = part_hist + static_cast<size_t>(t) * kBins1;
  int32_t* const oi = idx_out + static_cast<size_t>(t) * kTopK;
  float* const os = score_out ? score_out + static_cast<size_t>(t) * kTopK : nullptr;
  auto out = [&](int slot, uint32_t key, int p) {
    if (sorted) {
      stage[slot] = make_uint2(key, static_cast<uint32_t>(p));
    } else {
      __stcs(oi + slot, p);
      if (os) __stcs(os + slot, ordered_to_float(key));
    }
  };
  if (tid < 4) ctr[tid] = 0;
  for (int i = tid; i < kBins1; i += kMergeThreads) hist2[i] = 0u;
  // every key this thread visits (entries 4 g .. 4 g + 3 for g = tid + kMergeThreads j), requested
  // at once so that their latency overlaps the counts' (the lists hold at most kMaxChunks * kTopK
  // entries: kMergeJ 16-byte words per thread); empty slots are 0 and below every score
  constexpr int kMergeJ = kMaxChunks * kTopK / 4 / kMergeThreads;
  uint4 kq[kMergeJ];
#pragma unroll
  for (int j = 0; j < kMergeJ; ++j) {
    const int g = tid + kMergeThreads * j;
    kq[j] = g < n / 4 ? reinterpret_cast<const uint4*>(keys)[g] : make_uint4(0u, 0u, 0u, 0u);
  }
  // 1. boundary bin from the counts (two bins per thread), then clear them
  constexpr int kBPT = kBins1 / kMergeThreads;
  static_assert(kBPT == 2, "two bins per thread");
  uint32_t c[kBPT];
  uint32_t csum = 0;
#pragma unroll
  for (int i = 0; i < kBPT; ++i) {
    c[i] = qh[kBPT * tid + i];
    csum += c[i];
  }
#pragma unroll
  for (int i = 0; i < kBPT; ++i) qh[kBPT * tid + i] = 0u;
  if (tid == 0) {
    sh[0] = 0;
    sh[1] = 0;
  }
  uint32_t above_t = group_suffix_excl<kMergeThreads>(csum, tid, scratch, 1);
  if (above_t < static_cast<uint32_t>(kTopK) && static_cast<uint32_t>(kTopK) <= above_t + csum) {
    uint32_t cum = above_t;
#pragma unroll
    for (int i = kBPT - 1; i >= 0; --i) {
      if (cum + c[i] >= static_cast<uint32_t>(kTopK)) {
        sh[0] = kBPT * tid + i;
        sh[1] = static_cast<int>(cum);
        break;
      }
      cum += c[i];
    }
  }
  named_bar_sync(1, kMergeThreads);
  const uint32_t b1 = static_cast<uint32_t>(min(max(sh[0], 0), kBins1 - 1));
  const int above = min(max(sh[1], 0), kTopK);
  const int need = kTopK - above;
  // 2. second-level counts of b1's entries (a key of an empty slot is 0: never in b1, as b1
  // holds the kTopK-th largest of at least kTopK valid entries)
#pragma unroll
  for (int j = 0; j < kMergeJ; ++j)
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const uint32_t key = u4_get(kq[j], e);
      if (key != 0u && (key >> kBinShift) == b1)
        asm volatile("red.shared.add.u32 [%0], 1;" ::"r"(smem_u32(&hist2[(key >> kSubShift) & (kBins1 - 1)])) : "memory");
    }
  named_bar_sync(1, kMergeThreads);
#pragma unroll
  for (int i = 0; i < kBPT; ++i) {
    c[i] = hist2[kBPT * tid + i];
  }
  csum = c[0] + c[1];
  if (tid == 0) {
    sh[2] = 0;
    sh[3] = 0;
  }
  above_t = group_suffix_excl<kMergeThreads>(csum, tid, scratch, 1);
  if (above_t < static_cast<uint32_t>(need) && static_cast<uint32_t>(need) <= above_t + csum) {
    uint32_t cum = above_t;
#pragma unroll
    for (int i = kBPT - 1; i >= 0; --i) {
      if (cum + c[i] >= static_cast<uint32_t>(need)) {
        sh[2] = kBPT * tid + i;
        sh[3] = static_cast<int>(cum);
        break;
      }
      cum += c[i];
    }
  }
  named_bar_sync(1, kMergeThreads);
  const uint32_t b2 = static_cast<uint32_t>(min(max(sh[2], 0), kBins1 - 1));
  const int above2 = min(max(sh[3], 0), need);
  const uint32_t lo = (b1 << kBinShift) | (b2 << kSubShift), hi = lo + ((1u << kSubShift) - 1u);
  // 3. entries above lo to their slots, the entries of [lo, hi] to the list; positions are
  // read only for the 16-byte words that hold one of those (all such reads issued together)
  const uint32_t lt = lanemask_lt();
  constexpr int kHalfJ = kMergeJ / 2;   // positions are read for half of the words at a time (registers)
#pragma unroll
  for (int jh = 0; jh < kMergeJ; jh += kHalfJ) {
    int4 iq[kHalfJ];
#pragma unroll
    for (int jj = 0; jj < kHalfJ; ++jj) {
      const int j = jh + jj;
      const int g = tid + kMergeThreads * j;
      const bool any = u4_get(kq[j], 0) >= lo || u4_get(kq[j], 1) >= lo || u4_get(kq[j], 2) >= lo ||
                       u4_get(kq[j], 3) >= lo;
      iq[jj] = (any && g < n / 4) ? reinterpret_cast<const int4*>(pos)[g] : make_int4(-1, -1, -1, -1);
    }
#pragma unroll
    for (int jj = 0; jj < kHalfJ; ++jj) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const uint32_t key = u4_get(kq[jh + jj], e);
        const int p = i4_get(iq[jj], e);
        const bool up = p >= 0 && key > hi, mid = p >= 0 && key >= lo && key <= hi;
        const uint32_t bu = __ballot_sync(0xffffffffu, up), bm = __ballot_sync(0xffffffffu, mid);
        if (bu | bm) {
          int ou = 0, om = 0;
          if (lane == 0) {
            if (bu) ou = atomicAdd(&ctr[0], __popc(bu));
            if (bm) om = atomicAdd(&ctr[1], __popc(bm));
          }
          ou = __shfl_sync(0xffffffffu, ou, 0) + __popc(bu & lt);
          om = __shfl_sync(0xffffffffu, om, 0) + __popc(bm & lt);
          if (up && ou < kTopK) out(ou, key, p);
          if (mid && om < kMergeList) {
            lkeys[om] = key;
            lidx[om] = p;
          }
        }
      }
    }
  }
  named_bar_sync(1, kMergeThreads);
  const int m = ctr[1];
  const int base_slot = above + above2;   // slots taken by the entries above the sub-bin
  const int need3 = need - above2;
  int n_above;
  uint32_t kth;
  // 4. the exact need3-th largest key of the sub-bin
  if (m <= kMergeList) {
    kth = kth_largest<kMergeThreads>(lkeys, m, need3, lo, hi, hist, scratch, sh, tid, 1, &n_above);
  } else {
    // more entries in the sub-bin than the list holds (many equal scores): visit them in the
    // partial lists
    auto visit = [&](auto f) {
      for (int e = tid; e < n; e += kMergeThreads)
        if (pos[e] >= 0 && keys[e] >= lo && keys[e] <= hi) f(keys[e]);
    };
    kth = kth_window<kMergeThreads>(visit, need3, lo, hi, hist, scratch, sh, tid, 1, &n_above);
  }
  // 5. the sub-bin's entries above K*, then the first ties
  const int ties = need3 - n_above;
  auto fin = [&](uint32_t key, int p, bool ok) {
    const bool gt = ok && key > kth, eq = ok && key == kth;
    const uint32_t bg = __ballot_sync(0xffffffffu, gt), be = __ballot_sync(0xffffffffu, eq);
    if (bg | be) {
      int og = 0, oe = 0;
      if (lane == 0) {
        if (bg) og = atomicAdd(&ctr[2], __popc(bg));
        if (be) oe = atomicAdd(&ctr[3], __popc(be));
      }
      og = __shfl_sync(0xffffffffu, og, 0) + __popc(bg & lt);
      oe = __shfl_sync(0xffffffffu, oe, 0) + __popc(be & lt);
      if (gt && base_slot + og < kTopK) out(base_slot + og, key, p);
      if (eq && oe < ties) out(base_slot + n_above + oe, key, p);
    }
  };
  if (m <= kMergeList) {
    for (int base = 0; base < m; base += kMergeThreads) {
      const int e = base + tid;
      const bool ok = e < m;
      fin(ok ? lkeys[e] : 0u, ok ? lidx[e] : -1, ok);
    }
  } else {
    for (int base = 0; base < n; base += kMergeThreads) {
      const int e = base + tid;
      const bool ok = e < n && pos[e] >= 0 && keys[e] >= lo && keys[e] <= hi;
      fin(ok ? keys[e] : 0u, ok ? pos[e] : -1, ok);
    }
  }
  if (sorted) {
    named_bar_sync(1, kMergeThreads);
    sort_stage_and_emit<kMergeThreads>(stage, tid, 1, oi, os);
  }
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
  int num_sms;
  int qpi;            // queries per work item on the prefill path (256 / heads)
  int32_t* idx_out;   // [T, kTopK]: every row is padded when the offsets are malformed
  float* score_out;   // [T, kTopK] or null
  TopkWorkspace ws;
};

__device__ int block_exclusive_scan(int* a, int n, int* warp_sums) {
  // in-place exclusive scan of a[0..n) by kPrepThreads threads; returns the total.  Warp 0
  // scans all 32 warp sums, so the block must have exactly 32 warps (kPrepThreads = 1024):
  // with fewer, stale sums would enter the totals and the item list would be written out of
  // bounds.
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

// Key-chunk length of a split query with n keys: chunks of about `target` keys (a
// multiple of 128), at most kMaxChunks of them, of equal length but for the last.
__device__ __forceinline__ int chunk_len_for(int n, int target) {
  int nch = (n + target - 1) / target;
  nch = nch < 1 ? 1 : (nch > kMaxChunks ? kMaxChunks : nch);
  int c = (n + nch - 1) / nch;
  c = (c + kKeyTile - 1) / kKeyTile * kKeyTile;
  return c < kKeyTile ? kKeyTile : c;
}

// Sequence of query token t: the last b with q_seq_offsets[b] <= t.
__device__ __forceinline__ int sequence_of_token(const int32_t* qoff, int B, int t) {
  int lo = 0, hi = B - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (qoff[mid] <= t) lo = mid;
    else hi = mid - 1;
  }
  return lo;
}

constexpr int kPrepCopy = 2048;   // offset arrays up to this length are searched in shared memory
constexpr int kPrepTok = 1024;    // validated positions and chunk counts of up to this many queries stay in shared memory
constexpr int kLenBuckets = 1024; // item lengths in key tiles (longer items share the last bucket)

__global__ void __launch_bounds__(kPrepThreads) prep_kernel(PrepParams p) {
  __shared__ int warp_sums[32];
  __shared__ int bad;
  __shared__ unsigned long long total_keys;
  __shared__ int s_qoff[kPrepCopy + 1];   // copy of q_seq_offsets when B < kPrepCopy
  __shared__ int64_t s_coff[kPrepCopy + 1];   // copy of cache_offsets when B < kPrepCopy
  __shared__ int s_base[kPrepCopy + 1];   // copy of the items' owner bases when n_owners < kPrepCopy
  __shared__ int s_pe[kPrepTok];          // validated positions when T <= kPrepTok
  __shared__ int s_nch[kPrepTok];         // key chunks per query when T <= kPrepTok
  __shared__ int s_len[kLenBuckets];      // split path: items per length bucket, then bucket starts
  const TopkWorkspace& ws = p.ws;
  // the score kernel may start its prologue now; it waits for this grid's results
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  // every input is read once, up front; later phases read the shared copies
  const bool qoff_in_smem = p.B < kPrepCopy;
  if (qoff_in_smem)
    for (int b = threadIdx.x; b <= p.B; b += kPrepThreads) {
      s_qoff[b] = p.q_seq_offsets[b];
      s_coff[b] = p.cache_offsets[b];
    }
  const int32_t* qoff = qoff_in_smem ? s_qoff : p.q_seq_offsets;
  const int64_t* coff = qoff_in_smem ? s_coff : p.cache_offsets;
  const bool tok_in_smem = p.T <= kPrepTok;
  int* const pe = tok_in_smem ? s_pe : ws.pos_eff;      // validated positions (also written to ws.pos_eff)
  int* const nchk = tok_in_smem ? s_nch : ws.tok_nchunks;
  if (threadIdx.x == 0) {
    bad = 0;
    total_keys = 0;
  }
  __syncthreads();
  // 1. offsets
  for (int b = threadIdx.x; b <= p.B; b += kPrepThreads) {
    const int qo = qoff[b];
    const int64_t co = coff[b];
    bool ok = qo >= 0 && qo <= p.T && co >= 0 && co <= p.cache_rows;
    if (b == 0) ok = ok && qo == 0;
    if (b == p.B) ok = ok && qo == p.T;
    if (b > 0) ok = ok && qoff[b - 1] <= qo && coff[b - 1] <= co;
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
    // no query can be attributed to a sequence: every output row becomes padding
    const size_t n4 = static_cast<size_t>(p.T) * (kTopK / 4);
    for (size_t e = threadIdx.x; e < n4; e += kPrepThreads) {
      reinterpret_cast<int4*>(p.idx_out)[e] = make_int4(-1, -1, -1, -1);
      if (p.score_out) reinterpret_cast<float4*>(p.score_out)[e] = make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
    }
    return;
  }
  // 2. validated positions
  for (int t = threadIdx.x; t < p.T; t += kPrepThreads) {
    const int lo = sequence_of_token(qoff, p.B, t);
    const int64_t len = coff[lo + 1] - coff[lo];
    const int pos = p.positions[t];
    const bool ok = pos >= 0 && pos < len;
    if (!ok) atomicOr(ws.err, kErrBounds);
    pe[t] = ok ? pos : -1;
    if (tok_in_smem) ws.pos_eff[t] = ok ? pos : -1;
    ws.tok_nchunks[t] = 0;
    if (p.split && ok) atomicAdd(&total_keys, static_cast<unsigned long long>(pos) + 1ull);
  }
  __syncthreads();
  // split path: chunks sized so that about eight chunks per SM cover all the keys (more,
  // shorter chunks balance the SMs better than fewer, longer ones, and one epilogue group's
  // selection overlaps the other's next chunk; measured on 64 queries of 16 K..128 K keys:
  // 2, 4, 6, 8 chunks per SM took 0.297, 0.243, 0.231, 0.227 ms; the merge reads at most
  // kMaxChunks partial lists per query)
  long long tgt = (static_cast<long long>(total_keys) + 8ll * p.num_sms - 1) / (8ll * p.num_sms);
  tgt = (tgt + kKeyTile - 1) / kKeyTile * kKeyTile;
  const int target = static_cast<int>(tgt < kMinChunk ? kMinChunk : (tgt > (1 << 30) ? (1 << 30) : tgt));
  // 3. items per owner (sequence on the prefill path, query on the split path)
  const int n_owners = p.split ? p.T : p.B;
  int* const base = (n_owners < kPrepCopy) ? s_base : ws.seq_base;   // per-owner item counts, then bases
  for (int o = threadIdx.x; o < n_owners; o += kPrepThreads) {
    int c;
    if (p.split) {
      const int n = pe[o] + 1;
      const int cl = chunk_len_for(n, target);
      c = n > cl ? (n + cl - 1) / cl : 1;
      nchk[o] = c;
      if (tok_in_smem) ws.tok_nchunks[o] = c;
    } else {
      const int nq = qoff[o + 1] - qoff[o];
      c = (nq + p.qpi - 1) / p.qpi;
    }
    base[o] = c;
  }
  __syncthreads();
  const int total = block_exclusive_scan(base, n_owners, warp_sums);
  if (threadIdx.x == 0) {
    base[n_owners] = total;
    *ws.n_items = total;
    *ws.work_counter = 0;
  }
  __syncthreads();
  // 4. items.  Split path: item i is chunk `local` of query o; the items are written longest
  // first (a counting sort by length in key tiles, buckets in descending order), so that the
  // dynamically scheduled CTAs end on the shortest chunks and finish together.  Prefill path:
  // reverse order of (sequence, query group), which puts each sequence's longest prefixes
  // first.
  auto split_item = [&](int i) {
    const int t = owner_of(base, n_owners, i);
    const int local = i - base[t];
    const int n = pe[t] + 1;
    const int nch = nchk[t];
    const int cl = chunk_len_for(n, target);
    WorkItem wi;
    wi.pad0 = wi.pad1 = 0;
    wi.t0 = t;
    wi.nq = 1;
    wi.b = sequence_of_token(qoff, p.B, t);
    wi.k_begin = (nch > 1) ? local * cl : 0;
    wi.k_end = (nch > 1) ? min(n, (local + 1) * cl) : n;
    wi.chunk = (nch > 1) ? local : -1;
    return wi;
  };
  // bucket of an item: kLenBuckets - 1 - (length in tiles, capped), so ascending buckets hold
  // descending lengths
  auto len_bucket = [](const WorkItem& wi) {
    const int tiles = (wi.k_end - wi.k_begin + kKeyTile - 1) / kKeyTile;
    return kLenBuckets - 1 - (tiles < kLenBuckets - 1 ? tiles : kLenBuckets - 1);
  };
  if (p.split) {
    for (int b = threadIdx.x; b < kLenBuckets; b += kPrepThreads) s_len[b] = 0;
    __syncthreads();
    for (int i = threadIdx.x; i < total; i += kPrepThreads) atomicAdd(&s_len[len_bucket(split_item(i))], 1);
    __syncthreads();
    block_exclusive_scan(s_len, kLenBuckets, warp_sums);
    __syncthreads();
    for (int i = threadIdx.x; i < total; i += kPrepThreads) {
      const WorkItem wi = split_item(i);
      ws.items[atomicAdd(&s_len[len_bucket(wi)], 1)] = wi;
    }
  } else {
    for (int i = threadIdx.x; i < total; i += kPrepThreads) {
      const int b = owner_of(base, n_owners, i);
      const int local = i - base[b];
      WorkItem wi;
      wi.pad0 = wi.pad1 = 0;
      const int t0 = qoff[b] + local * p.qpi;
      const int nq = min(p.qpi, qoff[b + 1] - t0);
      int kend = 0;
      for (int j = 0; j < nq; ++j) kend = max(kend, pe[t0 + j] + 1);
      wi.t0 = t0;
      wi.nq = nq;
      wi.b = b;
      wi.k_begin = 0;
      wi.k_end = kend;
      wi.chunk = -1;
      ws.items[total - 1 - i] = wi;
    }
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

template <int QMAX, int STAGES, int ACC_BUFS, int NWG, int EW, bool ALT, bool SORTED, int EB, int H = kHeads>
cudaError_t launch_score(const CUtensorMap& tmQ, const CUtensorMap& tmK, const ScoreParams& p, int grid,
                         cudaStream_t s) {
  using C = ScoreCfg<QMAX, STAGES, ACC_BUFS, NWG, EW, ALT, EB, H>;
  auto kern = score_topk_kernel<QMAX, STAGES, ACC_BUFS, NWG, EW, ALT, SORTED, EB, H>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
  if (e != cudaSuccess) return e;
  if (C::kRegSplit) {
    // setmaxnreg.inc waits until the block's launch allocation can cover the request:
    // refuse to launch a split that does not fit it rather than wait forever
    cudaFuncAttributes fa;
    e = cudaFuncGetAttributes(&fa, kern);
    if (e != cudaSuccess) return e;
    const long launch_regs = static_cast<long>(fa.numRegs) * C::kThreads;
    const long split_regs = static_cast<long>(C::kCtrlRegs) * C::kEpiWarp0 * 32 +
                            static_cast<long>(C::kEpiRegs) * NWG * C::kGroupThreads;
    if (split_regs > launch_regs) return cudaErrorInvalidConfiguration;
  }
  // launched as a programmatic dependent of the prep kernel (which lets it start at once):
  // the prologue overlaps the prep kernel and griddepcontrol.wait orders the rest after it
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(C::kThreads);
  cfg.dynamicSmemBytes = C::kSmemBytes;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, tmQ, tmK, p);
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
  pp.num_sms = num_sms;
  pp.qpi = 256 / a.heads;
  pp.idx_out = a.idx_out;
  pp.score_out = a.score_out;
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
  sp.cand = ws.cand;
  sp.part_keys = ws.part_keys;
  sp.part_idx = ws.part_idx;
  sp.part_hist = ws.part_hist;
  sp.q_scale = a.q_scale;
  sp.key_scale = a.key_scale;
  sp.err = ws.err;
  sp.timeout_ns = a.timeout_ns;
  const int grid = num_sms < ws.cand_slots ? num_sms : ws.cand_slots;
  if (a.split) {
    if (a.heads == 64)
      e = a.sorted ? launch_score<1, 5, 4, 2, 4, true, true, 2, 64>(tmQ1, tmK, sp, grid, s)
                   : launch_score<1, 5, 4, 2, 4, true, false, 2, 64>(tmQ1, tmK, sp, grid, s);
    else if (a.fp8)   // 16 KB key tiles: twice the stages keep the same bytes in flight
      e = a.sorted ? launch_score<1, 10, 4, 2, 4, true, true, 1>(tmQ1, tmK, sp, grid, s)
                   : launch_score<1, 10, 4, 2, 4, true, false, 1>(tmQ1, tmK, sp, grid, s);
    else
      e = a.sorted ? launch_score<1, 5, 4, 2, 4, true, true, 2>(tmQ1, tmK, sp, grid, s)
                   : launch_score<1, 5, 4, 2, 4, true, false, 2>(tmQ1, tmK, sp, grid, s);
    if (e != cudaSuccess) return e;
    const int msmem = 2 * kMergeList * 4 + kTopK * 8 + kBins1 * 4;
    e = cudaFuncSetAttribute(merge_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, msmem);
    if (e != cudaSuccess) return e;
    // programmatic dependent of the score kernel, whose CTAs release it when the work list
    // runs dry: the merge's launch overlaps the score kernel's last items
    cudaLaunchConfig_t mc = {};
    mc.gridDim = dim3(a.T);
    mc.blockDim = dim3(kMergeThreads);
    mc.dynamicSmemBytes = msmem;
    mc.stream = s;
    cudaLaunchAttribute mattr[1];
    mattr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    mattr[0].val.programmaticStreamSerializationAllowed = 1;
    mc.attrs = mattr;
    mc.numAttrs = 1;
    return cudaLaunchKernelEx(&mc, merge_kernel, static_cast<const uint32_t*>(ws.part_keys),
                              static_cast<const int32_t*>(ws.part_idx), static_cast<const int*>(ws.tok_nchunks),
                              ws.part_hist, a.idx_out, a.score_out, a.sorted ? 1 : 0);
  }
  if (a.heads == 64)   // four queries x 64 heads per item
    return a.sorted ? launch_score<4, 3, 2, 2, 8, false, true, 2, 64>(tmQ8, tmK, sp, grid, s)
                    : launch_score<4, 3, 2, 2, 8, false, false, 2, 64>(tmQ8, tmK, sp, grid, s);
  if (a.fp8)
    return a.sorted ? launch_score<kPrefillQ, 6, 2, 2, 8, false, true, 1>(tmQ8, tmK, sp, grid, s)
                    : launch_score<kPrefillQ, 6, 2, 2, 8, false, false, 1>(tmQ8, tmK, sp, grid, s);
  return a.sorted ? launch_score<kPrefillQ, 3, 2, 2, 8, false, true, 2>(tmQ8, tmK, sp, grid, s)
                  : launch_score<kPrefillQ, 3, 2, 2, 8, false, false, 2>(tmQ8, tmK, sp, grid, s);
}

cudaError_t launch_wait_timeout_selftest(int* status, uint64_t timeout_ns, cudaStream_t s) {
  wait_timeout_selftest_kernel<<<1, 32, 0, s>>>(status, timeout_ns);
  return cudaGetLastError();
}

}  // namespace dsa
