// Row-wise top-k selection (velog.io DSA page, §1.2 Fine-grained Token Selection) over materialised scores.
//
// One CTA per row.  Scores are mapped to monotone uint32 order keys (order_key); the selected set is
// {key > T} plus the first `need` entries with key == T in ascending column order, T being the exact key of
// the k-th largest entry, which is "score descending, smaller column first on ties".  Rows with n <= k select
// every column.
//
// Sampled path (rows of 16384+ keys): see below; it reads the row about 1.1 times and falls back to the exact
// paths when its estimate does not hold.
// Fast path (two passes over the row): a 2048-bin histogram of the top 11 key bits gives the bin b* that
// holds the k-th largest key; a second pass appends every entry with bin >= b* (k entries plus the rest of
// bin b*) to shared memory, each warp owning a contiguous segment of the row and its own region, so the
// candidates stay in column order.  The exact threshold within bin b* (a 3-pass radix select on the low 21
// bits over the candidates) and the ordered output then run in shared memory only.
//
// Fallback (when a warp's region would overflow, e.g. on massive ties or on rows sorted by score): a 4-pass
// most-significant-digit radix select over the row (8-bit digits, per-warp histograms) and an ordered
// compaction with warp ballots, streaming the row six times.  Both paths give identical results.
#pragma once
#include "common.cuh"

namespace dsa {

struct TopkParams {
  const float* scores;
  long long ld;                 // row stride when row_off is null
  const long long* row_off;     // [rows] element offset of each row, or null
  const int* row_len;           // [rows] valid length of each row, or null
  int pos0;                     // row_len null: n_r = min(ld, pos0 + r + 1)
  int rows;
  int k;
  int* idx;                     // [rows, k]
  long long idx_ld;
  float* sel_scores;            // [rows, k] score of each selected column (-inf for padding), or null
  const unsigned* hist;         // [rows, 2048] each row's counts of the top 11 order-key bits, or null (the
                                // cluster kernel then reads them instead of counting; the rows kernel ignores it)
};

// Inverse of order_key on the keys it produces (+0.0 for a folded -0.0; NaN stays NaN)
__device__ __forceinline__ float key_score(uint32_t key) {
  return __uint_as_float((key & 0x80000000u) ? (key & 0x7FFFFFFFu) : ~key);
}

// CTA size: 512 threads (two CTAs per SM: the 64 registers per thread and ~107 KB of shared memory allow two).
// Fewer rows than SMs (a decode step) take topk_cluster_kernel, one cluster of CTAs per row.
constexpr int kTopkThreads = 512;
constexpr int kTopkBins = 2048;            // top 11 key bits
constexpr int kTopkSampleMin = 16384;      // rows at least this long take the sampled path

// Candidate slots per CTA, split into one region per warp.  The sampled path's threshold bin spans about 19 %
// in score, so on 128K-key rows it collects 4K+ candidates on average.
template <int NT>
constexpr int topk_candidates() { return 10240; }

template <int NT>
struct TopkSmem {
  static constexpr int W = NT / 32;
  static constexpr int REGION = topk_candidates<NT>() / W;   // candidates per warp region
  uint32_t hist[W][256];                   // radix select: per-warp histograms
  uint32_t bins[kTopkBins];                // top-11-bit histogram
  uint32_t cand_key[W][REGION];
  int cand_idx[W][REGION];
  int region_n[W];
  uint32_t s_need, s_digit, s_bin, s_overflow;
  int s_gt[W], s_eq[W];
  int s_out_base[W], s_eq_base[W];
};
static_assert(2 * sizeof(TopkSmem<kTopkThreads>) <= 228 * 1024 - 2048, "top-k shared memory: two CTAs per SM");

// Radix select on 32-bit keys among the entries that match (key & mask) == prefix: returns the exact k-th
// largest key and sets `need` to the number of entries equal to it that are taken.  each(visit) calls
// visit(key) for every entry this thread owns.  hist is a [TopkSmem<NT>::W][256] shared scratch; every thread of the
// CTA calls this.
template <int NT, typename Each>
__device__ __forceinline__ uint32_t radix_select(Each each, uint32_t prefix, uint32_t mask, int first_shift,
                                                 uint32_t& need, TopkSmem<NT>& sm) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  for (int shift = first_shift; shift >= 0; shift -= 8) {
    for (int i = lane; i < 256; i += 32) sm.hist[warp][i] = 0;
    __syncthreads();
    each([&](uint32_t key) {
      if ((key & mask) == prefix) atomicAdd(&sm.hist[warp][(key >> shift) & 255], 1u);
    });
    __syncthreads();
    // totals over the warps, one bin per thread (the top-11-bit histogram is no longer needed: its first 256 entries
    // hold the totals)
    for (int b = tid; b < 256; b += NT) {
      uint32_t c = 0;
#pragma unroll
      for (int w = 0; w < TopkSmem<NT>::W; ++w) c += sm.hist[w][b];
      sm.bins[b] = c;
    }
    __syncthreads();
    if (warp == 0) {
      // lane l owns bins 255-8l .. 248-8l (descending)
      uint32_t cnt[8];
      uint32_t tot = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        cnt[j] = sm.bins[255 - 8 * lane - j];
        tot += cnt[j];
      }
      uint32_t incl = tot;
#pragma unroll
      for (int d = 1; d < 32; d <<= 1) {
        const uint32_t v = __shfl_up_sync(0xffffffffu, incl, d);
        if (lane >= d) incl += v;
      }
      const uint32_t excl = incl - tot;
      if (excl < need && need <= incl) {
        uint32_t run = excl;
        int j = 0;
        for (; j < 8; ++j) {
          if (run + cnt[j] >= need) break;
          run += cnt[j];
        }
        sm.s_digit = static_cast<uint32_t>(255 - 8 * lane - j);
        sm.s_need = need - run;
      }
    }
    __syncthreads();
    prefix |= sm.s_digit << shift;
    mask |= 255u << shift;
    need = sm.s_need;
    __syncthreads();
  }
  return prefix;
}

// The bin (top 11 key bits) holding the kk-th largest counted key, from the histogram sm.bins: sets sm.s_bin
// (0xFFFFFFFF when fewer than kk keys were counted) and sm.s_need (keys of that bin still to take).  Thread t
// owns bins 2047 - B t .. 2048 - B (t + 1), B = 2048 / threads (descending order).  Every thread of the CTA calls this.
template <int NT>
__device__ __forceinline__ void topk_find_bin(uint32_t kk, TopkSmem<NT>& sm) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid == 0) sm.s_bin = 0xFFFFFFFFu;
  constexpr int BPT = kTopkBins / NT;       // bins per thread
  uint32_t c4[BPT], tot = 0;
#pragma unroll
  for (int j = 0; j < BPT; ++j) { c4[j] = sm.bins[kTopkBins - 1 - BPT * tid - j]; tot += c4[j]; }
  uint32_t incl = tot;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    const uint32_t v = __shfl_up_sync(0xffffffffu, incl, d);
    if (lane >= d) incl += v;
  }
  if (lane == 31) sm.s_gt[warp] = static_cast<int>(incl);
  __syncthreads();
  uint32_t wbase = 0;
  for (int w = 0; w < warp; ++w) wbase += static_cast<uint32_t>(sm.s_gt[w]);
  const uint32_t excl = wbase + incl - tot;
  if (excl < kk && kk <= excl + tot) {
    uint32_t run = excl;
    int j = 0;
    for (; j < BPT; ++j) {
      if (run + c4[j] >= kk) break;
      run += c4[j];
    }
    sm.s_bin = static_cast<uint32_t>(kTopkBins - 1 - BPT * tid - j);
    sm.s_need = kk - run;
  }
  __syncthreads();
}

// Pass over a 16-byte aligned row appending every key of bin >= bmin, in column order, to the per-warp regions
// (warp w owns columns w * seg .. + seg - 1, seg a multiple of four).  A key is in bin >= bmin exactly when the
// score is >= the float whose order key is bmin << 21, so the pass compares raw scores and forms order keys
// for the candidates only.  Lane l takes 16 consecutive columns of each 512-column step (four loads in
// flight); one warp scan of the lanes' counts places the candidates.  Sets sm.region_n, sm.s_eq[w] = the
// warp's uncapped candidate count and sm.s_overflow.
template <int NT>
__device__ __forceinline__ void topk_collect_vec(const float* x, int n, uint32_t bmin, TopkSmem<NT>& sm) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int seg = (((n + TopkSmem<NT>::W - 1) / TopkSmem<NT>::W) + 3) & ~3;
  const int seg0 = min(n, warp * seg), seg1 = min(n, seg0 + seg);
  const uint32_t kk = bmin << 21;
  uint32_t tb = (kk & 0x80000000u) ? (kk & 0x7FFFFFFFu) : ~kk;
  if (!(kk & 0x80000000u) && tb > 0xFF800000u) tb = 0xFF800000u;   // no float key lies below that of -inf
  const float thr = __uint_as_float(tb);
  const bool low = bmin == 0;    // bin 0 holds NaN (order key 0), which compares false: take every key
  int cnt = 0;
  for (int i00 = seg0; i00 < seg1; i00 += 512) {
    const int c0 = i00 + 16 * lane;
    float xv[16];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int col = c0 + 4 * u;
      if (col + 3 < seg1) {
        const float4 v = __ldcs(reinterpret_cast<const float4*>(x + col));   // last read of the row
        xv[4 * u] = v.x; xv[4 * u + 1] = v.y; xv[4 * u + 2] = v.z; xv[4 * u + 3] = v.w;
      } else {
#pragma unroll
        for (int e = 0; e < 4; ++e) xv[4 * u + e] = (col + e < seg1) ? x[col + e] : -INFINITY;
      }
    }
    int c = 0;
#pragma unroll
    for (int e = 0; e < 16; ++e) c += (c0 + e < seg1 && (low || xv[e] >= thr)) ? 1 : 0;
    int incl = c;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, d);
      if (lane >= d) incl += v;
    }
    const int tot = __shfl_sync(0xffffffffu, incl, 31);
    if (c) {
      int pos = cnt + incl - c;
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        if (c0 + e < seg1 && (low || xv[e] >= thr)) {
          if (pos < TopkSmem<NT>::REGION) {
            sm.cand_key[warp][pos] = order_key(xv[e]);
            sm.cand_idx[warp][pos] = c0 + e;
          }
          ++pos;
        }
      }
    }
    cnt += tot;
  }
  if (lane == 0) {
    sm.region_n[warp] = min(cnt, TopkSmem<NT>::REGION);
    sm.s_eq[warp] = cnt;
    if (cnt > TopkSmem<NT>::REGION) atomicOr(&sm.s_overflow, 1u);
  }
}

template <int NT>
__global__ void __launch_bounds__(NT, 2) topk_rows_kernel(const TopkParams p) {
  extern __shared__ __align__(16) uint8_t topk_smem_raw[];
  TopkSmem<NT>& sm = *reinterpret_cast<TopkSmem<NT>*>(topk_smem_raw);

  pdl_allow_next();
  pdl_wait();
  const int r = blockIdx.x;
  if (r >= p.rows) return;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const long long off = p.row_off ? p.row_off[r] : static_cast<long long>(r) * p.ld;
  const float* x = p.scores + off;
  long long nl = p.row_len ? p.row_len[r] : static_cast<long long>(p.pos0) + r + 1;
  if (!p.row_off && nl > p.ld) nl = p.ld;     // a row never extends past its stride
  const int n = static_cast<int>(nl < 0 ? 0 : nl);
  const int k = p.k;
  int* out = p.idx + static_cast<long long>(r) * p.idx_ld;
  float* sel_out = p.sel_scores ? p.sel_scores + static_cast<long long>(r) * p.idx_ld : nullptr;

  if (n <= k) {
    for (int i = tid; i < k; i += NT) {
      out[i] = (i < n) ? i : -1;
      if (sel_out) sel_out[i] = (i < n) ? x[i] : -INFINITY;
    }
    return;
  }
  const int seg = (n + TopkSmem<NT>::W - 1) / TopkSmem<NT>::W;
  const int seg0 = min(n, warp * seg), seg1 = min(n, seg0 + seg);
  uint32_t T = 0, need = 0;
  bool from_row = false;      // the compaction streams the row instead of the candidates
  bool have_T = false;

  // ---------------------------------------------------------------- sampled path (long 16-byte aligned rows)
  // A histogram of one eighth of the row (128-key blocks every 1024 keys) picks a bin b_est low enough that,
  // with a 1.25x margin, at least k keys of the row lie in bins >= b_est; one pass then collects those keys and
  // counts them exactly.  When they are at least k (and fit), the k-th largest key is among them, and the
  // exact selection runs on the candidates alone: the row is read about 1.1 times instead of twice, with an
  // eighth of the histogram atomics.  Otherwise the exact path below runs.
  if ((reinterpret_cast<uintptr_t>(x) & 15) == 0 && n >= kTopkSampleMin) {
    for (int i = tid; i < kTopkBins; i += NT) sm.bins[i] = 0;
    if (tid == 0) sm.s_overflow = 0;
    __syncthreads();
    const int nblk = n >> 10;
    for (int b0 = warp; b0 < nblk; b0 += 4 * TopkSmem<NT>::W) {
      float4 v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int b = b0 + u * TopkSmem<NT>::W;
        if (b < nblk) v[u] = reinterpret_cast<const float4*>(x + (static_cast<long long>(b) << 10))[lane];
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        if (b0 + u * TopkSmem<NT>::W >= nblk) break;
        atomicAdd(&sm.bins[order_key(v[u].x) >> 21], 1u);
        atomicAdd(&sm.bins[order_key(v[u].y) >> 21], 1u);
        atomicAdd(&sm.bins[order_key(v[u].z) >> 21], 1u);
        atomicAdd(&sm.bins[order_key(v[u].w) >> 21], 1u);
      }
    }
    __syncthreads();
    topk_find_bin(5u * static_cast<uint32_t>(k) / 32u + 16u, sm);   // k / 8 sampled keys with a 1.25x margin
    const uint32_t b_est = sm.s_bin;
    if (b_est != 0xFFFFFFFFu && b_est >= 1) {
      topk_collect_vec(x, n, b_est, sm);
      __syncthreads();
      int total = 0;
      for (int w = 0; w < TopkSmem<NT>::W; ++w) total += sm.s_eq[w];
      if (!sm.s_overflow && total >= k) {
        need = static_cast<uint32_t>(k);
        // every warp visits its own candidate region
        auto each = [&](auto visit) {
          for (int j = lane; j < sm.region_n[warp]; j += 32) visit(sm.cand_key[warp][j]);
        };
        T = radix_select(each, 0u, 0u, 24, need, sm);
        have_T = true;
      }
    }
    __syncthreads();
  }

  if (!have_T) {
  // ---------------------------------------------------------------- fast path, pass 1: top-11-bit histogram
  for (int i = tid; i < kTopkBins; i += NT) sm.bins[i] = 0;
  if (tid == 0) sm.s_overflow = 0;
  __syncthreads();
  if ((reinterpret_cast<uintptr_t>(x) & 15) == 0) {
    const float4* x4 = reinterpret_cast<const float4*>(x);
    const int n4 = n >> 2;
    for (int i = tid; i < n4; i += 4 * NT) {
      float4 v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u)
        if (i + u * NT < n4) v[u] = x4[i + u * NT];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        if (i + u * NT >= n4) break;
        atomicAdd(&sm.bins[order_key(v[u].x) >> 21], 1u);
        atomicAdd(&sm.bins[order_key(v[u].y) >> 21], 1u);
        atomicAdd(&sm.bins[order_key(v[u].z) >> 21], 1u);
        atomicAdd(&sm.bins[order_key(v[u].w) >> 21], 1u);
      }
    }
    for (int i = 4 * n4 + tid; i < n; i += NT) atomicAdd(&sm.bins[order_key(x[i]) >> 21], 1u);
  } else {
    for (int i = tid; i < n; i += NT) atomicAdd(&sm.bins[order_key(x[i]) >> 21], 1u);
  }
  __syncthreads();
  // bin b* holding the k-th largest key
  topk_find_bin(static_cast<uint32_t>(k), sm);
  const uint32_t bstar = sm.s_bin;
  const uint32_t need_bin = sm.s_need;
  // ---------------------------------------------------------------- pass 2: gather candidates in column order
  if ((reinterpret_cast<uintptr_t>(x) & 15) == 0) {
    topk_collect_vec(x, n, bstar, sm);
  } else {
    int cnt = 0;
    bool over = false;
    for (int i0 = seg0; i0 < seg1; i0 += 32) {
      const int i = i0 + lane;
      const uint32_t key = (i < seg1) ? order_key(x[i]) : 0u;
      const bool c = i < seg1 && (key >> 21) >= bstar;
      const uint32_t m = __ballot_sync(0xffffffffu, c);
      const int pos = cnt + __popc(m & ((1u << lane) - 1));
      if (c && pos < TopkSmem<NT>::REGION) {
        sm.cand_key[warp][pos] = key;
        sm.cand_idx[warp][pos] = i;
      }
      cnt += __popc(m);
      if (cnt > TopkSmem<NT>::REGION) over = true;
    }
    if (lane == 0) {
      sm.region_n[warp] = min(cnt, TopkSmem<NT>::REGION);
      if (over) atomicOr(&sm.s_overflow, 1u);
    }
  }
  __syncthreads();

  if (!sm.s_overflow) {
    // exact threshold inside bin b*, over the candidates (shared memory only)
    need = need_bin;
    auto each = [&](auto visit) {
      for (int j = lane; j < sm.region_n[warp]; j += 32) visit(sm.cand_key[warp][j]);
    };
    T = radix_select(each, bstar << 21, 0xFFE00000u, 16, need, sm);
    from_row = false;
  } else {
    need = static_cast<uint32_t>(k);
    auto each = [&](auto visit) {
      for (int i = tid; i < n; i += NT) visit(order_key(x[i]));
    };
    T = radix_select(each, 0u, 0u, 24, need, sm);
    from_row = true;
  }
  }
  // ---------------------------------------------------------------- ordered compaction
  // every warp walks its own span (a contiguous row segment, or its candidate region), in column order
  const int span = from_row ? seg1 - seg0 : sm.region_n[warp];
  auto key_at = [&](int j) -> uint32_t { return from_row ? order_key(x[seg0 + j]) : sm.cand_key[warp][j]; };
  auto col_at = [&](int j) -> int { return from_row ? seg0 + j : sm.cand_idx[warp][j]; };
  int gt = 0, eq = 0;
  for (int j = lane; j < span; j += 32) {
    const uint32_t key = key_at(j);
    gt += key > T;
    eq += key == T;
  }
#pragma unroll
  for (int d = 16; d > 0; d >>= 1) {
    gt += __shfl_xor_sync(0xffffffffu, gt, d);
    eq += __shfl_xor_sync(0xffffffffu, eq, d);
  }
  if (lane == 0) { sm.s_gt[warp] = gt; sm.s_eq[warp] = eq; }
  __syncthreads();
  if (tid == 0) {
    int base = 0, eqb = 0;
    for (int w = 0; w < TopkSmem<NT>::W; ++w) {
      sm.s_out_base[w] = base;
      sm.s_eq_base[w] = eqb;
      const int take_eq = max(0, min(sm.s_eq[w], static_cast<int>(need) - eqb));
      base += sm.s_gt[w] + take_eq;
      eqb += sm.s_eq[w];
    }
  }
  __syncthreads();
  int pos = sm.s_out_base[warp];
  int eq_rank = sm.s_eq_base[warp];
  for (int j0 = 0; j0 < span; j0 += 32) {
    const int j = j0 + lane;
    uint32_t key = 0;
    if (j < span) key = key_at(j);
    const bool is_eq = j < span && key == T;
    const uint32_t eq_mask = __ballot_sync(0xffffffffu, is_eq);
    const int my_eq_rank = eq_rank + __popc(eq_mask & ((1u << lane) - 1));
    const bool sel = j < span && (key > T || (is_eq && my_eq_rank < static_cast<int>(need)));
    const uint32_t sel_mask = __ballot_sync(0xffffffffu, sel);
    if (sel) {
      const int dst = pos + __popc(sel_mask & ((1u << lane) - 1));
      out[dst] = col_at(j);
      if (sel_out) sel_out[dst] = key_score(key);
    }
    pos += __popc(sel_mask);
    eq_rank += __popc(eq_mask);
  }
}

}  // namespace dsa
