// Top-k selection of a few long rows (velog.io DSA page, §1.2 Fine-grained Token Selection), one cluster of
// kTkcCluster CTAs per row.
//
// With fewer rows than SMs (a decode step: one row per sequence, up to 131K keys) one CTA per row leaves most of
// the GPU idle and serialises the row's passes on one SM.  Here the row is cut into kTkcCluster contiguous
// segments, one per CTA of a cluster, and the CTAs combine their counts through distributed shared memory:
//   1. every CTA builds the histogram of the top 11 order-key bits of its segment; the cluster's histogram (the
//      sum of the CTAs', read from each peer) gives the bin b* holding the k-th largest key, the same in every CTA;
//   2. every CTA collects the keys of bin >= b* of its segment into per-warp regions in column order;
//   3. a radix select over those candidates finds the exact k-th largest key T and the number `need` of keys
//      equal to T to take: each pass sums the CTAs' digit histograms (double-buffered, so one cluster barrier per
//      pass suffices), and every CTA picks the same digit;
//   4. the CTAs exchange their counts of keys > T and == T; each then writes its selected columns, in column order,
//      at its offset in the output row.
// The selection is "score descending, smaller column first on ties", identical to topk_rows_kernel's.  When a
// warp's candidate region would overflow (massive ties), the whole cluster takes a 4-pass radix select over the
// row segments instead, and the output walks the segments.
#pragma once
#include "topk.cuh"

namespace dsa {

constexpr int kTkcCluster = 8;          // CTAs per row (portable cluster size)
constexpr int kTkcThreads = 256;
constexpr int kTkcRegion = 384;         // candidate slots per warp (3072 per CTA)

struct TkcSmem {
  static constexpr int W = kTkcThreads / 32;
  uint32_t bins[kTopkBins];             // this CTA's top-11-bit histogram of its segment (peers read it)
  uint32_t merged[kTopkBins];           // the cluster's histogram (radix passes use its first 256 entries)
  uint32_t hist[W][256];                // radix pass: per-warp digit histograms
  uint32_t hist_cta[2][256];            // radix pass: this CTA's digit histogram, double-buffered (peers read it)
  uint32_t cand_key[W][kTkcRegion];
  int cand_idx[W][kTkcRegion];
  int region_n[W];
  int w_gt[W], w_eq[W], w_base[W], w_eqb[W];
  int cta_gt, cta_eq;                   // peers read them for the output offsets
  uint32_t cta_over;                    // peers read it: a warp region of this CTA overflowed
  uint32_t s_bin, s_need, s_digit;
};
static_assert(4 * (sizeof(TkcSmem) + 1024) <= 228 * 1024, "four cluster top-k CTAs per SM");

// The u32 at the same shared-memory offset as `local` in each of the cluster's eight CTAs, loaded by one block of
// eight loads, so that their latencies overlap.
__device__ __forceinline__ void cluster_load8(const void* local, uint32_t (&v)[kTkcCluster]) {
  static_assert(kTkcCluster == 8, "eight loads");
  const uint32_t a = smem_u32(local);
  asm volatile(
      "ld.shared::cluster.u32 %0, [%8];\n\tld.shared::cluster.u32 %1, [%9];\n\t"
      "ld.shared::cluster.u32 %2, [%10];\n\tld.shared::cluster.u32 %3, [%11];\n\t"
      "ld.shared::cluster.u32 %4, [%12];\n\tld.shared::cluster.u32 %5, [%13];\n\t"
      "ld.shared::cluster.u32 %6, [%14];\n\tld.shared::cluster.u32 %7, [%15];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7])
      : "r"(map_cluster(a, 0)), "r"(map_cluster(a, 1)), "r"(map_cluster(a, 2)), "r"(map_cluster(a, 3)),
        "r"(map_cluster(a, 4)), "r"(map_cluster(a, 5)), "r"(map_cluster(a, 6)), "r"(map_cluster(a, 7))
      : "memory");
}
// sum over the cluster's CTAs of the u32 at the same shared-memory offset as `local`
__device__ __forceinline__ uint32_t cluster_sum_u32(const void* local) {
  uint32_t v[kTkcCluster];
  cluster_load8(local, v);
  uint32_t s = 0;
#pragma unroll
  for (int q = 0; q < kTkcCluster; ++q) s += v[q];
  return s;
}

// Digit of a descending scan: the largest digit d with (count of digits > d) < need <= (count of digits >= d), over
// the 256 counts in sm.merged[0..255]; sets sm.s_digit and sm.s_need (entries of digit d still to take).  Run by
// warp 0; lane l owns digits 255 - 8 l .. 248 - 8 l.
__device__ __forceinline__ void tkc_pick_digit(uint32_t need, TkcSmem& sm) {
  const int lane = threadIdx.x & 31;
  uint32_t cnt[8], tot = 0;
#pragma unroll
  for (int j = 0; j < 8; ++j) { cnt[j] = sm.merged[255 - 8 * lane - j]; tot += cnt[j]; }
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

// Cluster-wide radix select on 32-bit keys among the entries with (key & mask) == prefix: returns the exact
// need-th largest key and sets `need` to the number of entries equal to it that are taken.  each(visit) visits
// every key this thread owns.  Every thread of every CTA of the cluster calls this with the same arguments.
template <typename Each>
__device__ __forceinline__ uint32_t tkc_radix_select(Each each, uint32_t prefix, uint32_t mask, int first_shift,
                                                     uint32_t& need, TkcSmem& sm) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int buf = 0;
  for (int shift = first_shift; shift >= 0; shift -= 8, buf ^= 1) {
    for (int i = lane; i < 256; i += 32) sm.hist[warp][i] = 0;
    __syncthreads();
    each([&](uint32_t key) {
      if ((key & mask) == prefix) atomicAdd(&sm.hist[warp][(key >> shift) & 255], 1u);
    });
    __syncthreads();
    for (int b = tid; b < 256; b += kTkcThreads) {
      uint32_t s = 0;
#pragma unroll
      for (int w = 0; w < TkcSmem::W; ++w) s += sm.hist[w][b];
      sm.hist_cta[buf][b] = s;
    }
    // every CTA's histogram of this pass is complete; the buffer of the previous pass is no longer read by any
    // peer (each read it before arriving here), so the next pass may overwrite it
    cluster_sync();
    for (int b = tid; b < 256; b += kTkcThreads) sm.merged[b] = cluster_sum_u32(&sm.hist_cta[buf][b]);
    __syncthreads();
    if (warp == 0) tkc_pick_digit(need, sm);
    __syncthreads();
    prefix |= sm.s_digit << shift;
    mask |= 255u << shift;
    need = sm.s_need;
  }
  return prefix;
}

__global__ void __cluster_dims__(kTkcCluster, 1, 1) __launch_bounds__(kTkcThreads, 4)
    topk_cluster_kernel(const TopkParams p) {
  extern __shared__ __align__(16) uint8_t tkc_smem_raw[];
  TkcSmem& sm = *reinterpret_cast<TkcSmem*>(tkc_smem_raw);
  constexpr int W = TkcSmem::W;
  pdl_allow_next();
  pdl_wait();
  const int r = blockIdx.x / kTkcCluster;
  const int rank = static_cast<int>(cluster_rank());
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (r >= p.rows) return;                       // whole clusters only: the grid is rows x kTkcCluster
  const long long off = p.row_off ? p.row_off[r] : static_cast<long long>(r) * p.ld;
  const float* x = p.scores + off;
  long long nl = p.row_len ? p.row_len[r] : static_cast<long long>(p.pos0) + r + 1;
  if (!p.row_off && nl > p.ld) nl = p.ld;
  const int n = static_cast<int>(nl < 0 ? 0 : nl);
  const int k = p.k;
  int* out = p.idx + static_cast<long long>(r) * p.idx_ld;
  float* sel_out = p.sel_scores ? p.sel_scores + static_cast<long long>(r) * p.idx_ld : nullptr;
  if (n <= k) {                                  // the same for every CTA of the cluster: no barrier is skipped
    if (rank == 0)
      for (int i = tid; i < k; i += kTkcThreads) {
        out[i] = (i < n) ? i : -1;
        if (sel_out) sel_out[i] = (i < n) ? x[i] : -INFINITY;
      }
    return;
  }
  const bool vec = (reinterpret_cast<uintptr_t>(x) & 15) == 0;
  // this CTA's segment (a multiple of four columns, so that it starts 16-byte aligned when the row does) and its
  // warps' sub-segments, all in column order
  const int cseg = (((n + kTkcCluster - 1) / kTkcCluster) + 3) & ~3;
  const int c0 = min(n, rank * cseg), c1 = min(n, c0 + cseg);
  const int wseg = (((c1 - c0 + W - 1) / W) + 3) & ~3;
  const int w0 = min(c1, c0 + warp * wseg), w1 = min(c1, w0 + wseg);

  // ---------------------------------------------------------------- 1. histograms, the cluster's bin b*
  // thread t scans bins 2047 - 8 t .. 2040 - 8 t (descending): c8[j] holds bin 2047 - 8 t - j
  constexpr int BPT = kTopkBins / kTkcThreads;
  static_assert(BPT == 8, "eight bins per thread");
  uint32_t c8[BPT];
  if (tid == 0) sm.s_bin = 0xFFFFFFFFu;
  if (p.hist) {
    // the row's histogram came with the scores (the decode indexer counts them as it writes them): each thread
    // loads its own eight bins, with two 16-byte loads in flight when the histogram is aligned
    const unsigned* h = p.hist + static_cast<long long>(r) * kTopkBins + (kTopkBins - BPT * (tid + 1));
    if ((reinterpret_cast<uintptr_t>(h) & 15) == 0) {
      const uint4 lo = reinterpret_cast<const uint4*>(h)[0], hi = reinterpret_cast<const uint4*>(h)[1];
      c8[0] = hi.w; c8[1] = hi.z; c8[2] = hi.y; c8[3] = hi.x;
      c8[4] = lo.w; c8[5] = lo.z; c8[6] = lo.y; c8[7] = lo.x;
    } else {
#pragma unroll
      for (int j = 0; j < BPT; ++j) c8[j] = h[BPT - 1 - j];
    }
  } else {
    for (int i = tid; i < kTopkBins; i += kTkcThreads) sm.bins[i] = 0;
    __syncthreads();
    if (vec) {
      for (int i0 = c0 + 4 * tid; i0 < c1; i0 += 16 * kTkcThreads) {
        float4 v[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int i = i0 + 4 * u * kTkcThreads;
          if (i + 3 < c1) {
            v[u] = *reinterpret_cast<const float4*>(x + i);
          } else {
            v[u].x = (i < c1) ? x[i] : NAN;
            v[u].y = (i + 1 < c1) ? x[i + 1] : NAN;
            v[u].z = (i + 2 < c1) ? x[i + 2] : NAN;
            v[u].w = NAN;
          }
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int i = i0 + 4 * u * kTkcThreads;
          if (i < c1) atomicAdd(&sm.bins[order_key(v[u].x) >> 21], 1u);
          if (i + 1 < c1) atomicAdd(&sm.bins[order_key(v[u].y) >> 21], 1u);
          if (i + 2 < c1) atomicAdd(&sm.bins[order_key(v[u].z) >> 21], 1u);
          if (i + 3 < c1) atomicAdd(&sm.bins[order_key(v[u].w) >> 21], 1u);
        }
      }
    } else {
      for (int i = c0 + tid; i < c1; i += kTkcThreads) atomicAdd(&sm.bins[order_key(x[i]) >> 21], 1u);
    }
    cluster_sync();                                // every CTA's histogram is complete
    {
      // the eight bins of this thread from every CTA: 64 loads issued before any is summed
      uint32_t v[BPT][kTkcCluster];
#pragma unroll
      for (int j = 0; j < BPT; ++j) cluster_load8(&sm.bins[tid + j * kTkcThreads], v[j]);
#pragma unroll
      for (int j = 0; j < BPT; ++j) {
        uint32_t s = 0;
#pragma unroll
        for (int q = 0; q < kTkcCluster; ++q) s += v[j][q];
        sm.merged[tid + j * kTkcThreads] = s;
      }
    }
    __syncthreads();
#pragma unroll
    for (int j = 0; j < BPT; ++j) c8[j] = sm.merged[kTopkBins - 1 - BPT * tid - j];
  }
  {
    // bin holding the k-th largest key of the row (the scan's barrier orders tid 0's reset of s_bin before the
    // write of the thread that finds it)
    uint32_t tot = 0;
#pragma unroll
    for (int j = 0; j < BPT; ++j) tot += c8[j];
    uint32_t incl = tot;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const uint32_t v = __shfl_up_sync(0xffffffffu, incl, d);
      if (lane >= d) incl += v;
    }
    if (lane == 31) sm.w_gt[warp] = static_cast<int>(incl);
    __syncthreads();
    uint32_t wbase = 0;
    for (int w = 0; w < warp; ++w) wbase += static_cast<uint32_t>(sm.w_gt[w]);
    const uint32_t excl = wbase + incl - tot;
    const uint32_t kk = static_cast<uint32_t>(k);
    if (excl < kk && kk <= excl + tot) {
      uint32_t run = excl;
      int j = 0;
      for (; j < BPT; ++j) {
        if (run + c8[j] >= kk) break;
        run += c8[j];
      }
      sm.s_bin = static_cast<uint32_t>(kTopkBins - 1 - BPT * tid - j);
      sm.s_need = kk - run;
    }
    __syncthreads();
  }
  const uint32_t bstar = sm.s_bin;               // n > k keys were counted, so the bin exists
  const uint32_t need_bin = sm.s_need;

  // ---------------------------------------------------------------- 2. candidates of bin >= b*, in column order
  // A key is in bin >= b* exactly when the score is >= the float whose order key is b* << 21, so the pass compares
  // raw scores.  Lane l takes 16 consecutive columns of each 512-column step of its warp's sub-segment (four
  // 16-byte loads when the row is aligned); one warp scan of the lanes' counts places the candidates.
  {
    const uint32_t kb = bstar << 21;
    uint32_t tb = (kb & 0x80000000u) ? (kb & 0x7FFFFFFFu) : ~kb;
    if (!(kb & 0x80000000u) && tb > 0xFF800000u) tb = 0xFF800000u;   // no float key lies below that of -inf
    const float thr = __uint_as_float(tb);
    const bool low = bstar == 0;               // bin 0 holds NaN too, which compares false: take every key
    int cnt = 0;
    // two 512-column steps per round: their eight 16-byte loads per lane are in flight together, then each step's
    // passing columns become a 16-bit mask (the data registers are free again) and the few candidates re-read
    // their scores (L1 hits) when they are written
    auto pass_mask = [&](int c0l) -> uint32_t {
      float xv[16];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int col = c0l + 4 * u;
        if (vec && col + 3 < w1) {
          const float4 v = *reinterpret_cast<const float4*>(x + col);
          xv[4 * u] = v.x; xv[4 * u + 1] = v.y; xv[4 * u + 2] = v.z; xv[4 * u + 3] = v.w;
        } else {
#pragma unroll
          for (int e = 0; e < 4; ++e) xv[4 * u + e] = (col + e < w1) ? x[col + e] : -INFINITY;
        }
      }
      uint32_t m = 0;
#pragma unroll
      for (int e = 0; e < 16; ++e) m |= (c0l + e < w1 && (low || xv[e] >= thr)) ? (1u << e) : 0u;
      return m;
    };
    auto place = [&](int c0l, uint32_t m) {
      const int c = __popc(m);
      int incl = c;
#pragma unroll
      for (int d = 1; d < 32; d <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, d);
        if (lane >= d) incl += v;
      }
      const int tot = __shfl_sync(0xffffffffu, incl, 31);
      int pos = cnt + incl - c;
      while (m) {
        const int e = __ffs(m) - 1;
        m &= m - 1;
        if (pos < kTkcRegion) {
          sm.cand_key[warp][pos] = order_key(x[c0l + e]);
          sm.cand_idx[warp][pos] = c0l + e;
        }
        ++pos;
      }
      cnt += tot;
    };
    for (int i00 = w0; i00 < w1; i00 += 1024) {
      const int ca = i00 + 16 * lane, cb = ca + 512;
      const uint32_t ma = pass_mask(ca), mb = pass_mask(cb);   // columns past w1 load nothing and never pass
      place(ca, ma);
      place(cb, mb);
    }
    if (lane == 0) {
      sm.region_n[warp] = min(cnt, kTkcRegion);
      sm.w_eq[warp] = cnt > kTkcRegion ? 1 : 0;
    }
  }
  __syncthreads();
  if (tid == 0) {
    uint32_t over = 0;
    for (int w = 0; w < W; ++w) over |= static_cast<uint32_t>(sm.w_eq[w]);
    sm.cta_over = over;
  }
  cluster_sync();                                // every CTA's overflow flag is set
  bool from_row = false;
  {
    uint32_t v[kTkcCluster];
    cluster_load8(&sm.cta_over, v);
    uint32_t over = 0;
#pragma unroll
    for (int q = 0; q < kTkcCluster; ++q) over |= v[q];
    from_row = over != 0;                        // the same decision in every CTA
  }

  // ---------------------------------------------------------------- 3. the exact threshold
  uint32_t need, T;
  if (!from_row) {
    need = need_bin;
    auto each = [&](auto visit) {
      for (int j = lane; j < sm.region_n[warp]; j += 32) visit(sm.cand_key[warp][j]);
    };
    T = tkc_radix_select(each, bstar << 21, 0xFFE00000u, 16, need, sm);
  } else {
    need = static_cast<uint32_t>(k);
    auto each = [&](auto visit) {
      for (int i = w0 + lane; i < w1; i += 32) visit(order_key(x[i]));
    };
    T = tkc_radix_select(each, 0u, 0u, 24, need, sm);
  }

  // ---------------------------------------------------------------- 4. ordered output
  const int span = from_row ? w1 - w0 : sm.region_n[warp];
  auto key_at = [&](int j) -> uint32_t { return from_row ? order_key(x[w0 + j]) : sm.cand_key[warp][j]; };
  auto col_at = [&](int j) -> int { return from_row ? w0 + j : sm.cand_idx[warp][j]; };
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
  if (lane == 0) { sm.w_gt[warp] = gt; sm.w_eq[warp] = eq; }
  __syncthreads();
  if (tid == 0) {
    int g = 0, e = 0;
    for (int w = 0; w < W; ++w) { g += sm.w_gt[w]; e += sm.w_eq[w]; }
    sm.cta_gt = g;
    sm.cta_eq = e;
  }
  cluster_sync();                                // every CTA's counts are set
  if (warp == 0) {
    // this CTA's place in the row: the entries the CTAs before it take (all eight CTAs' counts, loaded at once)
    uint32_t gv[kTkcCluster], ev[kTkcCluster];
    cluster_load8(&sm.cta_gt, gv);
    cluster_load8(&sm.cta_eq, ev);
    int base = 0, eqb = 0;
#pragma unroll
    for (int q = 0; q < kTkcCluster; ++q) {
      if (q < rank) {
        base += static_cast<int>(gv[q]) + max(0, min(static_cast<int>(ev[q]), static_cast<int>(need) - eqb));
        eqb += static_cast<int>(ev[q]);
      }
    }
    if (lane == 0) {
      for (int w = 0; w < W; ++w) {
        sm.w_base[w] = base;
        sm.w_eqb[w] = eqb;
        base += sm.w_gt[w] + max(0, min(sm.w_eq[w], static_cast<int>(need) - eqb));
        eqb += sm.w_eq[w];
      }
    }
  }
  __syncthreads();
  int pos = sm.w_base[warp];
  int eq_rank = sm.w_eqb[warp];
  for (int j0 = 0; j0 < span; j0 += 32) {
    const int j = j0 + lane;
    uint32_t key = 0;
    if (j < span) key = key_at(j);
    const bool is_eq = j < span && key == T;
    const uint32_t eq_mask = __ballot_sync(0xffffffffu, is_eq);
    const int my_eq_rank = eq_rank + __popc(eq_mask & ((1u << lane) - 1));
    const bool sel = j < span && (key > T || (is_eq && my_eq_rank < static_cast<int>(need)));
    const uint32_t sel_mask = __ballot_sync(0xffffffffu, sel);
    const int dst = pos + __popc(sel_mask & ((1u << lane) - 1));
    if (sel && dst < k) {                        // dst < k always; the bound keeps a fault out of other rows
      out[dst] = col_at(j);
      if (sel_out) sel_out[dst] = key_score(key);
    }
    pos += __popc(sel_mask);
    eq_rank += __popc(eq_mask);
  }
  cluster_sync();                                // no CTA leaves while a peer may still read its shared memory
}

}  // namespace dsa
