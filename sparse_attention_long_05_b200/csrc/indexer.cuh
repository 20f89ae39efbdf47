// Lightning-indexer kernel: I[t,s] = sum_j w[t,j] * ReLU(q_I[t,j] . k_I[s])   (velog.io DSA page, §1.1)
//
// Data layout on the tensor core.  One tcgen05 MMA computes, for a tile of 128 keys and a group of NT query
// tokens, D[s, (t, j)] = k_I[s] . q_I[t, j] with FP8 e4m3 operands and fp32 accumulation:
//   A = 128 keys x d_I   (K-major, TMA-loaded tile of k_I),
//   B = NT*H_I rows of q_I x d_I (K-major; rows (t, j) are consecutive in q_I's [T, H_I, d_I] layout),
//   D = 128 TMEM lanes (one per key) x NT*H_I fp32 columns.
// Because a key owns a TMEM lane, the ReLU and the head-weighted sum over j stay within a warp: the epilogue
// reads its lanes' columns, forms sum_j w[t,j] * max(x, 0) for each token of the stage (sixteen heads per thread,
// then a two-step shuffle over the four threads sharing a key), multiplies by the key scale (Gaussian mode; the
// query scale is folded into w), and writes I[t, s].
//
// Warp roles (one CTA per SM):
//   warp 0      TMA producer: q_I block of the work item, then one k_I tile per pipeline stage
//   warp 1      TMEM allocation + MMA issue (one elected thread)
//   warps 2..   epilogue warpgroup(s); warp w reads TMEM lanes 32*(w % 4) .. +31
// A ring of TMEM accumulators (2 of 256 columns; 4 of 64 in decode, two CTAs per SM) lets the
// epilogue of one (tile, group) overlap the MMAs of the next ones; with two epilogue warpgroups, each takes
// every other accumulator stage.  Tiles lying wholly above the causal diagonal of every token of the item are
// never loaded.
//
// Work items:
//   kModeScores  item = (block of NG*NT query rows, range of key tiles); writes scores [T, S] (tests,
//                materialised prefill chunks);
//   kModeDecode  item = (sequence b, range of its key tiles); one token per sequence; keys are the rows
//                [cache_off[b], cache_off[b] + len1[b]) of the flat key cache; writes the sequence's len1[b]
//                fp32 scores from score_off[b] on (one packed row per sequence).  The key tiles of all sequences,
//                laid end to end, are cut into gridDim.x equal ranges, one per CTA; a CTA's items are the pieces
//                of the sequences its range covers, so every CTA streams the same number of key tiles.
//   kModeSegments item = (segment, block of NG*NT query rows, range of key tiles); a segment is a run of query rows
//                of one sequence of a packed batch (its own query rows, key rows, positions and score rows), so
//                that one launch scores the rows of many sequences.
#pragma once
#include "common.cuh"

namespace dsa {

enum { kModeScores = 0, kModeDecode = 1, kModeSegments = 2 };

// kModeSegments: one run of consecutive query rows of one sequence
struct IndexerSeg {
  long long q_row0;     // row of q_I / w / q_scale holding the run's first query row
  long long key_row0;   // row of k_I / k_scale holding key 0 of the sequence
  long long out_base;   // score offset of (first query row, key 0)
  int pos0;             // position of the first query row in its sequence
  int n_rows;           // query rows of the run
  int S;                // keys the run sees (pos0 + n_rows)
  int ld;               // row stride of the run's scores
  int nsplit;           // key-range splits per query block
  int item0;            // first work item of the run
};

struct IndexerParams {
  const float* w;          // [T, H_I]
  const float* q_scale;    // [T] or null
  const float* k_scale;    // per key row, or null
  float* scores;           // output (see modes)
  long long ld;            // kModeScores: row stride of scores
  int T;                   // query rows (kModeScores) / sequences B (kModeDecode)
  int S;                   // kModeScores: number of keys
  int pos0;                // kModeScores: absolute position of query row 0
  int n_items;             // kModeScores: number of work items
  int nsplit;              // kModeScores: key-range splits per query block
  int split_tiles;         // kModeScores: key tiles per split
  const long long* cache_off;  // kModeDecode: [B] first cache row of each sequence
  const int* len1;             // kModeDecode: [B] keys of each sequence after the append (0: skip it)
  const long long* score_off;  // kModeDecode: [B] start of each sequence's score row
  const IndexerSeg* segs;      // kModeSegments: [n_segs]
  int n_segs;
  const int* page_table;       // kModeDecode, paged caches: [B, max_pages] page of each 'page_rows' positions
  int max_pages, page_rows;    // (page_rows a multiple of 128, so that a key tile lies in one page)
  long long k_rows, q_rows;    // rows of the key and query tensor maps (DSA_CHECKS builds check the loads)
  unsigned* hist;              // kModeDecode: [B, 2048] counts of the top 11 order-key bits of each sequence's
                               // scores, accumulated (zeroed by the caller), or null
};

struct IndexerItem {
  int q_row0;         // first query row of the item
  int n_tok;          // valid query rows in the item
  int pos0;           // absolute position of the item's first query row
  int tile0, tile1;   // key tile range [tile0, tile1)
  int n_keys;         // keys s < n_keys exist
  long long key_row0; // tensor-map row of key 0 (flat layouts)
  const int* pages;   // paged decode caches: the sequence's page-table row, else null
  int page_rows;
  long long out_base; // output offset of (first row, key 0)
  long long ld;       // row stride of the scores (kModeScores, kModeSegments)
};

// tensor-map row of key tile*128 + i of an item (i < 128)
__device__ __forceinline__ long long key_row(const IndexerItem& it, int tile, int i) {
  if (!it.pages) return it.key_row0 + static_cast<long long>(tile) * 128 + i;
  const int pos = tile * 128;
  return static_cast<long long>(it.pages[pos / it.page_rows]) * it.page_rows + pos % it.page_rows + i;
}

constexpr int kMaxDecodeSeqs = 1024;

template <int H_I, int D_I, int NT, int NG, int QBUF, int KSTAGES, int EPI_WG, int MODE>
struct IndexerCfg {
  static constexpr int N = NT * H_I;                 // MMA N
  static constexpr int TOK = NT * NG;                // query rows per item
  static constexpr int GBYTES = N * D_I;             // one group of q_I rows
  static constexpr int KBYTES = 128 * D_I;           // one key tile
  static constexpr int NUM_EPI_WARPS = 4 * EPI_WG;
  // CTAs per SM the launch relies on (decode: two, so that two sequences' chunks share an SM)
  static constexpr int CTAS_PER_SM = (MODE == kModeDecode) ? 2 : 1;
  static constexpr int ALIGN = 1024;
  // shared memory map (offsets from a 1024-byte aligned base)
  static constexpr int OFF_BAR = 0;                  // barriers + misc (2 KB)
  static constexpr int OFF_PREFIX = 2048;            // decode: per-sequence item prefix, key counts, cache offsets
  static constexpr int DEC_BYTES = 4 * (kMaxDecodeSeqs + 1) + 4 * kMaxDecodeSeqs + 8 * kMaxDecodeSeqs + 8;
  static constexpr int OFF_W = ((OFF_PREFIX + (MODE != kModeScores ? DEC_BYTES : 0) + 15) / 16) * 16;
  static constexpr int W_FLOATS = TOK * H_I;
  // decode: the CTA's histogram of its current item's scores (top 11 order-key bits), flushed to IndexerParams::hist
  static constexpr int OFF_HIST = OFF_W + QBUF * W_FLOATS * 4;
  static constexpr int HIST_BYTES = (MODE == kModeDecode) ? 2048 * 4 : 0;
  static constexpr int OFF_Q = ((OFF_HIST + HIST_BYTES + ALIGN - 1) / ALIGN) * ALIGN;
  static constexpr int OFF_K = OFF_Q + QBUF * NG * GBYTES;
  static constexpr int SMEM = OFF_K + KSTAGES * KBYTES + ALIGN;  // + alignment slack
  // accumulator ring: as many N-column accumulators as tensor memory holds (2 at N = 256), so that the MMAs
  // run that many (token group, key tile) steps ahead of the epilogue; decode keeps half of tensor memory
  // (4 x 64 columns) so that two CTAs share an SM
  static constexpr int NACC = (MODE == kModeDecode) ? 4 : ((512 / N) < 8 ? (512 / N) : 8);
  static constexpr uint32_t TMEM_COLS = static_cast<uint32_t>(NACC * N);
  // two epilogue warpgroups on alternate accumulator stages (H_I = 64 with two accumulators), each reading all N
  // columns of its stages; otherwise each warpgroup reads a column half of every stage
  static constexpr bool ALT_STAGES = (H_I == 64) && (EPI_WG == 2) && (NACC % 2 == 0) && ((N / EPI_WG) % 64 == 0);
  static constexpr int ACC_READERS = ALT_STAGES ? NUM_EPI_WARPS / 2 : NUM_EPI_WARPS;   // arrivals per stage
  // warps: 0 TMA producer, 1 MMA issue, EPI_WARP0.. the epilogue
  static constexpr int EPI_WARP0 = 2;
  static constexpr int NUM_THREADS = 32 * (EPI_WARP0 + NUM_EPI_WARPS);
  static_assert(TMEM_COLS == 256 || TMEM_COLS == 512, "tensor-memory allocation (power of two)");
  static constexpr uint32_t SW_LAYOUT = (D_I == 128) ? kLayoutSW128 : kLayoutSW64;
  static constexpr uint32_t SBO = (D_I == 128) ? 1024 : 512;
  static_assert(N <= 256 && N % 16 == 0, "MMA N");
  // the SM's 228 KB of shared memory, less 1 KB reserved per CTA, holds CTAS_PER_SM of them
  static_assert(CTAS_PER_SM * (SMEM + 1024) <= 228 * 1024, "CTAs per SM");
  static_assert(OFF_W % 16 == 0 && (W_FLOATS * 4) % 16 == 0, "head weights are read as 16-byte quads");
  static_assert(D_I == 128 || D_I == 64, "d_I");
  static_assert((N / EPI_WG) % H_I == 0 || H_I > N / EPI_WG, "epilogue column split");
};

// barrier slots (8 bytes each) in the barrier area
template <int QBUF, int KSTAGES, int NACC>
struct IndexerBars {
  static constexpr int Q_FULL = 0;
  static constexpr int Q_EMPTY = Q_FULL + QBUF;
  static constexpr int K_FULL = Q_EMPTY + QBUF;
  static constexpr int K_EMPTY = K_FULL + KSTAGES;
  static constexpr int ACC_FULL = K_EMPTY + KSTAGES;
  static constexpr int ACC_EMPTY = ACC_FULL + NACC;
  static constexpr int COUNT = ACC_EMPTY + NACC;
  static constexpr int OFF_TMEM = 8 * COUNT;         // u32: TMEM base address
  static constexpr int OFF_ABORT = OFF_TMEM + 4;     // int: abort flag
  static constexpr int OFF_NITEMS = OFF_TMEM + 8;    // int: key tiles of all sequences (decode)
  // DSA_CHECKS: ints [key tiles loaded, key tiles consumed by MMAs, accumulator stages committed, stage reads]
  static constexpr int OFF_CHECK = OFF_NITEMS + 4;
  static_assert(OFF_CHECK + 16 <= 2048, "barrier area");
};

// decode: the key-tile range [lo, hi) of this CTA over the tiles of all sequences laid end to end
struct TileRange {
  int lo, hi;
};

template <int MODE, int TOK>
__device__ __forceinline__ IndexerItem indexer_item(const IndexerParams& p, int i, const int* prefix,
                                                    TileRange tr) {
  IndexerItem it;
  if constexpr (MODE == kModeScores) {
    const int qb = i / p.nsplit, sp = i % p.nsplit;
    it.q_row0 = qb * TOK;
    it.n_tok = min(TOK, p.T - it.q_row0);
    it.pos0 = p.pos0 + it.q_row0;
    it.n_keys = p.S;
    it.key_row0 = 0;
    it.pages = nullptr;
    it.page_rows = 0;
    const int ntiles = (p.S + 127) / 128;
    it.tile0 = sp * p.split_tiles;
    it.tile1 = min(it.tile0 + p.split_tiles, ntiles);
    it.out_base = static_cast<long long>(it.q_row0) * p.ld;
    it.ld = p.ld;
  } else if constexpr (MODE == kModeSegments) {
    // binary search: prefix[sg] <= i < prefix[sg + 1] (prefix[sg] = the segment's first item)
    int lo = 0, hi = p.n_segs - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (prefix[mid] <= i) lo = mid; else hi = mid - 1;
    }
    const IndexerSeg sg = p.segs[lo];
    const int li = i - prefix[lo];
    const int qb = li / sg.nsplit, sp = li % sg.nsplit;
    it.q_row0 = static_cast<int>(sg.q_row0) + qb * TOK;
    it.n_tok = min(TOK, sg.n_rows - qb * TOK);
    it.pos0 = sg.pos0 + qb * TOK;
    it.n_keys = sg.S;
    it.key_row0 = sg.key_row0;
    it.pages = nullptr;
    it.page_rows = 0;
    const int ntiles = (sg.S + 127) / 128;
    it.tile0 = sp * p.split_tiles;
    it.tile1 = min(it.tile0 + p.split_tiles, ntiles);
    it.out_base = sg.out_base + static_cast<long long>(qb * TOK) * sg.ld;
    it.ld = sg.ld;
  } else {
    // item i is sequence b = i, clipped to the CTA's tile range (prefix[b] = its first tile in the joint order)
    const int b = i;
    const int* n1s = prefix + kMaxDecodeSeqs + 1;
    const long long* offs = reinterpret_cast<const long long*>(n1s + kMaxDecodeSeqs + 1);   // 8-byte aligned
    const int n = n1s[b];
    it.q_row0 = b;
    it.n_tok = 1;
    it.pos0 = n - 1;
    it.n_keys = n;
    it.key_row0 = offs[b];
    it.pages = p.page_table ? p.page_table + static_cast<long long>(b) * p.max_pages : nullptr;
    it.page_rows = p.page_rows;
    it.tile0 = max(tr.lo, prefix[b]) - prefix[b];
    it.tile1 = min(tr.hi, prefix[b + 1]) - prefix[b];
    it.out_base = p.score_off[b];
    it.ld = 0;
  }
  return it;
}

// last query position covered by group g of the item (or -1 when the group has no valid row)
template <int NT>
__device__ __forceinline__ int group_last_pos(const IndexerItem& it, int g) {
  if (g * NT >= it.n_tok) return -1;
  return it.pos0 + min(it.n_tok, (g + 1) * NT) - 1;
}
template <int NT>
__device__ __forceinline__ bool group_active(const IndexerItem& it, int tile, int g) {
  return tile * 128 < it.n_keys && tile * 128 <= group_last_pos<NT>(it, g);
}
__device__ __forceinline__ bool tile_active(const IndexerItem& it, int tile) {
  return tile * 128 < it.n_keys && tile * 128 <= it.pos0 + it.n_tok - 1;
}

template <int H_I, int D_I, int NT, int NG, int QBUF, int KSTAGES, int EPI_WG, int MODE>
__global__ void __launch_bounds__(IndexerCfg<H_I, D_I, NT, NG, QBUF, KSTAGES, EPI_WG, MODE>::NUM_THREADS,
                                  IndexerCfg<H_I, D_I, NT, NG, QBUF, KSTAGES, EPI_WG, MODE>::CTAS_PER_SM)
indexer_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
               const IndexerParams p) {
  using C = IndexerCfg<H_I, D_I, NT, NG, QBUF, KSTAGES, EPI_WG, MODE>;
  using Bars = IndexerBars<QBUF, KSTAGES, C::NACC>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + C::ALIGN - 1) &
                                             ~static_cast<uintptr_t>(C::ALIGN - 1));
  const uint32_t sbase = smem_u32(smem);
  auto bar = [&](int slot) -> uint32_t { return sbase + C::OFF_BAR + 8 * slot; };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Bars::OFF_ABORT);
  int* prefix = reinterpret_cast<int*>(smem + C::OFF_PREFIX);
  float* w_s = reinterpret_cast<float*>(smem + C::OFF_W);
  const uint32_t q_s = sbase + C::OFF_Q;
  const uint32_t k_s = sbase + C::OFF_K;
  const int warp = warp_id(), lane = lane_id();

  if (threadIdx.x == 0) {
    for (int i = 0; i < QBUF; ++i) { mbar_init(bar(Bars::Q_FULL + i), 1); mbar_init(bar(Bars::Q_EMPTY + i), 1); }
    for (int i = 0; i < KSTAGES; ++i) { mbar_init(bar(Bars::K_FULL + i), 1); mbar_init(bar(Bars::K_EMPTY + i), 1); }
    for (int i = 0; i < C::NACC; ++i) {
      mbar_init(bar(Bars::ACC_FULL + i), 1);
      mbar_init(bar(Bars::ACC_EMPTY + i), C::ACC_READERS);
    }
    *abort_flag = 0;
    if constexpr (kChecks) {
      for (int i = 0; i < 4; ++i) reinterpret_cast<int*>(smem + Bars::OFF_CHECK)[i] = 0;
    }
    fence_mbar_init();
  }
  pdl_allow_next();
  pdl_wait();
  if constexpr (MODE == kModeDecode) {
    // per sequence: keys n_b + 1, cache offset and key tiles, loaded by all threads in parallel; then an
    // exclusive scan of the tile counts by warp 0 (tiles of sequence b are prefix[b] .. prefix[b + 1] - 1 in the
    // joint order)
    int* n1s = prefix + kMaxDecodeSeqs + 1;
    long long* offs = reinterpret_cast<long long*>(n1s + kMaxDecodeSeqs + 1);
    int* cnts = prefix + 1;          // counts first, scanned in place below
    for (int b = threadIdx.x; b < p.T; b += blockDim.x) {
      const int n1 = p.len1[b];
      n1s[b] = n1;
      offs[b] = p.cache_off ? p.cache_off[b] : 0;     // paged caches: rows come from the page table
      cnts[b] = (n1 + 127) / 128;
    }
    __syncthreads();
    if (warp == 0) {
      int carry = 0;
      for (int b0 = 0; b0 < p.T; b0 += 32) {
        const int b = b0 + lane;
        const int c = (b < p.T) ? cnts[b] : 0;
        int incl = c;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
          const int v = __shfl_up_sync(0xffffffffu, incl, d);
          if (lane >= d) incl += v;
        }
        __syncwarp();
        if (b < p.T) prefix[b + 1] = carry + incl;    // cnts[b] aliases prefix[b + 1]: read before written
        carry += __shfl_sync(0xffffffffu, incl, 31);
        __syncwarp();
      }
      if (lane == 0) {
        prefix[0] = 0;
        *reinterpret_cast<int*>(smem + Bars::OFF_NITEMS) = carry;
      }
    }
  }
  if constexpr (MODE == kModeSegments) {
    for (int sgi = threadIdx.x; sgi < p.n_segs; sgi += blockDim.x) prefix[sgi] = p.segs[sgi].item0;
  }
  if (warp == 0 && lane == 0) { prefetch_tmap(&tm_q); prefetch_tmap(&tm_k); }
  if (warp == 1) {
    tmem_alloc(sbase + Bars::OFF_TMEM, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *reinterpret_cast<volatile uint32_t*>(smem + Bars::OFF_TMEM);
  // The CTA's items.  kModeScores: items blockIdx.x, + gridDim.x, ... below p.n_items.  kModeDecode: the
  // sequences whose tiles meet the CTA's range [lo, hi), skipping those without keys (every role walks the same
  // list, which must hold no empty item: each item loads its queries once).
  TileRange tr{0, 0};
  if constexpr (MODE == kModeDecode) {
    const long long tot = *reinterpret_cast<volatile int*>(smem + Bars::OFF_NITEMS);
    tr.lo = static_cast<int>(tot * blockIdx.x / gridDim.x);
    tr.hi = static_cast<int>(tot * (blockIdx.x + 1) / gridDim.x);
  }
  auto first_item = [&]() -> int {
    if constexpr (MODE == kModeDecode) {
      // the last sequence starting at or before lo: it holds tile lo (when lo < hi)
      int lo = 0, hi = p.T - 1;
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (prefix[mid] <= tr.lo) lo = mid; else hi = mid - 1;
      }
      return lo;
    } else {
      return static_cast<int>(blockIdx.x);
    }
  };
  auto has_item = [&](int i) -> bool {
    if constexpr (MODE == kModeDecode) return i < p.T && prefix[i] < tr.hi;
    else return i < p.n_items;
  };
  auto next_item = [&](int i) -> int {
    if constexpr (MODE == kModeDecode) {
      ++i;
      while (i < p.T && prefix[i + 1] == prefix[i]) ++i;     // sequences without keys
      return i;
    } else {
      return i + static_cast<int>(gridDim.x);
    }
  };

  // decode with a histogram: the sequence whose counts sit in the CTA's shared histogram, flushed when the next
  // item starts and at the end of the kernel (epilogue threads)
  [[maybe_unused]] int hist_b = -1;
  if (warp < C::EPI_WARP0) {
    if (warp == 0) {
      // ------------------------------------------------------------------ TMA producer
      if (lane == 0) {
        Pipe<KSTAGES> kp;
        int k_issued = 0;                 // k tiles issued so far
        int q_issued[QBUF] = {};          // per q buffer: loads issued
        uint32_t q_par[QBUF] = {};        // per q buffer: parity of its last load
        int qi = 0;
        bool ok = true;
        for (int item = first_item(); has_item(item) && ok; item = next_item(item), ++qi) {
          const IndexerItem it = indexer_item<MODE, C::TOK>(p, item, prefix, tr);
          const int qb = qi % QBUF;
          const uint32_t qph = (qi / QBUF) & 1;
          if (!mbar_wait(bar(Bars::Q_EMPTY + qb), qph ^ 1, abort_flag)) { ok = false; break; }
          mbar_arrive_expect_tx(bar(Bars::Q_FULL + qb), NG * C::GBYTES);
          for (int g = 0; g < NG; ++g) {
            check_that(it.q_row0 + g * NT < p.q_rows || g * NT >= it.n_tok);
            tma_load_2d(q_s + (qb * NG + g) * C::GBYTES, &tm_q, bar(Bars::Q_FULL + qb), 0,
                        (it.q_row0 + g * NT) * H_I);
          }
          q_issued[qb] += 1;
          q_par[qb] = qph;
          for (int tile = it.tile0; tile < it.tile1; ++tile) {
            if (!tile_active(it, tile)) continue;
            // the tile's row (a page-table load with paged caches) is looked up before the wait, so that the
            // load's latency overlaps it instead of delaying the copy
            const long long krow = key_row(it, tile, 0);
            if (!mbar_wait(bar(Bars::K_EMPTY + kp.stage), kp.phase ^ 1, abort_flag)) { ok = false; break; }
            mbar_arrive_expect_tx(bar(Bars::K_FULL + kp.stage), C::KBYTES);
            check_that(krow >= 0 && krow < p.k_rows);
            if constexpr (MODE == kModeDecode) {
              // the key cache streams through once per step: its lines go first, so that the score rows the
              // top-k reads next stay in L2
              tma_load_2d_hint(k_s + kp.stage * C::KBYTES, &tm_k, bar(Bars::K_FULL + kp.stage), 0,
                               static_cast<int>(krow), l2_policy_evict_first());
            } else {
              tma_load_2d(k_s + kp.stage * C::KBYTES, &tm_k, bar(Bars::K_FULL + kp.stage), 0, static_cast<int>(krow));
            }
            kp.advance();
            ++k_issued;
          }
        }
        if constexpr (kChecks) reinterpret_cast<int*>(smem + Bars::OFF_CHECK)[0] = k_issued;
        if (*abort_flag) {
          // leave no TMA write in flight into this CTA's shared memory: wait (bounded) for the last load
          // issued on every k stage and q buffer
          for (int st = 0; st < KSTAGES && st < k_issued; ++st)
            mbar_wait_drain(bar(Bars::K_FULL + st), st < kp.stage ? kp.phase : kp.phase ^ 1);
          for (int b = 0; b < QBUF; ++b)
            if (q_issued[b]) mbar_wait_drain(bar(Bars::Q_FULL + b), q_par[b]);
        }
      }
    } else if (warp == 1) {
      // ------------------------------------------------------------------ MMA issue
      if (lane == 0) {
        Pipe<KSTAGES> kp;
        Pipe<C::NACC> ap;
        constexpr uint32_t idesc = idesc_e4m3(128, C::N);
        int qi = 0;
        bool ok = true;
        [[maybe_unused]] int chk_tiles = 0, chk_stages = 0;
        for (int item = first_item(); has_item(item) && ok; item = next_item(item), ++qi) {
          const IndexerItem it = indexer_item<MODE, C::TOK>(p, item, prefix, tr);
          const int qb = qi % QBUF;
          if (!mbar_wait(bar(Bars::Q_FULL + qb), (qi / QBUF) & 1, abort_flag)) { ok = false; break; }
          tc_fence_after();
          for (int tile = it.tile0; tile < it.tile1 && ok; ++tile) {
            if (!tile_active(it, tile)) continue;
            if (!mbar_wait(bar(Bars::K_FULL + kp.stage), kp.phase, abort_flag)) { ok = false; break; }
            tc_fence_after();
            const uint64_t adesc = smem_desc(k_s + kp.stage * C::KBYTES, 16, C::SBO, C::SW_LAYOUT);
            for (int g = 0; g < NG; ++g) {
              if (!group_active<NT>(it, tile, g)) continue;
              if (!mbar_wait(bar(Bars::ACC_EMPTY + ap.stage), ap.phase ^ 1, abort_flag)) { ok = false; break; }
              tc_fence_after();
              const uint64_t bdesc = smem_desc(q_s + (qb * NG + g) * C::GBYTES, 16, C::SBO, C::SW_LAYOUT);
              const uint32_t d = tmem_base + ap.stage * C::N;
#pragma unroll
              for (int kk = 0; kk < D_I / 32; ++kk)   // K = 32 e4m3 (32 bytes) per instruction
                mma_f8_ss(d, adesc + 2 * kk, bdesc + 2 * kk, idesc, kk > 0 ? 1u : 0u);
              mma_commit(bar(Bars::ACC_FULL + ap.stage));
              ap.advance();
              if constexpr (kChecks) ++chk_stages;
            }
            mma_commit(bar(Bars::K_EMPTY + kp.stage));
            kp.advance();
            if constexpr (kChecks) ++chk_tiles;
          }
          mma_commit(bar(Bars::Q_EMPTY + qb));
        }
        if constexpr (kChecks) {
          reinterpret_cast<int*>(smem + Bars::OFF_CHECK)[1] = chk_tiles;
          reinterpret_cast<int*>(smem + Bars::OFF_CHECK)[2] = chk_stages;
        }
      }
    }
  } else {
    // ------------------------------------------------------------------ epilogue
    // Alternate stages (C::ALT_STAGES): warpgroup h reads the accumulator stages of parity h, all N columns.  The
    // two warps sharing a sub-partition then work on different stages, and one computes while the other waits
    // for its tensor-memory loads; with a column half each, both waited at the same moments and left the
    // sub-partition idle.
    constexpr int CPT = C::ALT_STAGES ? C::N : C::N / EPI_WG;   // accumulator columns per thread and stage
    constexpr int TOKS = (CPT >= H_I) ? CPT / H_I : 1;  // query rows per thread
    constexpr int INF_TOKS = (NT / EPI_WG > 0) ? NT / EPI_WG : 1;   // rows of a skipped group per thread
    // Packed epilogue (heads in pairs): w ReLU(x) is formed as w max(x, 0) for even heads (ALU pipe)
    // and as (w / 2)(x + |x|) for odd heads (FMA pipe, |x| as an operand modifier), so that the two pipes share
    // the ReLUs; the odd heads' weights are stored halved.  Both forms are exact for integer-valued inputs.
    constexpr bool kPacked = (H_I == 64) && ((C::N / EPI_WG) % 64 == 0);
    constexpr int P = kPacked ? 1 : ((H_I >= 16) ? 4 : 1);   // partial sums per row (ILP)
    // Fragment reads (kPacked): the accumulator is read in 16-lane x 256-bit fragments, so that a thread holds
    // four keys (lanes g, g + 8, g + 16, g + 24 of its warp's 32, g = lane / 4) and, of every eight columns, the
    // two columns 2c, 2c + 1 (c = lane % 4).  Each head weight a thread loads then serves four keys (the sixteen
    // weights of its heads lie together: four 16-byte loads per token), where per-key reads (one key per thread)
    // broadcast every weight to the whole warp.  Each thread sums its sixteen heads of a token, and two shuffle rounds
    // (lane ^ 1, lane ^ 2) add the four partial sums of a key, leaving thread (g, c) with key
    // g + 8 (c >> 1) + 16 (c & 1).
    const int e = warp - C::EPI_WARP0;
    const int quad = warp & 3;
    const int half = e >> 2;
    const int ethreads = 32 * C::NUM_EPI_WARPS;
    const int etid = e * 32 + lane;
    const uint32_t lane_addr = static_cast<uint32_t>(quad * 32) << 16;
    const int fc = lane & 3, fg = lane >> 2;        // fragment column pair and row (kPacked)
    const int key_lane = kPacked ? fg + 8 * (fc >> 1) + 16 * (fc & 1) : lane;   // this thread's key in the warp
    Pipe<C::NACC> ap;
    int qi = 0;
    bool ok = true;
    [[maybe_unused]] int chk_reads = 0;    // accumulator stages this warp read (DSA_CHECKS)
    for (int item = first_item(); has_item(item) && ok; item = next_item(item), ++qi) {
      const IndexerItem it = indexer_item<MODE, C::TOK>(p, item, prefix, tr);
      float* wq = w_s + (qi % QBUF) * C::W_FLOATS;
      named_bar_sync(1, ethreads);
      for (int i = etid; i < C::W_FLOATS; i += ethreads) {
        const int r = i / H_I, j = i % H_I;
        float v = 0.f;
        if (r < it.n_tok) {
          v = p.w[static_cast<long long>(it.q_row0 + r) * H_I + j];
          if (p.q_scale) v *= p.q_scale[it.q_row0 + r];
          if (kPacked && (j & 1)) v *= 0.5f;
        }
        // kPacked: head j = 8m + 2c + e goes to 16c + 2m + e, so that the sixteen weights of fragment column
        // pair c lie together (four 16-byte loads per token)
        wq[kPacked ? r * H_I + 16 * ((j >> 1) & 3) + 2 * (j >> 3) + (j & 1) : i] = v;
      }
      if constexpr (MODE == kModeDecode) {
        if (p.hist) {
          // each thread owns the same bins in every item: it flushes the previous item's counts and clears them
          unsigned* hs = reinterpret_cast<unsigned*>(smem + C::OFF_HIST);
          for (int i = etid; i < 2048; i += ethreads) {
            const unsigned v = hs[i];
            if (hist_b >= 0 && v) atomicAdd(p.hist + static_cast<long long>(hist_b) * 2048 + i, v);
            hs[i] = 0;
          }
          hist_b = it.q_row0;
        }
      }
      named_bar_sync(1, ethreads);
      // key scales are loaded ahead of their tile: a load issued at the start of its own tile would expose the
      // global-memory latency once per tile (the epilogue needs it a few hundred cycles later).  One tile ahead
      // in prefill; two in decode, whose tiles take about half a microsecond and whose paged caches put a
      // page-table load before the scale's.
      constexpr int KS_AHEAD = (MODE == kModeDecode) ? 2 : 1;
      auto kscale_of = [&](int tile) -> float {
        const int s = tile * 128 + quad * 32 + key_lane;
        return (p.k_scale && tile < it.tile1 && s < it.n_keys) ? p.k_scale[key_row(it, tile, quad * 32 + key_lane)]
                                                                : 1.f;
      };
      float kscale_ahead[KS_AHEAD];
#pragma unroll
      for (int a = 0; a < KS_AHEAD; ++a) kscale_ahead[a] = kscale_of(it.tile0 + a);
      for (int tile = it.tile0; tile < it.tile1; ++tile) {
        const int s = tile * 128 + quad * 32 + key_lane;      // key of this thread
        const bool key_ok = s < it.n_keys;
        const float kscale = kscale_ahead[0];
#pragma unroll
        for (int a = 0; a + 1 < KS_AHEAD; ++a) kscale_ahead[a] = kscale_ahead[a + 1];
        kscale_ahead[KS_AHEAD - 1] = kscale_of(tile + KS_AHEAD);
        for (int g = 0; g < NG; ++g) {
          if (g * NT >= it.n_tok) break;
          if (!group_active<NT>(it, tile, g)) {
            if constexpr (MODE != kModeDecode) {
              if (key_ok) {
#pragma unroll
                for (int tk = 0; tk < INF_TOKS; ++tk) {
                  const int r = g * NT + half * INF_TOKS + tk;
                  if (r < it.n_tok) p.scores[it.out_base + static_cast<long long>(r) * it.ld + s] = -INFINITY;
                }
              }
            }
            continue;
          }
          if (C::ALT_STAGES && (ap.stage & 1) != half) {   // the other warpgroup's stage
            ap.advance();
            continue;
          }
          // first row of this thread
          const int tok0 = g * NT + (C::ALT_STAGES ? 0 : half * (CPT / H_I > 0 ? CPT / H_I : 0));
          if (!mbar_wait(bar(Bars::ACC_FULL + ap.stage), ap.phase, abort_flag)) { ok = false; break; }
          tc_fence_after();
          float acc[TOKS][P];
#pragma unroll
          for (int tk = 0; tk < TOKS; ++tk)
#pragma unroll
            for (int q = 0; q < P; ++q) acc[tk][q] = 0.f;
          const uint32_t tcol = tmem_base + ap.stage * C::N + (C::ALT_STAGES ? 0 : half * CPT);
          if constexpr (kPacked) {
            // Chunks of 64 columns (one token) x 16 lanes: c = 2 * token + lane half.  A tcgen05.wait::ld waits for
            // every load in flight, so a load is hidden only behind the arithmetic done between its issue and the
            // next wait.  One chunk is loaded per chunk computed, LEAD chunks ahead, and the warp waits once per
            // SPAN chunks (a ring of LEAD + SPAN register buffers).  Two loads issued back to back, with no
            // arithmetic between them, ran far slower.
            constexpr int NCH = 2 * TOKS;
            constexpr int SPAN = C::ALT_STAGES ? 2 : 1;
            constexpr int LEAD = 2;
            constexpr int RD = LEAD + SPAN;
            uint64_t acc2[4];           // the current token: [key slot 2 * half + (row g: 0, row g + 8: 1)]
            auto chunk_addr = [&](int c) -> uint32_t {
              return lane_addr + (static_cast<uint32_t>(16 * (c & 1)) << 16) + tcol + 64 * (c >> 1);
            };
            uint32_t v[RD][32];
#pragma unroll
            for (int c = 0; c < LEAD && c < NCH; ++c) tmem_ld16x256_x8(chunk_addr(c), v[c]);
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < LEAD && c < NCH; ++c) tmem_regs_after_wait(v[c]);
            uint64_t ww[8];             // (w[8m + 2c], w[8m + 2c + 1] / 2) of the current token
            const bool odd1 = (fc & 1) != 0, odd2 = (fc & 2) != 0;
#pragma unroll
            for (int c = 0; c < NCH; ++c) {
              if (c + LEAD < NCH) tmem_ld16x256_x8(chunk_addr(c + LEAD), v[(c + LEAD) % RD]);
              const int tk = c >> 1, hl = c & 1;
              if (hl == 0) {
                const ulonglong2* wp = reinterpret_cast<const ulonglong2*>(wq + (tok0 + tk) * H_I + 16 * fc);
#pragma unroll
                for (int m = 0; m < 8; m += 2) {
                  const ulonglong2 q2 = wp[m >> 1];
                  ww[m] = q2.x;
                  ww[m + 1] = q2.y;
                }
              }
#pragma unroll
              for (int m = 0; m < 8; ++m) {
#pragma unroll
                for (int r = 0; r < 2; ++r) {
                  const float x0 = __uint_as_float(v[c % RD][4 * m + 2 * r]);
                  const float x1 = __uint_as_float(v[c % RD][4 * m + 2 * r + 1]);
                  const uint64_t a2 = pack_f32x2(fmaxf(x0, 0.f), x1 + fabsf(x1));
                  acc2[2 * hl + r] = (m == 0) ? mul_f32x2(ww[m], a2) : fma_f32x2(ww[m], a2, acc2[2 * hl + r]);
                }
              }
              if (hl == 1) {
                // the four partial sums of a key: lane ^ 1 trades lane halves, then lane ^ 2 trades rows g / g + 8
                float sm[4];
#pragma unroll
                for (int ks = 0; ks < 4; ++ks) {
                  float lo, hi;
                  unpack_f32x2(acc2[ks], lo, hi);
                  sm[ks] = lo + hi;
                }
                float t1[2];
#pragma unroll
                for (int r = 0; r < 2; ++r) {
                  const float keep = odd1 ? sm[2 + r] : sm[r];
                  const float send = odd1 ? sm[r] : sm[2 + r];
                  t1[r] = keep + __shfl_xor_sync(0xffffffffu, send, 1);
                }
                const float keep = odd2 ? t1[1] : t1[0];
                const float send = odd2 ? t1[0] : t1[1];
                acc[tk][0] = keep + __shfl_xor_sync(0xffffffffu, send, 2);
              }
              if (c % SPAN == SPAN - 1 && c + 1 - SPAN + LEAD < NCH) {   // loads issued since the last wait
                tmem_wait_ld_after(acc2[2 * hl], acc2[2 * hl + 1], acc[tk][0]);
#pragma unroll
                for (int b = 0; b < SPAN; ++b)
                  if (c + 1 - SPAN + LEAD + b < NCH) tmem_regs_after_wait(v[(c + 1 - SPAN + LEAD + b) % RD]);
              }
            }
          } else {
#pragma unroll
            for (int c0 = 0; c0 < CPT; c0 += 64) {
              uint32_t v0[32], v1[32];
              tmem_ld32(lane_addr + tcol + c0, v0);
              if (c0 + 32 < CPT) tmem_ld32(lane_addr + tcol + c0 + 32, v1);
              tmem_wait_ld();
#pragma unroll
              for (int i = 0; i < 64; ++i) {
                if (c0 + i >= CPT) break;
                const int col = c0 + i;
                const int tk = col / H_I, j = col % H_I;
                const float x = __uint_as_float(i < 32 ? v0[i] : v1[i - 32]);
                acc[tk][j % P] = fmaf(wq[(tok0 + tk) * H_I + j], fmaxf(x, 0.f), acc[tk][j % P]);
              }
            }
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(bar(Bars::ACC_EMPTY + ap.stage));
          ap.advance();
          if constexpr (kChecks) ++chk_reads;
          if (key_ok) {
#pragma unroll
            for (int tk = 0; tk < TOKS; ++tk) {
              const int r = tok0 + tk;
              if (r >= it.n_tok) continue;
              float sc = 0.f;
#pragma unroll
              for (int q = 0; q < P; ++q) sc += acc[tk][q];
              sc *= kscale;
              if constexpr (MODE != kModeDecode) {
                p.scores[it.out_base + static_cast<long long>(r) * it.ld + s] = (s <= it.pos0 + r) ? sc : -INFINITY;
              } else {
                p.scores[it.out_base + s] = sc;
                if (p.hist) atomicAdd(reinterpret_cast<unsigned*>(smem + C::OFF_HIST) + (order_key(sc) >> 21), 1u);
              }
            }
          }
        }
        if (!ok) break;
      }
    }
    if constexpr (kChecks) {
      if (lane == 0) atomicAdd(reinterpret_cast<int*>(smem + Bars::OFF_CHECK) + 3, chk_reads);
    }
  }

  // ------------------------------------------------------------------ teardown
  tc_fence_before();
  __syncthreads();
  if constexpr (MODE == kModeDecode) {
    if (p.hist && hist_b >= 0 && !*abort_flag) {      // the last item's counts (hist_b is set in epilogue threads)
      const unsigned* hs = reinterpret_cast<const unsigned*>(smem + C::OFF_HIST);
      for (int i = threadIdx.x - 32 * C::EPI_WARP0; i < 2048; i += 32 * C::NUM_EPI_WARPS) {
        const unsigned v = hs[i];
        if (v) atomicAdd(p.hist + static_cast<long long>(hist_b) * 2048 + i, v);
      }
    }
  }
  if constexpr (kChecks) {
    // every key tile loaded went through the MMAs, and every accumulator stage committed was read by the
    // ACC_READERS epilogue warps that take it (a wait that ran out has already recorded DSA_ERR_TIMEOUT)
    const int* chk = reinterpret_cast<const int*>(smem + Bars::OFF_CHECK);
    if (threadIdx.x == 0 && !*abort_flag) check_that(chk[0] == chk[1] && chk[3] == chk[2] * C::ACC_READERS);
  }
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

}  // namespace dsa
