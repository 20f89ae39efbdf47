// libdsa.so: C ABI of the DSA forward path on B200 (declarations and contracts in include/dsa.h).
//
// Host side only: argument checks, TMA tensor-map construction, launch configuration and the order of the
// kernels of the prefill and decode drivers.  Every step of the computation runs in the kernels included
// below.
#include <cmath>
#include <cstdint>
#include <cstdio>
#include <algorithm>
#include <atomic>
#include <mutex>
#include <vector>

#include "common.cuh"
#include "indexer.cuh"
#include "sparse_mla.cuh"
#include "topk.cuh"
#include "topk_cluster.cuh"

namespace dsa {

// ------------------------------------------------------------------------------------------ decode append
// Writes the new token's indexer key (+ scale) and latent entry at position ctx_len[b] of sequence b, n_b + 1
// into len1[b] (the number of keys the new token attends to) and the start of the sequence's score row into
// score_off[b].  Score rows are packed in sequence order, each padded to a multiple of 4 floats, so that every
// row starts on a 16-byte boundary (the top-k reads rows with 16-byte loads); they do not follow the cache
// layout.  A sequence whose cache range is invalid (cache_off < 0, ctx_len < 0, or the new row outside the
// cache) or whose score row would not fit in score_cap floats raises DSA_ERR_BAD_INDEX and gets len1 = 0: no
// kernel after this one reads or writes anything of it.

__device__ __forceinline__ bool decode_seq_valid(const long long* cache_off, const int* ctx_len,
                                                 long long cache_rows, int b) {
  const long long off = cache_off[b];
  const int n = ctx_len[b];
  return off >= 0 && n >= 0 && off + n < cache_rows;
}

// Paged caches: the caches are pools of pages of page_rows rows; row (page_table[b][pos / page_rows] * page_rows +
// pos % page_rows) holds position pos of sequence b.  A sequence is valid when its new position ctx_len[b] falls
// inside its table and every page up to it is in [0, num_pages).  Every thread of the CTA calls this.
__device__ __forceinline__ bool decode_seq_valid_paged(const int* page_table, int max_pages, int page_rows,
                                                       long long num_pages, const int* ctx_len, int b) {
  __shared__ int bad;
  const int n = ctx_len[b];
  if (threadIdx.x == 0) bad = (n < 0 || n / page_rows >= max_pages) ? 1 : 0;
  __syncthreads();
  if (!bad) {
    const int* row = page_table + static_cast<long long>(b) * max_pages;
    for (int j = threadIdx.x; j <= n / page_rows; j += blockDim.x)
      if (row[j] < 0 || row[j] >= num_pages) bad = 1;
  }
  __syncthreads();
  return bad == 0;
}

__device__ __forceinline__ long long padded4(long long n) { return (n + 3) & ~3ll; }

constexpr int kAppendThreads = 128;

// Cache layout of a decode step: flat (sequence b owns rows cache_off[b] ..) or paged (page_table non-null).
struct DecodeLayout {
  const long long* cache_off;   // flat: [B]
  long long cache_rows;         // flat: rows of the caches
  const int* page_table;        // paged: [B, max_pages], or null
  int max_pages, page_rows;
  long long num_pages;
};

__global__ void __launch_bounds__(kAppendThreads)
    decode_append_kernel(int B, DecodeLayout lay, const int* ctx_len, const uint8_t* k_new,
                         const float* k_scale_new, const uint16_t* c_new, uint8_t* k_cache, float* k_scale_cache,
                         uint16_t* c_cache, int d_I, int* len1, long long* score_off, long long score_cap,
                         unsigned* hist) {
  pdl_allow_next();
  pdl_wait();
  const int b = blockIdx.x;
  if (b >= B) return;
  // the sequence's score histogram, accumulated by the indexer (when the step uses one)
  if (hist)
    for (int i = threadIdx.x; i < kTopkBins; i += blockDim.x) hist[static_cast<long long>(b) * kTopkBins + i] = 0;
  // start of this sequence's score row: the padded lengths of the sequences before it that pass the cheap part
  // of their check (paged: the page-table entries of another sequence are not read here; a sequence that fails
  // only on those keeps its reserved row unused)
  __shared__ long long part[kAppendThreads / 32];
  long long acc = 0;
  for (int j = threadIdx.x; j < b; j += blockDim.x) {
    const int nj = ctx_len[j];
    if (lay.page_table ? (nj >= 0 && nj / lay.page_rows < lay.max_pages)
                       : decode_seq_valid(lay.cache_off, ctx_len, lay.cache_rows, j))
      acc += padded4(static_cast<long long>(nj) + 1);
  }
#pragma unroll
  for (int d = 16; d > 0; d >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, d);
  if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = acc;
  __syncthreads();
  long long s0 = 0;
#pragma unroll
  for (int w = 0; w < kAppendThreads / 32; ++w) s0 += part[w];
  const bool fits = s0 + padded4(static_cast<long long>(ctx_len[b]) + 1) <= score_cap;
  const bool valid = (lay.page_table ? decode_seq_valid_paged(lay.page_table, lay.max_pages, lay.page_rows,
                                                              lay.num_pages, ctx_len, b)
                                     : decode_seq_valid(lay.cache_off, ctx_len, lay.cache_rows, b)) && fits;
  if (!valid) {
    if (threadIdx.x == 0) { raise_status(DSA_ERR_BAD_INDEX); len1[b] = 0; score_off[b] = 0; }
    return;
  }
  const int n = ctx_len[b];
  const long long row = lay.page_table
      ? static_cast<long long>(lay.page_table[static_cast<long long>(b) * lay.max_pages + n / lay.page_rows]) *
            lay.page_rows + n % lay.page_rows
      : lay.cache_off[b] + n;
  const uint4* ks = reinterpret_cast<const uint4*>(k_new + static_cast<long long>(b) * d_I);
  uint4* kd = reinterpret_cast<uint4*>(k_cache + row * d_I);
  for (int i = threadIdx.x; i < d_I / 16; i += blockDim.x) kd[i] = ks[i];
  const uint4* cs = reinterpret_cast<const uint4*>(c_new + static_cast<long long>(b) * mla::D);
  uint4* cd = reinterpret_cast<uint4*>(c_cache + row * mla::D);
  for (int i = threadIdx.x; i < mla::D * 2 / 16; i += blockDim.x) cd[i] = cs[i];
  if (threadIdx.x == 0) {
    k_scale_cache[row] = k_scale_new[b];
    len1[b] = ctx_len[b] + 1;
    score_off[b] = s0;
  }
}

// ------------------------------------------------------------------------------------------ varlen prefill
// Row offset of every token of a packed batch of sequences: the first row of its own sequence (the largest b
// with cu[b] <= t, so an empty sequence never owns a token).
__global__ void varlen_row_off_kernel(const long long* cu, int nseq, long long total, long long* row_off) {
  const long long t = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (t >= total) return;
  int lo = 0, hi = nseq - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (cu[mid] <= t) lo = mid; else hi = mid - 1;
  }
  row_off[t] = cu[lo];
}

// Score-row offset and length of every row of a group of packed sequences for the top-k: row r of sequence b at
// position t reads the t + 1 scores at seq_off[b] + (t - k) * seq_ld[b] (rows t < k read nothing: every earlier key
// is selected).  cu: the group's sequence starts relative to its first row, nseq + 1 entries.
__global__ void varlen_score_rows_kernel(const long long* cu, int nseq, const long long* seq_off, const int* seq_ld,
                                         int k, long long* row_off, int* row_len) {
  pdl_allow_next();
  pdl_wait();
  const long long r = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (r >= cu[nseq]) return;
  int lo = 0, hi = nseq - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (cu[mid] <= r) lo = mid; else hi = mid - 1;
  }
  const long long t = r - cu[lo];
  row_len[r] = static_cast<int>(t + 1);
  row_off[r] = (t >= k) ? seq_off[lo] + (t - k) * seq_ld[lo] : 0;
}

// ------------------------------------------------------------------------------------------ bounded-wait self-check
// One CTA of two warps exercises the bounded mbarrier wait every pipeline of the library uses, on barriers
// that nothing arrives on.  Warp 0 waits from the start and runs out of budget (g_wait_limit cycles, about a
// second): it records DSA_ERR_TIMEOUT and raises the CTA's abort flag.  Warp 1 starts its wait half a budget
// later and must leave on the abort flag, well before its own budget ends.  result[2w] = 1 if warp w's wait
// succeeded, result[2w + 1] = its wait in units of 2^20 cycles.
__global__ void __launch_bounds__(64) wait_selfcheck_kernel(int* result) {
  __shared__ __align__(8) uint64_t bars[2];
  __shared__ int abort_flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bars[0]), 1);
    mbar_init(smem_u32(&bars[1]), 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (lane != 0) return;
  if (warp == 1) {
    const long long t0 = clock64();
    while (clock64() - t0 < (g_wait_limit >> 1)) {
    }
  }
  const long long t0 = clock64();
  const bool ok = mbar_wait(smem_u32(&bars[warp]), 0, &abort_flag);
  result[2 * warp] = ok ? 1 : 0;
  result[2 * warp + 1] = static_cast<int>((clock64() - t0) >> 20);
}

// ------------------------------------------------------------------------------------------ host helpers
namespace {

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// rank-2/3 tensor map; dims / strides innermost first (strides in bytes, rank-1 entries)
bool make_map(CUtensorMap* m, CUtensorMapDataType dt, int rank, const void* base, const cuuint64_t* dims,
              const cuuint64_t* strides, const cuuint32_t* box, CUtensorMapSwizzle sw) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint32_t es[3] = {1, 1, 1};
  return fn(m, dt, rank, const_cast<void*>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int num_sms() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
  return n;
}

template <typename K>
cudaError_t set_smem(K kernel, int bytes) {
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
}

std::atomic<unsigned long long> g_launches{0};

// Launch with programmatic stream serialisation (see pdl_wait): the kernel may be scheduled while its predecessor
// on the stream finishes, and waits for it on the device.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                       Args... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

dsa_status_t last_launch_status() {
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return cudaGetLastError() == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// floats of the decode score rows: every valid sequence's n_b + 1 keys, padded to a multiple of 4; sequences
// own disjoint cache ranges, so the rows need at most cache_rows + 3 B floats
size_t decode_score_cap(int B, int64_t cache_rows) { return size_t(cache_rows) + 4 * size_t(B); }

// ------------------------------------------------------------------------------------------ launchers
// A configuration that allocates all 512 TMEM columns runs one CTA per SM: at least 120 KB of shared memory is
// requested to keep a second CTA off the SM (its allocation would wait for the first CTA to finish).
constexpr int kMinIndexerSmem = 120 * 1024;

template <int H_I, int D_I, int NT, int NG, int QBUF, int KST, int EPI, int MODE>
dsa_status_t launch_indexer(const uint8_t* q_idx, int q_rows, const uint8_t* k_idx, long long k_rows,
                            const IndexerParams& p, int grid, cudaStream_t st) {
  using C = IndexerCfg<H_I, D_I, NT, NG, QBUF, KST, EPI, MODE>;
  CUtensorMap tq, tk;
  const cuuint64_t qd[2] = {static_cast<cuuint64_t>(D_I), static_cast<cuuint64_t>(q_rows) * H_I};
  const cuuint64_t qs[1] = {static_cast<cuuint64_t>(D_I)};
  const cuuint32_t qb[2] = {static_cast<cuuint32_t>(D_I), static_cast<cuuint32_t>(C::N)};
  const cuuint64_t kd[2] = {static_cast<cuuint64_t>(D_I), static_cast<cuuint64_t>(k_rows)};
  const cuuint32_t kb[2] = {static_cast<cuuint32_t>(D_I), 128u};
  const CUtensorMapSwizzle sw = (D_I == 128) ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
  if (!make_map(&tq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, q_idx, qd, qs, qb, sw)) return DSA_ERR_CUDA;
  if (!make_map(&tk, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, k_idx, kd, qs, kb, sw)) return DSA_ERR_CUDA;
  auto kern = indexer_kernel<H_I, D_I, NT, NG, QBUF, KST, EPI, MODE>;
  IndexerParams pk = p;
  pk.k_rows = k_rows;
  pk.q_rows = q_rows;
  const int smem = (C::TMEM_COLS == 512 && C::SMEM < kMinIndexerSmem) ? kMinIndexerSmem : C::SMEM;
  if (set_smem(kern, smem) != cudaSuccess) return DSA_ERR_CUDA;
  if (launch_pdl(kern, dim3(grid), dim3(C::NUM_THREADS), smem, st, tq, tk, pk) != cudaSuccess) return DSA_ERR_CUDA;
  return last_launch_status();
}

// scores [T, S] of query rows at positions pos0.. against keys 0..S-1 (materialised)
dsa_status_t run_indexer_scores(const uint8_t* q_idx, const float* q_scale, const uint8_t* k_idx,
                                const float* k_scale, const float* w, int T, int S, int H_I, int d_I, int pos0,
                                float* scores, long long ld, cudaStream_t st) {
  IndexerParams p{};
  p.w = w;
  p.q_scale = q_scale;
  p.k_scale = k_scale;
  p.scores = scores;
  p.ld = ld;
  p.T = T;
  p.S = S;
  p.pos0 = pos0;
  const int tok = (H_I == 64) ? 16 : 256;
  const int nqb = (T + tok - 1) / tok;
  const int ntiles = (S + 127) / 128;
  // Work items (query block x key-tile range) go round-robin to one persistent CTA per SM.  The key range is
  // split so that the items divide evenly over the SMs: cost = rounds x (tiles per item + ~2 tiles of per-item
  // setup: query block load, pipeline fill), the fewest splits winning ties.
  const int sms = num_sms();
  int best_split = 1;
  double best_cost = 1e300;
  for (int ns = 1; ns <= (ntiles < 64 ? ntiles : 64); ++ns) {
    const int per = (ntiles + ns - 1) / ns;
    const long long items = static_cast<long long>(nqb) * ((ntiles + per - 1) / per);
    const double cost = static_cast<double>((items + sms - 1) / sms) * (per + 2.0);
    if (cost < best_cost - 1e-9) { best_cost = cost; best_split = per; }
  }
  p.split_tiles = best_split;
  p.nsplit = (ntiles + p.split_tiles - 1) / p.split_tiles;
  p.n_items = nqb * p.nsplit;
  const int grid = p.n_items < sms ? p.n_items : sms;
  if (H_I == 64)
    return launch_indexer<64, 128, 4, 4, 1, 4, 2, kModeScores>(q_idx, T, k_idx, S, p, grid, st);
  return launch_indexer<4, 64, 64, 4, 1, 4, 2, kModeScores>(q_idx, T, k_idx, S, p, grid, st);
}

// Indexer scores of the runs of query rows in segs_host (one launch; segs_dev: a device copy of the table, written
// by the caller), into `scores`.  Chooses the key split and fills each run's nsplit and item0 in segs_host before
// the caller copies it.  Returns the number of items through *n_items.
void plan_segments(IndexerSeg* segs, int n_segs, int tok, int* split_tiles, int* n_items) {
  const int sms = num_sms();
  int best = 1;
  double best_cost = 1e300;
  for (int split = 1; split <= 64; ++split) {
    long long items = 0;
    for (int i = 0; i < n_segs; ++i) {
      const int nqb = (segs[i].n_rows + tok - 1) / tok, ntiles = (segs[i].S + 127) / 128;
      items += static_cast<long long>(nqb) * ((ntiles + split - 1) / split);
    }
    const double cost = static_cast<double>((items + sms - 1) / sms) * (split + 2.0);
    if (cost < best_cost - 1e-9) { best_cost = cost; best = split; }
  }
  int item = 0;
  for (int i = 0; i < n_segs; ++i) {
    const int nqb = (segs[i].n_rows + tok - 1) / tok, ntiles = (segs[i].S + 127) / 128;
    segs[i].nsplit = (ntiles + best - 1) / best;
    segs[i].item0 = item;
    item += nqb * segs[i].nsplit;
  }
  *split_tiles = best;
  *n_items = item;
}

dsa_status_t run_indexer_segments(const uint8_t* q_idx, long long q_rows, const float* q_scale, const uint8_t* k_idx,
                                  long long k_rows, const float* k_scale, const float* w, int H_I, int d_I,
                                  const IndexerSeg* segs_dev, int n_segs, int split_tiles, int n_items,
                                  float* scores, cudaStream_t st) {
  if (n_items <= 0) return DSA_OK;
  IndexerParams p{};
  p.w = w;
  p.q_scale = q_scale;
  p.k_scale = k_scale;
  p.scores = scores;
  p.segs = segs_dev;
  p.n_segs = n_segs;
  p.split_tiles = split_tiles;
  p.n_items = n_items;
  const int sms = num_sms();
  const int grid = n_items < sms ? n_items : sms;
  if (H_I == 64)
    return launch_indexer<64, 128, 4, 4, 1, 4, 2, kModeSegments>(q_idx, static_cast<int>(q_rows), k_idx, k_rows, p,
                                                                 grid, st);
  return launch_indexer<4, 64, 64, 4, 1, 4, 2, kModeSegments>(q_idx, static_cast<int>(q_rows), k_idx, k_rows, p, grid,
                                                             st);
}

#ifdef DSA_CHECKS
// DSA_CHECKS builds: every output row of a top-k launch holds min(k, n) entries, strictly ascending and in [0, n)
// for the row's n keys, then -1 padding.  One CTA per row; launched without the dependent-launch attribute, so
// it starts once the top-k has finished.
__global__ void __launch_bounds__(256) topk_check_kernel(const TopkParams p) {
  const int r = blockIdx.x;
  const long long n = p.row_len ? p.row_len[r] : (p.ld < p.pos0 + r + 1 ? p.ld : p.pos0 + r + 1);
  const int m = static_cast<int>(n < p.k ? (n > 0 ? n : 0) : p.k);
  const int* row = p.idx + static_cast<long long>(r) * p.idx_ld;
  bool good = true;
  for (int i = threadIdx.x; i < p.k; i += blockDim.x) {
    const int v = row[i];
    if (i < m) good &= v >= 0 && v < n && (i == 0 || v > row[i - 1]);
    else good &= v == -1;
  }
  if (!good) raise_status(DSA_ERR_CHECK);
}
#endif

dsa_status_t run_topk(const float* scores, long long ld, const long long* row_off, const int* row_len, int pos0,
                      int rows, int k, int* idx, long long idx_ld, cudaStream_t st, float* sel_scores = nullptr,
                      const unsigned* hist = nullptr) {
  if (rows <= 0) return DSA_OK;
  TopkParams p{scores, ld, row_off, row_len, pos0, rows, k, idx, idx_ld, sel_scores, hist};
  if (rows < num_sms()) {
    // fewer rows than SMs (decode): one cluster of kTkcCluster CTAs per row
    if (set_smem(topk_cluster_kernel, static_cast<int>(sizeof(TkcSmem))) != cudaSuccess) return DSA_ERR_CUDA;
    if (launch_pdl(topk_cluster_kernel, dim3(rows * kTkcCluster), dim3(kTkcThreads), sizeof(TkcSmem), st, p) !=
        cudaSuccess)
      return DSA_ERR_CUDA;
  } else {
    if (set_smem(topk_rows_kernel<kTopkThreads>, static_cast<int>(sizeof(TopkSmem<kTopkThreads>))) != cudaSuccess)
      return DSA_ERR_CUDA;
    if (launch_pdl(topk_rows_kernel<kTopkThreads>, dim3(rows), dim3(kTopkThreads), sizeof(TopkSmem<kTopkThreads>), st,
                   p) != cudaSuccess)
      return DSA_ERR_CUDA;
  }
#ifdef DSA_CHECKS
  {
    const dsa_status_t e = last_launch_status();
    if (e != DSA_OK) return e;
    topk_check_kernel<<<rows, 256, 0, st>>>(p);
  }
#endif
  return last_launch_status();
}

// Attention launch.  dense: kMlaSparse (every token gathers its index row), kMlaCausal (token t has the
// t - row_off[t] + 1 keys of its sequence) or kMlaCounts (token t has n_keys[t] keys); in the dense modes a
// token with at most k keys attends to all of them, read as contiguous tiles.
dsa_status_t run_mla(const uint16_t* q, const uint16_t* c, long long S, const int* idx, const long long* row_off,
                     int T, int H, int k, float scale, uint16_t* out, float* lse, cudaStream_t st,
                     int dense = kMlaSparse, const int* n_keys = nullptr, const int* page_table = nullptr,
                     int pt_stride = 0, int page_rows = 0, int pos0 = 0, const float* kl_lse = nullptr,
                     const float* kl_scores = nullptr, float* kl_out = nullptr) {
  if (T <= 0) return DSA_OK;
  CUtensorMap tq;
  const cuuint64_t qd[3] = {576, static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(T)};
  const cuuint64_t qs[2] = {576 * 2, static_cast<cuuint64_t>(H) * 576 * 2};
  const cuuint32_t qb[3] = {64, 128, 1};
  if (!make_map(&tq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, q, qd, qs, qb, CU_TENSOR_MAP_SWIZZLE_128B)) return DSA_ERR_CUDA;
  CUtensorMap tc;   // rows of c, one 64-column box high 1 row (the form tile::gather4 takes)
  const cuuint64_t cd[2] = {576, static_cast<cuuint64_t>(S)};
  const cuuint64_t cs[1] = {576 * 2};
  const cuuint32_t cb[2] = {64, 1};
  if (!make_map(&tc, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, c, cd, cs, cb, CU_TENSOR_MAP_SWIZZLE_128B)) return DSA_ERR_CUDA;
  CUtensorMap tcd;  // contiguous tiles of c: one 64-column box one key tile high (dense tokens)
  const cuuint32_t cbd[2] = {64, static_cast<cuuint32_t>(mla::NK)};
  if (!make_map(&tcd, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, c, cd, cs, cbd, CU_TENSOR_MAP_SWIZZLE_128B))
    return DSA_ERR_CUDA;
  MlaParams p{};
  p.dense = dense;
  p.pos0 = pos0;
  p.n_keys = n_keys;
  p.page_table = page_table;
  p.pt_stride = pt_stride;
  p.page_rows = page_rows;
  p.kl_lse = kl_lse;
  p.kl_scores = kl_scores;
  p.kl_out = kl_out;
  p.idx = idx;
  p.row_off = row_off;
  p.out = out;
  p.lse = lse;
  p.T = T;
  p.H = H;
  p.k = k;
  p.S = S;
  p.scale_log2 = scale * 1.4426950408889634f;
  // the instantiation with exactly the features this launch uses
  const bool dn = dense != kMlaSparse, pg = page_table != nullptr;
  auto kern = kl_out ? (dn ? sparse_mla_kernel<true, true, false> : sparse_mla_kernel<true, false, false>)
            : pg     ? sparse_mla_kernel<false, true, true>
            : dn     ? sparse_mla_kernel<false, true, false>
                     : sparse_mla_kernel<false, false, false>;
  if (pg && !dn) return DSA_ERR_INVALID_ARG;      // paged caches only come with per-token key counts
  if (set_smem(kern, mla::SMEM) != cudaSuccess) return DSA_ERR_CUDA;
  // KL mode: every CTA takes tokens of its own (the grid still comes in pairs, the kernel's cluster shape)
  const int per_cluster = kl_out ? 2 : 1;
  int clusters = num_sms() / 2;
  if (clusters > (T + per_cluster - 1) / per_cluster) clusters = (T + per_cluster - 1) / per_cluster;
  if (launch_pdl(kern, dim3(2 * clusters), dim3(mla::THREADS), mla::SMEM, st, tq, tc, tcd, p) != cudaSuccess)
    return DSA_ERR_CUDA;
  return last_launch_status();
}

// Causal rows [pos0, pos0 + T) of one sequence (row r at position pos0 + r, its keys from row 0 of c): the rows at
// positions below k (every earlier key selected) run on the dense instantiation, the others on the gathered one.
dsa_status_t run_mla_causal(const uint16_t* q, const uint16_t* c, long long S, const int* idx, int T, int H, int k,
                            float scale, uint16_t* out, float* lse, cudaStream_t st, int pos0,
                            const float* kl_lse = nullptr, const float* kl_scores = nullptr,
                            float* kl_out = nullptr) {
  const int nd = std::max(0, std::min(T, k - pos0));
  dsa_status_t e = DSA_OK;
  if (nd > 0)
    e = run_mla(q, c, S, idx, nullptr, nd, H, k, scale, out, lse, st, kMlaCausal, nullptr, nullptr, 0, 0, pos0,
                kl_lse, kl_scores, kl_out);
  if (e != DSA_OK || nd == T) return e;
  const size_t n = static_cast<size_t>(nd);
  return run_mla(q + n * H * 576, c, S, idx + n * k, nullptr, T - nd, H, k, scale, out ? out + n * H * 512 : nullptr,
                 lse ? lse + n * H : nullptr, st, kMlaSparse, nullptr, nullptr, 0, 0, 0,
                 kl_lse ? kl_lse + n * H : nullptr, kl_scores ? kl_scores + n * k : nullptr,
                 kl_out ? kl_out + n : nullptr);
}

// k: at least 128 and a multiple of 64 (slots of a last, half-filled 128-key tile are masked), at most KMAX
bool mla_k_ok(int k) { return k >= 128 && k % 64 == 0 && k <= mla::KMAX; }

bool indexer_shape_ok(int H_I, int d_I) { return (H_I == 64 && d_I == 128) || (H_I == 4 && d_I == 64); }

size_t prefill_chunk_rows(int L) {
  // rows of scores materialised per chunk: about 1 GiB of fp32 scores, at least 256 rows
  size_t r = (size_t(1) << 30) / (4 * size_t(L > 0 ? L : 1));
  if (r < 256) r = 256;
  if (r > size_t(L)) r = size_t(L);
  return r;
}

int round4(int n) { return (n + 3) & ~3; }

// Scores the varlen select holds at once: at least one sequence's blocked select (the longest), and up to 1 GiB
// for groups of sequences scored together.
size_t varlen_score_floats(int64_t total, int max_len) {
  const size_t one = prefill_chunk_rows(max_len) * size_t(max_len);
  const size_t all = size_t(total) * size_t(round4(max_len));
  const size_t cap = size_t(1) << 28;
  return std::max(one, std::min(all, cap));
}

// Group metadata of the varlen select: runs of query rows, relative sequence starts, score offsets and strides.
size_t varlen_meta_bytes(int nseq) {
  return align_up(size_t(nseq) * sizeof(IndexerSeg), 256) + align_up(size_t(nseq + 1) * 8 + size_t(nseq) * 12, 256);
}

// Steps 1-2 for rows [pos_begin, pos_end) of one causal sequence (row r attends to keys 0..r): q_idx, q_scale, w and
// idx_out point at row pos_begin; k_idx, k_scale hold keys 0..pos_end-1.  Rows t < k form one block whose
// selection needs no scores; later rows go in blocks of chunk_rows, each an indexer launch into `sc` (room for
// chunk_rows x pos_end scores) and a top-k launch.  With sel_scores (pointing at row pos_begin), the index score of
// every selected position is written too, and the indexer then also scores the rows t < k.
dsa_status_t select_rows(const uint8_t* q_idx, const float* q_scale, const uint8_t* k_idx, const float* k_scale,
                         const float* w, int H_I, int d_I, int k, int pos_begin, int pos_end, int32_t* idx_out,
                         float* sc, size_t chunk_rows, cudaStream_t st, float* sel_scores = nullptr) {
  for (int r0 = pos_begin, rows = 0; r0 < pos_end; r0 += rows) {
    rows = (r0 < k) ? std::min(k, pos_end) - r0 : static_cast<int>(std::min<size_t>(chunk_rows, pos_end - r0));
    const int s_eff = r0 + rows;   // keys beyond the block's last row are never selected (causal)
    const size_t i = static_cast<size_t>(r0 - pos_begin);
    // a block whose every row t has t + 1 <= k selects all of 0..t whatever the scores: no indexer launch (the
    // top-k kernel writes 0..t and the -1 padding of such rows without reading them)
    dsa_status_t e = DSA_OK;
    if (s_eff > k || sel_scores) {
      e = run_indexer_scores(q_idx + i * H_I * d_I, q_scale ? q_scale + i : nullptr, k_idx, k_scale, w + i * H_I,
                             rows, s_eff, H_I, d_I, r0, sc, s_eff, st);
      if (e != DSA_OK) return e;
    }
    e = run_topk(sc, s_eff, nullptr, nullptr, r0, rows, k, idx_out + i * k, k, st,
                 sel_scores ? sel_scores + i * k : nullptr);
    if (e != DSA_OK) return e;
  }
  return DSA_OK;
}

// Rows of the score block of an L-row prefill that starts at row r0: rows t < k form a block of their own, whose
// selection needs no scores; later blocks take prefill_chunk_rows(L) rows (the workspace's capacity at the
// longest key range).  Blocks sized to fill the workspace at every key range (many more rows early on) were
// measured slower for the indexer at 128K (98.2 against 96.0 ms per step) and are not used.
int prefill_block_rows(int L, int k, int r0) {
  if (r0 < 0 || r0 >= L) return 0;
  if (r0 < k) return std::min(k, L) - r0;
  return static_cast<int>(std::min<size_t>(prefill_chunk_rows(L), static_cast<size_t>(L - r0)));
}

// Host checks of a decode step's arguments, shared by both decode entry points (everything but the scratch).
dsa_status_t decode_args_status(int B, const int64_t* cache_off, const int32_t* ctx_len, const uint8_t* q_idx,
                                const float* w, const uint16_t* q, const uint8_t* k_new, const float* k_scale_new,
                                const uint16_t* c_new, const uint8_t* k_cache, const float* k_scale_cache,
                                const uint16_t* c_cache, int64_t cache_rows, int H_I, int d_I, int H, int k,
                                const int32_t* idx_out, const uint16_t* out) {
  if (B <= 0 || cache_rows <= 0 || H <= 0 || k <= 0 || !cache_off || !ctx_len || !q_idx || !w || !q || !k_new ||
      !k_scale_new || !c_new || !k_cache || !k_scale_cache || !c_cache || !out)
    return DSA_ERR_INVALID_ARG;
  if (H_I != 64 || d_I != 128 || H > 128 || !mla_k_ok(k) || B > kMaxDecodeSeqs) return DSA_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(q_idx) || !aligned16(q) || !aligned16(k_new) || !aligned16(c_new) || !aligned16(k_cache) ||
      !aligned16(c_cache) || !aligned16(out) || (idx_out && !aligned16(idx_out)))
    return DSA_ERR_ALIGNMENT;
  return DSA_OK;
}

size_t decode_ws_bytes(int B, size_t score_cap, int k) {
  return align_up(score_cap * 4, 256) + align_up(size_t(B) * 4, 256) + align_up(size_t(B) * 8, 256) +
         align_up(size_t(B) * k * 4, 256) + align_up(size_t(B) * kTopkBins * 4, 256);
}

// One decode step once the arguments are checked: append -> indexer over each sequence's keys -> top-k -> sparse
// MLA.  Workspace: score rows (packed, 16-byte aligned, score_cap floats), len1 [B], score_off [B], selected
// indices [B, k] (when idx_out is null), each sequence's score histogram [B, 2048] (top 11 order-key bits).
// With fewer sequences than SMs the indexer counts the histogram as it writes the scores, and the cluster top-k
// reads it instead of counting the row again and merging its CTAs' counts.
dsa_status_t run_decode(int B, const DecodeLayout& lay, const int32_t* ctx_len, const uint8_t* q_idx,
                        const float* q_scale, const float* w, const uint16_t* q, const uint8_t* k_new,
                        const float* k_scale_new, const uint16_t* c_new, uint8_t* k_cache, float* k_scale_cache,
                        uint16_t* c_cache, size_t score_cap, int H, int k, float scale, int32_t* idx_out,
                        uint16_t* out, float* lse, void* ws, cudaStream_t st) {
  constexpr int H_I = 64, d_I = 128;
  char* wsb = static_cast<char*>(ws);
  float* dscores = reinterpret_cast<float*>(wsb);
  size_t at = align_up(score_cap * 4, 256);
  int* len1 = reinterpret_cast<int*>(wsb + at);
  at += align_up(size_t(B) * 4, 256);
  long long* soff = reinterpret_cast<long long*>(wsb + at);
  at += align_up(size_t(B) * 8, 256);
  int32_t* idx = idx_out ? idx_out : reinterpret_cast<int32_t*>(wsb + at);
  at += align_up(size_t(B) * k * 4, 256);
  unsigned* hist = (B < num_sms()) ? reinterpret_cast<unsigned*>(wsb + at) : nullptr;
  if (launch_pdl(decode_append_kernel, dim3(B), dim3(kAppendThreads), 0, st, B, lay, ctx_len, k_new, k_scale_new,
                 c_new, k_cache, k_scale_cache, c_cache, d_I, len1, soff, static_cast<long long>(score_cap), hist) !=
      cudaSuccess)
    return DSA_ERR_CUDA;
  dsa_status_t e = last_launch_status();
  if (e != DSA_OK) return e;
  IndexerParams p{};
  p.w = w;
  p.q_scale = q_scale;
  p.k_scale = k_scale_cache;
  p.scores = dscores;
  p.T = B;
  p.cache_off = lay.cache_off;
  p.len1 = len1;
  p.score_off = soff;
  p.page_table = lay.page_table;
  p.max_pages = lay.max_pages;
  p.page_rows = lay.page_rows;
  p.hist = hist;
  using DecCfg = IndexerCfg<H_I, d_I, 1, 1, 2, 4, 1, kModeDecode>;
  e = launch_indexer<H_I, d_I, 1, 1, 2, 4, 1, kModeDecode>(q_idx, B, k_cache, lay.cache_rows, p,
                                                         DecCfg::CTAS_PER_SM * num_sms(), st);
  if (e != DSA_OK) return e;
  e = run_topk(dscores, 0, soff, len1, 0, B, k, idx, k, st, nullptr, hist);
  if (e != DSA_OK) return e;
  return run_mla(q, c_cache, lay.cache_rows, idx, lay.cache_off, B, H, k, scale, out, lse, st, kMlaCounts, len1,
                 lay.page_table, lay.max_pages, lay.page_rows);
}

}  // namespace
}  // namespace dsa

using namespace dsa;

extern "C" {

const char* dsa_status_string(dsa_status_t s) {
  switch (s) {
    case DSA_OK: return "DSA_OK";
    case DSA_ERR_INVALID_ARG: return "DSA_ERR_INVALID_ARG";
    case DSA_ERR_UNSUPPORTED_SHAPE: return "DSA_ERR_UNSUPPORTED_SHAPE";
    case DSA_ERR_ALIGNMENT: return "DSA_ERR_ALIGNMENT";
    case DSA_ERR_CUDA: return "DSA_ERR_CUDA";
    case DSA_ERR_TIMEOUT: return "DSA_ERR_TIMEOUT";
    case DSA_ERR_BAD_INDEX: return "DSA_ERR_BAD_INDEX";
    case DSA_ERR_WORKSPACE: return "DSA_ERR_WORKSPACE";
    case DSA_ERR_CHECK: return "DSA_ERR_CHECK";
  }
  return "DSA_UNKNOWN_STATUS";
}

dsa_status_t dsa_get_device_status(void* stream, int* device_status) {
  if (!device_status) return DSA_ERR_INVALID_ARG;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return DSA_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_dev_status, sizeof(int)) != cudaSuccess) return DSA_ERR_CUDA;
  const int zero = 0;
  if (cudaMemcpyToSymbol(g_dev_status, &zero, sizeof(int)) != cudaSuccess) return DSA_ERR_CUDA;
  *device_status = v;
  return DSA_OK;
}

int dsa_num_sms(void) { return num_sms(); }

int dsa_checks_enabled(void) { return kChecks ? 1 : 0; }

dsa_status_t dsa_indexer_scores(const uint8_t* q_idx, const float* q_scale, const uint8_t* k_idx,
                                const float* k_scale, const float* w, int T, int S, int H_I, int d_I, int pos0,
                                float* scores, void* stream) {
  if (T < 0 || S < 0 || pos0 < 0 || (T > 0 && (!q_idx || !w || !scores)) || (S > 0 && !k_idx))
    return DSA_ERR_INVALID_ARG;
  if (!indexer_shape_ok(H_I, d_I)) return DSA_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(q_idx) || !aligned16(k_idx)) return DSA_ERR_ALIGNMENT;
  if (T == 0 || S == 0) return DSA_OK;
  return run_indexer_scores(q_idx, q_scale, k_idx, k_scale, w, T, S, H_I, d_I, pos0, scores, S,
                            static_cast<cudaStream_t>(stream));
}

dsa_status_t dsa_topk(const float* scores, int rows, int64_t ld, const int32_t* row_len, int pos0, int k,
                      int32_t* idx, void* stream) {
  if (rows < 0 || ld < 0 || k <= 0 || pos0 < 0 || (rows > 0 && (!scores || !idx))) return DSA_ERR_INVALID_ARG;
  return run_topk(scores, ld, nullptr, row_len, pos0, rows, k, idx, k, static_cast<cudaStream_t>(stream));
}

dsa_status_t dsa_indexer_kl(const uint16_t* q, const uint16_t* c, int S, const int32_t* idx, const float* sel_scores,
                            const float* lse, int T, int H, int k, float scale, float* kl, void* stream) {
  if (T < 0 || S <= 0 || H <= 0 || k <= 0 || (T > 0 && (!q || !c || !idx || !sel_scores || !lse || !kl)))
    return DSA_ERR_INVALID_ARG;
  if (H > 128 || !mla_k_ok(k)) return DSA_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(q) || !aligned16(c) || !aligned16(idx)) return DSA_ERR_ALIGNMENT;
  return run_mla(q, c, S, idx, nullptr, T, H, k, scale, nullptr, nullptr, static_cast<cudaStream_t>(stream),
                 kMlaSparse, nullptr, nullptr, 0, 0, 0, lse, sel_scores, kl);
}

size_t dsa_prefill_kl_workspace_size(int L, int H_I, int d_I, int H, int k) {
  if (L <= 0 || k <= 0 || H <= 0) return 0;
  return dsa_prefill_workspace_size(L, H_I, d_I, H, k) + align_up(size_t(L) * size_t(k) * 4, 256) +
         align_up(size_t(L) * size_t(H) * 4, 256);
}

dsa_status_t dsa_forward_prefill_kl(const uint8_t* q_idx, const float* q_scale, const uint8_t* k_idx,
                                    const float* k_scale, const float* w, const uint16_t* q, const uint16_t* c,
                                    int L, int H_I, int d_I, int H, int k, float scale, int32_t* idx_out,
                                    uint16_t* out, float* lse, float* kl, void* ws, size_t ws_bytes, void* stream) {
  if (L <= 0 || H <= 0 || k <= 0 || !q_idx || !k_idx || !w || !q || !c || !out || !kl) return DSA_ERR_INVALID_ARG;
  if (!indexer_shape_ok(H_I, d_I) || H > 128 || !mla_k_ok(k)) return DSA_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(q_idx) || !aligned16(k_idx) || !aligned16(q) || !aligned16(c) || !aligned16(out) ||
      (idx_out && !aligned16(idx_out)))
    return DSA_ERR_ALIGNMENT;
  if (!ws || ws_bytes < dsa_prefill_kl_workspace_size(L, H_I, d_I, H, k)) return DSA_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // workspace: the prefill's (score block, selected indices), then the selected index scores [L, k] and lse [L, H]
  char* wsb = static_cast<char*>(ws);
  const size_t score_bytes = align_up(prefill_chunk_rows(L) * size_t(L) * 4, 256);
  int32_t* idx = idx_out ? idx_out : reinterpret_cast<int32_t*>(wsb + score_bytes);
  size_t at = dsa_prefill_workspace_size(L, H_I, d_I, H, k);
  float* sel = reinterpret_cast<float*>(wsb + at);
  at += align_up(size_t(L) * size_t(k) * 4, 256);
  float* lse_buf = lse ? lse : reinterpret_cast<float*>(wsb + at);
  dsa_status_t e = select_rows(q_idx, q_scale, k_idx, k_scale, w, H_I, d_I, k, 0, L, idx, reinterpret_cast<float*>(wsb),
                               prefill_chunk_rows(L), st, sel);
  if (e != DSA_OK) return e;
  e = run_mla_causal(q, c, L, idx, L, H, k, scale, out, lse_buf, st, 0);
  if (e != DSA_OK) return e;
  return run_mla_causal(q, c, L, idx, L, H, k, scale, nullptr, nullptr, st, 0, lse_buf, sel, kl);
}

dsa_status_t dsa_sparse_mla_attn(const uint16_t* q, const uint16_t* c, int S, const int32_t* idx, int T, int H,
                                 int k, float scale, uint16_t* out, float* lse, void* stream) {
  if (T < 0 || S <= 0 || H <= 0 || k <= 0 || (T > 0 && (!q || !c || !idx || !out))) return DSA_ERR_INVALID_ARG;
  if (H > 128 || !mla_k_ok(k)) return DSA_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(q) || !aligned16(c) || !aligned16(idx) || !aligned16(out)) return DSA_ERR_ALIGNMENT;
  return run_mla(q, c, S, idx, nullptr, T, H, k, scale, out, lse, static_cast<cudaStream_t>(stream));
}

size_t dsa_prefill_workspace_size(int L, int H_I, int d_I, int H, int k) {
  (void)H_I; (void)d_I; (void)H;
  if (L <= 0 || k <= 0) return 0;
  const size_t rows = prefill_chunk_rows(L);
  return align_up(rows * size_t(L) * 4, 256) + align_up(size_t(L) * size_t(k) * 4, 256);
}

dsa_status_t dsa_prefill_select(const uint8_t* q_idx, const float* q_scale, const uint8_t* k_idx,
                                const float* k_scale, const float* w, int L, int H_I, int d_I, int k,
                                int32_t* idx_out, void* ws, size_t ws_bytes, void* stream) {
  if (L <= 0 || k <= 0 || !q_idx || !k_idx || !w || !idx_out) return DSA_ERR_INVALID_ARG;
  if (!indexer_shape_ok(H_I, d_I)) return DSA_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(q_idx) || !aligned16(k_idx)) return DSA_ERR_ALIGNMENT;
  if (!ws || ws_bytes < align_up(prefill_chunk_rows(L) * size_t(L) * 4, 256)) return DSA_ERR_WORKSPACE;
  return select_rows(q_idx, q_scale, k_idx, k_scale, w, H_I, d_I, k, 0, L, idx_out, static_cast<float*>(ws),
                     prefill_chunk_rows(L), static_cast<cudaStream_t>(stream));
}

size_t dsa_prefill_rows_workspace_size(int row0, int nrows, int H_I, int d_I, int H, int k) {
  (void)H_I; (void)d_I; (void)H;
  if (row0 < 0 || nrows <= 0 || k <= 0) return 0;
  const int S = row0 + nrows;
  return align_up(prefill_chunk_rows(S) * size_t(S) * 4, 256) + align_up(size_t(nrows) * size_t(k) * 4, 256);
}

dsa_status_t dsa_forward_prefill_rows(const uint8_t* q_idx, const float* q_scale, const uint8_t* k_idx,
                                      const float* k_scale, const float* w, const uint16_t* q, const uint16_t* c,
                                      int row0, int nrows, int H_I, int d_I, int H, int k, float scale,
                                      int32_t* idx_out, uint16_t* out, float* lse, void* ws, size_t ws_bytes,
                                      void* stream) {
  if (row0 < 0 || nrows <= 0 || H <= 0 || k <= 0 || !q_idx || !k_idx || !w || !q || !c || !out)
    return DSA_ERR_INVALID_ARG;
  if (static_cast<long long>(row0) + nrows > INT32_MAX) return DSA_ERR_INVALID_ARG;
  if (!indexer_shape_ok(H_I, d_I) || H > 128 || !mla_k_ok(k)) return DSA_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(q_idx) || !aligned16(k_idx) || !aligned16(q) || !aligned16(c) || !aligned16(out) ||
      (idx_out && !aligned16(idx_out)))
    return DSA_ERR_ALIGNMENT;
  if (!ws || ws_bytes < dsa_prefill_rows_workspace_size(row0, nrows, H_I, d_I, H, k)) return DSA_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int S = row0 + nrows;
  const size_t score_bytes = align_up(prefill_chunk_rows(S) * size_t(S) * 4, 256);
  int32_t* idx = idx_out ? idx_out : reinterpret_cast<int32_t*>(static_cast<char*>(ws) + score_bytes);
  dsa_status_t e = select_rows(q_idx, q_scale, k_idx, k_scale, w, H_I, d_I, k, row0, S, idx, static_cast<float*>(ws),
                               prefill_chunk_rows(S), st);
  if (e != DSA_OK) return e;
  return run_mla_causal(q, c, S, idx, nrows, H, k, scale, out, lse, st, row0);
}

dsa_status_t dsa_forward_prefill(const uint8_t* q_idx, const float* q_scale, const uint8_t* k_idx,
                                 const float* k_scale, const float* w, const uint16_t* q, const uint16_t* c,
                                 int L, int H_I, int d_I, int H, int k, float scale, int32_t* idx_out,
                                 uint16_t* out, float* lse, void* ws, size_t ws_bytes, void* stream) {
  if (L <= 0 || H <= 0 || k <= 0 || !q_idx || !k_idx || !w || !q || !c || !out) return DSA_ERR_INVALID_ARG;
  if (!indexer_shape_ok(H_I, d_I) || H > 128 || !mla_k_ok(k)) return DSA_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(q_idx) || !aligned16(k_idx) || !aligned16(q) || !aligned16(c) || !aligned16(out) ||
      (idx_out && !aligned16(idx_out)))
    return DSA_ERR_ALIGNMENT;
  if (!ws || ws_bytes < dsa_prefill_workspace_size(L, H_I, d_I, H, k)) return DSA_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int32_t* idx = idx_out ? idx_out
                         : reinterpret_cast<int32_t*>(static_cast<char*>(ws) +
                                                      align_up(prefill_chunk_rows(L) * size_t(L) * 4, 256));
  dsa_status_t e = dsa_prefill_select(q_idx, q_scale, k_idx, k_scale, w, L, H_I, d_I, k, idx, ws, ws_bytes, stream);
  if (e != DSA_OK) return e;
  return run_mla_causal(q, c, L, idx, L, H, k, scale, out, lse, st, 0);
}

// ------------------------------------------------------------------------------------------ host-buffer prefill
namespace {
constexpr int kHostChunks = 16;         // token chunks of the host-buffer prefill's pipeline

// The host-buffer prefill's device copies, laid out after the prefill workspace.
struct HostPrefillLayout {
  size_t ws, q_idx, q_scale, k_idx, k_scale, w, q, c, out, lse, total;
};
HostPrefillLayout host_prefill_layout(int L, int H_I, int d_I, int H, int k) {
  HostPrefillLayout lo{};
  size_t at = dsa_prefill_workspace_size(L, H_I, d_I, H, k);
  auto take = [&](size_t bytes) { const size_t o = at; at += align_up(bytes, 256); return o; };
  lo.ws = 0;
  lo.q_idx = take(size_t(L) * H_I * d_I);
  lo.q_scale = take(size_t(L) * 4);
  lo.k_idx = take(size_t(L) * d_I);
  lo.k_scale = take(size_t(L) * 4);
  lo.w = take(size_t(L) * H_I * 4);
  lo.q = take(size_t(L) * H * 576 * 2);
  lo.c = take(size_t(L) * 576 * 2);
  lo.out = take(size_t(L) * H * 512 * 2);
  lo.lse = take(size_t(L) * H * 4);
  lo.total = at;
  return lo;
}

// One copy stream per direction and device, created on first use (the call allocates no memory).
struct CopyStreams {
  cudaStream_t h2d = nullptr, d2h = nullptr;
};
CopyStreams g_copy_streams[64];
std::mutex g_copy_mutex;

dsa_status_t copy_streams(CopyStreams* out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return DSA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_copy_mutex);
  CopyStreams& cs = g_copy_streams[dev];
  if (!cs.h2d && cudaStreamCreateWithFlags(&cs.h2d, cudaStreamNonBlocking) != cudaSuccess) return DSA_ERR_CUDA;
  if (!cs.d2h && cudaStreamCreateWithFlags(&cs.d2h, cudaStreamNonBlocking) != cudaSuccess) return DSA_ERR_CUDA;
  *out = cs;
  return DSA_OK;
}
}  // namespace

size_t dsa_prefill_host_workspace_size(int L, int H_I, int d_I, int H, int k) {
  if (L <= 0 || k <= 0 || H <= 0 || !indexer_shape_ok(H_I, d_I)) return 0;
  return host_prefill_layout(L, H_I, d_I, H, k).total;
}

dsa_status_t dsa_forward_prefill_host(const uint8_t* q_idx, const float* q_scale, const uint8_t* k_idx,
                                      const float* k_scale, const float* w, const uint16_t* q, const uint16_t* c,
                                      int L, int H_I, int d_I, int H, int k, float scale, int32_t* idx_out,
                                      uint16_t* out, float* lse, void* ws, size_t ws_bytes, void* stream) {
  if (L <= 0 || H <= 0 || k <= 0 || !q_idx || !k_idx || !w || !q || !c || !out) return DSA_ERR_INVALID_ARG;
  if (!indexer_shape_ok(H_I, d_I) || H > 128 || !mla_k_ok(k)) return DSA_ERR_UNSUPPORTED_SHAPE;
  if (!ws || ws_bytes < dsa_prefill_host_workspace_size(L, H_I, d_I, H, k)) return DSA_ERR_WORKSPACE;
  CopyStreams cs;
  dsa_status_t e = copy_streams(&cs);
  if (e != DSA_OK) return e;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const HostPrefillLayout lo = host_prefill_layout(L, H_I, d_I, H, k);
  char* d = static_cast<char*>(ws);
  uint8_t* dq_idx = reinterpret_cast<uint8_t*>(d + lo.q_idx);
  float* dq_scale = q_scale ? reinterpret_cast<float*>(d + lo.q_scale) : nullptr;
  uint8_t* dk_idx = reinterpret_cast<uint8_t*>(d + lo.k_idx);
  float* dk_scale = k_scale ? reinterpret_cast<float*>(d + lo.k_scale) : nullptr;
  float* dw = reinterpret_cast<float*>(d + lo.w);
  uint16_t* dq = reinterpret_cast<uint16_t*>(d + lo.q);
  uint16_t* dc = reinterpret_cast<uint16_t*>(d + lo.c);
  uint16_t* dout = reinterpret_cast<uint16_t*>(d + lo.out);
  float* dlse = reinterpret_cast<float*>(d + lo.lse);
  float* sc = reinterpret_cast<float*>(d);
  int32_t* didx = reinterpret_cast<int32_t*>(d + align_up(prefill_chunk_rows(L) * size_t(L) * 4, 256));
  // events: start, indexer inputs landed, per chunk its queries landed and its attention done, all copies back
  constexpr int NE = 2 + 2 * kHostChunks + 1;
  cudaEvent_t ev[NE] = {};
  for (int i = 0; i < NE; ++i)
    if (cudaEventCreateWithFlags(&ev[i], cudaEventDisableTiming) != cudaSuccess) {
      for (int j = 0; j < i; ++j) cudaEventDestroy(ev[j]);
      return DSA_ERR_CUDA;
    }
  cudaEvent_t& ev_start = ev[0];
  cudaEvent_t& ev_inputs = ev[1];
  cudaEvent_t* ev_q = ev + 2;
  cudaEvent_t* ev_att = ev + 2 + kHostChunks;
  cudaEvent_t& ev_done = ev[NE - 1];
  auto h2d = [&](void* dst, const void* src, size_t bytes) {
    return !src || cudaMemcpyAsync(dst, src, bytes, cudaMemcpyHostToDevice, cs.h2d) == cudaSuccess;
  };
  auto d2h = [&](void* dst, const void* src, size_t bytes) {
    return !dst || cudaMemcpyAsync(dst, src, bytes, cudaMemcpyDeviceToHost, cs.d2h) == cudaSuccess;
  };
  const size_t qrow = size_t(H) * 576 * 2, orow = size_t(H) * 512 * 2;
  bool ok = cudaEventRecord(ev_start, st) == cudaSuccess && cudaStreamWaitEvent(cs.h2d, ev_start, 0) == cudaSuccess &&
            cudaStreamWaitEvent(cs.d2h, ev_start, 0) == cudaSuccess;
  // host -> device: the indexer's inputs first, then c and the queries chunk by chunk
  ok = ok && h2d(dk_idx, k_idx, size_t(L) * d_I) && h2d(dk_scale, k_scale, size_t(L) * 4) &&
       h2d(dq_idx, q_idx, size_t(L) * H_I * d_I) && h2d(dq_scale, q_scale, size_t(L) * 4) &&
       h2d(dw, w, size_t(L) * H_I * 4) && cudaEventRecord(ev_inputs, cs.h2d) == cudaSuccess &&
       h2d(dc, c, size_t(L) * 576 * 2);
  int t0[kHostChunks + 1];
  for (int j = 0; j <= kHostChunks; ++j) t0[j] = static_cast<int>((static_cast<long long>(L) * j) / kHostChunks);
  for (int j = 0; j < kHostChunks && ok; ++j) {
    ok = h2d(reinterpret_cast<char*>(dq) + t0[j] * qrow, reinterpret_cast<const char*>(q) + t0[j] * qrow,
             size_t(t0[j + 1] - t0[j]) * qrow) &&
         cudaEventRecord(ev_q[j], cs.h2d) == cudaSuccess;
  }
  // compute, chunk by chunk: the chunk's rows' selection, then (once its queries landed) its attention
  ok = ok && cudaStreamWaitEvent(st, ev_inputs, 0) == cudaSuccess;
  for (int j = 0; j < kHostChunks && ok && e == DSA_OK; ++j) {
    const int n = t0[j + 1] - t0[j];
    if (n == 0) {
      ok = cudaEventRecord(ev_att[j], st) == cudaSuccess;
      continue;
    }
    e = select_rows(dq_idx + size_t(t0[j]) * H_I * d_I, dq_scale ? dq_scale + t0[j] : nullptr, dk_idx, dk_scale,
                    dw + size_t(t0[j]) * H_I, H_I, d_I, k, t0[j], t0[j + 1], didx + size_t(t0[j]) * k, sc,
                    prefill_chunk_rows(L), st);
    if (e != DSA_OK) break;
    ok = cudaStreamWaitEvent(st, ev_q[j], 0) == cudaSuccess;
    if (!ok) break;
    e = run_mla_causal(reinterpret_cast<const uint16_t*>(reinterpret_cast<const char*>(dq) + t0[j] * qrow), dc, L,
                       didx + size_t(t0[j]) * k, n, H, k, scale,
                       reinterpret_cast<uint16_t*>(reinterpret_cast<char*>(dout) + t0[j] * orow),
                       dlse + size_t(t0[j]) * H, st, t0[j]);
    if (e != DSA_OK) break;
    ok = cudaEventRecord(ev_att[j], st) == cudaSuccess;
    // device -> host of the chunk's results, on the other copy stream
    ok = ok && cudaStreamWaitEvent(cs.d2h, ev_att[j], 0) == cudaSuccess &&
         d2h(reinterpret_cast<char*>(out) + t0[j] * orow, reinterpret_cast<char*>(dout) + t0[j] * orow,
             size_t(n) * orow) &&
         d2h(lse ? lse + size_t(t0[j]) * H : nullptr, dlse + size_t(t0[j]) * H, size_t(n) * H * 4) &&
         d2h(idx_out ? idx_out + size_t(t0[j]) * k : nullptr, didx + size_t(t0[j]) * k, size_t(n) * k * 4);
  }
  // the caller's stream ends when every copy back has landed
  ok = ok && cudaEventRecord(ev_done, cs.d2h) == cudaSuccess && cudaStreamWaitEvent(st, ev_done, 0) == cudaSuccess;
  for (int i = 0; i < NE; ++i) cudaEventDestroy(ev[i]);     // released once the work that uses them completes
  if (e != DSA_OK) return e;
  return ok ? DSA_OK : DSA_ERR_CUDA;
}

size_t dsa_prefill_varlen_workspace_size(int nseq, int64_t total, int max_len, int H_I, int d_I, int H, int k) {
  (void)H_I; (void)d_I; (void)H;
  if (nseq <= 0 || total <= 0 || max_len <= 0 || k <= 0) return 0;
  return align_up(varlen_score_floats(total, max_len) * 4, 256) + align_up(size_t(total) * 8, 256) +
         align_up(size_t(nseq + 1) * 8, 256) + align_up(size_t(total) * size_t(k) * 4, 256) +
         align_up(size_t(total) * 8, 256) + align_up(size_t(total) * 4, 256) + varlen_meta_bytes(nseq);
}

dsa_status_t dsa_forward_prefill_varlen(int nseq, const int64_t* cu_seqlens, const uint8_t* q_idx,
                                        const float* q_scale, const uint8_t* k_idx, const float* k_scale,
                                        const float* w, const uint16_t* q, const uint16_t* c, int H_I, int d_I,
                                        int H, int k, float scale, int32_t* idx_out, uint16_t* out, float* lse,
                                        void* ws, size_t ws_bytes, void* stream) {
  if (nseq <= 0 || !cu_seqlens || H <= 0 || k <= 0 || !q_idx || !k_idx || !w || !q || !c || !out)
    return DSA_ERR_INVALID_ARG;
  if (cu_seqlens[0] != 0) return DSA_ERR_INVALID_ARG;
  int max_len = 0;
  for (int b = 0; b < nseq; ++b) {
    const int64_t len = cu_seqlens[b + 1] - cu_seqlens[b];
    if (len < 0 || cu_seqlens[b + 1] > INT32_MAX) return DSA_ERR_INVALID_ARG;
    if (len > max_len) max_len = static_cast<int>(len);
  }
  const int64_t total = cu_seqlens[nseq];
  if (total <= 0) return DSA_ERR_INVALID_ARG;
  if (!indexer_shape_ok(H_I, d_I) || H > 128 || !mla_k_ok(k)) return DSA_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(q_idx) || !aligned16(k_idx) || !aligned16(q) || !aligned16(c) || !aligned16(out) ||
      (idx_out && !aligned16(idx_out)))
    return DSA_ERR_ALIGNMENT;
  if (!ws || ws_bytes < dsa_prefill_varlen_workspace_size(nseq, total, max_len, H_I, d_I, H, k))
    return DSA_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // workspace: scores, per-token row offsets (attention), cu_seqlens, indices, per-row score offsets and lengths
  // (top-k), then the metadata of a group of sequences (runs of query rows, relative starts, score offsets, strides)
  char* wsb = static_cast<char*>(ws);
  const size_t budget = varlen_score_floats(total, max_len);
  float* sc = reinterpret_cast<float*>(wsb);
  size_t at = align_up(budget * 4, 256);
  long long* row_off = reinterpret_cast<long long*>(wsb + at);
  at += align_up(size_t(total) * 8, 256);
  long long* cu_dev = reinterpret_cast<long long*>(wsb + at);
  at += align_up(size_t(nseq + 1) * 8, 256);
  int32_t* idx = idx_out ? idx_out : reinterpret_cast<int32_t*>(wsb + at);
  at += align_up(size_t(total) * size_t(k) * 4, 256);
  long long* tk_off = reinterpret_cast<long long*>(wsb + at);
  at += align_up(size_t(total) * 8, 256);
  int* tk_len = reinterpret_cast<int*>(wsb + at);
  at += align_up(size_t(total) * 4, 256);
  char* meta = wsb + at;
  IndexerSeg* segs_dev = reinterpret_cast<IndexerSeg*>(meta);
  long long* gcu_dev = reinterpret_cast<long long*>(meta + align_up(size_t(nseq) * sizeof(IndexerSeg), 256));
  long long* soff_dev = gcu_dev + (nseq + 1);
  int* sld_dev = reinterpret_cast<int*>(soff_dev + nseq);
  if (cudaMemcpyAsync(cu_dev, cu_seqlens, size_t(nseq + 1) * 8, cudaMemcpyHostToDevice, st) != cudaSuccess)
    return DSA_ERR_CUDA;
  varlen_row_off_kernel<<<static_cast<unsigned>((total + 255) / 256), 256, 0, st>>>(cu_dev, nseq, total, row_off);
  dsa_status_t e = last_launch_status();
  if (e != DSA_OK) return e;
  // Steps 1-2.  Consecutive sequences are grouped while their scored rows (t >= k) fit the score buffer; a group
  // is one indexer launch over all of its sequences' scored rows and one top-k launch over all of its rows.  A
  // sequence whose scores alone exceed the buffer takes the blocked select of dsa_prefill_select.
  std::vector<IndexerSeg> segs;
  std::vector<long long> gcu, soff;
  std::vector<int> sld;
  const int tok = (H_I == 64) ? 16 : 256;
  for (int b = 0; b < nseq;) {
    const int64_t r0 = cu_seqlens[b];
    const int len = static_cast<int>(cu_seqlens[b + 1] - r0);
    const size_t need = (len > k) ? size_t(len - k) * size_t(round4(len)) : 0;
    if (need > budget) {
      e = select_rows(q_idx + r0 * H_I * d_I, q_scale ? q_scale + r0 : nullptr, k_idx + r0 * d_I,
                      k_scale ? k_scale + r0 : nullptr, w + r0 * H_I, H_I, d_I, k, 0, len, idx + r0 * k, sc,
                      prefill_chunk_rows(len), st);
      if (e != DSA_OK) return e;
      ++b;
      continue;
    }
    const int b0 = b;
    size_t used = 0;
    segs.clear();
    gcu.assign(1, 0);
    soff.clear();
    sld.clear();
    while (b < nseq && segs.size() < static_cast<size_t>(kMaxDecodeSeqs)) {
      const int64_t rb = cu_seqlens[b];
      const int lb = static_cast<int>(cu_seqlens[b + 1] - rb);
      const size_t nb = (lb > k) ? size_t(lb - k) * size_t(round4(lb)) : 0;
      if (used + nb > budget) break;
      if (nb) {
        IndexerSeg sg{};
        sg.q_row0 = rb + k;
        sg.key_row0 = rb;
        sg.out_base = static_cast<long long>(used);
        sg.pos0 = k;
        sg.n_rows = lb - k;
        sg.S = lb;
        sg.ld = round4(lb);
        segs.push_back(sg);
      }
      soff.push_back(static_cast<long long>(used));
      sld.push_back(round4(lb));
      used += nb;
      gcu.push_back(cu_seqlens[b + 1] - cu_seqlens[b0]);
      ++b;
    }
    const int ng = b - b0;
    int split = 1, n_items = 0;
    if (!segs.empty()) {
      plan_segments(segs.data(), static_cast<int>(segs.size()), tok, &split, &n_items);
      if (cudaMemcpyAsync(segs_dev, segs.data(), segs.size() * sizeof(IndexerSeg), cudaMemcpyHostToDevice, st) !=
          cudaSuccess)
        return DSA_ERR_CUDA;
      e = run_indexer_segments(q_idx, total, q_scale, k_idx, total, k_scale, w, H_I, d_I, segs_dev,
                               static_cast<int>(segs.size()), split, n_items, sc, st);
      if (e != DSA_OK) return e;
    }
    if (cudaMemcpyAsync(gcu_dev, gcu.data(), size_t(ng + 1) * 8, cudaMemcpyHostToDevice, st) != cudaSuccess ||
        cudaMemcpyAsync(soff_dev, soff.data(), size_t(ng) * 8, cudaMemcpyHostToDevice, st) != cudaSuccess ||
        cudaMemcpyAsync(sld_dev, sld.data(), size_t(ng) * 4, cudaMemcpyHostToDevice, st) != cudaSuccess)
      return DSA_ERR_CUDA;
    const long long grows = gcu[ng];
    if (grows > 0) {
      const long long rbase = cu_seqlens[b0];
      if (launch_pdl(varlen_score_rows_kernel, dim3(static_cast<unsigned>((grows + 255) / 256)), dim3(256), 0, st,
                     static_cast<const long long*>(gcu_dev), ng, static_cast<const long long*>(soff_dev),
                     static_cast<const int*>(sld_dev), k, tk_off + rbase, tk_len + rbase) != cudaSuccess)
        return DSA_ERR_CUDA;
      e = last_launch_status();
      if (e != DSA_OK) return e;
      e = run_topk(sc, 0, tk_off + rbase, tk_len + rbase, 0, static_cast<int>(grows), k, idx + rbase * k, k, st);
      if (e != DSA_OK) return e;
    }
  }
  return run_mla(q, c, static_cast<int>(total), idx, row_off, static_cast<int>(total), H, k, scale, out, lse, st,
                 kMlaCausal);
}

uint64_t dsa_launch_count(void) { return g_launches.load(); }

int dsa_prefill_block_rows(int L, int k, int r0) {
  if (L <= 0 || k <= 0) return 0;
  return prefill_block_rows(L, k, r0);
}

dsa_status_t dsa_check_bounded_wait(int32_t* result, void* stream) {
  if (!result) return DSA_ERR_INVALID_ARG;
  if (!aligned16(result)) return DSA_ERR_ALIGNMENT;
  wait_selfcheck_kernel<<<1, 64, 0, static_cast<cudaStream_t>(stream)>>>(result);
  return last_launch_status();
}

size_t dsa_checks_selftest_bytes(void) { return size_t(1) << 20; }

dsa_status_t dsa_checks_selftest(int which, void* scratch, void* stream) {
  if (!scratch || (which != 0 && which != 1)) return DSA_ERR_INVALID_ARG;
  if (!aligned16(scratch)) return DSA_ERR_ALIGNMENT;
#ifndef DSA_CHECKS
  return DSA_ERR_UNSUPPORTED_SHAPE;
#else
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  char* b = static_cast<char*>(scratch);
  if (cudaMemsetAsync(b, 0, dsa_checks_selftest_bytes(), st) != cudaSuccess) return DSA_ERR_CUDA;
  if (which == 0) {
    // a top-k output row of k = 4 over n = 10 keys, not ascending: [5, 3, 7, -1]
    static const int32_t row[4] = {5, 3, 7, -1};
    static const int32_t n = 10;
    int32_t* idx = reinterpret_cast<int32_t*>(b);
    int32_t* len = reinterpret_cast<int32_t*>(b + 256);
    // (copies from pageable memory: the source is read before cudaMemcpyAsync returns)
    if (cudaMemcpyAsync(idx, row, sizeof(row), cudaMemcpyHostToDevice, st) != cudaSuccess ||
        cudaMemcpyAsync(len, &n, sizeof(n), cudaMemcpyHostToDevice, st) != cudaSuccess)
      return DSA_ERR_CUDA;
    TopkParams p{nullptr, 10, nullptr, len, 0, 1, 4, idx, 4, nullptr};
    topk_check_kernel<<<1, 256, 0, st>>>(p);
    return last_launch_status();
  }
  // one decode-style token with n = 200 keys of a 256-row zero latent, k = 128, 8 heads; its first selected
  // entry (250) lies inside the latent but beyond the token's keys
  constexpr int S = 256, H = 8, k = 128;
  uint16_t* c = reinterpret_cast<uint16_t*>(b);                           // [S, 576] bf16 zeros
  uint16_t* q = reinterpret_cast<uint16_t*>(b + S * 1152);                 // [1, H, 576] bf16 zeros
  int32_t* idx = reinterpret_cast<int32_t*>(b + S * 1152 + 16384);         // [1, k]
  int32_t* nk = idx + k;                                                   // [1]
  uint16_t* out = reinterpret_cast<uint16_t*>(b + S * 1152 + 32768);       // [1, H, 512] bf16
  float* lse = reinterpret_cast<float*>(b + S * 1152 + 49152);             // [1, H]
  struct Planted {
    int32_t v[k + 1];
    Planted() {
      for (int j = 0; j < k; ++j) v[j] = j;
      v[0] = 250;   // idx row [250, 1, 2, ..., 127]
      v[k] = 200;   // n_keys
    }
  };
  static const Planted host;
  if (cudaMemcpyAsync(idx, host.v, sizeof(host.v), cudaMemcpyHostToDevice, st) != cudaSuccess) return DSA_ERR_CUDA;
  return run_mla(q, c, S, idx, nullptr, 1, H, k, 0.0416666679f, out, lse, st, kMlaCounts, nk);
#endif
}

#ifdef DSA_TRACE
// traced build only: copy the event stamps out and clear them
__attribute__((visibility("default"))) int dsa_trace_read(unsigned long long* host) {
  if (cudaMemcpyFromSymbol(host, g_trace, sizeof(g_trace)) != cudaSuccess) return DSA_ERR_CUDA;
  static unsigned long long zero[kTraceEvents][kTraceTiles];
  return cudaMemcpyToSymbol(g_trace, zero, sizeof(zero)) == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}
#endif

size_t dsa_decode_workspace_size(int B, int64_t cache_rows, int H_I, int d_I, int H, int k) {
  (void)H_I; (void)d_I; (void)H;
  if (B <= 0 || cache_rows <= 0 || k <= 0) return 0;
  return decode_ws_bytes(B, decode_score_cap(B, cache_rows), k);
}

dsa_status_t dsa_forward_decode(int B, const int64_t* cache_off, const int32_t* ctx_len, const uint8_t* q_idx,
                                const float* q_scale, const float* w, const uint16_t* q, const uint8_t* k_new,
                                const float* k_scale_new, const uint16_t* c_new, uint8_t* k_cache,
                                float* k_scale_cache, uint16_t* c_cache, int64_t cache_rows, int H_I, int d_I,
                                int H, int k, float scale, int32_t* idx_out, uint16_t* out, float* lse, void* ws,
                                size_t ws_bytes, void* stream) {
  const dsa_status_t chk = decode_args_status(B, cache_off, ctx_len, q_idx, w, q, k_new, k_scale_new, c_new, k_cache,
                                              k_scale_cache, c_cache, cache_rows, H_I, d_I, H, k, idx_out, out);
  if (chk != DSA_OK) return chk;
  if (!ws || ws_bytes < dsa_decode_workspace_size(B, cache_rows, H_I, d_I, H, k)) return DSA_ERR_WORKSPACE;
  DecodeLayout lay{};
  lay.cache_off = reinterpret_cast<const long long*>(cache_off);
  lay.cache_rows = cache_rows;
  return run_decode(B, lay, ctx_len, q_idx, q_scale, w, q, k_new, k_scale_new, c_new, k_cache, k_scale_cache,
                    c_cache, decode_score_cap(B, cache_rows), H, k, scale, idx_out, out, lse, ws,
                    static_cast<cudaStream_t>(stream));
}

size_t dsa_decode_paged_workspace_size(int B, int max_pages, int page_rows, int H_I, int d_I, int H, int k) {
  (void)H_I; (void)d_I; (void)H;
  if (B <= 0 || max_pages <= 0 || page_rows <= 0 || k <= 0) return 0;
  return decode_ws_bytes(B, decode_score_cap(B, static_cast<int64_t>(B) * max_pages * page_rows), k);
}

dsa_status_t dsa_forward_decode_paged(int B, const int32_t* page_table, int max_pages, int page_rows,
                                      const int32_t* ctx_len, const uint8_t* q_idx, const float* q_scale,
                                      const float* w, const uint16_t* q, const uint8_t* k_new,
                                      const float* k_scale_new, const uint16_t* c_new, uint8_t* k_cache,
                                      float* k_scale_cache, uint16_t* c_cache, int num_pages, int H_I, int d_I,
                                      int H, int k, float scale, int32_t* idx_out, uint16_t* out, float* lse,
                                      void* ws, size_t ws_bytes, void* stream) {
  if (!page_table || max_pages <= 0 || num_pages <= 0) return DSA_ERR_INVALID_ARG;
  if (page_rows <= 0 || page_rows % 128 != 0) return DSA_ERR_UNSUPPORTED_SHAPE;
  const int64_t pool_rows = static_cast<int64_t>(num_pages) * page_rows;
  if (pool_rows > INT32_MAX) return DSA_ERR_UNSUPPORTED_SHAPE;   // tensor-map row coordinates are 32-bit
  // every check of the flat call applies, with the page pools as the caches (any non-null cache_off passes)
  const dsa_status_t chk = decode_args_status(B, reinterpret_cast<const int64_t*>(page_table), ctx_len, q_idx, w, q,
                                              k_new, k_scale_new, c_new, k_cache, k_scale_cache, c_cache, pool_rows,
                                              H_I, d_I, H, k, idx_out, out);
  if (chk != DSA_OK) return chk;
  if (!ws || ws_bytes < dsa_decode_paged_workspace_size(B, max_pages, page_rows, H_I, d_I, H, k))
    return DSA_ERR_WORKSPACE;
  DecodeLayout lay{};
  lay.cache_rows = pool_rows;
  lay.page_table = page_table;
  lay.max_pages = max_pages;
  lay.page_rows = page_rows;
  lay.num_pages = num_pages;
  return run_decode(B, lay, ctx_len, q_idx, q_scale, w, q, k_new, k_scale_new, c_new, k_cache, k_scale_cache,
                    c_cache, decode_score_cap(B, static_cast<int64_t>(B) * max_pages * page_rows), H, k, scale,
                    idx_out, out, lse, ws, static_cast<cudaStream_t>(stream));
}

// ------------------------------------------------------------------------------------------ no-allocation decode
// Scratch of dsa_forward_decode_noalloc: a file-scope device array, so the call needs no workspace from the
// caller.  Every GPU that loads the library holds it until the process exits.
static constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

namespace {
// Device address of g_noalloc_scratch on each device, looked up with that device current (host code may not use
// the array's name as a device address).  The address belongs to the context that loaded the module: it is kept
// together with that context and looked up again when the device's current context is another one (after a
// cudaDeviceReset, for instance).
constexpr int kMaxDevices = 64;
struct ScratchAddr {
  void* ctx = nullptr;
  void* ptr = nullptr;
};
ScratchAddr g_noalloc[kMaxDevices];
std::mutex g_noalloc_mutex;

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
CtxGetCurrentFn ctx_get_current_fn() {
  static CtxGetCurrentFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(p);
  });
  return fn;
}

dsa_status_t noalloc_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return DSA_ERR_CUDA;
  CtxGetCurrentFn get_ctx = ctx_get_current_fn();
  CUcontext ctx = nullptr;   // null while this thread has no current context yet
  if (!get_ctx || get_ctx(&ctx) != CUDA_SUCCESS) return DSA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  ScratchAddr& a = g_noalloc[dev];
  if (!a.ptr || !ctx || a.ctx != static_cast<void*>(ctx)) {
    void* ptr = nullptr;
    // the lookup makes the device's primary context current when it is not yet
    if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || !ptr) return DSA_ERR_CUDA;
    if (get_ctx(&ctx) != CUDA_SUCCESS || !ctx) return DSA_ERR_CUDA;
    a.ctx = ctx;
    a.ptr = ptr;
  }
  *out = a.ptr;
  return DSA_OK;
}
}  // namespace

size_t dsa_decode_noalloc_scratch_bytes(void) { return kNoAllocScratchBytes; }

dsa_status_t dsa_forward_decode_noalloc(int B, const int64_t* cache_off, const int32_t* ctx_len,
                                        const uint8_t* q_idx, const float* q_scale, const float* w,
                                        const uint16_t* q, const uint8_t* k_new, const float* k_scale_new,
                                        const uint16_t* c_new, uint8_t* k_cache, float* k_scale_cache,
                                        uint16_t* c_cache, int64_t cache_rows, int H_I, int d_I, int H, int k,
                                        float scale, int32_t* idx_out, uint16_t* out, float* lse, void* stream) {
  const dsa_status_t chk = decode_args_status(B, cache_off, ctx_len, q_idx, w, q, k_new, k_scale_new, c_new, k_cache,
                                              k_scale_cache, c_cache, cache_rows, H_I, d_I, H, k, idx_out, out);
  if (chk != DSA_OK) return chk;
  if (dsa_decode_workspace_size(B, cache_rows, H_I, d_I, H, k) > kNoAllocScratchBytes) return DSA_ERR_WORKSPACE;
  void* scratch = nullptr;
  const dsa_status_t e = noalloc_scratch(&scratch);
  if (e != DSA_OK) return e;
  // the scratch needs no clearing: every byte a call reads there is written earlier in the same call
  return dsa_forward_decode(B, cache_off, ctx_len, q_idx, q_scale, w, q, k_new, k_scale_new, c_new, k_cache,
                            k_scale_cache, c_cache, cache_rows, H_I, d_I, H, k, scale, idx_out, out, lse, scratch,
                            kNoAllocScratchBytes, stream);
}

}  // extern "C"
