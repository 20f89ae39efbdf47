// Sparse MLA attention in MQA mode (velog.io DSA page, §1.2-§1.3): for each query token t and head h,
//   u[t,h] = softmax_{s in S_t}(scale * q[t,h] . c_s) . c_s[:512],   S_t = the selected latent entries.
//
// Why a 2-CTA cluster per token.  All 128 heads of a token share the same selected entries, so heads form
// the M = 128 dimension of the MMAs and every gathered entry is reused by all heads.  The output of one token
// (128 heads x 512 fp32) fills all 512 columns of one SM's tensor memory, leaving no room for the logits.
// The work is therefore split by role across the two CTAs of a cluster, each on its own SM:
//   score CTA (rank 0): keeps the token's queries on chip, gathers the 576-dim selected rows, computes
//     S = Q . C^T on tcgen05 (bf16 -> fp32), runs the online softmax (fp32, exp2 domain) and stores P (bf16)
//     plus per-head rescale factors and row sums straight into the value CTA's shared memory;
//   value CTA (rank 1): gathers the first 512 dims of the same rows, accumulates O += P . V on tcgen05 into
//     its tensor memory (two N = 256 halves), rescales O rows when a head's running maximum jumps (lazy:
//     only when the max grows by more than 2^8), and writes out = O / l in bf16.
// The QK^T and PV contractions (576 and 512 deep per key) are thus balanced across the two SMs, and no
// logit or probability ever leaves the chip.
//
// Data movement.
//   * Keys are processed in tiles of 128: the QK^T MMAs then have N = 128 (the tensor core ran the N = 64 ones
//     of 64-key tiles at about 40 % of its rate).  The score CTA's tensor memory holds Q chunks 0..7 (128 heads
//     x 64 dims each, 32 columns) in columns 0..255 and two 128-column S buffers, so the QK^T of tile g + 1
//     runs while the softmax reads tile g's logits.  Q chunk 8 (the 64 position dims) is the A operand of its
//     MMAs from shared memory, loaded for the next token as soon as the current token's last MMAs reading it
//     have retired.
//   * Selected rows are gathered by TMA tile::gather4 (four rows x one 64-column, 128-byte swizzled box per
//     instruction) into 128-key x 64-dim chunks in the K-major form the tensor core reads.  A pipeline stage
//     holds several chunks of one tile (three in the score CTA, four in the value CTA): each gather warp spends
//     about 300 ns per stage on its barrier handshake whatever the stage's size, so a stage gives each warp a
//     dozen or more gather4 to issue.  The ring is as deep as shared memory allows (three stages, 144 KB, in
//     the score CTA; two, 128 KB, in the value CTA): a gather takes about 1.5 us to land under load, so the
//     bytes in flight set the rate.  With every SM gathering random rows of a 151 MB latent and each stage
//     freed as soon as it landed, one SM's gathers ran at about 44 GB/s with two 48 KB stages, 66 with four,
//     and 73 with three 64 KB stages (near the TMA unit's limit of about 75).  Each stage is split over eight
//     gather warps (one warp issues gather4 only about every 50 ns; gather throughput per SM grows with the
//     issuing warps: about 12, 24, 45 and 73 GB/s with 1, 2, 4 and 8), each of which arrives on the stage's
//     barrier with its share of the bytes.  TMA
//     writes are in the async proxy, so the MMA warp consumes a stage as soon as its mbarrier completes,
//     with no proxy fence.  The same chunk bytes serve as the K-major B operand of QK^T (rows = keys) and
//     as the MN-major B operand of PV (rows = keys = K, 64 dims = N per atom; four chunks = N 256).
//   * P goes to the value CTA by st.async stores from the softmax threads, each completing its bytes on the
//     value CTA's P_FULL barrier: no staging buffer, and no bulk copy queued behind the gathers in the score
//     SM's TMA unit (such a copy took about 1.2 us per tile there).
//   * The token's selected-index row is prefetched into shared memory with one bulk copy.
//   * Q chunks 0..7 are staged by TMA (three shared-memory slots) and copied into tensor memory with
//     tcgen05.cp.  A copy may only overwrite a slot once the MMAs that last read it have completed, which the
//     MMA thread learns from tcgen05.commit barriers on the stages of a token's last tile: the next token's
//     chunks 0-2 are copied during that tile, chunks 3-5 and 6-7 in the next token's first tile, just
//     before the stages that read them.
//
// Warp roles (14 warps per CTA): w0 loader (index rows, Q chunks), w1 TMEM allocation + MMA issue (a
// warp-uniform loop; one elected lane issues the tcgen05 instructions),
// w2 w3 w8..w13 gathers, w4..w7 softmax (score CTA) or correction / epilogue (value CTA); warp w owns TMEM
// lanes (= heads) 32 * (w % 4) .. +31.
#pragma once
#include "common.cuh"

namespace dsa {

// How a token's keys are found.  kMlaSparse: the k entries of its index row are gathered.  The dense modes
// give each token the number n_t of keys its sequence shows it (positions 0..n_t-1, rows base..base+n_t-1 of
// c); a token with n_t <= k then selects all of them, whatever its index row says, and its keys are read as
// contiguous 128-row tiles, ceil(n_t / 128) of them (at least one), instead of ceil(k / 128) gathered tiles.
// kMlaCausal: n_t = pos0 + t - base + 1 (prefill rows at their positions, the launch's first row at position
// pos0); kMlaCounts: n_t = n_keys[t] (decode tokens after the append).
enum { kMlaSparse = 0, kMlaCausal = 1, kMlaCounts = 2 };

struct MlaParams {
  const int* idx;              // [T, k]
  const long long* row_off;    // [T] row of entry 0 of each token in c, or null (0)
  const int* n_keys;           // [T] keys of each token (kMlaCounts), else null
  uint16_t* out;               // [T, H, 512] bf16
  float* lse;                  // [T, H] or null
  int T, H, k;
  int dense;                   // kMlaSparse / kMlaCausal / kMlaCounts
  int pos0;                    // kMlaCausal: position of the launch's token 0 in its sequence
  // KL mode (kl_out non-null): no attention output; every CTA runs the score role on its own tokens and writes
  // kl_out[t] = KL(p_t || Softmax(I_t)) over the token's keys, p_t the heads' attention probabilities (from the
  // logits and the attention's lse [T, H]) summed and L1-normalised, I_t = kl_scores [T, k] (the index score of
  // each selected entry)
  const float* kl_lse;
  const float* kl_scores;
  float* kl_out;
  const int* page_table;       // paged c: [T, pt_stride] page of each page_rows positions of token t's keys, or null
  int pt_stride, page_rows;    // (page_rows a multiple of 128: a 128-key tile lies in one page)
  long long S;                 // rows of c
  float scale_log2;            // softmax scale * log2(e)
};

namespace mla {
// 128-key tiles: the QK^T MMAs have N = 128 (the tensor core ran N = 64 MMAs at about 40 % of its rate, N = 256
// ones near the full rate).  Two 128-column S buffers fit in tensor memory beside eight of the nine Q chunks; the
// ninth (the 64 position dims) is the A operand of its MMAs from shared memory.
constexpr int NK = 128;                   // keys per tile
constexpr int D = 576, DV = 512;
constexpr int QCHUNKS = D / 64;           // 9
constexpr int QTM = 8;                    // Q chunks in tensor memory (chunk 8 from shared memory)
constexpr int VCHUNKS = DV / 64;          // 8
constexpr int CHUNK_BYTES = NK * 128;     // 16 KB: 128 keys x 64 bf16
constexpr int QCHUNK_BYTES = 128 * 128;   // 16 KB: 128 heads x 64 bf16
constexpr int KMAX = 2048;                // largest selection handled (index row slot of 8 KB)
constexpr int QS = 3;                     // Q staging slots (score CTA)
constexpr int NPB = 2;                    // P buffers (value CTA)
constexpr int SCH = 3, VCH = 4;           // 64-dim chunks per gather stage (score CTA, value CTA)
constexpr int S_STAGE = SCH * CHUNK_BYTES, V_STAGE = VCH * CHUNK_BYTES;
constexpr int SPT_S = QCHUNKS / SCH, SPT_V = VCHUNKS / VCH;   // stages per 128-key tile: 3, 2
constexpr int NS_S = 3, NS_V = 2;         // gather stages per CTA (KL mode: NS_S - 1, its head sums in the last)
constexpr int THREADS = 448;
constexpr int GATHER_WARPS = 8;
constexpr int G4_PER_CHUNK = NK / 4;      // gather4 instructions per chunk (four rows each)
constexpr float RESCALE_LOG2 = 8.0f;      // lazy rescale threshold (factor 256)
constexpr int P_CHUNK = 128 * 128;        // one 64-key K chunk of P: 128 heads x 64 keys bf16
constexpr int P_BYTES = 2 * P_CHUNK;      // 128 heads x 128 keys bf16
constexpr int XFER = P_BYTES + 512 + 512; // P + alpha[128] + lsum[128]: the bytes of one tile to the value CTA
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t TQ = 0;                // score CTA: Q chunks 0..7 in columns 0..255
constexpr uint32_t TS = 256;              // score CTA: S buffers in columns 256..383 and 384..511
// barrier slots
constexpr int B_IDX_FULL = 0, B_IDX_EMPTY = 2;
constexpr int B_QST_FULL = 4, B_QST_EMPTY = B_QST_FULL + QS;
constexpr int B_RING_FULL = B_QST_EMPTY + QS, B_RING_EMPTY = B_RING_FULL + 16;
constexpr int B_S_FULL = B_RING_EMPTY + 16, B_S_EMPTY = B_S_FULL + 2, B_P_EMPTY = B_S_EMPTY + 2;
constexpr int B_P_FULL = B_P_EMPTY + NPB, B_P_READY = B_P_FULL + NPB;
// O_DONE: one barrier per P buffer (PV of tile g completes O_DONE[g % NPB]); a single barrier would be waited
// only now and then and could be two phases behind, where a parity test cannot tell the phases apart
constexpr int B_O_DONE = B_P_READY + NPB, B_O_FREE = B_O_DONE + NPB;
constexpr int B_QRET = B_O_FREE + 1;          // score CTA: stage s of a token's last tile retired (3 barriers)
constexpr int B_ROPE_FULL = B_QRET + SPT_S;   // score CTA: Q chunk 8 of a token staged
constexpr int B_ROPE_EMPTY = B_ROPE_FULL + 1; // score CTA: every MMA reading Q chunk 8 of a token retired
constexpr int B_RED_FULL = B_ROPE_EMPTY + 1;  // KL mode: the four warps' head sums of a tile written (2 buffers)
constexpr int B_RED_FREE = B_RED_FULL + 2;    // KL mode: the head sums of a tile read (2 buffers)
constexpr int B_COUNT = B_RED_FREE + 2;
// shared memory map (from a 1024-byte aligned base; both CTAs use the same barrier offsets)
constexpr int OFF_TMEM = 8 * B_COUNT;
constexpr int OFF_ABORT = OFF_TMEM + 4;
constexpr int OFF_CHECK = 576;                                  // DSA_CHECKS: per warp, key tiles walked (16 ints)
constexpr int OFF_IDX = 1024;                                   // both: 2 x 8 KB index rows
constexpr int OFF_QST = OFF_IDX + 2 * KMAX * 4;                 // score CTA: Q staging
constexpr int OFF_ROPE = OFF_QST + QS * QCHUNK_BYTES;           // score CTA: Q chunk 8 of the current token
constexpr int OFF_RING_S = OFF_ROPE + QCHUNK_BYTES;             // score CTA: gather ring
constexpr int OFF_RED = OFF_RING_S + (NS_S - 1) * S_STAGE;      // score CTA, KL mode: head sums [2][4][NK]
constexpr int OFF_PB = OFF_IDX + 2 * KMAX * 4;                  // value CTA: P buffers
constexpr int OFF_RING_V = OFF_PB + NPB * XFER;                 // value CTA: gather ring
constexpr int SMEM_S = OFF_RING_S + NS_S * S_STAGE;
constexpr int SMEM_V = OFF_RING_V + NS_V * V_STAGE;
constexpr int SMEM = (SMEM_S > SMEM_V ? SMEM_S : SMEM_V) + 1024;
static_assert(OFF_ABORT + 4 <= OFF_CHECK && OFF_CHECK + 64 <= OFF_IDX, "barrier area");
static_assert(OFF_QST % 1024 == 0 && OFF_ROPE % 1024 == 0 && OFF_RING_S % 1024 == 0, "1 KB aligned tiles");
static_assert(2 * 4 * NK * 4 <= S_STAGE, "KL mode: head sums in the ring's last stage");
static_assert(OFF_PB % 1024 == 0 && XFER % 1024 == 0 && OFF_RING_V % 1024 == 0, "1 KB aligned tiles");
static_assert(QCHUNKS % SCH == 0 && VCHUNKS % VCH == 0 && VCH * 64 == 256, "stage split");
static_assert(QTM == QCHUNKS - 1 && SPT_S == 3, "Q chunk 8 in the last score stage");
static_assert(TQ + 32 * QTM <= TS && TS + 2 * NK <= TMEM_COLS, "tensor memory columns");
static_assert((SCH * G4_PER_CHUNK) % GATHER_WARPS == 0 && (VCH * G4_PER_CHUNK) % GATHER_WARPS == 0,
              "gather4 split over warps");
static_assert((SCH * G4_PER_CHUNK) / GATHER_WARPS <= 32 && (VCH * G4_PER_CHUNK) / GATHER_WARPS <= 32,
              "one gather4 per lane");
static_assert(NS_S <= 16 && NS_V <= 16, "ring barrier slots");
static_assert(SMEM <= 232448, "shared memory per CTA");
}  // namespace mla

// The kernel is instantiated per feature set (DENSE: the dense modes; PAGED: a page table; KL: the objective), so that
// each launch runs code with none of the branches of the features it does not use: the attention's warps run from
// the instruction cache, and code for an unused feature in their loops showed up as instruction-fetch stalls.

// Row of c holding position `pos` (>= 0) of token t's keys: base + pos, or through the token's page-table row.
template <bool PAGED>
__device__ __forceinline__ long long mla_pos_row(const MlaParams& p, int t, long long base, long long pos) {
  if constexpr (!PAGED) {
    return base + pos;
  } else {
    const int* pr = p.page_table + static_cast<long long>(t) * p.pt_stride;
    return static_cast<long long>(pr[pos / p.page_rows]) * p.page_rows + pos % p.page_rows;
  }
}
// Whether selection entry e of token t names a row of c (an entry of -1 is padding; anything else outside the
// token's keys is an error).
template <bool PAGED>
__device__ __forceinline__ bool mla_valid(const MlaParams& p, int t, int e, long long base) {
  if (e < 0) return false;
  if (PAGED && e >= static_cast<long long>(p.pt_stride) * p.page_rows) return false;
  const long long r = mla_pos_row<PAGED>(p, t, base, e);
  return r >= 0 && r < p.S;
}
// Row of c gathered for selection entry e (in slot `slot` of its token's k entries).  An empty or invalid entry is
// masked out of the softmax but its stage still holds a row: it reads row `slot` (any row in [0, S) would do), so
// that the padding of short rows spreads over many L2 lines instead of hammering one.
template <bool PAGED>
__device__ __forceinline__ long long mla_row(const MlaParams& p, int t, int e, long long base, int slot) {
  const bool valid = mla_valid<PAGED>(p, t, e, base);
  if (!valid && e != -1) raise_status(DSA_ERR_BAD_INDEX);
  if constexpr (kChecks) {
    // DSA_CHECKS: where the token's key count n is known, a selected entry lies below it (causality)
    if (valid && p.dense != kMlaSparse) {
      const long long n = (p.dense == kMlaCausal) ? static_cast<long long>(p.pos0) + t - base + 1 : p.n_keys[t];
      check_that(e < n, DSA_ERR_BAD_INDEX);
    }
  }
  return valid ? mla_pos_row<PAGED>(p, t, base, e) : (slot < p.S ? slot : 0);
}

// mla_row of four consecutive entries over a page table: the four page-table loads are issued before any of
// them is used (checked one entry at a time, each load would wait behind the previous entry's check and possible
// status write, and a tile would pay four global-memory latencies in sequence).
__device__ __forceinline__ void mla_rows_paged(const MlaParams& p, int t, int4 e4, long long base, int slot,
                                               int (&r)[4]) {
  const int e[4] = {e4.x, e4.y, e4.z, e4.w};
  const int* pr = p.page_table + static_cast<long long>(t) * p.pt_stride;
  const long long lim = static_cast<long long>(p.pt_stride) * p.page_rows;
  int pg[4];
#pragma unroll
  for (int u = 0; u < 4; ++u) pg[u] = (e[u] >= 0 && e[u] < lim) ? __ldg(pr + e[u] / p.page_rows) : -1;
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const long long row = static_cast<long long>(pg[u]) * p.page_rows + e[u] % p.page_rows;
    const bool valid = pg[u] >= 0 && row < p.S;
    if (!valid && e[u] != -1) raise_status(DSA_ERR_BAD_INDEX);
    if constexpr (kChecks) {
      if (valid && p.dense != kMlaSparse) {
        const long long n = (p.dense == kMlaCausal) ? static_cast<long long>(p.pos0) + t - base + 1 : p.n_keys[t];
        check_that(e[u] < n, DSA_ERR_BAD_INDEX);
      }
    }
    r[u] = static_cast<int>(valid ? row : (slot + u < p.S ? slot + u : 0));
  }
}

// Number of keys n_t of token t when it takes the dense path (n_t <= k), -1 when its index row is gathered.
template <bool DENSE>
__device__ __forceinline__ int mla_dense_keys(const MlaParams& p, int t, long long base) {
  if constexpr (!DENSE) {
    return -1;
  } else {
    if (p.dense == kMlaSparse) return -1;
    const long long n = (p.dense == kMlaCausal) ? static_cast<long long>(p.pos0) + t - base + 1 : p.n_keys[t];
    if (n > p.k) return -1;
    return n > 0 ? static_cast<int>(n) : 0;
  }
}
// Which of the 128 keys of tile j of token t enter the softmax, as four warp-uniform ballots: lane l tests the keys
// in slots j NK + 4 l .. + 3, and key i of the tile is valid iff bit i / 4 of msk[i % 4] is set.  A gathered token's
// key is valid when its slot is below k and its entry names a row of c; a dense token's when its position is below n_t.
template <bool DENSE, bool PAGED>
__device__ __forceinline__ void mla_tile_masks(const MlaParams& p, int t, const int* ids, long long base, int nd, int j,
                                               int lane, uint32_t (&msk)[4]) {
  const int slot = j * mla::NK + 4 * lane;
  bool v[4];
  if (nd < 0) {
    const int4 e = (slot < p.k) ? *reinterpret_cast<const int4*>(ids + slot) : make_int4(-1, -1, -1, -1);
    v[0] = mla_valid<PAGED>(p, t, e.x, base);
    v[1] = mla_valid<PAGED>(p, t, e.y, base);
    v[2] = mla_valid<PAGED>(p, t, e.z, base);
    v[3] = mla_valid<PAGED>(p, t, e.w, base);
  } else {
#pragma unroll
    for (int u = 0; u < 4; ++u) v[u] = slot + u < nd;
  }
#pragma unroll
  for (int u = 0; u < 4; ++u) msk[u] = __ballot_sync(0xffffffffu, v[u]);
}
// 128-key tiles of a token: the tiles holding its k selection slots, or its n_t dense keys (at least one; slots past
// k or keys past n_t are masked)
__device__ __forceinline__ int mla_tiles(const MlaParams& p, int nd) {
  return max(1, ((nd < 0 ? p.k : nd) + mla::NK - 1) / mla::NK);
}

// position in a ring of `size` stages (size known at run time): stage index and pass parity, advanced
// incrementally so that no division runs in the per-chunk loops
struct RingPos {
  int stage = 0;
  uint32_t phase = 0;
  int size = 1;
  __device__ __forceinline__ void advance() {
    if (++stage == size) { stage = 0; phase ^= 1; }
  }
};

// every lane waits (bounded); the warp then agrees on the outcome so that it stays converged
template <bool kCluster = false>
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag) {
  const bool ok = mbar_wait<kCluster>(bar, parity, abort_flag);
  return __all_sync(0xffffffffu, ok);
}

// KL selects the indexer-objective instantiation (p.kl_out set): a separate kernel, so that the attention's code
// carries none of the objective's unrolled loops (the warps of the attention run from the instruction cache).
template <bool KL, bool DENSE, bool PAGED>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(mla::THREADS, 1)
sparse_mla_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_c,
                  const __grid_constant__ CUtensorMap tm_cd, const MlaParams p) {
  using namespace mla;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  auto bar = [&](int slot) -> uint32_t { return sbase + 8 * slot; };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + OFF_ABORT);
  const int warp = warp_id(), lane = lane_id();
  // 0 = score CTA, 1 = value CTA; in KL mode every CTA takes the score role on tokens of its own
  constexpr bool kl_mode = KL;
  const uint32_t rank = kl_mode ? 0u : cluster_rank();
  const int cluster = kl_mode ? static_cast<int>(blockIdx.x) : static_cast<int>(blockIdx.x >> 1);
  const int nclusters = kl_mode ? static_cast<int>(gridDim.x) : static_cast<int>(gridDim.x >> 1);
  const int nsr = (rank == 0) ? (KL ? NS_S - 1 : NS_S) : NS_V;
  const uint32_t ring = sbase + ((rank == 0) ? OFF_RING_S : OFF_RING_V);
  const int* idx_s = reinterpret_cast<const int*>(smem + OFF_IDX);

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(B_IDX_FULL + i), 1);
      mbar_init(bar(B_IDX_EMPTY + i), rank == 0 ? GATHER_WARPS + 4 : GATHER_WARPS);
    }
    for (int i = 0; i < 16; ++i) {
      mbar_init(bar(B_RING_FULL + i), GATHER_WARPS);     // each gather warp's arrive.expect_tx + TMA bytes
      mbar_init(bar(B_RING_EMPTY + i), 1);
    }
    if (rank == 0) {
      for (int i = 0; i < QS; ++i) { mbar_init(bar(B_QST_FULL + i), 1); mbar_init(bar(B_QST_EMPTY + i), 1); }
      for (int i = 0; i < 2; ++i) { mbar_init(bar(B_S_FULL + i), 1); mbar_init(bar(B_S_EMPTY + i), 4); }
      for (int i = 0; i < NPB; ++i) mbar_init(bar(B_P_EMPTY + i), 1);
      for (int i = 0; i < SPT_S; ++i) mbar_init(bar(B_QRET + i), 1);
      mbar_init(bar(B_ROPE_FULL), 1);
      mbar_init(bar(B_ROPE_EMPTY), 1);
      for (int i = 0; i < 2; ++i) { mbar_init(bar(B_RED_FULL + i), 4); mbar_init(bar(B_RED_FREE + i), 1); }
    } else {
      for (int i = 0; i < NPB; ++i) { mbar_init(bar(B_P_FULL + i), 1); mbar_init(bar(B_P_READY + i), 4); }
      for (int i = 0; i < NPB; ++i) mbar_init(bar(B_O_DONE + i), 1);
      mbar_init(bar(B_O_FREE), 4);
    }
    *abort_flag = 0;
    if constexpr (kChecks) {
      for (int i = 0; i < 16; ++i) reinterpret_cast<int*>(smem + OFF_CHECK)[i] = -1;
    }
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tm_c);
    if (DENSE && p.dense != kMlaSparse) prefetch_tmap(&tm_cd);
    if (rank == 0) prefetch_tmap(&tm_q);
  }
  if (warp == 1) {
    tmem_alloc(sbase + OFF_TMEM, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();        // both CTAs' barriers are initialised before any remote arrive
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + OFF_TMEM);
  // DSA_CHECKS: key tiles this thread's role walked over its tokens (every role of a CTA walks the same tokens)
  [[maybe_unused]] int chk_tiles = 0;
  [[maybe_unused]] bool chk_ran = false;
  // the set-up above touches no global memory; from here on the predecessor's results are read
  pdl_allow_next();
  pdl_wait();

  if (warp == 0) {
    // ===================================================================== loader
    if (lane == 0) {
      int qn = 0, ti = 0;
      bool ok = true;
      int idx_issued = 0, q_issued = 0;
      uint32_t idx_par[2] = {0, 0}, q_par[QS] = {};
      for (int t = cluster; t < p.T && ok; t += nclusters, ++ti) {
        const int is = ti & 1;
        if (!(ok = mbar_wait(bar(B_IDX_EMPTY + is), ((ti >> 1) & 1) ^ 1, abort_flag))) break;
        mbar_arrive_expect_tx(bar(B_IDX_FULL + is), p.k * 4);
        bulk_load(sbase + OFF_IDX + is * KMAX * 4, p.idx + static_cast<long long>(t) * p.k, p.k * 4,
                  bar(B_IDX_FULL + is));
        idx_par[is] = (ti >> 1) & 1;
        ++idx_issued;
        if (rank == 0) {
          // chunks 0..7 through the staging slots, copied into tensor memory by the MMA warp
          for (int c = 0; c < QTM; ++c, ++qn) {
            const int qs = qn % QS;
            if (!(ok = mbar_wait(bar(B_QST_EMPTY + qs), ((qn / QS) & 1) ^ 1, abort_flag))) break;
            mbar_arrive_expect_tx(bar(B_QST_FULL + qs), QCHUNK_BYTES);
            tma_load_3d(sbase + OFF_QST + qs * QCHUNK_BYTES, &tm_q, bar(B_QST_FULL + qs), 64 * c, 0, t);
            q_par[qs] = (qn / QS) & 1;
            ++q_issued;
          }
        }
      }
      if (*abort_flag) {
        for (int i = 0; i < 2 && i < idx_issued; ++i) mbar_wait_drain(bar(B_IDX_FULL + i), idx_par[i]);
        for (int i = 0; i < QS && i < q_issued; ++i) mbar_wait_drain(bar(B_QST_FULL + i), q_par[i]);
      }
    } else if (lane == 1 && rank == 0) {
      // chunk 8 (the position dims) of each token into its buffer, read by the MMAs from shared memory: loaded as
      // soon as the previous token's last MMAs reading it have retired, on a lane of its own so that the Q chunk
      // staging above never waits for it
      int ti = 0, issued = 0;
      bool ok = true;
      for (int t = cluster; t < p.T && ok; t += nclusters, ++ti) {
        if (!(ok = mbar_wait(bar(B_ROPE_EMPTY), (ti & 1) ^ 1, abort_flag))) break;
        mbar_arrive_expect_tx(bar(B_ROPE_FULL), QCHUNK_BYTES);
        tma_load_3d(sbase + OFF_ROPE, &tm_q, bar(B_ROPE_FULL), 64 * QTM, 0, t);
        ++issued;
      }
      if (*abort_flag && issued) mbar_wait_drain(bar(B_ROPE_FULL), (issued - 1) & 1);
    }
  } else if (warp == 2 || warp == 3 || warp >= 8) {
    // ===================================================================== gathers (TMA gather4)
    // Every stage is split over the eight gather warps: gather4 instruction i of a stage (i = 32 cc + rg)
    // fetches rows 4 rg .. 4 rg + 3 of the tile into its chunk cc; warp gw issues instructions
    // gw * per_warp .. + per_warp - 1, one per lane.  A dense token's full tiles are 128 contiguous rows: lane c
    // of gather warp 0 loads its chunk c as one 64 x 128 box, and the other warps arrive with no bytes.  Its
    // last, partial tile is gathered, its masked slots reading the token's last key row: the rows after the
    // sequence's last key may be memory the caller never wrote, and a NaN there would survive the zero
    // probability in P . V.
    const int gw = (warp < 8) ? warp - 2 : warp - 6;
    const int cps = (rank == 0) ? SCH : VCH;               // chunks per stage
    const int spt = (rank == 0) ? SPT_S : SPT_V;           // stages per tile
    const uint32_t sbytes = cps * CHUNK_BYTES;
    const int per_warp = cps * G4_PER_CHUNK / GATHER_WARPS; // 12 or 16
    const int gi = gw * per_warp + lane;
    const int cc = gi / G4_PER_CHUNK, rg = gi % G4_PER_CHUNK;
    const bool active = lane < per_warp;
    RingPos rp;
    rp.size = nsr;
    bool issued = false;               // this warp issued a load into the ring
    RingPos last;                      // ring position of its latest stage
    int ti = 0;
    bool ok = true;
    for (int t = cluster; t < p.T && ok; t += nclusters, ++ti) {
      const int is = ti & 1;
      if (!(ok = warp_wait(bar(B_IDX_FULL + is), (ti >> 1) & 1, abort_flag))) break;
      const int* ids = idx_s + is * KMAX;
      const long long base = p.row_off ? p.row_off[t] : 0;
      const int nd = mla_dense_keys<DENSE>(p, t, base);
      const int ntiles = mla_tiles(p, nd);
      if constexpr (kChecks) { chk_tiles += ntiles; chk_ran = true; }
      for (int j = 0; j < ntiles && ok; ++j) {
        const bool full_dense = nd >= 0 && (j + 1) * NK <= nd;    // 128 contiguous rows of keys
        const uint32_t tx = full_dense ? (gw == 0 ? sbytes : 0) : per_warp * 512;
        int r[4] = {0, 0, 0, 0};
        if (active && !full_dense) {
          const int slot = j * NK + 4 * rg;
          if (nd < 0) {
            // slots past the token's k entries (a k that is not a multiple of the tile) are padding
            const int4 e = (slot < p.k) ? *reinterpret_cast<const int4*>(ids + slot) : make_int4(-1, -1, -1, -1);
            if constexpr (PAGED) {
              mla_rows_paged(p, t, e, base, slot, r);
            } else {
              r[0] = static_cast<int>(mla_row<PAGED>(p, t, e.x, base, slot));
              r[1] = static_cast<int>(mla_row<PAGED>(p, t, e.y, base, slot + 1));
              r[2] = static_cast<int>(mla_row<PAGED>(p, t, e.z, base, slot + 2));
              r[3] = static_cast<int>(mla_row<PAGED>(p, t, e.w, base, slot + 3));
            }
          } else {
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const int pos = slot + u;
              r[u] = static_cast<int>(nd > 0 ? mla_pos_row<PAGED>(p, t, base, pos < nd ? pos : nd - 1)
                                             : (pos < p.S ? pos : 0));
            }
          }
        }
        for (int s = 0; s < spt; ++s, rp.advance()) {
          const int st = rp.stage;
          bool got = true;
          if (lane == 0) {
            got = mbar_wait(bar(B_RING_EMPTY + st), rp.phase ^ 1, abort_flag);
            if (got) {
              if (tx) mbar_arrive_expect_tx(bar(B_RING_FULL + st), tx);
              else mbar_arrive(bar(B_RING_FULL + st));
            }
          }
          if (!(ok = __shfl_sync(0xffffffffu, got, 0))) break;
          if (lane == 0 && gw == 0 && s == 0) DSA_TRACE_EVENT(rank == 0 ? 0 : 16, ti * ntiles + j);
          if (!full_dense) {
            if (active)
              tma_gather4(ring + st * sbytes + cc * CHUNK_BYTES + rg * 512, &tm_c, bar(B_RING_FULL + st),
                          64 * (s * cps + cc), r[0], r[1], r[2], r[3]);
          } else if (gw == 0 && lane < cps) {
            tma_load_2d(ring + st * sbytes + lane * CHUNK_BYTES, &tm_cd, bar(B_RING_FULL + st),
                        64 * (s * cps + lane), static_cast<int>(mla_pos_row<PAGED>(p, t, base, j * NK)));
          }
          issued = true;
          last = rp;
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(B_IDX_EMPTY + is));
    }
    if (lane == 0 && *abort_flag && issued) {
      // leave no gather in flight into this CTA's shared memory: bounded waits on the stages of the last pass
      // over the ring (stages up to this warp's last one in that pass' parity, the others one pass earlier)
      for (int st = 0; st < nsr; ++st)
        mbar_wait_drain(bar(B_RING_FULL + st), st <= last.stage ? last.phase : last.phase ^ 1);
    }
  } else if (warp == 1) {
    // ===================================================================== MMA issue
    // The whole warp runs the loop (every wait is warp-uniform); one elected lane issues each tcgen05 op.
    bool ok = true;
    int g = 0;
    RingPos rp;
    rp.size = nsr;
    int ti = 0;
    if (rank == 0) {
      // Q chunks 0..7 of a token live in tensor-memory slots 0..7, chunk 8 in its shared-memory buffer.
      // A copy overwrites a slot only after the MMAs that last read it have completed (tcgen05.commit barriers
      // QRET[s], stage s of a token's last tile): the next token's chunks 0..2 are copied during the last tile,
      // after the stage that follows stage 0 (stage 2 for a one-tile token, so that chunks leave the staging
      // slots in order), chunks 3..5 and 6..7 in its own first tile, just before stages 1 and 2 read them.
      constexpr uint32_t idesc = idesc_bf16(128, NK, false);
      int qn = 0;          // Q chunks copied into tensor memory so far (= 8 * token index + chunk)
      // copy the next `n` staged Q chunks (global chunk index qn ...) into their tensor-memory slots
      auto copy_q = [&](int n) -> bool {
        for (int i = 0; i < n; ++i, ++qn) {
          const int qs = qn % QS;
          if (!warp_wait(bar(B_QST_FULL + qs), (qn / QS) & 1, abort_flag)) return false;
          tc_fence_after();
          const uint32_t src = sbase + OFF_QST + qs * QCHUNK_BYTES;
          const uint32_t dst = tmem + TQ + 32 * (qn % QTM);
          if (elect_one()) {
#pragma unroll
            for (int s = 0; s < 4; ++s) tmem_cp_128x256b(dst + 8 * s, smem_desc(src + 32 * s, 16, 1024, kLayoutSW128));
            mma_commit(bar(B_QST_EMPTY + qs));
          }
          __syncwarp();
        }
        return true;
      };
      int nret = 0;        // tokens whose last tile committed the QRET barriers
      if (cluster < p.T) ok = copy_q(QTM);
      for (int t = cluster; t < p.T && ok; t += nclusters, ++ti) {
        const bool has_next = t + nclusters < p.T;
        const int ntiles = mla_tiles(p, mla_dense_keys<DENSE>(p, t, p.row_off ? p.row_off[t] : 0));
        if constexpr (kChecks) { chk_tiles += ntiles; chk_ran = true; }
        for (int j = 0; j < ntiles && ok; ++j, ++g) {
          const int sb = static_cast<int>(g & 1);
          const bool last = (j == ntiles - 1);
          if (!(ok = warp_wait(bar(B_S_EMPTY + sb), static_cast<uint32_t>((g >> 1) & 1) ^ 1, abort_flag))) break;
          DSA_TRACE_EVENT(2, g);
          tc_fence_after();
          for (int s = 0; s < SPT_S && ok; ++s, rp.advance()) {
            const int st = rp.stage;
            if (j == 0 && s > 0 && ti > 0) {
              // this token's chunks 3s .. 3s + 2 (6, 7) replace the previous token's, read last by its stage s
              if (!(ok = warp_wait(bar(B_QRET + s), static_cast<uint32_t>((nret - 1) & 1), abort_flag))) break;
              if (!(ok = copy_q(s == 1 ? 3 : 2))) break;
            }
            if (j == 0 && s == SPT_S - 1 &&
                !(ok = warp_wait(bar(B_ROPE_FULL), static_cast<uint32_t>(ti & 1), abort_flag)))
              break;
            if (!(ok = warp_wait(bar(B_RING_FULL + st), rp.phase, abort_flag))) break;
            DSA_TRACE_EVENT(12 + s, g);
            tc_fence_after();
            // the stage's three chunks: 12 MMAs issued as one block, then one commit
            const uint64_t bd = smem_desc(ring + st * S_STAGE, 16, 1024, kLayoutSW128);
            const uint64_t rd = smem_desc(sbase + OFF_ROPE, 16, 1024, kLayoutSW128);
            if (elect_one()) {
#pragma unroll
              for (int cc = 0; cc < SCH; ++cc) {
                const int qc = s * SCH + cc;
                const uint64_t b = bd + ((cc * CHUNK_BYTES) >> 4);
#pragma unroll
                for (int k = 0; k < 4; ++k) {  // K = 16 bf16 per instruction: 8 TMEM columns / 32 bytes of A, 32 bytes of B
                  const uint32_t acc = (s | cc | k) ? 1u : 0u;
                  if (qc < QTM) mma_bf16_ts(tmem + TS + NK * sb, tmem + TQ + 32 * qc + 8 * k, b + 2 * k, idesc, acc);
                  else mma_bf16_ss(tmem + TS + NK * sb, rd + 2 * k, b + 2 * k, idesc, acc);
                }
              }
              mma_commit(bar(B_RING_EMPTY + st));
              if (last && has_next) mma_commit(bar(B_QRET + s));
              if (last && s == SPT_S - 1) mma_commit(bar(B_ROPE_EMPTY));
            }
            __syncwarp();
            DSA_TRACE_EVENT(9 + s, g);
            if (last && has_next && s == (j == 0 ? SPT_S - 1 : 1)) {
              // the next token's chunks 0..2 overwrite this token's, read last by this tile's stage 0
              if (!(ok = warp_wait(bar(B_QRET), static_cast<uint32_t>(nret & 1), abort_flag))) break;
              if (!(ok = copy_q(3))) break;
            }
          }
          if (!ok) break;
          if (last && has_next) ++nret;
          DSA_TRACE_EVENT(3, g);
          if (elect_one()) mma_commit(bar(B_S_FULL + sb));
          __syncwarp();
        }
      }
    } else {
      constexpr uint32_t idesc = idesc_bf16(128, 256, true);
      for (int t = cluster; t < p.T && ok; t += nclusters, ++ti) {
        const int ntiles = mla_tiles(p, mla_dense_keys<DENSE>(p, t, p.row_off ? p.row_off[t] : 0));
        if constexpr (kChecks) { chk_tiles += ntiles; chk_ran = true; }
        for (int j = 0; j < ntiles && ok; ++j, ++g) {
          const int pb = static_cast<int>(g % NPB);
          if (j == 0 && !(ok = warp_wait(bar(B_O_FREE), (ti & 1) ^ 1, abort_flag))) break;
          if (!(ok = warp_wait(bar(B_P_READY + pb), static_cast<uint32_t>((g / NPB) & 1), abort_flag))) break;
          DSA_TRACE_EVENT(20, g);
          tc_fence_after();
          // P: two K-major chunks of 64 keys (128 heads x 128 bytes each, P_CHUNK apart)
          const uint64_t ad = smem_desc(sbase + OFF_PB + pb * XFER, 16, 1024, kLayoutSW128);
          for (int hh = 0; hh < SPT_V; ++hh, rp.advance()) {
            const int st = rp.stage;
            if (!(ok = warp_wait(bar(B_RING_FULL + st), rp.phase, abort_flag))) break;
            DSA_TRACE_EVENT(21 + hh, g);
            tc_fence_after();
            // MN-major V: 64-dim chunks 16 KB apart (LBO), 8-key row groups 1 KB apart (SBO)
            const uint64_t bd = smem_desc(ring + st * V_STAGE, CHUNK_BYTES, 1024, kLayoutSW128);
            if (elect_one()) {
#pragma unroll
              for (int k = 0; k < NK / 16; ++k)   // 16 keys per instruction: two 8-key groups = 2 KB of V
                mma_bf16_ss(tmem + 256 * hh, ad + (((k >> 2) * P_CHUNK) >> 4) + 2 * (k & 3), bd + ((k * 2048) >> 4),
                            idesc, (j == 0 && k == 0) ? 0u : 1u);
              mma_commit(bar(B_RING_EMPTY + st));
            }
            __syncwarp();
          }
          if (!ok) break;
          DSA_TRACE_EVENT(23, g);
          if (elect_one()) {
            mma_commit_mc(bar(B_P_EMPTY + pb), 0x1);   // P buffer pb free again (score CTA waits on it)
            mma_commit(bar(B_O_DONE + pb));
          }
          __syncwarp();
        }
      }
    }
  } else if constexpr (KL) {
    // ===================================================================== KL objective (warps 4..7)
    // Per tile, in two halves of 64 keys: each thread (one head) forms its head's probabilities of the half's keys
    // from the logits and the head's lse; a halving exchange sums them over the warp's 32 heads (lane l ends with
    // keys 2 l, 2 l + 1 of the half), and warp 4 adds the four warps' sums (handed over through double-buffered
    // shared memory under mbarriers) and accumulates the token's sums of a log a, a I, a and the log-sum-exp of I
    // over the valid keys.
    const int quad = warp & 3;
    const int h = quad * 32 + lane;
    const uint32_t lane_addr = static_cast<uint32_t>(quad * 32) << 16;
    float* red = reinterpret_cast<float*>(smem + OFF_RED);     // [2 buffers][4 warps][NK keys]
    constexpr float kLog2e = 1.4426950408889634f, kLn2 = 0.69314718055994531f;
    int g = 0;
    int ti = 0;
    bool ok = true;
    for (int t = cluster; t < p.T && ok; t += nclusters, ++ti) {
      const int is = ti & 1;
      if (!(ok = warp_wait(bar(B_IDX_FULL + is), (ti >> 1) & 1, abort_flag))) break;
      const int* ids = idx_s + is * KMAX;
      const long long base = p.row_off ? p.row_off[t] : 0;
      const int nd = mla_dense_keys<DENSE>(p, t, base);
      const int ntiles = mla_tiles(p, nd);
      if constexpr (kChecks) { chk_tiles += ntiles; chk_ran = true; }
      const bool head_on = h < p.H;
      const float lse2 = head_on ? p.kl_lse[static_cast<long long>(t) * p.H + h] * kLog2e : 0.f;
      const float inv_h = 1.f / static_cast<float>(p.H);
      float s_alog = 0.f, s_ai = 0.f, s_a = 0.f, m_i = -INFINITY, z_i = 0.f;   // warp 4, per lane
      for (int j = 0; j < ntiles && ok; ++j, ++g) {
        const int b = static_cast<int>(g & 1);     // S buffer and head-sum buffer of the tile
        const uint32_t use = static_cast<uint32_t>((g >> 1) & 1);
        uint32_t msk[4];   // key i of the tile enters the sums iff bit i / 4 of msk[i % 4] is set
        mla_tile_masks<DENSE, PAGED>(p, t, ids, base, nd, j, lane, msk);
        if (!(ok = warp_wait(bar(B_S_FULL + b), use, abort_flag))) break;
        tc_fence_after();
        if (!(ok = warp_wait(bar(B_RED_FREE + b), use ^ 1u, abort_flag))) break;
        float* rb = red + b * 4 * NK;
#pragma unroll
        for (int hq = 0; hq < 2; ++hq) {
          uint32_t v[64];
          {
            uint32_t (&v0)[32] = *reinterpret_cast<uint32_t(*)[32]>(&v[0]);
            uint32_t (&v1)[32] = *reinterpret_cast<uint32_t(*)[32]>(&v[32]);
            tmem_ld32(lane_addr + tmem + TS + NK * b + 64 * hq, v0);
            tmem_ld32(lane_addr + tmem + TS + NK * b + 64 * hq + 32, v1);
          }
          tmem_wait_ld();
          if (hq == 1) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(B_S_EMPTY + b));
          }
          float x[64];
#pragma unroll
          for (int i = 0; i < 64; ++i) {
            const int key = 64 * hq + i;
            const bool valid = (msk[key & 3] >> (key >> 2)) & 1u;
            x[i] = (valid && head_on) ? ex2_approx(fmaf(__uint_as_float(v[i]), p.scale_log2, -lse2)) : 0.f;
          }
          // sum over the warp's heads: five halving steps, each lane keeping the half its lane bit selects
#define DSA_KL_HALVE(O, N)                                                              \
  {                                                                                     \
    const bool up = (lane & (O)) != 0;                                                  \
    _Pragma("unroll") for (int i = 0; i < (N); ++i) {                                   \
      const float keep = up ? x[(N) + i] : x[i];                                        \
      const float send = up ? x[i] : x[(N) + i];                                        \
      x[i] = keep + __shfl_xor_sync(0xffffffffu, send, (O));                            \
    }                                                                                   \
  }
          DSA_KL_HALVE(16, 32)
          DSA_KL_HALVE(8, 16)
          DSA_KL_HALVE(4, 8)
          DSA_KL_HALVE(2, 4)
          DSA_KL_HALVE(1, 2)
#undef DSA_KL_HALVE
          rb[quad * NK + 64 * hq + 2 * lane] = x[0];
          rb[quad * NK + 64 * hq + 2 * lane + 1] = x[1];
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(B_RED_FULL + b));
        if (warp == 4) {
          if (!(ok = warp_wait(bar(B_RED_FULL + b), use, abort_flag))) break;
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            // key 64 hq + 2 lane + e of the tile (u = 2 hq + e): its bit is lane / 2 + 16 hq of msk[2 (lane % 2) + e]
            const int hq = u >> 1, e = u & 1;
            const int key = 64 * hq + 2 * lane + e;
            const uint32_t mw = (lane & 1) ? msk[2 + e] : msk[e];
            const bool valid = (mw >> (16 * hq + (lane >> 1))) & 1u;
            const float a = (rb[key] + rb[NK + key] + rb[2 * NK + key] + rb[3 * NK + key]) * inv_h;
            if (valid) {
              const float iv = p.kl_scores[static_cast<long long>(t) * p.k + j * NK + key];
              if (a > 0.f) s_alog += a * lg2_approx(a) * kLn2;
              s_ai += a * iv;
              s_a += a;
              if (iv > m_i) {
                z_i = (m_i == -INFINITY ? 0.f : z_i * ex2_approx((m_i - iv) * kLog2e)) + 1.f;
                m_i = iv;
              } else {
                z_i += ex2_approx((iv - m_i) * kLog2e);
              }
            }
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(bar(B_RED_FREE + b));
        }
      }
      if (ok && warp == 4) {
        // the token's divergence: p = a / sum(a) (L1-normalised), log Softmax(I) = I - lse(I)
        float mm = m_i;
#pragma unroll
        for (int d = 16; d > 0; d >>= 1) mm = fmaxf(mm, __shfl_xor_sync(0xffffffffu, mm, d));
        float z = (m_i == -INFINITY) ? 0.f : z_i * ex2_approx((m_i - mm) * kLog2e);
#pragma unroll
        for (int d = 16; d > 0; d >>= 1) {
          z += __shfl_xor_sync(0xffffffffu, z, d);
          s_alog += __shfl_xor_sync(0xffffffffu, s_alog, d);
          s_ai += __shfl_xor_sync(0xffffffffu, s_ai, d);
          s_a += __shfl_xor_sync(0xffffffffu, s_a, d);
        }
        if (lane == 0) {
          float kl = 0.f;
          if (s_a > 0.f && z > 0.f) {
            const float lse_i = mm + lg2_approx(z) * kLn2;
            kl = (s_alog - s_a * lg2_approx(s_a) * kLn2 - s_ai) / s_a + lse_i;
          }
          p.kl_out[t] = kl;
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(B_IDX_EMPTY + is));
    }
  } else if (rank == 0) {
    // ===================================================================== softmax (score CTA, warps 4..7)
    // Per tile: pass 1 reads the 128 logits of each head from tensor memory in two halves and takes the tile's
    // maximum; pass 2 forms the probabilities of the second half from the registers still holding it, reads the
    // first half again (after which the S buffer is released to the QK^T two tiles on), and stores P as bf16
    // straight into the value CTA's P buffer with st.async, each store completing its bytes on that CTA's P_FULL
    // barrier (no staging copy, and nothing queued behind the gathers in this SM's TMA unit).
    const int quad = warp & 3;
    const int h = quad * 32 + lane;
    const bool leader = (warp == 4 && lane == 0);
    const uint32_t lane_addr = static_cast<uint32_t>(quad * 32) << 16;
    const uint32_t pb_remote = map_cluster(sbase + OFF_PB, 1);
    const uint32_t pfull_remote = map_cluster(bar(B_P_FULL), 1);
    int g = 0;
    int ti = 0;
    bool ok = true;
    for (int t = cluster; t < p.T && ok; t += nclusters, ++ti) {
      const int is = ti & 1;
      if (!(ok = warp_wait(bar(B_IDX_FULL + is), (ti >> 1) & 1, abort_flag))) break;
      const int* ids = idx_s + is * KMAX;
      const long long base = p.row_off ? p.row_off[t] : 0;
      const int nd = mla_dense_keys<DENSE>(p, t, base);
      const int ntiles = mla_tiles(p, nd);
      if constexpr (kChecks) { chk_tiles += ntiles; chk_ran = true; }
      // l: sum of the bf16-rounded probabilities that enter P . V (normalises O exactly);
      // le: sum of the unrounded probabilities (for the log-sum-exp output)
      float m_ref = -INFINITY, l = 0.f, le = 0.f;
      for (int j = 0; j < ntiles && ok; ++j, ++g) {
        const int sb = static_cast<int>(g & 1), pb = static_cast<int>(g % NPB);
        const uint32_t s_tmem = lane_addr + tmem + TS + NK * sb;
        uint32_t msk[4];   // key i of the tile is valid iff bit i / 4 of msk[i % 4] is set
        mla_tile_masks<DENSE, PAGED>(p, t, ids, base, nd, j, lane, msk);
        const bool full_tile = (msk[0] & msk[1] & msk[2] & msk[3]) == 0xffffffffu;
        if (!(ok = warp_wait(bar(B_S_FULL + sb), static_cast<uint32_t>((g >> 1) & 1), abort_flag))) break;
        if (leader) DSA_TRACE_EVENT(4, g);
        tc_fence_after();
        uint32_t v[64];
        uint32_t (&v0)[32] = *reinterpret_cast<uint32_t(*)[32]>(&v[0]);
        uint32_t (&v1)[32] = *reinterpret_cast<uint32_t(*)[32]>(&v[32]);
        // masked keys become -inf (their probability is then 0)
        auto mask_half = [&](int hq) {
#pragma unroll
          for (int i = 0; i < 64; ++i) {
            const int key = 64 * hq + i;
            if (!((msk[key & 3] >> (key >> 2)) & 1u)) v[i] = __float_as_uint(-INFINITY);
          }
        };
        // pass 1: running max over the valid keys (raw logits; the scale is positive), as a 4-way tree
        float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int hq = 0; hq < 2; ++hq) {
          tmem_ld32(s_tmem + 64 * hq, v0);
          tmem_ld32(s_tmem + 64 * hq + 32, v1);
          tmem_wait_ld();
          if (!full_tile) mask_half(hq);
#pragma unroll
          for (int i = 0; i < 64; ++i) mx[i & 3] = fmaxf(mx[i & 3], __uint_as_float(v[i]));
        }
        if (leader) DSA_TRACE_EVENT(24, g);
        const float mraw = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
        const float mt = (mraw == -INFINITY) ? -INFINITY : mraw * p.scale_log2;
        float alpha = 1.f;
        if (mt > m_ref + RESCALE_LOG2) {
          alpha = (m_ref == -INFINITY) ? 0.f : ex2_approx(m_ref - mt);
          l *= alpha;
          le *= alpha;
          m_ref = mt;
        }
        // the value CTA's P buffer pb is free once its PV of tile g - NPB has completed
        if (!(ok = warp_wait<true>(bar(B_P_EMPTY + pb), static_cast<uint32_t>((g / NPB) & 1) ^ 1, abort_flag))) break;
        if (leader) {
          DSA_TRACE_EVENT(7, g);
          mbar_arrive_expect_tx_remote(pfull_remote + 8 * pb, XFER);
        }
        const uint32_t dst = pb_remote + pb * XFER, fb = pfull_remote + 8 * pb;
        // p = 2^(x * scale_log2 - m_ref) as one FMA + ex2, stored as one 64-key K chunk of P (128-byte swizzled
        // rows: 16-byte unit c of head h at unit c ^ (h % 8))
        const float neg_m = (m_ref == -INFINITY) ? 0.f : -m_ref;
        float ls0 = 0.f, ls1 = 0.f, lx0 = 0.f, lx1 = 0.f;
        auto emit_half = [&](int hq) {
          const uint32_t prow = dst + hq * P_CHUNK + h * 128;
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            uint32_t pk[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const float p0 = ex2_approx(fmaf(__uint_as_float(v[8 * c + 2 * i]), p.scale_log2, neg_m));
              const float p1 = ex2_approx(fmaf(__uint_as_float(v[8 * c + 2 * i + 1]), p.scale_log2, neg_m));
              const __nv_bfloat162 bb = __floats2bfloat162_rn(p0, p1);
              ls0 += __low2float(bb);
              ls1 += __high2float(bb);
              lx0 += p0;
              lx1 += p1;
              pk[i] = *reinterpret_cast<const uint32_t*>(&bb);
            }
            st_async_v4(prow + ((c ^ (h & 7)) << 4), make_uint4(pk[0], pk[1], pk[2], pk[3]), fb);
          }
        };
        emit_half(1);    // keys 64..127: still in v from pass 1
        tmem_ld32(s_tmem, v0);
        tmem_ld32(s_tmem + 32, v1);
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(B_S_EMPTY + sb));
        if (!full_tile) mask_half(0);
        emit_half(0);
        l += ls0 + ls1;
        le += lx0 + lx1;
        // per-head rescale factor and running row sum (the value CTA reads the sum of the token's last tile)
        st_async_b32(dst + P_BYTES + 4 * h, __float_as_uint(alpha), fb);
        st_async_b32(dst + P_BYTES + 512 + 4 * h, __float_as_uint(l), fb);
        if (leader) DSA_TRACE_EVENT(28, g);
        if (j == ntiles - 1 && p.lse && h < p.H)
          p.lse[static_cast<long long>(t) * p.H + h] =
              (le > 0.f) ? (m_ref + lg2_approx(le)) * 0.69314718055994531f : -INFINITY;
        ok = __shfl_sync(0xffffffffu, *abort_flag == 0, 0);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(B_IDX_EMPTY + is));
    }
  } else {
    // ===================================================================== correction + epilogue (value CTA)
    const int quad = warp & 3;
    const int h = quad * 32 + lane;
    const uint32_t lane_addr = static_cast<uint32_t>(quad * 32) << 16;
    int g = 0;
    int ti = 0;
    bool ok = true;
    for (int t = cluster; t < p.T && ok; t += nclusters, ++ti) {
      const int ntiles = mla_tiles(p, mla_dense_keys<DENSE>(p, t, p.row_off ? p.row_off[t] : 0));
      if constexpr (kChecks) { chk_tiles += ntiles; chk_ran = true; }
      float l = 0.f;
      for (int j = 0; j < ntiles; ++j, ++g) {
        const int pb = static_cast<int>(g % NPB);
        if (!(ok = warp_wait<true>(bar(B_P_FULL + pb), static_cast<uint32_t>((g / NPB) & 1), abort_flag))) break;
        if (warp == 4 && lane == 0) DSA_TRACE_EVENT(18, g);
        // P arrived by st.async; the PV MMA reads it through the async proxy
        fence_proxy_async_smem();
        const uint8_t* xb = smem + OFF_PB + pb * XFER;
        const float a = reinterpret_cast<const float*>(xb + P_BYTES)[h];
        if (j == ntiles - 1) l = reinterpret_cast<const float*>(xb + P_BYTES + 512)[h];
        if (j > 0 && __any_sync(0xffffffffu, a != 1.f)) {
          // wait until every PV up to tile g - 1 has landed in O, then scale the warp's rows of O
          if (!(ok = warp_wait(bar(B_O_DONE + (g - 1) % NPB), static_cast<uint32_t>(((g - 1) / NPB) & 1), abort_flag))) break;
          tc_fence_after();
          for (int cc = 0; cc < DV / 32; ++cc) {
            uint32_t v[32];
            tmem_ld32(lane_addr + tmem + 32 * cc, v);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] = __float_as_uint(__uint_as_float(v[i]) * a);
            tmem_st32(lane_addr + tmem + 32 * cc, v);
          }
          tmem_wait_st();
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(B_P_READY + pb));
        if (warp == 4 && lane == 0) DSA_TRACE_EVENT(19, g);
      }
      if (!ok) break;
      // epilogue: O / l -> bf16
      if (!(ok = warp_wait(bar(B_O_DONE + (g - 1) % NPB), static_cast<uint32_t>(((g - 1) / NPB) & 1), abort_flag))) break;
      tc_fence_after();
      const float inv = (l > 0.f) ? 1.f / l : 0.f;
      uint16_t* orow = p.out + (static_cast<long long>(t) * p.H + h) * DV;
      for (int cc = 0; cc < DV / 32; ++cc) {
        uint32_t v[32];
        tmem_ld32(lane_addr + tmem + 32 * cc, v);
        tmem_wait_ld();
        if (h < p.H) {
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const __nv_bfloat162 bb = __floats2bfloat162_rn(__uint_as_float(v[2 * i]) * inv,
                                                            __uint_as_float(v[2 * i + 1]) * inv);
            pk[i] = *reinterpret_cast<const uint32_t*>(&bb);
          }
          uint4* dst = reinterpret_cast<uint4*>(orow + 32 * cc);
#pragma unroll
          for (int i = 0; i < 4; ++i) dst[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(B_O_FREE));
    }
  }

  // ===================================================================== teardown
  if constexpr (kChecks) {
    // the threads of a warp that walked the key tiles agree on their count (first writer sets it)
    if (chk_ran && !*abort_flag) {
      const int old = atomicCAS(reinterpret_cast<int*>(smem + OFF_CHECK) + warp, -1, chk_tiles);
      check_that(old == -1 || old == chk_tiles);
    }
  }
  tc_fence_before();
  __syncthreads();
  if constexpr (kChecks) {
    // ... and so do the warps of the CTA
    if (threadIdx.x == 0 && !*abort_flag) {
      const int* chk = reinterpret_cast<const int*>(smem + OFF_CHECK);
      int ref = -1;
      for (int w = 0; w < THREADS / 32; ++w) {
        if (chk[w] < 0) continue;
        if (ref < 0) ref = chk[w];
        check_that(chk[w] == ref);
      }
    }
  }
  cluster_sync();       // no CTA leaves while its peer may still touch its shared memory
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

}  // namespace dsa
