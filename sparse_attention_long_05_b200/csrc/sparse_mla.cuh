// Sparse MLA attention in MQA mode (velog.io DSA page, §1.2-§1.3): for each query token t and head h,
//   u[t,h] = softmax_{s in S_t}(scale * q[t,h] . c_s) . c_s[:512],   S_t = the selected latent entries.
//
// Why a 2-CTA cluster per token.  All 128 heads of a token share the same selected entries, so heads form
// the M = 128 dimension of the MMAs and every gathered entry is reused by all heads.  The output of one token
// (128 heads x 512 fp32) fills all 512 columns of one SM's tensor memory, leaving no room for the logits.
// The work is therefore split by role across the two CTAs of a cluster, each on its own SM:
//   score CTA (rank 0): keeps the token's queries in tensor memory, gathers the 576-dim selected rows,
//     computes S = Q . C^T on tcgen05 (A from tensor memory, bf16 -> fp32), runs the online softmax (fp32,
//     exp2 domain) and ships P (bf16) plus per-head rescale factors and row sums to the value CTA with one
//     shared-to-shared bulk copy per 64-key tile;
//   value CTA (rank 1): gathers the first 512 dims of the same rows, accumulates O += P . V on tcgen05 into
//     its tensor memory (two N = 256 halves), rescales O rows when a head's running maximum jumps (lazy:
//     only when the max grows by more than 2^8), and writes out = O / l in bf16.
// The QK^T and PV contractions (576 and 512 deep per key) are thus balanced across the two SMs, and no
// logit or probability ever leaves the chip.
//
// Data movement.
//   * Selected rows are gathered with 16-byte cp.async copies by four warps per CTA into 64-key x 64-dim
//     stages laid out in the 128-byte swizzled K-major form the tensor core reads; a stage is handed to the
//     MMA warp through an mbarrier after the copies have landed and been fenced into the async proxy.  The
//     same stage bytes serve as the K-major B operand of QK^T (rows = keys) and as the MN-major B operand
//     of PV (rows = keys = K, 64 dims = N per atom).
//   * The token's selected-index row is prefetched into shared memory with one bulk copy.
//   * Q chunks (128 heads x 64 dims) are staged by TMA and copied into tensor memory with tcgen05.cp; the
//     next token's chunks replace the current ones during the current token's last tile, right after the
//     MMAs that last read them (tcgen05.mma and tcgen05.cp of one thread execute in issue order).
//
// Warp roles (10 warps per CTA): w0 loader (index rows, Q chunks), w1 TMEM allocation + MMA issue,
// w2 w3 w8 w9 gathers, w4..w7 softmax (score CTA) or correction / epilogue (value CTA); warp w owns TMEM
// lanes (= heads) 32 * (w % 4) .. +31.
#pragma once
#include "common.cuh"

namespace dsa {

struct MlaParams {
  const int* idx;              // [T, k]
  const long long* row_off;    // [T] row of entry 0 of each token in c, or null (0)
  const uint16_t* c;           // [S, 576] bf16 (gathered with cp.async)
  uint16_t* out;               // [T, H, 512] bf16
  float* lse;                  // [T, H] or null
  int T, H, k;
  long long S;                 // rows of c
  float scale_log2;            // softmax scale * log2(e)
};

namespace mla {
constexpr int NK = 64;                    // keys per tile
constexpr int D = 576, DV = 512;
constexpr int QCHUNKS = D / 64;           // 9
constexpr int VCHUNKS = DV / 64;          // 8
constexpr int CHUNK_BYTES = NK * 128;     // 8 KB: 64 keys x 64 bf16
constexpr int QCHUNK_BYTES = 128 * 128;   // 16 KB: 128 heads x 64 bf16
constexpr int KMAX = 2048;                // largest selection handled (index row slot of 8 KB)
constexpr int QS = 3;                     // Q staging slots (score CTA)
constexpr int NSB = 3;                    // S buffers in tensor memory (score CTA)
constexpr int NPB = 3;                    // P buffers (value CTA)
constexpr int NS_S = 15, NS_V = 16;       // gather stages per CTA
constexpr int GD = 12;                    // gather chunks in flight per thread before signalling
constexpr int THREADS = 320;
constexpr int GATHER_THREADS = 128;
constexpr float RESCALE_LOG2 = 8.0f;      // lazy rescale threshold (factor 256)
constexpr int P_BYTES = 128 * 128;        // 128 heads x 64 keys bf16
constexpr int XFER = P_BYTES + 512 + 512; // P + alpha[128] + lsum[128]
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t TQ = 0;                // score CTA: Q in columns 0..287
constexpr uint32_t TS = 320;              // score CTA: S buffers at 320, 384, 448
// barrier slots
constexpr int B_IDX_FULL = 0, B_IDX_EMPTY = 2;
constexpr int B_QST_FULL = 4, B_QST_EMPTY = B_QST_FULL + QS;
constexpr int B_RING_FULL = B_QST_EMPTY + QS, B_RING_EMPTY = B_RING_FULL + 16;
constexpr int B_S_FULL = B_RING_EMPTY + 16, B_S_EMPTY = B_S_FULL + NSB, B_P_EMPTY = B_S_EMPTY + NSB;
constexpr int B_P_FULL = B_P_EMPTY + NPB, B_P_READY = B_P_FULL + NPB;
constexpr int B_O_DONE = B_P_READY + NPB, B_O_FREE = B_O_DONE + 1;
constexpr int B_SLOT_FREE = B_O_FREE + 1, B_SLOT_WRITTEN = B_SLOT_FREE + 1;   // score CTA softmax handshakes
constexpr int B_COUNT = B_SLOT_WRITTEN + 1;
// shared memory map (from a 1024-byte aligned base; both CTAs use the same barrier offsets)
constexpr int OFF_TMEM = 8 * B_COUNT;
constexpr int OFF_ABORT = OFF_TMEM + 4;
constexpr int OFF_IDX = 2048;                                   // both: 2 x 8 KB index rows
constexpr int OFF_PST = OFF_IDX + 2 * KMAX * 4;                 // score CTA: 2 P staging slots
constexpr int OFF_QST = OFF_PST + 2 * XFER;                     // score CTA: Q staging
constexpr int OFF_RING_S = OFF_QST + QS * QCHUNK_BYTES;         // score CTA: gather ring
constexpr int OFF_PB = OFF_IDX + 2 * KMAX * 4;                  // value CTA: P buffers
constexpr int OFF_RING_V = OFF_PB + NPB * XFER;                 // value CTA: gather ring
constexpr int SMEM_S = OFF_RING_S + NS_S * CHUNK_BYTES;
constexpr int SMEM_V = OFF_RING_V + NS_V * CHUNK_BYTES;
constexpr int SMEM = (SMEM_S > SMEM_V ? SMEM_S : SMEM_V) + 1024;
static_assert(OFF_TMEM + 8 <= OFF_IDX, "barrier area");
static_assert(OFF_PST % 1024 == 0 && OFF_QST % 1024 == 0 && OFF_RING_S % 1024 == 0, "1 KB aligned tiles");
static_assert(OFF_PB % 1024 == 0 && XFER % 1024 == 0 && OFF_RING_V % 1024 == 0, "1 KB aligned tiles");
static_assert(NS_V % 4 == 0, "value stages come in groups of four 64-dim chunks");
static_assert(GD < NS_S && GD < NS_V, "gather signalling depth below the ring size");
static_assert(SMEM <= 232448, "shared memory per CTA");
}  // namespace mla

// row of c gathered for selection entry e of a token whose entries start at row `base`
__device__ __forceinline__ long long mla_row(int e, long long base, long long S) {
  const long long r = base + e;
  const bool valid = (e >= 0) && (r < S);
  if (!valid && e != -1) raise_status(DSA_ERR_BAD_INDEX);
  return valid ? r : (base < S ? base : 0);
}
__device__ __forceinline__ bool mla_valid(int e, long long base, long long S) { return e >= 0 && base + e < S; }

// every lane waits (bounded); the warp then agrees on the outcome so that it stays converged
template <bool kCluster = false>
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag) {
  const bool ok = mbar_wait<kCluster>(bar, parity, abort_flag);
  return __all_sync(0xffffffffu, ok);
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(mla::THREADS, 1)
sparse_mla_kernel(const __grid_constant__ CUtensorMap tm_q, const MlaParams p) {
  using namespace mla;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  auto bar = [&](int slot) -> uint32_t { return sbase + 8 * slot; };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + OFF_ABORT);
  const int warp = warp_id(), lane = lane_id();
  const uint32_t rank = cluster_rank();            // 0 = score CTA, 1 = value CTA
  const int cluster = blockIdx.x >> 1, nclusters = gridDim.x >> 1;
  const int ntiles = p.k / NK;
  const int nsr = (rank == 0) ? NS_S : NS_V;
  const uint32_t ring = sbase + ((rank == 0) ? OFF_RING_S : OFF_RING_V);
  const int* idx_s = reinterpret_cast<const int*>(smem + OFF_IDX);

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(B_IDX_FULL + i), 1);
      mbar_init(bar(B_IDX_EMPTY + i), rank == 0 ? 8 : 4);
    }
    for (int i = 0; i < 16; ++i) { mbar_init(bar(B_RING_FULL + i), 4); mbar_init(bar(B_RING_EMPTY + i), 1); }
    if (rank == 0) {
      for (int i = 0; i < QS; ++i) { mbar_init(bar(B_QST_FULL + i), 1); mbar_init(bar(B_QST_EMPTY + i), 1); }
      for (int i = 0; i < NSB; ++i) { mbar_init(bar(B_S_FULL + i), 1); mbar_init(bar(B_S_EMPTY + i), 4); }
      for (int i = 0; i < NPB; ++i) mbar_init(bar(B_P_EMPTY + i), 1);
      mbar_init(bar(B_SLOT_FREE), 1);
      mbar_init(bar(B_SLOT_WRITTEN), 4);
    } else {
      for (int i = 0; i < NPB; ++i) { mbar_init(bar(B_P_FULL + i), 1); mbar_init(bar(B_P_READY + i), 4); }
      mbar_init(bar(B_O_DONE), 1);
      mbar_init(bar(B_O_FREE), 4);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0 && rank == 0) prefetch_tmap(&tm_q);
  if (warp == 1) {
    tmem_alloc(sbase + OFF_TMEM, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();        // both CTAs' barriers are initialised before any remote arrive
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + OFF_TMEM);

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
          for (int c = 0; c < QCHUNKS; ++c, ++qn) {
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
    }
  } else if (warp == 2 || warp == 3 || warp == 8 || warp == 9) {
    // ===================================================================== gathers (cp.async)
    const int gw = (warp == 2) ? 0 : (warp == 3) ? 1 : (warp == 8) ? 2 : 3;
    const int gi = gw * 32 + lane;
    const int u = gi & 7, rb = gi >> 3;                   // 16-byte unit within a 128-byte row; first row
    const uint32_t swz = static_cast<uint32_t>((u ^ (rb & 7)) << 4);
    const int nch = (rank == 0) ? QCHUNKS : VCHUNKS;
    const char* cbytes = reinterpret_cast<const char*>(p.c);
    long long n = 0;
    int ti = 0;
    bool ok = true;
    for (int t = cluster; t < p.T && ok; t += nclusters, ++ti) {
      const int is = ti & 1;
      if (!(ok = warp_wait(bar(B_IDX_FULL + is), (ti >> 1) & 1, abort_flag))) break;
      const int* ids = idx_s + is * KMAX;
      const long long base = p.row_off ? p.row_off[t] : 0;
      for (int j = 0; j < ntiles && ok; ++j) {
        const char* src[4];
#pragma unroll
        for (int m = 0; m < 4; ++m)
          src[m] = cbytes + mla_row(ids[j * NK + rb + 16 * m], base, p.S) * (D * 2) + u * 16;
        for (int c = 0; c < nch; ++c, ++n) {
          const int st = static_cast<int>(n % nsr);
          if (!(ok = warp_wait(bar(B_RING_EMPTY + st), static_cast<uint32_t>((n / nsr) & 1) ^ 1, abort_flag)))
            break;
          const uint32_t dst = ring + st * CHUNK_BYTES + swz;
#pragma unroll
          for (int m = 0; m < 4; ++m) cp_async16(dst + (rb + 16 * m) * 128, src[m] + c * 128);
          cp_async_commit();
          if (n >= GD) {
            cp_async_wait<GD>();
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(B_RING_FULL + static_cast<int>((n - GD) % nsr)));
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(B_IDX_EMPTY + is));
    }
    // the last GD chunks: wait for them, fence, hand them over
    cp_async_wait<0>();
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0 && !*abort_flag)
      for (long long i = (n > GD ? n - GD : 0); i < n; ++i) mbar_arrive(bar(B_RING_FULL + static_cast<int>(i % nsr)));
  } else if (warp == 1) {
    // ===================================================================== MMA issue
    if (lane == 0) {
      bool ok = true;
      long long g = 0, n = 0;
      int ti = 0;
      if (rank == 0) {
        constexpr uint32_t idesc = idesc_bf16(128, NK, false);
        int qn = 0;
        // Q chunk c of the next staged token -> tensor memory columns TQ + 32c .. +31
        auto load_q = [&](int c) -> bool {
          const int qs = qn % QS;
          if (!mbar_wait(bar(B_QST_FULL + qs), (qn / QS) & 1, abort_flag)) return false;
          tc_fence_after();
          const uint32_t src = sbase + OFF_QST + qs * QCHUNK_BYTES;
#pragma unroll
          for (int s = 0; s < 4; ++s)
            tmem_cp_128x256b(tmem + TQ + 32 * c + 8 * s, smem_desc(src + 32 * s, 16, 1024, kLayoutSW128));
          mma_commit(bar(B_QST_EMPTY + qs));
          ++qn;
          return true;
        };
        if (cluster < p.T)
          for (int c = 0; c < QCHUNKS && ok; ++c) ok = load_q(c);
        for (int t = cluster; t < p.T && ok; t += nclusters, ++ti) {
          const bool has_next = t + nclusters < p.T;
          for (int j = 0; j < ntiles && ok; ++j, ++g) {
            const int sb = static_cast<int>(g % NSB);
            if (!(ok = mbar_wait(bar(B_S_EMPTY + sb), static_cast<uint32_t>((g / NSB) & 1) ^ 1, abort_flag))) break;
            tc_fence_after();
            for (int c = 0; c < QCHUNKS; ++c, ++n) {
              const int st = static_cast<int>(n % nsr);
              if (!(ok = mbar_wait(bar(B_RING_FULL + st), static_cast<uint32_t>((n / nsr) & 1), abort_flag))) break;
              tc_fence_after();
              const uint64_t bd = smem_desc(ring + st * CHUNK_BYTES, 16, 1024, kLayoutSW128);
#pragma unroll
              for (int s = 0; s < 4; ++s)     // K = 16 bf16 per instruction: 8 TMEM columns of A, 32 bytes of B
                mma_bf16_ts(tmem + TS + NK * sb, tmem + TQ + 32 * c + 8 * s, bd + 2 * s, idesc, (c | s) ? 1u : 0u);
              mma_commit(bar(B_RING_EMPTY + st));
              if (j == ntiles - 1 && has_next && !(ok = load_q(c))) break;
            }
            if (!ok) break;
            mma_commit(bar(B_S_FULL + sb));
          }
        }
      } else {
        constexpr uint32_t idesc = idesc_bf16(128, 256, true);
        for (int t = cluster; t < p.T && ok; t += nclusters, ++ti) {
          for (int j = 0; j < ntiles && ok; ++j, ++g) {
            const int pb = static_cast<int>(g % NPB);
            if (j == 0 && !(ok = mbar_wait(bar(B_O_FREE), (ti & 1) ^ 1, abort_flag))) break;
            if (!(ok = mbar_wait(bar(B_P_READY + pb), static_cast<uint32_t>((g / NPB) & 1), abort_flag))) break;
            tc_fence_after();
            const uint64_t ad = smem_desc(sbase + OFF_PB + pb * XFER, 16, 1024, kLayoutSW128);
            for (int hh = 0; hh < 2 && ok; ++hh) {
              const int st0 = static_cast<int>(n % nsr);
              for (int q = 0; q < 4 && ok; ++q)
                ok = mbar_wait(bar(B_RING_FULL + st0 + q), static_cast<uint32_t>(((n + q) / nsr) & 1), abort_flag);
              if (!ok) break;
              tc_fence_after();
              // MN-major V: 64-dim chunks 8 KB apart (LBO), 8-key row groups 1 KB apart (SBO)
              const uint64_t bd = smem_desc(ring + st0 * CHUNK_BYTES, CHUNK_BYTES, 1024, kLayoutSW128);
#pragma unroll
              for (int s = 0; s < 4; ++s)     // 16 keys per instruction: two 8-key groups = 2 KB of V
                mma_bf16_ss(tmem + 256 * hh, ad + 2 * s, bd + ((s * 2048) >> 4), idesc, (j == 0 && s == 0) ? 0u : 1u);
              for (int q = 0; q < 4; ++q) mma_commit(bar(B_RING_EMPTY + st0 + q));
              n += 4;
            }
            if (!ok) break;
            mma_commit_mc(bar(B_P_EMPTY + pb), 0x1);   // P buffer pb free again (score CTA waits on it)
            mma_commit(bar(B_O_DONE));
          }
        }
      }
    }
  } else if (rank == 0) {
    // ===================================================================== softmax (score CTA, warps 4..7)
    const int quad = warp & 3;
    const int h = quad * 32 + lane;
    const bool leader = (warp == 4 && lane == 0);
    const uint32_t lane_addr = static_cast<uint32_t>(quad * 32) << 16;
    const uint32_t pb_remote = map_cluster(sbase + OFF_PB, 1);
    const uint32_t pfull_remote = map_cluster(bar(B_P_FULL), 1);
    long long g = 0;
    int ti = 0;
    bool ok = true;
    for (int t = cluster; t < p.T && ok; t += nclusters, ++ti) {
      const int is = ti & 1;
      if (!(ok = warp_wait(bar(B_IDX_FULL + is), (ti >> 1) & 1, abort_flag))) break;
      const int* ids = idx_s + is * KMAX;
      const long long base = p.row_off ? p.row_off[t] : 0;
      // l: sum of the bf16-rounded probabilities that enter P . V (normalises O exactly);
      // le: sum of the unrounded probabilities (for the log-sum-exp output)
      float m_ref = -INFINITY, l = 0.f, le = 0.f;
      for (int j = 0; j < ntiles && ok; ++j, ++g) {
        const int sb = static_cast<int>(g % NSB), pb = static_cast<int>(g % NPB), b = static_cast<int>(g & 1);
        const int2 e = reinterpret_cast<const int2*>(ids + j * NK)[lane];
        const uint32_t m_even = __ballot_sync(0xffffffffu, mla_valid(e.x, base, p.S));
        const uint32_t m_odd = __ballot_sync(0xffffffffu, mla_valid(e.y, base, p.S));
        if (!(ok = warp_wait(bar(B_S_FULL + sb), static_cast<uint32_t>((g / NSB) & 1), abort_flag))) break;
        tc_fence_after();
        uint32_t v[64];
        {
          uint32_t (&v0)[32] = *reinterpret_cast<uint32_t(*)[32]>(&v[0]);
          uint32_t (&v1)[32] = *reinterpret_cast<uint32_t(*)[32]>(&v[32]);
          tmem_ld32(lane_addr + tmem + TS + NK * sb, v0);
          tmem_ld32(lane_addr + tmem + TS + NK * sb + 32, v1);
        }
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(B_S_EMPTY + sb));
        float mt = -INFINITY;
#pragma unroll
        for (int i = 0; i < NK; ++i) {
          const bool valid = ((i & 1) ? (m_odd >> (i >> 1)) : (m_even >> (i >> 1))) & 1u;
          const float x = valid ? __uint_as_float(v[i]) * p.scale_log2 : -INFINITY;
          v[i] = __float_as_uint(x);
          mt = fmaxf(mt, x);
        }
        float alpha = 1.f;
        if (mt > m_ref + RESCALE_LOG2) {
          alpha = (m_ref == -INFINITY) ? 0.f : ex2_approx(m_ref - mt);
          l *= alpha;
          le *= alpha;
          m_ref = mt;
        }
        uint32_t pk[NK / 2];
        float ls = 0.f, lx = 0.f;
#pragma unroll
        for (int i = 0; i < NK / 2; ++i) {
          const float x0 = __uint_as_float(v[2 * i]), x1 = __uint_as_float(v[2 * i + 1]);
          const float p0 = (x0 == -INFINITY) ? 0.f : ex2_approx(x0 - m_ref);
          const float p1 = (x1 == -INFINITY) ? 0.f : ex2_approx(x1 - m_ref);
          const __nv_bfloat162 bb = __floats2bfloat162_rn(p0, p1);
          ls += __low2float(bb) + __high2float(bb);
          lx += p0 + p1;
          pk[i] = *reinterpret_cast<const uint32_t*>(&bb);
        }
        l += ls;
        le += lx;
        // staging slot b was last read by the bulk copy of tile g - 2: the leader waits for that copy to
        // have read its source, then releases the slot to the four softmax warps
        if (leader) {
          bulk_wait_read<1>();
          mbar_arrive(bar(B_SLOT_FREE));
        }
        if (!(ok = warp_wait(bar(B_SLOT_FREE), static_cast<uint32_t>(g & 1), abort_flag))) break;
        uint8_t* st = smem + OFF_PST + b * XFER;
        uint8_t* prow = st + h * 128;
#pragma unroll
        for (int c = 0; c < 8; ++c)
          *reinterpret_cast<uint4*>(prow + ((c ^ (h & 7)) << 4)) =
              make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
        reinterpret_cast<float*>(st + P_BYTES)[h] = alpha;
        if (j == ntiles - 1) {
          reinterpret_cast<float*>(st + P_BYTES + 512)[h] = l;
          if (p.lse && h < p.H)
            p.lse[static_cast<long long>(t) * p.H + h] =
                (le > 0.f) ? (m_ref + lg2_approx(le)) * 0.69314718055994531f : -INFINITY;
        }
        fence_proxy_async_smem();     // the staging slot is read next by the bulk-copy (async) proxy
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(B_SLOT_WRITTEN));
        if (leader) {
          // all four warps wrote the slot; the value CTA's P buffer pb is free once its PV of tile g - NPB
          // has completed
          ok = mbar_wait(bar(B_SLOT_WRITTEN), static_cast<uint32_t>(g & 1), abort_flag) &&
               mbar_wait<true>(bar(B_P_EMPTY + pb), static_cast<uint32_t>((g / NPB) & 1) ^ 1, abort_flag);
          if (ok) {
            mbar_arrive_expect_tx_remote(pfull_remote + 8 * pb, XFER);
            bulk_copy_to_peer(pb_remote + pb * XFER, sbase + OFF_PST + b * XFER, XFER, pfull_remote + 8 * pb);
            bulk_commit();
          }
        }
        ok = __shfl_sync(0xffffffffu, ok, 0) && !*abort_flag;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(B_IDX_EMPTY + is));
    }
    if (leader) bulk_wait_read<0>();
  } else {
    // ===================================================================== correction + epilogue (value CTA)
    const int quad = warp & 3;
    const int h = quad * 32 + lane;
    const uint32_t lane_addr = static_cast<uint32_t>(quad * 32) << 16;
    long long g = 0;
    int ti = 0;
    bool ok = true;
    for (int t = cluster; t < p.T && ok; t += nclusters, ++ti) {
      float l = 0.f;
      for (int j = 0; j < ntiles; ++j, ++g) {
        const int pb = static_cast<int>(g % NPB);
        if (!(ok = warp_wait<true>(bar(B_P_FULL + pb), static_cast<uint32_t>((g / NPB) & 1), abort_flag))) break;
        const uint8_t* xb = smem + OFF_PB + pb * XFER;
        const float a = reinterpret_cast<const float*>(xb + P_BYTES)[h];
        if (j == ntiles - 1) l = reinterpret_cast<const float*>(xb + P_BYTES + 512)[h];
        if (j > 0 && __any_sync(0xffffffffu, a != 1.f)) {
          // wait until every PV up to tile g - 1 has landed in O, then scale the warp's rows of O
          if (!(ok = warp_wait(bar(B_O_DONE), static_cast<uint32_t>((g - 1) & 1), abort_flag))) break;
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
      }
      if (!ok) break;
      // epilogue: O / l -> bf16
      if (!(ok = warp_wait(bar(B_O_DONE), static_cast<uint32_t>((g - 1) & 1), abort_flag))) break;
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
  tc_fence_before();
  __syncthreads();
  cluster_sync();       // no CTA leaves while its peer may still touch its shared memory
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

}  // namespace dsa
