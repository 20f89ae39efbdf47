// Sparse MLA attention in MQA mode (velog.io DSA page, §1.2-§1.3): for each query token t and head h,
//   u[t,h] = softmax_{s in S_t}(scale * q[t,h] . c_s) . c_s[:512],   S_t = the selected latent entries.
//
// Why a 2-CTA cluster per token.  All 128 heads of a token share the same selected entries, so heads form
// the M = 128 dimension of the MMAs and every gathered entry is reused by all heads.  The output of one token
// (128 heads x 512 fp32) fills all 512 columns of one SM's tensor memory, leaving no room for the logits.
// The work is therefore split by role across the two CTAs of a cluster, each on its own SM:
//   score CTA (rank 0): gathers the 576-dim selected rows, S = Q . C^T on tcgen05 (bf16 -> fp32 in TMEM),
//     runs the online softmax (fp32, exp2 domain) and writes P (bf16) straight into the value CTA's shared
//     memory (distributed shared memory), plus per-head rescale factors and the final row sums;
//   value CTA (rank 1): gathers the first 512 dims of the same rows and accumulates O += P . V on tcgen05
//     into its tensor memory (two N = 256 halves), rescales O rows when a head's running maximum jumps
//     (lazy: only when the max grows by more than 2^8), and writes out = O / l in bf16.
// The QK^T and PV contractions (576 and 512 deep per key) are thus balanced across the two SMs, and no
// logit or probability ever leaves the chip.
//
// Gathers use TMA tile::gather4 (four rows of one 64-column, 128-byte swizzled box per instruction) into
// 64-key x 64-dim stages; the same stage bytes serve as the K-major B operand of QK^T (rows = keys) and as
// the MN-major B operand of PV (rows = keys = K, 64 dims = N per atom).
//
// Warp roles in each CTA: warp 0 = TMA producer, warp 1 = TMEM allocation + MMA issue, warps 2..5 = softmax
// (score CTA) or correction / epilogue (value CTA); warp w owns TMEM lanes (= heads) 32*(w % 4) .. +31.
#pragma once
#include "common.cuh"

namespace dsa {

struct MlaParams {
  const int* idx;              // [T, k]
  const long long* row_off;    // [T] row of entry 0 of each token in c, or null (0)
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
constexpr int NS = 9;                     // score-CTA gather stages
constexpr int NV = 20;                    // value-CTA gather stages (multiple of 4)
constexpr int THREADS = 192;
constexpr float RESCALE_LOG2 = 8.0f;      // lazy rescale threshold (factor 256)
// barrier slots
constexpr int B_Q_FULL = 0, B_Q_EMPTY = 1;
constexpr int B_KR_FULL = 2, B_KR_EMPTY = B_KR_FULL + NS;
constexpr int B_S_FULL = B_KR_EMPTY + NS, B_S_EMPTY = B_S_FULL + 2, B_P_EMPTY = B_S_EMPTY + 2;
constexpr int B_VR_FULL = B_P_EMPTY + 2, B_VR_EMPTY = B_VR_FULL + NV;
constexpr int B_P_FULL = B_VR_EMPTY + NV, B_P_READY = B_P_FULL + 2, B_O_DONE = B_P_READY + 2;
constexpr int B_O_FREE = B_O_DONE + 1;
constexpr int B_COUNT = B_O_FREE + 1;
// shared memory map (from a 1024-byte aligned base; both CTAs use the same barrier offsets)
constexpr int OFF_TMEM = 8 * B_COUNT;
constexpr int OFF_ABORT = OFF_TMEM + 4;
constexpr int OFF_ALPHA = 1024;           // value CTA: [2][128] fp32
constexpr int OFF_LSUM = OFF_ALPHA + 1024;  // value CTA: [128] fp32
constexpr int OFF_BIG = 4096;
constexpr int OFF_Q = OFF_BIG;                                 // score CTA
constexpr int OFF_KR = OFF_Q + QCHUNKS * QCHUNK_BYTES;         // score CTA
constexpr int OFF_P = OFF_BIG;                                 // value CTA: [2][128 x 64] bf16
constexpr int OFF_VR = OFF_P + 2 * 128 * 128;                  // value CTA
constexpr int SMEM_S = OFF_KR + NS * CHUNK_BYTES;
constexpr int SMEM_V = OFF_VR + NV * CHUNK_BYTES;
constexpr int SMEM = (SMEM_S > SMEM_V ? SMEM_S : SMEM_V) + 1024;
static_assert(OFF_TMEM + 8 <= OFF_ALPHA, "barrier area");
static_assert(NV % 4 == 0, "value stages come in groups of four 64-dim chunks");
}  // namespace mla

// row of c gathered for selection entry e of a token whose entries start at row `base`; marks validity
__device__ __forceinline__ int mla_row(int e, long long base, long long S, bool& valid) {
  const long long r = base + e;
  valid = (e >= 0) && (r < S);
  if (!valid && e != -1) raise_status(DSA_ERR_BAD_INDEX);
  return valid ? static_cast<int>(r) : static_cast<int>(base < S ? base : 0);
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(mla::THREADS, 1)
sparse_mla_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_c,
                  const MlaParams p) {
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

  if (threadIdx.x == 0) {
    if (rank == 0) {
      mbar_init(bar(B_Q_FULL), 1);
      mbar_init(bar(B_Q_EMPTY), 1);
      for (int i = 0; i < NS; ++i) { mbar_init(bar(B_KR_FULL + i), 1); mbar_init(bar(B_KR_EMPTY + i), 1); }
      for (int i = 0; i < 2; ++i) {
        mbar_init(bar(B_S_FULL + i), 1);
        mbar_init(bar(B_S_EMPTY + i), 128);
        mbar_init(bar(B_P_EMPTY + i), 1);
      }
    } else {
      for (int i = 0; i < NV; ++i) { mbar_init(bar(B_VR_FULL + i), 1); mbar_init(bar(B_VR_EMPTY + i), 1); }
      for (int i = 0; i < 2; ++i) { mbar_init(bar(B_P_FULL + i), 128); mbar_init(bar(B_P_READY + i), 128); }
      mbar_init(bar(B_O_DONE), 1);
      mbar_init(bar(B_O_FREE), 128);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) { prefetch_tmap(&tm_c); if (rank == 0) prefetch_tmap(&tm_q); }
  const uint32_t tmem_cols = (rank == 0) ? 128u : 512u;
  if (warp == 1) {
    tmem_alloc(sbase + OFF_TMEM, tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();        // both CTAs' barriers are initialised before any remote arrive
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + OFF_TMEM);

  if (warp == 0) {
    // ===================================================================== producers (both CTAs)
    const int nch = (rank == 0) ? QCHUNKS : VCHUNKS;
    const uint32_t ring = sbase + ((rank == 0) ? OFF_KR : OFF_VR);
    const int full0 = (rank == 0) ? B_KR_FULL : B_VR_FULL, empty0 = (rank == 0) ? B_KR_EMPTY : B_VR_EMPTY;
    const int nst = (rank == 0) ? NS : NV;
    int stage = 0;
    uint32_t phase = 0;
    long long issued = 0;
    int q_issued = 0;
    uint32_t q_par = 0;
    bool ok = true;
    int ti = 0;
    for (int t = cluster; t < p.T && ok; t += nclusters, ++ti) {
      if (rank == 0) {
        if (lane == 0) {
          ok = mbar_wait(bar(B_Q_EMPTY), (ti & 1) ^ 1, abort_flag);
          if (ok) {
            mbar_arrive_expect_tx(bar(B_Q_FULL), QCHUNKS * QCHUNK_BYTES);
            for (int c = 0; c < QCHUNKS; ++c)
              tma_load_3d(sbase + OFF_Q + c * QCHUNK_BYTES, &tm_q, bar(B_Q_FULL), 64 * c, 0, t);
            ++q_issued;
            q_par = ti & 1;
          }
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
      }
      const long long base = p.row_off ? p.row_off[t] : 0;
      const int* irow = p.idx + static_cast<long long>(t) * p.k;
      for (int j = 0; j < ntiles && ok; ++j) {
        const int2 e = *reinterpret_cast<const int2*>(irow + j * NK + 2 * lane);
        bool v0, v1;
        const int r0 = mla_row(e.x, base, p.S, v0), r1 = mla_row(e.y, base, p.S, v1);
        const int src = 2 * (lane & 15);
        const int a0 = __shfl_sync(0xffffffffu, r0, src), a1 = __shfl_sync(0xffffffffu, r1, src);
        const int a2 = __shfl_sync(0xffffffffu, r0, src + 1), a3 = __shfl_sync(0xffffffffu, r1, src + 1);
        for (int c = 0; c < nch; ++c) {
          if (lane == 0) {
            ok = mbar_wait(bar(empty0 + stage), phase ^ 1, abort_flag);
            if (ok) mbar_arrive_expect_tx(bar(full0 + stage), CHUNK_BYTES);
          }
          ok = __shfl_sync(0xffffffffu, ok, 0);
          if (!ok) break;
          if (lane < 16)
            tma_gather4(ring + stage * CHUNK_BYTES + lane * 512, &tm_c, bar(full0 + stage), 64 * c, a0, a1, a2, a3);
          ++issued;
          if (++stage == nst) { stage = 0; phase ^= 1; }
        }
      }
    }
    if (lane == 0 && *abort_flag) {
      for (int st = 0; st < nst && st < issued; ++st)
        mbar_wait_drain(bar(full0 + st), st < stage ? phase : phase ^ 1);
      if (rank == 0 && q_issued) mbar_wait_drain(bar(B_Q_FULL), q_par);
    }
  } else if (warp == 1) {
    // ===================================================================== MMA issue
    if (lane == 0) {
      bool ok = true;
      long long g = 0;
      int ti = 0;
      if (rank == 0) {
        constexpr uint32_t idesc = idesc_bf16(128, NK, false);
        Pipe<NS> kp;
        for (int t = cluster; t < p.T && ok; t += nclusters, ++ti) {
          if (!(ok = mbar_wait(bar(B_Q_FULL), ti & 1, abort_flag))) break;
          tc_fence_after();
          for (int j = 0; j < ntiles && ok; ++j, ++g) {
            const int sb = static_cast<int>(g & 1);
            if (!(ok = mbar_wait(bar(B_S_EMPTY + sb), ((g >> 1) & 1) ^ 1, abort_flag))) break;
            tc_fence_after();
            for (int c = 0; c < QCHUNKS; ++c) {
              if (!(ok = mbar_wait(bar(B_KR_FULL + kp.stage), kp.phase, abort_flag))) break;
              tc_fence_after();
              const uint64_t ad = smem_desc(sbase + OFF_Q + c * QCHUNK_BYTES, 16, 1024, kLayoutSW128);
              const uint64_t bd = smem_desc(sbase + OFF_KR + kp.stage * CHUNK_BYTES, 16, 1024, kLayoutSW128);
#pragma unroll
              for (int ks = 0; ks < 4; ++ks)     // K = 16 bf16 (32 bytes) per instruction
                mma_bf16_ss(tmem + sb * NK, ad + 2 * ks, bd + 2 * ks, idesc, (c | ks) ? 1u : 0u);
              mma_commit(bar(B_KR_EMPTY + kp.stage));
              kp.advance();
            }
            if (!ok) break;
            mma_commit(bar(B_S_FULL + sb));
          }
          mma_commit(bar(B_Q_EMPTY));
        }
      } else {
        constexpr uint32_t idesc = idesc_bf16(128, 256, true);
        Pipe<NV> vp;
        for (int t = cluster; t < p.T && ok; t += nclusters, ++ti) {
          for (int j = 0; j < ntiles && ok; ++j, ++g) {
            const int sb = static_cast<int>(g & 1);
            if (j == 0 && !(ok = mbar_wait(bar(B_O_FREE), (ti & 1) ^ 1, abort_flag))) break;
            if (!(ok = mbar_wait(bar(B_P_READY + sb), (g >> 1) & 1, abort_flag))) break;
            tc_fence_after();
            fence_proxy_async_smem();
            const uint64_t ad = smem_desc(sbase + OFF_P + sb * (128 * 128), 16, 1024, kLayoutSW128);
            for (int hh = 0; hh < 2 && ok; ++hh) {
              const int st0 = vp.stage;
              for (int q = 0; q < 4; ++q) {
                if (!(ok = mbar_wait(bar(B_VR_FULL + vp.stage), vp.phase, abort_flag))) break;
                vp.advance();
              }
              if (!ok) break;
              tc_fence_after();
              // MN-major V: 64-dim chunks 8 KB apart (LBO), 8-key row groups 1 KB apart (SBO)
              const uint64_t bd = smem_desc(sbase + OFF_VR + st0 * CHUNK_BYTES, CHUNK_BYTES, 1024, kLayoutSW128);
#pragma unroll
              for (int ks = 0; ks < 4; ++ks)     // 16 keys per instruction: two 8-key groups = 2 KB
                mma_bf16_ss(tmem + 256 * hh, ad + 2 * ks, bd + ((ks * 2048) >> 4), idesc,
                            (j == 0 && ks == 0) ? 0u : 1u);
              for (int q = 0; q < 4; ++q) mma_commit(bar(B_VR_EMPTY + st0 + q));
            }
            if (!ok) break;
            mma_commit_mc(bar(B_P_EMPTY + sb), 0x1);   // P buffer sb free again (score CTA)
            mma_commit(bar(B_O_DONE));
          }
        }
      }
    }
  } else if (rank == 0) {
    // ===================================================================== softmax (score CTA)
    const int quad = warp & 3;
    const int h = quad * 32 + lane;
    const uint32_t lane_addr = static_cast<uint32_t>(quad * 32) << 16;
    const uint32_t p_remote = map_cluster(sbase + OFF_P, 1);
    const uint32_t alpha_remote = map_cluster(sbase + OFF_ALPHA, 1);
    const uint32_t lsum_remote = map_cluster(sbase + OFF_LSUM, 1);
    const uint32_t pfull_remote = map_cluster(bar(B_P_FULL), 1);
    long long g = 0;
    bool ok = true;
    for (int t = p.T > 0 ? cluster : p.T; t < p.T && ok; t += nclusters) {
      const long long base = p.row_off ? p.row_off[t] : 0;
      const int* irow = p.idx + static_cast<long long>(t) * p.k;
      // l: sum of the bf16-rounded probabilities that enter P . V (normalises O exactly);
      // le: sum of the unrounded probabilities (for the log-sum-exp output)
      float m_ref = -INFINITY, l = 0.f, le = 0.f;
      for (int j = 0; j < ntiles; ++j, ++g) {
        const int sb = static_cast<int>(g & 1);
        const int2 e = *reinterpret_cast<const int2*>(irow + j * NK + 2 * lane);
        const uint32_t m_even = __ballot_sync(0xffffffffu, e.x >= 0 && base + e.x < p.S);
        const uint32_t m_odd = __ballot_sync(0xffffffffu, e.y >= 0 && base + e.y < p.S);
        if (!(ok = mbar_wait(bar(B_S_FULL + sb), (g >> 1) & 1, abort_flag))) break;
        tc_fence_after();
        uint32_t v[64];
        {
          uint32_t (&v0)[32] = *reinterpret_cast<uint32_t(*)[32]>(&v[0]);
          uint32_t (&v1)[32] = *reinterpret_cast<uint32_t(*)[32]>(&v[32]);
          tmem_ld32(lane_addr + tmem + sb * NK, v0);
          tmem_ld32(lane_addr + tmem + sb * NK + 32, v1);
        }
        tmem_wait_ld();
        tc_fence_before();
        mbar_arrive(bar(B_S_EMPTY + sb));
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
          const __nv_bfloat162 b = __floats2bfloat162_rn(p0, p1);
          ls += __low2float(b) + __high2float(b);
          lx += p0 + p1;
          pk[i] = *reinterpret_cast<const uint32_t*>(&b);
        }
        l += ls;
        le += lx;
        // P buffer sb of the value CTA is free once its PV of tile g - 2 has completed
        if (!(ok = mbar_wait<true>(bar(B_P_EMPTY + sb), ((g >> 1) & 1) ^ 1, abort_flag))) break;
        const uint32_t prow = p_remote + sb * (128 * 128) + h * 128;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const uint32_t dst = prow + ((c ^ (h & 7)) << 4);
          asm volatile("st.shared::cluster.v4.b32 [%0], {%1, %2, %3, %4};"
                       :: "r"(dst), "r"(pk[4 * c]), "r"(pk[4 * c + 1]), "r"(pk[4 * c + 2]), "r"(pk[4 * c + 3])
                       : "memory");
        }
        asm volatile("st.shared::cluster.f32 [%0], %1;" :: "r"(alpha_remote + 4 * (sb * 128 + h)), "f"(alpha) : "memory");
        if (j == ntiles - 1) {
          asm volatile("st.shared::cluster.f32 [%0], %1;" :: "r"(lsum_remote + 4 * h), "f"(l) : "memory");
          if (p.lse && h < p.H)
            p.lse[static_cast<long long>(t) * p.H + h] =
                (le > 0.f) ? (m_ref + lg2_approx(le)) * 0.69314718055994531f : -INFINITY;
        }
        fence_proxy_async();
        mbar_arrive_remote(pfull_remote + 8 * sb);
      }
    }
  } else {
    // ===================================================================== correction + epilogue (value CTA)
    const int quad = warp & 3;
    const int h = quad * 32 + lane;
    const uint32_t lane_addr = static_cast<uint32_t>(quad * 32) << 16;
    const float* alpha_s = reinterpret_cast<const float*>(smem + OFF_ALPHA);
    const float* lsum_s = reinterpret_cast<const float*>(smem + OFF_LSUM);
    long long g = 0;
    bool ok = true;
    for (int t = cluster; t < p.T && ok; t += nclusters) {
      for (int j = 0; j < ntiles; ++j, ++g) {
        const int sb = static_cast<int>(g & 1);
        if (!(ok = mbar_wait<true>(bar(B_P_FULL + sb), (g >> 1) & 1, abort_flag))) break;
        const float a = alpha_s[sb * 128 + h];
        if (j > 0 && a != 1.f) {
          // wait until every PV up to tile g - 1 has landed in O, then scale row h of O
          if (!(ok = mbar_wait(bar(B_O_DONE), static_cast<uint32_t>((g - 1) & 1), abort_flag))) break;
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
        mbar_arrive(bar(B_P_READY + sb));
      }
      if (!ok) break;
      // epilogue: O / l -> bf16
      if (!(ok = mbar_wait(bar(B_O_DONE), static_cast<uint32_t>((g - 1) & 1), abort_flag))) break;
      tc_fence_after();
      const float l = lsum_s[h];
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
            const __nv_bfloat162 b = __floats2bfloat162_rn(__uint_as_float(v[2 * i]) * inv,
                                                           __uint_as_float(v[2 * i + 1]) * inv);
            pk[i] = *reinterpret_cast<const uint32_t*>(&b);
          }
          uint4* dst = reinterpret_cast<uint4*>(orow + 32 * cc);
#pragma unroll
          for (int i = 0; i < 4; ++i) dst[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
        }
      }
      tc_fence_before();
      mbar_arrive(bar(B_O_FREE));
    }
  }

  // ===================================================================== teardown
  tc_fence_before();
  __syncthreads();
  cluster_sync();       // no CTA leaves while its peer may still touch its shared memory
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, tmem_cols);
  }
}

}  // namespace dsa
