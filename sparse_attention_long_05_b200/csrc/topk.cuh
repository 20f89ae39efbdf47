// Row-wise top-k selection (velog.io DSA page, §1.2 Fine-grained Token Selection) over materialised scores.
//
// One CTA per row.  Scores are mapped to monotone uint32 order keys (order_key), and the k-th largest key
// T is found exactly by a 4-pass most-significant-digit radix select (8-bit digits, per-warp shared-memory
// histograms, one warp scanning the 256 bins).  The selected set is then {key > T} plus the first
// `need` entries with key == T in ascending column order, which is exactly "score descending, smaller
// column first on ties".  A final ordered compaction writes the selected columns in ascending order: each
// warp owns a contiguous segment of the row, a counting pass gives every warp its output offset and its
// rank among the key == T entries, and a writing pass places the entries with warp ballots.
// Rows with n <= k select every column.  Nothing but the histograms lives in shared memory, so rows of any
// length (up to 2^31) are handled; the row is streamed from global memory (L2) six times.
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
};

constexpr int kTopkThreads = 512;
constexpr int kTopkWarps = kTopkThreads / 32;

__global__ void __launch_bounds__(kTopkThreads) topk_rows_kernel(const TopkParams p) {
  __shared__ uint32_t hist[kTopkWarps][256];
  __shared__ uint32_t s_need, s_digit;
  __shared__ int s_gt[kTopkWarps], s_eq[kTopkWarps];
  __shared__ int s_out_base[kTopkWarps], s_eq_base[kTopkWarps];

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

  if (n <= k) {
    for (int i = tid; i < k; i += kTopkThreads) out[i] = (i < n) ? i : -1;
    return;
  }

  // ---------------------------------------------------------------- radix select of the k-th largest key
  uint32_t prefix = 0, mask = 0, need = static_cast<uint32_t>(k);
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    for (int i = lane; i < 256; i += 32) hist[warp][i] = 0;
    __syncthreads();
    for (int i = tid; i < n; i += kTopkThreads) {
      const uint32_t key = order_key(x[i]);
      if ((key & mask) == prefix) atomicAdd(&hist[warp][(key >> shift) & 255], 1u);
    }
    __syncthreads();
    if (warp == 0) {
      // lane l owns bins 255-8l .. 248-8l (descending); totals over warps
      uint32_t cnt[8];
      uint32_t tot = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int bin = 255 - 8 * lane - j;
        uint32_t c = 0;
        for (int w = 0; w < kTopkWarps; ++w) c += hist[w][bin];
        cnt[j] = c;
        tot += c;
      }
      // inclusive scan of lane totals (descending bin order)
      uint32_t incl = tot;
#pragma unroll
      for (int d = 1; d < 32; d <<= 1) {
        const uint32_t v = __shfl_up_sync(0xffffffffu, incl, d);
        if (lane >= d) incl += v;
      }
      const uint32_t excl = incl - tot;
      // the lane whose range holds the need-th largest key
      const bool mine = excl < need && need <= incl;
      const uint32_t who = __ballot_sync(0xffffffffu, mine);
      if (mine) {
        uint32_t run = excl;
        int j = 0;
        for (; j < 8; ++j) {
          if (run + cnt[j] >= need) break;
          run += cnt[j];
        }
        s_digit = static_cast<uint32_t>(255 - 8 * lane - j);
        s_need = need - run;
      }
      (void)who;
    }
    __syncthreads();
    prefix |= s_digit << shift;
    mask |= 255u << shift;
    need = s_need;
    __syncthreads();
  }
  const uint32_t T = prefix;   // exact key of the k-th largest entry; `need` entries equal to T are taken

  // ---------------------------------------------------------------- ordered compaction
  const int seg = (n + kTopkWarps - 1) / kTopkWarps;
  const int seg0 = min(n, warp * seg), seg1 = min(n, seg0 + seg);
  int gt = 0, eq = 0;
  for (int i = seg0 + lane; i < seg1; i += 32) {
    const uint32_t key = order_key(x[i]);
    gt += key > T;
    eq += key == T;
  }
#pragma unroll
  for (int d = 16; d > 0; d >>= 1) {
    gt += __shfl_xor_sync(0xffffffffu, gt, d);
    eq += __shfl_xor_sync(0xffffffffu, eq, d);
  }
  if (lane == 0) { s_gt[warp] = gt; s_eq[warp] = eq; }
  __syncthreads();
  if (tid == 0) {
    int base = 0, eqb = 0;
    for (int w = 0; w < kTopkWarps; ++w) {
      s_out_base[w] = base;
      s_eq_base[w] = eqb;
      const int take_eq = max(0, min(s_eq[w], static_cast<int>(need) - eqb));
      base += s_gt[w] + take_eq;
      eqb += s_eq[w];
    }
  }
  __syncthreads();
  int pos = s_out_base[warp];
  int eq_rank = s_eq_base[warp];
  for (int i0 = seg0; i0 < seg1; i0 += 32) {
    const int i = i0 + lane;
    uint32_t key = 0;
    if (i < seg1) key = order_key(x[i]);
    const bool is_eq = i < seg1 && key == T;
    const uint32_t eq_mask = __ballot_sync(0xffffffffu, is_eq);
    const int my_eq_rank = eq_rank + __popc(eq_mask & ((1u << lane) - 1));
    const bool sel = i < seg1 && (key > T || (is_eq && my_eq_rank < static_cast<int>(need)));
    const uint32_t sel_mask = __ballot_sync(0xffffffffu, sel);
    if (sel) out[pos + __popc(sel_mask & ((1u << lane) - 1))] = i;
    pos += __popc(sel_mask);
    eq_rank += __popc(eq_mask);
  }
}

}  // namespace dsa
