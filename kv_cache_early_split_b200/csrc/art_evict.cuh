// art_evict.cuh -- random KV-cache eviction ahead of ART.
//
// intelligenzai.it, "La sorprendente sencillez de comprimir la memoria de la IA"
// (on arXiv 2609.03430, Random Attention): keep the tokens of the initial prompt
// and of the most recent window, drop the others uniformly at random inside each
// head (budgets of about 4x compression).  "Resumen Tecnico: ART" S2.4: ART runs
// on what such a cache policy keeps.
//
// Readings: per (batch, kv head), a sequence of length L <= budget keeps every
// position; otherwise it keeps [0, n_sink), [L - n_recent, L) and the
// m = budget - n_sink - n_recent middle positions j whose (key_j, j) pairs are the
// m smallest, key_j a caller-given uniform uint32.  Kept rows are packed in
// increasing position order.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace artk {
namespace evict {

constexpr int kSelThreads = 1024;

// Exclusive block-wide prefix sum of v (blockDim.x == kSelThreads); *total gets the sum.
__device__ __forceinline__ int block_exclusive_scan(int v, int* sm_warp, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, off);
    if (lane >= off) x += y;
  }
  if (lane == 31) sm_warp[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int s = sm_warp[lane];
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, s, off);
      if (lane >= off) s += y;
    }
    sm_warp[lane] = s;  // inclusive sums of the warps' totals
  }
  __syncthreads();
  const int before = (warp > 0) ? sm_warp[warp - 1] : 0;
  *total = sm_warp[31];
  __syncthreads();  // every thread has read sm_warp before the next use
  return before + x - v;
}

// kept[bh][0..budget): sorted kept positions (-1 past min(L, budget)); kept_lens[b] = min(L, budget).
// One block of kSelThreads per (batch, kv head).  A seq_len outside [1, L_max] keeps nothing.
__global__ void __launch_bounds__(kSelThreads) evict_select_kernel(const int32_t* __restrict__ seq_lens,
                                                                   const uint32_t* __restrict__ keys, int Hkv,
                                                                   int L_max, int n_sink, int n_recent, int budget,
                                                                   int32_t* __restrict__ kept,
                                                                   int32_t* __restrict__ kept_lens) {
  __shared__ unsigned hist[256];
  __shared__ int sm_warp[32];
  __shared__ unsigned s_prefix;
  __shared__ int s_rank;
  const int tid = threadIdx.x;
  const int bh = blockIdx.x, b = bh / Hkv;
  int L = seq_lens[b];
  if (L < 1 || L > L_max) L = 0;
  if (tid == 0 && bh % Hkv == 0) kept_lens[b] = min(L, budget);
  int32_t* out = kept + static_cast<long long>(bh) * budget;
  const uint32_t* kk = keys + static_cast<long long>(bh) * L_max;
  if (L <= budget) {
    for (int i = tid; i < budget; i += blockDim.x) out[i] = (i < L) ? i : -1;
    return;
  }
  const int lo = n_sink, hi = L - n_recent, m = budget - n_sink - n_recent;
  for (int i = tid; i < lo; i += blockDim.x) out[i] = i;
  for (int i = tid; i < n_recent; i += blockDim.x) out[budget - n_recent + i] = hi + i;
  if (m <= 0) return;

  // Radix select, most significant byte first: the m-th smallest key among kk[lo, hi).
  unsigned prefix = 0, mask = 0;
  int rank = m;  // 1-based rank still to locate among the keys that match `prefix` under `mask`
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int i = tid; i < 256; i += blockDim.x) hist[i] = 0;
    __syncthreads();
    for (int j = lo + tid; j < hi; j += blockDim.x) {
      const unsigned x = kk[j];
      if ((x & mask) == prefix) atomicAdd(&hist[(x >> shift) & 255u], 1u);
    }
    __syncthreads();
    if (tid == 0) {
      unsigned below = 0;
      int dg = 0;
      for (; dg < 255; ++dg) {
        if (below + hist[dg] >= static_cast<unsigned>(rank)) break;
        below += hist[dg];
      }
      s_prefix = prefix | (static_cast<unsigned>(dg) << shift);
      s_rank = rank - static_cast<int>(below);
    }
    __syncthreads();
    prefix = s_prefix;
    rank = s_rank;
    mask |= 255u << shift;
    __syncthreads();  // hist and s_* are rewritten by the next pass
  }
  // prefix is the threshold key; keep every smaller key and the first `rank` keys equal to it
  const unsigned thr = prefix;
  const int take_eq = rank;
  int base_keep = 0, base_eq = 0;
  for (int c0 = lo; c0 < hi; c0 += blockDim.x) {
    const int j = c0 + tid;
    const unsigned x = (j < hi) ? kk[j] : 0xffffffffu;
    const int less = (j < hi && x < thr) ? 1 : 0;
    const int eq = (j < hi && x == thr) ? 1 : 0;
    int tot_eq = 0, tot_keep = 0;
    const int pe = block_exclusive_scan(eq, sm_warp, &tot_eq);
    const int keep = (less || (eq && base_eq + pe < take_eq)) ? 1 : 0;
    const int pk = block_exclusive_scan(keep, sm_warp, &tot_keep);
    if (keep) out[lo + base_keep + pk] = j;
    base_keep += tot_keep;
    base_eq += tot_eq;
  }
}

// dst[bh][i] = src[bh][kept[bh][i]] row by row (rows of row_bytes, a multiple of 4); rows whose index is
// negative or not below L_max are zero.  grid: (B*Hkv, ceil(budget / warps per block)), one warp per row.
template <typename W>
__global__ void evict_compact_kernel(const uint8_t* __restrict__ src, const int32_t* __restrict__ kept, int L_max,
                                     int budget, int row_bytes, uint8_t* __restrict__ dst) {
  const int bh = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int i = blockIdx.y * (blockDim.x >> 5) + warp;
  if (i >= budget) return;
  const int j = kept[static_cast<long long>(bh) * budget + i];
  const bool ok = (j >= 0 && j < L_max);
  W* d = reinterpret_cast<W*>(dst + (static_cast<long long>(bh) * budget + i) * row_bytes);
  const W* s = reinterpret_cast<const W*>(src + (static_cast<long long>(bh) * L_max + (ok ? j : 0)) * row_bytes);
  const int nw = row_bytes / static_cast<int>(sizeof(W));
  for (int c = lane; c < nw; c += 32) {
    W v;
    if (ok) v = s[c];
    else memset(&v, 0, sizeof v);
    d[c] = v;
  }
}

}  // namespace evict
}  // namespace artk
