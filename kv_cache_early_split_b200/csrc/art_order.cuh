// art_order.cuh -- KV tile traversal orders for ART.
//
// "Resumen Tecnico: ART" (gist.science, arXiv 2606.00024), S2.4: ART composes
// with other KV-cache policies by changing the traversal sequence of the KV
// blocks ("recency first", "importance first"); full attention does not depend
// on that sequence, and block 0 is evaluated first.  The page names the two
// orders without defining them; this file implements these readings:
//   * a sequence is per (batch, kv head); split s walks its positions
//     [floor(s*n/S), floor((s+1)*n/S)), which hold a permutation of split s's
//     own tiles, the split's first tile first;
//   * recency first: then the split's other tiles from newest to oldest;
//   * importance first: then the split's other tiles by the score
//     max over the group's query heads of q_h . mu_t, mu_t the mean key of
//     tile t (a per-tile key summary), highest first, ties to the lower index.
// Sequences are int32 [B, Hkv, n_max] (n_max = ceil(L_max / T)) with -1 at
// positions >= ceil(L_b / T).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace artk {
namespace ord {

__device__ __forceinline__ bool len_ok(int L, int L_max) { return L >= 1 && L <= L_max; }

// First position of split s in a sequence of n tiles.
__device__ __forceinline__ int seg_start(int s, int n, int S) {
  return static_cast<int>((static_cast<long long>(s) * n) / S);
}

// grid: B * Hkv blocks; threads stride over the n_max positions.
__global__ void tile_order_recency_kernel(const int32_t* __restrict__ seq_lens, int Hkv, int L_max, int T, int S,
                                          int n_max, int32_t* __restrict__ out) {
  const int bh = blockIdx.x;
  const int b = bh / Hkv;
  const int L = seq_lens[b];
  const int n = len_ok(L, L_max) ? (L + T - 1) / T : 0;
  int32_t* o = out + static_cast<long long>(bh) * n_max;
  for (int k = threadIdx.x; k < n_max; k += blockDim.x) {
    int v = -1;
    if (k < n) {
      int s = 0;
      while (s + 1 < S && seg_start(s + 1, n, S) <= k) ++s;
      const int ta = seg_start(s, n, S), tb = seg_start(s + 1, n, S);
      v = (k == ta) ? ta : tb - (k - ta);
    }
    o[k] = v;
  }
}

template <typename TK>
__device__ __forceinline__ float to_f32(TK x);
template <>
__device__ __forceinline__ float to_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }

// Mean key of each tile.  grid: (B * Hkv, ceil(n_max / tiles_per_block)); block: d threads (one per
// element of the key, so each row is read with coalesced loads).  Tiles past the sequence get 0.
template <typename TK>
__global__ void tile_key_summary_kernel(const TK* __restrict__ k, const int32_t* __restrict__ seq_lens, int Hkv,
                                        int L_max, int d, int T, int n_max, int tiles_per_block,
                                        float* __restrict__ out) {
  const int bh = blockIdx.x;
  const int b = bh / Hkv;
  const int L = seq_lens[b];
  const int n = len_ok(L, L_max) ? (L + T - 1) / T : 0;
  const int i = threadIdx.x;
  const TK* kb = k + static_cast<long long>(bh) * L_max * d;
  const int t_lo = blockIdx.y * tiles_per_block;
  for (int t = t_lo; t < min(n_max, t_lo + tiles_per_block); ++t) {
    float mean = 0.f;
    if (t < n) {
      const int j0 = t * T, j1 = min(j0 + T, L);
      float s = 0.f;
      for (int j = j0; j < j1; ++j) s += to_f32(kb[static_cast<long long>(j) * d + i]);
      mean = s / static_cast<float>(j1 - j0);
    }
    out[(static_cast<long long>(bh) * n_max + t) * d + i] = mean;
  }
}

// Importance-first sequence of one (batch, kv head) per block of kImpThreads threads.  Dynamic
// shared memory: G*d floats of queries, then n_max scores.  Scores: one warp per tile, lanes over
// the key elements (coalesced summary rows), warp-shuffle sums.  Sequence: each tile's place in its
// split is the number of the split's other tiles ranked before it.
constexpr int kImpThreads = 1024;

template <typename TQ>
__global__ void __launch_bounds__(kImpThreads) tile_order_importance_kernel(
    const TQ* __restrict__ q, const float* __restrict__ summary, const int32_t* __restrict__ seq_lens, int Hq,
    int Hkv, int L_max, int d, int T, int S, int n_max, int32_t* __restrict__ out) {
  extern __shared__ float sh[];
  const int bh = blockIdx.x;
  const int b = bh / Hkv, kvh = bh % Hkv;
  const int G = Hq / Hkv;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr int NWP = kImpThreads / 32;
  float* qs = sh;
  float* sc = sh + G * d;
  const int L = seq_lens[b];
  const int n = len_ok(L, L_max) ? (L + T - 1) / T : 0;
  for (int x = threadIdx.x; x < G * d; x += blockDim.x)
    qs[x] = to_f32(q[(static_cast<long long>(b) * Hq + kvh * G) * d + x]);
  __syncthreads();
  const float* mu = summary + static_cast<long long>(bh) * n_max * d;
  for (int t = warp; t < n; t += NWP) {
    const float* row = mu + static_cast<long long>(t) * d;
    float best = -INFINITY;
    for (int g = 0; g < G; ++g) {
      float dot = 0.f;
      for (int x = lane; x < d; x += 32) dot = fmaf(qs[g * d + x], row[x], dot);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, off);
      best = fmaxf(best, dot);  // fmaxf drops a NaN operand
    }
    if (lane == 0) sc[t] = best;
  }
  __syncthreads();
  int32_t* o = out + static_cast<long long>(bh) * n_max;
  for (int t = threadIdx.x; t < n_max; t += blockDim.x) {
    if (t >= n) {
      o[t] = -1;
      continue;
    }
    int s = 0;
    while (s + 1 < S && seg_start(s + 1, n, S) <= t) ++s;
    const int ta = seg_start(s, n, S), tb = seg_start(s + 1, n, S);
    if (t == ta) {
      o[ta] = ta;
      continue;
    }
    // rank of t among the split's other tiles: higher score first, ties to the lower index
    const float st = sc[t];
    int rank = 0;
    for (int u = ta + 1; u < tb; ++u) {
      const float su = sc[u];
      rank += (su > st || (su == st && u < t)) ? 1 : 0;
    }
    o[ta + 1 + rank] = t;
  }
}

}  // namespace ord
}  // namespace artk
