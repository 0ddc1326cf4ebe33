// Two-pass decode attention over a q8 cache with the exact V skip (full attention, no ART).
//
// The skip rule (puntofijo.es, "La Elegancia de la Omision") leaves row j of tile t out of the
// numerator when exp(s_j - m'_t) < tau, m'_t the running maximum of the split's scores after tile
// t.  In one pass, m'_t needs the maxima of every earlier tile of the split, which a CTA that
// deals tiles with its neighbours only learns by waiting on them.  Split into passes instead:
//
//   pass 1 (q8_scores_kernel): s_j = q.k_j / sqrt(d) (log2 domain) for every row, the maximum of
//          every tile and of every chunk of CT tiles.  Reads K once, writes the scores.
//   pass 2 (q8_pv_kernel): m'_t = max(chunk maxima before the chunk, tile maxima of the chunk up
//          to t); weights p_j = 2^(s_j - m'_t) for the skip test, numerator and denominator taken
//          relative to the chunk's own reference max; V rows with every head below tau are not
//          dequantised, tiles with every row of every head below tau are not even read.
//   combine (q8_combine_kernel): the chunk states of every split merged per query head.
//
// Every step is a plain streaming kernel over the whole grid: no cluster barriers, no waits on
// other CTAs.  Each warp walks its rows in groups of RPI (one row per TPR lanes) and stages them
// through a ring of P groups in shared memory with cp.async, so that P groups per warp are in
// flight without holding registers.  Bytes: K and V (+ scales) once, plus 2 x 4 x GP bytes of
// scores per row.
#pragma once

#include <cuda.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "art_kernels.cuh"

namespace artk {
namespace q8two {

constexpr int NT = 256;  // threads per CTA
constexpr int NW = NT / 32;
constexpr int P = 8;       // ring slots per warp (row groups in flight)
constexpr int CTMAX = 32;  // tiles per chunk at most (one lane per tile in the in-chunk prefix)

struct Params {
  CUtensorMap tmK, tmV;  // tensor-core passes: K / V codes, boxes of 16 rows x 128 bytes, 128-byte swizzle
  const uint16_t* q;   // [B, Hq, D] bf16 bits
  const int8_t* k;     // [B, Hkv, L_max, D] codes
  const uint16_t* ks;  // [B, Hkv, L_max, D/32] fp16 bits
  const int8_t* v;
  const uint16_t* vs;
  const int32_t* seq_lens;  // [B]
  float* o;                 // [B, Hq, D]
  int32_t* tiles;           // [B, Hq] or NULL
  int32_t* ws_status;
  int32_t* ws_tiles_read;  // [B*Hkv*S]
  int32_t* ws_used;        // [B*Hq*S]
  float* scores;           // [B*Hkv][L_max][GP]  log2-domain scores (heads padded to GP)
  float* tmax;             // [B*Hkv][n_max][G]  tile maxima
  float* cmax;             // [B*Hkv*S][CPS][G]  chunk maxima
  float* part;             // [B*Hq*S][CPS][2 + D]  chunk states (m, l, acc)
  int32_t* vskip;          // [B*Hkv*S][2]  rows left out of every head's numerator, V tiles not read
  // ART on the two passes: per-tile probe records, the rule's stop tiles, the rule's settings
  float* probe;            // [B*Hq][n_max][REC]  m'_t, l_t, the tile's probe lanes of acc_t (own reference)
  int32_t* stop;           // [B*Hq*S]  absolute index of the last consumed tile of each split
  int B, Hq, Hkv, L_max, T, S, G, GP, CT, CPS, n_max;
  float qscale, tau;
  bool has_maps;  // tmK / tmV set
  bool art;       // the ART rule decides the tiles consumed (probe pass, rule, limited pass)
  int n_probe, patience;
  float eps_scale, eps_dir;
  int lanes[32];
};

constexpr int REC = 34;  // floats per probe record: m'_t, l_t, up to 32 probe lanes
static_assert(REC % 2 == 0, "records start on 8-byte boundaries");

// Smallest chunk: at least 128 rows per warp where that stays within CTMAX tiles.
__host__ __device__ inline int chunk_tiles_min(int T) {
  int ct = NW * (T >= 128 ? 1 : 128 / T);
  return ct > CTMAX ? CTMAX : ct;
}

__host__ __device__ constexpr int gp_of(int G) { return G <= 1 ? 1 : (G <= 2 ? 2 : (G <= 4 ? 4 : 8)); }

template <int D, int GP>
struct Geom {
  static constexpr int EPT = GP <= 4 ? 16 : 8;  // codes per thread of a row
  static constexpr int TPR = D / EPT;           // threads per row
  static constexpr int RPI = 32 / TPR;          // rows per group (one warp iteration)
  static constexpr int NB = D / 32;             // scale blocks per row
  static constexpr int HMASK = (TPR - 1) & ~(TPR / GP - 1);  // lane bits that name the head
  // one ring slot: codes [RPI][D] bytes, scales [RPI][NB] fp16, scores [RPI][GP] fp32 (pass 2)
  static constexpr int SLOT_CODES = RPI * D;
  static constexpr int SLOT_SCALES = RPI * NB * 2;
  static constexpr int SLOT_SCORES = RPI * GP * 4;
  static constexpr int SLOT = SLOT_CODES + SLOT_SCALES + SLOT_SCORES;
  static_assert(TPR >= GP && TPR <= 32 && 32 % TPR == 0, "a row must split evenly over a warp");
  static_assert(SLOT_CODES % 16 == 0 && SLOT_SCALES % 16 == 0 && SLOT_SCORES % 16 == 0, "16-byte slots");
};

// Head whose total transpose_reduce<GP, RL> leaves in this lane.
template <int GP, int RL>
__device__ __forceinline__ int head_of_lane(int lane) {
  int head = 0;
#pragma unroll
  for (int h = GP / 2, off = RL / 2; h >= 1; h >>= 1, off >>= 1)
    if (lane & off) head += h;
  return head;
}

// ---- cp.async (global -> shared, completion tracked per thread in commit groups)
template <int BYTES>
__device__ __forceinline__ void cp_async(uint32_t dst, const void* src) {
  if constexpr (BYTES == 16)
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
  else
    asm volatile("cp.async.ca.shared.global [%0], [%1], %2;" ::"r"(dst), "l"(src), "n"(BYTES) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Codes as float pairs (exponent-field insertion as in s8x8_to_f32; the subtraction is exact).
template <int EPT>
__device__ __forceinline__ void codes_to_f2(const uint32_t (&w)[EPT / 4], float2 (&f)[EPT / 2]) {
  const float2 bias = make_float2(-8388736.0f, -8388736.0f);
#pragma unroll
  for (int i = 0; i < EPT / 4; ++i) {
    const uint32_t u = w[i] ^ 0x80808080u;
    const float2 lo = make_float2(__uint_as_float(__byte_perm(u, 0x4B000000u, 0x7540u)),
                                  __uint_as_float(__byte_perm(u, 0x4B000000u, 0x7541u)));
    const float2 hi = make_float2(__uint_as_float(__byte_perm(u, 0x4B000000u, 0x7542u)),
                                  __uint_as_float(__byte_perm(u, 0x4B000000u, 0x7543u)));
    f[2 * i] = __fadd2_rn(lo, bias);
    f[2 * i + 1] = __fadd2_rn(hi, bias);
  }
}

// EPT codes of this lane from a ring slot
template <int EPT>
__device__ __forceinline__ void lds_codes(const uint8_t* p, uint32_t (&w)[EPT / 4]) {
  if constexpr (EPT == 16) {
    const uint4 x = *reinterpret_cast<const uint4*>(p);
    w[0] = x.x;
    w[1] = x.y;
    w[2] = x.z;
    w[3] = x.w;
  } else {
    const uint2 x = *reinterpret_cast<const uint2*>(p);
    w[0] = x.x;
    w[1] = x.y;
  }
}

struct Range {
  int L, t0, t1, c0, c1;
};

// Sequence, split and chunk of this CTA (blockIdx.x = chunk, blockIdx.y = (batch, kv head, split)).
// An invalid length reads as an empty sequence (the combine kernel reports it).
__device__ __forceinline__ Range cta_range(const Params& p) {
  Range r;
  const int unit = blockIdx.y;
  const int b = unit / p.S / p.Hkv;
  const int split = unit % p.S;
  r.L = p.seq_lens[b];
  if (r.L < 1 || r.L > p.L_max) r.L = 0;
  const int n_tiles = (r.L + p.T - 1) / p.T;
  r.t0 = static_cast<int>((static_cast<long long>(split) * n_tiles) / p.S);
  r.t1 = static_cast<int>((static_cast<long long>(split + 1) * n_tiles) / p.S);
  r.c0 = r.t0 + static_cast<int>(blockIdx.x) * p.CT;
  r.c1 = min(r.c0 + p.CT, r.t1);
  return r;
}

// The row groups of one warp, in order: tiles c0 + warp, c0 + warp + NW, ... of the chunk, ipt =
// T / RPI groups per tile.  The current group starts at row `row0` of tile `t` (group `ik` of the
// tile), whose rows end at `rend`.  Advanced incrementally: no divisions per group.
struct Walk {
  int t, row0, rend, ik;
  __device__ __forceinline__ void start(const Range& r, int warp, int T) {
    t = r.c0 + warp;
    row0 = t * T;
    rend = min(row0 + T, r.L);
    ik = 0;
  }
  __device__ __forceinline__ void next(const Range& r, int T, int ipt, int rpi) {
    row0 += rpi;
    if (++ik == ipt) {
      ik = 0;
      t += NW;
      row0 = t * T;
      rend = min(row0 + T, r.L);
    }
  }
};

// ------------------------------------------------------------------ pass 1: scores and maxima
template <int D, int GP>
__global__ void __launch_bounds__(NT, 2) q8_scores_kernel(const __grid_constant__ Params p) {
  using Gm = Geom<D, GP>;
  constexpr int EPT = Gm::EPT, TPR = Gm::TPR, RPI = Gm::RPI, NB = Gm::NB;
  constexpr int SLOT = Gm::SLOT_CODES + Gm::SLOT_SCALES;  // no scores in this pass's ring
  __shared__ __align__(16) uint8_t s_ring[NW][P][SLOT];
  __shared__ float s_cm[NW][GP];
  grid_dep_launch();  // pass 2's CTAs may take the SMs this grid leaves (they wait for its results)
  if (blockIdx.x == 0 && threadIdx.x < 2) p.vskip[blockIdx.y * 2 + threadIdx.x] = 0;  // counted by pass 2
  const Range r = cta_range(p);
  if (r.c0 >= r.t1) return;  // empty chunk
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int sub = lane % TPR, rsub = lane / TPR;
  const int unit = blockIdx.y;
  const int bk = unit / p.S;
  const int b = bk / p.Hkv, kvh = bk % p.Hkv;
  const int T = p.T, G = p.G;
  const int head = head_of_lane<GP, TPR>(lane);
  const bool writer = (sub % (TPR / GP)) == 0 && head < G;

  // query elements [sub*EPT, sub*EPT + EPT) of every head, scaled into the log2 domain
  float2 q2[GP][EPT / 2];
#pragma unroll
  for (int g = 0; g < GP; ++g) {
#pragma unroll
    for (int h = 0; h < EPT / 8; ++h) {
      float f[8];
      if (g < G) {
        const long long qrow = static_cast<long long>(b) * p.Hq + kvh * G + g;
        bf16x8_to_f32(*reinterpret_cast<const uint4*>(p.q + qrow * D + sub * EPT + 8 * h), f);
      } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) f[e] = 0.f;
      }
#pragma unroll
      for (int e = 0; e < 4; ++e) q2[g][4 * h + e] = make_float2(f[2 * e] * p.qscale, f[2 * e + 1] * p.qscale);
    }
  }

  const int8_t* kb = p.k + static_cast<long long>(bk) * p.L_max * D;
  const uint16_t* ksb = p.ks + static_cast<long long>(bk) * p.L_max * NB;
  float* scb = p.scores + static_cast<long long>(bk) * p.L_max * GP;
  const int ipt = T / RPI;
  const int nct = r.c1 - r.c0;
  const int niter = (warp < nct ? (nct - warp + NW - 1) / NW : 0) * ipt;
  const uint32_t ring = smem_u32(&s_ring[warp][0][0]);
  // rows past the end are not copied; their slot bytes are stale and their results unused
  Walk wi, wc;
  wi.start(r, warp, T);
  wc = wi;
  int ki = 0;
  auto issue = [&]() {
    if (ki < niter) {
      const int row = wi.row0 + rsub;
      if (row < wi.rend) {
        const uint32_t slot = ring + (ki & (P - 1)) * SLOT;
        cp_async<EPT>(slot + rsub * D + sub * EPT, kb + static_cast<long long>(row) * D + sub * EPT);
        if (sub == 0) cp_async<NB * 2>(slot + Gm::SLOT_CODES + rsub * NB * 2, ksb + static_cast<long long>(row) * NB);
      }
      wi.next(r, T, ipt, RPI);
    }
    ++ki;
    cp_async_commit();
  };

  float cm = -INFINITY, tm = -INFINITY;
  auto body = [&](int k) {
    const int row = wc.row0 + rsub;
    const uint8_t* slot = &s_ring[warp][k & (P - 1)][0];
    uint32_t cw[EPT / 4];
    lds_codes<EPT>(slot + rsub * D + sub * EPT, cw);
    const float sc = __half2float(
        __ushort_as_half(reinterpret_cast<const uint16_t*>(slot + Gm::SLOT_CODES)[rsub * NB + (sub * EPT) / 32]));
    float2 kf[EPT / 2];
    codes_to_f2<EPT>(cw, kf);
    float part[GP];
#pragma unroll
    for (int h = 0; h < GP; ++h) {
      float2 a = make_float2(0.f, 0.f);
#pragma unroll
      for (int i = 0; i < EPT / 2; ++i) a = __ffma2_rn(q2[h][i], kf[i], a);
      part[h] = (a.x + a.y) * sc;
    }
    int hd;
    const float tot = transpose_reduce<GP, TPR>(part, lane, hd);
    if (row < wc.rend) {
      tm = fmaxf(tm, tot);
      if (writer) scb[static_cast<long long>(row) * GP + head] = tot;
    }
    if (wc.ik == ipt - 1) {
      // last group of tile wc.t: its maximum per head over the lanes that hold that head
#pragma unroll
      for (int off = 1; off < 32; off <<= 1)
        if (!(off & Gm::HMASK)) tm = fmaxf(tm, __shfl_xor_sync(0xffffffffu, tm, off));
      if (lane < TPR && writer) p.tmax[(static_cast<long long>(bk) * p.n_max + wc.t) * G + head] = tm;
      cm = fmaxf(cm, tm);
      tm = -INFINITY;
    }
    wc.next(r, T, ipt, RPI);
  };

  // two groups per step (niter is a multiple of ipt, which is even): their chains interleave
#pragma unroll 1
  for (int k = 0; k < P - 2; ++k) issue();
#pragma unroll 1
  for (int k = 0; k < niter; k += 2) {
    issue();
    issue();
    cp_async_wait<P - 2>();  // groups k, k + 1 have landed (this lane's copies) ...
    __syncwarp();            // ... and every lane's
    body(k);
    body(k + 1);
    __syncwarp();  // every lane is done with these slots before they are refilled
  }
  cp_async_wait<0>();
  if (lane < TPR && (sub % (TPR / GP)) == 0) s_cm[warp][head] = cm;
  __syncthreads();
  if (static_cast<int>(threadIdx.x) < G) {
    float m = -INFINITY;
#pragma unroll
    for (int w = 0; w < NW; ++w) m = fmaxf(m, s_cm[w][threadIdx.x]);
    p.cmax[(static_cast<long long>(unit) * p.CPS + blockIdx.x) * G + threadIdx.x] = m;
  }
}

// ------------------------------------------------------------------ pass 1 on the tensor cores (d = 128, G <= 4)
// The same outputs as q8_scores_kernel, with the dot products on the tensor cores through warp-level
// m16n8k16 MMAs (f16 operands, fp32 accumulators): a warp takes 16 rows per group.  A = the rows'
// K codes, converted exactly to f16 in registers (codes are integers in [-127, 127]); B = the
// queries as 8 columns, the f16 part of each head's scaled query and the f16 of what that leaves
// over (≈ 22 bits), side by side (column 2h: head h's hi part, 2h + 1: its remainder), so lane
// (g, t) finds head t's two parts of rows g and g + 8 in its own accumulators.  Each 16-wide k-step
// lies inside one 32-wide scale block and accumulates into that block's accumulator, so each row's
// four K scales apply in fp32 after the MMAs, exactly as in the CUDA-core pass.  In block b, lane
// (g, t) supplies positions 32 b + 8 t .. + 3 to the first k-step and + 4 .. + 7 to the second, as
// MMA k-indices {2t, 2t+1, 2t+8, 2t+9} — 8 bytes of each row per block — and its B fragment uses
// the same order (a dot product does not depend on the order of its terms).
namespace mma16 {
constexpr int ROWS = 16;  // rows per group (the MMA's M)

__device__ __forceinline__ void mma_f16(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Four codes (one word) as two f16 pairs: (code 0, code 1) and (code 2, code 3).  u = c + 128 as a
// byte, 0x6400 | u is the f16 1024 + u, and subtracting 1152 leaves c exactly.
__device__ __forceinline__ void word_to_h2(uint32_t w, uint32_t& lo, uint32_t& hi) {
  const uint32_t u = w ^ 0x80808080u;
  const __half2 bias = __half2half2(__ushort_as_half(static_cast<unsigned short>(0x6480)));  // 1152
  uint32_t x = __byte_perm(u, 0x64646464u, 0x4140u), y = __byte_perm(u, 0x64646464u, 0x4342u);
  const __half2 a = __hsub2(*reinterpret_cast<const __half2*>(&x), bias);
  const __half2 b = __hsub2(*reinterpret_cast<const __half2*>(&y), bias);
  lo = *reinterpret_cast<const uint32_t*>(&a);
  hi = *reinterpret_cast<const uint32_t*>(&b);
}

__device__ __forceinline__ uint32_t pack_h2(float x, float y) {
  __half2 h = __floats2half2_rn(x, y);
  return *reinterpret_cast<uint32_t*>(&h);
}

// The codes of a step (two groups, 32 rows of one tile) arrive as one TMA box of 32 rows x 128 bytes
// with the 128-byte swizzle: the 16-byte chunk c of row R lands at chunk c ^ (R % 8), so a lane's
// reads of rows g and g + 8 (and the PV pass's of rows 2t .. 2t + 9) fall on distinct banks with no
// padding.  One copy instruction per 4 KiB: per-lane 16-byte copies, and then 2 KiB boxes, were
// what bounded the passes (measured with the arithmetic taken out).
constexpr int STEP = 32;
constexpr int BOX = STEP * 128;
constexpr int PB = 3;   // boxes per warp in flight, scores pass
constexpr int PBV = 2;  // PV pass (its scores and scales take the rest of the shared memory)
// Wait for slot sl's box (bounded; the warp agrees on the outcome).  On success the slot's pending bit
// clears and its parity flips; after a timeout (the status word has ART_ERR_TIMEOUT) the bit stays
// set, so that the caller stops issuing and drains the slots still pending before it leaves.
__device__ __forceinline__ bool wait_box(uint32_t bars, int sl, uint32_t& pend, uint32_t& phase, int32_t* status) {
  if (!((pend >> sl) & 1u)) return true;
  const bool ok = __all_sync(0xffffffffu, mbar_wait_bounded(bars + 8 * sl, (phase >> sl) & 1u, status));
  if (ok) {
    phase ^= 1u << sl;
    pend &= ~(1u << sl);
  }
  return ok;
}
// ... the drain: one more bounded wait on every slot still pending
__device__ __forceinline__ void drain_boxes(uint32_t bars, int slots, uint32_t pend, uint32_t phase, int32_t* status) {
  for (int sl = 0; sl < slots; ++sl)
    if ((pend >> sl) & 1u) mbar_wait_bounded(bars + 8 * sl, (phase >> sl) & 1u, status);
}

__device__ __forceinline__ uint32_t swz(int row, int byte) {
  return static_cast<uint32_t>(row * 128 + ((((byte >> 4) ^ row) & 7) << 4) + (byte & 15));
}
// dynamic shared memory of the scores pass: 1 KiB of alignment slack (the swizzle wants 1 KiB
// aligned boxes), then per warp PB boxes, PB x 32 rows of scales and PB barriers
constexpr int TSM_SCALES = NW * PB * BOX;
constexpr int TSM_BARS = TSM_SCALES + NW * PB * STEP * 8;
constexpr int TSMEM = 1024 + TSM_BARS + NW * PB * 8;
// the PV pass: per warp PBV boxes, PBV x 32 rows of V scales, PBV x 32 rows of scores (16 bytes each)
// and PBV barriers; after the rows, the same memory holds the warps' accumulators
constexpr int PSM_VS = NW * PBV * BOX;
constexpr int PSM_SC = PSM_VS + NW * PBV * STEP * 8;
constexpr int PSM_BARS = PSM_SC + NW * PBV * STEP * 16;
constexpr int PSMEM_RING = 1024 + PSM_BARS + NW * PBV * 8;
}  // namespace mma16

template <int GP>
__global__ void __launch_bounds__(NT, 2) q8_scores_mma_kernel(const __grid_constant__ Params p) {
  constexpr int D = 128, NB = 4;
  static_assert(GP <= 4, "4 heads (hi + lo) fill the MMA's 8 columns");
  extern __shared__ __align__(16) uint8_t s_dyn[];
  __shared__ float s_cm[NW][4];
  grid_dep_launch();  // pass 2's CTAs may take the SMs this grid leaves (they wait for its results)
  if (blockIdx.x == 0 && threadIdx.x < 2) p.vskip[blockIdx.y * 2 + threadIdx.x] = 0;  // counted by pass 2
  const Range r = cta_range(p);
  if (r.c0 >= r.t1) return;  // empty chunk
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 2, t = lane & 3;  // MMA fragment coordinates
  const int unit = blockIdx.y;
  const int bk = unit / p.S;
  const int b = bk / p.Hkv, kvh = bk % p.Hkv;
  const int T = p.T, G = p.G;

  // B fragments: column n = g is head g / 2's scaled query, its f16 part for even g, the remainder
  // for odd g; in step s (block s / 2) lane t holds positions 32 (s / 2) + 8 t + 4 (s % 2) + {0, 1}
  // (b0) and + {2, 3} (b1).
  uint32_t bq[8][2];
  {
    const int hq = g >> 1;
    const bool lo_part = (g & 1) != 0;
    const bool live = hq < G;
    const long long qrow = static_cast<long long>(b) * p.Hq + kvh * G + (live ? hq : 0);
#pragma unroll
    for (int s = 0; s < 8; ++s) {
      float f[4];
      const uint2 qw = *reinterpret_cast<const uint2*>(p.q + qrow * D + 32 * (s >> 1) + 8 * t + 4 * (s & 1));
      const uint32_t qv[2] = {qw.x, qw.y};
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        f[2 * e] = __uint_as_float(qv[e] << 16) * p.qscale;
        f[2 * e + 1] = __uint_as_float(qv[e] & 0xffff0000u) * p.qscale;
      }
      float v[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float h = __half2float(__float2half_rn(f[e]));
        v[e] = live ? (lo_part ? f[e] - h : h) : 0.f;
      }
      bq[s][0] = mma16::pack_h2(v[0], v[1]);
      bq[s][1] = mma16::pack_h2(v[2], v[3]);
    }
  }

  const uint16_t* ksb = p.ks + static_cast<long long>(bk) * p.L_max * NB;
  float* scb = p.scores + static_cast<long long>(bk) * p.L_max * GP;
  const int ipt = T / mma16::ROWS, ips = T / mma16::STEP;  // groups and steps per tile (T >= 32)
  const int nct = r.c1 - r.c0;
  const int nsteps = (warp < nct ? (nct - warp + NW - 1) / NW : 0) * ips;
  const uint32_t dyn = smem_u32(s_dyn), base = (dyn + 1023u) & ~1023u;
  uint8_t* const codes = s_dyn + (base - dyn) + warp * mma16::PB * mma16::BOX;
  uint8_t* const scales = s_dyn + (base - dyn) + mma16::TSM_SCALES + warp * mma16::PB * mma16::STEP * 8;
  const uint32_t bars = base + mma16::TSM_BARS + warp * mma16::PB * 8;
  if (lane == 0) {
    for (int i = 0; i < mma16::PB; ++i) mbar_init(bars + 8 * i, 1);
    fence_mbar_init();
  }
  __syncwarp();
  // copies of a step: one TMA box of 32 code rows (rows past the tensor's end read as zeros; rows
  // past the sequence are copied and their results dropped; a step wholly past it copies nothing)
  // and, lane l, row l's scales (8 B)
  Walk wi, wc;
  wi.start(r, warp, T);
  wc = wi;
  int ks = 0;
  uint32_t pend = 0u, phase = 0u;  // bit s: slot s has a box in flight / the parity it completes
  auto issue = [&]() {
    if (ks < nsteps) {
      const int sl = ks % mma16::PB;
      if (wi.row0 < wi.rend) {
        ART_DCHECK(wi.row0 >= 0 && wi.row0 < p.L_max, p.ws_status);
        if (lane == 0) {
          mbar_arrive_expect_tx(bars + 8 * sl, mma16::BOX);
          tma_load_3d(smem_u32(codes + sl * mma16::BOX), &p.tmK, bars + 8 * sl, 0, wi.row0, bk);
        }
        pend |= 1u << sl;
      }
      if (wi.row0 + lane < wi.rend)
        cp_async<8>(smem_u32(scales + sl * mma16::STEP * 8) + lane * 8, ksb + static_cast<long long>(wi.row0 + lane) * NB);
      wi.next(r, T, ips, mma16::STEP);
    }
    ++ks;
    cp_async_commit();
  };

  // head t (lanes with t < G), rows g and g + 8: the scores of a group ...
  float cm = -INFINITY, tm = -INFINITY;
  auto scores = [&](int sl, int half, float& v0, float& v1) {
    const uint8_t* box = codes + sl * mma16::BOX + half * mma16::ROWS * 128;  // rows 16 half .. (same swizzle phase)
    const uint8_t* ksl = scales + (sl * mma16::STEP + half * mma16::ROWS) * 8;
    float acc[NB][4];
#pragma unroll
    for (int j = 0; j < NB; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.f;
#pragma unroll
    for (int bb = 0; bb < NB; ++bb) {
      const uint2 w0 = *reinterpret_cast<const uint2*>(box + mma16::swz(g, 32 * bb + 8 * t));
      const uint2 w1 = *reinterpret_cast<const uint2*>(box + mma16::swz(g + 8, 32 * bb + 8 * t));
      uint32_t a[4];
      mma16::word_to_h2(w0.x, a[0], a[2]);
      mma16::word_to_h2(w1.x, a[1], a[3]);
      mma16::mma_f16(acc[bb], a, bq[2 * bb][0], bq[2 * bb][1]);
      mma16::word_to_h2(w0.y, a[0], a[2]);
      mma16::word_to_h2(w1.y, a[1], a[3]);
      mma16::mma_f16(acc[bb], a, bq[2 * bb + 1][0], bq[2 * bb + 1][1]);
    }
    // columns 2t (f16 part) and 2t + 1 (remainder) of head t, rows g (0, 1) and g + 8 (2, 3)
    const uint2 s0 = *reinterpret_cast<const uint2*>(ksl + g * 8);
    const uint2 s1 = *reinterpret_cast<const uint2*>(ksl + (g + 8) * 8);
    const float2 a0 = __half22float2(*reinterpret_cast<const __half2*>(&s0.x));
    const float2 a1 = __half22float2(*reinterpret_cast<const __half2*>(&s0.y));
    const float2 b0 = __half22float2(*reinterpret_cast<const __half2*>(&s1.x));
    const float2 b1 = __half22float2(*reinterpret_cast<const __half2*>(&s1.y));
    const float sc0[NB] = {a0.x, a0.y, a1.x, a1.y}, sc1[NB] = {b0.x, b0.y, b1.x, b1.y};
    v0 = 0.f;
    v1 = 0.f;
#pragma unroll
    for (int j = 0; j < NB; ++j) {
      v0 = fmaf(sc0[j], acc[j][0] + acc[j][1], v0);
      v1 = fmaf(sc1[j], acc[j][2] + acc[j][3], v1);
    }
  };
  // ... then stored, with the tile maxima, in walk order
  auto finish = [&](float v0, float v1) {
    if (t < G) {
      const int row0 = wc.row0 + g;
      if (row0 < wc.rend) {
        scb[static_cast<long long>(row0) * GP + t] = v0;
        tm = fmaxf(tm, v0);
      }
      if (row0 + 8 < wc.rend) {
        scb[static_cast<long long>(row0 + 8) * GP + t] = v1;
        tm = fmaxf(tm, v1);
      }
    }
    if (wc.ik == ipt - 1) {
      // last group of tile wc.t: the maximum of head t over the rows (lanes of the same t)
#pragma unroll
      for (int off = 4; off < 32; off <<= 1) tm = fmaxf(tm, __shfl_xor_sync(0xffffffffu, tm, off));
      ART_DCHECK(wc.t >= r.c0 && wc.t < r.c1 && wc.t < p.n_max, p.ws_status);
      if (g == 0 && t < G) p.tmax[(static_cast<long long>(bk) * p.n_max + wc.t) * G + t] = tm;
      cm = fmaxf(cm, tm);
      tm = -INFINITY;
    }
    wc.next(r, T, ipt, mma16::ROWS);
  };

  // the two groups of a step together, so that their loads, conversions and MMAs interleave
#pragma unroll 1
  for (int i = 0; i < mma16::PB; ++i) issue();
#pragma unroll 1
  for (int k = 0; k < nsteps; ++k) {
    const int sl = k % mma16::PB;
    cp_async_wait<mma16::PB - 1>();  // the scales of step k have landed (this lane's) ...
    if (!mma16::wait_box(bars, sl, pend, phase, p.ws_status)) break;  // ... its codes
    __syncwarp();  // ... and every lane's scales
    float x0, x1, y0, y1;
    scores(sl, 0, x0, x1);
    scores(sl, 1, y0, y1);
    finish(x0, x1);
    finish(y0, y1);
    __syncwarp();  // every lane is done with the slot before it is refilled
    issue();
  }
  mma16::drain_boxes(bars, mma16::PB, pend, phase, p.ws_status);  // (only after a timeout)
  cp_async_wait<0>();
  if (g == 0) s_cm[warp][t] = cm;
  __syncthreads();
  if (static_cast<int>(threadIdx.x) < G) {
    float m = -INFINITY;
#pragma unroll
    for (int w = 0; w < NW; ++w) m = fmaxf(m, s_cm[w][threadIdx.x]);
    p.cmax[(static_cast<long long>(unit) * p.CPS + blockIdx.x) * G + threadIdx.x] = m;
  }
}

// ------------------------------------------------------------------ pass 2 on the tensor cores (d = 128, G <= 4)
// The same outputs as q8_pv_kernel, with the weighted sum of V rows on the tensor cores: per group of
// 16 rows and per scale block, O^T += P'^T-shaped A (16 x 16: M = head g's weights times the V scale
// as f16 hi in row g and lo in row g + 8, K = the 16 rows) times B (16 rows x 8 positions of V, the
// codes converted exactly to f16).  In n-tile (block b, j) column n is position 32 b + 4 n + j, so a
// lane's V bytes for a row and block are one 4-byte word.  Weights, the skip test, the denominators
// and the counters are formed as in q8_pv_kernel: one lane per (row, head) pair, two pairs per lane.
namespace mma16 {
constexpr int PV_ACC = NW * 4 * 128 * 4;
constexpr int PV_SMEM = PSMEM_RING > PV_ACC ? PSMEM_RING : PV_ACC;
__device__ __forceinline__ uint32_t pack_hh(__half a, __half b) {
  __half2 h = __halves2half2(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}
}  // namespace mma16

// PASS 0: full attention (chunk states).  With the ART rule: PASS 1, the probe pass -- per tile and
// head the record (m'_t, l_t, the probe lanes of acc_t), each tile on its own reference m'_t, no chunk
// states -- and PASS 2, the limited pass -- chunk states over the tiles each head consumes (up to its
// stop tile from the rule), on a reference no later than its last consumed tile.
template <int GP, int PASS>
__global__ void __launch_bounds__(NT, 2) q8_pv_mma_kernel(const __grid_constant__ Params p) {
  constexpr int D = 128, NB = 4;
  static_assert(GP == 4, "one lane per (row, head) pair over 8 rows: four heads");
  static_assert(PASS >= 0 && PASS <= 2, "pass");
  extern __shared__ __align__(16) uint8_t s_dyn[];  // the ring while the rows stream, then the accumulators
  __shared__ float s_mp[CTMAX][4], s_ref[4];
  __shared__ int s_live[CTMAX];
  __shared__ float s_l[NW][4];
  __shared__ int s_plane[PASS == 1 ? 32 : 1];                   // the probe lanes (d positions)
  __shared__ __align__(16) float s_wg[PASS == 1 ? NW : 1][16][4];  // a group's weights, row x head
  __shared__ int s_stop[4];
  grid_dep_wait();  // pass 1's scores and maxima
  grid_dep_launch();
  const Range r = cta_range(p);
  if (r.c0 >= r.t1) return;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 2, t = lane & 3;
  const int unit = blockIdx.y;
  const int bk = unit / p.S, split = unit % p.S;
  const int b = bk / p.Hkv, kvh = bk % p.Hkv;
  const int T = p.T, G = p.G;
  const float tau = p.tau;
  const int nct = r.c1 - r.c0;  // <= CTMAX

  // running maxima m'_t, the chunk's reference and the tiles left unread, as in q8_pv_kernel; the
  // maxima of every head are loaded together (one round trip to memory, not one per head)
  if (warp == 0) {
    const float* cm = p.cmax + static_cast<long long>(unit) * p.CPS * G;
    const float* tmx = p.tmax + (static_cast<long long>(bk) * p.n_max + r.c0 + lane) * G;
    float mc[4], own4[4];
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      own4[h] = (h < G && lane < nct) ? tmx[h] : -INFINITY;
      mc[h] = -INFINITY;
    }
    for (int c = lane; c < static_cast<int>(blockIdx.x); c += 32)
#pragma unroll
      for (int h = 0; h < 4; ++h)
        if (h < G) mc[h] = fmaxf(mc[h], cm[c * G + h]);
    // the limited pass: each head's last consumed tile and their maximum (tiles past it are not read)
    const int my_stop = (PASS == 2 && lane < G) ? p.stop[(static_cast<long long>(b) * p.Hq + kvh * G + lane) * p.S + split] : -1;
    int smax = my_stop;
#pragma unroll
    for (int off = 1; off < 4; off <<= 1) smax = max(smax, __shfl_xor_sync(0xffffffffu, smax, off));
    smax = __shfl_sync(0xffffffffu, smax, 0);  // (lanes 0..3 hold the heads' stops)
    bool live = false;
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      if (h >= G) break;
      const float m = warp_max(mc[h]);
      const float own = own4[h];
      float x = own;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const float y = __shfl_up_sync(0xffffffffu, x, off);
        if (lane >= off) x = fmaxf(x, y);
      }
      const float mpj = fmaxf(m, x);
      if (lane < nct) {
        s_mp[lane][h] = mpj;
        if (!(exp2f(own - mpj) < tau)) live = true;
      }
      if (lane == 31) s_ref[h] = mpj;
    }
    if (PASS == 2) live = live && r.c0 + lane <= smax;
    if (lane < nct) s_live[lane] = live ? 1 : 0;
    const unsigned dead = __ballot_sync(0xffffffffu, lane < nct && !live);
    if (PASS != 2 && lane == 0 && dead) atomicAdd(&p.vskip[unit * 2 + 1], __popc(dead));
    if constexpr (PASS == 2) {  // the reference: m' at the last tile of the chunk the head consumes
      __syncwarp();
      if (lane < G) {
        const int last = min(r.c1 - 1, my_stop);
        s_ref[lane] = last >= r.c0 ? s_mp[last - r.c0][lane] : -INFINITY;
        s_stop[lane] = my_stop;
      }
    }
    if constexpr (PASS == 1) s_plane[lane] = lane < p.n_probe ? p.lanes[lane] : 0;
  }
  __syncthreads();

  const uint16_t* vsb = p.vs + static_cast<long long>(bk) * p.L_max * NB;
  const float* scb = p.scores + static_cast<long long>(bk) * p.L_max * GP;
  const int ipt = T / mma16::ROWS, ips = T / mma16::STEP;  // groups and steps per tile (T >= 32)
  const int nsteps = (warp < nct ? (nct - warp + NW - 1) / NW : 0) * ips;
  const uint32_t dyn = smem_u32(s_dyn), base = (dyn + 1023u) & ~1023u;
  uint8_t* const codes = s_dyn + (base - dyn) + warp * mma16::PBV * mma16::BOX;
  uint8_t* const vscales = s_dyn + (base - dyn) + mma16::PSM_VS + warp * mma16::PBV * mma16::STEP * 8;
  uint8_t* const srows = s_dyn + (base - dyn) + mma16::PSM_SC + warp * mma16::PBV * mma16::STEP * 16;
  const uint32_t bars = base + mma16::PSM_BARS + warp * mma16::PBV * 8;
  if (lane == 0) {
    for (int i = 0; i < mma16::PBV; ++i) mbar_init(bars + 8 * i, 1);
    fence_mbar_init();
  }
  // copies of a step (32 rows of a tile): one TMA box of V code rows (skipped for a tile left unread
  // and for a step wholly past the sequence), and per lane l the V scales (not for a tile left unread)
  // and the scores of row l; rows past the sequence are copied (codes) or not copied (scales, scores)
  // and weigh zero
  uint32_t pend = 0u, phase = 0u;  // bit s: slot s has a box in flight / the parity it completes
  Walk wi, wc;
  wi.start(r, warp, T);
  wc = wi;
  int ks = 0;
  // the V-scale areas of this warp's ring start as zeros: a row never copied then scales to a finite
  // value, and its weight (zero) keeps it out of the sum
  for (int i = lane; i < mma16::PBV * mma16::STEP * 2; i += 32) reinterpret_cast<uint32_t*>(vscales)[i] = 0u;
  __syncwarp();
  auto issue = [&]() {
    if (ks < nsteps) {
      const int sl = ks % mma16::PBV;
      ART_DCHECK(wi.t >= r.c0 && wi.t < r.c1 && wi.t - r.c0 < CTMAX && wi.row0 >= wi.t * T && wi.row0 < (wi.t + 1) * T, p.ws_status);
      ART_DCHECK(wi.row0 >= 0 && (wi.row0 < p.L_max || wi.row0 >= wi.rend), p.ws_status);
      const bool live_t = s_live[wi.t - r.c0] != 0;
      if (live_t && wi.row0 < wi.rend) {
        if (lane == 0) {
          mbar_arrive_expect_tx(bars + 8 * sl, mma16::BOX);
          tma_load_3d(smem_u32(codes + sl * mma16::BOX), &p.tmV, bars + 8 * sl, 0, wi.row0, bk);
        }
        pend |= 1u << sl;
      }
      if (wi.row0 + lane < wi.rend) {
        if (live_t)
          cp_async<8>(smem_u32(vscales + sl * mma16::STEP * 8) + lane * 8, vsb + static_cast<long long>(wi.row0 + lane) * NB);
        cp_async<16>(smem_u32(srows + sl * mma16::STEP * 16) + lane * 16, scb + static_cast<long long>(wi.row0 + lane) * GP);
      }
      wi.next(r, T, ips, mma16::STEP);
    }
    ++ks;
    cp_async_commit();
  };

  float acc[16][4];  // n-tile (block b, j) = 4 b + j
#pragma unroll
  for (int n = 0; n < 16; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.f;
  float pacc[4] = {0.f, 0.f, 0.f, 0.f};  // the probe pass: this lane's probe lane of each head, over the tile
  float l = 0.f, mp = 0.f, fac = 0.f;
  bool live = false;
  int nskip = 0;
  const bool head_ok = t < G;
  auto body = [&](int sl, int half) {
    if (wc.ik == 0) {  // a new tile: m'_t of this lane's head and the factor to the chunk's reference
      const int j = wc.t - r.c0;
      mp = head_ok ? s_mp[j][t] : 0.f;
      if constexpr (PASS == 0) fac = head_ok ? exp2f(mp - s_ref[t]) : 0.f;
      if constexpr (PASS == 1) fac = head_ok ? 1.f : 0.f;  // the tile's own reference
      if constexpr (PASS == 2) fac = (head_ok && wc.t <= s_stop[t]) ? exp2f(mp - s_ref[t]) : 0.f;
      live = s_live[j] != 0;
    }
    const uint8_t* box = codes + sl * mma16::BOX + half * mma16::ROWS * 128;  // rows 16 half .. (same swizzle phase)
    const uint8_t* vsl = vscales + (sl * mma16::STEP + half * mma16::ROWS) * 8;
    const uint8_t* ssl = srows + (sl * mma16::STEP + half * mma16::ROWS) * 16;
    // weights of rows g and g + 8 for head t
    float wk[2];
#pragma unroll
    for (int rr = 0; rr < 2; ++rr) {
      const int row = g + 8 * rr;
      const bool ok = head_ok && wc.row0 + row < wc.rend;
      const float sj = ok ? reinterpret_cast<const float*>(ssl + row * 16)[t] : -INFINITY;
      const float pj = exp2f(sj - mp);  // 0 for rows past the end and padded heads
      const float wj = pj * fac;
      l += wj;  // skipped rows stay in the denominator
      wk[rr] = (live && !(pj < tau) && pj > 0.f) ? wj : 0.f;
    }
    const unsigned kb0 = __ballot_sync(0xffffffffu, wk[0] > 0.f), kb1 = __ballot_sync(0xffffffffu, wk[1] > 0.f);
    if (PASS != 2 && t == 0) {  // rows g and g + 8 left out of every head's numerator
      if (wc.row0 + g < wc.rend && ((kb0 >> (4 * g)) & 0xFu) == 0u) ++nskip;
      if (wc.row0 + g + 8 < wc.rend && ((kb1 >> (4 * g)) & 0xFu) == 0u) ++nskip;
    }
    if constexpr (PASS == 1) {
      // the probe pass needs the probe lanes of the sums only: lane i < n_probe takes probe i over the
      // group's 16 rows and the heads (weights through shared memory), on the CUDA cores
      if (head_ok) {
        s_wg[warp][g][t] = wk[0];
        s_wg[warp][g + 8][t] = wk[1];
      } else if (t < 4) {
        s_wg[warp][g][t] = 0.f;
        s_wg[warp][g + 8][t] = 0.f;
      }
      __syncwarp();
      // up to 16 probe lanes: two lanes per probe lane, 8 rows each (the halves add at the flush)
      const bool halves = p.n_probe <= 16;
      const int pi = halves ? (lane & 15) : lane, r0 = halves ? (lane >> 4) * 8 : 0;
      if ((kb0 | kb1) != 0u && pi < p.n_probe) {
        const int pos = s_plane[pi], blk = pos >> 5;
#pragma unroll 4
        for (int row = r0; row < r0 + (halves ? 8 : mma16::ROWS); ++row) {
          const float code = static_cast<float>(static_cast<int8_t>(box[mma16::swz(row, pos)]));
          const float vv = code * __half2float(__ushort_as_half(reinterpret_cast<const uint16_t*>(vsl + row * 8)[blk]));
          const float4 w4 = *reinterpret_cast<const float4*>(&s_wg[warp][row][0]);
          pacc[0] = fmaf(w4.x, vv, pacc[0]);
          pacc[1] = fmaf(w4.y, vv, pacc[1]);
          pacc[2] = fmaf(w4.z, vv, pacc[2]);
          pacc[3] = fmaf(w4.w, vv, pacc[3]);
        }
      }
      __syncwarp();
    } else if ((kb0 | kb1) != 0u) {  // otherwise no row of the group is dequantised
      // A: head g's weights (g < 4) for rows 2t, 2t + 1, 2t + 8, 2t + 9 times each row's V scale
      const int src = 8 * t + (g & 3);
      const float w0 = __shfl_sync(0xffffffffu, wk[0], src), w1 = __shfl_sync(0xffffffffu, wk[0], src + 4);
      const float w2 = __shfl_sync(0xffffffffu, wk[1], src), w3 = __shfl_sync(0xffffffffu, wk[1], src + 4);
      const uint2 s0 = *reinterpret_cast<const uint2*>(vsl + (2 * t) * 8);
      const uint2 s1 = *reinterpret_cast<const uint2*>(vsl + (2 * t + 1) * 8);
      const uint2 s2 = *reinterpret_cast<const uint2*>(vsl + (2 * t + 8) * 8);
      const uint2 s3 = *reinterpret_cast<const uint2*>(vsl + (2 * t + 9) * 8);
      // (V scales of a row not copied: an earlier row's, or zero)
      const uint32_t sv[4][2] = {{s0.x, s0.y}, {s1.x, s1.y}, {s2.x, s2.y}, {s3.x, s3.y}};
      const int vrow[4] = {2 * t, 2 * t + 1, 2 * t + 8, 2 * t + 9};
      const __half2 bias = __half2half2(__ushort_as_half(static_cast<unsigned short>(0x6480)));  // 1152
#pragma unroll
      for (int bb = 0; bb < NB; ++bb) {
        uint32_t vw[4];  // this lane's 4 code bytes of each row, positions 32 b + 4 g .. + 3
#pragma unroll
        for (int i = 0; i < 4; ++i)
          vw[i] = *reinterpret_cast<const uint32_t*>(box + mma16::swz(vrow[i], 32 * bb + 4 * g)) ^ 0x80808080u;
        float sc[4];  // the four rows' scales of block bb
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float2 s2 = __half22float2(*reinterpret_cast<const __half2*>(&sv[i][bb >> 1]));
          sc[i] = (bb & 1) ? s2.y : s2.x;
        }
        uint32_t a[4] = {0u, 0u, 0u, 0u};
        if (g < 4) {  // weight x scale of rows (2t, 2t + 1) and (2t + 8, 2t + 9): f16 part and remainder
          const float2 x01 = __fmul2_rn(make_float2(w0, w1), make_float2(sc[0], sc[1]));
          const float2 x23 = __fmul2_rn(make_float2(w2, w3), make_float2(sc[2], sc[3]));
          const __half2 h01 = __float22half2_rn(x01), h23 = __float22half2_rn(x23);
          const float2 m1 = make_float2(-1.f, -1.f);
          const __half2 l01 = __float22half2_rn(__ffma2_rn(__half22float2(h01), m1, x01));
          const __half2 l23 = __float22half2_rn(__ffma2_rn(__half22float2(h23), m1, x23));
          a[0] = *reinterpret_cast<const uint32_t*>(&h01);
          a[1] = *reinterpret_cast<const uint32_t*>(&l01);
          a[2] = *reinterpret_cast<const uint32_t*>(&h23);
          a[3] = *reinterpret_cast<const uint32_t*>(&l23);
        }
        // B: rows (2t, 2t + 1) and (2t + 8, 2t + 9) at position 32 b + 4 g + j, for j = 0..3
        const uint32_t pa0 = __byte_perm(vw[0], vw[1], 0x5140u), pb0 = __byte_perm(vw[0], vw[1], 0x7362u);
        const uint32_t pa1 = __byte_perm(vw[2], vw[3], 0x5140u), pb1 = __byte_perm(vw[2], vw[3], 0x7362u);
        const uint32_t p0[2] = {pa0, pb0}, p1[2] = {pa1, pb1};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          uint32_t x0 = __byte_perm(p0[j >> 1], 0x64646464u, (j & 1) ? 0x4342u : 0x4140u);
          uint32_t x1 = __byte_perm(p1[j >> 1], 0x64646464u, (j & 1) ? 0x4342u : 0x4140u);
          const __half2 h0 = __hsub2(*reinterpret_cast<const __half2*>(&x0), bias);
          const __half2 h1 = __hsub2(*reinterpret_cast<const __half2*>(&x1), bias);
          mma16::mma_f16(acc[4 * bb + j], a, *reinterpret_cast<const uint32_t*>(&h0),
                         *reinterpret_cast<const uint32_t*>(&h1));
        }
      }
    }
    wc.next(r, T, ipt, mma16::ROWS);
  };
  // the probe pass, at the end of a tile: its records (head t's m'_t and denominator, head g's probe
  // lanes of the accumulators: f16 part in row g + remainder in row g + 8), then fresh sums
  auto flush = [&](int tile) {  // (the probe pass)
    float lt = l;  // head t's denominator over the tile (lanes of the same t)
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) lt += __shfl_xor_sync(0xffffffffu, lt, off);
    const long long rec0 = (static_cast<long long>(b) * p.Hq + kvh * G) * p.n_max + tile;  // head 0's
    ART_DCHECK(tile >= 0 && tile < p.n_max, p.ws_status);
    if (g == 0 && head_ok) {
      float* rc = p.probe + (rec0 + static_cast<long long>(t) * p.n_max) * REC;
      rc[0] = mp;
      rc[1] = lt;
    }
    if (p.n_probe <= 16) {  // the two halves of each probe lane
#pragma unroll
      for (int h = 0; h < 4; ++h) pacc[h] += __shfl_xor_sync(0xffffffffu, pacc[h], 16);
    }
    if (lane < p.n_probe) {  // probe `lane` of every head
#pragma unroll
      for (int h = 0; h < 4; ++h)
        if (h < G) p.probe[(rec0 + static_cast<long long>(h) * p.n_max) * REC + 2 + lane] = pacc[h];
    }
#pragma unroll
    for (int h = 0; h < 4; ++h) pacc[h] = 0.f;
    l = 0.f;
  };

#pragma unroll 1
  for (int k = 0; k < mma16::PBV - 1; ++k) issue();
#pragma unroll 1
  for (int k = 0; k < nsteps; ++k) {
    issue();                          // step k + PBV - 1, into the slot step k - 1 left
    cp_async_wait<mma16::PBV - 1>();  // step k's scales and scores (this lane's copies)
    const int sl = k % mma16::PBV;
    if (!mma16::wait_box(bars, sl, pend, phase, p.ws_status)) break;  // its V codes, when they were copied
    __syncwarp();
    const int t_step = wc.t;  // (a step never straddles two tiles)
#pragma unroll
    for (int half = 0; half < 2; ++half) body(sl, half);
    if constexpr (PASS == 1)
      if (wc.ik == 0) flush(t_step);  // the step ended its tile
    __syncwarp();
  }
  mma16::drain_boxes(bars, mma16::PBV, pend, phase, p.ws_status);  // (only after a timeout)
  cp_async_wait<0>();
  {
    int ns_w = nskip;
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) ns_w += __shfl_xor_sync(0xffffffffu, ns_w, off);
    if (lane == 0 && ns_w) atomicAdd(&p.vskip[unit * 2], ns_w);
  }
  if constexpr (PASS == 1) return;  // the records are the pass's output
  // the denominators: lanes of the same head t
#pragma unroll
  for (int off = 4; off < 32; off <<= 1) l += __shfl_xor_sync(0xffffffffu, l, off);
  __syncthreads();  // every warp is done with its ring before the accumulators overwrite it
  float* s_acc = reinterpret_cast<float*>(s_dyn);  // [NW][4][D]
  if (g < 4) {  // head g: hi (row g) + lo (row g + 8) at positions 32 b + 4 (2t) + j and 32 b + 4 (2t + 1) + j
#pragma unroll
    for (int bb = 0; bb < NB; ++bb)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        s_acc[(warp * 4 + g) * D + 32 * bb + 4 * (2 * t) + j] = acc[4 * bb + j][0] + acc[4 * bb + j][2];
        s_acc[(warp * 4 + g) * D + 32 * bb + 4 * (2 * t + 1) + j] = acc[4 * bb + j][1] + acc[4 * bb + j][3];
      }
  }
  if (lane < 4) s_l[warp][lane] = l;
  __syncthreads();
  for (int idx = threadIdx.x; idx < G * D; idx += NT) {
    const int h = idx / D, dd = idx % D;
    float a = 0.f;
#pragma unroll
    for (int w2 = 0; w2 < NW; ++w2) a += s_acc[(w2 * 4 + h) * D + dd];
    const long long hq = static_cast<long long>(b) * p.Hq + kvh * G + h;
    float* dst = p.part + ((hq * p.S + split) * p.CPS + blockIdx.x) * (2 + D);
    dst[2 + dd] = a;
    if (dd == 0) {
      float lsum = 0.f;
#pragma unroll
      for (int w2 = 0; w2 < NW; ++w2) lsum += s_l[w2][h];
      dst[0] = s_ref[h];
      dst[1] = lsum;
    }
  }
}

// ------------------------------------------------------------------ the ART rule over the probe records
// One CTA of RW warps per (query head, split), 32 * RW tiles of the split per round, thread = tile:
// the records' running merge (an inclusive scan of the online-softmax merge within each warp, the
// warps' totals and the state carried from earlier rounds prepended) gives every tile's probe
// x^(t) = acc^(t)[lanes] / l^(t); with the previous tile's probe (zeros before the first tile) the
// magnitude change | |x^(t)| - |x^(t-1)| | and the direction change 1 - cos =
// |x^(t)/|x^(t)| - x^(t-1)/|x^(t-1)||^2 / 2 (0 when both probes are zero, 1 when one is); a tile holds
// when both are below their thresholds, and the split stops at the first tile whose run of holding
// tiles reaches the patience ("Resumen Tecnico: ART", S2.2-S2.3).  Output: the stop tile (absolute
// index; the split's last tile when the rule never fires) and the tiles consumed.
constexpr int RW = 16;
constexpr int kNoStop = 0x7fffffff;
template <int PC>
struct RuleState {
  float m, l, a[PC];
};

template <int PC>
__global__ void __launch_bounds__(RW * 32) q8_rule_kernel(const __grid_constant__ Params p) {
  grid_dep_wait();  // the probe pass's records
  grid_dep_launch();
  __shared__ RuleState<PC> s_tot[RW];             // each warp's merged records
  __shared__ float s_lx[RW][PC], s_ln[RW];        // each warp's last probe and its norm
  __shared__ int s_allh[RW], s_trail[RW], s_first[RW];
  __shared__ RuleState<PC> s_carry;               // the state carried from earlier rounds ...
  __shared__ float s_cx[PC], s_cn;                // ... its probe and norm
  __shared__ int s_crun, s_stop;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int hq = static_cast<int>(blockIdx.x / p.S), split = static_cast<int>(blockIdx.x % p.S);
  int L = p.seq_lens[hq / p.Hq];
  if (L < 1 || L > p.L_max) L = 0;
  const int n = (L + p.T - 1) / p.T;
  const int ta = static_cast<int>((static_cast<long long>(split) * n) / p.S);
  const int tb = static_cast<int>((static_cast<long long>(split + 1) * n) / p.S);
  auto rescale = [](float x, float M) { return x == -INFINITY ? 0.f : exp2f(x - M); };
  // (m, l, a) <- earlier (mo, lo, ao) merged with (m, l, a)
  auto merge = [&](float& m, float& l, float (&a)[PC], float mo, float lo, const float* ao) {
    const float M = fmaxf(m, mo);
    const float cs = rescale(m, M), co = rescale(mo, M);
    l = cs * l + co * lo;
    m = M;
#pragma unroll
    for (int i = 0; i < PC; ++i) a[i] = cs * a[i] + co * ao[i];
  };
  if (threadIdx.x == 0) {
    s_carry.m = -INFINITY;
    s_carry.l = 0.f;
    s_cn = 0.f;
    s_crun = 0;
    s_stop = -1;
  }
  if (threadIdx.x < PC) s_carry.a[threadIdx.x] = s_cx[threadIdx.x] = 0.f;
  __syncthreads();
  for (int base = ta; base < tb; base += RW * 32) {
    const int tt = base + warp * 32 + lane;
    const bool valid = tt < tb;
    float m = -INFINITY, l = 0.f, a[PC];
#pragma unroll
    for (int i = 0; i < PC; ++i) a[i] = 0.f;
    if (valid) {  // (records are 136 bytes apart: 8-byte loads)
      const float2* rc = reinterpret_cast<const float2*>(p.probe + (static_cast<long long>(hq) * p.n_max + tt) * REC);
      const float2 ml = rc[0];
      m = ml.x;
      l = ml.y;
#pragma unroll
      for (int i = 0; i < PC; i += 2) {
        const float2 v = rc[1 + i / 2];
        a[i] = i < p.n_probe ? v.x : 0.f;
        a[i + 1] = i + 1 < p.n_probe ? v.y : 0.f;
      }
    }
#pragma unroll 1
    for (int off = 1; off < 32; off <<= 1) {  // the warp's inclusive scan
      const float mo = __shfl_up_sync(0xffffffffu, m, off), lo = __shfl_up_sync(0xffffffffu, l, off);
      float ao[PC];
#pragma unroll
      for (int i = 0; i < PC; ++i) ao[i] = __shfl_up_sync(0xffffffffu, a[i], off);
      if (lane >= off) merge(m, l, a, mo, lo, ao);
    }
    if (lane == 31) {
      s_tot[warp].m = m;
      s_tot[warp].l = l;
#pragma unroll
      for (int i = 0; i < PC; ++i) s_tot[warp].a[i] = a[i];
    }
    __syncthreads();
    {  // prepend the earlier warps' totals and the carried state
      float cm = s_carry.m, cl = s_carry.l, ca[PC];
#pragma unroll
      for (int i = 0; i < PC; ++i) ca[i] = s_carry.a[i];
      for (int u = 0; u < warp; ++u) {
        float tm = s_tot[u].m, tl = s_tot[u].l, tv[PC];
#pragma unroll
        for (int i = 0; i < PC; ++i) tv[i] = s_tot[u].a[i];
        merge(tm, tl, tv, cm, cl, ca);
        cm = tm;
        cl = tl;
#pragma unroll
        for (int i = 0; i < PC; ++i) ca[i] = tv[i];
      }
      merge(m, l, a, cm, cl, ca);
    }
    const float inv = l > 0.f ? 1.f / l : 0.f;
    float x[PC], sq = 0.f;
#pragma unroll
    for (int i = 0; i < PC; ++i) {
      x[i] = a[i] * inv;
      sq = fmaf(x[i], x[i], sq);
    }
    const float nrm = sqrtf(sq);
    if (lane == 31) {
#pragma unroll
      for (int i = 0; i < PC; ++i) s_lx[warp][i] = x[i];
      s_ln[warp] = nrm;
    }
    __syncthreads();
    float nrmp = __shfl_up_sync(0xffffffffu, nrm, 1);
    if (lane == 0) nrmp = warp == 0 ? s_cn : s_ln[warp - 1];
    const bool both = nrm > 0.f && nrmp > 0.f;
    const float in = both ? 1.f / nrm : 0.f, ip = both ? 1.f / nrmp : 0.f;
    float dd = 0.f;
#pragma unroll
    for (int i = 0; i < PC; ++i) {
      float xp = __shfl_up_sync(0xffffffffu, x[i], 1);
      if (lane == 0) xp = warp == 0 ? s_cx[i] : s_lx[warp - 1][i];
      const float dl = x[i] * in - xp * ip;
      dd = fmaf(dl, dl, dd);
    }
    const float d_scale = fabsf(nrm - nrmp);
    const float d_dir = (nrm == 0.f && nrmp == 0.f) ? 0.f : ((nrm == 0.f || nrmp == 0.f) ? 1.f : 0.5f * dd);
    const bool hold = valid && d_scale < p.eps_scale && d_dir < p.eps_dir;
    const unsigned hbits = __ballot_sync(0xffffffffu, hold);
    if (lane == 0) {
      s_allh[warp] = hbits == 0xffffffffu;
      s_trail[warp] = __clz(~hbits);  // holding tiles at the warp's end
    }
    __syncthreads();
    int crun = s_crun;  // the run of holding tiles entering this warp
    for (int u = 0; u < warp; ++u) crun = s_allh[u] ? crun + 32 : s_trail[u];
    const unsigned zeros = ~hbits & ((1u << lane) - 1u);
    const int run = !hold ? 0 : (zeros == 0u ? crun + lane + 1 : lane - (31 - __clz(zeros)));
    const unsigned rbits = __ballot_sync(0xffffffffu, hold && run >= p.patience);
    if (lane == 0) s_first[warp] = rbits ? tt + __ffs(rbits) - 1 : kNoStop;
    // the round's last tile carries its state into the next round
    const int last = min(base + RW * 32, tb) - 1;
    __syncthreads();
    int first = kNoStop;
#pragma unroll
    for (int u = 0; u < RW; ++u) first = min(first, s_first[u]);
    if (first != kNoStop) {
      if (threadIdx.x == 0) s_stop = first;
      break;  // (uniform: every thread saw the same minimum)
    }
    if (tt == last) {
      s_carry.m = m;
      s_carry.l = l;
#pragma unroll
      for (int i = 0; i < PC; ++i) {
        s_carry.a[i] = a[i];
        s_cx[i] = x[i];
      }
      s_cn = nrm;
      s_crun = run;
    }
    __syncthreads();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const int stop = s_stop >= 0 ? s_stop : tb - 1;  // every tile (an empty split: none)
    p.stop[static_cast<long long>(hq) * p.S + split] = stop;
    p.ws_used[static_cast<long long>(hq) * p.S + split] = stop - ta + 1;
  }
}

// ------------------------------------------------------------------ pass 2: weights, skip, PV
template <int D, int GP>
__global__ void __launch_bounds__(NT, 2) q8_pv_kernel(const __grid_constant__ Params p) {
  using Gm = Geom<D, GP>;
  constexpr int EPT = Gm::EPT, TPR = Gm::TPR, RPI = Gm::RPI, NB = Gm::NB, SLOT = Gm::SLOT;
  constexpr int RING = NW * P * SLOT, ACC = NW * GP * D * 4;
  // the ring while the rows stream, then the warps' accumulators
  __shared__ __align__(16) uint8_t s_buf[RING > ACC ? RING : ACC];
  __shared__ float s_mp[CTMAX][GP], s_ref[GP];
  __shared__ int s_live[CTMAX];
  __shared__ float s_l[NW][GP];
  grid_dep_wait();  // pass 1's scores and maxima
  grid_dep_launch();
  const Range r = cta_range(p);
  if (r.c0 >= r.t1) return;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int sub = lane % TPR, rsub = lane / TPR;
  const int unit = blockIdx.y;
  const int bk = unit / p.S, split = unit % p.S;
  const int b = bk / p.Hkv, kvh = bk % p.Hkv;
  const int T = p.T, G = p.G;
  const float tau = p.tau;
  const int nct = r.c1 - r.c0;  // <= CTMAX

  // Running maxima m'_t of the chunk's tiles (lane j: tile c0 + j): the maximum of the split's
  // chunks before this one, then the inclusive prefix maximum of the chunk's tile maxima.  ref
  // (m' at the chunk's last tile) is the reference of the chunk's weights.  A tile whose own
  // maximum already fails the skip test for every head has every row skipped: its V rows are not
  // read at all (the scores still feed the denominator).
  if (warp == 0) {
    const float* cm = p.cmax + static_cast<long long>(unit) * p.CPS * G;
    bool live = false;
    for (int g = 0; g < G; ++g) {
      float m = -INFINITY;
      for (int c = lane; c < static_cast<int>(blockIdx.x); c += 32) m = fmaxf(m, cm[c * G + g]);
      m = warp_max(m);
      const float own = lane < nct ? p.tmax[(static_cast<long long>(bk) * p.n_max + r.c0 + lane) * G + g]
                                   : -INFINITY;
      float x = own;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const float y = __shfl_up_sync(0xffffffffu, x, off);
        if (lane >= off) x = fmaxf(x, y);
      }
      const float mpj = fmaxf(m, x);
      if (lane < nct) {
        s_mp[lane][g] = mpj;
        if (!(exp2f(own - mpj) < tau)) live = true;
      }
      if (lane == 31) s_ref[g] = mpj;
    }
    if (lane < nct) s_live[lane] = live ? 1 : 0;
    const unsigned dead = __ballot_sync(0xffffffffu, lane < nct && !live);
    if (lane == 0 && dead) atomicAdd(&p.vskip[unit * 2 + 1], __popc(dead));
  }
  __syncthreads();

  const int8_t* vb = p.v + static_cast<long long>(bk) * p.L_max * D;
  const uint16_t* vsb = p.vs + static_cast<long long>(bk) * p.L_max * NB;
  const float* scb = p.scores + static_cast<long long>(bk) * p.L_max * GP;
  const int ipt = T / RPI;
  const int niter = (warp < nct ? (nct - warp + NW - 1) / NW : 0) * ipt;
  uint8_t* ring = s_buf + warp * P * SLOT;
  const uint32_t ring_a = smem_u32(ring);
  // rows past the end are not copied (stale slot bytes, zero weight); dead tiles copy scores only
  Walk wi, wc;
  wi.start(r, warp, T);
  wc = wi;
  int ki = 0;
  auto issue = [&]() {
    if (ki < niter) {
      const int row = wi.row0 + rsub;
      if (row < wi.rend) {
        const uint32_t slot = ring_a + (ki & (P - 1)) * SLOT;
        if (sub == 0) {
          const float* src = scb + static_cast<long long>(row) * GP;
          const uint32_t dst = slot + Gm::SLOT_CODES + Gm::SLOT_SCALES + rsub * GP * 4;
          if constexpr (GP == 8) {
            cp_async<16>(dst, src);
            cp_async<16>(dst + 16, src + 4);
          } else {
            cp_async<GP * 4>(dst, src);
          }
        }
        if (s_live[wi.t - r.c0]) {
          cp_async<EPT>(slot + rsub * D + sub * EPT, vb + static_cast<long long>(row) * D + sub * EPT);
          if (sub == 0) cp_async<NB * 2>(slot + Gm::SLOT_CODES + rsub * NB * 2, vsb + static_cast<long long>(row) * NB);
        }
      }
      wi.next(r, T, ipt, RPI);
    }
    ++ki;
    cp_async_commit();
  };

  // Weights: lane (pr, ph) = (lane / GP, lane % GP) forms the weight of head ph of row pr of each
  // group (RPI * GP <= 32 pairs) and accumulates that head's denominator; the lanes of a row then
  // fetch the row's weights by shuffle.
  constexpr int NPAIR = RPI * GP;
  static_assert(NPAIR <= 32, "one lane per (row, head) of a group");
  const int pr = lane / GP, ph = lane % GP;
  const bool pair = lane < NPAIR && ph < G;
  float2 acc[GP][EPT / 2];
#pragma unroll
  for (int h = 0; h < GP; ++h)
#pragma unroll
    for (int i = 0; i < EPT / 2; ++i) acc[h][i] = make_float2(0.f, 0.f);
  float l = 0.f, mp = 0.f, fac = 0.f;
  bool live = false;
  int nskip = 0;  // rows of this lane's row slot left out of every head's numerator
  auto body = [&](int k) {
    if (wc.ik == 0) {
      // a new tile: m'_t of this lane's head; fac = 2^(m'_t - ref) turns a skip-test weight into
      // a numerator weight
      const int j = wc.t - r.c0;
      mp = pair ? s_mp[j][ph] : 0.f;
      fac = pair ? exp2f(mp - s_ref[ph]) : 0.f;
      live = s_live[j] != 0;
    }
    const uint8_t* slot = ring + (k & (P - 1)) * SLOT;
    float wk = 0.f;
    {
      const bool ok = pair && wc.row0 + pr < wc.rend;
      const float sj = ok ? reinterpret_cast<const float*>(slot + Gm::SLOT_CODES + Gm::SLOT_SCALES)[lane] : -INFINITY;
      const float pj = exp2f(sj - mp);  // 0 for rows past the end and padded heads
      const float wj = pj * fac;
      l += wj;  // skipped rows stay in the denominator
      wk = (live && !(pj < tau) && pj > 0.f) ? wj : 0.f;
    }
    float w[GP];
    bool any = false;
#pragma unroll
    for (int h = 0; h < GP; ++h) {
      w[h] = __shfl_sync(0xffffffffu, wk, rsub * GP + h);
      any |= w[h] > 0.f;
    }
    if (sub == 0 && !any && wc.row0 + rsub < wc.rend) ++nskip;
    if (any) {  // otherwise the row is not dequantised
      uint32_t cw[EPT / 4];
      lds_codes<EPT>(slot + rsub * D + sub * EPT, cw);
      const float vsc = __half2float(
          __ushort_as_half(reinterpret_cast<const uint16_t*>(slot + Gm::SLOT_CODES)[rsub * NB + (sub * EPT) / 32]));
      float2 vf[EPT / 2];
      codes_to_f2<EPT>(cw, vf);
#pragma unroll
      for (int h = 0; h < GP; ++h) {
        const float wv = w[h] * vsc;
        const float2 w2 = make_float2(wv, wv);
#pragma unroll
        for (int i = 0; i < EPT / 2; ++i) acc[h][i] = __ffma2_rn(w2, vf[i], acc[h][i]);
      }
    }
    wc.next(r, T, ipt, RPI);
  };

  // two groups per step (niter is a multiple of ipt, which is even): their chains interleave
#pragma unroll 1
  for (int k = 0; k < P - 2; ++k) issue();
#pragma unroll 1
  for (int k = 0; k < niter; k += 2) {
    issue();
    issue();
    cp_async_wait<P - 2>();
    __syncwarp();
    body(k);
    body(k + 1);
    __syncwarp();
  }
  cp_async_wait<0>();
  {
    int ns_w = nskip;
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) ns_w += __shfl_xor_sync(0xffffffffu, ns_w, off);
    if (lane == 0 && ns_w) atomicAdd(&p.vskip[unit * 2], ns_w);
  }

  // sum over the row groups of the warp, then over the warps
#pragma unroll
  for (int off = GP; off < 32; off <<= 1) l += __shfl_xor_sync(0xffffffffu, l, off);  // lane h < GP: head h
#pragma unroll
  for (int off = TPR; off < 32; off <<= 1) {
#pragma unroll
    for (int h = 0; h < GP; ++h) {
#pragma unroll
      for (int i = 0; i < EPT / 2; ++i) {
        acc[h][i].x += __shfl_xor_sync(0xffffffffu, acc[h][i].x, off);
        acc[h][i].y += __shfl_xor_sync(0xffffffffu, acc[h][i].y, off);
      }
    }
  }
  __syncthreads();  // every warp is done with its ring before the accumulators overwrite it
  float* s_acc = reinterpret_cast<float*>(s_buf);  // [NW][GP][D]
  if (lane < TPR) {
#pragma unroll
    for (int h = 0; h < GP; ++h) {
#pragma unroll
      for (int i = 0; i < EPT / 2; ++i)
        *reinterpret_cast<float2*>(&s_acc[(warp * GP + h) * D + sub * EPT + 2 * i]) = acc[h][i];
    }
  }
  if (lane < GP) s_l[warp][lane] = l;
  __syncthreads();
  for (int idx = threadIdx.x; idx < G * D; idx += NT) {
    const int h = idx / D, dd = idx % D;
    float a = 0.f;
#pragma unroll
    for (int w2 = 0; w2 < NW; ++w2) a += s_acc[(w2 * GP + h) * D + dd];
    const long long hq = static_cast<long long>(b) * p.Hq + kvh * G + h;
    float* dst = p.part + ((hq * p.S + split) * p.CPS + blockIdx.x) * (2 + D);
    dst[2 + dd] = a;
    if (dd == 0) {
      float lsum = 0.f;
#pragma unroll
      for (int w2 = 0; w2 < NW; ++w2) lsum += s_l[w2][h];
      dst[0] = s_ref[h];
      dst[1] = lsum;
    }
  }
}

// ------------------------------------------------------------------ combine
// One CTA of D threads per (batch, query head), thread = output element: the chunk states of every
// split merged online (running maximum, rescaled sums), loads of 8 chunks in flight at a time;
// then the per-split counters of the caller's split layout.
template <int D>
__global__ void __launch_bounds__(D) q8_combine_kernel(const __grid_constant__ Params p) {
  constexpr int CU = 32;  // chunk states loaded per batch (a split of up to 32 chunks in one round trip)
  grid_dep_wait();  // pass 2's chunk states
  const int hq = blockIdx.x;
  const int dd = threadIdx.x;
  const int b = hq / p.Hq, h = hq % p.Hq;
  const int bk = b * p.Hkv + h / p.G;
  int L = p.seq_lens[b];
  const bool bad = (L < 1 || L > p.L_max);
  if (bad) L = 0;
  const int n_tiles = (L + p.T - 1) / p.T;
  const float* ph = p.part + static_cast<long long>(hq) * p.S * p.CPS * (2 + D);
  float M = -INFINITY, den = 0.f, num = 0.f;
  for (int s = 0; s < p.S; ++s) {
    const int ns = static_cast<int>((static_cast<long long>(s + 1) * n_tiles) / p.S) -
                   static_cast<int>((static_cast<long long>(s) * n_tiles) / p.S);
    const int nch = (ns + p.CT - 1) / p.CT;
    const float* pc = ph + static_cast<long long>(s) * p.CPS * (2 + D);
    for (int c0 = 0; c0 < nch; c0 += CU) {
      float m[CU], lc[CU], ac[CU];
#pragma unroll
      for (int u = 0; u < CU; ++u) {
        const bool in = c0 + u < nch;
        m[u] = in ? pc[(c0 + u) * (2 + D)] : -INFINITY;
        lc[u] = in ? pc[(c0 + u) * (2 + D) + 1] : 0.f;
        ac[u] = in ? pc[(c0 + u) * (2 + D) + 2 + dd] : 0.f;
      }
#pragma unroll
      for (int u = 0; u < CU; ++u) {
        if (m[u] == -INFINITY) continue;
        if (m[u] > M) {
          const float r = exp2f(M - m[u]);
          den *= r;
          num *= r;
          M = m[u];
        }
        const float w = exp2f(m[u] - M);
        den += w * lc[u];
        num += w * ac[u];
      }
    }
    if (dd == 0) {
      if (!p.art) p.ws_used[static_cast<long long>(hq) * p.S + s] = ns;  // (with ART: the rule's count)
      if (h % p.G == 0) p.ws_tiles_read[static_cast<long long>(bk) * p.S + s] = ns;  // every K tile is read
    }
  }
  p.o[static_cast<long long>(hq) * D + dd] = bad ? __int_as_float(0x7fc00000) : num / den;
  if (dd == 0) {
    int consumed = n_tiles;
    if (p.art) {
      consumed = 0;
      for (int s = 0; s < p.S; ++s) consumed += p.ws_used[static_cast<long long>(hq) * p.S + s];
    }
    if (p.tiles) p.tiles[hq] = consumed;
    if (bad && h == 0) atomicOr(p.ws_status, kStatusSeqLen);
  }
}

// ------------------------------------------------------------------ host side
struct Dims {
  int B, Hq, Hkv, d, L_max, T, S;
};

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Workspace arrays after the common ones (which end at `base`), sized for the smallest chunk.
struct Layout2 {
  size_t scores, tmax, cmax, part, vskip, probe, stop, end;
  int n_max, CT, CPS;
};

inline Layout2 layout2(const Dims& s, size_t base) {
  Layout2 q;
  const int G = s.Hq / s.Hkv;
  q.n_max = (s.L_max + s.T - 1) / s.T;
  q.CT = chunk_tiles_min(s.T);
  const int per_split = (q.n_max + s.S - 1) / s.S;
  q.CPS = (per_split + q.CT - 1) / q.CT;
  const size_t bk = size_t(s.B) * s.Hkv, units = bk * s.S;
  q.scores = align256(base);
  q.tmax = align256(q.scores + 4 * bk * size_t(s.L_max) * gp_of(G));
  q.cmax = align256(q.tmax + 4 * bk * size_t(q.n_max) * G);
  q.part = align256(q.cmax + 4 * units * size_t(q.CPS) * G);
  q.vskip = align256(q.part + 4 * units * G * size_t(q.CPS) * (size_t(s.d) + 2));
  q.probe = align256(q.vskip + 8 * units);
  q.stop = align256(q.probe + 4 * size_t(s.B) * s.Hq * size_t(q.n_max) * REC);
  q.end = align256(q.stop + 4 * units * G);
  return q;
}

inline size_t workspace_end(const Dims& s, size_t base) { return layout2(s, base).end; }

// (batch, kv head, split) units index blockIdx.y
inline bool grid_ok(const Dims& s) { return 1LL * s.B * s.Hkv * s.S <= 65535; }

// Tiles per chunk: the one in [smallest, CTMAX] whose grid (2 CTAs per SM) finishes soonest,
// counting a CTA's time as its tile count and the waves it takes.
inline int choose_ct(const Dims& s, int sms) {
  const int n_max = (s.L_max + s.T - 1) / s.T;
  const int per_split = (n_max + s.S - 1) / s.S;
  const long long units = 1LL * s.B * s.Hkv * s.S, slots = 2LL * sms;
  int best = chunk_tiles_min(s.T);
  long long best_cost = -1;
  for (int ct = best; ct <= CTMAX; ++ct) {
    const long long ctas = units * ((per_split + ct - 1) / ct);
    const long long cost = ((ctas + slots - 1) / slots) * ct;
    if (best_cost < 0 || cost < best_cost) {
      best_cost = cost;
      best = ct;
    }
  }
  return best;
}

// Launch a pass that reads the previous pass's results with programmatic stream serialisation: its
// CTAs may be scheduled while the previous grid finishes and wait in grid_dep_wait() for its results.
template <typename Kernel>
cudaError_t launch_after(Kernel kernel, dim3 grid, int threads, size_t smem, cudaStream_t st, const Params& p,
                         bool overlap = true) {
  cudaLaunchConfig_t lc = {};
  cudaLaunchAttribute attr[1];
  lc.gridDim = grid;
  lc.blockDim = dim3(static_cast<unsigned>(threads), 1, 1);
  lc.dynamicSmemBytes = smem;
  lc.stream = st;
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = overlap ? 1 : 0;
  lc.attrs = attr;
  lc.numAttrs = 1;
  return cudaLaunchKernelEx(&lc, kernel, p);
}

template <int D, int GP>
cudaError_t launch_dg(const Params& p, cudaStream_t st) {
  const dim3 grid(static_cast<unsigned>(p.CPS), static_cast<unsigned>(p.B * p.Hkv * p.S));
  bool mma = false;
  if constexpr (D == 128 && GP == 4) mma = p.T >= mma16::STEP;
  if (mma) {  // both passes on the tensor cores, fed by TMA
    if constexpr (D == 128 && GP == 4) {
      if (!p.has_maps) return cudaErrorInvalidValue;
      static bool attr_set[64] = {};  // the dynamic shared-memory limit, raised once per device
      int dev = 0;
      cudaError_t e = cudaGetDevice(&dev);
      if (e != cudaSuccess) return e;
      if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
      if (!attr_set[dev]) {
        e = cudaFuncSetAttribute(q8_scores_mma_kernel<GP>, cudaFuncAttributeMaxDynamicSharedMemorySize, mma16::TSMEM);
        if (e != cudaSuccess) return e;
        e = cudaFuncSetAttribute(q8_pv_mma_kernel<GP, 0>, cudaFuncAttributeMaxDynamicSharedMemorySize, mma16::PV_SMEM);
        if (e != cudaSuccess) return e;
        e = cudaFuncSetAttribute(q8_pv_mma_kernel<GP, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize, mma16::PV_SMEM);
        if (e != cudaSuccess) return e;
        e = cudaFuncSetAttribute(q8_pv_mma_kernel<GP, 2>, cudaFuncAttributeMaxDynamicSharedMemorySize, mma16::PV_SMEM);
        if (e != cudaSuccess) return e;
        attr_set[dev] = true;
      }
      q8_scores_mma_kernel<GP><<<grid, NT, mma16::TSMEM, st>>>(p);
      if (p.art) {  // probe pass, the rule, the limited pass, in plain stream order (measured: letting
                    // these launches overlap made the chain 20% slower)
        cudaError_t e2 = launch_after(q8_pv_mma_kernel<GP, 1>, grid, NT, mma16::PV_SMEM, st, p, false);
        if (e2 != cudaSuccess) return e2;
        const dim3 rule_grid(static_cast<unsigned>(p.B * p.Hq * p.S));
        e2 = p.n_probe <= 16 ? launch_after(q8_rule_kernel<16>, rule_grid, RW * 32, 0, st, p, false)
                             : launch_after(q8_rule_kernel<32>, rule_grid, RW * 32, 0, st, p, false);
        if (e2 != cudaSuccess) return e2;
        e2 = launch_after(q8_pv_mma_kernel<GP, 2>, grid, NT, mma16::PV_SMEM, st, p, false);
        if (e2 != cudaSuccess) return e2;
      } else {
        cudaError_t e2 = launch_after(q8_pv_mma_kernel<GP, 0>, grid, NT, mma16::PV_SMEM, st, p);
        if (e2 != cudaSuccess) return e2;
      }
    }
  } else {
    if (p.art) return cudaErrorInvalidValue;  // the rule runs on the tensor-core passes only
    q8_scores_kernel<D, GP><<<grid, NT, 0, st>>>(p);
    cudaError_t e2 = launch_after(q8_pv_kernel<D, GP>, grid, NT, 0, st, p);
    if (e2 != cudaSuccess) return e2;
  }
  cudaError_t e3 = launch_after(q8_combine_kernel<D>, dim3(static_cast<unsigned>(p.B * p.Hq)), D, 0, st, p,
                                !p.art);
  if (e3 != cudaSuccess) return e3;
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_d(const Params& p, cudaStream_t st) {
  if (p.GP == 1) return launch_dg<D, 1>(p, st);
  if (p.GP == 2) return launch_dg<D, 2>(p, st);
  if (p.GP == 4) return launch_dg<D, 4>(p, st);
  return launch_dg<D, 8>(p, st);
}

// The passes on the tensor cores (d = 128, 3 or 4 heads per kv head) take K and V codes through
// tensor maps (tma_box_maps); the others do not.
inline bool uses_maps(const Dims& s) { return s.d == 128 && gp_of(s.Hq / s.Hkv) == 4 && s.T >= mma16::STEP; }

// Enqueue the three kernels.  ws: the caller's workspace; tiles_read_off / used_off: the common
// per-split counters inside it; base: where the common arrays end; tmk / tmv: the code maps when
// uses_maps(s), else NULL.
// The rule's settings, for ART on the two passes (n_probe lanes in [0, 128), n_probe <= 32).
struct Rule {
  int n_probe, patience;
  float eps_scale, eps_dir;
  const int32_t* lanes;  // host
};

inline cudaError_t launch(const Dims& s, const uint16_t* q, const int8_t* k, const uint16_t* ks, const int8_t* v,
                          const uint16_t* vs, const int32_t* seq_lens, float tau, float* o, int32_t* tiles,
                          uint8_t* ws, size_t tiles_read_off, size_t used_off, size_t base, const CUtensorMap* tmk,
                          const CUtensorMap* tmv, const Rule* rule, cudaStream_t st) {
  static int sms_of[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (sms_of[dev] == 0) {
    int v_ = 0;
    e = cudaDeviceGetAttribute(&v_, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    sms_of[dev] = v_;
  }
  const Layout2 ql = layout2(s, base);
  Params p;
  p.has_maps = tmk != nullptr && tmv != nullptr;
  if (p.has_maps) {
    p.tmK = *tmk;
    p.tmV = *tmv;
  }
  p.q = q;
  p.k = k;
  p.ks = ks;
  p.v = v;
  p.vs = vs;
  p.seq_lens = seq_lens;
  p.o = o;
  p.tiles = tiles;
  p.ws_status = reinterpret_cast<int32_t*>(ws);
  p.ws_tiles_read = reinterpret_cast<int32_t*>(ws + tiles_read_off);
  p.ws_used = reinterpret_cast<int32_t*>(ws + used_off);
  p.scores = reinterpret_cast<float*>(ws + ql.scores);
  p.tmax = reinterpret_cast<float*>(ws + ql.tmax);
  p.cmax = reinterpret_cast<float*>(ws + ql.cmax);
  p.part = reinterpret_cast<float*>(ws + ql.part);
  p.vskip = reinterpret_cast<int32_t*>(ws + ql.vskip);
  p.probe = reinterpret_cast<float*>(ws + ql.probe);
  p.stop = reinterpret_cast<int32_t*>(ws + ql.stop);
  p.art = rule != nullptr;
  p.n_probe = rule ? rule->n_probe : 0;
  p.patience = rule ? rule->patience : 1;
  p.eps_scale = rule ? rule->eps_scale : 0.f;
  p.eps_dir = rule ? rule->eps_dir : 0.f;
  for (int i = 0; i < 32; ++i) p.lanes[i] = (rule && i < rule->n_probe) ? rule->lanes[i] : 0;
  p.B = s.B;
  p.Hq = s.Hq;
  p.Hkv = s.Hkv;
  p.L_max = s.L_max;
  p.T = s.T;
  p.S = s.S;
  p.G = s.Hq / s.Hkv;
  p.GP = gp_of(p.G);
  p.CT = choose_ct(s, sms_of[dev]);  // >= the layout's chunk, so at most its chunk count
  p.CPS = ((ql.n_max + s.S - 1) / s.S + p.CT - 1) / p.CT;
  p.n_max = ql.n_max;
  p.qscale = static_cast<float>(1.4426950408889634 / sqrt(static_cast<double>(s.d)));
  p.tau = tau;
  return s.d == 64 ? launch_d<64>(p, st) : launch_d<128>(p, st);
}

}  // namespace q8two
}  // namespace artk
