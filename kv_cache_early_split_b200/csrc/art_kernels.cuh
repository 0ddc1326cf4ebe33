// art_kernels.cuh -- sm_100a kernels for single-token decode attention with ART.
//
// What is computed (web pages, cited by title and section):
//   "Resumen Tecnico: ART (Terminacion de la Atencion en Tiempo de Ejecucion)"
//   (gist.science, arXiv 2606.00024):
//     S2.1  tile-wise online softmax: running max m, denominator l, numerator acc;
//     S2.2  probe x^(t) = fixed lanes of O^(t) = acc/l; d_scale = | |x_t| - |x_{t-1}| |;
//           d_dir = 1 - cos(x_t, x_{t-1}); terminate when both are below thresholds;
//     S2.3  ... on `patience` consecutive tiles;
//     S2.4  tile 0 always processed first.
//   "La paradoja de la eficiencia: como omitir redefine la velocidad de los LLM"
//   (puntofijo.es), "La Elegancia de la Omision": q8 V rows with negligible
//   softmax weight are not dequantised.
//
// Work decomposition (B200 design, not the pages'):
//   * one thread-block CLUSTER of C CTAs owns one (batch, kv head, split) unit; the
//     G = Hq/Hkv query heads of the group share every K/V tile read (GQA packing);
//   * tiles are dealt round-robin: in round r, CTA `rank` processes tile
//     t0 + r*C + rank.  Each CTA streams its tiles with 1-D bulk async copies
//     (cp.async.bulk, 16-byte aligned, fully coalesced) into an NSTAGE-deep ring
//     of shared-memory stages completed by mbarriers;
//   * full attention: each CTA keeps its own online-softmax state; the C states
//     are merged through distributed shared memory at the end;
//   * ART: the rule is sequential per head, so each CTA computes the tile-LOCAL
//     state (m_t, l_t, acc_t) of its tile, publishes (m_t, l_t, acc_t[probe
//     lanes]) in its shared memory, and after one cluster barrier every CTA
//     reads all C publications and replays the rule for the round in tile order
//     (a prefix scan of the associative merge followed by the per-tile
//     metrics).  The replay is identical in every CTA, so they agree on the stop
//     tile without a second barrier.  Each CTA then merges its own tile into its
//     owned state only if the tile lies at or before its head's stop tile: the
//     union of owned states is exactly the sequential ART result;
//   * q8 V-skip needs the running max m' after each tile: tile maxima are
//     exchanged the same way before the PV step.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "art_device.cuh"

namespace artk {

constexpr int NT = 256;  // threads per CTA
constexpr int NW = NT / 32;
constexpr int PMAX = 32;  // max probe lanes
constexpr int CMAX = 16;  // max cluster size
constexpr int GMAX = 8;   // max query heads per kv head

enum : int { KV_F32 = 0, KV_BF16 = 1, KV_Q8 = 2 };
enum : int { MODE_FULL = 0, MODE_ART = 1, MODE_SKIP = 2, MODE_SKIP_ART = 3 };

struct Params {
  const void* q;
  const void* k;
  const void* v;
  const uint16_t* ks;  // q8 K scales (fp16 bits)
  const uint16_t* vs;  // q8 V scales
  const int32_t* seq_lens;
  float* o;
  int32_t* tiles;
  float* ws_partial;   // [B*Hq*S][2+d] (S > 1)
  int32_t* ws_used;    // [B*Hq*S] tiles consumed per split
  int32_t* ws_tiles_read;  // [B*Hkv*S]
  int32_t* ws_status;
  const int32_t* order;  // NULL or [B*Hkv][n_max] tile traversal sequences
  int n_max;             // ceil(L_max / T)
  // paged cache: NULL, or [B][max_pages] page of each page_size run of positions; K/V (and q8
  // scales) are then page pools [num_pages][Hkv][page_size][...]
  const int32_t* block_table;
  int page_size, max_pages, num_pages;
  int B, Hq, Hkv, L_max, T, S, G, C, nstage, n_probe, patience;
  float qscale;  // log2(e)/sqrt(d): scores live in the log2 domain
  float eps_scale, eps_dir, tau;
  int emask;  // bit e set when some probe lane sits at element e of a lane chunk
  int8_t lanes[PMAX];
};

template <int KIND, int D>
struct KvGeom {
  static constexpr int ESZ = KIND == KV_F32 ? 4 : (KIND == KV_BF16 ? 2 : 1);
  static constexpr int LB = KIND == KV_Q8 ? 8 : 16;  // bytes per lane chunk
  static constexpr int EPC = LB / ESZ;              // elements per lane chunk
  static constexpr int CH = D * ESZ / LB;           // lane chunks per row
  static constexpr int ROWB = D * ESZ;              // bytes per K/V row
  static constexpr int SCB = KIND == KV_Q8 ? (D / 32) * 2 : 0;  // scale bytes per row
  static constexpr int RPW = 32 / CH;               // rows per warp in the score step
  static constexpr int NSUB = NT / CH;              // position subsets in the PV step
  static_assert(CH <= 32 && 32 % CH == 0, "row must split evenly over a warp");
};

// Shared-memory layout (byte offsets), identical on host and device.
struct Layout {
  uint32_t k, v, ks, vs, stage;  // inside one stage
  uint32_t bar, sc, p, ppart, pub, pubm, rule_f, rule_i, rx, misc_f, misc_i, red, l2p, total;
};

__host__ __device__ inline uint32_t align_up(uint32_t x, uint32_t a) { return (x + a - 1) / a * a; }

// rule_f per head: [0]=m [1]=l [2]=|x_prev| [3]=m_run(skip) [4..4+PMAX)=acc probe [4+PMAX..)=x_prev
constexpr int RF_M = 0, RF_L = 1, RF_NRM = 2, RF_MRUN = 3, RF_A = 4, RF_XP = 4 + PMAX;
constexpr int RF_SIZE = 4 + 2 * PMAX;
// rule_i per head: run, stopped, used (tiles consumed in this split), stop index this round
constexpr int RI_RUN = 0, RI_STOPPED = 1, RI_USED = 2, RI_STOPREL = 3, RI_SIZE = 4;
// pub per slot per head: m, l, probe[PMAX]
constexpr int PUB_SIZE = 2 + PMAX;
// misc_f per head: mref (reference max of the current tile), l_t (its
// denominator), mown (running max of this CTA's own tiles, full attention)
constexpr int MF_MREF = 0, MF_LT = 1, MF_MOWN = 2, MF_SIZE = 4;

template <int KIND, int D, int GP>
__host__ __device__ inline Layout make_layout(int T, int nstage, int C) {
  using Gm = KvGeom<KIND, D>;
  Layout L;
  uint32_t o = 0;
  L.k = 0;
  o = T * Gm::ROWB;
  L.v = o;
  o += T * Gm::ROWB;
  L.ks = o;
  o = align_up(o + T * Gm::SCB, 16);
  L.vs = o;
  o = align_up(o + T * Gm::SCB, 16);
  L.stage = align_up(o, 128);
  o = L.stage * nstage;
  L.bar = o;
  o = align_up(o + 8 * nstage, 16);
  L.sc = o;  // scores [GP][T]
  o += 4 * GP * T;
  L.p = o;  // weights [T][GP]
  o += 4 * GP * T;
  L.ppart = o;  // probe partials [NW][GP][PMAX]
  o += 4 * NW * GP * PMAX;
  L.pub = o;  // [2][GP][PUB_SIZE]
  o += 4 * 2 * GP * PUB_SIZE;
  L.pubm = o;  // [2][GP]
  o += 4 * 2 * GP;
  L.rule_f = o;  // [GP][RF_SIZE]
  o += 4 * GP * RF_SIZE;
  L.rule_i = o;  // [GP][RI_SIZE]
  o += 4 * GP * RI_SIZE;
  L.rx = o;  // [GP][2][C][PMAX] scanned numerators and probes
  o += 4 * GP * 2 * C * PMAX;
  L.misc_f = o;  // [GP][MF_SIZE]
  o += 4 * GP * MF_SIZE;
  L.misc_i = o;  // [8]: all_stopped, tiles_read
  o += 4 * 8;
  L.red = o;  // final: [GP][D] numerators + [GP] m + [GP] l
  o += 4 * (GP * D + 2 * GP);
  L.l2p = o;  // lane -> probe index [D] int8
  o += D;
  L.total = align_up(o, 128);
  return L;
}

// ---------------------------------------------------------------- conversions
__device__ __forceinline__ void bf16x8_to_f32(const uint4 w, float (&f)[8]) {
  const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(u[i] << 16);
    f[2 * i + 1] = __uint_as_float(u[i] & 0xffff0000u);
  }
}

// int8 -> float by exponent-field insertion (IEEE-754 binary32): the float with
// bit pattern 0x4B000000 | u equals 2^23 + u for 0 <= u < 2^23.  A signed code
// c becomes u = c + 128 by flipping its top bit, so value = float - (2^23 + 128).
__device__ __forceinline__ void s8x8_to_f32(const uint2 w, float (&f)[8]) {
  const uint32_t u[2] = {w.x ^ 0x80808080u, w.y ^ 0x80808080u};
#pragma unroll
  for (int h = 0; h < 2; ++h) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t bits = __byte_perm(u[h], 0x4B000000u, 0x7540u | i);
      f[4 * h + i] = __uint_as_float(bits) - 8388736.0f;
    }
  }
}

// Load one lane chunk (EPC elements) of a K/V row from shared memory as floats.
template <int KIND>
__device__ __forceinline__ void load_chunk(const uint8_t* ptr, float (&f)[KIND == KV_F32 ? 4 : 8]) {
  if constexpr (KIND == KV_F32) {
    const float4 w = *reinterpret_cast<const float4*>(ptr);
    f[0] = w.x;
    f[1] = w.y;
    f[2] = w.z;
    f[3] = w.w;
  } else if constexpr (KIND == KV_BF16) {
    bf16x8_to_f32(*reinterpret_cast<const uint4*>(ptr), f);
  } else {
    s8x8_to_f32(*reinterpret_cast<const uint2*>(ptr), f);
  }
}

// Sum GP per-lane partials over groups of RL consecutive lanes (RL a power of
// two >= GP).  The first log2(GP) butterfly levels also split the head set in
// half (each lane sends the half it gives up), so afterwards every lane holds
// the group total of one head (`head`), held by RL/GP lanes of the group.
template <int GP, int RL>
__device__ __forceinline__ float transpose_reduce(float (&v)[GP], int lane, int& head) {
  head = 0;
#pragma unroll
  for (int h = GP / 2, off = RL / 2; h >= 1; h >>= 1, off >>= 1) {
    const bool upper = (lane & off) != 0;
#pragma unroll
    for (int i = 0; i < h; ++i) {
      const float send = upper ? v[i] : v[i + h];
      const float keep = upper ? v[i + h] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, off);
    }
    if (upper) head += h;
  }
#pragma unroll
  for (int off = RL / (2 * GP); off >= 1; off >>= 1) v[0] += __shfl_xor_sync(0xffffffffu, v[0], off);
  return v[0];
}

// acc[g][e] += p_j[g] * v_j[chunk pv_c, element e] over this thread's positions.
// Rows whose weights are all zero (q8 V-skip) are not dequantised.
template <int KIND, int D, int GP, bool SKIP>
__device__ __forceinline__ void pv_tile(float (&acc)[GP][KvGeom<KIND, D>::EPC], const uint8_t* vtile,
                                        const uint8_t* vscale, const float* s_p, int rows, int pv_r,
                                        int pv_c) {
  using Gm = KvGeom<KIND, D>;
  constexpr int EPC = Gm::EPC;
  for (int j = pv_r; j < rows; j += Gm::NSUB) {
    float w[GP];
    bool any = false;
#pragma unroll
    for (int g = 0; g < GP; ++g) {
      w[g] = s_p[j * GP + g];
      any |= (w[g] != 0.f);
    }
    if (SKIP && !any) continue;  // the V row is not dequantised at all
    float vf[EPC];
    load_chunk<KIND>(vtile + j * Gm::ROWB + pv_c * Gm::LB, vf);
    if constexpr (KIND == KV_Q8) {
      const float sc = __half2float(
          __ushort_as_half(reinterpret_cast<const uint16_t*>(vscale)[j * (D / 32) + (pv_c * EPC) / 32]));
#pragma unroll
      for (int g = 0; g < GP; ++g) w[g] *= sc;
    }
#pragma unroll
    for (int g = 0; g < GP; ++g)
#pragma unroll
      for (int e = 0; e < EPC; ++e) acc[g][e] = fmaf(w[g], vf[e], acc[g][e]);
  }
}

// ------------------------------------------------------------------ main kernel
template <int KIND, int D, int GP, int MODE>
__global__ void __launch_bounds__(NT, 1) art_decode_kernel(const __grid_constant__ Params p) {
  constexpr bool ART = (MODE == MODE_ART || MODE == MODE_SKIP_ART);
  constexpr bool SKIP = (MODE == MODE_SKIP || MODE == MODE_SKIP_ART);
  using Gm = KvGeom<KIND, D>;
  constexpr int EPC = Gm::EPC, CH = Gm::CH, ROWB = Gm::ROWB, SCB = Gm::SCB;
  constexpr int RPW = Gm::RPW, NSUB = Gm::NSUB;
  static_assert(GP <= CH, "heads must fit the score reduction");
  static_assert(GP <= NW, "one warp per head in the softmax step");

  extern __shared__ __align__(128) uint8_t smem[];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int C = p.C, T = p.T, G = p.G, P = p.n_probe;
  const int rank = (C > 1) ? static_cast<int>(cluster_ctarank()) : 0;
  const int unit = blockIdx.x / C;
  const int split = unit % p.S;
  const int bk = unit / p.S;
  const int kvh = bk % p.Hkv;
  const int b = bk / p.Hkv;
  const Layout Ly = make_layout<KIND, D, GP>(T, p.nstage, C);

  float* s_sc = reinterpret_cast<float*>(smem + Ly.sc);
  float* s_p = reinterpret_cast<float*>(smem + Ly.p);
  float* s_ppart = reinterpret_cast<float*>(smem + Ly.ppart);
  float* s_pub = reinterpret_cast<float*>(smem + Ly.pub);
  float* s_pubm = reinterpret_cast<float*>(smem + Ly.pubm);
  float* s_rf = reinterpret_cast<float*>(smem + Ly.rule_f);
  int32_t* s_ri = reinterpret_cast<int32_t*>(smem + Ly.rule_i);
  float* s_rx = reinterpret_cast<float*>(smem + Ly.rx);
  float* s_mf = reinterpret_cast<float*>(smem + Ly.misc_f);
  int32_t* s_mi = reinterpret_cast<int32_t*>(smem + Ly.misc_i);
  float* s_red = reinterpret_cast<float*>(smem + Ly.red);
  int8_t* s_l2p = reinterpret_cast<int8_t*>(smem + Ly.l2p);
  const uint32_t bar0 = smem_u32(smem + Ly.bar);

  // ---- sequence, split and rounds (identical in every CTA of the cluster)
  int L = p.seq_lens[b];
  const bool bad_len = (L < 1 || L > p.L_max);
  if (bad_len) L = 0;
  const int n_tiles = (L + T - 1) / T;
  const int t0 = static_cast<int>((static_cast<long long>(split) * n_tiles) / p.S);
  const int t1 = static_cast<int>((static_cast<long long>(split + 1) * n_tiles) / p.S);
  const int ns = t1 - t0;
  const int my_tiles = ns > rank ? (ns - rank + C - 1) / C : 0;
  const int rounds = (MODE == MODE_FULL) ? my_tiles : (ns + C - 1) / C;
  // Tile at position q of this split's traversal sequence (the natural order without one).  An
  // entry outside the split is replaced by the natural tile (the producer flags it).
  const int32_t* ord_seq = p.order ? p.order + (static_cast<long long>(b) * p.Hkv + kvh) * p.n_max : nullptr;
  auto phys_of = [&](int q) -> int {
    if (!ord_seq) return q;
    const int e = __ldg(ord_seq + q);
    return (e >= t0 && e < t1) ? e : q;
  };

  // ---- shared-memory initialisation
  if (tid == 0) {
    for (int i = 0; i < p.nstage; ++i) mbar_init(bar0 + 8 * i, 1);
    fence_mbar_init();
    if (bad_len && rank == 0) atomicOr(p.ws_status, kStatusSeqLen);
  }
  for (int i = tid; i < D; i += NT) s_l2p[i] = -1;
  for (int i = tid; i < GP * T; i += NT) s_p[i] = 0.f;
  for (int i = tid; i < GP * D + 2 * GP; i += NT) s_red[i] = 0.f;
  if (tid < GP) {
    float* rf = s_rf + tid * RF_SIZE;
    rf[RF_M] = -INFINITY;
    rf[RF_L] = 0.f;
    rf[RF_NRM] = 0.f;
    rf[RF_MRUN] = -INFINITY;
    for (int i = 0; i < PMAX; ++i) rf[RF_A + i] = rf[RF_XP + i] = 0.f;
    int32_t* ri = s_ri + tid * RI_SIZE;
    ri[RI_RUN] = 0;
    ri[RI_STOPPED] = (tid < G) ? 0 : 1;
    ri[RI_USED] = ns;
    ri[RI_STOPREL] = -1;
  }
  if (tid < GP) s_mf[tid * MF_SIZE + MF_MOWN] = -INFINITY;
  if (tid == 0) s_mi[0] = 0;
  __syncthreads();
  if (tid < P) s_l2p[p.lanes[tid]] = static_cast<int8_t>(tid);
  fence_proxy_async_smem();
  __syncthreads();

  // ---- producer: issue the bulk copies of this CTA's tile with ordinal `ord`
  const uint8_t* gk = static_cast<const uint8_t*>(p.k);
  const uint8_t* gv = static_cast<const uint8_t*>(p.v);
  const long long slab_row0 = (static_cast<long long>(b) * p.Hkv + kvh) * p.L_max;
  auto issue = [&](int ord) -> bool {
    if (ord >= my_tiles) return false;
    const int tq = t0 + ord * C + rank;
    const int t = phys_of(tq);
    if (ord_seq && t != __ldg(ord_seq + tq)) atomicOr(p.ws_status, kStatusOrder);
    const int rows = min(T, L - t * T);
    const int stage = ord % p.nstage;
    const uint32_t bar = bar0 + 8 * stage;
    uint8_t* st = smem + stage * Ly.stage;
    long long row = slab_row0 + static_cast<long long>(t) * T;
    if (p.block_table) {  // the tile lies inside one page (page_size is a multiple of T)
      const int pos0 = t * T;
      int pg = __ldg(p.block_table + static_cast<long long>(b) * p.max_pages + pos0 / p.page_size);
      if (pg < 0 || pg >= p.num_pages) {
        atomicOr(p.ws_status, kStatusPage);
        pg = 0;
      }
      row = (static_cast<long long>(pg) * p.Hkv + kvh) * p.page_size + pos0 % p.page_size;
    }
    ART_DCHECK(t >= t0 && t < t1 && rows >= 1 && rows <= T, p.ws_status);
    ART_DCHECK(p.block_table || t * T + rows <= p.L_max, p.ws_status);
    ART_DCHECK(stage < p.nstage, p.ws_status);
    uint32_t bytes = 2u * rows * ROWB;
    uint32_t sbytes = 0;
    if constexpr (KIND == KV_Q8) {
      const int unit_rows = 16 / SCB;  // rows per 16-byte granule of scales
      sbytes = static_cast<uint32_t>((rows + unit_rows - 1) / unit_rows * unit_rows) * SCB;
      bytes += 2u * sbytes;
    }
    mbar_arrive_expect_tx(bar, bytes);
    bulk_g2s(smem_u32(st + Ly.k), gk + row * ROWB, rows * ROWB, bar);
    bulk_g2s(smem_u32(st + Ly.v), gv + row * ROWB, rows * ROWB, bar);
    if constexpr (KIND == KV_Q8) {
      bulk_g2s(smem_u32(st + Ly.ks), reinterpret_cast<const uint8_t*>(p.ks) + row * SCB, sbytes, bar);
      bulk_g2s(smem_u32(st + Ly.vs), reinterpret_cast<const uint8_t*>(p.vs) + row * SCB, sbytes, bar);
    }
    return true;
  };
  int issued = 0;  // meaningful in thread 0 only
  if (tid == 0) {
    while (issued < p.nstage && issue(issued)) ++issued;
  }

  // ---- query registers for the score step: lane chunk sc_c of every head
  const int sc_c = lane % CH;
  const int sc_rs = lane / CH;
  float qr[GP][EPC];
#pragma unroll
  for (int g = 0; g < GP; ++g) {
    if (g < G) {
      const long long qrow = static_cast<long long>(b) * p.Hq + kvh * G + g;
      if constexpr (KIND == KV_F32) {
        const float4 w = *reinterpret_cast<const float4*>(static_cast<const float*>(p.q) + qrow * D + sc_c * EPC);
        qr[g][0] = w.x * p.qscale;
        qr[g][1] = w.y * p.qscale;
        qr[g][2] = w.z * p.qscale;
        qr[g][3] = w.w * p.qscale;
      } else {
        float f[8];
        bf16x8_to_f32(*reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(p.q) + qrow * D + sc_c * 8), f);
#pragma unroll
        for (int e = 0; e < 8; ++e) qr[g][e] = f[e] * p.qscale;
      }
    } else {
#pragma unroll
      for (int e = 0; e < EPC; ++e) qr[g][e] = 0.f;
    }
  }

  // ---- PV mapping and owned state
  const int pv_c = tid % CH;
  const int pv_r = tid / CH;
  float acc_o[GP][EPC];
  float acc_t[GP][EPC];  // tile-local numerator (ART modes only)
  float m_own[GP], l_own[GP];
#pragma unroll
  for (int g = 0; g < GP; ++g) {
    m_own[g] = -INFINITY;
    l_own[g] = 0.f;
#pragma unroll
    for (int e = 0; e < EPC; ++e) acc_o[g][e] = 0.f;
  }

  int waited = 0;
  bool all_stopped = false;
  for (int r = 0; r < rounds; ++r) {
    const int t = t0 + r * C + rank;
    const bool have = (MODE == MODE_FULL) ? true : (t < t1);
    const int rows = have ? min(T, L - phys_of(t) * T) : 0;
    const int stage = r % p.nstage;
    const int slot = r & 1;
    const uint8_t* st = smem + stage * Ly.stage;
    if (have) {
      mbar_wait_bounded(bar0 + 8 * stage, (r / p.nstage) & 1, p.ws_status);
      ++waited;
    }

    // -------- scores: s[g][j] = (q_g . k_j) * log2(e)/sqrt(d)
    if (have) {
      for (int j0 = 0; j0 < T; j0 += NW * RPW) {
        const int j = j0 + warp * RPW + sc_rs;
        float part[GP];
#pragma unroll
        for (int g = 0; g < GP; ++g) part[g] = 0.f;
        if (j < rows) {
          float kf[EPC];
          load_chunk<KIND>(st + Ly.k + j * ROWB + sc_c * Gm::LB, kf);
          float sc = 1.f;
          if constexpr (KIND == KV_Q8)
            sc = __half2float(__ushort_as_half(
                reinterpret_cast<const uint16_t*>(st + Ly.ks)[j * (D / 32) + (sc_c * EPC) / 32]));
#pragma unroll
          for (int g = 0; g < GP; ++g) {
            float a = 0.f;
#pragma unroll
            for (int e = 0; e < EPC; ++e) a = fmaf(qr[g][e], kf[e], a);
            part[g] = a * sc;
          }
        }
        int head;
        const float tot = transpose_reduce<GP, CH>(part, lane, head);
        if (j < rows && head < G && (lane % (CH / GP)) == 0) s_sc[head * T + j] = tot;
      }
    }
    __syncthreads();

    // -------- reference max per head
    if constexpr (SKIP) {
      // exchange tile maxima so that every CTA knows the running max m' after its tile
      if (warp < G) {
        float mx = -INFINITY;
        for (int j = lane; j < rows; j += 32) mx = fmaxf(mx, s_sc[warp * T + j]);
        mx = warp_max(mx);
        if (lane == 0) s_pubm[slot * GP + warp] = mx;
      }
      if (C > 1) cluster_sync_all(); else __syncthreads();
      if (warp < G) {
        const int nv = min(C, t1 - (t0 + r * C));
        float v = -INFINITY, vall = -INFINITY;
        if (lane < nv) {
          const float x = (C > 1) ? ld_dsmem_f32(map_to_rank(smem_u32(s_pubm + slot * GP + warp), lane))
                                  : s_pubm[slot * GP + warp];
          vall = x;
          if (lane <= rank) v = x;
        }
        v = warp_max(v);
        vall = warp_max(vall);
        float* rf = s_rf + warp * RF_SIZE;
        if (lane == 0) {
          s_mf[warp * MF_SIZE + MF_MREF] = fmaxf(rf[RF_MRUN], v);
        }
        __syncwarp();
        if (lane == 0) rf[RF_MRUN] = fmaxf(rf[RF_MRUN], vall);
      }
      __syncthreads();
    }

    // -------- weights p_j = 2^(s_j - mref), tile denominator
    if (warp < G && have) {
      const int g = warp;
      float mref;
      if constexpr (SKIP) {
        mref = s_mf[g * MF_SIZE + MF_MREF];
      } else {
        float mx = -INFINITY;
        for (int j = lane; j < rows; j += 32) mx = fmaxf(mx, s_sc[g * T + j]);
        mx = warp_max(mx);
        mref = ART ? mx : fmaxf(s_mf[g * MF_SIZE + MF_MOWN], mx);
      }
      float lsum = 0.f;
      for (int j = lane; j < T; j += 32) {
        float pj = 0.f;
        if (j < rows) {
          pj = exp2f(s_sc[g * T + j] - mref);
          lsum += pj;
          if (SKIP && pj < p.tau) pj = 0.f;  // left out of the numerator only
        }
        s_p[j * GP + g] = pj;
      }
      lsum = warp_sum(lsum);
      if (lane == 0) {
        s_mf[g * MF_SIZE + MF_MREF] = mref;
        s_mf[g * MF_SIZE + MF_LT] = lsum;
        s_mf[g * MF_SIZE + MF_MOWN] = fmaxf(s_mf[g * MF_SIZE + MF_MOWN], mref);
      }
    }
    __syncthreads();

    // -------- PV: acc[g][e] += p_j[g] * v_j[chunk e]
    if (have) {
      if constexpr (ART) {
#pragma unroll
        for (int g = 0; g < GP; ++g)
#pragma unroll
          for (int e = 0; e < EPC; ++e) acc_t[g][e] = 0.f;
        pv_tile<KIND, D, GP, SKIP>(acc_t, st + Ly.v, st + Ly.vs, s_p, rows, pv_r, pv_c);
      } else {
#pragma unroll
        for (int g = 0; g < GP; ++g) {
          if (g < G) {
            const float mref = s_mf[g * MF_SIZE + MF_MREF];
            const float alpha = rescale(m_own[g], mref);
            m_own[g] = mref;
            l_own[g] = alpha * l_own[g] + s_mf[g * MF_SIZE + MF_LT];
#pragma unroll
            for (int e = 0; e < EPC; ++e) acc_o[g][e] *= alpha;
          }
        }
        pv_tile<KIND, D, GP, SKIP>(acc_o, st + Ly.v, st + Ly.vs, s_p, rows, pv_r, pv_c);
      }
    }

    if constexpr (ART) {
      // -------- probe lanes of the tile-local numerator -> publication slot
      if (have) {
#pragma unroll
        for (int e = 0; e < EPC; ++e) {
          if ((p.emask >> e) & 1) {  // uniform over the CTA
            const int pidx = s_l2p[pv_c * EPC + e];
#pragma unroll
            for (int g = 0; g < GP; ++g) {
              float x = acc_t[g][e];
#pragma unroll
              for (int off = CH; off < 32; off <<= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
              if (lane < CH && pidx >= 0 && g < G) s_ppart[(warp * GP + g) * PMAX + pidx] = x;
            }
          }
        }
      }
      __syncthreads();
      for (int i = tid; i < GP * PUB_SIZE; i += NT) {
        const int g = i / PUB_SIZE, k = i % PUB_SIZE;
        float val = 0.f;
        if (have && g < G) {
          if (k == 0) {
            val = s_mf[g * MF_SIZE + MF_MREF];
          } else if (k == 1) {
            val = s_mf[g * MF_SIZE + MF_LT];
          } else if (k - 2 < P) {
            for (int w = 0; w < NW; ++w) val += s_ppart[(w * GP + g) * PMAX + (k - 2)];
          }
        } else if (k == 0) {
          val = -INFINITY;
        }
        s_pub[(slot * GP + g) * PUB_SIZE + k] = val;
      }
      if (C > 1) cluster_sync_all(); else __syncthreads();

      // -------- replay the rule for the C tiles of this round, one warp per head
      if (warp < G) {
        const int g = warp;
        float* rf = s_rf + g * RF_SIZE;
        int32_t* ri = s_ri + g * RI_SIZE;
        if (ri[RI_STOPPED]) {
          if (lane == 0) ri[RI_STOPREL] = -2;  // stopped in an earlier round
        } else {
          const int round_start = t0 + r * C;
          const int nv = min(C, t1 - round_start);
          const int c = lane;
          const uint32_t my_pub = smem_u32(s_pub + (slot * GP + g) * PUB_SIZE);
          const uint32_t src = (C > 1 && c < nv) ? map_to_rank(my_pub, c) : my_pub;
          float mc = -INFINITY, lc = 0.f;
          if (c < nv) {
            mc = (C > 1) ? ld_dsmem_f32(src) : s_pub[(slot * GP + g) * PUB_SIZE];
            lc = (C > 1) ? ld_dsmem_f32(src + 4) : s_pub[(slot * GP + g) * PUB_SIZE + 1];
          }
          // inclusive scan of (m, l) over the round's tiles; keep per-level coefficients
          float cself[4], cother[4];
#pragma unroll
          for (int lv = 0; lv < 4; ++lv) {
            const int off = 1 << lv;
            cself[lv] = 1.f;
            cother[lv] = 0.f;
            if (off < C) {
              const float mo = __shfl_up_sync(0xffffffffu, mc, off);
              const float lo = __shfl_up_sync(0xffffffffu, lc, off);
              if (c >= off) {
                const float M = fmaxf(mc, mo);
                const float a = rescale(mc, M), bo = rescale(mo, M);
                lc = a * lc + bo * lo;
                mc = M;
                cself[lv] = a;
                cother[lv] = bo;
              }
            }
          }
          // prepend the state carried from earlier rounds
          const float mR = rf[RF_M], lR = rf[RF_L];
          const float Mf = fmaxf(mR, mc);
          const float aR = rescale(mR, Mf), aS = rescale(mc, Mf);
          const float lf = aR * lR + aS * lc;
          const float inv_l = 1.f / lf;
          float* rxa = s_rx + (g * 2 + 0) * C * PMAX;
          float* rxx = s_rx + (g * 2 + 1) * C * PMAX;
          float nrm2 = 0.f;
          for (int i = 0; i < P; ++i) {
            float a = 0.f;
            if (c < nv) a = (C > 1) ? ld_dsmem_f32(src + 8 + 4 * i) : s_pub[(slot * GP + g) * PUB_SIZE + 2 + i];
#pragma unroll
            for (int lv = 0; lv < 4; ++lv) {
              const int off = 1 << lv;
              if (off < C) {
                const float ao = __shfl_up_sync(0xffffffffu, a, off);
                a = cself[lv] * a + cother[lv] * ao;
              }
            }
            a = aR * rf[RF_A + i] + aS * a;
            const float x = a * inv_l;
            if (c < C) {
              rxa[c * PMAX + i] = a;
              rxx[c * PMAX + i] = x;
            }
            nrm2 = fmaf(x, x, nrm2);
          }
          const float nrm = sqrtf(nrm2);
          float nrm_prev = __shfl_up_sync(0xffffffffu, nrm, 1);
          if (c == 0) nrm_prev = rf[RF_NRM];
          __syncwarp();
          float dd2 = 0.f;
          if (c < nv && nrm > 0.f && nrm_prev > 0.f) {
            const float in = 1.f / nrm, ip = 1.f / nrm_prev;
            for (int i = 0; i < P; ++i) {
              const float xp = (c > 0) ? rxx[(c - 1) * PMAX + i] : rf[RF_XP + i];
              const float dlt = rxx[c * PMAX + i] * in - xp * ip;
              dd2 = fmaf(dlt, dlt, dd2);
            }
          }
          const float d_scale = fabsf(nrm - nrm_prev);
          float d_dir;
          if (nrm == 0.f && nrm_prev == 0.f)
            d_dir = 0.f;
          else if (nrm == 0.f || nrm_prev == 0.f)
            d_dir = 1.f;
          else
            d_dir = 0.5f * dd2;
          const bool hold = (c < nv) && (d_scale < p.eps_scale) && (d_dir < p.eps_dir);
          const uint32_t mask = __ballot_sync(0xffffffffu, hold);
          int run = ri[RI_RUN];
          int stop = -1;
          for (int cc = 0; cc < nv; ++cc) {
            run = ((mask >> cc) & 1u) ? run + 1 : 0;
            if (run >= p.patience) {
              stop = cc;
              break;
            }
          }
          const int srcl = (stop >= 0) ? stop : nv - 1;
          const float m_out = __shfl_sync(0xffffffffu, Mf, srcl);
          const float l_out = __shfl_sync(0xffffffffu, lf, srcl);
          const float nrm_out = __shfl_sync(0xffffffffu, nrm, srcl);
          __syncwarp();
          if (lane < P) {
            rf[RF_A + lane] = rxa[srcl * PMAX + lane];
            rf[RF_XP + lane] = rxx[srcl * PMAX + lane];
          }
          if (lane == 0) {
            rf[RF_M] = m_out;
            rf[RF_L] = l_out;
            rf[RF_NRM] = nrm_out;
            ri[RI_RUN] = run;
            ri[RI_STOPREL] = stop;
            if (stop >= 0) {
              ri[RI_STOPPED] = 1;
              ri[RI_USED] = round_start + stop + 1 - t0;
            }
          }
        }
      }
      __syncthreads();

      // -------- merge this CTA's tile into its owned state where the rule allows
      all_stopped = true;
#pragma unroll
      for (int g = 0; g < GP; ++g) {
        if (g < G) {
          const int stop = s_ri[g * RI_SIZE + RI_STOPREL];
          all_stopped &= (s_ri[g * RI_SIZE + RI_STOPPED] != 0);
          const bool take = have && stop != -2 && (stop < 0 || rank <= stop);
          if (take) {
            const float mt = s_mf[g * MF_SIZE + MF_MREF], lt = s_mf[g * MF_SIZE + MF_LT];
            const float M = fmaxf(m_own[g], mt);
            const float a = rescale(m_own[g], M), bt = rescale(mt, M);
            m_own[g] = M;
            l_own[g] = a * l_own[g] + bt * lt;
#pragma unroll
            for (int e = 0; e < EPC; ++e) acc_o[g][e] = a * acc_o[g][e] + bt * acc_t[g][e];
          }
        }
      }
    }

    __syncthreads();  // the stage buffer and the per-tile scratch are free again
    if (tid == 0 && !all_stopped && issued == r + p.nstage) {
      if (issue(issued)) ++issued;
    }
    if (ART && all_stopped) break;
  }

  // ---- drain copies that were prefetched past the stop tile
  if (tid == 0) {
    for (int ord = waited; ord < issued; ++ord)
      mbar_wait_bounded(bar0 + 8 * (ord % p.nstage), (ord / p.nstage) & 1, p.ws_status);
  }

  // ---- reduce the owned numerators over the position subsets of this CTA
  // (warp shuffles, then warps add in a fixed order: the result is deterministic)
#pragma unroll
  for (int g = 0; g < GP; ++g) {
#pragma unroll
    for (int e = 0; e < EPC; ++e) {
      float x = acc_o[g][e];
#pragma unroll
      for (int off = CH; off < 32; off <<= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
      acc_o[g][e] = x;
    }
  }
  for (int w = 0; w < NW; ++w) {
    if (warp == w && lane < CH) {
#pragma unroll
      for (int g = 0; g < GP; ++g)
#pragma unroll
        for (int e = 0; e < EPC; ++e)
          if (g < G) s_red[g * D + pv_c * EPC + e] += acc_o[g][e];
    }
    __syncthreads();
  }
  if (tid == 0) {
#pragma unroll
    for (int g = 0; g < GP; ++g) {
      s_red[GP * D + g] = m_own[g];
      s_red[GP * D + GP + g] = l_own[g];
    }
    s_mi[1] = issued;
  }
  if (C > 1) cluster_sync_all(); else __syncthreads();

  // ---- rank 0 merges the C owned states and writes the result
  if (rank == 0) {
    const uint32_t red_base = smem_u32(s_red);
    for (int idx = tid; idx < G * D; idx += NT) {
      const int g = idx / D, dd = idx % D;
      float M = -INFINITY;
      for (int c = 0; c < C; ++c) {
        const float mc = (C > 1) ? ld_dsmem_f32(map_to_rank(red_base + 4 * (GP * D + g), c)) : s_red[GP * D + g];
        M = fmaxf(M, mc);
      }
      float den = 0.f, num = 0.f;
      for (int c = 0; c < C; ++c) {
        float mc, lc, ac;
        if (C > 1) {
          mc = ld_dsmem_f32(map_to_rank(red_base + 4 * (GP * D + g), c));
          lc = ld_dsmem_f32(map_to_rank(red_base + 4 * (GP * D + GP + g), c));
          ac = ld_dsmem_f32(map_to_rank(red_base + 4 * (g * D + dd), c));
        } else {
          mc = s_red[GP * D + g];
          lc = s_red[GP * D + GP + g];
          ac = s_red[g * D + dd];
        }
        if (mc == -INFINITY) continue;
        const float w = exp2f(mc - M);
        den += w * lc;
        num += w * ac;
      }
      const long long hq = static_cast<long long>(b) * p.Hq + kvh * G + g;
      if (p.S == 1) {
        p.o[hq * D + dd] = bad_len ? __int_as_float(0x7fc00000) : num / den;
      } else {
        float* part = p.ws_partial + (hq * p.S + split) * (D + 2);
        if (dd == 0) {
          part[0] = M;
          part[1] = den;
        }
        part[2 + dd] = num;
      }
    }
    if (tid < G) {
      const long long hq = static_cast<long long>(b) * p.Hq + kvh * G + tid;
      const int used = bad_len ? 0 : (ART ? s_ri[tid * RI_SIZE + RI_USED] : ns);
      p.ws_used[hq * p.S + split] = used;
      if (p.S == 1 && p.tiles) p.tiles[hq] = used;
    }
    if (tid == 0) {
      int total = 0;
      const uint32_t a = smem_u32(s_mi + 1);
      for (int c = 0; c < C; ++c) total += (C > 1) ? ld_dsmem_s32(map_to_rank(a, c)) : s_mi[1];
      p.ws_tiles_read[(static_cast<long long>(b) * p.Hkv + kvh) * p.S + split] = total;
    }
  }
  if (C > 1) cluster_sync_all();  // peers stay resident until rank 0 has read them
}

// ------------------------------------------------------------------ split combine
// One warp per (batch, query head): O = sum_s 2^(m_s-M) acc_s / sum_s 2^(m_s-M) l_s.
// With internal splits of one caller split (full attention only), also the caller's per-split
// counters: used_out[hq] = tiles consumed, tread_out[b*Hkv + kvh] = the sum of tread_in over the splits.
template <int D>
__global__ void __launch_bounds__(256) art_combine_kernel(const float* __restrict__ part,
                                                          const int32_t* __restrict__ used,
                                                          float* __restrict__ o,
                                                          int32_t* __restrict__ tiles, int n_heads,
                                                          int S, int32_t* __restrict__ used_out = nullptr,
                                                          const int32_t* __restrict__ tread_in = nullptr,
                                                          int32_t* __restrict__ tread_out = nullptr,
                                                          int G = 1) {
  const int hq = blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (hq >= n_heads) return;
  const float* ph = part + static_cast<long long>(hq) * S * (D + 2);
  float M = -INFINITY;
  for (int s = 0; s < S; ++s) M = fmaxf(M, ph[s * (D + 2)]);
  float den = 0.f;
  float num[D / 32];
#pragma unroll
  for (int i = 0; i < D / 32; ++i) num[i] = 0.f;
  int tsum = 0;
  for (int s = 0; s < S; ++s) {
    const float ms = ph[s * (D + 2)];
    tsum += used[static_cast<long long>(hq) * S + s];
    if (ms == -INFINITY) continue;
    const float w = exp2f(ms - M);
    den += w * ph[s * (D + 2) + 1];
#pragma unroll
    for (int i = 0; i < D / 32; ++i) num[i] += w * ph[s * (D + 2) + 2 + lane + 32 * i];
  }
#pragma unroll
  for (int i = 0; i < D / 32; ++i) o[static_cast<long long>(hq) * D + lane + 32 * i] = num[i] / den;
  if (lane == 0 && tiles) tiles[hq] = tsum;
  if (lane == 0 && used_out) used_out[hq] = tsum;
  if (lane == 0 && tread_out && hq % G == 0) {
    const int bk = hq / G;  // batch * Hkv + kv head
    int t = 0;
    for (int s2 = 0; s2 < S; ++s2) t += tread_in[static_cast<long long>(bk) * S + s2];
    tread_out[bk] = t;
  }
}

}  // namespace artk
