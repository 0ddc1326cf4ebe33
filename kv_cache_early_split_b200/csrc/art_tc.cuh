// art_tc.cuh -- tensor-core (tcgen05 + TMA) decode kernel for bf16 K/V, d = 128,
// tile 64 or 128, up to 8 query heads per kv head; full attention and ART.
//
// Same computation as art_decode_kernel (web pages, cited by title and section):
//   "Resumen Tecnico: ART" (gist.science, arXiv 2606.00024) S2.1 tile-wise online
//   softmax; S2.2 probe of the normalised partial output, d_scale / d_direction,
//   both below threshold; S2.3 patience; S2.4 tile 0 first.
//
// The GQA group's G query heads against a K/V block of 128 positions are two
// real dense contractions, so they run on the 5th-generation tensor cores:
//   S^T[128 pos x 16]  = K_blk[128 x 128 d] . Q^T      (A: K, K-major, 128-byte swizzle)
//   O_t^T[128 d x 16]  = V_t^T[128 d x T]  . P_t^T      (A: V, MN-major, 128-byte swizzle)
// with accumulators in tensor memory.  P is split into bf16 hi + lo parts
// (columns 0..7 and 8..15) so that the weights keep ~16 bits of precision.
// Full attention treats a whole 128-position block as one tile (the tile size
// has no effect on its result); ART keeps the caller's tiles.
//
// Warp roles (384 threads, one CTA per SM):
//   warp 0       TMA producer: K/V blocks (4 tiled 3-D TMA loads, 64 KiB) into a 3-deep ring
//   warp 1       MMA issuer (one lane) and tensor-memory owner
//   warp 2       ART controller: per round, reads all CTAs' publications through
//                distributed shared memory and replays the rule in tile order.
//   warp 3       second ART controller when the replay of a round needs two or more
//                passes over the heads (each warp takes half of them); idle otherwise
//   warps 4..11  two epilogue warpgroups (thread = TMEM lane); warpgroup wg takes the
//                CTA's own blocks wg, wg + 2, ...: scores -> per-tile max / weights ->
//                P^T in smem; O readback (thread = d row) -> online merge in registers;
//                ART publication.  While one warpgroup waits on a barrier or the tensor
//                cores, the other works on the next block.
// Blocks are dealt round-robin over the cluster exactly as in art_decode_kernel; the
// CTA's own block r belongs to ART round r.
//
// ART exchange without back-pressure barriers: rounds cycle through NSLOT publication
// slots and a warpgroup merges round r - LAG after publishing round r (LAG = NWG = 2:
// its own previous round).  Before a warpgroup publishes round x it has merged round
// x-NWG-LAG, so its controller has decided that round, so every CTA had published it,
// so every CTA had merged round x-2*NWG-2*LAG, so every controller had decided -- and
// finished reading -- every round up to x-2*NWG-2*LAG = x-NSLOT: the slot is free.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "art_device.cuh"
#include "art_kernels.cuh"

namespace artk {
namespace tc {

constexpr int BLK = 128;  // positions per block (= MMA M for the scores)
constexpr int D = 128;
constexpr int NSTG = 3;
constexpr int NWG = 2;  // epilogue warpgroups, taking alternate blocks
constexpr int NWARP = 4 + 4 * NWG;
constexpr int NTHR = NWARP * 32;
constexpr int KT_MAX = 2;  // ART tiles per block (tile 64)
constexpr int STAGE_BYTES = 4 * 16384;
constexpr uint32_t TMEM_COLS = 128;
constexpr int WARP_TMA = 0, WARP_MMA = 1, WARP_CTL = 2, WARP_EPI0 = 4;
constexpr int BAR_EPI = 1;  // named barriers BAR_EPI + wg: the 128 threads of epilogue warpgroup wg
constexpr int BAR_CTL = 3;  // named barrier of the two controller warps
constexpr int LAG = 2;      // a round is merged LAG rounds after it was published (LAG % NWG == 0)
constexpr int NSLOT = 2 * NWG + 2 * LAG;
static_assert(LAG % NWG == 0, "a warpgroup merges its own rounds");

struct TcParams {
  CUtensorMap tmK;  // 64-byte aligned (first members); box 64 d x 128 positions
  CUtensorMap tmV;
  CUtensorMap tmK64;  // box 64 d x 64 positions (ordered traversal with tile 64)
  CUtensorMap tmV64;
  const int32_t* order;  // NULL or [B*Hkv][n_max] tile traversal sequences (ART only)
  int n_max;
  // paged cache: NULL, or [B][max_pages] page of each page_size run of positions; tmK64/tmV64 then
  // map the page pools [num_pages*Hkv][page_size][128] (page_size a multiple of 64)
  const int32_t* block_table;
  int page_size, max_pages, num_pages;
  const uint16_t* q;
  const int32_t* seq_lens;
  float* o;
  int32_t* tiles;
  float* ws_partial;
  int32_t* ws_used;
  int32_t* ws_tiles_read;
  int32_t* ws_status;
  int B, Hq, Hkv, L_max, T, S, G, C, n_probe, patience;
  int spec_tiles;  // ART: bound on the tiles read past the safe point (0: none)
  float qscale, eps_scale, eps_dir;
  float tau;      // q8: V-skip threshold (rows with weight below tau leave the numerator); 0 = off
  float log2tau;  // q8: log2(tau) (scores live in the log2 domain)
  int8_t lanes[PMAX];
};

// ---- q8 cache (int8 codes in 32-element blocks along d, one fp16 scale per block)
// A raw stage holds one 128-position block as loaded: K codes, V codes (128 B per row), then the
// K and V scales (8 B per row).  The converter warpgroup turns codes into f16 MMA operands.
constexpr int Q8_NRAW = 2;
constexpr uint32_t Q8_RAW_K = 0, Q8_RAW_V = 16384, Q8_RAW_KS = 32768, Q8_RAW_VS = 33792, Q8_RAW_BYTES = 34816;
constexpr uint32_t Q8_SCL_BYTES = 2048;  // a scale-ring entry: K scales [128][4], then V scales [128][4]
constexpr int Q8_NP = 32;                // P' columns: 4 scale blocks x (4 hi + 4 lo) for up to 4 heads
// maxima exchange of the V skip, per round: this CTA's caller-tile maxima [KT_MAX][GMAX], then its
// block maxima [GMAX]
constexpr uint32_t MXS_FLOATS = KT_MAX * GMAX + GMAX;

// ---- shared-memory map (byte offsets from a 1024-aligned base), per kind of KV cache
//   bf16: NSTG stages of K and V exactly as TMA loads them (they are the MMA operands themselves);
//   q8:   Q8_NRAW raw stages, one K operand and two V operands in f16 written by the converter
//         warpgroup, a two-entry ring of the blocks' scales for the epilogue, and the maxima
//         exchange areas of the V skip.
template <bool Q8>
struct Lay {
  static constexpr int NWARP = Q8 ? 16 : 12;  // q8: + the converter warpgroup (warps 12..15)
  static constexpr int NTHR = NWARP * 32;
  static constexpr uint32_t TMEM_COLS = Q8 ? 256 : 128;
  static constexpr uint32_t STAGE = 0;
  static constexpr uint32_t KCV = Q8_NRAW * Q8_RAW_BYTES;
  static constexpr uint32_t VCV = KCV + 32768;
  static constexpr uint32_t SCL = VCV + 2 * 32768;
  static constexpr uint32_t Q = Q8 ? SCL + 2 * Q8_SCL_BYTES : NSTG * STAGE_BYTES;  // 2 halves x 2 KiB
  static constexpr uint32_t PBUF = Q8 ? 128 * Q8_NP * 2 : 4096;  // one P buffer
  static constexpr uint32_t P = Q + 4096;
  static constexpr uint32_t BAR = P + 2 * PBUF;                                 // mbarriers
  static constexpr uint32_t WRED = BAR + 512;                                   // [2][4][GMAX] per-warp maxima
  static constexpr uint32_t WSUM = WRED + 4 * 2 * 4 * GMAX;                     // [2][4][GMAX] per-warp sums
  static constexpr uint32_t TST = WSUM + 4 * 2 * 4 * GMAX;                      // [NSLOT][KT][GMAX][2] tile (m, l)
  static constexpr uint32_t DEC = TST + 4 * NSLOT * KT_MAX * GMAX * 2;          // [NSLOT][GMAX] int
  static constexpr uint32_t CTL = DEC + 4 * NSLOT * GMAX;                       // [16] int
  static constexpr uint32_t RF = CTL + 4 * 16;                                  // [GMAX][RF_SIZE] float
  static constexpr uint32_t RI = RF + 4 * GMAX * RF_SIZE;                       // [GMAX][RI_SIZE] int
  static constexpr uint32_t L2P = RI + 4 * GMAX * RI_SIZE;                      // [D] int8
  static constexpr uint32_t MXS = L2P + D;                                      // q8: [NSLOT][MXS_FLOATS]
  static constexpr uint32_t MXL = MXS + (Q8 ? 4 * NSLOT * MXS_FLOATS : 0);      // q8: [NWG][2][CMAX][GMAX]
  static constexpr uint32_t MXP = MXL + (Q8 ? 4 * NWG * 2 * CMAX * GMAX : 0);   // q8: [NWG][GMAX]
  static constexpr uint32_t PUB = MXP + (Q8 ? 4 * NWG * GMAX : 0);              // [NSLOT] publication slots
  static_assert(RF % 16 == 0 && PUB % 16 == 0 && TST % 16 == 0 && DEC % 16 == 0, "vector access");
  static_assert(Q % 1024 == 0 && (!Q8 || (KCV % 1024 == 0 && VCV % 1024 == 0)), "swizzled operands");
};
constexpr uint32_t OFF_STAGE = Lay<false>::STAGE;
constexpr uint32_t OFF_P = Lay<false>::P;
enum : int {
  B_FULL = 0, B_EMPTY = B_FULL + NSTG, B_SFULL = B_EMPTY + NSTG, B_SFREE = B_SFULL + 2,
  B_OFULL = B_SFREE + 2, B_XFULL = B_OFULL + 2, B_DEC = B_XFULL + NSLOT,
  B_DRAIN = B_DEC + NSLOT,  // [3]: tensor-core ops of the MMA warp, of warpgroup 0's and 1's leaders
  B_COUNT = B_DRAIN + 3,
  // q8 only: raw stage full / empty, K operand full / empty, V operands full / empty, scale ring
  // full / empty, maxima exchange of round r (slot r % NSLOT)
  B_RAWF = B_COUNT, B_RAWE = B_RAWF + Q8_NRAW, B_KCVF = B_RAWE + Q8_NRAW, B_KCVE = B_KCVF + 1,
  B_VCVF = B_KCVE + 1, B_VCVE = B_VCVF + 2, B_SCLF = B_VCVE + 2, B_SCLE = B_SCLF + 2, B_MXF = B_SCLE + 2,
  B_COUNT_Q8 = B_MXF + NSLOT
};
static_assert(B_COUNT_Q8 * 8 <= 512, "barrier area");
// Publication slot of a kernel with GP heads per kv head and probe capacity PC, one entry per
// (tile i of the block, head g), e = i * GP + g:  m_t[KT_MAX * GP], l_t[KT_MAX * GP], then the PC
// probe lanes of O_t per entry (rows of PC floats, 16-byte aligned for vector loads).
template <int GP, int PC, bool Q8 = false>
struct Pub {
  static constexpr uint32_t NE = KT_MAX * GP;
  static constexpr uint32_t OFF_L = NE, OFF_X = 2 * NE;  // float offsets inside a slot
  static constexpr uint32_t SLOT = 4 * NE * (2 + PC);
  static constexpr uint32_t SMEM_BYTES = Lay<Q8>::PUB + NSLOT * SLOT + 1024;  // + alignment slack
  static_assert((4 * OFF_X) % 16 == 0 && SLOT % 16 == 0, "probe rows 16-byte aligned");
  static_assert(SMEM_BYTES <= 232448, "shared memory per block");
};
constexpr uint32_t SMEM_BYTES = Pub<GMAX, PMAX>::SMEM_BYTES;  // the largest bf16 instantiation
constexpr uint32_t SMEM_BYTES_Q8 = Pub<4, PMAX, true>::SMEM_BYTES;
// final reduction (aliases stage 0 after the pipeline has drained):
// [NWG][GMAX][D] numerators, then [NWG][GMAX] m, [NWG][GMAX] l, [4] ints (slot 0 ends up holding
// the CTA's combined state)
constexpr uint32_t OFF_RED = 0;
constexpr uint32_t RED_M = NWG * GMAX * D, RED_L = RED_M + NWG * GMAX, RED_I = RED_L + NWG * GMAX;
// merge tables (floats): [CMAX][GMAX] per-rank maxima / weights, [CMAX][GMAX] per-rank
// denominators, [GMAX] merged max, [GMAX] merged denominators
constexpr uint32_t RED_W = RED_I + 8, RED_LT = RED_W + CMAX * GMAX, RED_MG = RED_LT + CMAX * GMAX,
                   RED_DN = RED_MG + GMAX;
static_assert(4 * (RED_DN + GMAX) <= STAGE_BYTES, "final reduction fits stage 0");
enum : int { CTL_EXIT = 0, CTL_EXIT_ROUND, CTL_ABORT, CTL_ISSUED, CTL_CONSUMED, CTL_TREAD, CTL_TMEM,
             CTL_STOPFLAG = 8,    // [2 rounds][2 controller warps]: all of the warp's heads stopped
             CTL_SAFE = 12,      // tiles the split will consume whatever the rest holds (decided so far)
             CTL_DECIDED = 13 };  // rounds decided so far

__device__ __forceinline__ uint32_t s_col(int b) { return 16u * b; }
// q8: S buffer b holds 4 accumulators of 16 columns (one per 32-wide scale block of d); O buffer b
// holds KT_MAX tiles of Q8_NP columns
__device__ __forceinline__ uint32_t s_col_q8(int b) { return 64u * b; }
__device__ __forceinline__ uint32_t o_col_q8(int b, int i) { return 128u + 64u * b + 32u * i; }
constexpr uint32_t idS8 = idesc_f16(128, 16, false, false);
constexpr uint32_t idO8 = idesc_f16(128, Q8_NP, true, true);
constexpr int BAR_CNV = 4;  // named barrier of the q8 converter warpgroup
// instruction descriptors: scores S^T = K . Q^T (both K-major); output O_t^T = V_t^T . P_t^T (both MN-major)
constexpr uint32_t idS = idesc_bf16(128, 16, false, false);
constexpr uint32_t idO = idesc_bf16(128, 16, true, true);
__device__ __forceinline__ uint32_t o_col(int b, int i) { return 32u + 32u * b + 16u * i; }

// A wait gives up after this many SM clock cycles (about one second at B200 clocks), sets the
// timeout bit of the status word and aborts the CTA.  A test build may set a short limit
// (ART_TC_WAIT_LIMIT_CYCLES) to drive that path; the drains keep their own limit, so a CTA that
// aborted still waits for the copies and tensor-core ops it issued.
#ifndef ART_TC_WAIT_LIMIT_CYCLES
#define ART_TC_WAIT_LIMIT_CYCLES 2000000000LL
#endif
constexpr long long kWaitLimitCycles = ART_TC_WAIT_LIMIT_CYCLES;
constexpr long long kDrainLimitCycles = 2000000000LL;
// Longest single sleep of a waiting thread between checks of the exit / abort flags.
constexpr uint32_t kSuspendNs = 2000;

// Bounded wait that also gives up when the CTA aborted (a timeout elsewhere) or,
// with watch_exit, when the ART controller ended the run.  Returns true when the
// phase completed.  The barrier is polled before any clock is read, and the
// limit uses the SM cycle counter (cheap) rather than the global timer.
__device__ __forceinline__ bool wait_phase(uint32_t bar, uint32_t parity, volatile int* ctl, bool watch_exit,
                                        int32_t* status, bool cluster_scope) {
  if (cluster_scope ? mbar_try_wait_cluster(bar, parity) : mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (true) {
    if (cluster_scope ? mbar_try_wait_cluster_sleep(bar, parity, kSuspendNs) : mbar_try_wait_sleep(bar, parity, kSuspendNs))
      return true;
    if (ctl[CTL_ABORT]) return false;
    if (watch_exit && ctl[CTL_EXIT]) {
      __threadfence_block();
      return cluster_scope ? mbar_try_wait_cluster(bar, parity) : mbar_try_wait(bar, parity);
    }
    if (clock64() - t0 > kWaitLimitCycles) {
      atomicOr(status, kStatusTimeout);
      ctl[CTL_ABORT] = 1;
      return false;
    }
  }
}

// Wait for asynchronous work the CTA has in flight (copies into its shared memory, tensor-core
// ops on its tensor memory) before that memory is reused or released.  Bounded by the wait limit
// only: a CTA that aborted still waits for what it issued.
__device__ __forceinline__ void drain_wait(uint32_t bar, uint32_t parity, int32_t* status) {
  if (mbar_try_wait(bar, parity)) return;
  const long long t0 = clock64();
  while (!mbar_try_wait_sleep(bar, parity, kSuspendNs)) {
    if (clock64() - t0 > kDrainLimitCycles) {
      atomicOr(status, kStatusTimeout);
      return;
    }
  }
}

// Wait for the controller's decision of round rp; false when it will never come
// (the run ended before that round, or the CTA aborted).
__device__ __forceinline__ bool wait_decision_phase(uint32_t bar, uint32_t parity, int rp, volatile int* ctl,
                                                 int32_t* status) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (true) {
    if (mbar_try_wait_sleep(bar, parity, kSuspendNs)) return true;
    if (ctl[CTL_ABORT]) return false;
    if (ctl[CTL_EXIT]) {
      __threadfence_block();
      if (rp > ctl[CTL_EXIT_ROUND]) return false;
    }
    if (clock64() - t0 > kWaitLimitCycles) {
      atomicOr(status, kStatusTimeout);
      ctl[CTL_ABORT] = 1;
      return false;
    }
  }
}

// GP: query heads per kv head (padded to 1, 2, 4 or 8); MODE: full or ART;
// PC: probe-lane capacity of the rule replay (16 or 32, lanes beyond n_probe are zero).
// ORD / PAGED: a traversal sequence / a paged cache; a kernel without them carries none of that
// code (the ART epilogue and the producer are sensitive to their instruction footprint).
// NCW: the ART controller: 0 = the sequential controller of a single-CTA cluster; 1 or 2 = the scan
// controller of a cluster on one warp or two (half of the heads each).
template <int GP, int MODE, int PC, bool ORD, bool PAGED, int NCW, bool Q8 = false>
__global__ void __launch_bounds__(Lay<Q8>::NTHR, 1) art_decode_tc_kernel(const __grid_constant__ TcParams p) {
  constexpr bool ART = (MODE == MODE_ART);
  using LY = Lay<Q8>;
  using PB = Pub<GP, PC, Q8>;
  constexpr int NT_ = LY::NTHR;
  static_assert(!Q8 || (GP == 4 && !ORD && !PAGED), "q8 cache: 3 or 4 query heads per kv head, natural order, contiguous");
  static_assert(GP >= 1 && GP <= 8, "up to 8 query heads per kv head");
  static_assert(PC == 16 || PC == 32, "probe capacity");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int C = p.C, G = p.G, P = p.n_probe;
  const int T = p.T;
  const int KT = ART ? BLK / T : 1;  // tiles per block (full attention: the block is one tile)
  const int TE = ART ? T : BLK;      // positions per tile inside the kernel
  const int rank = (C > 1) ? static_cast<int>(cluster_ctarank()) : 0;
  const int unit = blockIdx.x / C;
  const int split = unit % p.S;
  const int bk = unit / p.S;
  const int kvh = bk % p.Hkv;
  const int b = bk / p.Hkv;

  int L = p.seq_lens[b];
  const bool bad_len = (L < 1 || L > p.L_max);
  if (bad_len) L = 0;
  const int n_tiles = (L + T - 1) / T;
  const int t0 = static_cast<int>((static_cast<long long>(split) * n_tiles) / p.S);
  const int t1 = static_cast<int>((static_cast<long long>(split + 1) * n_tiles) / p.S);
  const int ns = t1 - t0;
  const int pbeg = t0 * T;
  const int pend = min(t1 * T, L);
  const int nblk = pend > pbeg ? (pend - pbeg + BLK - 1) / BLK : 0;
  const int my_blocks = nblk > rank ? (nblk - rank + C - 1) / C : 0;
  const int R = (nblk + C - 1) / C;
  const int zc = b * p.Hkv + kvh;
  // Tile at position q of this split's traversal sequence (ART with a sequence; natural order
  // otherwise).  An entry outside the split is replaced by the natural tile (the producer flags it).
  const int32_t* ord_seq = (ORD && ART && p.order) ? p.order + static_cast<long long>(zc) * p.n_max : nullptr;
  const int32_t* const btab = PAGED ? p.block_table : nullptr;
  auto phys_of = [&](int q) -> int {
    if (!ord_seq) return q;
    const int e = __ldg(ord_seq + q);
    return (e >= t0 && e < t1) ? e : q;
  };
  // tiles of own block jl that lie inside the split
  auto block_tiles = [&](int jl) -> int {
    if (!ART) return 1;
    const int j = jl * C + rank;
    return min(KT, t1 - (t0 + j * KT));
  };

  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + LY::BAR);
  auto bar = [&](int i) { return smem_u32(&bars[i]); };
  volatile int* ctl = reinterpret_cast<volatile int*>(sm + LY::CTL);
  float* wred = reinterpret_cast<float*>(sm + LY::WRED);
  float* wsum = reinterpret_cast<float*>(sm + LY::WSUM);
  float* tst = reinterpret_cast<float*>(sm + LY::TST);
  float* pub = reinterpret_cast<float*>(sm + LY::PUB);
  int* dec = reinterpret_cast<int*>(sm + LY::DEC);
  float* rf = reinterpret_cast<float*>(sm + LY::RF);
  int* ri = reinterpret_cast<int*>(sm + LY::RI);
  int8_t* l2p = reinterpret_cast<int8_t*>(sm + LY::L2P);

  // ---------------------------------------------------------------- setup
  if (tid == 0) {
    for (int s = 0; s < NSTG; ++s) {
      mbar_init(bar(B_FULL + s), 1);
      mbar_init(bar(B_EMPTY + s), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(B_SFULL + s), 1);
      mbar_init(bar(B_SFREE + s), 128);
      mbar_init(bar(B_OFULL + s), 1);
    }
    for (int s = 0; s < NSLOT; ++s) {
      mbar_init(bar(B_XFULL + s), C);
      mbar_init(bar(B_DEC + s), 1);
    }
    for (int s = 0; s < 3; ++s) mbar_init(bar(B_DRAIN + s), 1);
    if constexpr (Q8) {
      for (int s = 0; s < Q8_NRAW; ++s) {
        mbar_init(bar(B_RAWF + s), 1);
        mbar_init(bar(B_RAWE + s), 1);
      }
      mbar_init(bar(B_KCVF), 1);
      mbar_init(bar(B_KCVE), 1);
      for (int s = 0; s < 2; ++s) {
        mbar_init(bar(B_VCVF + s), 1);
        mbar_init(bar(B_VCVE + s), 1);
        mbar_init(bar(B_SCLF + s), 1);
        mbar_init(bar(B_SCLE + s), 128);
      }
      for (int s = 0; s < NSLOT; ++s) mbar_init(bar(B_MXF + s), C);
    }
    fence_mbar_init();
    if (bad_len && rank == 0) atomicOr(p.ws_status, kStatusSeqLen);
  }
  if (tid < 16) ctl[tid] = (tid == CTL_SAFE) ? min(ns, p.patience) : 0;  // no head stops before `patience` tiles
  for (int i = tid; i < D; i += NT_) l2p[i] = -1;
  for (int i = tid; i < static_cast<int>(2 * LY::PBUF / 16); i += NT_) reinterpret_cast<uint4*>(sm + LY::P)[i] = make_uint4(0, 0, 0, 0);
  if (ART)
    for (int i = tid; i < static_cast<int>(NSLOT * PB::SLOT / 16); i += NT_)
      reinterpret_cast<uint4*>(sm + LY::PUB)[i] = make_uint4(0, 0, 0, 0);
  if (tid < GMAX) {
    float* r = rf + tid * RF_SIZE;
    r[RF_M] = -INFINITY;
    r[RF_L] = 0.f;
    r[RF_NRM] = 0.f;
    for (int k = 0; k < PMAX; ++k) r[RF_A + k] = r[RF_XP + k] = 0.f;
    int* q = ri + tid * RI_SIZE;
    q[RI_RUN] = 0;
    q[RI_STOPPED] = (tid < G) ? 0 : 1;
    q[RI_USED] = ns;
    q[RI_STOPREL] = -1;
  }
  // Q^T as the scores' B operand: K-major, 128-byte swizzle, 16 rows x 2 halves of 64 d.  bf16: row
  // n = head n.  q8 (f16 operands on both sides): row n < 8 = f16 of head n, row 8 + n = the f16 of
  // what that leaves over (bf16 -> f16 hi + lo keeps q to ~22 bits).
  for (int i = tid; i < 16 * 16; i += NT_) {
    const int n = i >> 4, c = i & 15, h = c >> 3, cc = c & 7;
    uint4 w = make_uint4(0, 0, 0, 0);
    if constexpr (Q8) {
      const int hn = n & 7;
      if (hn < G) {
        const uint4 qv = *reinterpret_cast<const uint4*>(p.q + (static_cast<long long>(b) * p.Hq + kvh * G + hn) * D + c * 8);
        uint32_t qw[4] = {qv.x, qv.y, qv.z, qv.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float x0 = __uint_as_float(qw[k] << 16), x1 = __uint_as_float(qw[k] & 0xffff0000u);
          __half2 hh = __floats2half2_rn(x0, x1);
          if (n >= 8) {
            const float2 f = __half22float2(hh);
            hh = __floats2half2_rn(x0 - f.x, x1 - f.y);
          }
          qw[k] = *reinterpret_cast<uint32_t*>(&hh);
        }
        w = make_uint4(qw[0], qw[1], qw[2], qw[3]);
      }
    } else {
      if (n < G) w = *reinterpret_cast<const uint4*>(p.q + (static_cast<long long>(b) * p.Hq + kvh * G + n) * D + c * 8);
    }
    *reinterpret_cast<uint4*>(sm + LY::Q + h * 2048 + n * 128 + ((cc ^ (n & 7)) * 16)) = w;
  }
  if (warp == WARP_MMA) tmem_alloc(smem_u32(sm + LY::CTL + 4 * CTL_TMEM), LY::TMEM_COLS);
  __syncthreads();
  if (tid < P) l2p[p.lanes[tid]] = static_cast<int8_t>(tid);
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (C > 1) cluster_sync_all();  // every CTA's barriers exist before any remote arrive
  const uint32_t tmem = static_cast<uint32_t>(ctl[CTL_TMEM]);

  // owned online-softmax state of the epilogue threads (thread = d row)
  float acc[GP], m_own[GP], l_own[GP];
#pragma unroll
  for (int g = 0; g < GP; ++g) {
    acc[g] = 0.f;
    m_own[g] = -INFINITY;
    l_own[g] = 0.f;
  }

  // ---------------------------------------------------------------- roles
  // (the safe point once every head has stopped: no further round is read)
  constexpr int kNothingSafe = -(1 << 30);
  if (warp == WARP_TMA) {
    // ART with a bound on speculative reads: round jl is read only once it begins fewer than
    // spec_tiles tiles past the safe point.  Until then the thread sleeps on the decision barrier
    // of the next undecided round and re-reads the safe point and the decision count (so a phase
    // of the barrier that completed twice meanwhile costs one sleep, never a lost wake-up).  The
    // decision of round jl - 1 always puts round jl before the safe point unless the run has ended,
    // so the wait never needs round jl itself.  false: the run ended, or the CTA aborted.
    auto spec_ok = [&](int jl) -> bool {
      if (!ART || p.spec_tiles <= 0) return true;
      long long tw = 0;
      while (jl * (C * KT) >= ctl[CTL_SAFE] + p.spec_tiles) {
        if (ctl[CTL_EXIT] || ctl[CTL_ABORT]) return false;
        const int dn = ctl[CTL_DECIDED];
        if (!mbar_try_wait_sleep(bar(B_DEC + dn % NSLOT), (dn / NSLOT) & 1, kSuspendNs)) {
          if (tw == 0) tw = clock64();
          if (clock64() - tw > kWaitLimitCycles) {
            atomicOr(p.ws_status, kStatusTimeout);
            ctl[CTL_ABORT] = 1;
            return false;
          }
        }
        __threadfence_block();
      }
      return true;
    };
    if (Q8 && lane == 0) {
      // q8: per own block, the K and V codes (tensor maps over [B*Hkv][L_max][128] bytes, box 128 x
      // 128 rows) and the K and V scales (over [B*Hkv][L_max/2][16 bytes], box 16 x 64: two rows'
      // scales per 16 bytes) into raw stage jl % Q8_NRAW; positions past L_max are zero-filled
      int issued = 0, tiles_read = 0;
      for (int jl = 0; jl < my_blocks; ++jl) {
        if (ART && (ctl[CTL_EXIT] || !spec_ok(jl))) break;
        const int rs = jl % Q8_NRAW;
        if (jl >= Q8_NRAW && !wait_phase(bar(B_RAWE + rs), ((jl / Q8_NRAW) - 1) & 1, ctl, ART, p.ws_status, false))
          break;
        const int j = jl * C + rank;
        const int p0 = pbeg + j * BLK;
        ART_DCHECK(j < nblk && p0 >= 0 && p0 < p.L_max && (p0 & 1) == 0, p.ws_status);  // (scales: row pairs)
        const uint32_t fb = bar(B_RAWF + rs);
        const uint32_t st = smem_u32(sm + rs * Q8_RAW_BYTES);
        mbar_arrive_expect_tx(fb, Q8_RAW_BYTES);
        tma_load_3d(st + Q8_RAW_K, &p.tmK, fb, 0, p0, zc);
        tma_load_3d(st + Q8_RAW_V, &p.tmV, fb, 0, p0, zc);
        tma_load_3d(st + Q8_RAW_KS, &p.tmK64, fb, 0, p0 / 2, zc);
        tma_load_3d(st + Q8_RAW_VS, &p.tmV64, fb, 0, p0 / 2, zc);
        ++issued;
        tiles_read += min(BLK / T, t1 - (t0 + j * (BLK / T)));
      }
      ctl[CTL_ISSUED] = issued;
      ctl[CTL_TREAD] = tiles_read;
    } else if (lane == 0) {
      int issued = 0, tiles_read = 0;
      // paged cache in natural order: the page ids of a block follow from its position, so those of
      // the next block are loaded while this one's copies are issued and the next stage frees up
      const bool pg_ahead = btab && !ord_seq;
      const int32_t* bt_row = btab ? btab + static_cast<long long>(b) * p.max_pages : nullptr;
      auto page_ids = [&](int jl, int (&pg)[2]) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int lp = pbeg + (jl * C + rank) * BLK + 64 * h;
          pg[h] = (jl < my_blocks && lp < L) ? __ldg(bt_row + lp / p.page_size) : 0;
        }
      };
      int pg_cur[2] = {0, 0}, pg_next[2] = {0, 0};
      if (pg_ahead) page_ids(0, pg_cur);
      for (int jl = 0; jl < my_blocks; ++jl) {
        if (ART && (ctl[CTL_EXIT] || !spec_ok(jl))) break;
        const int stage = jl % NSTG;
        if (jl >= NSTG && !wait_phase(bar(B_EMPTY + stage), ((jl / NSTG) - 1) & 1, ctl, ART, p.ws_status, false)) break;
        const int j = jl * C + rank;
        const uint32_t fb = bar(B_FULL + stage);
        const uint32_t st = smem_u32(sm + OFF_STAGE + stage * STAGE_BYTES);
        if (!btab && (!ord_seq || T == BLK)) {
          // one 128-position run: the block, or its one (reordered) tile of 128
          int p0 = pbeg + j * BLK;
          if (ord_seq) {
            const int ph = phys_of(t0 + j);
            if (ph != __ldg(ord_seq + t0 + j)) atomicOr(p.ws_status, kStatusOrder);
            p0 = ph * BLK;
          }
          ART_DCHECK(j < nblk && p0 >= 0 && p0 < L, p.ws_status);
          mbar_arrive_expect_tx(fb, STAGE_BYTES);
          tma_load_3d(st, &p.tmK, fb, 0, p0, zc);
          tma_load_3d(st + 16384, &p.tmK, fb, 64, p0, zc);
          tma_load_3d(st + 32768, &p.tmV, fb, 0, p0, zc);
          tma_load_3d(st + 49152, &p.tmV, fb, 64, p0, zc);
        } else {
          // two 64-position halves, each from its own place (a tile of a traversal sequence, a
          // page of a paged cache), loaded when it starts inside the sequence; rows not loaded
          // are masked by the epilogue
          int lp[2];
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            if (ord_seq && T != BLK) {
              const int tq = t0 + j * KT + h;
              lp[h] = -1;
              if (tq < t1) {
                const int ph = phys_of(tq);
                if (ph != __ldg(ord_seq + tq)) atomicOr(p.ws_status, kStatusOrder);
                lp[h] = ph * 64;
              }
            } else if (ord_seq) {
              const int ph = phys_of(t0 + j);
              if (h == 0 && ph != __ldg(ord_seq + t0 + j)) atomicOr(p.ws_status, kStatusOrder);
              lp[h] = ph * BLK + 64 * h;
            } else {
              lp[h] = pbeg + j * BLK + 64 * h;
            }
            if (lp[h] >= L) lp[h] = -1;
          }
          mbar_arrive_expect_tx(fb, ((lp[0] >= 0) + (lp[1] >= 0)) * (STAGE_BYTES / 2));
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            if (lp[h] < 0) continue;
            int r = lp[h], z = zc;
            if (btab) {
              int pg = pg_ahead ? pg_cur[h] : __ldg(bt_row + lp[h] / p.page_size);
              if (pg < 0 || pg >= p.num_pages) {
                atomicOr(p.ws_status, kStatusPage);
                pg = 0;
              }
              r = lp[h] % p.page_size;
              z = pg * p.Hkv + kvh;
            }
            const uint32_t off = h * 8192;  // 64 rows of 128 bytes: whole swizzle atoms
            tma_load_3d(st + off, &p.tmK64, fb, 0, r, z);
            tma_load_3d(st + 16384 + off, &p.tmK64, fb, 64, r, z);
            tma_load_3d(st + 32768 + off, &p.tmV64, fb, 0, r, z);
            tma_load_3d(st + 49152 + off, &p.tmV64, fb, 64, r, z);
          }
        }
        if (pg_ahead) {
          page_ids(jl + 1, pg_next);
          pg_cur[0] = pg_next[0];
          pg_cur[1] = pg_next[1];
        }
        ++issued;
        tiles_read += min(BLK / T, t1 - (t0 + j * (BLK / T)));
      }
      ctl[CTL_ISSUED] = issued;
      ctl[CTL_TREAD] = tiles_read;
    }
  } else if (warp == WARP_MMA) {
    if (lane == 0) {
      const uint32_t q_addr = smem_u32(sm + LY::Q);
      // The scores of every own block, in order: K/V landed, S buffer free.  (The PV product of
      // a block is issued by the leader of the epilogue warpgroup that wrote its weights.)
      // Descriptors are built once per operand buffer and stepped by constant offsets: the
      // address field (bits 0-13, 16-byte units) of a shared-memory address below 256 KB never
      // carries into the next field.
      const uint64_t qd0 = smem_desc(q_addr, 16, 1024, 2);
      int consumed = 0;
      if constexpr (Q8) {
        // q8: scores from the converted K operand (f16 codes) into 4 accumulators, one per scale
        // block of 32 d (2 MMAs of 16 d each); the epilogue applies each row's block scales
        const uint64_t kd0 = smem_desc(smem_u32(sm + LY::KCV), 16, 1024, 2);
        for (int jl = 0; jl < my_blocks; ++jl) {
          const int bb = jl & 1;
          if (!wait_phase(bar(B_KCVF), jl & 1, ctl, ART, p.ws_status, false)) break;
          if (jl >= 2 && !wait_phase(bar(B_SFREE + bb), ((jl >> 1) - 1) & 1, ctl, ART, p.ws_status, false)) break;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            constexpr uint32_t kq[8] = {0, 2, 4, 6, 1024, 1026, 1028, 1030};
            constexpr uint32_t qq[8] = {0, 2, 4, 6, 128, 130, 132, 134};
            umma_bf16(tmem + s_col_q8(bb) + 16u * (kk >> 1), kd0 + kq[kk], qd0 + qq[kk], idS8, kk & 1);
          }
          umma_commit(bar(B_SFULL + bb));
          umma_commit(bar(B_KCVE));  // the K operand may be overwritten once these scores are done
        }
      }
      for (int jl = 0; !Q8 && jl < my_blocks; ++jl) {
        const int stage = jl % NSTG, bb = jl & 1;
        if (!wait_phase(bar(B_FULL + stage), (jl / NSTG) & 1, ctl, ART, p.ws_status, false)) break;
        consumed = jl + 1;
        if (jl >= 2 && !wait_phase(bar(B_SFREE + bb), ((jl >> 1) - 1) & 1, ctl, ART, p.ws_status, false)) break;
        tc_fence_after();
        const uint64_t kd0 = smem_desc(smem_u32(sm + OFF_STAGE + stage * STAGE_BYTES), 16, 1024, 2);
        const uint32_t dcol = tmem + s_col(bb);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          constexpr uint32_t kq[8] = {0, 2, 4, 6, 1024, 1026, 1028, 1030};  // (h * 16384 + (kk & 3) * 32) / 16
          constexpr uint32_t qq[8] = {0, 2, 4, 6, 128, 130, 132, 134};      // (h * 2048 + (kk & 3) * 32) / 16
          umma_bf16(dcol, kd0 + kq[kk], qd0 + qq[kk], idS, kk > 0);
        }
        umma_commit(bar(B_SFULL + bb));
      }
      if (!Q8) ctl[CTL_CONSUMED] = consumed;  // (q8: the converter consumes the raw stages)
      // every tensor-core op this thread issued has completed before the drain barrier fires
      umma_commit(bar(B_DRAIN));
      drain_wait(bar(B_DRAIN), 0, p.ws_status);
    }
    __syncwarp();
  } else if (Q8 && warp >= WARP_EPI0 + 4 * NWG) {
    // ------------------------------------------------------------ q8 converter warpgroup
    // Thread ct owns row ct of each block: its K codes become the f16 K operand (once the previous
    // block's scores have read it), its scales go to the scale ring (once the epilogue has read
    // the entry's previous block), its V codes become the f16 V operand (once the PV product two
    // blocks back has read it); then the raw stage is released.  Waits are taken by thread 0 and
    // shared through the warpgroup's named barrier.
    const int ct = tid - 32 * (WARP_EPI0 + 4 * NWG);
    const bool cl = (ct == 0);
    auto cv_wait = [&](uint32_t bar_, uint32_t parity) -> bool {
      bool ok = true;
      if (cl) ok = wait_phase(bar_, parity, ctl, ART, p.ws_status, false);
      return named_barrier_and(BAR_CNV, 128, ok);
    };
    int consumed = 0;
    for (int jl = 0; jl < my_blocks; ++jl) {
      const int rs = jl % Q8_NRAW, vb = jl & 1;
      const uint8_t* raw = sm + rs * Q8_RAW_BYTES;
      if (!cv_wait(bar(B_RAWF + rs), (jl / Q8_NRAW) & 1)) break;
      consumed = jl + 1;
      if (jl >= 1 && !cv_wait(bar(B_KCVE), (jl - 1) & 1)) break;
      convert_code_row(raw + Q8_RAW_K, sm + LY::KCV, ct);
      if (jl >= 2 && !cv_wait(bar(B_SCLE + vb), ((jl >> 1) - 1) & 1)) break;
      uint8_t* scl = sm + LY::SCL + vb * Q8_SCL_BYTES;
      *reinterpret_cast<uint2*>(scl + ct * 8) = *reinterpret_cast<const uint2*>(raw + Q8_RAW_KS + ct * 8);
      *reinterpret_cast<uint2*>(scl + 1024 + ct * 8) = *reinterpret_cast<const uint2*>(raw + Q8_RAW_VS + ct * 8);
      fence_proxy_async_smem();  // the K operand is read by the tensor cores
      named_barrier(BAR_CNV, 128);
      if (cl) {
        mbar_arrive(bar(B_KCVF));
        mbar_arrive(bar(B_SCLF + vb));
      }
      if (jl >= 2 && !cv_wait(bar(B_VCVE + vb), ((jl >> 1) - 1) & 1)) break;
      convert_code_row(raw + Q8_RAW_V, sm + LY::VCV + vb * 32768, ct);
      fence_proxy_async_smem();
      named_barrier(BAR_CNV, 128);
      if (cl) {
        mbar_arrive(bar(B_VCVF + vb));
        mbar_arrive(bar(B_RAWE + rs));
      }
    }
    if (cl) ctl[CTL_CONSUMED] = consumed;
  } else if (warp >= WARP_EPI0) {
    // ------------------------------------------------------------ epilogue warpgroups
    // Warpgroup wg takes the own blocks jl = wg, wg + NWG, ... (TMEM and smem buffers
    // bb = jl & 1 = wg).  All 128 threads of a warpgroup take every branch together:
    // mbarrier waits are done by one leader thread and their outcome is shared with a
    // reducing named barrier of that warpgroup.
    const int wg = (warp - WARP_EPI0) >> 2;
    const int bar_epi = BAR_EPI + wg;
    const int wq = warp & 3;
    const int er = 32 * wq + lane;  // TMEM lane: position row of S, d row of O
    const bool leader = (er == 0);
    const uint32_t lane_base = static_cast<uint32_t>(32 * wq) << 16;
    const int w_n = TE / 32;           // warps per tile
    const int w_lo = (er / TE) * w_n;  // first warp of this row's tile
    // reductions over the warps of one tile run over all four warps with a predicate
    // (fixed trip count, no loop branches)
    auto in_tile = [&](int w, int lo) { return w >= lo && w < lo + w_n; };
    auto epi_wait = [&](uint32_t bb_, uint32_t parity, bool watch_exit) -> bool {
      bool ok = true;
      if (leader) ok = wait_phase(bb_, parity, ctl, watch_exit, p.ws_status, false);
      return named_barrier_and(bar_epi, 128, ok);
    };
    // ot: this block's tile outputs; pnd: the warpgroup's previous round (published, not
    // merged yet: a round is merged LAG = NWG rounds, i.e. one own round, after publication)
    static_assert(LAG == NWG, "one pending own round");
    float ot[KT_MAX][GP], pnd[KT_MAX][GP];
#pragma unroll
    for (int i = 0; i < KT_MAX; ++i)
#pragma unroll
      for (int g = 0; g < GP; ++g) ot[i][g] = pnd[i][g] = 0.f;
    int ntl_p = 0;
    auto merge_tile = [&](int g, float mt, float lt, float o) {
      const float M = fmaxf(m_own[g], mt);
      const float a = rescale_fast(m_own[g], M), bt = rescale_fast(mt, M);
      acc[g] = a * acc[g] + bt * o;
      l_own[g] = a * l_own[g] + bt * lt;
      m_own[g] = M;
    };
    // merge the pending tiles `pt` (ntlp of them) of round rp by that round's decision.  The
    // decisions and tile statistics are loaded first (vector loads), then every (tile, head) is
    // merged without branches: a tile past its head's stop tile merges with weight 0.
    auto merge_round = [&](int rp, const float (&pt)[KT_MAX][GP], int ntlp) {
      const int sp = rp % NSLOT;
      int dv[GP];
      float tm[KT_MAX][GP], tl[KT_MAX][GP];
      if constexpr (GP >= 4) {
#pragma unroll
        for (int g = 0; g < GP; g += 4) {
          const int4 d4 = *reinterpret_cast<const int4*>(dec + sp * GMAX + g);
          dv[g] = d4.x, dv[g + 1] = d4.y, dv[g + 2] = d4.z, dv[g + 3] = d4.w;
        }
      } else {
#pragma unroll
        for (int g = 0; g < GP; ++g) dv[g] = dec[sp * GMAX + g];
      }
#pragma unroll
      for (int i = 0; i < KT_MAX; ++i) {
        const float* ts = tst + (sp * KT_MAX + i) * GMAX * 2;
        if constexpr (GP >= 2) {
#pragma unroll
          for (int g = 0; g < GP; g += 2) {
            const float4 v = *reinterpret_cast<const float4*>(ts + 2 * g);
            tm[i][g] = v.x, tl[i][g] = v.y, tm[i][g + 1] = v.z, tl[i][g + 1] = v.w;
          }
        } else {
          tm[i][0] = ts[0], tl[i][0] = ts[1];
        }
      }
#pragma unroll
      for (int i = 0; i < KT_MAX; ++i) {
        const int q = rank * KT + i;
#pragma unroll
        for (int g = 0; g < GP; ++g) {
          const int d = dv[g];
          const bool take = i < ntlp && g < G && (d == -1 || (d >= 0 && q <= d));
          // statistics of a tile that is not taken may be stale or unset: select, never scale by 0
          const float M = fmaxf(m_own[g], tm[i][g]);
          const float a = rescale_fast(m_own[g], M), bt = rescale_fast(tm[i][g], M);
          const float na = a * acc[g] + bt * pt[i][g], nl = a * l_own[g] + bt * tl[i][g];
          acc[g] = take ? na : acc[g];
          l_own[g] = take ? nl : l_own[g];
          m_own[g] = take ? M : m_own[g];
        }
      }
    };
    // wait (leader) for the controller's decision of round rp; false if it will never come
    auto wait_decision = [&](int rp) -> bool {
      bool got = true;
      if (leader) got = wait_decision_phase(bar(B_DEC + rp % NSLOT), (rp / NSLOT) & 1, rp, ctl, p.ws_status);
      return named_barrier_and(bar_epi, 128, got);
    };

    // scores -> weights -> P^T (hi, lo) in smem for own block jl; false if the run ended
    auto s_phase = [&](int jl) -> bool {
      const int bb = jl & 1, stage = jl % NSTG;
      const int j = jl * C + rank;
      // this row's KV position (the load is issued before the wait and used after it)
      const int tq = t0 + j * KT + er / TE;
      const int ph = (ord_seq && tq < t1) ? phys_of(tq) : 0;
      if (!epi_wait(bar(B_SFULL + bb), (jl >> 1) & 1, ART)) return false;
      tc_fence_after();
      float sv[8];
      tmem_ld8(tmem + lane_base + s_col(bb), sv);
      tmem_ld_wait();
      tc_fence_before();
      mbar_arrive(bar(B_SFREE + bb));
      const int pos = ord_seq ? ph * T + (er % TE) : pbeg + j * BLK + er;
      const bool valid = ord_seq ? (tq < t1 && pos < L) : (pos < pend);
      float s2[GP], red[GP], pw[GP];
#pragma unroll
      for (int g = 0; g < GP; ++g) red[g] = s2[g] = (valid && g < G) ? sv[g] * p.qscale : -INFINITY;
      {
        const float wm = warp_reduce_heads<GP, true>(red, lane);
        if ((lane & (32 / GP - 1)) == 0) wred[(bb * 4 + wq) * GMAX + lane / (32 / GP)] = wm;
      }
      named_barrier(bar_epi, 128);
#pragma unroll
      for (int g = 0; g < GP; ++g) {
        float mt = -INFINITY;
#pragma unroll
        for (int w = 0; w < 4; ++w)
          if (in_tile(w, w_lo)) mt = fmaxf(mt, wred[(bb * 4 + w) * GMAX + g]);
        red[g] = pw[g] = (s2[g] == -INFINITY) ? 0.f : ex2_fast(s2[g] - mt);
      }
      {
        const float ws = warp_reduce_heads<GP, false>(red, lane);
        if ((lane & (32 / GP - 1)) == 0) wsum[(bb * 4 + wq) * GMAX + lane / (32 / GP)] = ws;
      }
      uint8_t* prow = sm + OFF_P + bb * 4096 + (er >> 3) * 256 + (er & 7) * 16;
#pragma unroll
      for (int g = 0; g < GP; ++g) {
        const __nv_bfloat16 h = __float2bfloat16_rn(pw[g]);
        const __nv_bfloat16 l = __float2bfloat16_rn(pw[g] - __bfloat162float(h));
        reinterpret_cast<uint16_t*>(prow)[g] = __bfloat16_as_ushort(h);
        reinterpret_cast<uint16_t*>(prow + 128)[g] = __bfloat16_as_ushort(l);
      }
      if (!valid) {  // V rows of positions past the end must not reach the MMA
        uint8_t* vrow = sm + OFF_STAGE + stage * STAGE_BYTES + 32768 + er * 128;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          reinterpret_cast<uint4*>(vrow)[c] = make_uint4(0, 0, 0, 0);
          reinterpret_cast<uint4*>(vrow + 16384)[c] = make_uint4(0, 0, 0, 0);
        }
      }
      // every thread's weights (and zeroed V rows) are written: the leader issues the PV product
      fence_proxy_async_smem();
      named_barrier(bar_epi, 128);
      if (leader) {
        tc_fence_after();
        const int ntl = block_tiles(jl);
        const uint64_t vd0 = smem_desc(smem_u32(sm + OFF_STAGE + stage * STAGE_BYTES + 32768), 16384, 1024, 2);
        const uint64_t pd0 = smem_desc(smem_u32(sm + OFF_P + bb * 4096), 256, 128, 0);
        // 8 MMAs of 16 positions each, unrolled so that the operand offsets are constants; MMA u
        // belongs to tile u * 16 / TE and starts that tile's accumulator when it is its first
        const int tsh = (TE == 64) ? 6 : 7;
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int i = (u * 16) >> tsh;
          if (i < ntl) umma_bf16(tmem + o_col(bb, i), vd0 + (u * 128u), pd0 + (u * 32u), idO, ((u * 16) & (TE - 1)) != 0);
        }
        umma_commit(bar(B_OFULL + bb));
        umma_commit(bar(B_EMPTY + stage));
      }
      return true;
    };
    // ---- q8: the V skip's threshold.  Row j of caller tile t (T positions) leaves head g's
    // numerator when its score s_j < m'_t + log2(tau), m'_t the running maximum of the split's
    // scores after tile t = max(every tile of earlier rounds, every tile of the round's lower-ranked
    // CTAs, this block's caller tiles up to t).  Each CTA publishes its round's caller-tile and block
    // maxima and signals every CTA of the cluster (rounds without a block of the CTA too); threads
    // 0..GP-1 of the warpgroup keep the maximum over all rounds up to two back (mrun2) and take the
    // round before from the exchange.
    float mrun2 = -INFINITY;
    auto mx_publish = [&](int r, int bbx, bool has_block) {
      float* mo = reinterpret_cast<float*>(sm + LY::MXS) + (r % NSLOT) * MXS_FLOATS;
      const int ksn = BLK / T, wnt = T / 32;
      if (er < KT_MAX * GP) {
        const int i = er / GP, g = er % GP;
        float mt = -INFINITY;
        if (has_block && i < ksn && g < G) {
#pragma unroll
          for (int w = 0; w < 4; ++w)
            if (w >= i * wnt && w < (i + 1) * wnt) mt = fmaxf(mt, wred[(bbx * 4 + w) * GMAX + g]);
        }
        mo[i * GMAX + g] = mt;
      }
      if (er < GP) {
        float mb = -INFINITY;
        if (has_block && er < G) {
#pragma unroll
          for (int w = 0; w < 4; ++w) mb = fmaxf(mb, wred[(bbx * 4 + w) * GMAX + er]);
        }
        mo[KT_MAX * GMAX + er] = mb;
      }
      named_barrier(bar_epi, 128);
      if (er < C) {
        if (C > 1) {
          fence_acq_rel_cluster();
          mbar_arrive_cluster_relaxed(map_to_rank(bar(B_MXF + r % NSLOT), er));
        } else {
          mbar_arrive(bar(B_MXF + r % NSLOT));
        }
      }
    };
    auto mx_threshold = [&](int r, float (&thr)[GP]) -> bool {
      bool ok = true;
      if (leader) {
        ok = wait_phase(bar(B_MXF + r % NSLOT), (r / NSLOT) & 1, ctl, ART, p.ws_status, C > 1);
        if (ok && r >= 1)
          ok = wait_phase(bar(B_MXF + (r - 1) % NSLOT), ((r - 1) / NSLOT) & 1, ctl, ART, p.ws_status, C > 1);
      }
      if (!named_barrier_and(bar_epi, 128, ok)) return false;
      float* mxl = reinterpret_cast<float*>(sm + LY::MXL) + wg * 2 * CMAX * GMAX;
      const uint32_t mxs = smem_u32(sm + LY::MXS);
      if (er < C * GP) {  // block maxima of CTA c, this round and the round before
        const int c = er / GP, g = er % GP;
        const uint32_t a0 = mxs + 4 * ((r % NSLOT) * MXS_FLOATS + KT_MAX * GMAX + g);
        mxl[c * GMAX + g] = ld_smem_f32(C > 1 ? map_to_rank(a0, c) : a0, C > 1);
        float pv = -INFINITY;
        if (r >= 1) {
          const uint32_t a1 = mxs + 4 * (((r - 1) % NSLOT) * MXS_FLOATS + KT_MAX * GMAX + g);
          pv = ld_smem_f32(C > 1 ? map_to_rank(a1, c) : a1, C > 1);
        }
        mxl[CMAX * GMAX + c * GMAX + g] = pv;
      }
      named_barrier(bar_epi, 128);
      float* mxp = reinterpret_cast<float*>(sm + LY::MXP) + wg * GMAX;
      if (er < GP) {
        float pre = mrun2, nxt = mrun2;
        for (int c = 0; c < C; ++c) {
          const float vp = mxl[CMAX * GMAX + c * GMAX + er], vc = mxl[c * GMAX + er];
          pre = fmaxf(pre, vp);
          nxt = fmaxf(nxt, fmaxf(vp, vc));
          if (c < rank) pre = fmaxf(pre, vc);
        }
        mxp[er] = pre;
        mrun2 = nxt;
      }
      named_barrier(bar_epi, 128);
      const float* mo = reinterpret_cast<const float*>(sm + LY::MXS) + (r % NSLOT) * MXS_FLOATS;
      const int ic = (T == 64) ? (er >> 6) : 0;  // this row's caller tile inside the block
#pragma unroll
      for (int g = 0; g < GP; ++g) {
        float m = mxp[g];
#pragma unroll
        for (int i = 0; i < KT_MAX; ++i)
          if (i <= ic) m = fmaxf(m, mo[i * GMAX + g]);
        thr[g] = m + p.log2tau;
      }
      return true;
    };
    // q8: scores -> weights -> P'^T in smem -> PV product for own block jl; false if the run ended.
    // S buffer bb holds, per scale block of 32 d, the products with q's f16 hi part (columns 0..7)
    // and lo part (8..15); s = sum over blocks of (hi + lo) x the row's K scale of the block.  P'
    // has, per scale block, f16 hi and lo parts of p x (the row's V scale of the block): columns
    // 8 * block + {0..3 hi, 4..7 lo} for the 4 heads; a (row, head) below the V-skip threshold
    // gets 0 there (its weight stays in the denominator).
    auto s_phase_q8 = [&](int jl) -> bool {
      const int bb = jl & 1;
      const int j = jl * C + rank;
      bool ok = true;
      if (leader)
        ok = wait_phase(bar(B_SFULL + bb), (jl >> 1) & 1, ctl, ART, p.ws_status, false) &&
             wait_phase(bar(B_SCLF + bb), (jl >> 1) & 1, ctl, ART, p.ws_status, false);
      if (!named_barrier_and(bar_epi, 128, ok)) return false;
      tc_fence_after();
      float sh[4][4], sl[4][4];
#pragma unroll
      for (int bk = 0; bk < 4; ++bk) {
        tmem_ld4(tmem + lane_base + s_col_q8(bb) + 16u * bk, sh[bk]);
        tmem_ld4(tmem + lane_base + s_col_q8(bb) + 16u * bk + 8u, sl[bk]);
      }
      const uint8_t* scl = sm + LY::SCL + bb * Q8_SCL_BYTES;
      const uint2 ksw = *reinterpret_cast<const uint2*>(scl + er * 8);
      const uint2 vsw = *reinterpret_cast<const uint2*>(scl + 1024 + er * 8);
      mbar_arrive(bar(B_SCLE + bb));
      tmem_ld_wait();
      tc_fence_before();
      mbar_arrive(bar(B_SFREE + bb));
      auto h2f = [](uint32_t bits) { return __half2float(__ushort_as_half(static_cast<unsigned short>(bits & 0xffffu))); };
      const float ks[4] = {h2f(ksw.x), h2f(ksw.x >> 16), h2f(ksw.y), h2f(ksw.y >> 16)};
      const float vs[4] = {h2f(vsw.x), h2f(vsw.x >> 16), h2f(vsw.y), h2f(vsw.y >> 16)};
      const int pos = pbeg + j * BLK + er;
      const bool valid = pos < pend;
      float s2[GP], red[GP], pw[GP];
#pragma unroll
      for (int g = 0; g < GP; ++g) {
        float sg = 0.f;
#pragma unroll
        for (int bk = 0; bk < 4; ++bk) sg = fmaf(ks[bk], sh[bk][g] + sl[bk][g], sg);
        red[g] = s2[g] = (valid && g < G) ? sg * p.qscale : -INFINITY;
      }
      {
        const float wm = warp_reduce_heads<GP, true>(red, lane);
        if ((lane & (32 / GP - 1)) == 0) wred[(bb * 4 + wq) * GMAX + lane / (32 / GP)] = wm;
      }
      named_barrier(bar_epi, 128);
      const bool skip_on = p.tau > 0.f;
      if (skip_on) mx_publish(jl, bb, true);
#pragma unroll
      for (int g = 0; g < GP; ++g) {
        float mt = -INFINITY;
#pragma unroll
        for (int w = 0; w < 4; ++w)
          if (in_tile(w, w_lo)) mt = fmaxf(mt, wred[(bb * 4 + w) * GMAX + g]);
        red[g] = pw[g] = (s2[g] == -INFINITY) ? 0.f : ex2_fast(s2[g] - mt);
      }
      {
        const float ws = warp_reduce_heads<GP, false>(red, lane);
        if ((lane & (32 / GP - 1)) == 0) wsum[(bb * 4 + wq) * GMAX + lane / (32 / GP)] = ws;
      }
      float thr[GP];
#pragma unroll
      for (int g = 0; g < GP; ++g) thr[g] = -INFINITY;
      if (skip_on && !mx_threshold(jl, thr)) return false;
      uint8_t* prow = sm + LY::P + bb * LY::PBUF + (er >> 3) * 512 + (er & 7) * 16;
#pragma unroll
      for (int bk = 0; bk < 4; ++bk) {
        uint32_t hw[2], lw[2];
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
          const int g0 = 2 * h2;
          const float x0 = (s2[g0] < thr[g0]) ? 0.f : pw[g0] * vs[bk];
          const float x1 = (s2[g0 + 1] < thr[g0 + 1]) ? 0.f : pw[g0 + 1] * vs[bk];
          __half2 hh = __floats2half2_rn(x0, x1);
          const float2 f = __half22float2(hh);
          __half2 ll = __floats2half2_rn(x0 - f.x, x1 - f.y);
          hw[h2] = *reinterpret_cast<uint32_t*>(&hh);
          lw[h2] = *reinterpret_cast<uint32_t*>(&ll);
        }
        *reinterpret_cast<uint4*>(prow + bk * 128) = make_uint4(hw[0], hw[1], lw[0], lw[1]);
      }
      // every thread's weights are written: the leader issues the PV product once the converter
      // has written this block's V operand
      fence_proxy_async_smem();
      named_barrier(bar_epi, 128);
      if (leader && wait_phase(bar(B_VCVF + bb), (jl >> 1) & 1, ctl, ART, p.ws_status, false)) {
        tc_fence_after();
        const int ntl = block_tiles(jl);
        const uint64_t vd0 = smem_desc(smem_u32(sm + LY::VCV + bb * 32768), 16384, 1024, 2);
        const uint64_t pd0 = smem_desc(smem_u32(sm + LY::P + bb * LY::PBUF), 512, 128, 0);
        const int tsh = (TE == 64) ? 6 : 7;
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int i = (u * 16) >> tsh;
          if (i < ntl) umma_bf16(tmem + o_col_q8(bb, i), vd0 + (u * 128u), pd0 + (u * 64u), idO8, ((u * 16) & (TE - 1)) != 0);
        }
        umma_commit(bar(B_OFULL + bb));
        umma_commit(bar(B_VCVE + bb));
      }
      return true;
    };
    // O_t readback (thread = d row) for own block jl into ot; tile stats to tst; false if the run ended
    auto o_phase = [&](int jl, int& ntl) -> bool {
      const int bb = jl & 1;
      ntl = block_tiles(jl);
      if (!epi_wait(bar(B_OFULL + bb), (jl >> 1) & 1, ART)) {
        ntl = 0;
        return false;
      }
      tc_fence_after();
#pragma unroll
      for (int i = 0; i < KT_MAX; ++i) {
        if (i < ntl) {
          if constexpr (Q8) {
            // rows of warp wq are the d rows of scale block wq: its 8 columns (4 hi, 4 lo)
            float ov[8];
            tmem_ld8(tmem + lane_base + o_col_q8(bb, i) + 8u * wq, ov);
            tmem_ld_wait();
#pragma unroll
            for (int g = 0; g < GP; ++g) ot[i][g] = ov[g] + ov[4 + g];
          } else {
            float ov[16];
            tmem_ld16(tmem + lane_base + o_col(bb, i), ov);
            tmem_ld_wait();
#pragma unroll
            for (int g = 0; g < GP; ++g) ot[i][g] = ov[g] + ov[8 + g];
          }
        }
      }
      tc_fence_before();  // O of buffer bb is read: the next PV into it comes after a warpgroup barrier
      if (!ART) {  // the block is one tile: every thread merges it into its own state
#pragma unroll
        for (int g = 0; g < GP; ++g) {
          float mt = -INFINITY, lt = 0.f;
#pragma unroll
          for (int w = 0; w < 4; ++w) {
            mt = fmaxf(mt, wred[(bb * 4 + w) * GMAX + g]);
            lt += wsum[(bb * 4 + w) * GMAX + g];
          }
          if (g < G) merge_tile(g, mt, lt, ot[0][g]);
        }
      } else {
        // ART: this block's tiles go to publication slot jl % NSLOT.  One thread per (tile, head)
        // forms the tile's (m_t, l_t) from the per-warp maxima and sums and writes it to the slot
        // and to the CTA's own copy (tst, read by the merge); the threads of the probe lanes write
        // their lanes of O_t.  The warpgroup barrier that follows orders these writes before the
        // round is signalled.
        const int sl = jl % NSLOT;
        float* ps = pub + sl * (PB::SLOT / 4);
        if (er < KT_MAX * GP) {
          const int i = er / GP, g = er % GP;
          if (i < ntl && g < G) {
            float mt = -INFINITY, lt = 0.f;
#pragma unroll
            for (int w = 0; w < 4; ++w)
              if (in_tile(w, i * w_n)) {
                mt = fmaxf(mt, wred[(bb * 4 + w) * GMAX + g]);
                lt += wsum[(bb * 4 + w) * GMAX + g];
              }
            tst[(sl * KT_MAX + i) * GMAX * 2 + g * 2 + 0] = mt;
            tst[(sl * KT_MAX + i) * GMAX * 2 + g * 2 + 1] = lt;
            ps[er] = mt;
            ps[PB::OFF_L + er] = lt;
          }
        }
        const int pi = l2p[er];
        if (pi >= 0) {
#pragma unroll
          for (int i = 0; i < KT_MAX; ++i)
#pragma unroll
            for (int g = 0; g < GP; ++g)
              if (i < ntl && g < G) ps[PB::OFF_X + (i * GP + g) * PC + pi] = ot[i][g];
        }
      }
      return true;
    };

    // q8 with the V skip: every round takes part in the maxima exchange, blocks or not
    const bool mx_on = Q8 && p.tau > 0.f;
    const int iters = (ART || mx_on) ? R : my_blocks;
    bool streaming = true;
    for (int r = wg; r < iters; r += NWG) {  // own block r of the CTA = ART round r
      int ntl = 0;
      if (r < my_blocks && streaming) {
        if constexpr (Q8)
          streaming = s_phase_q8(r);
        else
          streaming = s_phase(r);
      } else if (mx_on && streaming && r >= my_blocks) {
        mx_publish(r, r & 1, false);
      }
      if (r < my_blocks && streaming) streaming = o_phase(r, ntl);
      if (!ART) {
        if (!streaming) break;  // aborted
        continue;
      }
      // Merge, in order, the warpgroup's rounds lo, lo + NWG, .., hi (r - LAG held in pnd,
      // r in ot) by their decisions.  A single call site keeps the loop body small.
      auto merge_span = [&](int lo, int hi) -> bool {
#pragma unroll 1
        for (int rk = lo; rk <= hi; rk += NWG) {
          if (!wait_decision(rk)) return false;
          const bool cur = (rk == r);
          float tmp[KT_MAX][GP];
#pragma unroll
          for (int i = 0; i < KT_MAX; ++i)
#pragma unroll
            for (int g = 0; g < GP; ++g) tmp[i][g] = cur ? ot[i][g] : pnd[i][g];
          merge_round(rk, tmp, cur ? ntl : ntl_p);
        }
        return true;
      };
      // Once the controller has ended the run, merge every round it decided and leave.
      // Otherwise publish round r, then merge round r - LAG by its decision (after the
      // warpgroup's last round, everything still pending).  Both paths share one merge site.
      const bool leaving = named_barrier_or(bar_epi, 128, leader && (ctl[CTL_EXIT] || ctl[CTL_ABORT]));
      int m_hi;
      if (leaving) {
        const bool aborted = named_barrier_or(bar_epi, 128, leader && ctl[CTL_ABORT] != 0);
        const int er_round = ctl[CTL_EXIT_ROUND];  // written before the exit flag, never changed after
        m_hi = aborted ? -1 : min(r, er_round);
      } else {
        // round r is in its publication slot (written by o_phase; the barrier above ordered the
        // warpgroup's writes): signal every CTA's controller.  Across CTAs the slot is read through
        // distributed shared memory, so the signalling thread first fences at cluster scope; a
        // single CTA needs only the barrier's own release.
        const int sl = r % NSLOT;
        if (er < C) {
          if (C > 1) {
            fence_acq_rel_cluster();
            mbar_arrive_cluster_relaxed(map_to_rank(bar(B_XFULL + sl), er));
          } else {
            mbar_arrive(bar(B_XFULL + sl));
          }
        }
        m_hi = (r + NWG >= iters) ? r : r - LAG;
      }
      merge_span(r >= LAG ? r - LAG : r, m_hi);
      if (leaving) break;
#pragma unroll
      for (int i = 0; i < KT_MAX; ++i)
#pragma unroll
        for (int g = 0; g < GP; ++g) pnd[i][g] = ot[i][g];
      ntl_p = ntl;
    }
    // every PV product this warpgroup's leader issued has completed before the CTA moves on
    if (leader) {
      umma_commit(bar(B_DRAIN + 1 + wg));
      drain_wait(bar(B_DRAIN + 1 + wg), 0, p.ws_status);
    }
  } else if (warp == WARP_CTL || (NCW == 2 && warp == WARP_CTL + 1)) {
    // NCW = 0: the sequential controller of a single-CTA cluster; 1 or 2: the scan controller of a
    // cluster on one warp (one pass over the heads) or two (half of the heads each)
    // ------------------------------------------------------------ ART controller(s)
    const int TQ = C * KT;    // tiles per round (power of two <= 32)
    const int HPP = 32 / TQ;  // heads per pass
    const int cw = (NCW == 0) ? 0 : warp - WARP_CTL;  // NCW 2: which half of the heads
    if constexpr (ART && NCW == 0) {
      // Single-CTA cluster: a round is this CTA's KT tiles, replayed one after another.  Head g
      // owns LPH lanes holding CPL probe lanes each; its carried state (m, l, probe accumulators,
      // previous probe and norm, run) lives in registers across rounds.  Norms and the direction
      // change are reduced over the head's lanes with xor shuffles.
      constexpr int LPH = (32 / GP) < PC ? (32 / GP) : PC;
      constexpr int CPL = PC / LPH;
      const int g = lane / LPH, j = lane % LPH;
      const bool active = g < G;
      const int gs = active ? g : 0;
      float m = -INFINITY, l = 0.f, nrmp = 0.f, a[CPL], xp[CPL];
#pragma unroll
      for (int k = 0; k < CPL; ++k) a[k] = xp[k] = 0.f;
      int run = 0;
      bool stopped = !active;
      auto group_sum = [&](float v) {
#pragma unroll
        for (int o = LPH / 2; o >= 1; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        return v;
      };
#pragma unroll 1
      for (int r = 0; r < R; ++r) {
        const int sl = r % NSLOT;
        int okw = 1;
        if (lane == 0) okw = wait_phase(bar(B_XFULL + sl), (r / NSLOT) & 1, ctl, false, p.ws_status, false);
        if (!__shfl_sync(0xffffffffu, okw, 0)) break;
        const int nv = max(0, min(KT, t1 - (t0 + r * KT)));
        const float* ps = pub + sl * (PB::SLOT / 4);
        const bool was_stopped = stopped;
        int stop_q = -1;
#pragma unroll 1
        for (int q = 0; q < nv; ++q) {
          const int e = q * GP + gs;
          const float mt = ps[e], lt = ps[PB::OFF_L + e];
          float at[CPL];
#pragma unroll
          for (int k = 0; k < CPL; ++k) at[k] = ps[PB::OFF_X + e * PC + j * CPL + k];
          const float M = fmaxf(m, mt);
          const float al = rescale_fast(m, M), be = rescale_fast(mt, M);
          const float nl = al * l + be * lt;
          const float inv_l = __fdividef(1.f, nl);
          float na[CPL], x[CPL], sq = 0.f;
#pragma unroll
          for (int k = 0; k < CPL; ++k) {
            na[k] = al * a[k] + be * at[k];
            x[k] = na[k] * inv_l;
            sq = fmaf(x[k], x[k], sq);
          }
          const float nrm = __fsqrt_rn(group_sum(sq));
          const bool both = nrm > 0.f && nrmp > 0.f;
          const float in = both ? __fdividef(1.f, nrm) : 0.f, ip = both ? __fdividef(1.f, nrmp) : 0.f;
          float dq = 0.f;
#pragma unroll
          for (int k = 0; k < CPL; ++k) {
            const float dl = x[k] * in - xp[k] * ip;
            dq = fmaf(dl, dl, dq);
          }
          const float dd2 = group_sum(dq);
          const float d_scale = fabsf(nrm - nrmp);
          const float d_dir = (nrm == 0.f && nrmp == 0.f) ? 0.f : ((nrm == 0.f || nrmp == 0.f) ? 1.f : 0.5f * dd2);
          const bool hold = (d_scale < p.eps_scale) && (d_dir < p.eps_dir);
          if (!stopped) {  // a stopped head keeps its state (it still takes part in the shuffles)
            m = M;
            l = nl;
            nrmp = nrm;
#pragma unroll
            for (int k = 0; k < CPL; ++k) {
              a[k] = na[k];
              xp[k] = x[k];
            }
            run = hold ? run + 1 : 0;
            if (run >= p.patience) {
              stopped = true;
              stop_q = q;
            }
          }
        }
        if (active && j == 0) {
          dec[sl * GMAX + g] = was_stopped ? -2 : stop_q;
          if (stop_q >= 0) {
            ri[g * RI_SIZE + RI_STOPPED] = 1;
            ri[g * RI_SIZE + RI_USED] = r * KT + stop_q + 1;
          }
        }
        const bool all = __ballot_sync(0xffffffffu, active && !stopped) == 0u;
        // the safe point: tiles decided so far plus what the head farthest from stopping still needs
        const int rem = __reduce_max_sync(0xffffffffu, (active && !stopped) ? p.patience - run : 0);
        __syncwarp();
        if (lane == 0) {
          ctl[CTL_SAFE] = all ? kNothingSafe : min(ns, (r + 1) * KT + rem);
          ctl[CTL_DECIDED] = r + 1;
          __threadfence_block();
          mbar_arrive(bar(B_DEC + sl));
          if (all) {
            ctl[CTL_EXIT_ROUND] = r;
            __threadfence_block();
            ctl[CTL_EXIT] = 1;
          }
        }
        __syncwarp();
        if (all) break;
      }
    } else if constexpr (ART && NCW >= 1) {
      // Scan controller: lane (hh, q) takes tile q of the round for head g0 + hh.
      const int hh = lane / TQ, q = lane % TQ;
      const int c = q / KT, i = q % KT;
      const int seg0 = hh * TQ;  // first lane of this head's segment
      const unsigned segmask = (TQ == 32) ? 0xffffffffu : ((1u << TQ) - 1u);
      const bool remote = C > 1;  // the tile's publication lives in CTA c of the cluster
      const uint32_t pub_c = remote ? map_to_rank(smem_u32(pub), c) : smem_u32(pub);
      ART_DCHECK(c < C && TQ <= 32 && (32 % TQ) == 0, p.ws_status);
      // The part of a round that needs no earlier round: this lane's tile (m, l, probe) from the CTA
      // that computed it (tiles at or past nv stay empty) ...  The probe lanes are held as pairs:
      // the arithmetic below runs on packed f32x2 instructions.
      auto load_tile = [&](uint32_t slot, bool valid, int g, float& m, float& l, float2 (&a)[PC / 2]) {
        m = -INFINITY;
        l = 0.f;
#pragma unroll
        for (int k = 0; k < PC / 2; ++k) a[k] = make_float2(0.f, 0.f);
        if (valid) {
          const uint32_t e = static_cast<uint32_t>(i * GP + g);
          m = ld_smem_f32(slot + 4 * e, remote);
          l = ld_smem_f32(slot + 4 * (PB::OFF_L + e), remote);
          const uint32_t px = slot + 4 * (PB::OFF_X + e * PC);
#pragma unroll
          for (int k = 0; k < PC; k += 4) {
            const float4 v = ld_smem_v4(px + 4 * k, remote);
            a[k / 2] = make_float2(v.x, v.y);
            a[k / 2 + 1] = make_float2(v.z, v.w);
          }
        }
      };
      // ... merged with the round's earlier tiles of the same head: an inclusive scan over the head's
      // segment of TQ lanes.
      auto scan_tiles = [&](float& m, float& l, float2 (&a)[PC / 2]) {
        // a loop, not unrolled: the controller's instruction footprint costs more than the loop
#pragma unroll 1
        for (int off = 1; off < TQ; off <<= 1) {
          const float mo = __shfl_up_sync(0xffffffffu, m, off, TQ);
          const float lo = __shfl_up_sync(0xffffffffu, l, off, TQ);
          const bool take = q >= off;
          const float M = fmaxf(m, mo);
          const float cs = take ? rescale_fast(m, M) : 1.f;
          const float co = take ? rescale_fast(mo, M) : 0.f;
          l = cs * l + co * lo;
          m = take ? M : m;
          const float2 cs2 = make_float2(cs, cs), co2 = make_float2(co, co);
#pragma unroll
          for (int k = 0; k < PC / 2; ++k) {
            const float2 ao = make_float2(__shfl_up_sync(0xffffffffu, a[k].x, off, TQ),
                                          __shfl_up_sync(0xffffffffu, a[k].y, off, TQ));
            a[k] = __ffma2_rn(cs2, a[k], __fmul2_rn(co2, ao));
          }
        }
      };
      // The part that needs the state carried over from earlier rounds: prepend it, evaluate the rule
      // at every tile of the round, find the stop, and carry the state of the head's last replayed
      // tile (the stop, or the round's last tile) into the next round.
      auto replay_round = [&](int r, int sl, int nv, int g, float m, float l, float2 (&a)[PC / 2]) {
        const bool active = g < G;
        const int gs = active ? g : 0;
        float* R_f = rf + gs * RF_SIZE;
        int* R_i = ri + gs * RI_SIZE;
        const bool stopped_before = !active || R_i[RI_STOPPED] != 0;
        const bool valid = !stopped_before && q < nv;
        const float4 st = *reinterpret_cast<const float4*>(R_f);  // m, l, |x_prev|, -
        const float mR = st.x, lR = st.y;
        const float Mf = fmaxf(mR, m);
        const float aR = rescale_fast(mR, Mf), aS = rescale_fast(m, Mf);
        l = aR * lR + aS * l;
        m = Mf;
        const float inv_l = __fdividef(1.f, l);
        const float2 aR2 = make_float2(aR, aR), aS2 = make_float2(aS, aS), il2 = make_float2(inv_l, inv_l);
        float2 x[PC / 2], sq[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
        for (int k = 0; k < PC; k += 4) {
          const float4 ar = *reinterpret_cast<const float4*>(R_f + RF_A + k);
          a[k / 2] = __ffma2_rn(aR2, make_float2(ar.x, ar.y), __fmul2_rn(aS2, a[k / 2]));
          a[k / 2 + 1] = __ffma2_rn(aR2, make_float2(ar.z, ar.w), __fmul2_rn(aS2, a[k / 2 + 1]));
          x[k / 2] = __fmul2_rn(a[k / 2], il2);
          x[k / 2 + 1] = __fmul2_rn(a[k / 2 + 1], il2);
          sq[0] = __ffma2_rn(x[k / 2], x[k / 2], sq[0]);
          sq[1] = __ffma2_rn(x[k / 2 + 1], x[k / 2 + 1], sq[1]);
        }
        const float nrm = __fsqrt_rn((sq[0].x + sq[1].x) + (sq[0].y + sq[1].y));
        float nrmp = __shfl_up_sync(0xffffffffu, nrm, 1, TQ);
        if (q == 0) nrmp = st.z;
        const bool both = nrm > 0.f && nrmp > 0.f;
        const float in = both ? __fdividef(1.f, nrm) : 0.f, ip = both ? __fdividef(1.f, nrmp) : 0.f;
        const float2 in2 = make_float2(in, in), nip2 = make_float2(-ip, -ip);
        float2 dq[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
        for (int k = 0; k < PC; k += 4) {
          const float4 xr = *reinterpret_cast<const float4*>(R_f + RF_XP + k);
          const float2 xrv[2] = {make_float2(xr.x, xr.y), make_float2(xr.z, xr.w)};
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            float2 xp = make_float2(__shfl_up_sync(0xffffffffu, x[k / 2 + u].x, 1, TQ),
                                    __shfl_up_sync(0xffffffffu, x[k / 2 + u].y, 1, TQ));
            if (q == 0) xp = xrv[u];
            const float2 dl = __ffma2_rn(x[k / 2 + u], in2, __fmul2_rn(xp, nip2));
            dq[u] = __ffma2_rn(dl, dl, dq[u]);
          }
        }
        const float dd2 = (dq[0].x + dq[1].x) + (dq[0].y + dq[1].y);
        const float d_scale = fabsf(nrm - nrmp);
        const float d_dir = (nrm == 0.f && nrmp == 0.f) ? 0.f : ((nrm == 0.f || nrmp == 0.f) ? 1.f : 0.5f * dd2);
        const bool hold = valid && (d_scale < p.eps_scale) && (d_dir < p.eps_dir);
        // patience, for every tile of the round at once: the run ending at tile q is the number
        // of consecutive holding tiles up to q (plus the carried run when they reach back to the
        // round's first tile); the head stops at the first tile whose run reaches the patience.
        const unsigned hbits = (__ballot_sync(0xffffffffu, hold) >> seg0) & segmask;
        const int run0 = stopped_before ? 0 : R_i[RI_RUN];
        const unsigned zeros = ~hbits & ((1u << q) - 1u);
        const int runq = !((hbits >> q) & 1u) ? 0 : (zeros == 0u ? run0 + q + 1 : q - (31 - __clz(zeros)));
        const bool reach = hold && runq >= p.patience;
        const unsigned rbits = (__ballot_sync(0xffffffffu, reach) >> seg0) & segmask;
        const int stop = (!stopped_before && rbits != 0u) ? __ffs(rbits) - 1 : -1;
        const int srcq = (stop >= 0) ? stop : nv - 1;
        if (active && !stopped_before && nv > 0 && q == srcq) {
          *reinterpret_cast<float4*>(R_f) = make_float4(m, l, nrm, 0.f);
#pragma unroll
          for (int k = 0; k < PC; k += 4) {
            *reinterpret_cast<float4*>(R_f + RF_A + k) = make_float4(a[k / 2].x, a[k / 2].y, a[k / 2 + 1].x, a[k / 2 + 1].y);
            *reinterpret_cast<float4*>(R_f + RF_XP + k) = make_float4(x[k / 2].x, x[k / 2].y, x[k / 2 + 1].x, x[k / 2 + 1].y);
          }
          R_i[RI_RUN] = runq;
          if (stop >= 0) {
            R_i[RI_STOPPED] = 1;
            R_i[RI_USED] = r * TQ + stop + 1;
          }
        }
        if (active && q == 0) dec[sl * GMAX + g] = stopped_before ? -2 : stop;
        __syncwarp();
      };
      if constexpr (NCW == 1) {
        // One warp, one pass over every head per round.  The loads of round r + 1 are issued before
        // round r is replayed whenever every CTA has already published it, so that their latency
        // (distributed shared memory) overlaps the replay.  (Rounds dealt alternately to two warps,
        // each scanning one round while the other replays the previous one, ran several times slower.)
        const int g = hh;
        auto tile_valid = [&](int r) { return g < G && q < t1 - (t0 + r * TQ); };
        float m, l;
        float2 a[PC / 2];
        int okw = 1;
        if (R > 0) {
          if (lane == 0) okw = wait_phase(bar(B_XFULL), 0, ctl, false, p.ws_status, true);
          okw = __shfl_sync(0xffffffffu, okw, 0);
          if (okw) load_tile(pub_c, tile_valid(0), g, m, l, a);
        }
        for (int r = 0; okw && r < R; ++r) {
          const int sl = r % NSLOT;
          const int nv = max(0, min(TQ, t1 - (t0 + r * TQ)));
          scan_tiles(m, l, a);
          const int r1 = r + 1, sl1 = r1 % NSLOT;
          float m1, l1;
          float2 a1[PC / 2];
          int pre = 0;
          if (r1 < R) {
            if (lane == 0) pre = mbar_test_wait_cluster(bar(B_XFULL + sl1), (r1 / NSLOT) & 1);
            pre = __shfl_sync(0xffffffffu, pre, 0);
            if (pre) load_tile(pub_c + sl1 * PB::SLOT, tile_valid(r1), g, m1, l1, a1);
          }
          replay_round(r, sl, nv, g, m, l, a);
          if (lane == 0) {
            bool all = true;
            int rem = 0;  // the safe point, as in the sequential controller
            for (int gg = 0; gg < G; ++gg) {
              const bool sg = ri[gg * RI_SIZE + RI_STOPPED] != 0;
              all &= sg;
              if (!sg) rem = max(rem, p.patience - ri[gg * RI_SIZE + RI_RUN]);
            }
            ctl[CTL_SAFE] = all ? kNothingSafe : min(ns, (r + 1) * TQ + rem);
            ctl[CTL_DECIDED] = r + 1;
            __threadfence_block();
            mbar_arrive(bar(B_DEC + sl));
            if (all) {
              ctl[CTL_EXIT_ROUND] = r;
              __threadfence_block();
              ctl[CTL_EXIT] = 1;
            }
          }
          __syncwarp();
          if (ctl[CTL_EXIT] || r1 >= R) break;
          if (!pre) {
            if (lane == 0) okw = wait_phase(bar(B_XFULL + sl1), (r1 / NSLOT) & 1, ctl, false, p.ws_status, true);
            okw = __shfl_sync(0xffffffffu, okw, 0);
            if (!okw) break;
            load_tile(pub_c + sl1 * PB::SLOT, tile_valid(r1), g, m1, l1, a1);
          }
          m = m1;
          l = l1;
#pragma unroll
          for (int k = 0; k < PC / 2; ++k) a[k] = a1[k];
        }
      } else {
        // Two warps, each replaying half of the heads, round after round.
        for (int r = 0; r < R; ++r) {
          const int sl = r % NSLOT;
          int okw = 1;
          if (lane == 0) okw = wait_phase(bar(B_XFULL + sl), (r / NSLOT) & 1, ctl, false, p.ws_status, true);
          okw = __shfl_sync(0xffffffffu, okw, 0);
          okw = named_barrier_and(BAR_CTL, 64, okw != 0);  // both warps leave together
          if (!okw) break;
          const int nv = max(0, min(TQ, t1 - (t0 + r * TQ)));
          for (int g0 = cw * HPP; g0 < G; g0 += 2 * HPP) {
            const int g = g0 + hh;
            const bool sb = g >= G || ri[g * RI_SIZE + RI_STOPPED] != 0;
            float m, l;
            float2 a[PC / 2];
            load_tile(pub_c + sl * PB::SLOT, !sb && q < nv, g, m, l, a);
            scan_tiles(m, l, a);
            replay_round(r, sl, nv, g, m, l, a);
          }
          // this warp's heads all stopped?  (flags double-buffered by round: the named barrier
          // keeps the two warps within one round of each other)
          if (lane == 0) {
            bool mine = true;
            for (int g0 = cw * HPP; g0 < G; g0 += 2 * HPP)
              for (int gg = g0; gg < min(G, g0 + HPP); ++gg) mine &= (ri[gg * RI_SIZE + RI_STOPPED] != 0);
            ctl[CTL_STOPFLAG + 2 * (r & 1) + cw] = mine ? 1 : 0;
          }
          named_barrier(BAR_CTL, 64);  // both warps' decisions and flags are written
          const bool all = ctl[CTL_STOPFLAG + 2 * (r & 1)] && ctl[CTL_STOPFLAG + 2 * (r & 1) + 1];
          if (cw == 0 && lane == 0) {
            int rem = 0;  // the safe point, as in the sequential controller
            for (int gg = 0; gg < G; ++gg)
              if (ri[gg * RI_SIZE + RI_STOPPED] == 0) rem = max(rem, p.patience - ri[gg * RI_SIZE + RI_RUN]);
            ctl[CTL_SAFE] = all ? kNothingSafe : min(ns, (r + 1) * TQ + rem);
            ctl[CTL_DECIDED] = r + 1;
            __threadfence_block();
            mbar_arrive(bar(B_DEC + sl));
            if (all) {
              ctl[CTL_EXIT_ROUND] = r;
              __threadfence_block();
              ctl[CTL_EXIT] = 1;
            }
          }
          __syncwarp();
          if (all) break;
        }
      }
    }
  }

  __syncthreads();  // (1) every role has left its loop
  // drain: copies that were issued but never consumed still land in shared memory
  if (warp == WARP_TMA && lane == 0) {
    for (int ord = ctl[CTL_CONSUMED]; ord < ctl[CTL_ISSUED]; ++ord) {
      if (Q8)
        drain_wait(bar(B_RAWF + ord % Q8_NRAW), (ord / Q8_NRAW) & 1, p.ws_status);
      else
        drain_wait(bar(B_FULL + ord % NSTG), (ord / NSTG) & 1, p.ws_status);
    }
  }
  __syncthreads();  // (2) the ring is quiet: stage 0 can hold the final reduction
  float* red = reinterpret_cast<float*>(sm + OFF_RED);
  int* redi = reinterpret_cast<int*>(sm + OFF_RED + 4 * RED_I);
  // 1. the CTA's two warpgroup states become one (warpgroup 1 hands its state to warpgroup 0)
  const int er_ = 32 * (warp & 3) + lane;
  if (warp >= WARP_EPI0 + 4 && warp < WARP_EPI0 + 4 * NWG) {  // warpgroup 1 (not the q8 converter)
#pragma unroll
    for (int g = 0; g < GP; ++g)
      if (g < G) red[(GMAX + g) * D + er_] = acc[g];
    if (er_ == 0) {
#pragma unroll
      for (int g = 0; g < GP; ++g) {
        red[RED_M + GMAX + g] = m_own[g];
        red[RED_L + GMAX + g] = l_own[g];
      }
    }
  }
  if (tid == 0) redi[0] = ctl[CTL_TREAD];
  __syncthreads();
  if (warp >= WARP_EPI0 && warp < WARP_EPI0 + 4) {
#pragma unroll
    for (int g = 0; g < GP; ++g) {
      if (g >= G) continue;
      const float m1 = red[RED_M + GMAX + g], l1 = red[RED_L + GMAX + g];
      const float M = fmaxf(m_own[g], m1);
      const float w0 = rescale_fast(m_own[g], M), w1 = rescale_fast(m1, M);
      red[g * D + er_] = w0 * acc[g] + w1 * red[(GMAX + g) * D + er_];
      if (er_ == 0) {
        red[RED_M + g] = M;
        red[RED_L + g] = w0 * l_own[g] + w1 * l1;
      }
    }
  }

  // ---------------------------------------------------------------- cluster merge and output
  // 2. every CTA of the cluster merges a share of the (head, d) outputs over the C states: the
  //    per-rank weights 2^(m_c - M) and the denominators are tabulated once, then each output
  //    element takes C loads from the ranks' shared memory
  if (C > 1) cluster_sync_all(); else __syncthreads();
  const uint32_t rb = smem_u32(red);
  float* wt = red + RED_W;    // [CMAX][GMAX]: the ranks' maxima, then their weights 2^(m_c - M)
  float* lt = red + RED_LT;   // [CMAX][GMAX] the ranks' denominators
  float* mg = red + RED_MG;   // [GMAX] merged max
  float* den = red + RED_DN;  // [GMAX] merged denominator
  if (tid < C * G) {
    const int cc = tid / G, g = tid % G;
    wt[cc * GMAX + g] = (C > 1) ? ld_dsmem_f32(map_to_rank(rb + 4 * (RED_M + g), cc)) : red[RED_M + g];
    lt[cc * GMAX + g] = (C > 1) ? ld_dsmem_f32(map_to_rank(rb + 4 * (RED_L + g), cc)) : red[RED_L + g];
  }
  __syncthreads();
  if (tid < G) {
    float M = -INFINITY;
    for (int cc = 0; cc < C; ++cc) M = fmaxf(M, wt[cc * GMAX + tid]);
    float dsum = 0.f;
    for (int cc = 0; cc < C; ++cc) {
      const float w = rescale_fast(wt[cc * GMAX + tid], M);
      wt[cc * GMAX + tid] = w;
      dsum += w * lt[cc * GMAX + tid];
    }
    mg[tid] = M;
    den[tid] = dsum;
  }
  __syncthreads();
  const int share = (G * D + C - 1) / C;
  for (int idx = rank * share + tid; idx < min(G * D, (rank + 1) * share); idx += NT_) {
    const int g = idx / D, dd = idx % D;
    float num = 0.f;
#pragma unroll 4
    for (int cc = 0; cc < C; ++cc) {
      const float ac = (C > 1) ? ld_dsmem_f32(map_to_rank(rb + 4 * (g * D + dd), cc)) : red[g * D + dd];
      num = fmaf(wt[cc * GMAX + g], ac, num);
    }
    const long long hq = static_cast<long long>(b) * p.Hq + kvh * G + g;
    if (p.S == 1) {
      p.o[hq * D + dd] = bad_len ? __int_as_float(0x7fc00000) : num / den[g];
    } else {
      float* part = p.ws_partial + (hq * p.S + split) * (D + 2);
      if (dd == 0) {
        part[0] = mg[g];
        part[1] = den[g];
      }
      part[2 + dd] = num;
    }
  }
  if (rank == 0) {
    if (tid < G) {
      const long long hq = static_cast<long long>(b) * p.Hq + kvh * G + tid;
      const int used = bad_len ? 0 : (ART ? ri[tid * RI_SIZE + RI_USED] : ns);
      ART_DCHECK(used >= 0 && used <= ns && hq < static_cast<long long>(p.B) * p.Hq, p.ws_status);
      p.ws_used[hq * p.S + split] = used;
      if (p.S == 1 && p.tiles) p.tiles[hq] = used;
    }
    if (tid == 0) {
      int total = 0;
      const uint32_t a = smem_u32(redi);
      for (int cc = 0; cc < C; ++cc) total += (C > 1) ? ld_dsmem_s32(map_to_rank(a, cc)) : redi[0];
      p.ws_tiles_read[(static_cast<long long>(b) * p.Hkv + kvh) * p.S + split] = total;
    }
  }
  if (C > 1) cluster_sync_all();
  if (warp == WARP_MMA) {
    tc_fence_after();
    tmem_dealloc(tmem, LY::TMEM_COLS);
  }
}

}  // namespace tc
}  // namespace artk
