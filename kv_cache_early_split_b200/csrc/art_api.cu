// art_api.cu -- host side of the C ABI declared in include/art_decode.h:
// argument validation, workspace layout, launch configuration (cluster size,
// pipeline depth) and kernel dispatch.  No memory is allocated here.
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>
#include <string.h>

#include <mutex>

#include "art_decode.h"
#include "art_evict.cuh"
#include "art_kernels.cuh"
#include "art_order.cuh"
#include "art_q8_two.cuh"
#include "art_tc_pick.cuh"

namespace {

using artk::Layout;
using artk::Params;

constexpr size_t kWsHeader = 256;  // status word lives at offset 0
constexpr int kMaxDynSmem = 232448;  // 227 KB per block on sm_100
constexpr int kSmemPerSm = 233472;   // 228 KB per SM
constexpr int kSmemReservedPerBlock = 1024;

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Full attention with one caller split may run as up to this many internal splits (same result:
// attention does not depend on how the positions are grouped) when that fills more SMs.
constexpr int kFullSplitsMax = 4;

struct WsLayout {
  size_t tiles_read, used, partial, int_tiles_read, int_used, int_partial, total;
};

bool shape_ok(const art_shape* s) {
  return s && s->B >= 1 && s->Hq >= 1 && s->Hkv >= 1 && s->d >= 1 && s->L_max >= 1 && s->tile >= 1 &&
         s->num_splits >= 1;
}

WsLayout ws_layout(const art_shape* s) {
  WsLayout w;
  const size_t units = size_t(s->B) * s->Hkv * s->num_splits;
  const size_t heads = size_t(s->B) * s->Hq * s->num_splits;
  w.tiles_read = kWsHeader;
  w.used = align256(w.tiles_read + 4 * units);
  w.partial = align256(w.used + 4 * heads);
  // internal splits of full attention (one caller split, up to kFullSplitsMax parts per sequence)
  const size_t iunits = size_t(s->B) * s->Hkv * kFullSplitsMax, iheads = size_t(s->B) * s->Hq * kFullSplitsMax;
  w.int_tiles_read = align256(w.partial + 4 * heads * (size_t(s->d) + 2));
  w.int_used = align256(w.int_tiles_read + 4 * iunits);
  w.int_partial = align256(w.int_used + 4 * iheads);
  w.total = (s->num_splits == 1) ? align256(w.int_partial + 4 * iheads * (size_t(s->d) + 2))
                                 : w.int_tiles_read;
  return w;
}

using KernelFn = void (*)(Params);

struct KernelInfo {
  KernelFn fn;
  Layout (*layout)(int T, int nstage, int C);
  int epc;
};

template <int KIND, int D, int GP, int MODE>
Layout layout_thunk(int T, int nstage, int C) {
  return artk::make_layout<KIND, D, GP>(T, nstage, C);
}

template <int KIND, int D, int GP, int MODE>
KernelInfo info() {
  return KernelInfo{&artk::art_decode_kernel<KIND, D, GP, MODE>, &layout_thunk<KIND, D, GP, MODE>,
                    artk::KvGeom<KIND, D>::EPC};
}

template <int KIND, int D, int MODE>
bool pick_gp(int G, KernelInfo* out) {
  if (G == 1) *out = info<KIND, D, 1, MODE>();
  else if (G == 2) *out = info<KIND, D, 2, MODE>();
  else if (G <= 4) *out = info<KIND, D, 4, MODE>();
  else if (G <= 8) *out = info<KIND, D, 8, MODE>();
  else return false;
  return true;
}

template <int KIND, int MODE>
bool pick_d(int d, int G, KernelInfo* out) {
  if (d == 64) return pick_gp<KIND, 64, MODE>(G, out);
  if (d == 128) return pick_gp<KIND, 128, MODE>(G, out);
  return false;
}

bool pick_kernel(int kind, int mode, int d, int G, KernelInfo* out) {
  using namespace artk;
  if (kind == KV_F32 && mode == MODE_FULL) return pick_d<KV_F32, MODE_FULL>(d, G, out);
  if (kind == KV_F32 && mode == MODE_ART) return pick_d<KV_F32, MODE_ART>(d, G, out);
  if (kind == KV_BF16 && mode == MODE_FULL) return pick_d<KV_BF16, MODE_FULL>(d, G, out);
  if (kind == KV_BF16 && mode == MODE_ART) return pick_d<KV_BF16, MODE_ART>(d, G, out);
  if (kind == KV_Q8 && mode == MODE_SKIP) return pick_d<KV_Q8, MODE_SKIP>(d, G, out);
  if (kind == KV_Q8 && mode == MODE_SKIP_ART) return pick_d<KV_Q8, MODE_SKIP_ART>(d, G, out);
  return false;
}

// Per-device facts and per-kernel attributes, set once.
std::mutex g_mu;
struct DevInfo {
  int sms = 0;
};
DevInfo g_dev[64];
struct AttrEntry {
  KernelFn fn;
  int device;
};
AttrEntry g_attr[512];
int g_attr_n = 0;

art_status prepare(KernelFn fn, int* sms) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return ART_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_dev[dev].sms == 0) {
    int v = 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return ART_ERR_CUDA;
    g_dev[dev].sms = v;
  }
  *sms = g_dev[dev].sms;
  for (int i = 0; i < g_attr_n; ++i)
    if (g_attr[i].fn == fn && g_attr[i].device == dev) return ART_OK;
  if (cudaFuncSetAttribute(reinterpret_cast<const void*>(fn), cudaFuncAttributeMaxDynamicSharedMemorySize,
                           kMaxDynSmem) != cudaSuccess)
    return ART_ERR_CUDA;
  if (cudaFuncSetAttribute(reinterpret_cast<const void*>(fn), cudaFuncAttributeNonPortableClusterSizeAllowed, 1) !=
      cudaSuccess)
    return ART_ERR_CUDA;
  if (g_attr_n < 512) g_attr[g_attr_n++] = AttrEntry{fn, dev};
  return ART_OK;
}

struct LaunchCfg {
  int C, nstage;
  uint32_t smem;
};

struct OccEntry {
  KernelFn fn;
  int device, tile, nstage, per_sm;
};
OccEntry g_occ[1024];
int g_occ_n = 0;

// Pipeline depth and resident CTAs per SM for a kernel and tile size: prefer
// two resident CTAs per SM with an (at least) three-deep ring, else one CTA
// with the deepest ring that fits.  Occupancy comes from the runtime, so the
// register count of the compiled kernel is taken into account.
bool pick_depth(const KernelInfo& ki, int tile, int* nstage, int* per_sm) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  {
    std::lock_guard<std::mutex> lock(g_mu);
    for (int i = 0; i < g_occ_n; ++i)
      if (g_occ[i].fn == ki.fn && g_occ[i].device == dev && g_occ[i].tile == tile) {
        *nstage = g_occ[i].nstage;
        *per_sm = g_occ[i].per_sm;
        return *nstage > 0;
      }
  }
  int best_ns = 0, best_occ = 0;
  for (int ns = 4; ns >= 2; --ns) {
    const Layout L = ki.layout(tile, ns, artk::CMAX);
    if (L.total > static_cast<uint32_t>(kMaxDynSmem)) continue;
    int occ = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, ki.fn, artk::NT, L.total) != cudaSuccess) return false;
    if (occ < 1) continue;
    const bool better = (best_ns == 0) || (occ >= 2 && best_occ < 2 && ns >= 3);
    if (better) {
      best_ns = ns;
      best_occ = occ;
    }
  }
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_occ_n < 1024) g_occ[g_occ_n++] = OccEntry{ki.fn, dev, tile, best_ns, best_occ};
  *nstage = best_ns;
  *per_sm = best_occ;
  return best_ns > 0;
}

// Cluster size: fill the GPU in one wave -- the largest power-of-two C with
// units*C no more than the resident-CTA count (and no more CTAs than tiles).
bool choose_config(const KernelInfo& ki, const art_shape* s, int sms, int max_tiles_per_split, LaunchCfg* out) {
  const int units = s->B * s->Hkv * s->num_splits;
  int nstage = 0, per_sm = 0;
  if (!pick_depth(ki, s->tile, &nstage, &per_sm)) return false;
  const int target = sms * (per_sm > 2 ? 2 : per_sm);
  int C = 1;
  while (C < artk::CMAX && units * (2 * C) <= target && 2 * C <= max_tiles_per_split) C *= 2;
  // shrink the cluster until every cluster of the grid is resident at once (one wave): a cluster of
  // C CTAs needs C free SMs in one GPC, so large clusters can leave a tail wave behind
  while (C > 1) {
    cudaLaunchConfig_t lc;
    memset(&lc, 0, sizeof lc);
    cudaLaunchAttribute attr[1];
    lc.gridDim = dim3(static_cast<unsigned>(units * C), 1, 1);
    lc.blockDim = dim3(artk::NT, 1, 1);
    lc.dynamicSmemBytes = ki.layout(s->tile, nstage, C).total;
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = C;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    lc.attrs = attr;
    lc.numAttrs = 1;
    int nclusters = 0;
    if (cudaOccupancyMaxActiveClusters(&nclusters, ki.fn, &lc) == cudaSuccess && nclusters >= units) break;
    cudaGetLastError();  // clear a sticky-free query error
    C /= 2;
  }
  out->C = C;
  out->nstage = nstage;
  out->smem = ki.layout(s->tile, nstage, C).total;
  return true;
}

art_status validate_params(const art_params* a, int d, int epc, int* emask);

// ---------------------------------------------------------------------------
// Tensor-core path: bf16 K/V, d = 128, tile 64 or 128, up to 8 heads per kv head.
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
std::mutex g_enc_mu;
EncodeTiledFn g_encode = nullptr;

EncodeTiledFn encode_fn() {
  std::lock_guard<std::mutex> lock(g_enc_mu);
  if (!g_encode) {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult qr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &qr) != cudaSuccess ||
        qr != cudaDriverEntryPointSuccess || !fn)
      return nullptr;
    g_encode = reinterpret_cast<EncodeTiledFn>(fn);
  }
  return g_encode;
}

bool tc_eligible(int kind, int mode, const art_shape* s, const art_paged_kv* pg = nullptr) {
  const int G = s->Hq / s->Hkv;
  if (kind == artk::KV_Q8)  // q8: 3 or 4 heads per kv head, contiguous cache, natural order
    return (mode == artk::MODE_SKIP || mode == artk::MODE_SKIP_ART) && s->d == 128 &&
           (s->tile == 64 || s->tile == 128) && (G == 3 || G == 4) && !pg && s->L_max % 2 == 0;
  return kind == artk::KV_BF16 && (mode == artk::MODE_FULL || mode == artk::MODE_ART) && s->d == 128 &&
         (s->tile == 64 || s->tile == 128) && G >= 1 && G <= 8 && (!pg || pg->page_size % 64 == 0);
}

// q8 codes [B*Hkv][L_max][128] (bytes) as a 3-D tensor map, box 128 bytes x 128 rows, no swizzle.
bool make_q8_code_map(CUtensorMap* m, const void* base, const art_shape* s) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[3] = {128, static_cast<cuuint64_t>(s->L_max), static_cast<cuuint64_t>(s->B) * s->Hkv};
  const cuuint64_t strides[2] = {128, static_cast<cuuint64_t>(s->L_max) * 128};
  const cuuint32_t box[3] = {128, 128, 1};
  const cuuint32_t es[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// q8 codes [B*Hkv][L_max][128] for the two-pass tensor-core path: box 128 bytes x 32 rows, 128-byte
// swizzle (two row groups of the MMA per copy).
bool make_q8_group_map(CUtensorMap* m, const void* base, const art_shape* s) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[3] = {128, static_cast<cuuint64_t>(s->L_max), static_cast<cuuint64_t>(s->B) * s->Hkv};
  const cuuint64_t strides[2] = {128, static_cast<cuuint64_t>(s->L_max) * 128};
  const cuuint32_t box[3] = {128, artk::q8two::mma16::STEP, 1};
  const cuuint32_t es[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// q8 scales [B*Hkv][L_max][4] fp16 viewed as [B*Hkv][L_max/2][16 bytes] (two rows per 16 bytes),
// box 16 bytes x 64: the scales of 128 positions (L_max even).
bool make_q8_scale_map(CUtensorMap* m, const void* base, const art_shape* s) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[3] = {16, static_cast<cuuint64_t>(s->L_max / 2), static_cast<cuuint64_t>(s->B) * s->Hkv};
  const cuuint64_t strides[2] = {16, static_cast<cuuint64_t>(s->L_max) * 8};
  const cuuint32_t box[3] = {16, 64, 1};
  const cuuint32_t es[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// A bf16 page pool [num_pages*Hkv][page_size][128] as a 3-D tensor map; box = 64 d x 64 positions.
bool make_pool_map(CUtensorMap* m, const void* base, const art_shape* s, const art_paged_kv* pg) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[3] = {128, static_cast<cuuint64_t>(pg->page_size),
                              static_cast<cuuint64_t>(pg->num_pages) * s->Hkv};
  const cuuint64_t strides[2] = {256, static_cast<cuuint64_t>(pg->page_size) * 256};
  const cuuint32_t box[3] = {64, 64, 1};
  const cuuint32_t es[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// K/V [B*Hkv][L_max][128] bf16 as a 3-D tensor map; box = 64 d x `rows` positions (128 or 64),
// 128-byte swizzle.
bool make_kv_map(CUtensorMap* m, const void* base, const art_shape* s, unsigned rows = 128) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[3] = {128, static_cast<cuuint64_t>(s->L_max), static_cast<cuuint64_t>(s->B) * s->Hkv};
  const cuuint64_t strides[2] = {256, static_cast<cuuint64_t>(s->L_max) * 256};
  const cuuint32_t box[3] = {64, rows, 1};
  const cuuint32_t es[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

using artk::tc::TcFn;

// The tensor-core kernel for G heads per kv head; ord: a traversal sequence; paged: a paged cache;
// ncw: ART controller warps.
TcFn tc_pick(int mode, int G, int n_probe, bool ord, bool paged, int ncw) {
  const int pc = n_probe <= 16 ? 16 : 32;
  if (G == 1) return artk::tc::kernel_gp1(mode, pc, ord, paged, ncw);
  if (G == 2) return artk::tc::kernel_gp2(mode, pc, ord, paged, ncw);
  if (G <= 4) return artk::tc::kernel_gp4(mode, pc, ord, paged, ncw);
  return artk::tc::kernel_gp8(mode, pc, ord, paged, ncw);
}

// ART controller for cluster size C: 0 (the sequential controller) for a single CTA; else the scan
// controller, on two warps when one round's rule replay needs two or more passes of a warp over the
// heads (a pass covers 32 / (C * tiles per block) heads).
int tc_ncw(int mode, int G, int C, int kt) {
  if (mode != artk::MODE_ART) return 1;
  if (C == 1) return 0;
  const int hpp = 32 / (C * kt);
  return (G + hpp - 1) / hpp >= 2 ? 2 : 1;
}

// kind KV_BF16, or KV_Q8 (mode MODE_SKIP / MODE_SKIP_ART; ks, vs the scales, tau the V-skip threshold)
art_status launch_tc(int kind, int mode, const art_shape* s, const void* q, const void* k, const void* v,
                     const uint16_t* ks, const uint16_t* vs, float tau, const int32_t* seq_lens,
                     const art_params* a, const int32_t* order, float* o, int32_t* tiles, void* ws, void* stream,
                     const art_paged_kv* pg) {
  const int G = s->Hq / s->Hkv;
  const bool q8 = kind == artk::KV_Q8;
  if (q8) mode = (mode == artk::MODE_SKIP_ART) ? artk::MODE_ART : artk::MODE_FULL;
  const unsigned nthr = q8 ? artk::tc::Lay<true>::NTHR : artk::tc::Lay<false>::NTHR;
  const uint32_t smem = q8 ? artk::tc::SMEM_BYTES_Q8 : artk::tc::SMEM_BYTES;
  const bool ord = order != nullptr, paged = pg != nullptr;
  const int n_probe = a ? a->n_probe : 0;
  artk::tc::TcParams p;
  memset(&p, 0, sizeof p);
  if (a) {
    int emask = 0;
    const art_status st = validate_params(a, s->d, 8, &emask);
    if (st != ART_OK) return st;
    p.eps_scale = a->eps_scale;
    p.eps_dir = a->eps_dir;
    p.patience = a->patience;
    p.n_probe = a->n_probe;
    p.spec_tiles = a->max_spec_tiles;
    for (int i = 0; i < a->n_probe; ++i) p.lanes[i] = static_cast<int8_t>(a->probe_lanes[i]);
  }
  p.tau = q8 ? tau : 0.f;
  p.log2tau = (q8 && tau > 0.f) ? static_cast<float>(log2(static_cast<double>(tau))) : -INFINITY;
  if (q8) {
    if (!make_q8_code_map(&p.tmK, k, s) || !make_q8_code_map(&p.tmV, v, s) || !make_q8_scale_map(&p.tmK64, ks, s) ||
        !make_q8_scale_map(&p.tmV64, vs, s))
      return ART_ERR_CUDA;
  } else if (pg) {  // the paged path loads 64-position halves from the page pools
    if (!make_pool_map(&p.tmK64, k, s, pg) || !make_pool_map(&p.tmV64, v, s, pg)) return ART_ERR_CUDA;
    p.block_table = pg->block_table;
    p.page_size = pg->page_size;
    p.max_pages = pg->max_pages_per_seq;
    p.num_pages = pg->num_pages;
  } else {
    if (!make_kv_map(&p.tmK, k, s) || !make_kv_map(&p.tmV, v, s)) return ART_ERR_CUDA;
    if (order && s->tile == 64 && (!make_kv_map(&p.tmK64, k, s, 64) || !make_kv_map(&p.tmV64, v, s, 64)))
      return ART_ERR_CUDA;
  }
  p.order = order;
  p.n_max = (s->L_max + s->tile - 1) / s->tile;
  int sms = 0;
  auto pick = [&](int ncw) -> TcFn {
    return q8 ? artk::tc::kernel_q8(mode, n_probe <= 16 ? 16 : 32, ncw) : tc_pick(mode, G, n_probe, ord, paged, ncw);
  };
  art_status st = prepare(reinterpret_cast<KernelFn>(pick(1)), &sms);
  if (st != ART_OK) return st;
  // one CTA per SM; cluster size C: power of two, units*C <= SMs, C*tiles_per_block <= 32 (one rule lane
  // per tile of a round), no more CTAs than 128-position blocks in a split, and every cluster resident
  // at once (a cluster of C CTAs needs C free SMs of one GPC, so large clusters can leave a tail wave)
  const int kt = 128 / s->tile;
  const long long max_tiles = (s->L_max + s->tile - 1) / s->tile;
  struct Pick {
    int C, units;
    TcFn fn;
  };
  auto choose = [&](int S_, Pick* out) -> art_status {
    const int units_ = s->B * s->Hkv * S_;
    const long long max_blocks = ((max_tiles + S_ - 1) / S_ * s->tile + 127) / 128;
    int C_ = 1;
    while (C_ < artk::CMAX && 1LL * units_ * (2 * C_) <= sms && 2 * C_ * kt <= 32 && 2 * C_ <= max_blocks) C_ *= 2;
    TcFn fn_ = nullptr;
    while (true) {
      fn_ = pick(tc_ncw(mode, G, C_, kt));
      const art_status st_ = prepare(reinterpret_cast<KernelFn>(fn_), &sms);
      if (st_ != ART_OK) return st_;
      if (C_ == 1) break;
      cudaLaunchConfig_t lc;
      memset(&lc, 0, sizeof lc);
      cudaLaunchAttribute attr[1];
      lc.gridDim = dim3(static_cast<unsigned>(units_ * C_), 1, 1);
      lc.blockDim = dim3(nthr, 1, 1);
      lc.dynamicSmemBytes = smem;
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = C_;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      lc.attrs = attr;
      lc.numAttrs = 1;
      int nclusters = 0;
      if (cudaOccupancyMaxActiveClusters(&nclusters, fn_, &lc) == cudaSuccess && nclusters >= units_) break;
      cudaGetLastError();
      C_ /= 2;
    }
    *out = Pick{C_, units_, fn_};
    return ART_OK;
  };
  Pick pk;
  st = choose(s->num_splits, &pk);
  if (st != ART_OK) return st;
  // Full attention with one caller split: split each sequence internally when that puts more CTAs to
  // work at once (the combine kernel merges the parts and reports the caller's counters).
  int S_run = s->num_splits;
  // (not for q8: the V skip's running maximum is a property of the split)
  if (mode == artk::MODE_FULL && s->num_splits == 1 && !q8) {
    for (int f = 2; f <= kFullSplitsMax && f <= max_tiles; f *= 2) {
      Pick q2;
      st = choose(f, &q2);
      if (st != ART_OK) return st;
      if (1LL * q2.units * q2.C > 1LL * pk.units * pk.C && 1LL * q2.units * q2.C <= sms) {
        pk = q2;
        S_run = f;
      }
    }
  }
  const int C = pk.C, units = pk.units;
  const TcFn fn = pk.fn;
  const WsLayout w = ws_layout(s);
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  p.q = static_cast<const uint16_t*>(q);
  p.seq_lens = seq_lens;
  p.o = o;
  p.tiles = tiles;
  p.ws_status = reinterpret_cast<int32_t*>(wsb);
  const bool internal = S_run != s->num_splits;  // full attention split internally
  p.ws_tiles_read = reinterpret_cast<int32_t*>(wsb + (internal ? w.int_tiles_read : w.tiles_read));
  p.ws_used = reinterpret_cast<int32_t*>(wsb + (internal ? w.int_used : w.used));
  p.ws_partial = reinterpret_cast<float*>(wsb + (internal ? w.int_partial : w.partial));
  p.B = s->B;
  p.Hq = s->Hq;
  p.Hkv = s->Hkv;
  p.L_max = s->L_max;
  p.T = s->tile;
  p.S = S_run;
  p.G = G;
  p.C = C;
  p.qscale = static_cast<float>(1.4426950408889634 / sqrt(128.0));

  cudaLaunchConfig_t lc;
  memset(&lc, 0, sizeof lc);
  cudaLaunchAttribute attr[1];
  lc.gridDim = dim3(static_cast<unsigned>(units * C), 1, 1);
  lc.blockDim = dim3(nthr, 1, 1);
  lc.dynamicSmemBytes = smem;
  lc.stream = static_cast<cudaStream_t>(stream);
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  lc.attrs = attr;
  lc.numAttrs = 1;
  if (cudaLaunchKernelEx(&lc, fn, p) != cudaSuccess) return ART_ERR_CUDA;
  if (S_run > 1) {
    const int heads = s->B * s->Hq;
    if (internal)  // also the caller's one-split counters
      artk::art_combine_kernel<128><<<(heads + 7) / 8, 256, 0, lc.stream>>>(
          p.ws_partial, p.ws_used, o, tiles, heads, S_run, reinterpret_cast<int32_t*>(wsb + w.used),
          p.ws_tiles_read, reinterpret_cast<int32_t*>(wsb + w.tiles_read), G);
    else
      artk::art_combine_kernel<128><<<(heads + 7) / 8, 256, 0, lc.stream>>>(p.ws_partial, p.ws_used, o, tiles,
                                                                             heads, S_run);
    if (cudaGetLastError() != cudaSuccess) return ART_ERR_CUDA;
  }
  return ART_OK;
}

art_status validate_common(const art_shape* s, const void* q, const void* k, const void* v,
                           const int32_t* seq_lens, const float* o, void* ws, size_t ws_bytes) {
  if (!shape_ok(s)) return ART_ERR_INVALID_ARG;
  if (!q || !k || !v || !seq_lens || !o) return ART_ERR_INVALID_ARG;
  if (s->Hq % s->Hkv != 0) return ART_ERR_INVALID_ARG;
  const int G = s->Hq / s->Hkv;
  if (G > artk::GMAX) return ART_ERR_UNSUPPORTED;
  if (s->d != 64 && s->d != 128) return ART_ERR_UNSUPPORTED;
  if (s->tile != 16 && s->tile != 32 && s->tile != 64 && s->tile != 128 && s->tile != 256) return ART_ERR_UNSUPPORTED;
  auto mis = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) != 0; };
  if (mis(q) || mis(k) || mis(v) || mis(o)) return ART_ERR_INVALID_ARG;
  if (!ws || ws_bytes < art_workspace_bytes(s) || mis(ws)) return ART_ERR_WORKSPACE;
  // index arithmetic stays in 64-bit on the device; keep the grid within limits
  const long long units = 1LL * s->B * s->Hkv * s->num_splits;
  if (units * artk::CMAX > 0x7fffffffLL) return ART_ERR_UNSUPPORTED;
  return ART_OK;
}

art_status validate_paged(const art_shape* s, const art_paged_kv* pg) {
  if (!pg || !pg->block_table || (reinterpret_cast<uintptr_t>(pg->block_table) & 3u)) return ART_ERR_INVALID_ARG;
  if (pg->page_size < 1 || pg->num_pages < 1 || pg->max_pages_per_seq < 1) return ART_ERR_INVALID_ARG;
  if (pg->page_size % s->tile != 0) return ART_ERR_UNSUPPORTED;
  if (1LL * pg->max_pages_per_seq * pg->page_size < s->L_max) return ART_ERR_INVALID_ARG;
  if (1LL * pg->num_pages * s->Hkv * pg->page_size > 0x7fffffffLL) return ART_ERR_UNSUPPORTED;
  return ART_OK;
}

art_status validate_params(const art_params* a, int d, int epc, int* emask) {
  if (!a || !a->probe_lanes) return ART_ERR_INVALID_ARG;
  if (a->n_probe < 1 || a->n_probe > artk::PMAX || a->patience < 1 || a->max_spec_tiles < 0)
    return ART_ERR_INVALID_ARG;
  uint64_t seen[2] = {0, 0};
  *emask = 0;
  for (int i = 0; i < a->n_probe; ++i) {
    const int l = a->probe_lanes[i];
    if (l < 0 || l >= d) return ART_ERR_INVALID_ARG;
    if (seen[l >> 6] & (1ull << (l & 63))) return ART_ERR_INVALID_ARG;
    seen[l >> 6] |= 1ull << (l & 63);
    *emask |= 1 << (l % epc);
  }
  return ART_OK;
}

// The one-pass kernel on the CUDA cores (any dtype, d 64 / 128, a thread-block cluster per split).
art_status launch_cluster(int kind, int mode, const art_shape* s, const void* q, const void* k, const void* v,
                          const uint16_t* ks, const uint16_t* vs, const int32_t* seq_lens, const art_params* a,
                          float tau, float* o, int32_t* tiles, void* ws, void* stream,
                          const int32_t* order = nullptr, const art_paged_kv* pg = nullptr) {
  const int G = s->Hq / s->Hkv;
  KernelInfo ki;
  if (!pick_kernel(kind, mode, s->d, G, &ki)) return ART_ERR_UNSUPPORTED;
  Params p;
  memset(&p, 0, sizeof p);
  p.emask = 0;
  if (a) {
    const art_status st = validate_params(a, s->d, ki.epc, &p.emask);
    if (st != ART_OK) return st;
    p.eps_scale = a->eps_scale;
    p.eps_dir = a->eps_dir;
    p.patience = a->patience;
    p.n_probe = a->n_probe;
    for (int i = 0; i < a->n_probe; ++i) p.lanes[i] = static_cast<int8_t>(a->probe_lanes[i]);
  }
  int sms = 0;
  art_status st = prepare(ki.fn, &sms);
  if (st != ART_OK) return st;
  const int max_tiles = (s->L_max + s->tile - 1) / s->tile;
  const int max_tiles_per_split = (max_tiles + s->num_splits - 1) / s->num_splits;
  LaunchCfg cfg;
  if (!choose_config(ki, s, sms, max_tiles_per_split, &cfg)) return ART_ERR_UNSUPPORTED;

  const WsLayout w = ws_layout(s);
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  p.q = q;
  p.k = k;
  p.v = v;
  p.ks = ks;
  p.vs = vs;
  p.seq_lens = seq_lens;
  p.o = o;
  p.tiles = tiles;
  p.ws_status = reinterpret_cast<int32_t*>(wsb);
  p.ws_tiles_read = reinterpret_cast<int32_t*>(wsb + w.tiles_read);
  p.ws_used = reinterpret_cast<int32_t*>(wsb + w.used);
  p.ws_partial = reinterpret_cast<float*>(wsb + w.partial);
  p.B = s->B;
  p.Hq = s->Hq;
  p.Hkv = s->Hkv;
  p.L_max = s->L_max;
  p.T = s->tile;
  p.S = s->num_splits;
  p.G = G;
  p.C = cfg.C;
  p.nstage = cfg.nstage;
  p.qscale = static_cast<float>(1.4426950408889634 / sqrt(static_cast<double>(s->d)));
  p.tau = tau;
  p.order = order;
  p.n_max = max_tiles;
  if (pg) {
    p.block_table = pg->block_table;
    p.page_size = pg->page_size;
    p.max_pages = pg->max_pages_per_seq;
    p.num_pages = pg->num_pages;
  }

  cudaLaunchConfig_t lc;
  memset(&lc, 0, sizeof lc);
  cudaLaunchAttribute attr[1];
  lc.gridDim = dim3(static_cast<unsigned>(s->B * s->Hkv * s->num_splits * cfg.C), 1, 1);
  lc.blockDim = dim3(artk::NT, 1, 1);
  lc.dynamicSmemBytes = cfg.smem;
  lc.stream = static_cast<cudaStream_t>(stream);
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = cfg.C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  lc.attrs = attr;
  lc.numAttrs = 1;
  if (cudaLaunchKernelEx(&lc, ki.fn, p) != cudaSuccess) return ART_ERR_CUDA;
  if (s->num_splits > 1) {
    const int heads = s->B * s->Hq;
    const dim3 grid((heads + 7) / 8);
    if (s->d == 64)
      artk::art_combine_kernel<64><<<grid, 256, 0, lc.stream>>>(p.ws_partial, p.ws_used, o, tiles, heads,
                                                                 s->num_splits);
    else
      artk::art_combine_kernel<128><<<grid, 256, 0, lc.stream>>>(p.ws_partial, p.ws_used, o, tiles, heads,
                                                                  s->num_splits);
    if (cudaGetLastError() != cudaSuccess) return ART_ERR_CUDA;
  }
  return ART_OK;
}

art_status launch(int kind, int mode, const art_shape* s, const void* q, const void* k, const void* v,
                  const uint16_t* ks, const uint16_t* vs, const int32_t* seq_lens, const art_params* a,
                  float tau, float* o, int32_t* tiles, void* ws, void* stream, const int32_t* order = nullptr,
                  const art_paged_kv* pg = nullptr) {
  if (tc_eligible(kind, mode, s, pg))
    return launch_tc(kind, mode, s, q, k, v, ks, vs, tau, seq_lens, a, order, o, tiles, ws, stream, pg);
  return launch_cluster(kind, mode, s, q, k, v, ks, vs, seq_lens, a, tau, o, tiles, ws, stream, order, pg);
}

// Two-pass q8 decode (full attention with the V skip): the kernels, their workspace arrays (after
// the common ones) and their launch shape live in art_q8_two.cuh.
artk::q8two::Dims q8_dims(const art_shape* s) {
  return artk::q8two::Dims{s->B, s->Hq, s->Hkv, s->d, s->L_max, s->tile, s->num_splits};
}

size_t q8_ws_total(const art_shape* s) { return artk::q8two::workspace_end(q8_dims(s), ws_layout(s).total); }

// Full attention on any shape; ART (the rule over per-tile probe records) on the tensor-core passes.
bool q8two_eligible(const art_shape* s, const art_params* params, size_t ws_bytes) {
  if (params && !artk::q8two::uses_maps(q8_dims(s))) return false;
  return ws_bytes >= q8_ws_total(s) && artk::q8two::grid_ok(q8_dims(s));
}

art_status launch_q8two(const art_shape* s, const void* q, const int8_t* k, const uint16_t* ks, const int8_t* v,
                        const uint16_t* vs, const int32_t* seq_lens, float tau, const art_params* params, float* o,
                        int32_t* tiles, void* ws, void* stream) {
  const WsLayout w = ws_layout(s);
  CUtensorMap tmk, tmv;
  const bool maps = artk::q8two::uses_maps(q8_dims(s));
  if (maps && (!make_q8_group_map(&tmk, k, s) || !make_q8_group_map(&tmv, v, s))) return ART_ERR_CUDA;
  artk::q8two::Rule rule{};
  if (params)
    rule = artk::q8two::Rule{params->n_probe, params->patience, params->eps_scale, params->eps_dir,
                             params->probe_lanes};
  const cudaError_t e = artk::q8two::launch(q8_dims(s), static_cast<const uint16_t*>(q), k, ks, v, vs, seq_lens,
                                            tau, o, tiles, static_cast<uint8_t*>(ws), w.tiles_read, w.used, w.total,
                                            maps ? &tmk : nullptr, maps ? &tmv : nullptr, params ? &rule : nullptr,
                                            static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? ART_OK : ART_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// Scratch memory for art_decode_attn_terminate_noalloc.  The array is a
// file-scope device variable: every GPU that loads this library holds it until
// the process exits.  Host code may not pass the symbol itself to a kernel (on
// the host it only names a stand-in); its device address is looked up once per
// device with cudaGetSymbolAddress while that device is current.
constexpr size_t kNoAllocScratchBytes = size_t(4) << 20;  // 4 MiB
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_noalloc_mu;
void* g_noalloc_ptr[64] = {};

// Device address of g_noalloc_scratch on the current device (set up on first use).
art_status noalloc_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return ART_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return ART_ERR_CUDA;
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return ART_OK;
}

}  // namespace

extern "C" {

size_t art_workspace_bytes(const art_shape* shape) {
  if (!shape_ok(shape)) return 0;
  return ws_layout(shape).total;
}

size_t art_q8_workspace_bytes(const art_shape* shape) {
  if (!shape_ok(shape)) return 0;
  return q8_ws_total(shape);
}

size_t art_workspace_vskip_offset(const art_shape* shape) {
  if (!shape_ok(shape) || shape->Hq % shape->Hkv != 0) return 0;
  return artk::q8two::layout2(q8_dims(shape), ws_layout(shape).total).vskip;
}

size_t art_workspace_tiles_read_offset(const art_shape* shape) {
  if (!shape_ok(shape)) return 0;
  return ws_layout(shape).tiles_read;
}

size_t art_workspace_split_tiles_offset(const art_shape* shape) {
  if (!shape_ok(shape)) return 0;
  return ws_layout(shape).used;
}

art_status art_decode_attn_full(const art_shape* shape, art_dtype dtype, const void* q, const void* k,
                                const void* v, const int32_t* seq_lens, float* o, int32_t* tiles, void* ws,
                                size_t ws_bytes, void* stream) {
  art_status st = validate_common(shape, q, k, v, seq_lens, o, ws, ws_bytes);
  if (st != ART_OK) return st;
  if (dtype != ART_F32 && dtype != ART_BF16) return ART_ERR_INVALID_ARG;
  const int kind = dtype == ART_F32 ? artk::KV_F32 : artk::KV_BF16;
  return launch(kind, artk::MODE_FULL, shape, q, k, v, nullptr, nullptr, seq_lens, nullptr, 0.f, o, tiles, ws,
                stream);
}

art_status art_decode_attn_terminate(const art_shape* shape, art_dtype dtype, const void* q, const void* k,
                                     const void* v, const int32_t* seq_lens, const art_params* params, float* o,
                                     int32_t* tiles, void* ws, size_t ws_bytes, void* stream) {
  art_status st = validate_common(shape, q, k, v, seq_lens, o, ws, ws_bytes);
  if (st != ART_OK) return st;
  if (dtype != ART_F32 && dtype != ART_BF16) return ART_ERR_INVALID_ARG;
  if (!params) return ART_ERR_INVALID_ARG;
  const int kind = dtype == ART_F32 ? artk::KV_F32 : artk::KV_BF16;
  return launch(kind, artk::MODE_ART, shape, q, k, v, nullptr, nullptr, seq_lens, params, 0.f, o, tiles, ws,
                stream);
}

// Allocation-free variant of art_decode_attn_terminate: the workspace is the
// library's own device array (g_noalloc_scratch) instead of caller memory.
// Nothing in that array has to start at zero: the kernels write every word
// they later read (the status word is only ever OR-ed into, and this entry
// point has no way to read it back), so no clearing is enqueued.
art_status art_decode_attn_terminate_noalloc(const art_shape* shape, art_dtype dtype, const void* q,
                                             const void* k, const void* v, const int32_t* seq_lens,
                                             const art_params* params, float* o, int32_t* tiles,
                                             void* stream) {
  if (!shape_ok(shape)) return ART_ERR_INVALID_ARG;
  if (art_workspace_bytes(shape) > kNoAllocScratchBytes) return ART_ERR_WORKSPACE;
  void* scratch = nullptr;  // looking the address up enqueues no work
  const art_status sst = noalloc_scratch(&scratch);
  if (sst != ART_OK) return sst;
  return art_decode_attn_terminate(shape, dtype, q, k, v, seq_lens, params, o, tiles, scratch,
                                   kNoAllocScratchBytes, stream);
}

art_status art_decode_attn_q8_skipv_path(const art_shape* shape, const void* q_bf16, const int8_t* k_q,
                                         const uint16_t* k_scale_f16, const int8_t* v_q,
                                         const uint16_t* v_scale_f16, const int32_t* seq_lens, float tau,
                                         const art_params* params, float* o, int32_t* tiles, void* ws,
                                         size_t ws_bytes, int32_t path, void* stream) {
  art_status st = validate_common(shape, q_bf16, k_q, v_q, seq_lens, o, ws, ws_bytes);
  if (st != ART_OK) return st;
  if (!k_scale_f16 || !v_scale_f16) return ART_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(k_scale_f16) & 15u) || (reinterpret_cast<uintptr_t>(v_scale_f16) & 15u))
    return ART_ERR_INVALID_ARG;
  if (isnan(tau)) return ART_ERR_INVALID_ARG;
  if (path < ART_Q8_AUTO || path > ART_Q8_CLUSTER) return ART_ERR_INVALID_ARG;
  const long long scale_row_bytes = (shape->d / 32) * 2;
  if ((1LL * shape->L_max * scale_row_bytes) % 16 != 0) return ART_ERR_UNSUPPORTED;
  const int mode = params ? artk::MODE_SKIP_ART : artk::MODE_SKIP;
  if (params) {
    int emask = 0;
    st = validate_params(params, shape->d, 8, &emask);
    if (st != ART_OK) return st;
  }
  const bool tc = tc_eligible(artk::KV_Q8, mode, shape);
  const bool two = q8two_eligible(shape, params, ws_bytes);
  if (path == ART_Q8_TENSOR_CORE && !tc) return ART_ERR_UNSUPPORTED;
  if (path == ART_Q8_TWO_PASS && !two) return ART_ERR_UNSUPPORTED;
  // automatic choice: two streaming passes when the workspace allows (full attention on every
  // shape, ART on the tensor-core passes: the fastest q8 paths), else the tensor-core decode kernel,
  // else the cluster kernel
  if (path == ART_Q8_TWO_PASS || (path == ART_Q8_AUTO && two))
    return launch_q8two(shape, q_bf16, k_q, k_scale_f16, v_q, v_scale_f16, seq_lens, tau, params, o, tiles, ws,
                        stream);
  if (path == ART_Q8_TENSOR_CORE || (path == ART_Q8_AUTO && tc))
    return launch_tc(artk::KV_Q8, mode, shape, q_bf16, k_q, v_q, k_scale_f16, v_scale_f16, tau, seq_lens, params,
                     nullptr, o, tiles, ws, stream, nullptr);
  // the one-pass cluster kernel on the CUDA cores
  KernelInfo ki;
  if (!pick_kernel(artk::KV_Q8, mode, shape->d, shape->Hq / shape->Hkv, &ki)) return ART_ERR_UNSUPPORTED;
  return launch_cluster(artk::KV_Q8, mode, shape, q_bf16, k_q, v_q, k_scale_f16, v_scale_f16, seq_lens, params,
                        tau, o, tiles, ws, stream);
}

art_status art_decode_attn_q8_skipv(const art_shape* shape, const void* q_bf16, const int8_t* k_q,
                                    const uint16_t* k_scale_f16, const int8_t* v_q, const uint16_t* v_scale_f16,
                                    const int32_t* seq_lens, float tau, const art_params* params, float* o,
                                    int32_t* tiles, void* ws, size_t ws_bytes, void* stream) {
  return art_decode_attn_q8_skipv_path(shape, q_bf16, k_q, k_scale_f16, v_q, v_scale_f16, seq_lens, tau, params, o,
                                       tiles, ws, ws_bytes, ART_Q8_AUTO, stream);
}

art_status art_decode_attn_terminate_ordered(const art_shape* shape, art_dtype dtype, const void* q,
                                             const void* k, const void* v, const int32_t* seq_lens,
                                             const art_params* params, const int32_t* tile_order, float* o,
                                             int32_t* tiles, void* ws, size_t ws_bytes, void* stream) {
  art_status st = validate_common(shape, q, k, v, seq_lens, o, ws, ws_bytes);
  if (st != ART_OK) return st;
  if (dtype != ART_F32 && dtype != ART_BF16) return ART_ERR_INVALID_ARG;
  if (!params || !tile_order || (reinterpret_cast<uintptr_t>(tile_order) & 3u)) return ART_ERR_INVALID_ARG;
  const int kind = dtype == ART_F32 ? artk::KV_F32 : artk::KV_BF16;
  return launch(kind, artk::MODE_ART, shape, q, k, v, nullptr, nullptr, seq_lens, params, 0.f, o, tiles, ws,
                stream, tile_order);
}

art_status art_decode_attn_paged(const art_shape* shape, art_dtype dtype, const void* q, const void* k_pages,
                                 const void* v_pages, const art_paged_kv* pages, const int32_t* seq_lens,
                                 const art_params* params, const int32_t* tile_order, float* o, int32_t* tiles,
                                 void* ws, size_t ws_bytes, void* stream) {
  art_status st = validate_common(shape, q, k_pages, v_pages, seq_lens, o, ws, ws_bytes);
  if (st != ART_OK) return st;
  if (dtype != ART_F32 && dtype != ART_BF16) return ART_ERR_INVALID_ARG;
  st = validate_paged(shape, pages);
  if (st != ART_OK) return st;
  if (tile_order && (!params || (reinterpret_cast<uintptr_t>(tile_order) & 3u))) return ART_ERR_INVALID_ARG;
  const int kind = dtype == ART_F32 ? artk::KV_F32 : artk::KV_BF16;
  return launch(kind, params ? artk::MODE_ART : artk::MODE_FULL, shape, q, k_pages, v_pages, nullptr, nullptr,
                seq_lens, params, 0.f, o, tiles, ws, stream, tile_order, pages);
}

art_status art_decode_attn_q8_skipv_paged(const art_shape* shape, const void* q_bf16, const int8_t* k_q_pages,
                                          const uint16_t* k_scale_pages, const int8_t* v_q_pages,
                                          const uint16_t* v_scale_pages, const art_paged_kv* pages,
                                          const int32_t* seq_lens, float tau, const art_params* params, float* o,
                                          int32_t* tiles, void* ws, size_t ws_bytes, void* stream) {
  art_status st = validate_common(shape, q_bf16, k_q_pages, v_q_pages, seq_lens, o, ws, ws_bytes);
  if (st != ART_OK) return st;
  if (!k_scale_pages || !v_scale_pages) return ART_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(k_scale_pages) & 15u) || (reinterpret_cast<uintptr_t>(v_scale_pages) & 15u))
    return ART_ERR_INVALID_ARG;
  if (isnan(tau)) return ART_ERR_INVALID_ARG;
  st = validate_paged(shape, pages);
  if (st != ART_OK) return st;
  // every tile's scale run starts on a 16-byte boundary: page_size * (d/32) * 2 bytes per page slab
  if ((1LL * pages->page_size * (shape->d / 32) * 2) % 16 != 0) return ART_ERR_UNSUPPORTED;
  const int mode = params ? artk::MODE_SKIP_ART : artk::MODE_SKIP;
  return launch(artk::KV_Q8, mode, shape, q_bf16, k_q_pages, v_q_pages, k_scale_pages, v_scale_pages, seq_lens,
                params, tau, o, tiles, ws, stream, nullptr, pages);
}

art_status art_evict_random_select(const art_shape* shape, const int32_t* seq_lens, const uint32_t* rand_keys,
                                   int32_t n_sink, int32_t n_recent, int32_t budget, int32_t* kept,
                                   int32_t* kept_lens, void* stream) {
  if (!shape_ok(shape) || !seq_lens || !rand_keys || !kept || !kept_lens) return ART_ERR_INVALID_ARG;
  if (n_sink < 0 || n_recent < 0 || budget < 1 || 1LL * n_sink + n_recent > budget) return ART_ERR_INVALID_ARG;
  const unsigned grid = static_cast<unsigned>(shape->B) * shape->Hkv;
  artk::evict::evict_select_kernel<<<grid, artk::evict::kSelThreads, 0, static_cast<cudaStream_t>(stream)>>>(
      seq_lens, rand_keys, shape->Hkv, shape->L_max, n_sink, n_recent, budget, kept, kept_lens);
  return cudaGetLastError() == cudaSuccess ? ART_OK : ART_ERR_CUDA;
}

art_status art_evict_compact(const art_shape* shape, art_kv_format format, const void* src,
                             const uint16_t* src_scale, const int32_t* kept, int32_t budget, void* dst,
                             uint16_t* dst_scale, void* stream) {
  if (!shape_ok(shape) || !src || !kept || !dst || budget < 1) return ART_ERR_INVALID_ARG;
  if (format != ART_KV_F32 && format != ART_KV_BF16 && format != ART_KV_Q8) return ART_ERR_INVALID_ARG;
  const bool q8 = format == ART_KV_Q8;
  if (q8 != (src_scale != nullptr) || q8 != (dst_scale != nullptr)) return ART_ERR_INVALID_ARG;
  if (q8 && shape->d % 32 != 0) return ART_ERR_UNSUPPORTED;
  const int esz = format == ART_KV_F32 ? 4 : (format == ART_KV_BF16 ? 2 : 1);
  const int row_bytes = shape->d * esz;
  if (row_bytes % 16 != 0) return ART_ERR_UNSUPPORTED;
  auto mis = [](const void* p, unsigned a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) != 0; };
  if (mis(src, 16) || mis(dst, 16) || (q8 && (mis(src_scale, 4) || mis(dst_scale, 4)))) return ART_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  constexpr int kWarps = 8;
  const dim3 grid(static_cast<unsigned>(shape->B) * shape->Hkv, (budget + kWarps - 1) / kWarps);
  if (grid.y > 65535u) return ART_ERR_UNSUPPORTED;
  artk::evict::evict_compact_kernel<uint4><<<grid, 32 * kWarps, 0, st>>>(
      static_cast<const uint8_t*>(src), kept, shape->L_max, budget, row_bytes, static_cast<uint8_t*>(dst));
  if (q8)
    artk::evict::evict_compact_kernel<uint32_t><<<grid, 32 * kWarps, 0, st>>>(
        reinterpret_cast<const uint8_t*>(src_scale), kept, shape->L_max, budget, (shape->d / 32) * 2,
        reinterpret_cast<uint8_t*>(dst_scale));
  return cudaGetLastError() == cudaSuccess ? ART_OK : ART_ERR_CUDA;
}

art_status art_tile_order_recency(const art_shape* shape, const int32_t* seq_lens, int32_t* tile_order,
                                  void* stream) {
  if (!shape_ok(shape) || !seq_lens || !tile_order) return ART_ERR_INVALID_ARG;
  const int n_max = (shape->L_max + shape->tile - 1) / shape->tile;
  const unsigned grid = static_cast<unsigned>(shape->B) * shape->Hkv;
  artk::ord::tile_order_recency_kernel<<<grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(
      seq_lens, shape->Hkv, shape->L_max, shape->tile, shape->num_splits, n_max, tile_order);
  return cudaGetLastError() == cudaSuccess ? ART_OK : ART_ERR_CUDA;
}

art_status art_tile_key_summary(const art_shape* shape, art_dtype dtype, const void* k, const int32_t* seq_lens,
                                float* summary, void* stream) {
  if (!shape_ok(shape) || !k || !seq_lens || !summary) return ART_ERR_INVALID_ARG;
  if (shape->d != 64 && shape->d != 128) return ART_ERR_UNSUPPORTED;
  const int n_max = (shape->L_max + shape->tile - 1) / shape->tile;
  constexpr int kTilesPerBlock = 8;
  const dim3 grid(static_cast<unsigned>(shape->B) * shape->Hkv, (n_max + kTilesPerBlock - 1) / kTilesPerBlock);
  if (grid.y > 65535u) return ART_ERR_UNSUPPORTED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (dtype == ART_F32)
    artk::ord::tile_key_summary_kernel<float><<<grid, shape->d, 0, st>>>(
        static_cast<const float*>(k), seq_lens, shape->Hkv, shape->L_max, shape->d, shape->tile, n_max,
        kTilesPerBlock, summary);
  else if (dtype == ART_BF16)
    artk::ord::tile_key_summary_kernel<__nv_bfloat16><<<grid, shape->d, 0, st>>>(
        static_cast<const __nv_bfloat16*>(k), seq_lens, shape->Hkv, shape->L_max, shape->d, shape->tile, n_max,
        kTilesPerBlock, summary);
  else
    return ART_ERR_INVALID_ARG;
  return cudaGetLastError() == cudaSuccess ? ART_OK : ART_ERR_CUDA;
}

art_status art_tile_order_importance(const art_shape* shape, art_dtype dtype, const void* q, const float* summary,
                                     const int32_t* seq_lens, int32_t* tile_order, void* stream) {
  if (!shape_ok(shape) || !q || !summary || !seq_lens || !tile_order) return ART_ERR_INVALID_ARG;
  if (shape->Hq % shape->Hkv != 0) return ART_ERR_INVALID_ARG;
  if (dtype != ART_F32 && dtype != ART_BF16) return ART_ERR_INVALID_ARG;
  const int n_max = (shape->L_max + shape->tile - 1) / shape->tile;
  const size_t smem = 4 * (static_cast<size_t>(shape->Hq / shape->Hkv) * shape->d + n_max);
  if (smem > 200 * 1024) return ART_ERR_UNSUPPORTED;
  const unsigned grid = static_cast<unsigned>(shape->B) * shape->Hkv;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (dtype == ART_F32) {
    auto fn = &artk::ord::tile_order_importance_kernel<float>;
    if (smem > 48 * 1024 &&
        cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) != cudaSuccess)
      return ART_ERR_CUDA;
    fn<<<grid, artk::ord::kImpThreads, smem, st>>>(static_cast<const float*>(q), summary, seq_lens, shape->Hq, shape->Hkv,
                                shape->L_max, shape->d, shape->tile, shape->num_splits, n_max, tile_order);
  } else {
    auto fn = &artk::ord::tile_order_importance_kernel<__nv_bfloat16>;
    if (smem > 48 * 1024 &&
        cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) != cudaSuccess)
      return ART_ERR_CUDA;
    fn<<<grid, artk::ord::kImpThreads, smem, st>>>(static_cast<const __nv_bfloat16*>(q), summary, seq_lens, shape->Hq, shape->Hkv,
                                shape->L_max, shape->d, shape->tile, shape->num_splits, n_max, tile_order);
  }
  return cudaGetLastError() == cudaSuccess ? ART_OK : ART_ERR_CUDA;
}

art_status art_read_device_status(void* ws, void* stream) {
  if (!ws) return ART_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int32_t h = 0;
  if (cudaStreamSynchronize(s) != cudaSuccess) return ART_ERR_CUDA;
  if (cudaMemcpyAsync(&h, ws, sizeof h, cudaMemcpyDeviceToHost, s) != cudaSuccess) return ART_ERR_CUDA;
  if (cudaMemsetAsync(ws, 0, sizeof h, s) != cudaSuccess) return ART_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return ART_ERR_CUDA;
  if (h & artk::kStatusSeqLen) return ART_ERR_SEQLEN;
  if (h & artk::kStatusTimeout) return ART_ERR_TIMEOUT;
  if (h & artk::kStatusOrder) return ART_ERR_ORDER;
  if (h & artk::kStatusPage) return ART_ERR_PAGE;
  if (h & artk::kStatusIndex) return ART_ERR_INDEX;
  return ART_OK;
}

const char* art_kernel_name(const art_shape* shape, art_dtype dtype, int32_t kv_q8, int32_t with_art) {
  if (!shape_ok(shape)) return nullptr;
  int kind, mode;
  if (kv_q8) {
    kind = artk::KV_Q8;
    mode = with_art ? artk::MODE_SKIP_ART : artk::MODE_SKIP;
  } else {
    if (dtype != ART_F32 && dtype != ART_BF16) return nullptr;
    kind = dtype == ART_F32 ? artk::KV_F32 : artk::KV_BF16;
    mode = with_art ? artk::MODE_ART : artk::MODE_FULL;
  }
  if (mode == artk::MODE_SKIP && (shape->d == 64 || shape->d == 128) && shape->Hq % shape->Hkv == 0 &&
      shape->Hq / shape->Hkv <= artk::GMAX)  // two passes, given the q8 workspace
    return artk::q8two::uses_maps(q8_dims(shape)) ? "q8_pv_mma_kernel" : "q8_pv_kernel";
  if (mode == artk::MODE_SKIP_ART && shape->Hq % shape->Hkv == 0 && artk::q8two::uses_maps(q8_dims(shape)))
    return "q8_pv_mma_kernel";  // the probe and limited passes, given the q8 workspace
  if (tc_eligible(kind, mode, shape)) return "art_decode_tc_kernel";
  KernelInfo ki;
  if (!pick_kernel(kind, mode, shape->d, shape->Hq / shape->Hkv, &ki)) return nullptr;
  return "art_decode_kernel";
}

const char* art_status_string(art_status status) {
  switch (status) {
    case ART_OK: return "ART_OK";
    case ART_ERR_INVALID_ARG: return "ART_ERR_INVALID_ARG";
    case ART_ERR_UNSUPPORTED: return "ART_ERR_UNSUPPORTED";
    case ART_ERR_WORKSPACE: return "ART_ERR_WORKSPACE";
    case ART_ERR_CUDA: return "ART_ERR_CUDA";
    case ART_ERR_TIMEOUT: return "ART_ERR_TIMEOUT";
    case ART_ERR_SEQLEN: return "ART_ERR_SEQLEN";
    case ART_ERR_ORDER: return "ART_ERR_ORDER";
    case ART_ERR_PAGE: return "ART_ERR_PAGE";
    case ART_ERR_INDEX: return "ART_ERR_INDEX";
  }
  return "ART_ERR_UNKNOWN";
}

}  // extern "C"
