// libsqa C ABI: argument checks, TMA tensor maps, launches.
// The declarations and their contracts are in include/sqa.h.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <algorithm>
#include <climits>
#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <mutex>

#include "sqa.h"
#include "attn_bwd.cuh"
#include "attn_fwd.cuh"
#include "decode.cuh"
#include "gemm.cuh"

// Per-device status word written by kernels whose bounded waits ran out.
__device__ int g_sqa_status;

namespace {

using sqa::AttnCfg;
using sqa::AttnParams;
using sqa::BwdParams;
using sqa::DecodeCfg;
using sqa::DecodeParams;
using sqa::DkdvCfg;
using sqa::DqCfg;
using sqa::GemmCfg;
using sqa::GemmParams;

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

constexpr int kMaxDevices = 64;
constexpr unsigned long long kDefaultWaitNs = 2000000000ull;  // 2 s

struct DeviceState {
  bool ready = false;
  int* status = nullptr;
  int sms = 0;
};

// Attention kernels, one per head size. The template's second argument marks
// the column pairs (of every 8) whose exp2 is evaluated by the FMA-pipe
// polynomial; the rest use the MUFU unit: all-MUFU at d = 64, two eighths at
// d = 128, where the exponentials balance the tensor work.
using AttnKernel = void (*)(const CUtensorMap, const CUtensorMap, const CUtensorMap, const AttnParams);
constexpr int kEmu64 = 0x00, kEmu128 = 0x03;
AttnKernel attn_kernel(int d) {
  return d == 64 ? sqa::attn_fwd_kernel<64, kEmu64> : sqa::attn_fwd_kernel<128, kEmu128>;
}

std::mutex g_mu;
DeviceState g_dev[kMaxDevices];
EncodeTiledFn g_encode = nullptr;
std::atomic<unsigned long long> g_wait_ns{kDefaultWaitNs};

// One-time per-device set-up: status word address, SM count, shared-memory opt-in.
int device_state(DeviceState** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return SQA_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_mu);
  DeviceState& st = g_dev[dev];
  if (!st.ready) {
    if (!g_encode) {
      void* fn = nullptr;
      cudaDriverEntryPointQueryResult q;
      if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault, &q) !=
              cudaSuccess ||
          q != cudaDriverEntryPointSuccess || !fn)
        return SQA_ERR_CUDA;
      g_encode = reinterpret_cast<EncodeTiledFn>(fn);
    }
    if (cudaGetSymbolAddress(reinterpret_cast<void**>(&st.status), g_sqa_status) != cudaSuccess) return SQA_ERR_CUDA;
    if (cudaDeviceGetAttribute(&st.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return SQA_ERR_CUDA;
    if (cudaFuncSetAttribute(attn_kernel(64), cudaFuncAttributeMaxDynamicSharedMemorySize,
                             AttnCfg<64>::SMEM_BYTES) != cudaSuccess ||
        cudaFuncSetAttribute(attn_kernel(128), cudaFuncAttributeMaxDynamicSharedMemorySize,
                             AttnCfg<128>::SMEM_BYTES) != cudaSuccess)
      return SQA_ERR_CUDA;
    {
      // The kernels re-split their registers between warpgroups at run time;
      // the split is only valid for the per-thread count they were built for.
      cudaFuncAttributes a64, a128;
      if (cudaFuncGetAttributes(&a64, attn_kernel(64)) != cudaSuccess ||
          cudaFuncGetAttributes(&a128, attn_kernel(128)) != cudaSuccess)
        return SQA_ERR_CUDA;
      if (a64.numRegs != AttnCfg<64>::REGS_LAUNCH || a128.numRegs != AttnCfg<128>::REGS_LAUNCH)
        return SQA_ERR_UNSUPPORTED;
    }
    if (cudaFuncSetAttribute(sqa::gemm_bf16_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             GemmCfg::SMEM_BYTES) != cudaSuccess ||
        cudaFuncSetAttribute(sqa::bwd_dkdv_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             DkdvCfg<64>::SMEM_BYTES) != cudaSuccess ||
        cudaFuncSetAttribute(sqa::bwd_dkdv_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             DkdvCfg<128>::SMEM_BYTES) != cudaSuccess ||
        cudaFuncSetAttribute(sqa::bwd_dq_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             DqCfg<64>::SMEM_BYTES) != cudaSuccess ||
        cudaFuncSetAttribute(sqa::bwd_dq_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             DqCfg<128>::SMEM_BYTES) != cudaSuccess ||
        cudaFuncSetAttribute(sqa::decode_split_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             DecodeCfg<64>::SMEM_BYTES) != cudaSuccess ||
        cudaFuncSetAttribute(sqa::decode_split_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             DecodeCfg<128>::SMEM_BYTES) != cudaSuccess)
      return SQA_ERR_CUDA;
    st.ready = true;
  }
  *out = &st;
  return SQA_OK;
}

bool aligned16(const void* p) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Tensor maps are cached per process: a map is a pure function of what it is
// encoded from (address, data type, sizes, strides, box, swizzle, promotion),
// so a hit returns exactly the map a fresh encode would, whatever happened to
// the memory in between. Direct-mapped, keyed by all of those inputs; a miss
// encodes and replaces the slot.
struct MapKey {
  uintptr_t base;
  uint32_t dtype, rank, swizzle, promo;
  cuuint64_t dims[5], strides[4];
  cuuint32_t box[5];
  bool operator==(const MapKey& o) const {
    if (base != o.base || dtype != o.dtype || rank != o.rank || swizzle != o.swizzle || promo != o.promo) return false;
    for (uint32_t i = 0; i < rank; ++i)
      if (dims[i] != o.dims[i] || box[i] != o.box[i] || (i + 1 < rank && strides[i] != o.strides[i])) return false;
    return true;
  }
};
struct MapSlot {
  bool used = false;
  MapKey key;
  CUtensorMap map;
};
constexpr int kMapSlots = 256;
std::mutex g_map_mu;
MapSlot g_maps[kMapSlots];

int encode_cached(CUtensorMap* m, CUtensorMapDataType dtype, int rank, const void* base, const cuuint64_t* dims,
                  const cuuint64_t* strides, const cuuint32_t* box, CUtensorMapSwizzle swizzle,
                  CUtensorMapL2promotion promo) {
  MapKey k{};
  k.base = reinterpret_cast<uintptr_t>(base);
  k.dtype = (uint32_t)dtype;
  k.rank = (uint32_t)rank;
  k.swizzle = (uint32_t)swizzle;
  k.promo = (uint32_t)promo;
  uint64_t h = k.base * 0x9E3779B97F4A7C15ull ^ ((uint64_t)k.dtype << 1) ^ ((uint64_t)k.swizzle << 7);
  for (int i = 0; i < rank; ++i) {
    k.dims[i] = dims[i];
    k.box[i] = box[i];
    if (i + 1 < rank) k.strides[i] = strides[i];
    h = (h ^ (dims[i] + 0x1000193ull * box[i] + (i + 1 < rank ? strides[i] : 0))) * 0x100000001B3ull;
  }
  MapSlot& slot = g_maps[(h >> 32) % kMapSlots];
  {
    std::lock_guard<std::mutex> lk(g_map_mu);
    if (slot.used && slot.key == k) {
      *m = slot.map;
      return SQA_OK;
    }
  }
  const cuuint32_t es[5] = {1, 1, 1, 1, 1};
  const CUresult r = g_encode(m, dtype, (cuuint32_t)rank, const_cast<void*>(base), dims, strides, box, es,
                              CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, promo, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return SQA_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_map_mu);
  slot.used = true;
  slot.key = k;
  slot.map = *m;
  return SQA_OK;
}

// Tiled bf16 tensor map with 128-byte swizzle. dims/box innermost first;
// strides in bytes for dims 1..rank-1.
int encode_map(CUtensorMap* m, const void* base, int rank, const cuuint64_t* dims, const cuuint64_t* strides,
               const cuuint32_t* box) {
  return encode_cached(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, base, dims, strides, box,
                       CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B);
}

// Tiled fp32 map over `rows` rows of `cols` floats, `ld` floats apart (ld a
// multiple of 4); boxes of `box_cols` x 1, no swizzle; columns >= cols read as zero.
int encode_rows_f32(CUtensorMap* m, const float* base, long long rows, int cols, int ld, int box_cols) {
  const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)ld * 4};
  const cuuint32_t box[2] = {(cuuint32_t)box_cols, 1};
  return encode_cached(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, base, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_NONE,
                       CU_TENSOR_MAP_L2_PROMOTION_L2_128B);
}

int check_attn_args(const void* q, const void* k, const void* v, const void* out, int B, int N, int H_q, int H_kv,
                    int d, int causal, float scale) {
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return SQA_ERR_INVALID_ARG;
  if (B < 1 || N < 1 || H_q < 1 || H_kv < 1 || H_kv > H_q) return SQA_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return SQA_ERR_INVALID_ARG;
  if (!(scale > 0.0f) || !std::isfinite(scale)) return SQA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return SQA_ERR_UNSUPPORTED;
  // element counts must fit the 64-bit offsets; tensor-map strides < 2^40 bytes
  const long double elems = (long double)B * N * H_q * d;
  if (elems * 2 >= (long double)(1ull << 40)) return SQA_ERR_INVALID_ARG;
  return SQA_OK;
}

// Heads stacked per 128-row tile: the largest power of two (<= 128) dividing
// H_q / H_kv when the groups are even; otherwise one head per tile.
int heads_per_tile(int H_q, int H_kv) {
  if (H_q % H_kv != 0) return 1;
  const int R = H_q / H_kv;
  int P = 1;
  while (P * 2 <= 128 && R % (P * 2) == 0) P *= 2;
  return P;
}

// How one forward call covers its work: `main_items` tile pairs in one launch,
// then (non-causal) the pairs left for a partial last wave as key-split
// clusters of two CTAs, `tail_ctas` of them, one tile (tail_singles) or a whole
// pair per cluster. Non-causal items all cost the same, so the pairs left for a
// partial last wave take about half as long when their keys are split: one
// tile per unit when four CTAs per pair still fit in one wave (more SMs), else
// the whole pair per unit (two tiles per SM keep the exponential unit busier
// than one).
struct AttnPlan {
  long long pairs, n_pairs, n_hb, main_items, tail_ctas;
  int P, log2P, tpt, tail_singles;
};
AttnPlan plan_attn(int sms, int B, int N, int Nk, int H_q, int H_kv, int causal, int BM, int BN) {
  AttnPlan a{};
  a.P = heads_per_tile(H_q, H_kv);
  while ((1 << a.log2P) < a.P) ++a.log2P;
  a.tpt = BM / a.P;
  a.n_pairs = ((long long)N + 2 * a.tpt - 1) / (2 * a.tpt);
  a.n_hb = H_q / a.P;
  a.pairs = a.n_pairs * a.n_hb * B;
  const long long n_kv_all = ((long long)Nk + BN - 1) / BN;
  const long long rem = a.pairs % sms;
  a.main_items = a.pairs;
  if (!causal && rem > 0 && n_kv_all >= 2) {
    if (4 * rem <= sms) {
      a.main_items = a.pairs - rem;
      a.tail_ctas = 4 * rem;
      a.tail_singles = 1;
    } else if (2 * rem <= sms) {
      a.main_items = a.pairs - rem;
      a.tail_ctas = 2 * rem;
    }
  }
  return a;
}

template <int D>
// N query rows at global positions q0 .. q0 + N - 1 against Nk keys (Nk < 0:
// Nk = N, the whole-sequence case).
int launch_attn(const DeviceState* st, const void* q, const void* k, const void* v, void* out, int B, int N, int H_q,
                int H_kv, int causal, float scale, cudaStream_t stream, float* lse = nullptr, int Nk = -1,
                int q0 = 0, int* ready = nullptr) {
  using C = AttnCfg<D>;
  if (Nk < 0) Nk = N;
  const AttnPlan plan = plan_attn(st->sms, B, N, Nk, H_q, H_kv, causal, C::BM, C::BN);
  const int P = plan.P, log2P = plan.log2P, tpt = plan.tpt;
  const long long n_pairs = plan.n_pairs, n_hb = plan.n_hb;
  const long long main_items = plan.main_items, tail_ctas = plan.tail_ctas;
  const int tail_singles = plan.tail_singles;
  if (plan.pairs > INT_MAX || tail_ctas > INT_MAX) return SQA_ERR_INVALID_ARG;

  CUtensorMap tq, tk, tv;
  {
    const cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)H_q, (cuuint64_t)N, (cuuint64_t)B};
    const cuuint64_t strides[3] = {(cuuint64_t)D * 2, (cuuint64_t)H_q * D * 2, (cuuint64_t)N * H_q * D * 2};
    const cuuint32_t box[4] = {64, (cuuint32_t)P, (cuuint32_t)tpt, 1};
    if (int e = encode_map(&tq, q, 4, dims, strides, box)) return e;
  }
  {
    const cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)H_kv, (cuuint64_t)Nk, (cuuint64_t)B};
    const cuuint64_t strides[3] = {(cuuint64_t)D * 2, (cuuint64_t)H_kv * D * 2, (cuuint64_t)Nk * H_kv * D * 2};
    const cuuint32_t box[4] = {64, 1, (cuuint32_t)C::BN, 1};
    if (int e = encode_map(&tk, k, 4, dims, strides, box)) return e;
    if (int e = encode_map(&tv, v, 4, dims, strides, box)) return e;
  }
  AttnParams p;
  p.Nk = Nk;
  p.q0 = q0;
  p.out = reinterpret_cast<__nv_bfloat16*>(out);
  p.B = B;
  p.N = N;
  p.H_q = H_q;
  p.H_kv = H_kv;
  p.P = P;
  p.log2P = log2P;
  p.tpt = tpt;
  p.n_pairs = (int)n_pairs;
  p.n_hb = (int)n_hb;
  p.causal = causal;
  p.scale_log2 = (float)((double)scale * 1.4426950408889634);  // scale * log2(e)
  p.status = st->status;
  p.timeout_ns = g_wait_ns.load();
  p.lse = lse;
  p.ready = ready;
  const AttnKernel kern = attn_kernel(D);
  if (main_items > 0) {
    p.item0 = 0;
    p.singles = 0;
    p.kv_split = 1;
    kern<<<(unsigned)main_items, C::THREADS, C::SMEM_BYTES, stream>>>(tq, tk, tv, p);
    if (cudaGetLastError() != cudaSuccess) return SQA_ERR_CUDA;
  }
  if (tail_ctas > 0) {
    // clusters of two; a programmatic dependent of the main launch, so that it
    // takes SMs as that grid's last wave frees them (it reads nothing it writes)
    p.item0 = (int)main_items;
    p.singles = tail_singles;
    p.kv_split = 2;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)tail_ctas);
    cfg.blockDim = dim3(C::THREADS);
    cfg.dynamicSmemBytes = C::SMEM_BYTES;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = main_items > 0 ? 2 : 1;
    if (cudaLaunchKernelEx(&cfg, kern, tq, tk, tv, p) != cudaSuccess) return SQA_ERR_CUDA;
  }
  return cudaGetLastError() == cudaSuccess ? SQA_OK : SQA_ERR_CUDA;
}

struct GemmOperands {
  const void* x;
  long long M;
  int K;
  int n_w;
  const void* w[3];
  int w_rows[3];
  int N_out;
  int n_y;
  void* y[3];
  int y_cols[3];  // width of each output (its row stride)
  // x written by the kernel launched just before on the same stream: this GEMM
  // is its programmatic dependent and waits per 128-row block on `ready`
  const int* ready = nullptr;
  int ready_per_row = 0;
  int order = 0, order_B = 1, order_TB = 1;   // row-block order (GemmParams)
  int* zero_ptr = nullptr;                    // counters to zero for a later kernel
  int zero_count = 0;
};

int launch_gemm(const DeviceState* st, const GemmOperands& g, cudaStream_t stream) {
  using C = GemmCfg;
  if (g.M > INT_MAX) return SQA_ERR_INVALID_ARG;
  CUtensorMap tx, tw[3];
  {
    const cuuint64_t dims[2] = {(cuuint64_t)g.K, (cuuint64_t)g.M};
    const cuuint64_t strides[1] = {(cuuint64_t)g.K * 2};
    const cuuint32_t box[2] = {64, 128};
    if (int e = encode_map(&tx, g.x, 2, dims, strides, box)) return e;
  }
  GemmParams p;
  p.w_seg_start[0] = 0;
  for (int i = 0; i < 3; ++i) {
    const int idx = i < g.n_w ? i : 0;
    const cuuint64_t dims[2] = {(cuuint64_t)g.K, (cuuint64_t)g.w_rows[idx]};
    const cuuint64_t strides[1] = {(cuuint64_t)g.K * 2};
    const cuuint32_t box[2] = {64, 64};
    if (int e = encode_map(&tw[i], g.w[idx], 2, dims, strides, box)) return e;
    if (i < g.n_w) p.w_seg_start[i + 1] = p.w_seg_start[i] + g.w_rows[i];
  }
  p.M = (int)g.M;
  p.K = g.K;
  p.N_out = g.N_out;
  p.tiles_m = (int)((g.M + C::BM - 1) / C::BM);
  p.tiles_n = (g.N_out + C::BN - 1) / C::BN;
  p.n_seg_w = g.n_w;
  p.n_seg_y = g.n_y;
  p.y_seg_start[0] = 0;
  for (int i = 0; i < 3; ++i) {
    p.y_ptr[i] = reinterpret_cast<__nv_bfloat16*>(i < g.n_y ? g.y[i] : g.y[0]);
    p.y_ld[i] = i < g.n_y ? g.y_cols[i] : g.y_cols[0];
    if (i < g.n_y) p.y_seg_start[i + 1] = p.y_seg_start[i] + g.y_cols[i];
  }
  p.ready = g.ready;
  p.ready_per_row = g.ready_per_row;
  p.order = g.order;
  p.order_B = g.order_B;
  p.order_TB = g.order_TB;
  p.zero_ptr = g.zero_ptr;
  p.zero_count = g.zero_count;
  p.status = st->status;
  p.timeout_ns = g_wait_ns.load();
  const long long tiles = (long long)p.tiles_m * p.tiles_n;
  if (tiles > INT_MAX) return SQA_ERR_INVALID_ARG;
  const int grid = (int)(tiles < st->sms ? tiles : st->sms);
  if (g.ready == nullptr) {
    sqa::gemm_bf16_kernel<<<grid, C::THREADS, C::SMEM_BYTES, stream>>>(tx, tw[0], tw[1], tw[2], p);
    return cudaGetLastError() == cudaSuccess ? SQA_OK : SQA_ERR_CUDA;
  }
  // programmatic dependent of the previous launch on `stream`
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(C::THREADS);
  cfg.dynamicSmemBytes = C::SMEM_BYTES;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, sqa::gemm_bf16_kernel, tx, tw[0], tw[1], tw[2], p) != cudaSuccess) return SQA_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? SQA_OK : SQA_ERR_CUDA;
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// The layer's per-128-row-block counters of stored attention rows.
size_t layer_ready_bytes(int B, int N) { return align256((((size_t)B * N + 127) / 128) * sizeof(int)); }

// lse2 / dsum rows: a multiple of 4 floats so that every row starts 16-byte aligned.
int bwd_row_ld(int N) { return (N + 3) & ~3; }
size_t bwd_vec_bytes(int B, int N, int H_q) { return align256((size_t)B * H_q * bwd_row_ld(N) * 4); }

// Decode work split: the keys of each (b, g, head block) are cut into `splits`
// ranges of whole 64-key tiles. The split count minimises a small cost model:
// waves of the 296 resident CTAs (two per SM on 148 SMs) times the tiles one
// CTA streams plus about three tiles' worth of pipeline fill. Few long CTAs
// when the cache is small (one wave), enough CTAs to fill whole waves when it
// is large. A pure function of the sizes, so the workspace size is too.
struct DecodeSplit {
  int hblocks, splits, tiles_per_split, n_parts, heads_per_cta;
};
DecodeSplit decode_split(int B, int N, int H_q, int H_kv, int d) {
  constexpr long long kResident = 2 * 148;   // decode_split_kernel CTAs resident at once
  constexpr long long kFillTiles = 3;        // pipeline fill of one CTA, in tiles
  DecodeSplit r;
  r.heads_per_cta = 16 * (d == 64 ? DecodeCfg<64>::RB : DecodeCfg<128>::RB);
  const int r_max = (H_q + H_kv - 1) / H_kv;
  r.hblocks = (r_max + r.heads_per_cta - 1) / r.heads_per_cta;
  const long long n_tiles = (N + 63) / 64;
  const long long base = (long long)B * H_kv * r.hblocks;
  // more splits than eight waves' worth only add partials
  const long long s_max = std::max(1LL, std::min(n_tiles, (8 * kResident + base - 1) / base));
  long long best_tps = n_tiles, best_cost = -1;
  for (long long sp = 1; sp <= s_max; ++sp) {
    const long long tps = (n_tiles + sp - 1) / sp;
    const long long ctas = base * ((n_tiles + tps - 1) / tps);
    const long long cost = ((ctas + kResident - 1) / kResident) * (tps + kFillTiles);
    if (best_cost < 0 || cost < best_cost) {
      best_cost = cost;
      best_tps = tps;
    }
  }
  r.tiles_per_split = (int)best_tps;
  r.splits = (int)((n_tiles + best_tps - 1) / best_tps);
  r.n_parts = 4 * r.splits;
  return r;
}

template <int D>
int launch_decode(const DeviceState* st, const void* q, const void* k, const void* v, void* out, void* workspace,
                  int B, int N, int H_q, int H_kv, float scale, cudaStream_t stream) {
  using C = DecodeCfg<D>;
  const DecodeSplit sp = decode_split(B, N, H_q, H_kv, D);
  if ((long long)B * H_kv > 65535 || sp.hblocks > 65535) return SQA_ERR_INVALID_ARG;
  CUtensorMap tk, tv;
  {
    const cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)H_kv, (cuuint64_t)N, (cuuint64_t)B};
    const cuuint64_t strides[3] = {(cuuint64_t)D * 2, (cuuint64_t)H_kv * D * 2, (cuuint64_t)N * H_kv * D * 2};
    const cuuint32_t box[4] = {64, 1, (cuuint32_t)C::BK, 1};
    if (int e = encode_map(&tk, k, 4, dims, strides, box)) return e;
    if (int e = encode_map(&tv, v, 4, dims, strides, box)) return e;
  }
  DecodeParams p;
  p.q = reinterpret_cast<const __nv_bfloat16*>(q);
  p.part = reinterpret_cast<float*>(workspace);
  p.out = reinterpret_cast<__nv_bfloat16*>(out);
  p.B = B;
  p.N = N;
  p.H_q = H_q;
  p.H_kv = H_kv;
  p.splits = sp.splits;
  p.tiles_per_split = sp.tiles_per_split;
  p.n_parts = sp.n_parts;
  p.heads_per_cta = sp.heads_per_cta;
  p.scale_log2 = (float)((double)scale * 1.4426950408889634);
  p.status = st->status;
  p.timeout_ns = g_wait_ns.load();
  const dim3 grid((unsigned)sp.splits, (unsigned)sp.hblocks, (unsigned)(B * H_kv));
  sqa::decode_split_kernel<D><<<grid, C::THREADS, C::SMEM_BYTES, stream>>>(tk, tv, p);
  if (cudaGetLastError() != cudaSuccess) return SQA_ERR_CUDA;
  const long long rows = (long long)B * H_q;
  if (rows > INT_MAX) return SQA_ERR_INVALID_ARG;
  // programmatic dependent launch: the combine's launch overlaps the split's
  // tail; the kernel's griddepcontrol.wait orders it after the split grid
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)rows);
  cfg.blockDim = dim3(128);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, sqa::decode_combine_kernel<D>, p) != cudaSuccess) return SQA_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? SQA_OK : SQA_ERR_CUDA;
}

template <int D>
int launch_attn_bwd(const DeviceState* st, const void* q, const void* k, const void* v, const void* out,
                    const void* dout, const float* lse, void* dq, void* dk, void* dv, void* workspace, int B, int N,
                    int H_q, int H_kv, int causal, float scale, cudaStream_t stream) {
  const int P = heads_per_tile(H_q, H_kv);
  int log2P = 0;
  while ((1 << log2P) < P) ++log2P;
  const int tpt = 128 / P;
  const long long n_kt = ((long long)N + 127) / 128;
  const long long n_qt = ((long long)N + tpt - 1) / tpt;
  const long long n_hb = H_q / P;
  const long long grid_kv = n_kt * H_kv * B, grid_q = n_qt * n_hb * B;
  const long long rows = (long long)B * N * H_q;
  if (grid_kv > INT_MAX || grid_q > INT_MAX || (rows + 7) / 8 > INT_MAX) return SQA_ERR_INVALID_ARG;
  const int ld = bwd_row_ld(N);
  float* lse2 = reinterpret_cast<float*>(workspace);
  float* dsum = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(workspace) + bwd_vec_bytes(B, N, H_q));

  // dK/dV kernel: Q_j, dO_j of 64 queries of one head, K/V tiles of 128 keys;
  // dQ kernel: 128-row stacked Q/dO tiles as in the forward, K_j/V_j of 64 keys.
  CUtensorMap tq1, tdo1, tqP, tdoP, tk128, tv128, tk64, tv64, tl, td;
  {
    const cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)H_q, (cuuint64_t)N, (cuuint64_t)B};
    const cuuint64_t strides[3] = {(cuuint64_t)D * 2, (cuuint64_t)H_q * D * 2, (cuuint64_t)N * H_q * D * 2};
    const cuuint32_t box1[4] = {64, 1, (cuuint32_t)DkdvCfg<D>::BQ, 1};
    const cuuint32_t boxP[4] = {64, (cuuint32_t)P, (cuuint32_t)tpt, 1};
    if (int e = encode_map(&tq1, q, 4, dims, strides, box1)) return e;
    if (int e = encode_map(&tdo1, dout, 4, dims, strides, box1)) return e;
    if (int e = encode_map(&tqP, q, 4, dims, strides, boxP)) return e;
    if (int e = encode_map(&tdoP, dout, 4, dims, strides, boxP)) return e;
  }
  {
    const cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)H_kv, (cuuint64_t)N, (cuuint64_t)B};
    const cuuint64_t strides[3] = {(cuuint64_t)D * 2, (cuuint64_t)H_kv * D * 2, (cuuint64_t)N * H_kv * D * 2};
    const cuuint32_t box128[4] = {64, 1, 128, 1};
    const cuuint32_t box64[4] = {64, 1, (cuuint32_t)DqCfg<D>::BK, 1};
    if (int e = encode_map(&tk128, k, 4, dims, strides, box128)) return e;
    if (int e = encode_map(&tv128, v, 4, dims, strides, box128)) return e;
    if (int e = encode_map(&tk64, k, 4, dims, strides, box64)) return e;
    if (int e = encode_map(&tv64, v, 4, dims, strides, box64)) return e;
  }
  if (int e = encode_rows_f32(&tl, lse2, (long long)B * H_q, N, ld, DkdvCfg<D>::BQ)) return e;
  if (int e = encode_rows_f32(&td, dsum, (long long)B * H_q, N, ld, DkdvCfg<D>::BQ)) return e;

  BwdParams p;
  p.q = reinterpret_cast<const __nv_bfloat16*>(q);
  p.k = reinterpret_cast<const __nv_bfloat16*>(k);
  p.v = reinterpret_cast<const __nv_bfloat16*>(v);
  p.dout = reinterpret_cast<const __nv_bfloat16*>(dout);
  p.dq = reinterpret_cast<__nv_bfloat16*>(dq);
  p.dk = reinterpret_cast<__nv_bfloat16*>(dk);
  p.dv = reinterpret_cast<__nv_bfloat16*>(dv);
  p.nlse2 = lse2;
  p.ndsum = dsum;
  p.ld = ld;
  p.B = B;
  p.N = N;
  p.H_q = H_q;
  p.H_kv = H_kv;
  p.P = P;
  p.log2P = log2P;
  p.tpt = tpt;
  p.n_hb = (int)n_hb;
  p.causal = causal;
  p.scale = scale;
  p.scale_log2 = (float)((double)scale * 1.4426950408889634);
  p.status = st->status;
  p.timeout_ns = g_wait_ns.load();

  sqa::bwd_prep_kernel<D><<<(unsigned)((rows + 7) / 8), 256, 0, stream>>>(
      reinterpret_cast<const __nv_bfloat16*>(out), reinterpret_cast<const __nv_bfloat16*>(dout), lse, dsum, lse2, B,
      N, H_q, ld);
  if (cudaGetLastError() != cudaSuccess) return SQA_ERR_CUDA;
  sqa::bwd_dkdv_kernel<D><<<(unsigned)grid_kv, DkdvCfg<D>::THREADS, DkdvCfg<D>::SMEM_BYTES, stream>>>(
      tq1, tdo1, tk128, tv128, tl, td, p);
  if (cudaGetLastError() != cudaSuccess) return SQA_ERR_CUDA;
  sqa::bwd_dq_kernel<D><<<(unsigned)grid_q, DqCfg<D>::THREADS, DqCfg<D>::SMEM_BYTES, stream>>>(tqP, tdoP, tk64, tv64, p);
  return cudaGetLastError() == cudaSuccess ? SQA_OK : SQA_ERR_CUDA;
}

__global__ void wait_probe_kernel(int* status, unsigned long long ns) {
  __shared__ alignas(8) uint64_t barrier;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    sqa::mbar_init(sqa::smem_u32(&barrier), 1);
    abort_flag = 0;
    sqa::fence_mbar_init();
  }
  __syncthreads();
  sqa::WaitCtl c{&abort_flag, status, ns};
  sqa::mbar_wait_warp(sqa::smem_u32(&barrier), 0, c);  // nothing arrives: must give up
}

// Evaluates the attention kernels' FMA-pipe exp2 (sqa::exp2_poly2, on pairs)
// beside CUDA's exp2f, for checking the polynomial against the library routine.
__global__ void exp2_poly_probe_kernel(const float* x, float* poly, float* ref, long long n) {
  const long long stride = 2LL * gridDim.x * blockDim.x;
  for (long long i = 2LL * (blockIdx.x * (long long)blockDim.x + threadIdx.x); i < n; i += stride) {
    const bool pair = i + 1 < n;
    const float a = x[i], b = pair ? x[i + 1] : a;
    const float2 p = sqa::exp2_poly2(make_float2(a, b));
    poly[i] = p.x;
    ref[i] = exp2f(a);
    if (pair) {
      poly[i + 1] = p.y;
      ref[i + 1] = exp2f(b);
    }
  }
}

// Layer sizes whose every tensor, workspace region and tensor-map stride stays
// below 2^40 bytes, and whose projection widths fit the kernels' int fields.
bool layer_sizes_fit(int B, int N, int d_model, int H_q, int H_kv, int d_head) {
  const long double M = (long double)B * N;
  const long double lim = (long double)(1ull << 40);
  if (M > INT_MAX) return false;
  if ((long double)H_q * d_head + 2.0L * H_kv * d_head > INT_MAX) return false;
  if (M * d_model * 2 >= lim || M * (2.0L * H_q + 2.0L * H_kv) * d_head * 2 >= lim) return false;
  if ((long double)d_model * H_q * d_head * 2 >= lim) return false;
  return true;
}

// Every argument check of the layer entry points, before anything else.
int check_layer_args(const void* x, const void* Wq, const void* Wk, const void* Wv, const void* Wo, const void* out,
                     int B, int N, int d_model, int H_q, int H_kv, int d_head, int causal, float scale) {
  if (!aligned16(x) || !aligned16(Wq) || !aligned16(Wk) || !aligned16(Wv) || !aligned16(Wo) || !aligned16(out))
    return SQA_ERR_INVALID_ARG;
  if (d_model < 8 || d_model % 8 != 0) return SQA_ERR_INVALID_ARG;
  if (B < 1 || N < 1 || H_q < 1 || H_kv < 1 || H_kv > H_q) return SQA_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return SQA_ERR_INVALID_ARG;
  if (!(scale > 0.0f) || !std::isfinite(scale)) return SQA_ERR_INVALID_ARG;
  if (d_head != 64 && d_head != 128) return SQA_ERR_UNSUPPORTED;
  if (!layer_sizes_fit(B, N, d_model, H_q, H_kv, d_head)) return SQA_ERR_INVALID_ARG;
  return SQA_OK;
}

// One thread evaluates a bounds check that fails, with no access behind it:
// records SQA_ERR_BOUNDS where the checks are compiled in (debug builds).
__global__ void bounds_probe_kernel(int* status, int n) {
  const int idx = n;   // one past the end of an n-element range
  sqa::in_bounds(idx < n, status);
}

}  // namespace

extern "C" {

int sqa_attn_fwd(const void* q, const void* k, const void* v, void* out, int B, int N, int H_q, int H_kv, int d_head,
                 int causal, float scale, void* stream) {
  if (int e = check_attn_args(q, k, v, out, B, N, H_q, H_kv, d_head, causal, scale)) return e;
  DeviceState* st = nullptr;
  if (int e = device_state(&st)) return e;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  return d_head == 64 ? launch_attn<64>(st, q, k, v, out, B, N, H_q, H_kv, causal, scale, s)
                      : launch_attn<128>(st, q, k, v, out, B, N, H_q, H_kv, causal, scale, s);
}

int sqa_attn_fwd_lse(const void* q, const void* k, const void* v, void* out, float* lse, int B, int N, int H_q,
                     int H_kv, int d_head, int causal, float scale, void* stream) {
  if (int e = check_attn_args(q, k, v, out, B, N, H_q, H_kv, d_head, causal, scale)) return e;
  if (!aligned16(lse)) return SQA_ERR_INVALID_ARG;
  DeviceState* st = nullptr;
  if (int e = device_state(&st)) return e;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  return d_head == 64 ? launch_attn<64>(st, q, k, v, out, B, N, H_q, H_kv, causal, scale, s, lse)
                      : launch_attn<128>(st, q, k, v, out, B, N, H_q, H_kv, causal, scale, s, lse);
}

int sqa_attn_fwd_rows(const void* q, const void* k, const void* v, void* out, int B, int N_q, int N_k, int q_offset,
                      int H_q, int H_kv, int d_head, int causal, float scale, void* stream) {
  if (N_k < 1 || N_q < 1 || q_offset < 0 || (long long)q_offset + N_q > N_k) return SQA_ERR_INVALID_ARG;
  if (int e = check_attn_args(q, k, v, out, B, N_k, H_q, H_kv, d_head, causal, scale)) return e;
  DeviceState* st = nullptr;
  if (int e = device_state(&st)) return e;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  return d_head == 64
             ? launch_attn<64>(st, q, k, v, out, B, N_q, H_q, H_kv, causal, scale, s, nullptr, N_k, q_offset)
             : launch_attn<128>(st, q, k, v, out, B, N_q, H_q, H_kv, causal, scale, s, nullptr, N_k, q_offset);
}

int sqa_attn_fwd_grids(int B, int N, int H_q, int H_kv, int d_head, int causal) {
  if (B < 1 || N < 1 || H_q < 1 || H_kv < 1 || H_kv > H_q || (causal != 0 && causal != 1)) return 0;
  if (d_head != 64 && d_head != 128) return 0;
  DeviceState* st = nullptr;
  if (device_state(&st) != SQA_OK) return 0;
  const AttnPlan a = d_head == 64 ? plan_attn(st->sms, B, N, N, H_q, H_kv, causal, AttnCfg<64>::BM, AttnCfg<64>::BN)
                                  : plan_attn(st->sms, B, N, N, H_q, H_kv, causal, AttnCfg<128>::BM, AttnCfg<128>::BN);
  return (a.main_items > 0 ? 1 : 0) + (a.tail_ctas > 0 ? 1 : 0);
}

size_t sqa_attn_bwd_workspace_bytes(int B, int N, int H_q) {
  if (B < 1 || N < 1 || H_q < 1) return 0;
  return 2 * bwd_vec_bytes(B, N, H_q);
}

int sqa_attn_bwd(const void* q, const void* k, const void* v, const void* out, const void* dout, const float* lse,
                 void* dq, void* dk, void* dv, void* workspace, size_t workspace_bytes, int B, int N, int H_q,
                 int H_kv, int d_head, int causal, float scale, void* stream) {
  if (int e = check_attn_args(q, k, v, out, B, N, H_q, H_kv, d_head, causal, scale)) return e;
  if (!aligned16(dout) || !aligned16(lse) || !aligned16(dq) || !aligned16(dk) || !aligned16(dv))
    return SQA_ERR_INVALID_ARG;
  const size_t need = sqa_attn_bwd_workspace_bytes(B, N, H_q);
  if (workspace == nullptr || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0 || workspace_bytes < need)
    return SQA_ERR_WORKSPACE;
  DeviceState* st = nullptr;
  if (int e = device_state(&st)) return e;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  return d_head == 64
             ? launch_attn_bwd<64>(st, q, k, v, out, dout, lse, dq, dk, dv, workspace, B, N, H_q, H_kv, causal, scale, s)
             : launch_attn_bwd<128>(st, q, k, v, out, dout, lse, dq, dk, dv, workspace, B, N, H_q, H_kv, causal, scale,
                                    s);
}

size_t sqa_decode_workspace_bytes(int B, int N, int H_q, int H_kv, int d_head) {
  if (B < 1 || N < 1 || H_q < 1 || H_kv < 1 || H_kv > H_q || (d_head != 64 && d_head != 128)) return 0;
  const DecodeSplit sp = decode_split(B, N, H_q, H_kv, d_head);
  return align256((size_t)B * H_q * sp.n_parts * (d_head + 2) * 4);
}

int sqa_decode_fwd(const void* q, const void* k_cache, const void* v_cache, void* out, void* workspace,
                   size_t workspace_bytes, int B, int N, int H_q, int H_kv, int d_head, float scale, void* stream) {
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out)) return SQA_ERR_INVALID_ARG;
  if (B < 1 || N < 1 || H_q < 1 || H_kv < 1 || H_kv > H_q) return SQA_ERR_INVALID_ARG;
  if (!(scale > 0.0f) || !std::isfinite(scale)) return SQA_ERR_INVALID_ARG;
  if (d_head != 64 && d_head != 128) return SQA_ERR_UNSUPPORTED;
  if ((long double)B * N * H_kv * d_head * 2 >= (long double)(1ull << 40)) return SQA_ERR_INVALID_ARG;
  const size_t need = sqa_decode_workspace_bytes(B, N, H_q, H_kv, d_head);
  if (workspace == nullptr || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0 || workspace_bytes < need)
    return SQA_ERR_WORKSPACE;
  DeviceState* st = nullptr;
  if (int e = device_state(&st)) return e;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  return d_head == 64 ? launch_decode<64>(st, q, k_cache, v_cache, out, workspace, B, N, H_q, H_kv, scale, s)
                      : launch_decode<128>(st, q, k_cache, v_cache, out, workspace, B, N, H_q, H_kv, scale, s);
}

size_t sqa_layer_workspace_bytes(int B, int N, int d_model, int H_q, int H_kv, int d_head) {
  if (B < 1 || N < 1 || d_model < 8 || H_q < 1 || H_kv < 1 || H_kv > H_q || d_head < 1) return 0;
  if (!layer_sizes_fit(B, N, d_model, H_q, H_kv, d_head)) return 0;
  const size_t M = (size_t)B * N;
  return align256(M * H_q * d_head * 2) * 2 + align256(M * H_kv * d_head * 2) * 2 + layer_ready_bytes(B, N);
}

int sqa_layer_fwd(const void* x, const void* Wq, const void* Wk, const void* Wv, const void* Wo, void* out,
                  void* workspace, size_t workspace_bytes, int B, int N, int d_model, int H_q, int H_kv, int d_head,
                  int causal, float scale, void* stream) {
  if (int e = check_layer_args(x, Wq, Wk, Wv, Wo, out, B, N, d_model, H_q, H_kv, d_head, causal, scale)) return e;
  const long long M = (long long)B * N;
  const size_t need = sqa_layer_workspace_bytes(B, N, d_model, H_q, H_kv, d_head);
  if (workspace == nullptr || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0 || workspace_bytes < need)
    return SQA_ERR_WORKSPACE;
  DeviceState* st = nullptr;
  if (int e = device_state(&st)) return e;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);

  uint8_t* ws = reinterpret_cast<uint8_t*>(workspace);
  const size_t q_bytes = align256((size_t)M * H_q * d_head * 2);
  const size_t kv_bytes = align256((size_t)M * H_kv * d_head * 2);
  void* Q = ws;
  void* K = ws + q_bytes;
  void* V = ws + q_bytes + kv_bytes;
  void* A = ws + q_bytes + 2 * kv_bytes;
  // one counter per 128-row block of A: rows of A the attention kernel has stored
  int* ready = reinterpret_cast<int*>(ws + 2 * q_bytes + 2 * kv_bytes);
  const int n_blocks = (int)((M + 127) / 128);

  GemmOperands g1{};
  g1.x = x;
  g1.M = M;
  g1.K = d_model;
  g1.n_w = 3;
  g1.w[0] = Wq; g1.w[1] = Wk; g1.w[2] = Wv;
  g1.w_rows[0] = H_q * d_head; g1.w_rows[1] = H_kv * d_head; g1.w_rows[2] = H_kv * d_head;
  g1.N_out = (H_q + 2 * H_kv) * d_head;
  g1.n_y = 3;
  g1.y[0] = Q; g1.y[1] = K; g1.y[2] = V;
  g1.y_cols[0] = H_q * d_head; g1.y_cols[1] = H_kv * d_head; g1.y_cols[2] = H_kv * d_head;
  g1.zero_ptr = ready;   // zeroed before the attention kernel starts (stream order)
  g1.zero_count = n_blocks;
  if (int e = launch_gemm(st, g1, s)) return e;

  if (int e = d_head == 64 ? launch_attn<64>(st, Q, K, V, A, B, N, H_q, H_kv, causal, scale, s, nullptr, -1, 0, ready)
                           : launch_attn<128>(st, Q, K, V, A, B, N, H_q, H_kv, causal, scale, s, nullptr, -1, 0, ready))
    return e;

  GemmOperands g2{};
  g2.x = A;
  g2.M = M;
  g2.K = H_q * d_head;
  g2.n_w = 1;
  g2.w[0] = Wo;
  g2.w_rows[0] = d_model;
  g2.N_out = d_model;
  g2.n_y = 1;
  g2.y[0] = out;
  g2.y_cols[0] = d_model;
  // Wo consumes A's row blocks as the attention kernel completes them; causal
  // work runs longest (latest query tiles) first, so blocks go latest first
  g2.ready = ready;
  g2.ready_per_row = H_q;
  if (causal && N % 128 == 0) {
    g2.order = 1;
    g2.order_B = B;
    g2.order_TB = N / 128;
  }
  return launch_gemm(st, g2, s);
}

// ---------------------------------------------------------------------------
// Layer forward with library-owned scratch (no allocation by anyone per call).
//
// Some callers cannot allocate device memory for the layer's workspace: a
// framework that owns all device memory through its own allocator and budget,
// or a plugin interface that hands the library only its input and output
// buffers. For them the library keeps one fixed scratch array per device, sized
// SQA_STATIC_WORKSPACE_BYTES, that lives from library load until process exit.
static __device__ __align__(256) unsigned char g_sqa_static_ws[SQA_STATIC_WORKSPACE_BYTES];

namespace {
std::mutex g_static_mu;
void* g_static_ws_ptr[kMaxDevices] = {};

// Once per device, with that device current: the array's device address. In
// host code the array's name is only a host-side stand-in, so the address must
// come from the runtime.
int static_workspace(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return SQA_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_static_mu);
  if (!g_static_ws_ptr[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_sqa_static_ws) != cudaSuccess || ptr == nullptr) return SQA_ERR_CUDA;
    g_static_ws_ptr[dev] = ptr;
  }
  *out = g_static_ws_ptr[dev];
  return SQA_OK;
}
}  // namespace

int sqa_layer_fwd_static_ws(const void* x, const void* Wq, const void* Wk, const void* Wv, const void* Wo, void* out,
                            int B, int N, int d_model, int H_q, int H_kv, int d_head, int causal, float scale,
                            void* stream) {
  if (int e = check_layer_args(x, Wq, Wk, Wv, Wo, out, B, N, d_model, H_q, H_kv, d_head, causal, scale)) return e;
  const size_t need = sqa_layer_workspace_bytes(B, N, d_model, H_q, H_kv, d_head);
  if (need == 0) return SQA_ERR_INVALID_ARG;
  if (need > (size_t)SQA_STATIC_WORKSPACE_BYTES) return SQA_ERR_WORKSPACE;  // problem too large for the array
  void* ws = nullptr;
  if (int e = static_workspace(&ws)) return e;
  // Q, K, V and the attention output are written in full before they are read,
  // so nothing in the array has to start at zero.
  return sqa_layer_fwd(x, Wq, Wk, Wv, Wo, out, ws, (size_t)SQA_STATIC_WORKSPACE_BYTES, B, N, d_model, H_q, H_kv,
                       d_head, causal, scale, stream);
}

int sqa_linear_fwd(const void* x, const void* W, void* y, long long M, int K, int N_out, void* stream) {
  if (!aligned16(x) || !aligned16(W) || !aligned16(y)) return SQA_ERR_INVALID_ARG;
  if (M < 1 || M > INT_MAX || K < 8 || K % 8 != 0 || N_out < 8 || N_out % 8 != 0) return SQA_ERR_INVALID_ARG;
  if ((long double)M * K * 2 >= (long double)(1ull << 40) || (long double)N_out * K * 2 >= (long double)(1ull << 40))
    return SQA_ERR_INVALID_ARG;
  DeviceState* st = nullptr;
  if (int e = device_state(&st)) return e;
  GemmOperands g{};
  g.x = x;
  g.M = M;
  g.K = K;
  g.n_w = 1;
  g.w[0] = W;
  g.w_rows[0] = N_out;
  g.N_out = N_out;
  g.n_y = 1;
  g.y[0] = y;
  g.y_cols[0] = N_out;
  return launch_gemm(st, g, reinterpret_cast<cudaStream_t>(stream));
}

int sqa_device_status(void* stream) {
  DeviceState* st = nullptr;
  if (int e = device_state(&st)) return e;
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return SQA_ERR_CUDA;
  int v = 0;
  const int zero = 0;
  if (cudaMemcpyFromSymbol(&v, g_sqa_status, sizeof v) != cudaSuccess) return SQA_ERR_CUDA;
  if (cudaMemcpyToSymbol(g_sqa_status, &zero, sizeof zero) != cudaSuccess) return SQA_ERR_CUDA;
  return v;
}

unsigned long long sqa_set_wait_limit_ns(unsigned long long ns) {
  return g_wait_ns.exchange(ns == 0 ? kDefaultWaitNs : ns);
}

int sqa_check_wait_timeout(unsigned long long limit_ns, void* stream) {
  if (limit_ns < 1000ull || limit_ns > 10000000000ull) return SQA_ERR_INVALID_ARG;
  DeviceState* st = nullptr;
  if (int e = device_state(&st)) return e;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  wait_probe_kernel<<<1, 32, 0, s>>>(st->status, limit_ns);
  if (cudaGetLastError() != cudaSuccess) return SQA_ERR_CUDA;
  return sqa_device_status(stream);
}

int sqa_check_exp2_poly(const float* x, float* poly, float* ref, long long n, void* stream) {
  if (x == nullptr || poly == nullptr || ref == nullptr || n < 1 || n > (1LL << 31)) return SQA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(poly) | reinterpret_cast<uintptr_t>(ref)) & 3u)
    return SQA_ERR_INVALID_ARG;
  DeviceState* st = nullptr;
  if (int e = device_state(&st)) return e;
  const long long pairs = (n + 1) / 2;
  const long long blocks = std::min<long long>((pairs + 255) / 256, 8LL * st->sms);
  exp2_poly_probe_kernel<<<(unsigned)blocks, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(x, poly, ref, n);
  return cudaGetLastError() == cudaSuccess ? SQA_OK : SQA_ERR_CUDA;
}

int sqa_check_bounds_report(void* stream) {
  DeviceState* st = nullptr;
  if (int e = device_state(&st)) return e;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  bounds_probe_kernel<<<1, 1, 0, s>>>(st->status, 16);
  if (cudaGetLastError() != cudaSuccess) return SQA_ERR_CUDA;
  return sqa_device_status(stream);
}

const char* sqa_status_string(int status) {
  switch (status) {
    case SQA_OK: return "SQA_OK";
    case SQA_ERR_INVALID_ARG: return "SQA_ERR_INVALID_ARG";
    case SQA_ERR_UNSUPPORTED: return "SQA_ERR_UNSUPPORTED";
    case SQA_ERR_CUDA: return "SQA_ERR_CUDA";
    case SQA_ERR_TIMEOUT: return "SQA_ERR_TIMEOUT";
    case SQA_ERR_WORKSPACE: return "SQA_ERR_WORKSPACE";
    case SQA_ERR_BOUNDS: return "SQA_ERR_BOUNDS";
    default: return "SQA_ERR_UNKNOWN";
  }
}

int sqa_version(void) { return 100; }

}  // extern "C"
