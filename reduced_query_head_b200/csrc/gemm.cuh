// Projection GEMM on sm_100a: Y[M, N_out] = X[M, K] * W[N_out, K]^T, bf16 in,
// fp32 accumulate in TMEM, bf16 out. This is the no-bias linear layer of the
// attention block (GQA explainer, "PyTorchでのGQA実装": q_proj, k_proj,
// v_proj, o_proj with bias=False, weight [out_features, in_features]).
//
// W may be given as up to three row segments (Wq | Wk | Wv) with separate
// tensor maps, and Y's columns may be routed to up to three outputs (Q | K | V),
// so the fused QKV projection reads x once and writes the [B,N,H,d] views
// directly. Segment boundaries are multiples of 64 rows/columns.
//
// Persistent kernel, one CTA per SM, 128 x 256 output tiles, 64-deep K blocks
// in a 4-stage TMA ring, two TMEM accumulators so the epilogue of one tile
// overlaps the main loop of the next.
//
// Streaming X from a kernel still running (the layer's output projection):
// with `ready` set, the kernel is launched as a programmatic dependent of the
// attention kernel that writes X, and the producer waits, per 128-row block of
// X, until that block's counter shows every row written (the writer adds its
// rows with release semantics), then orders the async-proxy loads after that
// observation. Row blocks are visited in the order the attention kernel
// finishes them, so the projection runs on the SMs its tail frees.
//   warp 0      TMA producer
//   warp 1      MMA issuer + TMEM owner
//   warps 2-5   epilogue (TMEM lane quarter = warp % 4)
#pragma once

#include "sm100.cuh"

namespace sqa {

struct GemmParams {
  int M, K, N_out;
  int tiles_m, tiles_n;
  int n_seg_w;                 // row segments of W (1..3)
  int w_seg_start[4];          // segment i covers rows [start[i], start[i+1])
  int n_seg_y;                 // column segments of Y (1..3)
  int y_seg_start[4];
  __nv_bfloat16* y_ptr[3];
  long long y_ld[3];           // row stride (elements) of each output
  // X written while this kernel runs: row block tm is ready once ready[tm] reaches
  // (rows in the block) * ready_per_row; nullptr when X is complete at launch.
  const int* ready;
  int ready_per_row;
  // Row-block order: 0 = natural; 1 = B batches of TB blocks each, the last
  // block of every batch first (the order a causal longest-first attention
  // finishes its query tiles).
  int order, order_B, order_TB;
  // Counters of a later kernel, zeroed by CTA 0 at start (nullptr: none).
  int* zero_ptr;
  int zero_count;
  int* status;
  unsigned long long timeout_ns;
};

// Row block and column block of the tile-th output tile.
__device__ __forceinline__ void gemm_tile_coords(const GemmParams& p, int tile, int& tm, int& tn) {
  const int mo = tile / p.tiles_n;
  tn = tile - mo * p.tiles_n;
  tm = p.order ? (mo % p.order_B) * p.order_TB + (p.order_TB - 1 - mo / p.order_B) : mo;
}

__device__ __forceinline__ int ld_acquire_gpu(const int* ptr) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(ptr) : "memory");
  return v;
}

// Wait (bounded) until *ptr >= target; false on time-out or abort.
__device__ __forceinline__ bool wait_counter(const int* ptr, int target, const WaitCtl& c) {
  if (ld_acquire_gpu(ptr) >= target) return true;
  const uint64_t t0 = global_timer_ns();
  while (true) {
    __nanosleep(128);
    if (ld_acquire_gpu(ptr) >= target) return true;
    if (*c.abort_flag) return false;
    if (global_timer_ns() - t0 > c.timeout_ns) {
      *c.abort_flag = 1;
      atomicCAS(c.status, kStatusOk, kStatusTimeout);
      return false;
    }
  }
}

struct GemmCfg {
  static constexpr int BM = 128, BN = 256, BK = 64, STAGES = 4;
  static constexpr int A_BYTES = BM * BK * 2;      // 16 KB
  static constexpr int B_BYTES = BN * BK * 2;      // 32 KB
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int OFF_BAR = STAGES * STAGE_BYTES;
  // full[S], empty[S], acc_full[2], acc_empty[2], drain
  static constexpr int BAR_FULL = 0, BAR_EMPTY = STAGES, BAR_ACCF = 2 * STAGES, BAR_ACCE = 2 * STAGES + 2,
                       BAR_DRAIN = 2 * STAGES + 4, N_BARS = 2 * STAGES + 5;
  static constexpr int OFF_MISC = OFF_BAR + N_BARS * 8;
  static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;
  static constexpr int THREADS = 192;
  static constexpr uint32_t TMEM_COLS = 512;
};

__global__ void __launch_bounds__(192, 1)
    gemm_bf16_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w0,
                     const __grid_constant__ CUtensorMap tm_w1, const __grid_constant__ CUtensorMap tm_w2,
                     const GemmParams p) {
  using C = GemmCfg;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile uint32_t* tmem_slot = misc;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);
  auto bar = [&](int i) { return smem_u32(&bars[i]); };

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n_tiles = p.tiles_m * p.tiles_n;
  const int k_blocks = (p.K + C::BK - 1) / C::BK;
  WaitCtl ctl{abort_flag, p.status, p.timeout_ns};

  if (tid == 0) {
    for (int i = 0; i < C::N_BARS; ++i) mbar_init(bar(i), (i == C::BAR_ACCE || i == C::BAR_ACCE + 1) ? 4 : 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (blockIdx.x == 0 && p.zero_ptr != nullptr)
    for (int i = tid; i < p.zero_count; i += blockDim.x) p.zero_ptr[i] = 0;
  if (warp == 1) {
    tmem_alloc(smem_u32((const void*)tmem_slot), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&tm_x);
      tma_prefetch_desc(&tm_w0);
      if (p.n_seg_w > 1) tma_prefetch_desc(&tm_w1);
      if (p.n_seg_w > 2) tma_prefetch_desc(&tm_w2);
      int it = 0;  // global k-block counter across tiles
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < n_tiles; tile += gridDim.x) {
        int tm, tn;
        gemm_tile_coords(p, tile, tm, tn);
        if (!in_bounds(tm >= 0 && tm < p.tiles_m && tn >= 0 && tn < p.tiles_n, p.status)) { ok = false; break; }
        if (p.ready != nullptr) {
          // every row of this block of X written (acquire), then the async proxy may read it
          const int rows = min(C::BM, p.M - tm * C::BM);
          if (!wait_counter(p.ready + tm, rows * p.ready_per_row, ctl)) { ok = false; break; }
          asm volatile("fence.proxy.async.global;" ::: "memory");
        }
        for (int kb = 0; kb < k_blocks; ++kb, ++it) {
          const int s = it % C::STAGES;
          const int round = it / C::STAGES;
          if (round > 0 && !mbar_wait(bar(C::BAR_EMPTY + s), (round - 1) & 1, ctl)) { ok = false; break; }
          const uint32_t a_dst = sbase + s * C::STAGE_BYTES;
          const uint32_t b_dst = a_dst + C::A_BYTES;
          mbar_arrive_expect_tx(bar(C::BAR_FULL + s), C::STAGE_BYTES);
          tma_load_2d(a_dst, &tm_x, bar(C::BAR_FULL + s), kb * C::BK, tm * C::BM);
#pragma unroll
          for (int q = 0; q < C::BN / 64; ++q) {
            const int row = tn * C::BN + q * 64;
            int seg = 0;
            if (p.n_seg_w > 1 && row >= p.w_seg_start[1]) seg = 1;
            if (p.n_seg_w > 2 && row >= p.w_seg_start[2]) seg = 2;
            const void* map = seg == 0 ? (const void*)&tm_w0 : seg == 1 ? (const void*)&tm_w1 : (const void*)&tm_w2;
            // rows past the last segment's end read as zero (a partial last N tile)
            if (!in_bounds(row - p.w_seg_start[seg] >= 0, p.status)) continue;
            tma_load_2d(b_dst + q * 64 * 128, map, bar(C::BAR_FULL + s), kb * C::BK, row - p.w_seg_start[seg]);
          }
        }
      }
      // drain the copies in flight
      volatile int zero = 0;
      WaitCtl drain{&zero, p.status, drain_limit_ns(p.timeout_ns)};
      for (int j = max(0, it - C::STAGES); j < it; ++j)
        mbar_wait(bar(C::BAR_FULL + j % C::STAGES), (j / C::STAGES) & 1, drain);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t IDESC = idesc_bf16_f32(C::BM, C::BN, 0, 0);
      int it = 0, local = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < n_tiles; tile += gridDim.x, ++local) {
        const int a = local & 1;
        const int use = local >> 1;
        if (use > 0 && !mbar_wait(bar(C::BAR_ACCE + a), (use - 1) & 1, ctl)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem + a * C::BN;
        for (int kb = 0; kb < k_blocks; ++kb, ++it) {
          const int s = it % C::STAGES;
          if (!mbar_wait(bar(C::BAR_FULL + s), (it / C::STAGES) & 1, ctl)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_addr = sbase + s * C::STAGE_BYTES;
          const uint32_t b_addr = a_addr + C::A_BYTES;
#pragma unroll
          for (int kk = 0; kk < C::BK / 16; ++kk)
            umma_ss(d_tmem, sdesc_sw128(a_addr + kk * 32, 16, 1024), sdesc_sw128(b_addr + kk * 32, 16, 1024),
                    IDESC, (kb > 0 || kk > 0) ? 1u : 0u);
          umma_commit(bar(C::BAR_EMPTY + s));
        }
        if (ok) umma_commit(bar(C::BAR_ACCF + a));
      }
      umma_commit(bar(C::BAR_DRAIN));
      volatile int zero = 0;
      WaitCtl drain{&zero, p.status, drain_limit_ns(p.timeout_ns)};
      mbar_wait(bar(C::BAR_DRAIN), 0, drain);
    }
  } else {
    // epilogue warps 2..5
    const int quarter = warp & 3;
    const int row_in_tile = quarter * 32 + lane;
    const uint32_t lane_base = tmem + (uint32_t(quarter * 32) << 16);
    int local = 0;
    for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x, ++local) {
      const int a = local & 1;
      const int use = local >> 1;
      if (!mbar_wait_warp(bar(C::BAR_ACCF + a), use & 1, ctl)) break;
      tc_fence_after();
      int tm, tn;
      gemm_tile_coords(p, tile, tm, tn);
      const long long row = (long long)tm * C::BM + row_in_tile;
      const bool row_ok = row < p.M;
#pragma unroll 1
      for (int c = 0; c < C::BN; c += 32) {
        uint32_t r[32];
        __syncwarp();   // after the per-lane stores: the TMEM load is warp-collective
        tmem_ld32(lane_base + a * C::BN + c, r);
        const int col = tn * C::BN + c;
        if (row_ok && col < p.N_out) {
          int seg = 0;
          if (p.n_seg_y > 1 && col >= p.y_seg_start[1]) seg = 1;
          if (p.n_seg_y > 2 && col >= p.y_seg_start[2]) seg = 2;
          if (!in_bounds(col - p.y_seg_start[seg] + 32 <= p.y_ld[seg] || col + 32 > p.N_out, p.status)) continue;
          __nv_bfloat16* dst = p.y_ptr[seg] + row * p.y_ld[seg] + (col - p.y_seg_start[seg]);
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            if (col + v * 8 < p.N_out) {
              uint4 w;
              w.x = pack_bf16x2(__uint_as_float(r[v * 8 + 0]), __uint_as_float(r[v * 8 + 1]));
              w.y = pack_bf16x2(__uint_as_float(r[v * 8 + 2]), __uint_as_float(r[v * 8 + 3]));
              w.z = pack_bf16x2(__uint_as_float(r[v * 8 + 4]), __uint_as_float(r[v * 8 + 5]));
              w.w = pack_bf16x2(__uint_as_float(r[v * 8 + 6]), __uint_as_float(r[v * 8 + 7]));
              *reinterpret_cast<uint4*>(dst + v * 8) = w;
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(C::BAR_ACCE + a));
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
  // Streaming mode (a programmatic dependent of the attention grid): do not
  // complete before that grid, so work ordered after the layer on the stream
  // finds it complete. A no-op otherwise.
  if (p.ready != nullptr) asm volatile("griddepcontrol.wait;" ::: "memory");
}

}  // namespace sqa
