// Decode attention on sm_100a: one new token per sequence against its K/V cache.
//
//   out[b,i,:] = sum_u softmax_u(scale * q[b,i,:] . k[b,u,g(i),:]) v[b,u,g(i),:],
//   u over all N cached keys, g(i) = floor(i * H_kv / H_q).
// This is the autoregressive step of the GQA explainer ("背景と動機" and the
// KV-cache table): every query head of a group reads the same cached K/V, so
// a step streams B * N * H_kv * d * 2 elements from HBM whatever H_q is (the
// reason fewer query heads do not speed decoding up).
//
// Memory-bound: the kernels stream each group's K/V once.
//   decode_split_kernel   one CTA per (split of the keys, block of the group's
//                         query heads, (b, g)). A producer warp streams
//                         64-key K/V tiles through a TMA ring; four consumer
//                         warps each take 16 keys of every tile, compute
//                         S = Q K^T and O += P V with mma.sync (16 head rows
//                         per block), keep an online softmax in registers and
//                         write an unnormalised partial (m, l, o) per head.
//                         (Merging the four warps in shared memory first
//                         measured slower: barriers and atomics per CTA.)
//   decode_combine_kernel merges the partials of each (b, i) into out (one
//                         CTA per head row; each thread folds a 16-column
//                         slice of a strided set of parts into its own running
//                         maximum, in one pass). It is launched as a
//                         programmatic dependent of the split grid, so its
//                         launch overlaps the split's last wave.
#pragma once

#include "sm100.cuh"

namespace sqa {

struct DecodeParams {
  const __nv_bfloat16* q;   // [B, H_q, D]
  float* part;              // [B, H_q, n_parts, D + 2]: m (log2 units), l, o[D]; one part per consumer warp
  __nv_bfloat16* out;       // [B, H_q, D]
  int B, N, H_q, H_kv;
  int splits, tiles_per_split, n_parts;   // n_parts = splits * 4 (one per consumer warp)
  int heads_per_cta;        // 16 * row blocks
  float scale_log2;
  int* status;
  unsigned long long timeout_ns;
};

template <int D>
struct DecodeCfg {
  static constexpr int KCH = D / 64;                 // 128-byte column chunks
  static constexpr int BK = 64;                      // keys per tile
  static constexpr int RB = (D == 64) ? 2 : 1;       // 16-row head blocks per CTA
  static constexpr int STAGES = (D == 64) ? 4 : 3;   // two CTAs per SM either way
  static constexpr int T_BYTES = BK * D * 2;         // K or V tile
  static constexpr int T_CHUNK = BK * 128;
  static constexpr int STAGE_BYTES = 2 * T_BYTES;
  static constexpr int OFF_BAR = STAGES * STAGE_BYTES;
  static constexpr int BAR_FULL = 0, BAR_EMPTY = STAGES, N_BARS = 2 * STAGES;
  static constexpr int OFF_MISC = OFF_BAR + N_BARS * 8;
  static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;
  static constexpr int THREADS = 160;                // warps 0-3 consumers, warp 4 producer
};

// ------------------------------------------------------------------ mma.sync helpers
__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void ldmatrix_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                                  uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
// Byte address of (row, 16-byte chunk c) in a 128-byte-swizzled tile: the
// chunk index is XORed with row % 8 (the TMA SWIZZLE_128B layout).
__device__ __forceinline__ uint32_t sw128(uint32_t base, int row, int c) {
  return base + (uint32_t)row * 128u + (uint32_t)((c ^ (row & 7)) << 4);
}

template <int D>
__global__ void __launch_bounds__(160)
    decode_split_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                        const DecodeParams p) {
  using C = DecodeCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC);
  auto bar = [&](int i) { return smem_u32(&bars[i]); };
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  const int split = blockIdx.x, hblk = blockIdx.y, bg = blockIdx.z;
  const int b = bg / p.H_kv, g = bg - b * p.H_kv;
  // query heads of group g under g(i) = floor(i * H_kv / H_q); this CTA's block of them
  const int i0 = (int)(((long long)g * p.H_q + p.H_kv - 1) / p.H_kv);
  const int i1 = (int)(((long long)(g + 1) * p.H_q + p.H_kv - 1) / p.H_kv);
  const int h_lo = i0 + hblk * p.heads_per_cta, h_hi = min(i1, h_lo + p.heads_per_cta);
  if (h_lo >= h_hi) return;  // uniform over the CTA, before any barrier exists
  const int n_tiles = (p.N + C::BK - 1) / C::BK;
  const int t_begin = split * p.tiles_per_split;
  const int n_t = max(0, min(n_tiles, t_begin + p.tiles_per_split) - t_begin);

  WaitCtl ctl{abort_flag, p.status, p.timeout_ns};
  if (threadIdx.x == 0) {
    for (int i = 0; i < C::N_BARS; ++i) mbar_init(bar(i), i >= C::BAR_EMPTY ? 4 : 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == 4) {
    if (lane == 0) {
      int filled = 0;
      for (int j = 0; j < n_t; ++j) {
        const int st = j % C::STAGES, round = j / C::STAGES;
        if (round > 0 && !mbar_wait(bar(C::BAR_EMPTY + st), (round - 1) & 1, ctl)) break;
        if (!in_bounds((t_begin + j) * C::BK < p.N && g < p.H_kv && b < p.B, p.status)) break;
        const uint32_t dst = sbase + st * C::STAGE_BYTES;
        const uint32_t full = bar(C::BAR_FULL + st);
        mbar_arrive_expect_tx(full, C::STAGE_BYTES);
#pragma unroll
        for (int c = 0; c < C::KCH; ++c) {
          tma_load_4d(dst + c * C::T_CHUNK, &tm_k, full, c * 64, g, (t_begin + j) * C::BK, b);
          tma_load_4d(dst + C::T_BYTES + c * C::T_CHUNK, &tm_v, full, c * 64, g, (t_begin + j) * C::BK, b);
        }
        filled = j + 1;
      }
      volatile int zero = 0;
      WaitCtl drain{&zero, p.status, drain_limit_ns(p.timeout_ns)};
      for (int j = max(0, filled - C::STAGES); j < filled; ++j)
        mbar_wait(bar(C::BAR_FULL + j % C::STAGES), (j / C::STAGES) & 1, drain);
    }
    return;
  }

  // ---- consumer warp w: keys [16w, 16w + 16) of every tile
  const int g4 = lane >> 2, t4 = lane & 3;
  const int nrb = (h_hi - h_lo + 15) >> 4;  // 16-row head blocks in use (1..RB)
  // Q as mma A fragments, rows = heads h_lo + 16 rb + {g4, g4 + 8}; rows past h_hi are zero
  uint32_t qa[C::RB][D / 16][4];
#pragma unroll
  for (int rb = 0; rb < C::RB; ++rb) {
    const int r0 = h_lo + rb * 16 + g4, r1 = r0 + 8;
    const uint32_t* q0 = reinterpret_cast<const uint32_t*>(p.q + ((size_t)b * p.H_q + (r0 < h_hi ? r0 : h_lo)) * D);
    const uint32_t* q1 = reinterpret_cast<const uint32_t*>(p.q + ((size_t)b * p.H_q + (r1 < h_hi ? r1 : h_lo)) * D);
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
      qa[rb][ks][0] = r0 < h_hi ? q0[ks * 8 + t4] : 0u;
      qa[rb][ks][1] = r1 < h_hi ? q1[ks * 8 + t4] : 0u;
      qa[rb][ks][2] = r0 < h_hi ? q0[ks * 8 + 4 + t4] : 0u;
      qa[rb][ks][3] = r1 < h_hi ? q1[ks * 8 + 4 + t4] : 0u;
    }
  }
  float o[C::RB][D / 8][4];
  float m[C::RB][2], l[C::RB][2];
#pragma unroll
  for (int rb = 0; rb < C::RB; ++rb) {
    m[rb][0] = m[rb][1] = -INFINITY;
    l[rb][0] = l[rb][1] = 0.f;
#pragma unroll
    for (int nb = 0; nb < D / 8; ++nb) o[rb][nb][0] = o[rb][nb][1] = o[rb][nb][2] = o[rb][nb][3] = 0.f;
  }
  const float sl2 = p.scale_log2;
  bool ok = true;
  for (int j = 0; j < n_t; ++j) {
    const int st = j % C::STAGES;
    if (!mbar_wait_warp(bar(C::BAR_FULL + st), (j / C::STAGES) & 1, ctl)) { ok = false; break; }
    const uint32_t kb = sbase + st * C::STAGE_BYTES, vb = kb + C::T_BYTES;
    const int key0 = (t_begin + j) * C::BK + 16 * warp;
    // K fragments (B of S = Q K^T): matrix (lane >> 3): keys 8 * (lane >> 4) .. +7, d chunk ks*16 + 8*((lane>>3)&1)
    uint32_t kf[D / 16][4];
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
      const int row = 16 * warp + ((lane >> 4) << 3) + (lane & 7);
      const int ch = 2 * (ks & 3) + ((lane >> 3) & 1);
      ldmatrix_x4(sw128(kb + (ks >> 2) * C::T_CHUNK, row, ch), kf[ks][0], kf[ks][1], kf[ks][2], kf[ks][3]);
    }
    // V fragments (B of O += P V), transposed: matrix (lane >> 3): keys 8*((lane>>3)&1) .. +7, d cols np*16 + 8*(lane>>4)
    uint32_t vf[D / 16][4];
#pragma unroll
    for (int np = 0; np < D / 16; ++np) {
      const int row = 16 * warp + (((lane >> 3) & 1) << 3) + (lane & 7);
      const int ch = 2 * (np & 3) + (lane >> 4);
      ldmatrix_x4_trans(sw128(vb + (np >> 2) * C::T_CHUNK, row, ch), vf[np][0], vf[np][1], vf[np][2], vf[np][3]);
    }
    // every shared-memory read of this stage is done: release it
    __syncwarp();
    if (lane == 0) mbar_arrive(bar(C::BAR_EMPTY + st));
    const bool tail = key0 + 16 > p.N;
#pragma unroll
    for (int rb = 0; rb < C::RB; ++rb) {
      if (rb >= nrb) break;
      float s[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks) {
        mma_bf16_16816(s[0], qa[rb][ks], kf[ks][0], kf[ks][1]);
        mma_bf16_16816(s[1], qa[rb][ks], kf[ks][2], kf[ks][3]);
      }
      // s[nb][0..1]: row g4, keys key0 + 8 nb + 2 t4 + {0,1}; s[nb][2..3]: row g4 + 8
#pragma unroll
      for (int nb = 0; nb < 2; ++nb)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          float x = s[nb][e] * sl2;
          if (tail && key0 + 8 * nb + 2 * t4 + (e & 1) >= p.N) x = -INFINITY;
          s[nb][e] = x;
        }
      float mx0 = fmaxf(fmaxf(s[0][0], s[0][1]), fmaxf(s[1][0], s[1][1]));
      float mx1 = fmaxf(fmaxf(s[0][2], s[0][3]), fmaxf(s[1][2], s[1][3]));
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
      const float mn0 = fmaxf(m[rb][0], mx0), mn1 = fmaxf(m[rb][1], mx1);
      // a row with no visible key yet keeps m = -inf: subtract 0 instead (every p is 0)
      const float ref0 = mn0 == -INFINITY ? 0.f : mn0, ref1 = mn1 == -INFINITY ? 0.f : mn1;
      const float c0 = ex2_approx(m[rb][0] - ref0), c1 = ex2_approx(m[rb][1] - ref1);
      m[rb][0] = mn0;
      m[rb][1] = mn1;
      float pr[2][4];
#pragma unroll
      for (int nb = 0; nb < 2; ++nb) {
        pr[nb][0] = ex2_approx(s[nb][0] - ref0);
        pr[nb][1] = ex2_approx(s[nb][1] - ref0);
        pr[nb][2] = ex2_approx(s[nb][2] - ref1);
        pr[nb][3] = ex2_approx(s[nb][3] - ref1);
      }
      l[rb][0] = l[rb][0] * c0 + (pr[0][0] + pr[0][1] + pr[1][0] + pr[1][1]);
      l[rb][1] = l[rb][1] * c1 + (pr[0][2] + pr[0][3] + pr[1][2] + pr[1][3]);
      uint32_t pa[4];
      pa[0] = pack_bf16x2(pr[0][0], pr[0][1]);
      pa[1] = pack_bf16x2(pr[0][2], pr[0][3]);
      pa[2] = pack_bf16x2(pr[1][0], pr[1][1]);
      pa[3] = pack_bf16x2(pr[1][2], pr[1][3]);
#pragma unroll
      for (int np = 0; np < D / 16; ++np) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          float(&acc)[4] = o[rb][2 * np + h];
          acc[0] *= c0;
          acc[1] *= c0;
          acc[2] *= c1;
          acc[3] *= c1;
          mma_bf16_16816(acc, pa, vf[np][2 * h], vf[np][2 * h + 1]);
        }
      }
    }
  }
  if (!ok) return;
  // ---- partial of this warp: m (log2 units), l, unnormalised o, per head row
  const int pi = split * 4 + warp;
#pragma unroll
  for (int rb = 0; rb < C::RB; ++rb) {
    if (rb >= nrb) break;
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      float lt = l[rb][half];
      lt += __shfl_xor_sync(0xffffffffu, lt, 1);
      lt += __shfl_xor_sync(0xffffffffu, lt, 2);
      const int r = h_lo + rb * 16 + g4 + 8 * half;
      if (r < h_hi && in_bounds(r < p.H_q && pi < p.n_parts && b < p.B, p.status)) {
        float* dst = p.part + (((size_t)b * p.H_q + r) * p.n_parts + pi) * (D + 2);
        if (t4 == 0) {
          dst[0] = m[rb][half];
          dst[1] = lt;
        }
#pragma unroll
        for (int nb = 0; nb < D / 8; ++nb)
          *reinterpret_cast<float2*>(dst + 2 + nb * 8 + 2 * t4) =
              make_float2(o[rb][nb][2 * half], o[rb][nb][2 * half + 1]);
      }
    }
  }
  // the combine grid (launched as a programmatic dependent) may be scheduled
  // once every CTA of this grid got here or exited; its griddepcontrol.wait
  // still waits for this grid to complete and its writes to be visible
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// One CTA of 128 threads per (b, i): merge the partials of all splits and
// warps in one pass. Thread t owns the 16-column slice t % (D/16) of the parts
// t / (D/16), t / (D/16) + G, ... (G part groups) and folds them into a
// running (max, l, o) of its own, with the loads of four parts issued before
// any is used; the G groups' states are then merged with their own maxima.
// Parts that saw no key hold m = -inf and weigh nothing.
template <int D>
__global__ void __launch_bounds__(128) decode_combine_kernel(const DecodeParams p) {
  constexpr int CW = D / 16, G = 128 / CW, U = 4;
  __shared__ float gacc[G][D];
  __shared__ float gm[G], gl[G];
  const int row = blockIdx.x;   // b * H_q + i
  const int t = threadIdx.x;
  // launched as a programmatic dependent of the split grid: wait until that
  // grid has completed and its partials are visible (a no-op otherwise)
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const float* base = p.part + (size_t)row * p.n_parts * (D + 2);
  const int c = t % CW, pg = t / CW;
  float mm = -INFINITY, L = 0.f, acc[16];
#pragma unroll
  for (int x = 0; x < 16; ++x) acc[x] = 0.f;
  for (int k0 = pg; k0 < p.n_parts; k0 += U * G) {
    float2 ml[U];
    float v[U][16];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int k = k0 + u * G;
      if (k < p.n_parts) {
        const float* pk = base + (size_t)k * (D + 2);
        ml[u] = *reinterpret_cast<const float2*>(pk);
        // the o slice starts 8 bytes into the 8-byte-aligned part: float2 loads
#pragma unroll
        for (int x = 0; x < 8; ++x) {
          const float2 f2 = *reinterpret_cast<const float2*>(pk + 2 + 16 * c + 2 * x);
          v[u][2 * x] = f2.x;
          v[u][2 * x + 1] = f2.y;
        }
      } else {
        ml[u] = make_float2(-INFINITY, 0.f);
#pragma unroll
        for (int x = 0; x < 16; ++x) v[u][x] = 0.f;
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const float mn = fmaxf(mm, ml[u].x);
      const bool any = mn != -INFINITY;
      const float a = any ? ex2_approx(mm - mn) : 0.f;      // rescale of what is held (0 if nothing yet)
      const float w = any ? ex2_approx(ml[u].x - mn) : 0.f;
      L = L * a + w * ml[u].y;
#pragma unroll
      for (int x = 0; x < 16; ++x) acc[x] = acc[x] * a + w * v[u][x];
      mm = mn;
    }
  }
#pragma unroll
  for (int x = 0; x < 16; ++x) gacc[pg][16 * c + x] = acc[x];
  if (c == 0) {
    gm[pg] = mm;
    gl[pg] = L;
  }
  __syncthreads();
  if (t < D / 2) {
    float M = -INFINITY;
#pragma unroll 8
    for (int g2 = 0; g2 < G; ++g2) M = fmaxf(M, gm[g2]);
    float sx = 0.f, sy = 0.f, sl = 0.f;
#pragma unroll 4
    for (int g2 = 0; g2 < G; ++g2) {
      const float w = gm[g2] != -INFINITY ? ex2_approx(gm[g2] - M) : 0.f;
      sx += w * gacc[g2][2 * t];
      sy += w * gacc[g2][2 * t + 1];
      sl += w * gl[g2];
    }
    const float inv = 1.0f / sl;
    if (in_bounds(row < p.B * p.H_q, p.status))
      *reinterpret_cast<uint32_t*>(p.out + (size_t)row * D + 2 * t) = pack_bf16x2(sx * inv, sy * inv);
  }
}

}  // namespace sqa
