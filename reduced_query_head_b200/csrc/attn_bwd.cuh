// Backward pass of decoupled-head attention on sm_100a.
//
// With S = scale * Q_i K_g^T, P = softmax(S) and O_i = P V_g (query head i,
// group g = floor(i * H_kv / H_q)), an upstream gradient dO_i gives
//   dP = dO_i V_g^T,  dS = P * (dP - D),  D = rowsum(dO_i * O_i)
//   dQ_i = scale * dS K_g,  dK_g += scale * dS^T Q_i,  dV_g += P^T dO_i.
// The sums over i make the K/V gradients group-aware: every query head that
// reads a group adds its share (the repetition of the GQA explainer's module,
// "PyTorchでのGQA実装", expand). P is recomputed from the forward's row
// log-sum-exp instead of being stored.
//
// Three kernels:
//   bwd_prep   D and the log-sum-exp in log2 units, laid out [B, H_q, N]
//   bwd_dkdv   one CTA per (128-key tile, group, batch); loops over the group's
//              heads and the query tiles, accumulating dK and dV in TMEM
//   bwd_dq     one CTA per 128-row query tile (heads of a group stacked as in
//              the forward); loops over the key tiles, accumulating dQ in TMEM
// Both main kernels keep S^T/S and dP^T/dP in TMEM and write P^T/dS^T (dS) back
// over them as bf16, so the second-stage MMAs read their A operand from TMEM.
#pragma once

#include "sm100.cuh"

namespace sqa {

// ---------------------------------------------------------------- prep
// One warp per row (b, t, i): D = sum_c dO * O (fp32) and lse2 = lse * log2(e),
// both stored negated (-D, -lse2) so that the main kernels add them with a
// plain fused multiply-add. Outputs are [B * H_q] rows of `ld` >= N floats (ld
// a multiple of 4, so that the rows can be TMA-loaded); columns >= N are never
// written.
template <int D>
__global__ void __launch_bounds__(256) bwd_prep_kernel(const __nv_bfloat16* __restrict__ out,
                                                       const __nv_bfloat16* __restrict__ dout,
                                                       const float* __restrict__ lse, float* __restrict__ ndsum,
                                                       float* __restrict__ nlse2, int B, int N, int H_q, int ld) {
  const long long rows = (long long)B * N * H_q;
  const long long row = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  constexpr int PER = D / 32;  // 2 or 4 elements per lane
  const __nv_bfloat16* o = out + row * D + lane * PER;
  const __nv_bfloat16* g = dout + row * D + lane * PER;
  float acc = 0.f;
#pragma unroll
  for (int u = 0; u < PER; ++u) acc = fmaf(__bfloat162float(o[u]), __bfloat162float(g[u]), acc);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if (lane == 0) {
    // row = (b * N + t) * H_q + i  ->  [b, i, t]
    const long long i = row % H_q;
    const long long bt = row / H_q;
    const long long t = bt % N, b = bt / N;
    ndsum[(b * H_q + i) * ld + t] = -acc;
    nlse2[(b * H_q + i) * ld + t] = lse[(b * H_q + i) * N + t] * -1.4426950408889634f;
  }
}

struct BwdParams {
  const __nv_bfloat16* q;     // [B, N, H_q, D]
  const __nv_bfloat16* k;     // [B, N, H_kv, D]
  const __nv_bfloat16* v;     // [B, N, H_kv, D]
  const __nv_bfloat16* dout;  // [B, N, H_q, D]
  __nv_bfloat16* dq;    // [B, N, H_q, D]
  __nv_bfloat16* dk;    // [B, N, H_kv, D]
  __nv_bfloat16* dv;    // [B, N, H_kv, D]
  const float* nlse2;   // [B, H_q] rows of ld: -(log-sum-exp in log2 units)
  const float* ndsum;   // [B, H_q] rows of ld: -rowsum(dO * O)
  int ld;               // row stride of lse2 / dsum
  int B, N, H_q, H_kv;
  int P, log2P, tpt;    // dq kernel: heads stacked per tile, tokens per tile
  int n_hb;             // dq kernel: head blocks = H_q / P
  int causal;
  float scale;          // softmax scale
  float scale_log2;     // scale * log2(e)
  int* status;
  unsigned long long timeout_ns;
};



// Both main kernels run a two-buffer pipeline: TMEM buffer b (b = step & 1)
// holds the step's scores in its first half and dP in its second. Both
// elementwise warpgroups work on every step, each on its own half of the
// step's columns, and write P / dS back as bf16 behind the columns they have
// already read (the MMA reads each K16 step of the A operand from wherever its
// warpgroup put it). The MMA issuers are split by product, so every TMEM
// region has one issuing thread and in-order issue orders its reuse.
// dQ kernel (96-key steps, 192-column buffers): warp 1 issues S, warp 3 issues
// dP and dQ += dS K_j into one dQ accumulator; Q and dO are TMEM operands at
// d = 64 and shared-memory operands at d = 128.
// dK/dV kernel (64-query steps): at d = 64 K and V sit in TMEM, so all four products
// are TS; warp 1 issues S^T and dV, warp 3 dP^T and dK, and every TMEM region
// (scores or dP half of a buffer, one accumulator) has a single issuer. At
// d = 128 there is no TMEM left for K and V: the score products read them from
// shared memory (SS), with the same split of the products between the issuers.
//   warp 0      TMA producer
//   warp 1      MMA issuer 0 + TMEM owner
//   warp 3      MMA issuer 1
//   warps 4-7   elementwise, first half of every step's columns (thread = TMEM lane = tile row)
//   warps 8-11  elementwise, second half of every step's columns

// 16 columns of the elementwise step from the scores s and dP read from TMEM:
// p = exp2(s * scale_log2 - lse2), ds = p * (dP - D), both packed to bf16
// pairs (low half = even column). nl / nd hold -lse2 / -D per column pair.
__device__ __forceinline__ void bwd_chunk(const uint32_t (&rs)[16], const uint32_t (&rd)[16], float sl2,
                                          const float2 (&nl)[8], const float2 (&nd)[8], uint32_t (&pp)[8],
                                          uint32_t (&pd)[8]) {
  const float2 s2 = make_float2(sl2, sl2);
#pragma unroll
  for (int w = 0; w < 8; ++w) {
    const float2 x = ffma2(make_float2(__uint_as_float(rs[2 * w]), __uint_as_float(rs[2 * w + 1])), s2, nl[w]);
    const float2 pe = make_float2(ex2_approx(x.x), ex2_approx(x.y));
    const float2 g = fadd2(make_float2(__uint_as_float(rd[2 * w]), __uint_as_float(rd[2 * w + 1])), nd[w]);
    const float2 ds = fmul2(pe, g);
    pp[w] = pack_bf16x2(pe.x, pe.y);
    pd[w] = pack_bf16x2(ds.x, ds.y);
  }
}

// ---------------------------------------------------------------- dK, dV
template <int D>
struct DkdvCfg {
  static constexpr int KCH = D / 64;                   // 128-byte column chunks
  static constexpr int BQ = 64;                        // queries per step
  // d = 64: K and V rows in TMEM (A operands of the score products); d = 128:
  // from shared memory. Two issuers either way, split by product.
  static constexpr bool KV_TMEM = (D == 64);
  static constexpr int NI = 2;
  static constexpr int STAGES = (D == 64) ? 8 : 4;
  static constexpr int KV_BYTES = 128 * D * 2;         // K or V tile, 128 keys
  static constexpr int KV_CHUNK = 128 * 128;           // one column chunk of it
  static constexpr int T_BYTES = BQ * D * 2;           // Q_j or dO_j, 64 queries
  static constexpr int T_CHUNK = BQ * 128;
  static constexpr int STAGE_BYTES = 2 * T_BYTES;
  static constexpr int VEC_BYTES = BQ * 4;             // -lse2 or -D of the step's queries
  static constexpr int OFF_K = 0, OFF_V = KV_BYTES, OFF_STAGE = KV_TMEM ? 0 : 2 * KV_BYTES;
  static constexpr int OFF_VEC = OFF_STAGE + STAGES * STAGE_BYTES;   // [STAGES][-lse2 | -D]
  static constexpr int OFF_BAR = OFF_VEC + STAGES * 2 * VEC_BYTES;
  static constexpr int BAR_KV = 0, BAR_FULL = 1, BAR_EMPTY = 1 + STAGES, BAR_S = 1 + 2 * STAGES,
                       BAR_P = BAR_S + 2, BAR_DONE = BAR_P + 2, BAR_DRAIN = BAR_DONE + 2, N_BARS = BAR_DRAIN + 2;
  static constexpr int OFF_MISC = OFF_BAR + N_BARS * 8;
  static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;
  static constexpr int THREADS = 384;
  static constexpr uint32_t TMEM_COLS = 512;
  // dV at COL_ACC, dK D columns after it; K and V rows (KV_TMEM) after those
  static constexpr uint32_t COL_ACC = 256, COL_KT = COL_ACC + 2 * D, COL_VT = COL_KT + D / 2;
  static_assert(COL_ACC + 2 * D <= TMEM_COLS && (!KV_TMEM || COL_VT + D / 2 <= TMEM_COLS), "TMEM budget");
  static_assert(STAGE_BYTES % 1024 == 0 && OFF_STAGE % 1024 == 0, "tile alignment");
};

// One CTA per (128-key tile u, KV group g, batch b). Steps walk the group's
// query heads and, per head, the 64-query tiles that can see key tile u
// (all of them, or those from 128u on when causal). Thread = key row:
// S^T = K Q_j^T and dP^T = V dO_j^T, then dV += P^T dO_j and dK += dS^T Q_j
// with P^T and dS^T read from TMEM.
template <int D>
__global__ void __launch_bounds__(384, 1)
    bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
                    const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                    const __grid_constant__ CUtensorMap tm_lse2, const __grid_constant__ CUtensorMap tm_dsum,
                    const BwdParams p) {
  using C = DkdvCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile uint32_t* tmem_slot = misc;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);
  auto bar = [&](int i) { return smem_u32(&bars[i]); };
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  // ---- work item: causal items run longest (small u) first
  const int n_kt = (p.N + 127) / 128;
  const int L = blockIdx.x;
  int u, rest;
  if (p.causal) {
    u = L / (p.B * p.H_kv);
    rest = L - u * (p.B * p.H_kv);
  } else {
    u = L % n_kt;
    rest = L / n_kt;
  }
  const int g = rest % p.H_kv, b = rest / p.H_kv;
  // query heads of group g under g(i) = floor(i * H_kv / H_q)
  const int i0 = (int)(((long long)g * p.H_q + p.H_kv - 1) / p.H_kv);
  const int i1 = (int)(((long long)(g + 1) * p.H_q + p.H_kv - 1) / p.H_kv);
  const int n_qt = (p.N + C::BQ - 1) / C::BQ;
  const int t_start = p.causal ? 2 * u : 0;
  const int per_head = n_qt - t_start;
  const int n_steps = (i1 - i0) * per_head;

  WaitCtl ctl{abort_flag, p.status, p.timeout_ns};
  if (tid == 0) {
    // KV_TMEM: the 8 elementwise warps arrive on BAR_KV after writing K / V
    // into TMEM; S and EMPTY then take one commit from each issuer
    for (int i = 0; i < C::N_BARS; ++i) {
      int cnt = 1;
      if (i == C::BAR_P || i == C::BAR_P + 1 || (C::KV_TMEM && i == C::BAR_KV)) cnt = 8;
      else if (C::NI == 2 && ((i >= C::BAR_S && i < C::BAR_S + 2) || (i >= C::BAR_EMPTY && i < C::BAR_EMPTY + C::STAGES))) cnt = 2;
      mbar_init(bar(i), cnt);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
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
      if (!C::KV_TMEM) {
        mbar_arrive_expect_tx(bar(C::BAR_KV), 2 * C::KV_BYTES);
#pragma unroll
        for (int c = 0; c < C::KCH; ++c) {
          tma_load_4d(sbase + C::OFF_K + c * C::KV_CHUNK, &tm_k, bar(C::BAR_KV), c * 64, g, u * 128, b);
          tma_load_4d(sbase + C::OFF_V + c * C::KV_CHUNK, &tm_v, bar(C::BAR_KV), c * 64, g, u * 128, b);
        }
      }
      int filled = 0;
      for (int s = 0; s < n_steps; ++s) {
        const int st = s % C::STAGES, round = s / C::STAGES;
        if (round > 0 && !mbar_wait(bar(C::BAR_EMPTY + st), (round - 1) & 1, ctl)) break;
        const int i = i0 + s / per_head, t = t_start + s % per_head;
        if (!in_bounds(i < p.H_q && t * C::BQ < p.N && g < p.H_kv && b < p.B, p.status)) break;
        const uint32_t dst = sbase + C::OFF_STAGE + st * C::STAGE_BYTES;
        const uint32_t vec = sbase + C::OFF_VEC + st * 2 * C::VEC_BYTES;
        const uint32_t full = bar(C::BAR_FULL + st);
        mbar_arrive_expect_tx(full, C::STAGE_BYTES + 2 * C::VEC_BYTES);
#pragma unroll
        for (int c = 0; c < C::KCH; ++c) {
          tma_load_4d(dst + c * C::T_CHUNK, &tm_q, full, c * 64, i, t * C::BQ, b);
          tma_load_4d(dst + C::T_BYTES + c * C::T_CHUNK, &tm_do, full, c * 64, i, t * C::BQ, b);
        }
        tma_load_2d(vec, &tm_lse2, full, t * C::BQ, b * p.H_q + i);
        tma_load_2d(vec + C::VEC_BYTES, &tm_dsum, full, t * C::BQ, b * p.H_q + i);
        filled = s + 1;
      }
      volatile int zero = 0;
      WaitCtl drain{&zero, p.status, drain_limit_ns(p.timeout_ns)};
      if (!C::KV_TMEM) mbar_wait(bar(C::BAR_KV), 0, drain);
      for (int s = max(0, filled - C::STAGES); s < filled; ++s)
        mbar_wait(bar(C::BAR_FULL + s % C::STAGES), (s / C::STAGES) & 1, drain);
    }
  } else if (warp == 1 || (C::NI == 2 && warp == 3)) {
    if (lane == 0) {
      const int me = warp == 1 ? 0 : 1;
      constexpr uint32_t IDESC_S = idesc_bf16_f32(128, C::BQ, 0, 0);
      constexpr uint32_t IDESC_G = idesc_bf16_f32(128, D, 0, 1);
      // Descriptors are built once; a byte offset `o` inside shared memory is
      // added as o >> 4 to the start-address field (no carry: smem < 256 KB).
      const uint64_t dK = sdesc_sw128(sbase + C::OFF_K, 16, 1024), dV = sdesc_sw128(sbase + C::OFF_V, 16, 1024);
      const uint64_t dQk = sdesc_sw128(sbase + C::OFF_STAGE, 16, 1024);
      const uint64_t dDk = sdesc_sw128(sbase + C::OFF_STAGE + C::T_BYTES, 16, 1024);
      const uint64_t dQm = sdesc_sw128(sbase + C::OFF_STAGE, C::T_CHUNK, 1024);
      const uint64_t dDm = sdesc_sw128(sbase + C::OFF_STAGE + C::T_BYTES, C::T_CHUNK, 1024);
      const uint32_t col_dv = tmem + C::COL_ACC, col_dk = col_dv + D;
      bool ok = mbar_wait(bar(C::BAR_KV), 0, ctl);
      {
        // issuer 0: S^T = K Q_s^T into the buffer's first half, dV += P^T dO_s;
        // issuer 1: dP^T = V dO_s^T into its second half, dK += dS^T Q_s.
        // Each TMEM region has one issuing thread, whose MMAs run in issue order.
        const uint64_t d_score = me ? dDk : dQk, d_grad = me ? dQm : dDm;
        const uint64_t d_kv = me ? dV : dK;
        const uint32_t col_acc = me ? col_dk : col_dv, half = me ? 64u : 0u;
        auto issue_score = [&](int s) -> bool {
          const int st = s % C::STAGES;
          if (!mbar_wait(bar(C::BAR_FULL + st), (s / C::STAGES) & 1, ctl)) return false;
          tc_fence_after();
          const uint64_t so = (uint64_t)(st * (C::STAGE_BYTES >> 4));
          const uint32_t buf = tmem + (uint32_t)(s & 1) * 128 + half;
          if constexpr (C::KV_TMEM) {
            const uint32_t col_a = tmem + (me ? C::COL_VT : C::COL_KT);
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk)
              umma_ts(buf, col_a + kk * 8, d_score + so + (uint64_t)(((kk & 3) * 32) >> 4), IDESC_S, kk > 0);
          } else {
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint64_t ok_ = ((kk >> 2) * C::KV_CHUNK + (kk & 3) * 32) >> 4;
              const uint64_t oq = ((kk >> 2) * C::T_CHUNK + (kk & 3) * 32) >> 4;
              umma_ss(buf, d_kv + ok_, d_score + so + oq, IDESC_S, kk > 0);
            }
          }
          umma_commit(bar(C::BAR_S + (s & 1)));
          return true;
        };
        if (ok) ok = issue_score(0);
        if (ok && n_steps > 1) ok = issue_score(1);
        for (int s = 0; ok && s < n_steps; ++s) {
          if (!mbar_wait_spin(bar(C::BAR_P + (s & 1)), (s >> 1) & 1, ctl)) { ok = false; break; }
          tc_fence_after();
          const int st = s % C::STAGES;
          const uint64_t so = (uint64_t)(st * (C::STAGE_BYTES >> 4));
          const uint32_t buf = tmem + (uint32_t)(s & 1) * 128 + half;
#pragma unroll
          for (int kk = 0; kk < C::BQ / 16; ++kk)
            // queries 16kk.. were packed by warpgroup kk/2 into its 32 columns, chunk kk%2
            // (B operands MN-major: d contiguous)
            umma_ts(col_acc, buf + (uint32_t)(32 * (kk >> 1) + 8 * (kk & 1)), d_grad + so + (uint64_t)((kk * 16 * 128) >> 4),
                    IDESC_G, (s > 0 || kk > 0) ? 1u : 0u);
          umma_commit(bar(C::BAR_EMPTY + st));
          // S^T / dP^T of step s + 2 overwrite what this issuer's own products just read
          if (s + 2 < n_steps) ok = issue_score(s + 2);
        }
      }
      if (ok) umma_commit(bar(C::BAR_DONE + me));
      umma_commit(bar(C::BAR_DRAIN + me));
      volatile int zero = 0;
      WaitCtl drain{&zero, p.status, drain_limit_ns(p.timeout_ns)};
      mbar_wait(bar(C::BAR_DRAIN + me), 0, drain);
    }
  } else if (warp >= 4) {
    const int wg = (warp - 4) >> 2;          // 0: columns 0-31 of each step, 1: columns 32-63
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const int key = u * 128 + row;
    const uint32_t lane_base = tmem + (uint32_t(quarter * 32) << 16);
    const int half = 32 * wg;   // this warpgroup's 32 query columns of every step
    const float sl2 = p.scale_log2;
    if constexpr (C::KV_TMEM) {
      // this key's row of K (warpgroup 0) or V (warpgroup 1) into its TMEM lane; zero past N
      static_assert(D == 64, "one 32-column TMEM store per row");
      const __nv_bfloat16* src = (wg == 0 ? p.k : p.v) + (((size_t)b * p.N + (key < p.N ? key : 0)) * p.H_kv + g) * D;
      const uint4* s4 = reinterpret_cast<const uint4*>(src);
      uint32_t r[D / 2];
#pragma unroll
      for (int x = 0; x < D / 8; ++x) {
        const uint4 a = key < p.N ? s4[x] : make_uint4(0u, 0u, 0u, 0u);
        r[4 * x] = a.x; r[4 * x + 1] = a.y; r[4 * x + 2] = a.z; r[4 * x + 3] = a.w;
      }
      __syncwarp();   // the TMEM store is warp-collective
      tmem_st32(lane_base + (wg == 0 ? C::COL_KT : C::COL_VT), r);
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(C::BAR_KV));
    }
    bool ok = true;
    for (int s = 0; s < n_steps; ++s) {
      const int st = s % C::STAGES;
      const int t = t_start + s % per_head;
      const uint32_t buf = lane_base + (uint32_t)(s & 1) * 128 + (uint32_t)half;
      if (!mbar_wait_warp(bar(C::BAR_S + (s & 1)), (s >> 1) & 1, ctl) ||
          !mbar_wait_warp(bar(C::BAR_FULL + st), (s / C::STAGES) & 1, ctl)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const float4* vl4 = reinterpret_cast<const float4*>(smem + C::OFF_VEC + st * 2 * C::VEC_BYTES) + half / 4;
      const float4* vd4 = vl4 + C::BQ / 4;
      // a key above a query of the step only on the two diagonal tiles; ragged ends
      const bool need_mask = (p.causal && t < 2 * u + 2) || (t * C::BQ + C::BQ > p.N) || (key >= p.N);
      // two 16-column chunks; chunk 1's TMEM load is in flight while chunk 0 is computed
      uint32_t a0[16], b0[16], a1[16], b1[16];
      tmem_ld16x2_nowait(buf, buf + 64, a0, b0);
      tmem_ld_wait16x2(a0, b0);
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        uint32_t(&ra)[16] = k ? a1 : a0;
        uint32_t(&rb)[16] = k ? b1 : b0;
        if (k == 0) tmem_ld16x2_nowait(buf + 16, buf + 64 + 16, a1, b1);
        // masked scores become -inf (p = 0) in a pass of their own, so the
        // arithmetic stays one straight block
        if (need_mask) {
#pragma unroll
          for (int x = 0; x < 16; ++x) {
            const int q = t * C::BQ + half + k * 16 + x;
            if (q >= p.N || key >= p.N || (p.causal && key > q)) ra[x] = __float_as_uint(-INFINITY);
          }
        }
        float2 nl[8], nd[8];
#pragma unroll
        for (int w = 0; w < 4; ++w) {
          const float4 l4 = vl4[k * 4 + w], d4 = vd4[k * 4 + w];
          nl[2 * w] = make_float2(l4.x, l4.y);
          nl[2 * w + 1] = make_float2(l4.z, l4.w);
          nd[2 * w] = make_float2(d4.x, d4.y);
          nd[2 * w + 1] = make_float2(d4.z, d4.w);
        }
        uint32_t pp[8], pd[8];
        bwd_chunk(ra, rb, sl2, nl, nd, pp, pd);
        // chunk k packs into [8k, 8k + 8) of this half: behind the columns already read
        tmem_st8(buf + k * 8, pp);
        tmem_st8(buf + 64 + k * 8, pd);
        if (k == 0) tmem_ld_wait16x2(a1, b1);
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(C::BAR_P + (s & 1)));
    }
    // epilogue: warpgroup 0 writes dV, warpgroup 1 writes dK (x scale)
    if (ok && mbar_wait_warp(bar(C::BAR_DONE), 0, ctl) && (C::NI == 1 || mbar_wait_warp(bar(C::BAR_DONE + 1), 0, ctl))) {
      tc_fence_after();
      const bool store = key < p.N && in_bounds(g < p.H_kv && b < p.B, p.status);
      const size_t base = (((size_t)b * p.N + (store ? key : 0)) * p.H_kv + g) * D;
      __nv_bfloat16* dst = (wg == 0 ? p.dv : p.dk) + base;
      const float mul = wg == 0 ? 1.0f : p.scale;
      const uint32_t col0 = lane_base + C::COL_ACC + (wg == 0 ? 0u : (uint32_t)D);
#pragma unroll
      for (int c = 0; c < D; c += 32) {
        uint32_t r[32];
        __syncwarp();   // after the per-lane stores: the TMEM load is warp-collective
        tmem_ld32(col0 + c, r);
        uint4 w[4];
        uint32_t* wp = reinterpret_cast<uint32_t*>(w);
#pragma unroll
        for (int x = 0; x < 16; ++x)
          wp[x] = pack_bf16x2(__uint_as_float(r[2 * x]) * mul, __uint_as_float(r[2 * x + 1]) * mul);
        if (store) {
          uint4* d4 = reinterpret_cast<uint4*>(dst + c);
#pragma unroll
          for (int x = 0; x < 4; ++x) d4[x] = w[x];
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// ---------------------------------------------------------------- dQ
template <int D>
struct DqCfg {
  static constexpr int KCH = D / 64;
  // Issuer 0 issues S, issuer 1 issues dP and dQ, so one dQ accumulator
  // suffices and the TMEM it frees holds 96-key steps.
  static constexpr int BK = 96;                        // keys per step
  static constexpr int STAGES = (D == 64) ? 8 : 3;
  // d = 64: Q and dO live in TMEM as the A operands of the score products (TS
  // form); at d = 128 the score buffers and the dQ accumulator fill TMEM and
  // they stay in shared memory (SS form).
  static constexpr bool A_TMEM = (D == 64);
  static constexpr int Q_BYTES = 128 * D * 2;          // Q or dO tile, 128 rows
  static constexpr int Q_CHUNK = 128 * 128;
  static constexpr int T_BYTES = BK * D * 2;           // K_j or V_j, BK keys
  static constexpr int T_CHUNK = BK * 128;
  static constexpr int STAGE_BYTES = 2 * T_BYTES;
  static constexpr int OFF_Q = 0, OFF_DO = Q_BYTES, OFF_STAGE = A_TMEM ? 0 : 2 * Q_BYTES;
  static constexpr int OFF_BAR = OFF_STAGE + STAGES * STAGE_BYTES;
  static constexpr int BAR_QD = 0, BAR_FULL = 1, BAR_EMPTY = 1 + STAGES, BAR_S = 1 + 2 * STAGES,
                       BAR_P = BAR_S + 2, BAR_DONE = BAR_P + 2, BAR_DRAIN = BAR_DONE + 2, N_BARS = BAR_DRAIN + 2;
  static constexpr int OFF_MISC = OFF_BAR + N_BARS * 8;
  static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;
  static constexpr int THREADS = 384;
  static constexpr uint32_t TMEM_COLS = 512;
  // TMEM buffer b at b * BUF: scores in [0, BK), dP in [BK, 2 BK). Then the dQ
  // accumulator, then the Q / dO rows (A_TMEM).
  static constexpr uint32_t BUF = 2 * BK;
  static constexpr uint32_t COL_DQ = 2 * BUF, COL_QT = COL_DQ + D, COL_DOT = COL_QT + D / 2;
  static_assert(COL_DQ + D <= TMEM_COLS && (!A_TMEM || COL_DOT + D / 2 <= TMEM_COLS), "TMEM budget");
  // elementwise: each warpgroup owns CPW key columns of a step, in NCH chunks
  // of 16; chunk k of warpgroup w packs its dS into [w*CPW + 8k, +8) of the
  // buffer's dP half, behind the columns it has already read
  static constexpr int CPW = BK / 2, NCH = CPW / 16;
  static_assert(CPW % 16 == 0, "chunking");
  __host__ __device__ static constexpr uint32_t ds_col(int kk) {
    return (uint32_t)((16 * kk / CPW) * CPW + 8 * ((16 * kk % CPW) / 16));
  }
  static_assert(STAGE_BYTES % 1024 == 0 && OFF_STAGE % 1024 == 0, "tile alignment");
};

// One CTA per 128-row query tile: P heads of one group stacked as in the
// forward (row r = token_local * P + head offset), so each K/V tile serves all
// P heads. Steps walk BK-key tiles (96 at d = 64, 64 at d = 128):
// S = Q K_j^T, dP = dO V_j^T, then dQ += dS K_j with dS read from TMEM.
template <int D>
__global__ void __launch_bounds__(384, 1)
    bwd_dq_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
                  const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                  const BwdParams p) {
  using C = DqCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile uint32_t* tmem_slot = misc;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);
  auto bar = [&](int i) { return smem_u32(&bars[i]); };
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  // ---- work item (query tile qt, head block hb, batch b); causal: longest first
  const int n_qt = (p.N + p.tpt - 1) / p.tpt;
  const int L = blockIdx.x;
  int qt, rest;
  if (p.causal) {
    qt = n_qt - 1 - L / (p.B * p.n_hb);
    rest = L % (p.B * p.n_hb);
  } else {
    qt = L % n_qt;
    rest = L / n_qt;
  }
  const int hb = rest % p.n_hb, b = rest / p.n_hb;
  const int head0 = hb * p.P;
  const int g = (int)(((long long)head0 * p.H_kv) / p.H_q);
  const int t0 = qt * p.tpt;
  const int t_last = min(p.N - 1, t0 + p.tpt - 1);
  const int n_kv = p.causal ? (t_last / C::BK + 1) : (p.N + C::BK - 1) / C::BK;

  WaitCtl ctl{abort_flag, p.status, p.timeout_ns};
  if (tid == 0) {
    // S and EMPTY take one commit from each issuer
    for (int i = 0; i < C::N_BARS; ++i) {
      int cnt = 1;
      if (i == C::BAR_P || i == C::BAR_P + 1 || (C::A_TMEM && i == C::BAR_QD)) cnt = 8;
      else if ((i >= C::BAR_S && i < C::BAR_S + 2) || (i >= C::BAR_EMPTY && i < C::BAR_EMPTY + C::STAGES))
        cnt = 2;
      mbar_init(bar(i), cnt);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
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
      if (!C::A_TMEM) {
        mbar_arrive_expect_tx(bar(C::BAR_QD), 2 * C::Q_BYTES);
#pragma unroll
        for (int c = 0; c < C::KCH; ++c) {
          if (!in_bounds(head0 + p.P <= p.H_q && t0 < p.N && b < p.B, p.status)) break;
          tma_load_4d(sbase + C::OFF_Q + c * C::Q_CHUNK, &tm_q, bar(C::BAR_QD), c * 64, head0, t0, b);
          tma_load_4d(sbase + C::OFF_DO + c * C::Q_CHUNK, &tm_do, bar(C::BAR_QD), c * 64, head0, t0, b);
        }
      }
      int filled = 0;
      for (int j = 0; j < n_kv; ++j) {
        const int st = j % C::STAGES, round = j / C::STAGES;
        if (round > 0 && !mbar_wait(bar(C::BAR_EMPTY + st), (round - 1) & 1, ctl)) break;
        if (!in_bounds(j * C::BK < p.N && g < p.H_kv && b < p.B, p.status)) break;
        const uint32_t dst = sbase + C::OFF_STAGE + st * C::STAGE_BYTES;
        const uint32_t full = bar(C::BAR_FULL + st);
        mbar_arrive_expect_tx(full, C::STAGE_BYTES);
#pragma unroll
        for (int c = 0; c < C::KCH; ++c) {
          tma_load_4d(dst + c * C::T_CHUNK, &tm_k, full, c * 64, g, j * C::BK, b);
          tma_load_4d(dst + C::T_BYTES + c * C::T_CHUNK, &tm_v, full, c * 64, g, j * C::BK, b);
        }
        filled = j + 1;
      }
      volatile int zero = 0;
      WaitCtl drain{&zero, p.status, drain_limit_ns(p.timeout_ns)};
      if (!C::A_TMEM) mbar_wait(bar(C::BAR_QD), 0, drain);
      for (int j = max(0, filled - C::STAGES); j < filled; ++j)
        mbar_wait(bar(C::BAR_FULL + j % C::STAGES), (j / C::STAGES) & 1, drain);
    }
  } else if (warp == 1 || warp == 3) {
    if (lane == 0) {
      const int me = warp == 1 ? 0 : 1;
      constexpr uint32_t IDESC_S = idesc_bf16_f32(128, C::BK, 0, 0);
      constexpr uint32_t IDESC_G = idesc_bf16_f32(128, D, 0, 1);
      // descriptors built once; offsets added as o >> 4 (see the dK/dV kernel)
      const uint64_t dQ = sdesc_sw128(sbase + C::OFF_Q, 16, 1024), dO = sdesc_sw128(sbase + C::OFF_DO, 16, 1024);
      const uint64_t dKk = sdesc_sw128(sbase + C::OFF_STAGE, 16, 1024);
      const uint64_t dVk = sdesc_sw128(sbase + C::OFF_STAGE + C::T_BYTES, 16, 1024);
      const uint64_t dKm = sdesc_sw128(sbase + C::OFF_STAGE, C::T_CHUNK, 1024);
      bool ok = mbar_wait(bar(C::BAR_QD), 0, ctl);
      {
        // issuer 0: S_j = Q K_j^T into the buffer's first half; issuer 1:
        // dP_j = dO V_j^T into its second half, then dQ += dS_j K_j with dS_j
        // read from that half. Each half has one issuing thread, so in-order
        // issue puts dP(j + 2) after the dQ(j) that read the same columns.
        auto issue_score = [&](int j) -> bool {
          const int st = j % C::STAGES;
          if (!mbar_wait(bar(C::BAR_FULL + st), (j / C::STAGES) & 1, ctl)) return false;
          tc_fence_after();
          const uint64_t so = (uint64_t)(st * (C::STAGE_BYTES >> 4));
          const uint32_t dst = tmem + (uint32_t)(j & 1) * C::BUF + (me ? (uint32_t)C::BK : 0u);
          const uint64_t b_desc = me ? dVk : dKk;
          if constexpr (C::A_TMEM) {
            const uint32_t a_col = tmem + (me ? C::COL_DOT : C::COL_QT);
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk)
              umma_ts(dst, a_col + kk * 8, b_desc + so + (uint64_t)(((kk & 3) * 32) >> 4), IDESC_S, kk > 0);
          } else {
            const uint64_t a_desc = me ? dO : dQ;
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint64_t oq = ((kk >> 2) * C::Q_CHUNK + (kk & 3) * 32) >> 4;
              const uint64_t ok_ = ((kk >> 2) * C::T_CHUNK + (kk & 3) * 32) >> 4;
              umma_ss(dst, a_desc + oq, b_desc + so + ok_, IDESC_S, kk > 0);
            }
          }
          umma_commit(bar(C::BAR_S + (j & 1)));
          return true;
        };
        if (me == 0) {
          for (int j = 0; ok && j < n_kv; ++j) {
            // buffer j & 1 is free once the elementwise warps have read S(j - 2)
            if (j >= 2 && !mbar_wait_spin(bar(C::BAR_P + (j & 1)), ((j - 2) >> 1) & 1, ctl)) { ok = false; break; }
            if (!issue_score(j)) { ok = false; break; }
            umma_commit(bar(C::BAR_EMPTY + j % C::STAGES));
          }
        } else {
          if (ok && n_kv > 0) ok = issue_score(0);
          if (ok && n_kv > 1) ok = issue_score(1);
          for (int j = 0; ok && j < n_kv; ++j) {
            if (!mbar_wait_spin(bar(C::BAR_P + (j & 1)), (j >> 1) & 1, ctl)) { ok = false; break; }
            tc_fence_after();
            const int st = j % C::STAGES;
            const uint64_t so = (uint64_t)(st * (C::STAGE_BYTES >> 4));
            const uint32_t ds = tmem + (uint32_t)(j & 1) * C::BUF + (uint32_t)C::BK;
#pragma unroll
            for (int kk = 0; kk < C::BK / 16; ++kk)
              // dQ += dS K_j (K as an MN-major B operand: d contiguous)
              umma_ts(tmem + C::COL_DQ, ds + C::ds_col(kk), dKm + so + (uint64_t)((kk * 16 * 128) >> 4), IDESC_G,
                      (j > 0 || kk > 0) ? 1u : 0u);
            umma_commit(bar(C::BAR_EMPTY + st));
            if (j + 2 < n_kv) ok = issue_score(j + 2);
          }
        }
      }
      if (ok) umma_commit(bar(C::BAR_DONE + me));
      umma_commit(bar(C::BAR_DRAIN + me));
      volatile int zero = 0;
      WaitCtl drain{&zero, p.status, drain_limit_ns(p.timeout_ns)};
      mbar_wait(bar(C::BAR_DRAIN + me), 0, drain);
    }
  } else if (warp >= 4) {
    const int wg = (warp - 4) >> 2;
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const int token = t0 + (row >> p.log2P);
    const int head = head0 + (row & (p.P - 1));
    const bool row_ok = token < p.N;
    const uint32_t lane_base = tmem + (uint32_t(quarter * 32) << 16);
    const int half = C::CPW * wg;   // this warpgroup's first key column of every step
    const float sl2 = p.scale_log2;
    float nl_r = 0.f, nd_r = 0.f;
    if (row_ok) {
      const size_t ri = ((size_t)b * p.H_q + head) * p.ld + token;
      nl_r = p.nlse2[ri];
      nd_r = p.ndsum[ri];
    }
    if (C::A_TMEM) {
      // this row of Q (warpgroup 0) or dO (warpgroup 1) into the TMEM lane
      const __nv_bfloat16* src = (wg == 0 ? p.q : p.dout) + (((size_t)b * p.N + (row_ok ? token : 0)) * p.H_q + head) * D;
      uint32_t r[32];
      const uint4* s4 = reinterpret_cast<const uint4*>(src);
#pragma unroll
      for (int x = 0; x < 8; ++x) {
        const uint4 a = row_ok ? s4[x] : make_uint4(0u, 0u, 0u, 0u);
        r[4 * x] = a.x; r[4 * x + 1] = a.y; r[4 * x + 2] = a.z; r[4 * x + 3] = a.w;
      }
      __syncwarp();   // the TMEM store is warp-collective
      tmem_st32(lane_base + (wg == 0 ? C::COL_QT : C::COL_DOT), r);
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(C::BAR_QD));
    }
    float2 nl[8], nd[8];
#pragma unroll
    for (int w = 0; w < 8; ++w) {
      nl[w] = make_float2(nl_r, nl_r);
      nd[w] = make_float2(nd_r, nd_r);
    }
    bool ok = true;
    for (int j = 0; j < n_kv; ++j) {
      // this warpgroup's score columns of buffer j & 1, and its dP columns
      const uint32_t buf = lane_base + (uint32_t)(j & 1) * C::BUF + (uint32_t)half;
      const uint32_t dpb = buf + (uint32_t)C::BK;
      if (!mbar_wait_warp(bar(C::BAR_S + (j & 1)), (j >> 1) & 1, ctl)) { ok = false; break; }
      tc_fence_after();
      // keys above t0 only in the last tiles when causal; keys past N in the last tile
      const bool need_mask = !row_ok || (j * C::BK + C::BK > p.N) || (p.causal && j * C::BK + C::BK - 1 > t0);
      // NCH 16-column chunks; chunk k + 1's TMEM load is in flight while chunk k is computed
      uint32_t ra2[2][16], rb2[2][16];
      tmem_ld16x2_nowait(buf, dpb, ra2[0], rb2[0]);
      tmem_ld_wait16x2(ra2[0], rb2[0]);
#pragma unroll
      for (int k = 0; k < C::NCH; ++k) {
        uint32_t(&ra)[16] = ra2[k & 1];
        uint32_t(&rb)[16] = rb2[k & 1];
        if (k + 1 < C::NCH) tmem_ld16x2_nowait(buf + 16 * (k + 1), dpb + 16 * (k + 1), ra2[(k + 1) & 1], rb2[(k + 1) & 1]);
        if (need_mask) {   // masked scores -> -inf (p = 0), outside the arithmetic block
#pragma unroll
          for (int x = 0; x < 16; ++x) {
            const int key = j * C::BK + half + k * 16 + x;
            if (!row_ok || key >= p.N || (p.causal && key > token)) ra[x] = __float_as_uint(-INFINITY);
          }
        }
        uint32_t pp[8], pd[8];
        bwd_chunk(ra, rb, sl2, nl, nd, pp, pd);
        // dS of chunk k into [8k, 8k + 8) of this warpgroup's dP columns (already read)
        tmem_st8(dpb + k * 8, pd);
        if (k + 1 < C::NCH) tmem_ld_wait16x2(ra2[(k + 1) & 1], rb2[(k + 1) & 1]);
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(C::BAR_P + (j & 1)));
    }
    // epilogue: each warpgroup writes half of the row's d columns (x scale) of
    // issuer 1's accumulator
    const bool acc_ready = ok && mbar_wait_warp(bar(C::BAR_DONE + 1), 0, ctl);
    if (acc_ready) {
      tc_fence_after();
      const bool st = row_ok && in_bounds(head < p.H_q && b < p.B, p.status);
      __nv_bfloat16* dst = p.dq + (((size_t)b * p.N + (st ? token : 0)) * p.H_q + (st ? head : 0)) * D;
#pragma unroll
      for (int c = wg * (D / 2); c < (wg + 1) * (D / 2); c += 32) {
        uint32_t r[32];
        __syncwarp();   // after the per-lane stores: the TMEM load is warp-collective
        tmem_ld32(lane_base + C::COL_DQ + c, r);
        uint4 w[4];
        uint32_t* wp = reinterpret_cast<uint32_t*>(w);
#pragma unroll
        for (int x = 0; x < 16; ++x)
          wp[x] = pack_bf16x2(__uint_as_float(r[2 * x]) * p.scale, __uint_as_float(r[2 * x + 1]) * p.scale);
        if (st) {
          uint4* d4 = reinterpret_cast<uint4*>(dst + c);
#pragma unroll
          for (int x = 0; x < 4; ++x) d4[x] = w[x];
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace sqa
