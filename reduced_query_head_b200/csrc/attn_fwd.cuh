// Forward attention with decoupled head counts on sm_100a.
//
// out[b,t,i,:] = softmax_u(scale * q[b,t,i,:] . k[b,u,g(i),:]) v[b,u,g(i),:],
// g(i) = floor(i * H_kv / H_q), keys u in [0, N) or u <= t when causal.
// This is scaled-dot-product attention with per-group key/value sharing as in
// the GQA explainer ("MHA・MQA・GQAの関係" equations and the head-to-group
// diagram); Sparse Query Attention is the same computation with fewer query
// heads ("Sparse Query Attention (SQA)", abstract).
//
// One CTA owns two 128-row query tiles of one (batch, head block), or one
// tile when the host splits the last non-causal pairs to fill the final wave. A head
// block is P consecutive query heads of one KV group (P a power of two
// dividing H_q/H_kv), stacked so that tile row r = token_local * P + head
// offset: every key/value tile brought into shared memory serves all P heads.
//
// Warp roles (12 warps):
//   warp 0   TMA producer: Q0/Q1 once, then K_j and V_j into a ring of stages
//   warps 1, 3  MMA issuers, one per query tile k: S_k = Q_k K_j^T into TMEM,
//            O_k += P_k V_j with P_k read from TMEM
//   warp 2   owns the TMEM allocation
//   warps 4-7 / 8-11  softmax for tile 0 / tile 1 (thread = row = TMEM lane):
//            online softmax with a lazily rescaled running max, P written
//            back to TMEM as bf16, epilogue O / l -> bf16 -> global.
// Each tile's S, P and O have TMEM columns of their own, so S_k(j+1) is issued
// as soon as softmax k has read S_k(j) and overlaps softmax(j). A step takes
// BN keys: 128 at d=64; 80 at d=128, the widest step whose S, P and O for two
// tiles fit the 512 columns.
//
// TMEM columns, d=64:  S0 [0,128), S1 [128,256), O0 [256,320), O1 [320,384),
//                      P0 [384,448), P1 [448,512);
//               d=128: S0 [0,80), P0 [80,120), S1 [128,208), P1 [208,248),
//                      O0 [256,384), O1 [384,512).
// Every wait is bounded; on time-out the kernel records the status, drains
// its own copies and MMAs, frees TMEM and returns.
#pragma once

#include "sm100.cuh"

namespace sqa {

struct AttnParams {
  __nv_bfloat16* out;   // [B, N, H_q, D]
  int B, N, H_q, H_kv;  // N: query rows of this call
  int Nk;               // keys (N_k >= q0 + N); N_k = N and q0 = 0 for whole-sequence attention
  int q0;               // global position of query row 0 (causal masks compare global positions)
  int P, log2P;         // heads stacked per tile
  int tpt;              // tokens per 128-row tile = 128 / P
  int n_pairs;          // tile pairs per (batch, head block)
  // This launch runs pair items item0, item0 + 1, ...: one unit per pair, or
  // (singles) one unit per tile of a pair. With kv_split = 2 (non-causal, a
  // cluster of two CTAs per unit) each CTA of the cluster takes half of the
  // key tiles and rank 1 hands its partial rows to rank 0, which merges them.
  int item0, singles, kv_split;
  int n_hb;             // head blocks = H_q / P
  int causal;
  float scale_log2;     // scale * log2(e)
  float* lse;           // optional [B, H_q, N]: natural log of sum_u exp(scale q.k_u), or nullptr
  // optional, layer mode: after its rows are stored, each tile adds its count of
  // stored (token, head) rows to ready[(b * N + token) / 128] (release), for the
  // output projection launched as this grid's programmatic dependent
  int* ready;
  int* status;
  unsigned long long timeout_ns;
};

template <int D>
struct AttnCfg {
  static constexpr int BM = 128;
  static constexpr int BN = (D == 64) ? 128 : 80;      // keys per step
  static constexpr int KCH = D / 64;                    // 128-byte column chunks
  static constexpr int STAGES = (D == 64) ? 4 : 3;
  static constexpr int Q_BYTES = BM * D * 2;            // one Q tile
  static constexpr int KV_BYTES = BN * D * 2;           // one K (or V) tile
  static constexpr int CHUNK_Q = BM * 128;              // bytes per column chunk
  static constexpr int CHUNK_KV = BN * 128;
  // shared-memory map (offsets from a 1024-aligned base)
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + 2 * Q_BYTES;
  static constexpr int OFF_V = OFF_K + STAGES * KV_BYTES;
  static constexpr int OFF_BAR = OFF_V + STAGES * KV_BYTES;
  // barriers
  static constexpr int BAR_Q = 0;
  static constexpr int BAR_KF = 1;                      // [STAGES] K tile landed
  static constexpr int BAR_VF = BAR_KF + STAGES;        // [STAGES] V tile landed
  static constexpr int BAR_KVE = BAR_VF + STAGES;       // [STAGES] stage free again
  static constexpr int BAR_S = BAR_KVE + STAGES;        // [2] S_k ready in TMEM
  static constexpr int BAR_SFREE = BAR_S + 2;           // [2] S_k read out by softmax (4 warps)
  static constexpr int BAR_P = BAR_SFREE + 2;           // [2] P_k written, O_k corrected (4 warps)
  static constexpr int BAR_PV = BAR_P + 2;              // [2] O_k += P_k V done
  static constexpr int BAR_O = BAR_PV + 2;              // [2] last PV of tile k done
  static constexpr int BAR_DRAIN = BAR_O + 2;            // [2] per MMA thread
  static constexpr int N_BARS = BAR_DRAIN + 2;
  static constexpr int OFF_MISC = OFF_BAR + N_BARS * 8;  // tmem base (u32), abort flag (u32)
  static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;  // + alignment slack
  static constexpr int THREADS = 384;
  static constexpr int REGS_LAUNCH = 168, REGS_CTRL = 56, REGS_SOFTMAX = 224;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t COL_S0 = 0, COL_S1 = 128;
  static constexpr uint32_t COL_O0 = 256, COL_O1 = 256 + D;
  // d=64: P0/P1 after the accumulators; d=128 (80-key steps): each P right after its S
  static constexpr uint32_t COL_P0 = (D == 64) ? 256 + 2 * D : BN;
  static constexpr uint32_t COL_P1 = (D == 64) ? 256 + 2 * D + 64 : 128 + BN;
  static_assert(COL_P0 + BN / 2 <= ((D == 64) ? COL_P1 : COL_S1), "TMEM map");
  static_assert(COL_P1 + BN / 2 <= ((D == 64) ? TMEM_COLS : COL_O0), "TMEM map");
  static_assert(COL_O1 + D <= ((D == 64) ? COL_P0 : TMEM_COLS), "TMEM map");
};

// EMU: bit u of this mask set = column pair u of every 8 takes 2^x from the
// polynomial on the FMA pipe instead of the MUFU unit.
template <int D, int EMU>
__global__ void __launch_bounds__(384, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const AttnParams p) {
  using C = AttnCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile uint32_t* tmem_slot = misc;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);
  auto bar = [&](int i) { return smem_u32(&bars[i]); };

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  // A dependent launch (the last wave's split units, the layer's output
  // projection) may be scheduled once every CTA of this grid has started: it
  // then takes only SMs this grid's last wave frees. It reads nothing this grid
  // writes, except row blocks it waits for by their counters.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  // ---- work item
  // Causal: query-tile pair outermost, longest first, so the short items fill
  // the tail. Non-causal: all items cost the same, so the query-tile pair is
  // innermost and CTAs running together read the same head block's K/V from L2.
  // The pairs left for a last, partial wave of a non-causal grid run in a
  // second launch whose units split the keys over two CTAs (the host decides).
  const int split = p.kv_split;
  const int rank = split > 1 ? (int)cluster_rank() : 0;
  const int unit = (int)blockIdx.x / split;
  int item, single = -1;
  if (p.singles) {
    item = p.item0 + (unit >> 1);
    single = unit & 1;                   // which tile of the pair this unit runs
  } else {
    item = p.item0 + unit;
  }
  int qp, rest;
  if (p.causal) {
    const int per_pair = p.n_hb * p.B;
    qp = item / per_pair;
    rest = item - qp * per_pair;
    qp = p.n_pairs - 1 - qp;
  } else {
    qp = item % p.n_pairs;
    rest = item / p.n_pairs;
  }
  const int hb = rest % p.n_hb;
  const int b = rest / p.n_hb;
  const int head0 = hb * p.P;
  const int g = (int)(((long long)head0 * p.H_kv) / p.H_q);
  const int n_kv_all = (p.Nk + C::BN - 1) / C::BN;
  int t0[2], n_kv[2];
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    t0[k] = (qp * 2 + k) * p.tpt;
    if (single >= 0) t0[k] = (k == 0) ? (qp * 2 + single) * p.tpt : p.N;  // one tile, in slot 0
    if (t0[k] >= p.N) {
      n_kv[k] = 0;
    } else if (p.causal) {
      const int last = p.q0 + min(t0[k] + p.tpt - 1, p.N - 1);  // global position of the tile's last row
      n_kv[k] = min(last / C::BN + 1, n_kv_all);
    } else {
      n_kv[k] = n_kv_all;
    }
  }
  // Split units (non-causal, at least two key tiles): rank 0 takes key tiles
  // [0, half), rank 1 [half, n_kv_all).
  int kv0 = 0;
  if (split > 1) {
    const int half = n_kv_all / 2;
    kv0 = rank ? half : 0;
#pragma unroll
    for (int k = 0; k < 2; ++k)
      if (n_kv[k] > 0) n_kv[k] = rank ? n_kv_all - half : half;
  }
  const int n_max = max(n_kv[0], n_kv[1]);

  WaitCtl ctl{abort_flag, p.status, p.timeout_ns};

  if (tid == 0) {
    const uint32_t active_tiles = (n_kv[0] > 0) + (n_kv[1] > 0);
    for (int i = 0; i < C::N_BARS; ++i) {
      const bool per_warp = (i >= C::BAR_SFREE && i < C::BAR_SFREE + 2) || (i >= C::BAR_P && i < C::BAR_P + 2);
      const bool kv_empty = i >= C::BAR_KVE && i < C::BAR_KVE + C::STAGES;
      // a K/V stage is free once every MMA thread that uses it has committed it
      mbar_init(bar(i), per_warp ? 4 : (kv_empty && active_tiles > 1) ? 2 : 1);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 2) {
    tmem_alloc(smem_u32((const void*)tmem_slot), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // Register split: the kernel launches with REGS_LAUNCH per thread (the host
  // checks this before launching). Warpgroup 0 (producer, MMA, TMEM owner)
  // gives registers back, the two softmax warpgroups take them:
  // 128*REGS_CTRL + 256*REGS_SOFTMAX <= 384*REGS_LAUNCH.
  static_assert(128 * C::REGS_CTRL + 256 * C::REGS_SOFTMAX <= 384 * C::REGS_LAUNCH, "register split");
  if (warp < 4) regs_release<C::REGS_CTRL>();

  if (warp == 0) {
    // ======================= TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      // Q of the tiles that have rows (a pair's second tile may lie past N)
      mbar_arrive_expect_tx(bar(C::BAR_Q), ((n_kv[0] > 0) + (n_kv[1] > 0)) * C::Q_BYTES);
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        if (n_kv[k] == 0) continue;
#pragma unroll
        for (int c = 0; c < C::KCH; ++c) {
          // a failed check loads nothing: the barrier then never completes, and
          // the waits on it end by their time limit
          if (!in_bounds(head0 + p.P <= p.H_q && t0[k] >= 0 && t0[k] < p.N && b < p.B, p.status)) continue;
          tma_load_4d(sbase + C::OFF_Q + k * C::Q_BYTES + c * C::CHUNK_Q, &tm_q, bar(C::BAR_Q), c * 64, head0,
                      t0[k], b);
        }
      }
      int filled = 0;
      for (int j = 0; j < n_max; ++j) {
        const int s = j % C::STAGES;
        const int round = j / C::STAGES;
        if (round > 0 && !mbar_wait(bar(C::BAR_KVE + s), (round - 1) & 1, ctl)) break;
        if (!in_bounds((kv0 + j) * C::BN < p.Nk && g < p.H_kv && s < C::STAGES, p.status)) break;
        mbar_arrive_expect_tx(bar(C::BAR_KF + s), C::KV_BYTES);
#pragma unroll
        for (int c = 0; c < C::KCH; ++c)
          tma_load_4d(sbase + C::OFF_K + s * C::KV_BYTES + c * C::CHUNK_KV, &tm_k, bar(C::BAR_KF + s), c * 64, g,
                      (kv0 + j) * C::BN, b);
        mbar_arrive_expect_tx(bar(C::BAR_VF + s), C::KV_BYTES);
#pragma unroll
        for (int c = 0; c < C::KCH; ++c)
          tma_load_4d(sbase + C::OFF_V + s * C::KV_BYTES + c * C::CHUNK_KV, &tm_v, bar(C::BAR_VF + s), c * 64, g,
                      (kv0 + j) * C::BN, b);
        filled = j + 1;
      }
      // Drain: wait (bounded) for the copies this thread issued, so none lands after exit.
      volatile int zero = 0;
      WaitCtl drain{&zero, p.status, drain_limit_ns(p.timeout_ns)};
      mbar_wait(bar(C::BAR_Q), 0, drain);
      for (int j = max(0, filled - C::STAGES); j < filled; ++j) {
        const int s = j % C::STAGES;
        mbar_wait(bar(C::BAR_KF + s), (j / C::STAGES) & 1, drain);
        mbar_wait(bar(C::BAR_VF + s), (j / C::STAGES) & 1, drain);
      }
    }
  } else if (warp == 1 || warp == 3) {
    // ======================= MMA issuers: one thread per tile
    // Each tile's S/PV chain runs on its own thread, so a slow step of one
    // tile never holds up the other (issue blocks until the tensor core
    // accepts the MMA). Both threads feed the same tensor core; they touch
    // disjoint TMEM columns and meet only on the K/V stage barriers.
    const int k = warp == 1 ? 0 : 1;
    if (lane == 0) {
      constexpr uint32_t IDESC_S = idesc_bf16_f32(C::BM, C::BN, 0, 0);
      constexpr uint32_t IDESC_O = idesc_bf16_f32(C::BM, D, 0, 1);
      const uint32_t col_s = k ? C::COL_S1 : C::COL_S0;
      const uint32_t col_o = k ? C::COL_O1 : C::COL_O0;
      const uint32_t col_p = k ? C::COL_P1 : C::COL_P0;
      const int nk = n_kv[k];
      // Descriptors are built once; a byte offset o inside shared memory is
      // added as o >> 4 to the start-address field (no carry: smem < 256 KB).
      const uint64_t dq = sdesc_sw128(sbase + C::OFF_Q + k * C::Q_BYTES, 16, 1024);
      const uint64_t dk0 = sdesc_sw128(sbase + C::OFF_K, 16, 1024);
      const uint64_t dv0 = sdesc_sw128(sbase + C::OFF_V, C::CHUNK_KV, 1024);
      auto issue_s = [&](int s) {
        const uint64_t dk = dk0 + (uint64_t)((s * C::KV_BYTES) >> 4);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t off = ((kk >> 2) * C::CHUNK_Q + (kk & 3) * 32) >> 4;
          const uint64_t offk = ((kk >> 2) * C::CHUNK_KV + (kk & 3) * 32) >> 4;
          umma_ss(tmem + col_s, dq + off, dk + offk, IDESC_S, kk > 0);
        }
      };
      auto issue_pv = [&](int s, int j) {
        const uint64_t dv = dv0 + (uint64_t)((s * C::KV_BYTES) >> 4);
#pragma unroll
        for (int kk = 0; kk < C::BN / 16; ++kk) {
          umma_ts(tmem + col_o, tmem + col_p + kk * 8, dv + (uint64_t)((kk * 16 * 128) >> 4), IDESC_O,
                  (j > 0 || kk > 0) ? 1u : 0u);
        }
      };
      bool ok = nk > 0 && mbar_wait(bar(C::BAR_Q), 0, ctl) && mbar_wait(bar(C::BAR_KF + 0), 0, ctl);
      if (ok) {
        tc_fence_after();
        issue_s(0);
        umma_commit(bar(C::BAR_S + k));
      }
      for (int j = 0; ok && j < nk; ++j) {
        const int s = j % C::STAGES;
        const uint32_t ph = (j / C::STAGES) & 1;
        const int s1 = (j + 1) % C::STAGES;
        const uint32_t ph1 = ((j + 1) / C::STAGES) & 1;
        const bool more = j + 1 < nk;
        {
          // S(j+1) as soon as the softmax has read S(j): overlaps softmax(j).
          // This thread spins on its hand-offs (a suspended wait wakes a few
          // hundred cycles after the phase completes).
          if (more) {
            if (!mbar_wait_spin(bar(C::BAR_SFREE + k), j & 1, ctl) || !mbar_wait(bar(C::BAR_KF + s1), ph1, ctl)) {
              ok = false;
              break;
            }
            tc_fence_after();
            issue_s(s1);
            umma_commit(bar(C::BAR_S + k));
          }
        }
        if (!mbar_wait(bar(C::BAR_VF + s), ph, ctl) || !mbar_wait_spin(bar(C::BAR_P + k), j & 1, ctl)) {
          ok = false;
          break;
        }
        tc_fence_after();
        issue_pv(s, j);
        umma_commit(bar(C::BAR_PV + k));
        if (!more) umma_commit(bar(C::BAR_O + k));
        umma_commit(bar(C::BAR_KVE + s));
      }
      // Drain: every MMA issued above has finished before TMEM is released.
      umma_commit(bar(C::BAR_DRAIN + k));
      volatile int zero = 0;
      WaitCtl drain{&zero, p.status, drain_limit_ns(p.timeout_ns)};
      mbar_wait(bar(C::BAR_DRAIN + k), 0, drain);
    }
  } else if (warp >= 4) {
    // ======================= softmax + epilogue, one thread per tile row
    regs_claim<C::REGS_SOFTMAX>();
    const int k = (warp - 4) >> 2;
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t lane_base = tmem + (uint32_t(quarter * 32) << 16);
    const uint32_t s_addr = lane_base + (k ? C::COL_S1 : C::COL_S0);
    const uint32_t o_addr = lane_base + (k ? C::COL_O1 : C::COL_O0);
    const uint32_t p_addr = lane_base + (k ? C::COL_P1 : C::COL_P0);
    const int token = t0[k] + (row >> p.log2P);
    const int head = head0 + (row & (p.P - 1));
    const float sl2 = p.scale_log2;
    const float2 sl2x2 = make_float2(sl2, sl2);
    const int nk = n_kv[k];
    const int t_first = p.q0 + t0[k];   // global position of the tile's first row
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < nk; ++j) {
      if (!mbar_wait_warp(bar(C::BAR_S + k), j & 1, ctl)) { ok = false; break; }
      tc_fence_after();
      constexpr int NC = C::BN;
      float s[NC];
      if constexpr (NC == 128) {
        uint32_t r[128];
        tmem_ld128(s_addr, r);
#pragma unroll
        for (int u = 0; u < 128; ++u) s[u] = __uint_as_float(r[u]);
      } else {
        static_assert(NC == 80, "score columns");
        uint32_t r[64], r2[16];
        tmem_ld64(s_addr, r);
        tmem_ld16(s_addr + 64, r2);
#pragma unroll
        for (int u = 0; u < 64; ++u) s[u] = __uint_as_float(r[u]);
#pragma unroll
        for (int u = 0; u < 16; ++u) s[64 + u] = __uint_as_float(r2[u]);
      }
      // S_k is in registers: the next S_k may be written.
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(C::BAR_SFREE + k));

      const int key0 = (kv0 + j) * C::BN;
      const bool tail = key0 + C::BN > p.Nk;
      const bool diag = p.causal && (key0 + C::BN - 1 > t_first);
      if (tail || diag) {
        const int lim = p.causal ? min(p.q0 + token, p.Nk - 1) : p.Nk - 1;  // last visible key
#pragma unroll
        for (int u = 0; u < NC; ++u)
          if (key0 + u > lim) s[u] = -INFINITY;
      }
      // row maximum: eight independent 3-input chains, then a short tree
      float m8[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) m8[i] = fmax3(s[i], s[8 + i], s[16 + i]);
#pragma unroll
      for (int u = 24; u < NC - 8; u += 16)
#pragma unroll
        for (int i = 0; i < 8; ++i) m8[i] = fmax3(m8[i], s[u + i], s[u + 8 + i]);
#pragma unroll
      for (int i = 0; i < 8; ++i) m8[i] = fmaxf(m8[i], s[NC - 8 + i]);
      const float mx = fmax3(fmax3(m8[0], m8[1], m8[2]), fmax3(m8[3], m8[4], m8[5]), fmaxf(m8[6], m8[7]));
      const float m_new = fmaxf(m, mx);
      // Keep the stale maximum unless it grew by more than 2^8 in the exp2
      // domain: O / l is exact either way, and P stays <= 256.
      const bool need = (j == 0) || ((m_new - m) * sl2 > 8.0f);
      const float m_use = need ? m_new : m;
      const float f = (need && j > 0) ? ex2_approx((m - m_new) * sl2) : 1.0f;
      const bool rescale = (j > 0) && __any_sync(0xffffffffu, need);
      const float2 nms = make_float2(-m_use * sl2, -m_use * sl2);
      uint32_t pk[NC / 2];
      float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
      for (int u = 0; u < NC / 2; ++u) {
        const float2 x = ffma2(make_float2(s[2 * u], s[2 * u + 1]), sl2x2, nms);
        float2 e;
        if ((EMU >> (u & 7)) & 1) {
          e = exp2_poly2(x);
        } else {
          e.x = ex2_approx(x.x);
          e.y = ex2_approx(x.y);
        }
        acc[u & 3] = fadd2(acc[u & 3], e);
        pk[u] = pack_bf16x2(e.x, e.y);   // P(j) packed as it is made
      }
      const float2 a01 = fadd2(acc[0], acc[1]), a23 = fadd2(acc[2], acc[3]);
      const float2 a = fadd2(a01, a23);
      l = l * f + (a.x + a.y);
      // P_k and O_k are free once PV_k(j-1) has completed.
      if (j > 0) {
        if (!mbar_wait_warp(bar(C::BAR_PV + k), (j - 1) & 1, ctl)) { ok = false; break; }
        tc_fence_after();
      }
      if constexpr (NC == 128) {
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          uint32_t r[32];
#pragma unroll
          for (int u = 0; u < 32; ++u) r[u] = pk[c * 32 + u];
          tmem_st32(p_addr + c * 32, r);
        }
      } else {
        uint32_t r[32], r8[8];
#pragma unroll
        for (int u = 0; u < 32; ++u) r[u] = pk[u];
#pragma unroll
        for (int u = 0; u < 8; ++u) r8[u] = pk[32 + u];
        tmem_st32(p_addr, r);
        tmem_st8(p_addr + 32, r8);
      }
      if (rescale) {
#pragma unroll 1
        for (int c = 0; c < D; c += 32) {
          uint32_t r[32];
          tmem_ld32(o_addr + c, r);
#pragma unroll
          for (int u = 0; u < 32; ++u) r[u] = __float_as_uint(__uint_as_float(r[u]) * f);
          tmem_st32(o_addr + c, r);
        }
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(C::BAR_P + k));
      m = m_use;
    }
    const bool have_o = ok && nk > 0 && mbar_wait_warp(bar(C::BAR_O + k), 0, ctl);
    if (have_o) tc_fence_after();
    const bool store = token < p.N;
    // Output rows: O = (a0 * O_tmem + a1 * part) * inv_l, the row's log-sum-exp
    // (natural log) for the backward, and the layer's row-block counters.
    auto store_rows = [&](float a0, const float* part, float a1, float inv_l, float lse_row) {
      // per lane: the warp-collective TMEM loads below run on every lane either way
      const bool st = store && in_bounds(head < p.H_q && b < p.B && token >= 0, p.status);
      if (p.lse != nullptr && st) p.lse[((size_t)b * p.H_q + head) * p.N + token] = lse_row;
      __nv_bfloat16* dst = p.out + (((size_t)b * p.N + (st ? token : 0)) * p.H_q + (st ? head : 0)) * D;
#pragma unroll
      for (int c = 0; c < D; c += 32) {
        uint32_t r[32];
        __syncwarp();              // after the per-lane stores: the TMEM load is warp-collective
        tmem_ld32(o_addr + c, r);
        float o[32];
#pragma unroll
        for (int u = 0; u < 32; ++u) o[u] = __uint_as_float(r[u]) * a0;
        if (part != nullptr) {
#pragma unroll
          for (int u = 0; u < 32; ++u) o[u] = fmaf(part[c + u], a1, o[u]);
        }
        uint4 w[4];
        uint32_t* wp = reinterpret_cast<uint32_t*>(w);
#pragma unroll
        for (int u = 0; u < 16; ++u) wp[u] = pack_bf16x2(o[2 * u] * inv_l, o[2 * u + 1] * inv_l);
        if (st) {
          uint4* d4 = reinterpret_cast<uint4*>(dst + c);
#pragma unroll
          for (int u = 0; u < 4; ++u) d4[u] = w[u];
        }
      }
      if (p.ready != nullptr) {
        // Publish this warp's rows: each lane's stores, then one release add
        // per 128-row block of [B * N] the warp's consecutive tokens touch
        // (at most two).
        __threadfence();
        __syncwarp();
        const long long flat = (long long)b * p.N + token;
        const int mb = (int)(flat >> 7);
        const int mb0 = __shfl_sync(0xffffffffu, mb, 0);
        const unsigned in0 = __ballot_sync(0xffffffffu, st && mb == mb0);
        const unsigned in1 = __ballot_sync(0xffffffffu, st && mb != mb0);
        const int n_blocks = (int)(((long long)p.B * p.N + 127) >> 7);
        if (lane == 0 && (in0 | in1) != 0u && in_bounds(mb0 >= 0 && mb0 + (in1 ? 1 : 0) < n_blocks, p.status)) {
          __threadfence();
          if (in0) atomicAdd(p.ready + mb0, __popc(in0));
          if (in1) atomicAdd(p.ready + mb0 + 1, __popc(in1));
        }
      }
    };
    constexpr float kLn2 = 0.69314718055994531f;
    if (split > 1) {
      // The two halves of the key range meet in rank 0. Partial row of tile k,
      // row r: (D unnormalised O values, m * scale * log2(e), l) at
      // OFF_Q + (k * 128 + r) * (D + 4) floats in rank 0's shared memory.
      cluster_sync_all();  // both CTAs are past their main loops: rank 0's Q/K/V buffers are free
      float* mrg = reinterpret_cast<float*>(smem + C::OFF_Q) + ((size_t)k * C::BM + row) * (D + 4);
      static_assert(C::OFF_Q + 2 * C::BM * (D + 4) * 4 <= C::OFF_BAR, "merge buffer");
      if (rank == 1 && have_o) {
        const uint32_t dst = map_shared_to_rank(smem_u32(mrg), 0);
#pragma unroll
        for (int c = 0; c < D; c += 32) {
          uint32_t r[32];
          tmem_ld32(o_addr + c, r);
#pragma unroll
          for (int v = 0; v < 8; ++v)
            st_cluster_v4(dst + (c + 4 * v) * 4, __uint_as_float(r[4 * v]), __uint_as_float(r[4 * v + 1]),
                          __uint_as_float(r[4 * v + 2]), __uint_as_float(r[4 * v + 3]));
        }
        st_cluster_v4(dst + D * 4, m * sl2, l, 0.f, 0.f);
      }
      cluster_sync_all();  // rank 1's partial rows are in rank 0's shared memory
      if (rank == 0 && have_o) {
        const float m0 = m * sl2, m1 = mrg[D], l1 = mrg[D + 1];
        const float mm = fmaxf(m0, m1);
        const float a0 = ex2_approx(m0 - mm), a1 = ex2_approx(m1 - mm);
        const float lt = l * a0 + l1 * a1;
        store_rows(a0, mrg, a1, 1.0f / lt, (mm + __log2f(lt)) * kLn2);
      }
    } else if (have_o) {
      // l sums exp2(s*sl2 - m*sl2), so ln(sum_u exp(scale*s_u)) = (m*sl2 + log2(l)) * ln(2)
      store_rows(1.0f, nullptr, 0.f, 1.0f / l, (m * sl2 + __log2f(l)) * kLn2);
    }
  }
  // Every thread of a split unit takes part in the two cluster barriers.
  if (split > 1 && warp < 4) {
    cluster_sync_all();
    cluster_sync_all();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
  // Launched as a programmatic dependent (a split last wave after its main
  // grid), this grid must not complete before that grid: work ordered after
  // this call on the stream relies on both. A no-op otherwise.
  asm volatile("griddepcontrol.wait;" ::: "memory");
}

}  // namespace sqa
