// bwd_dq_sm100.cuh -- the query-side half of the recompute backward: dQ
// (bf16, head dimension 64 or 128) for sm_100a.
//
// Same recompute as bwd_dkdv_sm100.cuh, with queries as rows:
//   S  = Q K^T          P  = exp(scale S - LSE)
//   dP = dO V^T         dS = P * (dP - D) * scale
//   dQ += dS K
// (fanfani.net "FlashAttention", "The backward pass, and where the memory
// saving comes from": the score blocks are rebuilt from Q, K and the stored
// per-row statistics). Giving dQ its own pass costs the two recomputed
// products S and dP a second time, but dQ then accumulates in tensor memory
// over all key tiles and is written once, in bf16: no f32 accumulator in
// global memory, no reductions from every key tile into it, and the result
// does not depend on the order in which CTAs finish.
//
// One CTA per (128-query tile, batch, query head). Q and dO are loaded once
// into tensor memory as the A operands of S and dP; dS goes back into tensor
// memory as the A operand of dQ += dS K. K and V stream through shared memory
// 64 keys at a time, and S and dP are double-buffered, so the tensor core
// computes sub-tile j+1 while the compute warpgroups turn sub-tile j into dS.
//
// Roles (12 warps):
//   warps 0-3, 4-7  compute warpgroups: thread = query row (TMEM lane);
//                   warpgroup h owns key columns [32h, 32h+32) of every
//                   64-key sub-tile
//   warp 8          TMA producer (K and V sub-tiles)
//   warp 9          TMEM allocator and MMA issuer
//   warps 10, 11    idle
// TMEM (columns): Q at 0, dO at d/2, dQ at d, then S0, S1, dP0, dP1 (64 each).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include "sm100_ptx.cuh"

namespace fa {

template <int HD>
struct BwdQCfg {
  static constexpr int BM = 128;                  // query rows per CTA
  static constexpr int NK = 64;                   // keys per sub-step
  static constexpr int SUB_BYTES = NK * HD * 2;   // one 64-row bf16 sub-tile (K or V)
  static constexpr int STAGE_BYTES = 2 * SUB_BYTES;
  static constexpr int STAGES = HD == 64 ? 8 : 6;
  static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES;
  static constexpr int THREADS = 384;
  static constexpr int HEAD_GROUP = 8;            // query heads scheduled together
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t T_Q = 0;
  static constexpr uint32_t T_DO = HD / 2;
  static constexpr uint32_t T_DQ = HD;
  static constexpr uint32_t T_S0 = 2 * HD;        // S buffer b at T_S0 + 64 b
  static constexpr uint32_t T_DP0 = 2 * HD + 2 * NK;
  static_assert(T_DP0 + 2 * NK <= TMEM_COLS, "tensor memory overflow");
  static_assert(SMEM_BYTES <= 232448, "shared memory overflow");
};

struct BwdQParams {
  const __nv_bfloat16* q;  // [B*Hq][N][d]
  const __nv_bfloat16* dO;
  const float* ws_delta;   // [B*Hq][Npad]
  const float* ws_lse2;    // [B*Hq][Npad]
  __nv_bfloat16* dq;       // [B*Hq][N][d]
  int N, Npad, Hq, Hkv, BH, num_tiles;
  float scale_log2;
  float scale;
  int causal;
  unsigned long long timeout_ns;
};

template <int HD>
__global__ void __launch_bounds__(384, 1)
    fa_bwd_dq_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                     const BwdQParams p) {
  using C = BwdQCfg<HD>;
  constexpr int ST = C::STAGES;
  constexpr int KCH = HD / 64;

  extern __shared__ uint8_t smem_raw[];
  __shared__ uint64_t bar_full[ST], bar_empty[ST];
  __shared__ uint64_t bar_sfull[2], bar_dpfull[2], bar_dsfull[2];
  __shared__ uint64_t bar_q, bar_final;
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;

  const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // Work item: groups of HEAD_GROUP (batch, query head) pairs (a GQA group's
  // heads are adjacent, so their K and V stay in L2 together); inside a group
  // the heaviest (last, when causal) query tiles start first.
  const int per_group = C::HEAD_GROUP * p.num_tiles;
  const int g = static_cast<int>(blockIdx.x) / per_group;
  const int in_group = min(C::HEAD_GROUP, p.BH - g * C::HEAD_GROUP);
  const int r = static_cast<int>(blockIdx.x) - g * per_group;
  const int qt = p.num_tiles - 1 - r / in_group;
  const int bhq = g * C::HEAD_GROUP + r % in_group;
  const int b = bhq / p.Hq;
  const int hq = bhq - b * p.Hq;
  const int bhkv = b * p.Hkv + hq / (p.Hq / p.Hkv);
  const int q0 = qt * C::BM;
  const int n_sub_all = (p.N + C::NK - 1) / C::NK;
  const int steps = p.causal ? min(n_sub_all, (q0 + C::BM) / C::NK) : n_sub_all;

  WaitCtl wc{&abort_flag, p.timeout_ns};

  if (threadIdx.x == 0) {
    abort_flag = 0;
    for (int s = 0; s < ST; ++s) {
      mbar_init(smem_u32(&bar_full[s]), 1);
      mbar_init(smem_u32(&bar_empty[s]), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(smem_u32(&bar_sfull[s]), 1);
      mbar_init(smem_u32(&bar_dpfull[s]), 1);
      mbar_init(smem_u32(&bar_dsfull[s]), 256);
    }
    mbar_init(smem_u32(&bar_q), 256);
    mbar_init(smem_u32(&bar_final), 1);
    fence_mbar_init();
  }
  if (warp == 9) {
    tmem_alloc(smem_u32(&tmem_slot), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;

  if (warp == 8) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_v);
      int issued = 0;
      for (int t = 0; t < steps; ++t) {
        const int s = t % ST;
        if (!mbar_wait(smem_u32(&bar_empty[s]), ((t / ST) & 1) ^ 1, wc)) break;
        const uint32_t st = base + s * C::STAGE_BYTES;
        const uint32_t fb = smem_u32(&bar_full[s]);
        mbar_arrive_expect_tx(fb, 2 * C::SUB_BYTES);
        for (int c = 0; c < KCH; ++c) {
          tma_load_3d(st + c * 8192, &tm_k, fb, c * 64, t * C::NK, bhkv);
          tma_load_3d(st + C::SUB_BYTES + c * 8192, &tm_v, fb, c * 64, t * C::NK, bhkv);
        }
        issued = t + 1;
      }
      for (int t = max(0, issued - ST); t < issued; ++t)
        (void)mbar_wait_drain(smem_u32(&bar_full[t % ST]), (t / ST) & 1, p.timeout_ns);
    }
  } else if (warp == 9) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t id_s = idesc_bf16_f32(128, C::NK, false, false);  // S, dP: M=queries, N=64 keys
      constexpr uint32_t id_g = idesc_bf16_f32(128, HD, false, true);      // dQ: N=d, B (K) MN-major
      // S(t) = Q K^T or dP(t) = dO V^T into buffer t & 1
      auto issue_pair = [&](int t) {
        const int bf = t & 1;
        if (!mbar_wait(smem_u32(&bar_full[t % ST]), (t / ST) & 1, wc)) return false;
        tc_fence_after();
        const uint32_t st = base + (t % ST) * C::STAGE_BYTES;
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk)
          mma_bf16_ts(tmem + C::T_S0 + bf * C::NK, tmem + C::T_Q + kk * 8,
                      sdesc_sw128(st + (kk >> 2) * 8192 + (kk & 3) * 32, 16, 1024), id_s, kk > 0);
        mma_commit(smem_u32(&bar_sfull[bf]));
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk)
          mma_bf16_ts(tmem + C::T_DP0 + bf * C::NK, tmem + C::T_DO + kk * 8,
                      sdesc_sw128(st + C::SUB_BYTES + (kk >> 2) * 8192 + (kk & 3) * 32, 16, 1024), id_s, kk > 0);
        mma_commit(smem_u32(&bar_dpfull[bf]));
        return true;
      };
      bool ok = mbar_wait(smem_u32(&bar_q), 0, wc);
      if (ok) tc_fence_after();
      for (int t = 0; ok && t < 2 && t < steps; ++t) ok = issue_pair(t);
      for (int t = 0; ok && t < steps; ++t) {
        const int bf = t & 1;
        if (!mbar_wait(smem_u32(&bar_dsfull[bf]), (t >> 1) & 1, wc)) { ok = false; break; }
        tc_fence_after();
        // dQ += dS K: A = dS in TMEM (warpgroup h's 32 keys in columns
        // [32h, 32h+16) of the S buffer), B = the K sub-tile as keys x d
        const uint32_t kst = base + (t % ST) * C::STAGE_BYTES;
#pragma unroll
        for (int kk = 0; kk < C::NK / 16; ++kk)
          mma_bf16_ts(tmem + C::T_DQ, tmem + C::T_S0 + bf * C::NK + (kk >> 1) * 32 + (kk & 1) * 8,
                      sdesc_sw128(kst + kk * 2048, 8192, 1024), id_g, (t > 0 || kk > 0));
        mma_commit(smem_u32(&bar_empty[t % ST]));  // K and V of sub-step t are consumed
        // the buffer's next products may overwrite dS(t): dQ(t) was issued first
        if (t + 2 < steps && !issue_pair(t + 2)) { ok = false; break; }
      }
      mma_commit(smem_u32(&bar_final));
      (void)mbar_wait_drain(smem_u32(&bar_final), 0, p.timeout_ns);
    }
  } else if (warp < 8) {
    // ---------------------------------------------------- compute warpgroups
    const int h = warp >> 2;
    const int rrow = (warp & 3) * 32 + lane;  // query row within the tile (TMEM lane)
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const int qrow = q0 + rrow;
    const bool q_live = qrow < p.N;
    {
      // Q (warpgroup 0) or dO (warpgroup 1) of this query row into tensor memory
      const __nv_bfloat16* src = (h == 0 ? p.q : p.dO) + (static_cast<size_t>(bhq) * p.N + (q_live ? qrow : 0)) * HD;
      load_rows_to_tmem<HD>(tmem + lane_base + (h == 0 ? C::T_Q : C::T_DO), src, q_live);
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(smem_u32(&bar_q));
    }
    // per-row statistics: padding rows carry LSE2 = +inf and D = 0
    const float lse2 = p.ws_lse2[static_cast<size_t>(bhq) * p.Npad + qrow];
    const float dlt = p.ws_delta[static_cast<size_t>(bhq) * p.Npad + qrow];
    const int kc = 32 * h;  // first key column of this warpgroup in a sub-step
    bool ok = true;
    for (int t = 0; t < steps; ++t) {
      const int bf = t & 1;
      const uint32_t ph = (t >> 1) & 1;
      const int key0 = t * C::NK + kc;
      if (!warp_wait(smem_u32(&bar_sfull[bf]), ph, wc)) { ok = false; break; }
      tc_fence_after();
      float pf[32];
      {
        uint32_t s[32];
        tmem_ld32(tmem + lane_base + C::T_S0 + bf * C::NK + kc, s);
#pragma unroll
        for (int c = 0; c < 32; ++c) pf[c] = ex2_approx(fmaf(__uint_as_float(s[c]), p.scale_log2, -lse2));
        // keys past N, and keys after the query when causal, get no weight
        const int lim = min(p.causal ? qrow + 1 : p.N, p.N) - key0;  // keys [key0, key0 + lim) visible
        if (lim < 32) {
#pragma unroll
          for (int c = 0; c < 32; ++c)
            if (c >= lim) pf[c] = 0.f;
        }
      }
      if (!warp_wait(smem_u32(&bar_dpfull[bf]), ph, wc)) { ok = false; break; }
      tc_fence_after();
      {
        uint32_t g[32];
        tmem_ld32(tmem + lane_base + C::T_DP0 + bf * C::NK + kc, g);
        uint32_t w[16];
#pragma unroll
        for (int x = 0; x < 16; ++x)
          w[x] = pack_bf16x2(pf[2 * x] * (__uint_as_float(g[2 * x]) - dlt) * p.scale,
                             pf[2 * x + 1] * (__uint_as_float(g[2 * x + 1]) - dlt) * p.scale);
        tmem_st16(tmem + lane_base + C::T_S0 + bf * C::NK + kc, w);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(smem_u32(&bar_dsfull[bf]));
    }
    // epilogue: warpgroup h writes dQ columns [h d/2, (h+1) d/2) of its row
    if (ok && warp_wait(smem_u32(&bar_final), 0, wc)) {
      tc_fence_after();
      __nv_bfloat16* out = p.dq + (static_cast<size_t>(bhq) * p.N + (q_live ? qrow : 0)) * HD + h * (HD / 2);
#pragma unroll
      for (int c = 0; c < HD / 64; ++c) {
        uint32_t rr[32];
        tmem_ld32(tmem + lane_base + C::T_DQ + h * (HD / 2) + c * 32, rr);
        uint4 w[4];
        uint32_t* wp = reinterpret_cast<uint32_t*>(w);
#pragma unroll
        for (int x = 0; x < 16; ++x) wp[x] = pack_bf16x2(__uint_as_float(rr[2 * x]), __uint_as_float(rr[2 * x + 1]));
        if (q_live) {
#pragma unroll
          for (int x = 0; x < 4; ++x) reinterpret_cast<uint4*>(out + c * 32)[x] = w[x];
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace fa
