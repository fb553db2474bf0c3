// bwd_dkdv_sm100.cuh -- the key-side half of the recompute backward: dK and
// dV (bf16, head dimension 64 or 128) for sm_100a.
//
// The forward keeps only O and the per-row log-sum-exp; the backward rebuilds
// every score block from Q, K and those statistics instead of reading a
// stored score matrix (fanfani.net "FlashAttention", "The backward pass, and
// where the memory saving comes from"; synthetic.wiki "FlashAttention:
// attention's bottleneck is the wire, not the maths", "The backward pass buys
// memory with recompute"). The gradient is the textbook derivative of the
// softmax; per block, with keys as rows (the transposed products):
//   S^T  = K Q^T                  P^T  = exp(scale S^T - LSE)
//   dP^T = V dO^T                 dS^T = P^T * (dP^T - D) * scale
//   dV  += P^T dO                 dK  += dS^T Q
// with D = rowsum(dO * O) from the prep kernel. dQ is formed by a separate
// kernel (bwd_dq_sm100.cuh), so this one never adds into shared memory
// outside the CTA.
//
// One CTA per (128-key tile, batch, KV head, head slice). K and V are loaded
// once into tensor memory, where they are the A operand of S^T and dP^T; P^T
// and dS^T are written back into tensor memory as the A operand of dV and dK.
// So every MMA reads only its B operand (a Q or dO sub-tile) from shared
// memory: the form that runs at the full tensor rate. To fit tensor memory
// (512 columns: K and V take d/2 each, dV and dK d each), the CTA walks the
// query heads of its slice and their query rows 64 at a time.
//
// Roles (12 warps):
//   warps 0-3, 4-7  compute warpgroups: thread = key row (TMEM lane);
//                   warpgroup h owns query columns [32h, 32h+32) of every
//                   64-query sub-step
//   warp 8          TMA producer (Q and dO sub-tiles, LSE2 and D rows)
//   warp 9          TMEM allocator and MMA issuer
//   warps 10, 11    idle
// TMEM (columns): K at 0, V at d/2, dV at d, dK at 2d, then NBUF S^T and NBUF
// dP^T buffers of 64 columns (one each at d = 128, two each at d = 64).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include "sm100_ptx.cuh"

namespace fa {

template <int HD>
struct BwdKVCfg {
  static constexpr int NQ = 64;                          // queries per sub-step
  static constexpr int NBUF = HD == 64 ? 2 : 1;          // S^T / dP^T buffers
  static constexpr int SUB_BYTES = NQ * HD * 2;          // one 64-row bf16 sub-tile
  static constexpr int STAGE_BYTES = 2 * SUB_BYTES + 1024;  // Q, dO, LSE2 + D (padded)
  static constexpr int STAGES = HD == 64 ? 8 : 6;
  static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES;
  static constexpr int THREADS = 384;
  static constexpr int KV_GROUP = 8;  // (batch, KV head) pairs scheduled together
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t T_K = 0;
  static constexpr uint32_t T_V = HD / 2;
  static constexpr uint32_t T_DV = HD;
  static constexpr uint32_t T_DK = 2 * HD;
  static constexpr uint32_t T_S0 = 3 * HD;               // buffer b at T_S0 + 64 b
  static constexpr uint32_t T_DP0 = 3 * HD + NBUF * NQ;  // buffer b at T_DP0 + 64 b
  static_assert(T_DP0 + NBUF * NQ <= TMEM_COLS, "tensor memory overflow");
  static_assert(SMEM_BYTES <= 232448, "shared memory overflow");
};

struct BwdKVParams {
  const __nv_bfloat16* k;  // [B*Hkv][N][d]
  const __nv_bfloat16* v;
  const float* ws_delta;   // [B*Hq][Npad]
  const float* ws_lse2;    // [B*Hq][Npad], LSE * log2(e), +inf in padding rows
  __nv_bfloat16* dk;
  __nv_bfloat16* dv;
  float* dk_acc;  // [B*Hkv][N][d] f32, used when head_split > 1
  float* dv_acc;
  int N, Npad, Hq, Hkv, num_tiles;
  int head_split;  // CTAs sharing the query heads of one (KV head, key tile)
  int BHkv;
  float scale_log2;
  float scale;
  int causal;
  unsigned long long timeout_ns;
};

// A 128-row bf16 operand (K or V of this CTA's key tile) into tensor memory:
// thread r (TMEM lane r of its warp's quarter) copies row `row` of `src`
// (zeros when `live` is false) into columns [col, col + HD/2), two elements
// per column, lower index in the low half -- the layout of an MMA A operand.
template <int HD>
FA_DEV void load_rows_to_tmem(uint32_t taddr, const __nv_bfloat16* row_ptr, bool live) {
  const uint4* src = reinterpret_cast<const uint4*>(row_ptr);
#pragma unroll
  for (int c = 0; c < HD / 64; ++c) {
    uint32_t r[32];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const uint4 w = live ? __ldg(src + c * 8 + i) : make_uint4(0u, 0u, 0u, 0u);
      r[4 * i] = w.x;
      r[4 * i + 1] = w.y;
      r[4 * i + 2] = w.z;
      r[4 * i + 3] = w.w;
    }
    tmem_st32(taddr + c * 32, r);
  }
}

template <int HD>
__global__ void __launch_bounds__(384, 1)
    fa_bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
                       const BwdKVParams p) {
  using C = BwdKVCfg<HD>;
  constexpr int ST = C::STAGES, NBUF = C::NBUF;
  constexpr int KCH = HD / 64;

  extern __shared__ uint8_t smem_raw[];
  __shared__ uint64_t bar_full[ST], bar_empty[ST];
  __shared__ uint64_t bar_sfull[NBUF], bar_dpfull[NBUF], bar_pfull[NBUF], bar_dsfull[NBUF];
  __shared__ uint64_t bar_kv, bar_final;
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;

  const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
  uint8_t* const gbase = smem_raw + (base - smem_u32(smem_raw));

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // Block order: groups of KV_GROUP (batch, KV head) pairs whose K, V, Q and
  // dO stay in L2 together; inside a group the key tiles go heaviest first
  // (tile 0 sees every query when causal), each over its head slices.
  const int per_kv = p.num_tiles * p.head_split;
  const int grp = static_cast<int>(blockIdx.x) / (C::KV_GROUP * per_kv);
  const int in_grp = min(C::KV_GROUP, p.BHkv - grp * C::KV_GROUP);
  const int r0 = static_cast<int>(blockIdx.x) - grp * C::KV_GROUP * per_kv;
  const int kt = r0 / (in_grp * p.head_split);
  const int r1 = r0 - kt * in_grp * p.head_split;
  const int bhkv = grp * C::KV_GROUP + r1 / p.head_split;
  const int slice = r1 - (r1 / p.head_split) * p.head_split;
  const int k0 = kt * 128;
  const int b = bhkv / p.Hkv;
  const int hkv = bhkv - b * p.Hkv;
  const int group = p.Hq / p.Hkv;
  const int heads = group / p.head_split;
  const int h_first = slice * heads;
  const int n_sub = (p.N + C::NQ - 1) / C::NQ;       // 64-query sub-tiles per head
  const int i_begin = p.causal ? 2 * kt : 0;          // first sub-tile that sees the keys
  const int per_head = n_sub - i_begin;
  const int steps = heads * per_head;

  WaitCtl wc{&abort_flag, p.timeout_ns};

  if (threadIdx.x == 0) {
    abort_flag = 0;
    for (int s = 0; s < ST; ++s) {
      mbar_init(smem_u32(&bar_full[s]), 1);
      mbar_init(smem_u32(&bar_empty[s]), 1);
    }
    for (int s = 0; s < NBUF; ++s) {
      mbar_init(smem_u32(&bar_sfull[s]), 1);
      mbar_init(smem_u32(&bar_dpfull[s]), 1);
      mbar_init(smem_u32(&bar_pfull[s]), 256);
      mbar_init(smem_u32(&bar_dsfull[s]), 256);
    }
    mbar_init(smem_u32(&bar_kv), 256);
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

  // sub-step t -> (query head, first query row)
  auto step_rows = [&](int t, int& bhq, int& q0) {
    const int hh = t / per_head;
    q0 = (i_begin + (t - hh * per_head)) * C::NQ;
    bhq = b * p.Hq + hkv * group + h_first + hh;
  };

  if (warp == 8) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      prefetch_tmap(&tm_q);
      prefetch_tmap(&tm_do);
      int issued = 0;
      for (int t = 0; t < steps; ++t) {
        int bhq, q0;
        step_rows(t, bhq, q0);
        const int s = t % ST;
        if (!mbar_wait(smem_u32(&bar_empty[s]), ((t / ST) & 1) ^ 1, wc)) break;
        const uint32_t st = base + s * C::STAGE_BYTES;
        const uint32_t fb = smem_u32(&bar_full[s]);
        mbar_arrive_expect_tx(fb, 2 * C::SUB_BYTES + 512);
        for (int c = 0; c < KCH; ++c) {
          tma_load_3d(st + c * 8192, &tm_q, fb, c * 64, q0, bhq);
          tma_load_3d(st + C::SUB_BYTES + c * 8192, &tm_do, fb, c * 64, q0, bhq);
        }
        const size_t roff = static_cast<size_t>(bhq) * p.Npad + q0;
        bulk_load(st + 2 * C::SUB_BYTES, p.ws_lse2 + roff, 256, fb);
        bulk_load(st + 2 * C::SUB_BYTES + 256, p.ws_delta + roff, 256, fb);
        issued = t + 1;
      }
      // leave nothing in flight into shared memory: wait for the loads of
      // the stages still outstanding (they may not have been consumed when a
      // bounded wait gave up)
      for (int t = max(0, issued - ST); t < issued; ++t)
        (void)mbar_wait_drain(smem_u32(&bar_full[t % ST]), (t / ST) & 1, p.timeout_ns);
    }
  } else if (warp == 9) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t id_s = idesc_bf16_f32(128, C::NQ, false, false);  // S^T, dP^T: M=keys, N=64 queries
      constexpr uint32_t id_g = idesc_bf16_f32(128, HD, false, true);      // dV, dK: N=d, B MN-major
      // S^T(t) or dP^T(t): A = K or V in TMEM, B = the Q or dO sub-tile (K-major)
      auto issue_sd = [&](int t, uint32_t a_col, uint32_t d_col, uint32_t sub_off, uint32_t bar) {
        const uint32_t src = base + (t % ST) * C::STAGE_BYTES + sub_off;
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk)
          mma_bf16_ts(tmem + d_col, tmem + a_col + kk * 8,
                      sdesc_sw128(src + (kk >> 2) * 8192 + (kk & 3) * 32, 16, 1024), id_s, kk > 0);
        mma_commit(bar);
      };
      // dV += P^T dO or dK += dS^T Q: A = P^T / dS^T in TMEM (warpgroup h's
      // 32 queries in columns [32h, 32h+16) of the buffer), B = the sub-tile
      // as queries x d (MN-major)
      auto issue_grad = [&](int t, uint32_t a_col, uint32_t d_col, uint32_t sub_off, bool first) {
        const uint32_t src = base + (t % ST) * C::STAGE_BYTES + sub_off;
#pragma unroll
        for (int kk = 0; kk < C::NQ / 16; ++kk)
          mma_bf16_ts(tmem + d_col, tmem + a_col + (kk >> 1) * 32 + (kk & 1) * 8,
                      sdesc_sw128(src + kk * 2048, 8192, 1024), id_g, !(first && kk == 0));
      };
      auto issue_pair = [&](int t) {  // S^T(t) and dP^T(t) into buffer t % NBUF
        const int bf = t % NBUF;
        if (!mbar_wait(smem_u32(&bar_full[t % ST]), (t / ST) & 1, wc)) return false;
        tc_fence_after();
        issue_sd(t, C::T_K, C::T_S0 + bf * C::NQ, 0, smem_u32(&bar_sfull[bf]));
        issue_sd(t, C::T_V, C::T_DP0 + bf * C::NQ, C::SUB_BYTES, smem_u32(&bar_dpfull[bf]));
        return true;
      };
      bool ok = mbar_wait(smem_u32(&bar_kv), 0, wc);
      if (ok) tc_fence_after();
      for (int t = 0; ok && t < NBUF && t < steps; ++t) ok = issue_pair(t);
      for (int t = 0; ok && t < steps; ++t) {
        const int bf = t % NBUF;
        const uint32_t ph = (t / NBUF) & 1;
        if (!mbar_wait(smem_u32(&bar_pfull[bf]), ph, wc)) { ok = false; break; }
        tc_fence_after();
        issue_grad(t, C::T_S0 + bf * C::NQ, C::T_DV, C::SUB_BYTES, t == 0);
        // With one buffer, S^T(t+1) may overwrite P^T(t) once dV(t) is issued
        // (MMAs run in issue order); dP^T(t+1) waits for dK(t) likewise.
        if (NBUF == 1 && t + 1 < steps) {
          if (!mbar_wait(smem_u32(&bar_full[(t + 1) % ST]), ((t + 1) / ST) & 1, wc)) { ok = false; break; }
          tc_fence_after();
          issue_sd(t + 1, C::T_K, C::T_S0, 0, smem_u32(&bar_sfull[0]));
        }
        if (!mbar_wait(smem_u32(&bar_dsfull[bf]), ph, wc)) { ok = false; break; }
        tc_fence_after();
        issue_grad(t, C::T_DP0 + bf * C::NQ, C::T_DK, 0, t == 0);
        mma_commit(smem_u32(&bar_empty[t % ST]));  // Q and dO of sub-step t are consumed
        if (NBUF == 1 && t + 1 < steps) issue_sd(t + 1, C::T_V, C::T_DP0, C::SUB_BYTES, smem_u32(&bar_dpfull[0]));
        if (NBUF == 2 && t + 2 < steps) {
          if (!issue_pair(t + 2)) { ok = false; break; }
        }
      }
      // bar_final completes when every MMA issued above has completed, on
      // the normal path and after a bounded wait gave up alike; wait for it
      // so that no MMA is in flight when tensor memory is released
      mma_commit(smem_u32(&bar_final));
      (void)mbar_wait_drain(smem_u32(&bar_final), 0, p.timeout_ns);
    }
  } else if (warp < 8) {
    // ---------------------------------------------------- compute warpgroups
    const int h = warp >> 2;
    const int row = (warp & 3) * 32 + lane;  // key row within the tile (TMEM lane)
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const int key = k0 + row;
    const bool key_live = key < p.N;
    // K (warpgroup 0) or V (warpgroup 1) of this key row into tensor memory
    {
      const __nv_bfloat16* src = (h == 0 ? p.k : p.v) + (static_cast<size_t>(bhkv) * p.N + (key_live ? key : 0)) * HD;
      load_rows_to_tmem<HD>(tmem + lane_base + (h == 0 ? C::T_K : C::T_V), src, key_live);
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(smem_u32(&bar_kv));
    }
    const int qc = 32 * h;  // first query column of this warpgroup in a sub-step
    bool ok = true;
    for (int t = 0; t < steps; ++t) {
      int bhq, q0;
      step_rows(t, bhq, q0);
      const int bf = t % NBUF;
      const uint32_t ph = (t / NBUF) & 1;
      const float* srow = reinterpret_cast<const float*>(gbase + (t % ST) * C::STAGE_BYTES + 2 * C::SUB_BYTES);
      const float4* l4 = reinterpret_cast<const float4*>(srow + qc);
      const float4* d4 = reinterpret_cast<const float4*>(srow + 64 + qc);
      if (!warp_wait(smem_u32(&bar_full[t % ST]), (t / ST) & 1, wc)) { ok = false; break; }
      if (!warp_wait(smem_u32(&bar_sfull[bf]), ph, wc)) { ok = false; break; }
      tc_fence_after();
      // ---- P^T = exp2(S^T * scale * log2 e - LSE2), masked
      const bool diag = p.causal && (q0 < k0 + 128);  // some query of the sub-step precedes some key
      float pf[32];
      {
        uint32_t s[32];
        tmem_ld32(tmem + lane_base + C::T_S0 + bf * C::NQ + qc, s);
        uint32_t pk[16];
#pragma unroll
        for (int x = 0; x < 8; ++x) {
          const float4 L = l4[x];
          pf[4 * x] = ex2_approx(fmaf(__uint_as_float(s[4 * x]), p.scale_log2, -L.x));
          pf[4 * x + 1] = ex2_approx(fmaf(__uint_as_float(s[4 * x + 1]), p.scale_log2, -L.y));
          pf[4 * x + 2] = ex2_approx(fmaf(__uint_as_float(s[4 * x + 2]), p.scale_log2, -L.z));
          pf[4 * x + 3] = ex2_approx(fmaf(__uint_as_float(s[4 * x + 3]), p.scale_log2, -L.w));
        }
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          const bool hidden = !key_live || (diag && q0 + qc + c < key);
          if (hidden) pf[c] = 0.f;
        }
#pragma unroll
        for (int x = 0; x < 16; ++x) pk[x] = pack_bf16x2(pf[2 * x], pf[2 * x + 1]);
        tmem_st16(tmem + lane_base + C::T_S0 + bf * C::NQ + qc, pk);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(smem_u32(&bar_pfull[bf]));
      // ---- dS^T = P^T (dP^T - D) scale
      if (!warp_wait(smem_u32(&bar_dpfull[bf]), ph, wc)) { ok = false; break; }
      tc_fence_after();
      {
        uint32_t g[32];
        tmem_ld32(tmem + lane_base + C::T_DP0 + bf * C::NQ + qc, g);
        uint32_t w[16];
#pragma unroll
        for (int x = 0; x < 8; ++x) {
          const float4 Dv = d4[x];
          const float e0 = pf[4 * x] * (__uint_as_float(g[4 * x]) - Dv.x) * p.scale;
          const float e1 = pf[4 * x + 1] * (__uint_as_float(g[4 * x + 1]) - Dv.y) * p.scale;
          const float e2 = pf[4 * x + 2] * (__uint_as_float(g[4 * x + 2]) - Dv.z) * p.scale;
          const float e3 = pf[4 * x + 3] * (__uint_as_float(g[4 * x + 3]) - Dv.w) * p.scale;
          w[2 * x] = pack_bf16x2(e0, e1);
          w[2 * x + 1] = pack_bf16x2(e2, e3);
        }
        tmem_st16(tmem + lane_base + C::T_DP0 + bf * C::NQ + qc, w);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(smem_u32(&bar_dsfull[bf]));
    }
    // epilogue: warpgroup 0 writes dV, warpgroup 1 writes dK (dS carries the
    // scale): bf16 rows, or, when the group's heads are split over several
    // CTAs, f32 rows added into the accumulators
    if (ok && warp_wait(smem_u32(&bar_final), 0, wc)) {
      tc_fence_after();
      const size_t row_off = (static_cast<size_t>(bhkv) * p.N + (key_live ? key : 0)) * HD;
      __nv_bfloat16* out = (h == 0 ? p.dv : p.dk) + row_off;
      float* acc = p.head_split > 1 ? (h == 0 ? p.dv_acc : p.dk_acc) + row_off : nullptr;
      const uint32_t col = h == 0 ? C::T_DV : C::T_DK;
#pragma unroll
      for (int c = 0; c < HD / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(tmem + lane_base + col + c * 32, r);
        if (p.head_split > 1) {
          if (key_live) {
#pragma unroll
            for (int x = 0; x < 8; ++x)
              red_add_v4_f32(acc + c * 32 + 4 * x, __uint_as_float(r[4 * x]), __uint_as_float(r[4 * x + 1]),
                             __uint_as_float(r[4 * x + 2]), __uint_as_float(r[4 * x + 3]));
          }
        } else {
          uint4 w[4];
          uint32_t* wp = reinterpret_cast<uint32_t*>(w);
#pragma unroll
          for (int x = 0; x < 16; ++x) wp[x] = pack_bf16x2(__uint_as_float(r[2 * x]), __uint_as_float(r[2 * x + 1]));
          if (key_live) {
#pragma unroll
            for (int x = 0; x < 4; ++x) reinterpret_cast<uint4*>(out + c * 32)[x] = w[x];
          }
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
