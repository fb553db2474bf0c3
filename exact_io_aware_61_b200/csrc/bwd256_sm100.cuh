// bwd256_sm100.cuh -- recompute backward for head dimension 256 (bf16) on
// sm_100a.
//
// Same gradient as the d = 64 / 128 kernel (bwd2_sm100.cuh): scores are
// recomputed from Q and K and the weights rebuilt from the stored LSE
// (fanfani.net "FlashAttention", "The backward pass, and where the memory
// saving comes from"):
//   P  = exp(scale S - LSE)     dV = P^T dO      dP = dO V^T
//   dS = P * (dP - D)           dQ = scale dS K  dK = scale dS^T Q
//
// At d = 256 the f32 dK and dV of a 128-key tile would fill all 512 columns
// of tensor memory, so this kernel takes 64-key tiles and accumulates them
// transposed, with the head dimension on the TMEM lanes:
//   dV^T [256 x 64] += dO^T P,  dK^T [256 x 64] += Q^T dS
// each as two 128-lane halves of 64 columns. S and dP have the 128 query
// rows on the lanes (64 columns each), and dQ = dS K leaves in two
// 128-column halves (the second over the S and dP columns, free by then).
// TMEM: dV^T 0..127 | dK^T 128..255 | S 256..319 | dP 320..383 | dQ half 0
// 384..511; dQ half 1 at 256..383.
//
// One CTA per (64-key tile, batch, KV head, head slice); it loops over its
// slice of the group's query heads and the 128-row query tiles that see the
// key tile (all of them without the mask). Shared memory holds K and V of
// the key tile (32 KB each), one Q and one dO tile (64 KB each) with their
// LSE and D rows, and P and dS (16 KB each): 225 KB.
// Roles (16 warps):
//   warps 0-7   two compute warpgroups; thread = query row, warpgroup h
//               owns key columns [32h, 32h + 32): P (bf16) and dS (bf16)
//               into 128-byte-swizzled shared tiles [query][key], which are
//               the B operands of dV^T and dK^T and the A operand of dQ
//   warps 8-11  dQ drain: loads dQ from TMEM in 64-column pieces (16x256b
//               shape), frees each as far as the next MMA needs it, and adds
//               it into the f32 accumulator, each warp-wide reduction 256
//               contiguous bytes of one row
//   warp 12     TMA producer; warp 13 TMEM allocator and MMA issuer
// Per step (query tile t) the issuer runs S, dP, dV^T (once P is in shared
// memory), dK^T (once dS is), dQ half 1, dQ half 0.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <utility>

#include "sm100_ptx.cuh"

namespace fa {

struct Bwd256Cfg {
  static constexpr int HD = 256;
  static constexpr int BK = 64;                  // keys per CTA
  static constexpr int BQ = 128;                 // queries per step
  static constexpr int KV_BYTES = BK * HD * 2;   // 32 KB: four [64 keys][64 d] chunks of 8 KB
  static constexpr int KV_CHUNK = BK * 128;
  static constexpr int Q_BYTES = BQ * HD * 2;    // 64 KB: four [128 q][64 d] chunks of 16 KB
  static constexpr int Q_CHUNK = BQ * 128;
  static constexpr int STATS_BYTES = 1024;       // LSE2, D of the tile's 128 rows
  static constexpr int PS_BYTES = BQ * BK * 2;   // 16 KB: [128 q][64 keys], one 128-byte row per query
  static constexpr int SMEM_BYTES = 1024 + 2 * KV_BYTES + 2 * Q_BYTES + STATS_BYTES + 2 * PS_BYTES;
  static constexpr int THREADS = 512;
  // Launch with 128 registers per thread (16 warps, 4 per SM sub-partition),
  // then redistribute per warpgroup: the drain holds a whole 128-column half
  // of the dQ tile, so that its columns are freed before any reduction.
  static constexpr int LAUNCH_REGS = 128;
  static constexpr int COMPUTE_REGS = 136;
  static constexpr int DRAIN_REGS = 144;
  static constexpr int OTHER_REGS = 96;
  static_assert(128 * (2 * COMPUTE_REGS + DRAIN_REGS + OTHER_REGS) <= THREADS * LAUNCH_REGS,
                "register split exceeds the launch allocation");
  static constexpr int KV_GROUP = 4;             // (batch, KV head) pairs scheduled together (their working set stays in L2)
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t T_DV = 0, T_DK = 128, T_S = 256, T_DP = 320, T_DQ0 = 384, T_DQ1 = 256;
};
static_assert(Bwd256Cfg::SMEM_BYTES <= 231424, "shared memory beyond the 227 KB per block, with the static part");

struct Bwd256Params {
  const float* ws_delta;  // [B*Hq][Npad]
  const float* ws_lse2;   // [B*Hq][Npad]
  float* dq_acc;          // [B*Hq][N][256]
  __nv_bfloat16* dk;      // [B*Hkv][N][256]
  __nv_bfloat16* dv;
  float* dk_acc;          // f32 [B*Hkv][N][256], used when head_split > 1
  float* dv_acc;
  int N, Npad, Hq, Hkv, num_tiles;  // num_tiles: 64-key tiles
  int head_split, BHkv;
  float scale_log2, scale;
  int causal;
  unsigned long long timeout_ns;
};

// The dQ drain's reductions of one set of 8 rows (RB .. RB + 7 of the warp's 32)
// over a 64-column piece. On entry lane 4 g + c holds, in x[k], columns
// 8k + 2c, 8k + 2c + 1 of row RB + g (k = 0..7: the 16x256b layout). An 8 x 8
// transpose over the lane groups g (three butterfly stages of XOR shuffles;
// the register indices stay compile-time constants) leaves in x[j] columns
// 8g + 2c, 8g + 2c + 1 of row RB + j, so that each reduction instruction of
// the warp covers 256 contiguous bytes of one row (whole lines: L2 takes
// those about 1.7 times faster than 32-byte pieces of 8 rows).
// x[J] (row RB + J, 1 KB per row of 256 floats) into the accumulator, the
// row offset an immediate of the instruction
template <int RB, int J>
FA_DEV void drain_red(float* base, const float (&x)[8][2], int live) {
  if (RB + J < live) red_add_v2_f32<(RB + J) * Bwd256Cfg::HD * 4>(base, x[J][0], x[J][1]);
}

template <int RB, size_t... J>
FA_DEV void drain_reds(float* base, const float (&x)[8][2], int live, std::index_sequence<J...>) {
  (drain_red<RB, static_cast<int>(J)>(base, x, live), ...);
}

template <int RB>
FA_DEV void drain_rowset(float* base, float (&x)[8][2], int g, int live) {
#pragma unroll
  for (int s = 0; s < 3; ++s) {
    const int m = 1 << s;
    const bool hi = (g & m) != 0;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      if (k & m) continue;
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const float send = hi ? x[k][e] : x[k | m][e];
        const float recv = __shfl_xor_sync(0xffffffffu, send, 4 * m);
        if (hi) x[k][e] = recv;
        else x[k | m][e] = recv;
      }
    }
  }
  drain_reds<RB>(base, x, live, std::make_index_sequence<8>{});
}

// 16 warps, 4 per SM sub-partition: 16384 / 128 -> 128 registers at launch.
__global__ void __launch_bounds__(512, 1)
    fa_bwd256_main_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                          const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                          const Bwd256Params p) {
  using C = Bwd256Cfg;
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint64_t bar_kv, bar_qfull, bar_qempty, bar_dofull, bar_doempty, bar_sfull, bar_dpfull;
  __shared__ uint64_t bar_pfull, bar_pempty, bar_dsfull, bar_dsempty;
  __shared__ uint64_t bar_dq0full, bar_dq1full, bar_dq0free, bar_dq1afree, bar_dq1bfree, bar_final;
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;

  const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
  uint8_t* const gbase = smem_raw + (base - smem_u32(smem_raw));
  const uint32_t sK = base;
  const uint32_t sV = sK + C::KV_BYTES;
  const uint32_t sQ = sV + C::KV_BYTES;
  const uint32_t sDO = sQ + C::Q_BYTES;
  const uint32_t sST = sDO + C::Q_BYTES;  // LSE2 [128] then D [128]
  const uint32_t sP = sST + C::STATS_BYTES;
  const uint32_t sDS = sP + C::PS_BYTES;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // Block order: groups of KV_GROUP (batch, KV head) pairs (their K, V, Q, dO
  // stay in L2 together); inside a group the key tiles go heaviest first.
  const int per_kv = p.num_tiles * p.head_split;
  const int grp = static_cast<int>(blockIdx.x) / (C::KV_GROUP * per_kv);
  const int in_grp = min(C::KV_GROUP, p.BHkv - grp * C::KV_GROUP);
  const int r0 = static_cast<int>(blockIdx.x) - grp * C::KV_GROUP * per_kv;
  const int kt = r0 / (in_grp * p.head_split);
  const int r1 = r0 - kt * in_grp * p.head_split;
  const int bhkv = grp * C::KV_GROUP + r1 / p.head_split;
  const int slice = r1 - (r1 / p.head_split) * p.head_split;
  const int b = bhkv / p.Hkv;
  const int hkv = bhkv - b * p.Hkv;
  const int k0 = kt * C::BK;
  const int group = p.Hq / p.Hkv;
  const int heads = group / p.head_split;
  const int h_first = slice * heads;
  const int n_qt = (p.N + C::BQ - 1) / C::BQ;
  const int i_begin = p.causal ? k0 / C::BQ : 0;  // first query tile that sees key tile kt
  const int per_head = n_qt - i_begin;
  const int steps = heads * per_head;

  WaitCtl wc{&abort_flag, p.timeout_ns};

  if (threadIdx.x == 0) {
    abort_flag = 0;
    mbar_init(smem_u32(&bar_kv), 1);
    mbar_init(smem_u32(&bar_qfull), 1);
    mbar_init(smem_u32(&bar_qempty), 1);
    mbar_init(smem_u32(&bar_dofull), 1);
    mbar_init(smem_u32(&bar_doempty), 1);
    mbar_init(smem_u32(&bar_sfull), 1);
    mbar_init(smem_u32(&bar_dpfull), 1);
    mbar_init(smem_u32(&bar_pempty), 1);
    mbar_init(smem_u32(&bar_dsempty), 1);
    mbar_init(smem_u32(&bar_dq0full), 1);
    mbar_init(smem_u32(&bar_dq1full), 1);
    mbar_init(smem_u32(&bar_final), 1);
    mbar_init(smem_u32(&bar_pfull), 256);
    mbar_init(smem_u32(&bar_dsfull), 256);
    mbar_init(smem_u32(&bar_dq0free), 128);
    mbar_init(smem_u32(&bar_dq1afree), 128);
    mbar_init(smem_u32(&bar_dq1bfree), 128);
    fence_mbar_init();
  }
  if (warp == 13) {
    tmem_alloc(smem_u32(&tmem_slot), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;

  auto step_tile = [&](int t, int& bhq, int& q0) {
    const int hh = t / per_head;
    q0 = (i_begin + (t - hh * per_head)) * C::BQ;
    bhq = b * p.Hq + hkv * group + h_first + hh;
  };

  if (warp >= 12) {
    set_max_regs<C::OTHER_REGS, C::LAUNCH_REGS>();
    if (warp == 12) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      prefetch_tmap(&tm_q);
      prefetch_tmap(&tm_do);
      mbar_arrive_expect_tx(smem_u32(&bar_kv), 2 * C::KV_BYTES);
      for (int c = 0; c < 4; ++c) {
        tma_load_3d(sK + c * C::KV_CHUNK, &tm_k, smem_u32(&bar_kv), c * 64, k0, bhkv);
        tma_load_3d(sV + c * C::KV_CHUNK, &tm_v, smem_u32(&bar_kv), c * 64, k0, bhkv);
      }
      int q_issued = 0, do_issued = 0;
      for (int t = 0; t < steps; ++t) {
        int bhq, q0;
        step_tile(t, bhq, q0);
        if (!mbar_wait(smem_u32(&bar_qempty), (t & 1) ^ 1, wc)) break;
        const uint32_t qb = smem_u32(&bar_qfull);
        mbar_arrive_expect_tx(qb, C::Q_BYTES + C::STATS_BYTES);
        for (int c = 0; c < 4; ++c) tma_load_3d(sQ + c * C::Q_CHUNK, &tm_q, qb, c * 64, q0, bhq);
        const size_t roff = static_cast<size_t>(bhq) * p.Npad + q0;
        bulk_load(sST, p.ws_lse2 + roff, 512, qb);
        bulk_load(sST + 512, p.ws_delta + roff, 512, qb);
        q_issued = t + 1;
        if (!mbar_wait(smem_u32(&bar_doempty), (t & 1) ^ 1, wc)) break;
        const uint32_t db = smem_u32(&bar_dofull);
        mbar_arrive_expect_tx(db, C::Q_BYTES);
        for (int c = 0; c < 4; ++c) tma_load_3d(sDO + c * C::Q_CHUNK, &tm_do, db, c * 64, q0, bhq);
        do_issued = t + 1;
      }
      // leave no copy in flight into shared memory
      (void)mbar_wait_drain(smem_u32(&bar_kv), 0, p.timeout_ns);
      if (q_issued > 0) (void)mbar_wait_drain(smem_u32(&bar_qfull), (q_issued - 1) & 1, p.timeout_ns);
      if (do_issued > 0) (void)mbar_wait_drain(smem_u32(&bar_dofull), (do_issued - 1) & 1, p.timeout_ns);
    }
    } else if (warp == 13) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t id_s = idesc_bf16_f32(128, 64, false, false);   // S, dP: [q x keys]
      constexpr uint32_t id_t = idesc_bf16_f32(128, 64, true, true);     // dV^T, dK^T: [d x keys]
      constexpr uint32_t id_q = idesc_bf16_f32(128, 128, false, true);   // dQ half: [q x d]
      bool ok = mbar_wait(smem_u32(&bar_kv), 0, wc);
      for (int t = 0; ok && t < steps; ++t) {
        const uint32_t ph = t & 1;
        // S = Q K^T over d: the S columns are free once the drain has read
        // the first 64 columns of dQ(t-1) half 1 from them
        if (!mbar_wait(smem_u32(&bar_qfull), ph, wc)) { ok = false; break; }
        if (t > 0 && !mbar_wait(smem_u32(&bar_dq1afree), ph ^ 1, wc)) { ok = false; break; }
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 16; ++kk)
          mma_bf16_ss(tmem + C::T_S, sdesc_sw128(sQ + (kk >> 2) * C::Q_CHUNK + (kk & 3) * 32, 16, 1024),
                      sdesc_sw128(sK + (kk >> 2) * C::KV_CHUNK + (kk & 3) * 32, 16, 1024), id_s, kk > 0);
        mma_commit(smem_u32(&bar_sfull));
        // dP = dO V^T, in the columns of dQ(t-1) half 1's last 64
        if (!mbar_wait(smem_u32(&bar_dofull), ph, wc)) { ok = false; break; }
        if (t > 0 && !mbar_wait(smem_u32(&bar_dq1bfree), ph ^ 1, wc)) { ok = false; break; }
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 16; ++kk)
          mma_bf16_ss(tmem + C::T_DP, sdesc_sw128(sDO + (kk >> 2) * C::Q_CHUNK + (kk & 3) * 32, 16, 1024),
                      sdesc_sw128(sV + (kk >> 2) * C::KV_CHUNK + (kk & 3) * 32, 16, 1024), id_s, kk > 0);
        mma_commit(smem_u32(&bar_dpfull));
        // dV^T += dO^T P (two 128-row halves of d)
        if (!mbar_wait(smem_u32(&bar_pfull), ph, wc)) { ok = false; break; }
        tc_fence_after();
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_bf16_ss(tmem + C::T_DV + h * 64, sdesc_sw128(sDO + 2 * h * C::Q_CHUNK + kk * 2048, C::Q_CHUNK, 1024),
                        sdesc_sw128(sP + kk * 2048, 8192, 1024), id_t, t > 0 || kk > 0);
        mma_commit(smem_u32(&bar_doempty));
        mma_commit(smem_u32(&bar_pempty));
        // dK^T += Q^T dS
        if (!mbar_wait(smem_u32(&bar_dsfull), ph, wc)) { ok = false; break; }
        tc_fence_after();
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_bf16_ss(tmem + C::T_DK + h * 64, sdesc_sw128(sQ + 2 * h * C::Q_CHUNK + kk * 2048, C::Q_CHUNK, 1024),
                        sdesc_sw128(sDS + kk * 2048, 8192, 1024), id_t, t > 0 || kk > 0);
        mma_commit(smem_u32(&bar_qempty));
        // dQ = dS K in two 128-column halves: half 1 first, over S and dP
        // (both read by the compute warps before they formed dS), so the
        // drain frees those columns, which S(t+1) needs, as early as it can;
        // half 0 into its own columns once the drain has read half 0 of dQ(t-1)
        tc_fence_after();
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          const int h = 1 - i;
          if (h == 0 && t > 0 && !mbar_wait(smem_u32(&bar_dq0free), ph ^ 1, wc)) { ok = false; break; }
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_bf16_ss(tmem + (h == 0 ? C::T_DQ0 : C::T_DQ1), sdesc_sw128(sDS + kk * 32, 16, 1024),
                        sdesc_sw128(sK + 2 * h * C::KV_CHUNK + kk * 2048, C::KV_CHUNK, 1024), id_q, kk > 0);
          mma_commit(smem_u32(h == 0 ? &bar_dq0full : &bar_dq1full));
        }
        if (!ok) break;
        mma_commit(smem_u32(&bar_dsempty));
      }
      // no MMA may be in flight when tensor memory is released
      mma_commit(smem_u32(&bar_final));
      (void)mbar_wait_drain(smem_u32(&bar_final), 0, p.timeout_ns);
    }
    }  // warps 14, 15: idle
  } else if (warp < 8) {
    set_max_regs<C::COMPUTE_REGS, C::LAUNCH_REGS>();
    // ---------------------------------------------------- compute warpgroups
    // Thread = query row r of the step's tile (TMEM lane r); warpgroup h
    // owns key columns [32h, 32h + 32), i.e. 16-byte chunks 4h .. 4h + 3 of
    // the row's 128 bytes in the P and dS tiles (stored at chunk ^ (r & 7),
    // the 128-byte swizzle).
    const int h = warp >> 2;
    const int r = threadIdx.x & 127;
    const uint32_t lane_base = ((warp & 3) * 32u) << 16;
    const float* stats = reinterpret_cast<const float*>(gbase + (sST - base));
    uint8_t* p_row = gbase + (sP - base) + r * 128;
    uint8_t* ds_row = gbase + (sDS - base) + r * 128;
    const int key_first = k0 + 32 * h;
    bool ok = true;
    for (int t = 0; t < steps; ++t) {
      int bhq, q0;
      step_tile(t, bhq, q0);
      const uint32_t ph = t & 1;
      const int q = q0 + r;
      if (!warp_wait(smem_u32(&bar_qfull), ph, wc)) { ok = false; break; }
      if (!warp_wait(smem_u32(&bar_sfull), ph, wc)) { ok = false; break; }
      tc_fence_after();
      const float lse2 = stats[r];
      const float dlt = stats[128 + r];
      uint32_t sr[32];
      tmem_ld32(tmem + lane_base + C::T_S + 32 * h, sr);
      // keys past N (zero-filled rows) and, causal, keys after the query get
      // weight 0; queries past N have LSE2 = +inf, so weight 0 as well
      const int lim = min(p.causal ? q + 1 : p.N, p.N) - key_first;  // keys [key_first, key_first + lim) visible
      uint32_t pk[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        float p0 = ex2_approx(fmaf(__uint_as_float(sr[2 * j]), p.scale_log2, -lse2));
        float p1 = ex2_approx(fmaf(__uint_as_float(sr[2 * j + 1]), p.scale_log2, -lse2));
        if (2 * j >= lim) p0 = 0.f;
        if (2 * j + 1 >= lim) p1 = 0.f;
        pk[j] = pack_bf16x2(p0, p1);
      }
      if (t > 0 && !warp_wait(smem_u32(&bar_pempty), ph ^ 1, wc)) { ok = false; break; }  // dV^T(t-1) read P
#pragma unroll
      for (int c = 0; c < 4; ++c)
        *reinterpret_cast<uint4*>(p_row + (((4 * h + c) ^ (r & 7)) * 16)) =
            make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
      fence_proxy_async_smem();
      mbar_arrive(smem_u32(&bar_pfull));
      // dS = P (dP - D) scale
      if (!warp_wait(smem_u32(&bar_dpfull), ph, wc)) { ok = false; break; }
      tc_fence_after();
      uint32_t dr[32];
      tmem_ld32(tmem + lane_base + C::T_DP + 32 * h, dr);
      uint32_t w[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const float e0 = bf16_lo(pk[j]) * (__uint_as_float(dr[2 * j]) - dlt) * p.scale;
        const float e1 = bf16_hi(pk[j]) * (__uint_as_float(dr[2 * j + 1]) - dlt) * p.scale;
        w[j] = pack_bf16x2(e0, e1);
      }
      if (t > 0 && !warp_wait(smem_u32(&bar_dsempty), ph ^ 1, wc)) { ok = false; break; }  // dK^T, dQ (t-1) read dS
#pragma unroll
      for (int c = 0; c < 4; ++c)
        *reinterpret_cast<uint4*>(ds_row + (((4 * h + c) ^ (r & 7)) * 16)) =
            make_uint4(w[4 * c], w[4 * c + 1], w[4 * c + 2], w[4 * c + 3]);
      fence_proxy_async_smem();
      tc_fence_before();  // S and dP have been read: dQ half 1 may overwrite them
      mbar_arrive(smem_u32(&bar_dsfull));
    }
    // epilogue: warpgroup 0 writes dV, warpgroup 1 dK. Thread = head-dim
    // index r of each 128-row half; 64 keys along the columns.
    if (ok && warp_wait(smem_u32(&bar_final), 0, wc)) {
      tc_fence_after();
      const uint32_t col = h == 0 ? C::T_DV : C::T_DK;
      __nv_bfloat16* out = h == 0 ? p.dv : p.dk;
      float* acc = h == 0 ? p.dv_acc : p.dk_acc;
#pragma unroll
      for (int half = 0; half < 2; ++half) {
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          uint32_t v[32];
          tmem_ld32(tmem + lane_base + col + half * 64 + c * 32, v);
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int key = k0 + c * 32 + j;
            if (key < p.N) {
              const size_t idx = (static_cast<size_t>(bhkv) * p.N + key) * C::HD + half * 128 + r;
              if (p.head_split > 1) atomicAdd(acc + idx, __uint_as_float(v[j]));
              else out[idx] = __float2bfloat16_rn(__uint_as_float(v[j]));
            }
          }
        }
      }
    }
  } else {
    set_max_regs<C::DRAIN_REGS, C::LAUNCH_REGS>();
    // ------------------------------------------------------------ dQ drain
    // dQ(t) leaves TMEM in four 64-column pieces: half 1 first (in the order
    // the MMAs produce the halves), and of it first the piece over the S
    // columns, which S(t+1) waits for, then the piece over the dP columns.
    // Each piece is loaded in the 16x256b shape (32 rows x 64 columns a warp),
    // its columns freed as far as the next MMA needs them, transposed across
    // the lanes (drain_rowset) and added into the f32 accumulator with 8-byte
    // reductions, each warp instruction 256 contiguous bytes of one row.
    const uint32_t lane_base = ((warp & 3) * 32u) << 16;
    const int wrow = (warp & 3) * 32;  // the warp's 32 rows of the tile
    const int g = lane >> 2, c = lane & 3;
    bool ok = true;
    for (int t = 0; ok && t < steps; ++t) {
      int bhq, q0;
      step_tile(t, bhq, q0);
      const uint32_t ph = t & 1;
      float* tile = p.dq_acc + (static_cast<size_t>(bhq) * p.N + q0) * C::HD;
      const int live = p.N - q0 - wrow;  // rows of the warp's 32 inside N
#pragma unroll 1
      for (int i = 0; i < 4; ++i) {
        const int half = i < 2 ? 1 : 0;
        const int piece = i & 1;
        if (piece == 0 && !warp_wait(smem_u32(half == 0 ? &bar_dq0full : &bar_dq1full), ph, wc)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t src = tmem + lane_base + (half == 0 ? C::T_DQ0 : C::T_DQ1) + piece * 64;
        uint32_t va[32], vb[32];
        tmem_ld_16x256b_x8_async(src, va);                // rows g, g + 8 of the warp's 32
        tmem_ld_16x256b_x8_async(src + (16u << 16), vb);  // rows g + 16, g + 24
        tmem_wait_ld32(va);
        tmem_tie32(vb);
        if (half == 1 || piece == 1) {
          tc_fence_before();
          mbar_arrive(smem_u32(half == 1 ? (piece == 0 ? &bar_dq1afree : &bar_dq1bfree) : &bar_dq0free));
        }
        float x0[8][2], x1[8][2], x2[8][2], x3[8][2];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          x0[k][0] = __uint_as_float(va[4 * k]);
          x0[k][1] = __uint_as_float(va[4 * k + 1]);
          x1[k][0] = __uint_as_float(va[4 * k + 2]);
          x1[k][1] = __uint_as_float(va[4 * k + 3]);
          x2[k][0] = __uint_as_float(vb[4 * k]);
          x2[k][1] = __uint_as_float(vb[4 * k + 1]);
          x3[k][0] = __uint_as_float(vb[4 * k + 2]);
          x3[k][1] = __uint_as_float(vb[4 * k + 3]);
        }
        // after the transposes lane 4 g + c writes columns 8g + 2c, +1 of each row
        float* base = tile + static_cast<size_t>(wrow) * C::HD + half * 128 + piece * 64 + 8 * g + 2 * c;
        drain_rowset<0>(base, x0, g, live);
        drain_rowset<8>(base, x1, g, live);
        drain_rowset<16>(base, x2, g, live);
        drain_rowset<24>(base, x3, g, live);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 13) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace fa
