// bwd_sm100.cuh -- recompute-based attention backward for bf16 on sm_100a.
//
// The forward keeps only O and the per-row log-sum-exp; the backward
// recomputes every score tile from Q and K and rebuilds the weights from the
// stored statistics without a second pass (fanfani.net "FlashAttention", "The
// backward pass, and where the memory saving comes from"; synthetic.wiki
// "FlashAttention: attention's bottleneck is the wire, not the maths", "The
// backward pass buys memory with recompute"). The gradient is the textbook
// derivative of the softmax:
//   P  = exp(scale S - LSE)         dV = P^T dO
//   dP = dO V^T                     D  = rowsum(dO * O)
//   dS = P * (dP - D)               dQ = scale dS K,  dK = scale dS^T Q
//
// Three kernels, in stream order:
//   fa_bwd_prep_kernel   D and LSE * log2(e) into 128-row-padded workspace
//                        rows (+inf / 0 in the padding so padded queries
//                        get zero weight), and zeroes the f32 dQ accumulator
//   fa_bwd_main_kernel   one CTA per (key tile of 128, batch, KV head); loops
//                        over the query heads of the group and the query
//                        tiles that see the key tile; dK, dV accumulate in
//                        TMEM; each dQ tile is added into the f32
//                        accumulator with a TMA reduce-add
//   fa_bwd_dq_kernel     f32 accumulator -> bf16 dQ
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include "sm100_ptx.cuh"

namespace fa {

// -------------------------------------------------------------- preprocess

struct BwdPrepParams {
  const __nv_bfloat16* o;
  const __nv_bfloat16* dO;
  const float* lse;
  float* ws_delta;  // [B*Hq][Npad]
  float* ws_lse2;   // [B*Hq][Npad]
  float* dq_acc;    // [B*Hq][N][d]
  int N, Npad;
};

// 8 threads per row, 32 rows per 256-thread block; 1-D grid of
// (Npad / 32) * B*Hq blocks.
template <int HD>
__global__ void __launch_bounds__(256) fa_bwd_prep_kernel(const BwdPrepParams p) {
  constexpr int PER = HD / 8;  // elements per thread
  const int blocks_per_head = p.Npad / 32;
  const size_t bh = blockIdx.x / blocks_per_head;
  const int sub = threadIdx.x & 7;
  const int row = static_cast<int>(blockIdx.x % blocks_per_head) * 32 + (threadIdx.x >> 3);
  float acc = 0.f;
  const bool live = row < p.N;
  if (live) {
    const size_t off = (bh * p.N + row) * HD + sub * PER;
    const uint4* o4 = reinterpret_cast<const uint4*>(p.o + off);
    const uint4* d4 = reinterpret_cast<const uint4*>(p.dO + off);
    float4* z4 = reinterpret_cast<float4*>(p.dq_acc + off);
#pragma unroll
    for (int i = 0; i < PER / 8; ++i) {
      const uint4 a = o4[i], g = d4[i];
      const uint32_t av[4] = {a.x, a.y, a.z, a.w};
      const uint32_t gv[4] = {g.x, g.y, g.z, g.w};
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        acc = fmaf(bf16_lo(av[t]), bf16_lo(gv[t]), acc);
        acc = fmaf(bf16_hi(av[t]), bf16_hi(gv[t]), acc);
      }
      z4[2 * i] = make_float4(0.f, 0.f, 0.f, 0.f);
      z4[2 * i + 1] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }
  acc += __shfl_xor_sync(0xffffffffu, acc, 1);
  acc += __shfl_xor_sync(0xffffffffu, acc, 2);
  acc += __shfl_xor_sync(0xffffffffu, acc, 4);
  if (sub == 0 && row < p.Npad) {
    const size_t w = bh * p.Npad + row;
    p.ws_delta[w] = live ? acc : 0.f;
    p.ws_lse2[w] = live ? p.lse[bh * p.N + row] * 1.4426950408889634f : INFINITY;
  }
}

// ------------------------------------------------------------ dQ convert

// grid-stride over float4 groups of the accumulator: dq = bf16(acc).
__global__ void __launch_bounds__(256) fa_bwd_dq_kernel(const float* __restrict__ acc,
                                                        __nv_bfloat16* __restrict__ dq, size_t n4) {
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n4;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const float4 v = reinterpret_cast<const float4*>(acc)[i];
    uint2 w;
    w.x = pack_bf16x2(v.x, v.y);
    w.y = pack_bf16x2(v.z, v.w);
    reinterpret_cast<uint2*>(dq)[i] = w;
  }
}

// ------------------------------------------------------------ main kernel

template <int HD>
struct BwdCfg {
  static constexpr int BK = 128;  // keys per CTA
  static constexpr int BQ = 128;  // queries per step
  static constexpr int QST = HD == 64 ? 2 : 1;  // stages of (Q, dO, LSE, D)
  static constexpr int TILE = 128 * HD * 2;     // one 128-row bf16 tile
  static constexpr int DS_BYTES = 128 * 128 * 2;
  static constexpr int DQ_CHUNK = 128 * 32 * 4;  // 128 rows x 32 f32 (one TMA box)
  static constexpr int STAGE_BYTES = 2 * TILE + 2 * 512;
  static constexpr int SMEM_BYTES = 1024 + 2 * TILE + QST * STAGE_BYTES + DS_BYTES + 2 * DQ_CHUNK;
  static constexpr int THREADS = 192;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t T_S = 0;     // S^T, then P^T (bf16) in its first 64 columns
  static constexpr uint32_t T_DP = 128;  // dP^T, then the dQ tile
  static constexpr uint32_t T_DV = 256;
  static constexpr uint32_t T_DK = 256 + HD;
};

struct BwdParams {
  const float* ws_delta;
  const float* ws_lse2;
  __nv_bfloat16* dk;
  __nv_bfloat16* dv;
  int N, Npad, Hq, Hkv, num_tiles;
  float scale_log2;  // scale * log2(e)
  float scale;
  int causal;
  unsigned long long timeout_ns;
};

template <int HD>
__global__ void __launch_bounds__(192, 1)
    fa_bwd_main_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                       const __grid_constant__ CUtensorMap tm_dq, const BwdParams p) {
  using C = BwdCfg<HD>;
  constexpr int QST = C::QST;
  constexpr int KCH = HD / 64;

  extern __shared__ uint8_t smem_raw[];
  __shared__ uint64_t bar_kv, bar_qfull[QST], bar_qempty[QST];
  __shared__ uint64_t bar_sfull, bar_dpfull, bar_pfull, bar_dsfull, bar_dqfull, bar_tfree, bar_final, bar_wg;
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;

  const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
  const uint32_t sK = base;
  const uint32_t sV = sK + C::TILE;
  const uint32_t sStage = sV + C::TILE;  // per stage: Q, dO, LSE2[128], D[128]
  const uint32_t sDS = sStage + QST * C::STAGE_BYTES;
  const uint32_t sDQ = sDS + C::DS_BYTES;
  const uint8_t* gen_base = smem_raw + (base - smem_u32(smem_raw));

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // 1-D grid, head-major; key tile 0 sees the most query tiles under the
  // causal mask, so it starts first.
  const int bhkv = static_cast<int>(blockIdx.x) / p.num_tiles;
  const int kt = static_cast<int>(blockIdx.x) - bhkv * p.num_tiles;
  const int k0 = kt * C::BK;
  const int b = bhkv / p.Hkv;
  const int hkv = bhkv - b * p.Hkv;
  const int group = p.Hq / p.Hkv;
  const int i_begin = p.causal ? kt : 0;
  const int per_head = p.num_tiles - i_begin;
  const int steps = group * per_head;

  WaitCtl wc{&abort_flag, p.timeout_ns};

  if (threadIdx.x == 0) {
    abort_flag = 0;
    mbar_init(smem_u32(&bar_kv), 1);
    for (int s = 0; s < QST; ++s) {
      mbar_init(smem_u32(&bar_qfull[s]), 1);
      mbar_init(smem_u32(&bar_qempty[s]), 1);
    }
    mbar_init(smem_u32(&bar_sfull), 1);
    mbar_init(smem_u32(&bar_dpfull), 1);
    mbar_init(smem_u32(&bar_pfull), 128);
    mbar_init(smem_u32(&bar_dsfull), 128);
    mbar_init(smem_u32(&bar_dqfull), 1);
    mbar_init(smem_u32(&bar_tfree), 128);
    mbar_init(smem_u32(&bar_final), 1);
    mbar_init(smem_u32(&bar_wg), 128);
    fence_mbar_init();
  }
  if (warp == 5) {
    tmem_alloc(smem_u32(&tmem_slot), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;

  if (warp == 4) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      mbar_arrive_expect_tx(smem_u32(&bar_kv), 2 * C::TILE);
      for (int c = 0; c < KCH; ++c) {
        tma_load_3d(sK + c * 16384, &tm_k, smem_u32(&bar_kv), c * 64, k0, bhkv);
        tma_load_3d(sV + c * 16384, &tm_v, smem_u32(&bar_kv), c * 64, k0, bhkv);
      }
      for (int t = 0; t < steps; ++t) {
        const int hh = t / per_head;
        const int i = i_begin + (t - hh * per_head);
        const int bhq = b * p.Hq + hkv * group + hh;
        const int s = t % QST;
        if (!mbar_wait(smem_u32(&bar_qempty[s]), ((t / QST) & 1) ^ 1, wc)) break;
        const uint32_t st = sStage + s * C::STAGE_BYTES;
        const uint32_t fb = smem_u32(&bar_qfull[s]);
        mbar_arrive_expect_tx(fb, C::STAGE_BYTES);
        for (int c = 0; c < KCH; ++c) {
          tma_load_3d(st + c * 16384, &tm_q, fb, c * 64, i * C::BQ, bhq);
          tma_load_3d(st + C::TILE + c * 16384, &tm_do, fb, c * 64, i * C::BQ, bhq);
        }
        const size_t roff = static_cast<size_t>(bhq) * p.Npad + static_cast<size_t>(i) * C::BQ;
        bulk_load(st + 2 * C::TILE, p.ws_lse2 + roff, 512, fb);
        bulk_load(st + 2 * C::TILE + 512, p.ws_delta + roff, 512, fb);
      }
    }
  } else if (warp == 5) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t id_kk = idesc_bf16_f32(128, 128, false, false);  // S^T, dP^T
      constexpr uint32_t id_kmn = idesc_bf16_f32(128, HD, false, true);   // dV, dK
      constexpr uint32_t id_mnmn = idesc_bf16_f32(128, HD, true, true);   // dQ
      bool ok = mbar_wait(smem_u32(&bar_kv), 0, wc);
      for (int t = 0; ok && t < steps; ++t) {
        const int s = t % QST;
        const uint32_t st = sStage + s * C::STAGE_BYTES;
        const uint32_t sQ = st, sDO = st + C::TILE;
        if (!mbar_wait(smem_u32(&bar_qfull[s]), (t / QST) & 1, wc)) break;
        if (t > 0 && !mbar_wait(smem_u32(&bar_tfree), (t - 1) & 1, wc)) break;
        tc_fence_after();
        // S^T = K Q^T   (M = keys, N = queries, K = d)
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) {
          const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
          mma_bf16_ss(tmem + C::T_S, sdesc_sw128(sK + off, 16, 1024), sdesc_sw128(sQ + off, 16, 1024), id_kk,
                      kk > 0);
        }
        mma_commit(smem_u32(&bar_sfull));
        // dP^T = V dO^T
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) {
          const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
          mma_bf16_ss(tmem + C::T_DP, sdesc_sw128(sV + off, 16, 1024), sdesc_sw128(sDO + off, 16, 1024), id_kk,
                      kk > 0);
        }
        mma_commit(smem_u32(&bar_dpfull));
        // dV += P^T dO   (A = P^T in TMEM, B = dO: K = queries, N = d, MN-major)
        if (!mbar_wait(smem_u32(&bar_pfull), t & 1, wc)) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_bf16_ts(tmem + C::T_DV, tmem + C::T_S + kk * 8, sdesc_sw128(sDO + kk * 2048, 16384, 1024), id_kmn,
                      (t > 0 || kk > 0));
        // dK += dS^T Q   (A = dS^T K-major in smem, B = Q MN-major)
        if (!mbar_wait(smem_u32(&bar_dsfull), t & 1, wc)) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
          mma_bf16_ss(tmem + C::T_DK, sdesc_sw128(sDS + off, 16, 1024), sdesc_sw128(sQ + kk * 2048, 16384, 1024),
                      id_kmn, (t > 0 || kk > 0));
        }
        // dQ = dS K   (A = dS MN-major: the same bytes read transposed; B = K MN-major)
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_bf16_ss(tmem + C::T_DP, sdesc_sw128(sDS + kk * 2048, 16384, 1024),
                      sdesc_sw128(sK + kk * 2048, 16384, 1024), id_mnmn, kk > 0);
        mma_commit(smem_u32(&bar_qempty[s]));
        mma_commit(smem_u32(&bar_dqfull));
      }
      mma_commit(smem_u32(&bar_final));
    }
  } else {
    // ------------------------------------------------ compute warpgroup
    const int tid = threadIdx.x;  // key row (S^T, dP^T, dK, dV) and query row (dQ)
    const uint32_t lane_base = (warp * 32u) << 16;
    const int key = k0 + tid;
    bool ok = true;
    uint32_t wg_phase = 0;
    // bounded barrier over the 128 compute threads
    auto wg_sync = [&]() -> bool {
      mbar_arrive(smem_u32(&bar_wg));
      const bool r = warp_wait(smem_u32(&bar_wg), wg_phase, wc);
      wg_phase ^= 1u;
      return r;
    };
    for (int t = 0; t < steps && ok; ++t) {
      const int hh = t / per_head;
      const int i = i_begin + (t - hh * per_head);
      const int bhq = b * p.Hq + hkv * group + hh;
      const int s = t % QST;
      const uint8_t* st_gen = gen_base + (sStage - base) + s * C::STAGE_BYTES;
      const float* lse2 = reinterpret_cast<const float*>(st_gen + 2 * C::TILE);
      const float* delta = lse2 + 128;
      if (!warp_wait(smem_u32(&bar_qfull[s]), (t / QST) & 1, wc)) { ok = false; break; }
      if (!warp_wait(smem_u32(&bar_sfull), t & 1, wc)) { ok = false; break; }
      tc_fence_after();
      // P^T row: this key against the 128 queries of tile i
      const int q0 = i * C::BQ;
      const bool diag = p.causal && (i == kt);
      const bool key_live = key < p.N;
      float pr[128];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t r[32];
        tmem_ld32(tmem + lane_base + C::T_S + c * 32, r);
#pragma unroll
        for (int x = 0; x < 32; ++x) {
          const int qc = c * 32 + x;
          float v = ex2_approx(fmaf(__uint_as_float(r[x]), p.scale_log2, -lse2[qc]));
          if (diag && (q0 + qc < key)) v = 0.f;
          pr[qc] = key_live ? v : 0.f;
        }
      }
      {
        uint32_t pk[32];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
#pragma unroll
          for (int x = 0; x < 32; ++x) pk[x] = pack_bf16x2(pr[h * 64 + 2 * x], pr[h * 64 + 2 * x + 1]);
          tmem_st32(tmem + lane_base + C::T_S + h * 32, pk);
        }
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(smem_u32(&bar_pfull));
      // dS^T row = P^T * (dP^T - D) * scale -> smem (bf16, 128B-swizzled, [key][query])
      if (!warp_wait(smem_u32(&bar_dpfull), t & 1, wc)) { ok = false; break; }
      tc_fence_after();
      uint8_t* ds_row = const_cast<uint8_t*>(gen_base) + (sDS - base) + tid * 128;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t r[32];
        tmem_ld32(tmem + lane_base + C::T_DP + c * 32, r);
        uint32_t w[16];
#pragma unroll
        for (int x = 0; x < 16; ++x) {
          const int q_a = c * 32 + 2 * x, q_b = q_a + 1;
          const float a = pr[q_a] * (__uint_as_float(r[2 * x]) - delta[q_a]) * p.scale;
          const float bb = pr[q_b] * (__uint_as_float(r[2 * x + 1]) - delta[q_b]) * p.scale;
          w[x] = pack_bf16x2(a, bb);
        }
        // 32 queries = 64 bytes = 4 chunks of 16 B; block c/2, chunk (c%2)*4 + u
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int chunk = ((c & 1) * 4 + u) ^ (tid & 7);
          uint4* dst = reinterpret_cast<uint4*>(ds_row + (c >> 1) * 16384 + chunk * 16);
          *dst = make_uint4(w[4 * u], w[4 * u + 1], w[4 * u + 2], w[4 * u + 3]);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(smem_u32(&bar_dsfull));
      // dQ tile (row tid = query q0 + tid) -> smem -> TMA reduce-add into the accumulator
      if (!warp_wait(smem_u32(&bar_dqfull), t & 1, wc)) { ok = false; break; }
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < HD / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(tmem + lane_base + C::T_DP + c * 32, r);
        const int buf = c & 1;
        if (tid == 0 && (c >= 2 || t > 0)) bulk_wait_group_read<1>();
        if (!wg_sync()) { ok = false; break; }
        uint8_t* drow = const_cast<uint8_t*>(gen_base) + (sDQ - base) + buf * C::DQ_CHUNK + tid * 128;
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int chunk = u ^ (tid & 7);
          *reinterpret_cast<uint4*>(drow + chunk * 16) = make_uint4(r[4 * u], r[4 * u + 1], r[4 * u + 2], r[4 * u + 3]);
        }
        fence_proxy_async_smem();
        if (!wg_sync()) { ok = false; break; }
        if (tid == 0) {
          tma_reduce_add_3d(&tm_dq, sDQ + buf * C::DQ_CHUNK, c * 32, q0, bhq);
          bulk_commit_group();
        }
      }
      if (!ok) break;
      tc_fence_before();
      mbar_arrive(smem_u32(&bar_tfree));
    }
    // dK, dV rows of this key tile
    if (ok && warp_wait(smem_u32(&bar_final), 0, wc)) {
      tc_fence_after();
      const bool live = key < p.N;
      const size_t roff = (static_cast<size_t>(bhkv) * p.N + (live ? key : 0)) * HD;
#pragma unroll
      for (int which = 0; which < 2; ++which) {
        __nv_bfloat16* out = (which == 0 ? p.dv : p.dk) + roff;
        const uint32_t col = which == 0 ? C::T_DV : C::T_DK;
#pragma unroll
        for (int c = 0; c < HD / 32; ++c) {
          uint32_t r[32];
          tmem_ld32(tmem + lane_base + col + c * 32, r);
          uint4 w[4];
          uint32_t* wp = reinterpret_cast<uint32_t*>(w);
#pragma unroll
          for (int x = 0; x < 16; ++x) wp[x] = pack_bf16x2(__uint_as_float(r[2 * x]), __uint_as_float(r[2 * x + 1]));
          if (live) {
            uint4* dst = reinterpret_cast<uint4*>(out + c * 32);
#pragma unroll
            for (int x = 0; x < 4; ++x) dst[x] = w[x];
          }
        }
      }
    }
    if (tid == 0) bulk_wait_all();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace fa
