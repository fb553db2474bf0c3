// bwd2_sm100.cuh -- pipelined recompute backward (bf16, head dimension 64 or
// 128) for sm_100a.
//
// The forward keeps only O and the per-row log-sum-exp; the backward
// recomputes every score tile from Q and K and rebuilds the weights from the
// stored statistics without a second pass (fanfani.net "FlashAttention", "The
// backward pass, and where the memory saving comes from"; synthetic.wiki
// "FlashAttention: attention's bottleneck is the wire, not the maths", "The
// backward pass buys memory with recompute"). The gradient is the textbook
// derivative of the softmax:
//   P  = exp(scale S - LSE)         dV = P^T dO
//   dP = dO V^T                     D  = rowsum(dO * O)   (prep kernel)
//   dS = P * (dP - D)               dQ = scale dS K,  dK = scale dS^T Q
//
// One CTA per (128-key tile, batch, KV head, head slice); it loops over its
// slice of the query heads of the group and the query tiles that see its key
// tile. With one slice (the usual case) it writes dK and dV in bf16; when the
// host splits the group over several CTAs (too few CTAs for the SMs
// otherwise, as with one KV head), each CTA adds its f32 share into dK/dV
// accumulators that a conversion kernel rounds afterwards. Roles (16 warps):
//   warps 0-7   two compute warpgroups; warpgroup h owns query columns
//               [64h, 64h + 64): P^T = exp2(S^T * scale * log2 e - LSE2) ->
//               bf16 over its own S^T columns in TMEM (A operand of dV),
//               then dS^T = P^T (dP^T - D) scale (bf16) -> shared memory,
//               where it is the A operand of dK (read as keys x queries) and
//               of dQ (read as queries x keys)
//   warps 8-11  dQ drain: the dQ tile leaves TMEM at once, then is added to
//               the f32 accumulator with TMA tensor reduce-adds
//   warp 12     TMA producer (K, V once; Q, LSE2, D double-buffered; dO)
//   warp 13     TMEM allocator and MMA issuer; warps 14, 15 idle
// MMA order per step t (query tile):
//   dP^T(t) [once dQ(t-1) left TMEM], dV += P^T dO, S^T(t+1) [over P^T(t),
//   which dV(t) has read], dQ(t) [into the dP^T columns], dK += dS^T Q: the
//   next step's scores are ready while the compute warpgroups form dS^T(t),
//   dQ(t) reaches the drain without waiting for dK(t), and the drain empties
//   dQ(t) while they work on step t+1.
// TMEM: S^T / P^T at 0, dP^T / dQ at 128, dV at 256, dK at 256 + d.
// Every MMA runs 128 x 128 (or 128 x d) per instruction, the size at which
// operands in shared memory and in tensor memory both keep the tensor core
// at its full rate.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include "sm100_ptx.cuh"
#include "bwd_sm100.cuh"  // ws_seq_base

namespace fa {

template <int HD>
struct Bwd2Cfg {
  static constexpr int TILE = 128 * HD * 2;  // one 128-row bf16 tile
  static constexpr int QST = 2;              // stages of (Q, LSE2, D)
  static constexpr int DOST = HD == 64 ? 2 : 1;
  static constexpr int QSTAGE_BYTES = TILE + 1024;
  static constexpr int DS_BYTES = 128 * 128 * 2;
  // dQ staging: one 32-row x 32-column f32 box per drain warp (its own rows
  // of the tile), each added to the accumulator with a TMA reduce-add
  static constexpr int DQ_BOX_ROWS = 32;
  static constexpr int DQ_BOX_BYTES = DQ_BOX_ROWS * 32 * 4;
  static constexpr int DQ_STAGE_BYTES = 4 * DQ_BOX_BYTES;
  static constexpr int SMEM_BYTES =
      1024 + 2 * TILE + QST * QSTAGE_BYTES + DOST * TILE + DS_BYTES + DQ_STAGE_BYTES;
  static constexpr int THREADS = 512;
  // Launch with 128 registers per thread (16 warps, 4 per SM sub-partition),
  // then redistribute per warpgroup: 128 x (2 compute + drain + other) =
  // 512 x 128. The drain holds a whole dQ row (HD registers), so at d = 64 it
  // gives registers to the compute warpgroups.
  static constexpr int LAUNCH_REGS = 128;
  static constexpr int COMPUTE_REGS = HD == 64 ? 136 : 120;
  static constexpr int DRAIN_REGS = HD == 64 ? 136 : 168;
  static constexpr int OTHER_REGS = 104;
  static_assert(128 * (2 * COMPUTE_REGS + DRAIN_REGS + OTHER_REGS) <= THREADS * LAUNCH_REGS,
                "register split exceeds the launch allocation");
  static constexpr int KV_GROUP = 8;  // (batch, KV head) pairs scheduled together
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t T_S = 0;
  static constexpr uint32_t T_DP = 128;
  static constexpr uint32_t T_DV = 256;
  static constexpr uint32_t T_DK = 256 + HD;
};

struct Bwd2Params {
  const float* ws_delta;
  const float* ws_lse2;
  float* dq_acc;
  __nv_bfloat16* dk;
  __nv_bfloat16* dv;
  float* dk_acc;   // [B*Hkv][N][d] f32, used when head_split > 1
  float* dv_acc;
  int N, Npad, Hq, Hkv, num_tiles;
  int head_split;  // CTAs sharing the query heads of one (KV head, key tile)
  int BHkv;        // B * Hkv
  float scale_log2;
  float scale;
  int causal;
  unsigned long long timeout_ns;
  // Packed variable-length batches (the VARLEN kernel only): sequence s owns
  // query tokens cu_q[s] .. cu_q[s+1]-1 of Q, dO [total_q][Hq][d] and key
  // tokens cu_k[s] .. cu_k[s+1]-1 of K, V, dK, dV [total_k][Hkv][d]; its
  // queries are its last positions. The dQ accumulator is laid out like Q.
  // Each query head's workspace row (Npad floats) holds sequence s from
  // ws_seq_base(s), so every 128-row tile starts on a 16-byte boundary.
  // num_tiles covers the longest key sequence.
  const int* cu_q;
  const int* cu_k;
  int batch, total_q, total_k, max_seqlen_q, max_seqlen_k;
  // PARTIAL kernel (one key block of a longer sequence): the causal diagonal
  // moved by diag_shift keys, query i sees key j iff j <= i + diag_shift; dK
  // and dV are added into dk_acc, dv_acc (f32, not zeroed here).
  int diag_shift;
};


// 16 warps, 4 per SM sub-partition: 16384 / 128 -> 128 registers at launch.
// VARLEN: packed variable-length batches (see Bwd2Params); the tensor maps are
// then rank-3 views {d, heads, tokens} with a {64 or 32, 1, 128} box, which
// lands in shared memory like the dense box.
// PARTIAL: dense layout, shifted diagonal, dK/dV added into f32 accumulators.
template <int HD, bool VARLEN = false, bool PARTIAL = false>
__global__ void __launch_bounds__(512, 1)
    fa_bwd2_main_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                        const __grid_constant__ CUtensorMap tm_dq, const Bwd2Params p) {
  using C = Bwd2Cfg<HD>;
  constexpr int QST = C::QST, DOST = C::DOST;
  constexpr int KCH = HD / 64;

  extern __shared__ uint8_t smem_raw[];
  __shared__ uint64_t bar_kv, bar_qfull[QST], bar_qempty[QST], bar_dofull[DOST], bar_doempty[DOST];
  __shared__ uint64_t bar_sfull, bar_pfull, bar_dpfull, bar_dsfull, bar_dqfull, bar_dqfree, bar_final;
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;

  const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
  uint8_t* const gbase = smem_raw + (base - smem_u32(smem_raw));
  const uint32_t sK = base;
  const uint32_t sV = sK + C::TILE;
  const uint32_t sQ = sV + C::TILE;                    // stage s: Q at +s*QSTAGE, LSE2/D after Q
  const uint32_t sDO = sQ + QST * C::QSTAGE_BYTES;
  const uint32_t sDS = sDO + DOST * C::TILE;
  const uint32_t sDQ = sDS + C::DS_BYTES;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // Block order (dense): groups of KV_GROUP (batch, KV head) pairs, whose K,
  // V, Q and dO stay in L2 together; inside a group the key tiles go
  // heaviest first (tile 0 has the most work when causal), each over the
  // group's heads and head slices, so the last blocks to start are the
  // shortest. Variable-length: every (sequence, KV head, slice) at one key
  // tile index, tile indices from 0 up; CTAs past their sequence's keys
  // leave at once.
  int kt, bhkv, slice, b, hkv;
  int q_len, k_len, q_tok = 0, k_tok = 0, ws_base = 0;
  if constexpr (VARLEN) {
    const int per_kt = p.batch * p.Hkv * p.head_split;
    kt = static_cast<int>(blockIdx.x) / per_kt;
    const int r0 = static_cast<int>(blockIdx.x) - kt * per_kt;
    b = r0 / (p.Hkv * p.head_split);
    const int r1 = r0 - b * p.Hkv * p.head_split;
    hkv = r1 / p.head_split;
    slice = r1 - hkv * p.head_split;
    bhkv = hkv;
    q_tok = p.cu_q[b];
    k_tok = p.cu_k[b];
    q_len = p.cu_q[b + 1] - q_tok;
    k_len = p.cu_k[b + 1] - k_tok;
    const bool bad = q_tok < 0 || k_tok < 0 || q_len < 0 || k_len < q_len || q_len > p.max_seqlen_q ||
                     k_len > p.max_seqlen_k || q_tok + q_len > p.total_q || k_tok + k_len > p.total_k;
    if (bad) {
      if (threadIdx.x == 0) atomicCAS(&g_status, 0, kStatusInvalid);
      return;
    }
    if (kt * 128 >= k_len) return;  // no keys of this sequence here
    ws_base = ws_seq_base(q_tok, b);
  } else {
    const int per_kv = p.num_tiles * p.head_split;
    const int grp = static_cast<int>(blockIdx.x) / (C::KV_GROUP * per_kv);
    const int in_grp = min(C::KV_GROUP, p.BHkv - grp * C::KV_GROUP);
    const int r0 = static_cast<int>(blockIdx.x) - grp * C::KV_GROUP * per_kv;
    kt = r0 / (in_grp * p.head_split);
    const int r1 = r0 - kt * in_grp * p.head_split;
    bhkv = grp * C::KV_GROUP + r1 / p.head_split;
    slice = r1 - (r1 / p.head_split) * p.head_split;
    b = bhkv / p.Hkv;
    hkv = bhkv - b * p.Hkv;
    q_len = k_len = p.N;
  }
  const int k0 = kt * 128;
  const int group = p.Hq / p.Hkv;
  const int heads = group / p.head_split;  // query heads of this CTA's slice
  const int h_first = slice * heads;
  // query i of the sequence sits at key position kv_off + i (its last
  // positions when it has fewer queries than keys)
  const int kv_off = k_len - q_len + (PARTIAL ? p.diag_shift : 0);
  const int i_begin = p.causal ? max(0, (k0 - kv_off) / 128) : 0;  // first query tile that sees key tile kt
  const int per_head = (q_len + 127) / 128 - i_begin;
  const int steps = heads * max(per_head, 0);
  if (steps == 0) {
    // no query sees this key tile (a sequence without queries, or a shifted
    // diagonal): its keys get zero gradients, already zero (or left as they
    // are) in f32 accumulators
    if (p.head_split == 1 && !PARTIAL && threadIdx.x < 256) {
      const int key = k0 + (threadIdx.x & 127);
      if (key < k_len) {
        const size_t row = VARLEN ? static_cast<size_t>(k_tok + key) * p.Hkv + hkv : static_cast<size_t>(bhkv) * p.N + key;
        __nv_bfloat16* out = (threadIdx.x < 128 ? p.dv : p.dk) + row * HD;
#pragma unroll
        for (int i = 0; i < HD / 8; ++i) reinterpret_cast<uint4*>(out)[i] = make_uint4(0u, 0u, 0u, 0u);
      }
    }
    return;
  }

  WaitCtl wc{&abort_flag, p.timeout_ns};

  if (threadIdx.x == 0) {
    abort_flag = 0;
    mbar_init(smem_u32(&bar_kv), 1);
    for (int s = 0; s < QST; ++s) {
      mbar_init(smem_u32(&bar_qfull[s]), 1);
      mbar_init(smem_u32(&bar_qempty[s]), 1);
    }
    for (int s = 0; s < DOST; ++s) {
      mbar_init(smem_u32(&bar_dofull[s]), 1);
      mbar_init(smem_u32(&bar_doempty[s]), 1);
    }
    mbar_init(smem_u32(&bar_sfull), 1);
    mbar_init(smem_u32(&bar_pfull), 256);
    mbar_init(smem_u32(&bar_dpfull), 1);
    mbar_init(smem_u32(&bar_dsfull), 256);
    mbar_init(smem_u32(&bar_dqfull), 1);
    mbar_init(smem_u32(&bar_dqfree), 128);
    mbar_init(smem_u32(&bar_final), 1);
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

  // step t: query tile q0 of query head hq (dense: row bhq = b Hq + hq of the
  // [B Hq] heads; variable-length: hq itself, the sequence being fixed)
  auto step_tile = [&](int t, int& bhq, int& q0) {
    const int hh = t / per_head;
    q0 = (i_begin + (t - hh * per_head)) * 128;
    bhq = (VARLEN ? 0 : b * p.Hq) + hkv * group + h_first + hh;
  };
  // TMA coordinates (y, z) of row r of query head row bhq / of the key tile
  auto q_yz = [&](int bhq, int r, int& y, int& z) {
    y = VARLEN ? bhq : r;
    z = VARLEN ? q_tok + r : bhq;
  };

  if (warp >= 12) {
    set_max_regs<C::OTHER_REGS, C::LAUNCH_REGS>();
    if (warp == 12) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      prefetch_tmap(&tm_q);
      prefetch_tmap(&tm_do);
      mbar_arrive_expect_tx(smem_u32(&bar_kv), 2 * C::TILE);
      const int ky = VARLEN ? hkv : k0, kz = VARLEN ? k_tok + k0 : bhkv;
      for (int c = 0; c < KCH; ++c) {
        tma_load_3d(sK + c * 16384, &tm_k, smem_u32(&bar_kv), c * 64, ky, kz);
        tma_load_3d(sV + c * 16384, &tm_v, smem_u32(&bar_kv), c * 64, ky, kz);
      }
      int q_issued = 0, do_issued = 0;
      for (int t = 0; t < steps; ++t) {
        int bhq, q0;
        step_tile(t, bhq, q0);
        const int sq = t % QST, sd = t % DOST;
        if (!mbar_wait(smem_u32(&bar_qempty[sq]), ((t / QST) & 1) ^ 1, wc)) break;
        const uint32_t qst = sQ + sq * C::QSTAGE_BYTES;
        const uint32_t qb = smem_u32(&bar_qfull[sq]);
        mbar_arrive_expect_tx(qb, C::QSTAGE_BYTES);
        int qy, qz;
        q_yz(bhq, q0, qy, qz);
        for (int c = 0; c < KCH; ++c) tma_load_3d(qst + c * 16384, &tm_q, qb, c * 64, qy, qz);
        const size_t roff = static_cast<size_t>(bhq) * p.Npad + ws_base + q0;
        bulk_load(qst + C::TILE, p.ws_lse2 + roff, 512, qb);
        bulk_load(qst + C::TILE + 512, p.ws_delta + roff, 512, qb);
        q_issued = t + 1;
        if (!mbar_wait(smem_u32(&bar_doempty[sd]), ((t / DOST) & 1) ^ 1, wc)) break;
        const uint32_t db = smem_u32(&bar_dofull[sd]);
        mbar_arrive_expect_tx(db, C::TILE);
        for (int c = 0; c < KCH; ++c) tma_load_3d(sDO + sd * C::TILE + c * 16384, &tm_do, db, c * 64, qy, qz);
        do_issued = t + 1;
      }
      // leave no copy in flight into shared memory (a bounded wait elsewhere
      // may have given up before these stages were consumed)
      (void)mbar_wait_drain(smem_u32(&bar_kv), 0, p.timeout_ns);
      for (int t = max(0, q_issued - QST); t < q_issued; ++t)
        (void)mbar_wait_drain(smem_u32(&bar_qfull[t % QST]), (t / QST) & 1, p.timeout_ns);
      for (int t = max(0, do_issued - DOST); t < do_issued; ++t)
        (void)mbar_wait_drain(smem_u32(&bar_dofull[t % DOST]), (t / DOST) & 1, p.timeout_ns);
    }
  } else if (warp == 13) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t id_kk = idesc_bf16_f32(128, 128, false, false);  // S^T, dP^T
      constexpr uint32_t id_kmn = idesc_bf16_f32(128, HD, false, true);   // dV, dK
      constexpr uint32_t id_mnmn = idesc_bf16_f32(128, HD, true, true);   // dQ
      auto issue_s = [&](int t) {
        const uint32_t qst = sQ + (t % QST) * C::QSTAGE_BYTES;
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) {
          const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
          mma_bf16_ss(tmem + C::T_S, sdesc_sw128(sK + off, 16, 1024), sdesc_sw128(qst + off, 16, 1024), id_kk,
                      kk > 0);
        }
        mma_commit(smem_u32(&bar_sfull));
      };
      bool ok = mbar_wait(smem_u32(&bar_kv), 0, wc) && mbar_wait(smem_u32(&bar_qfull[0]), 0, wc);
      if (ok) {
        tc_fence_after();
        issue_s(0);
      }
      for (int t = 0; ok && t < steps; ++t) {
        const int sq = t % QST, sd = t % DOST;
        const uint32_t qst = sQ + sq * C::QSTAGE_BYTES;
        const uint32_t dob = sDO + sd * C::TILE;
        if (t > 0 && !mbar_wait(smem_u32(&bar_dqfree), (t - 1) & 1, wc)) break;
        if (!mbar_wait(smem_u32(&bar_dofull[sd]), (t / DOST) & 1, wc)) break;
        tc_fence_after();
        // dP^T = V dO^T
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) {
          const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
          mma_bf16_ss(tmem + C::T_DP, sdesc_sw128(sV + off, 16, 1024), sdesc_sw128(dob + off, 16, 1024), id_kk,
                      kk > 0);
        }
        mma_commit(smem_u32(&bar_dpfull));
        // dV += P^T dO
        if (!mbar_wait(smem_u32(&bar_pfull), t & 1, wc)) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_bf16_ts(tmem + C::T_DV, tmem + C::T_S + (kk >> 2) * 64 + (kk & 3) * 8,
                      sdesc_sw128(dob + kk * 2048, 16384, 1024), id_kmn,
                      (t > 0 || kk > 0));
        mma_commit(smem_u32(&bar_doempty[sd]));
        // S^T(t+1) may overwrite P^T(t) now (MMAs run in issue order, dV(t)
        // first); dS^T(t) lives in shared memory, so the next step's scores
        // are computed while the compute warpgroups form dS^T(t)
        if (t + 1 < steps) {
          if (!mbar_wait(smem_u32(&bar_qfull[(t + 1) % QST]), ((t + 1) / QST) & 1, wc)) break;
          tc_fence_after();
          issue_s(t + 1);
        }
        // dQ = dS K (A = dS^T's shared-memory tile read as queries x keys,
        // M-major), then dK += dS^T Q (the same tile as keys x queries,
        // K-major). dQ goes first: the drain, and through it dP^T(t+1), wait
        // for it, while nothing waits for dK before the next step's dK.
        if (!mbar_wait(smem_u32(&bar_dsfull), t & 1, wc)) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_bf16_ss(tmem + C::T_DP, sdesc_sw128(sDS + kk * 2048, 16384, 1024),
                      sdesc_sw128(sK + kk * 2048, 16384, 1024), id_mnmn, kk > 0);
        mma_commit(smem_u32(&bar_dqfull));
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_bf16_ss(tmem + C::T_DK, sdesc_sw128(sDS + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024),
                      sdesc_sw128(qst + kk * 2048, 16384, 1024), id_kmn, (t > 0 || kk > 0));
        // the Q stage and the dS tile are free once dK(t) has completed
        mma_commit(smem_u32(&bar_qempty[sq]));
      }
      // bar_final completes once every MMA issued above has completed (on
      // the normal path and after a bounded wait gave up alike); no MMA may
      // be in flight when tensor memory is released
      mma_commit(smem_u32(&bar_final));
      (void)mbar_wait_drain(smem_u32(&bar_final), 0, p.timeout_ns);
    }
    }  // warps 14, 15: idle
  } else if (warp < 8) {
    set_max_regs<C::COMPUTE_REGS, C::LAUNCH_REGS>();
    // ---------------------------------------------------- compute warpgroups
    // Warpgroup `half` owns query columns [64 half, 64 half + 64) of every
    // step: it turns its S^T columns into P^T (bf16, written over its own
    // S^T columns 64 half .. 64 half + 31) and later its dP^T columns into
    // dS^T (bf16, written over S^T columns 64 half + 32 .. 64 half + 63, and
    // into shared-memory block `half`). Both warpgroups cover all 128 key
    // rows (TMEM lane = key).
    const int half = warp >> 2;
    const int tid = threadIdx.x & 127;  // key row k0 + tid
    const int cb = half * 64;           // first query column of this warpgroup
    const uint32_t lane_base = ((warp & 3) * 32u) << 16;
    const int key = k0 + tid;
    const bool key_live = key < k_len;
    uint8_t* ds_row = gbase + (sDS - base) + half * 16384 + tid * 128;
    bool ok = true;
    for (int t = 0; t < steps; ++t) {
      int bhq, q0;
      step_tile(t, bhq, q0);
      const int sq = t % QST;
      const float* lse2 = reinterpret_cast<const float*>(gbase + (sQ - base) + sq * C::QSTAGE_BYTES + C::TILE);
      const float4* l4 = reinterpret_cast<const float4*>(lse2 + cb);
      const float4* d4 = reinterpret_cast<const float4*>(lse2 + 128 + cb);
      if (!warp_wait(smem_u32(&bar_qfull[sq]), (t / QST) & 1, wc)) { ok = false; break; }
      if (!warp_wait(smem_u32(&bar_sfull), t & 1, wc)) { ok = false; break; }
      tc_fence_after();
      // ---- P^T = exp2(S^T * scale * log2 e - LSE2), masked; kept in
      // registers too, since S^T(t+1) overwrites these columns once dV(t) has
      // read them
      // some element of the tile is masked: a key after its query (causal),
      // or, variable-length, a query past the sequence's end (its workspace
      // row may belong to the next sequence, so the weight is zeroed here;
      // dense padding rows have LSE = +inf and weigh 0 already)
      const bool mask = VARLEN    ? (p.causal && k0 + 127 > kv_off + q0) || q0 + 128 > q_len
                        : PARTIAL ? p.causal && k0 + 127 > kv_off + q0
                                  : p.causal && q0 == k0;
      uint32_t pk[32];
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        uint32_t rr[32];
        tmem_ld32(tmem + lane_base + C::T_S + cb + 32 * u, rr);
#pragma unroll
        for (int x = 0; x < 8; ++x) {
          const float4 L = l4[u * 8 + x];
          const int qa = cb + u * 32 + 4 * x;  // query column of element 0
          float pv[4];
          pv[0] = ex2_approx(fmaf(__uint_as_float(rr[4 * x]), p.scale_log2, -L.x));
          pv[1] = ex2_approx(fmaf(__uint_as_float(rr[4 * x + 1]), p.scale_log2, -L.y));
          pv[2] = ex2_approx(fmaf(__uint_as_float(rr[4 * x + 2]), p.scale_log2, -L.z));
          pv[3] = ex2_approx(fmaf(__uint_as_float(rr[4 * x + 3]), p.scale_log2, -L.w));
          if (mask) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int qi = q0 + qa + e;
              if (VARLEN ? (p.causal && key > kv_off + qi) || qi >= q_len : PARTIAL ? key > kv_off + qi : qi < key)
                pv[e] = 0.f;
            }
          }
          pk[u * 16 + 2 * x] = key_live ? pack_bf16x2(pv[0], pv[1]) : 0u;
          pk[u * 16 + 2 * x + 1] = key_live ? pack_bf16x2(pv[2], pv[3]) : 0u;
        }
        uint32_t half_pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) half_pk[i] = pk[u * 16 + i];
        tmem_st16(tmem + lane_base + C::T_S + cb + u * 16, half_pk);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(smem_u32(&bar_pfull));
      // ---- dS^T = P^T (dP^T - D) * scale -> shared memory
      // dS(t-1) consumed: dK(t-1), the last MMA to read it, completes the
      // release of Q stage (t-1) % QST
      if (t > 0 && !warp_wait(smem_u32(&bar_qempty[(t - 1) % QST]), ((t - 1) / QST) & 1, wc)) { ok = false; break; }
      if (!warp_wait(smem_u32(&bar_dpfull), t & 1, wc)) { ok = false; break; }
      tc_fence_after();
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        uint32_t r[32];
        tmem_ld32(tmem + lane_base + C::T_DP + cb + u * 32, r);
        uint32_t w[16];
#pragma unroll
        for (int x = 0; x < 8; ++x) {
          const float4 Dv = d4[u * 8 + x];
          const uint32_t p01 = pk[u * 16 + 2 * x], p23 = pk[u * 16 + 2 * x + 1];
          const float e0 = bf16_lo(p01) * (__uint_as_float(r[4 * x]) - Dv.x) * p.scale;
          const float e1 = bf16_hi(p01) * (__uint_as_float(r[4 * x + 1]) - Dv.y) * p.scale;
          const float e2 = bf16_lo(p23) * (__uint_as_float(r[4 * x + 2]) - Dv.z) * p.scale;
          const float e3 = bf16_hi(p23) * (__uint_as_float(r[4 * x + 3]) - Dv.w) * p.scale;
          w[2 * x] = pack_bf16x2(e0, e1);
          w[2 * x + 1] = pack_bf16x2(e2, e3);
        }
        // 32 queries = 64 bytes = four 16-byte chunks: chunk u*4 + v, swizzled by row
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          const int chunk = (u * 4 + v) ^ (tid & 7);
          *reinterpret_cast<uint4*>(ds_row + chunk * 16) = make_uint4(w[4 * v], w[4 * v + 1], w[4 * v + 2], w[4 * v + 3]);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(smem_u32(&bar_dsfull));
    }
    // epilogue: warpgroup 0 writes dV, warpgroup 1 writes dK (dS carries the
    // scale): bf16 rows, or, when the group's heads are split over several
    // CTAs, f32 rows added into the accumulators
    if (ok && warp_wait(smem_u32(&bar_final), 0, wc)) {
      tc_fence_after();
      const size_t row_off = VARLEN ? (static_cast<size_t>(k_tok + (key_live ? key : 0)) * p.Hkv + hkv) * HD
                                    : (static_cast<size_t>(bhkv) * p.N + (key_live ? key : 0)) * HD;
      __nv_bfloat16* out = (half == 0 ? p.dv : p.dk) + row_off;
      const bool to_acc = p.head_split > 1 || PARTIAL;
      float* acc = to_acc ? (half == 0 ? p.dv_acc : p.dk_acc) + row_off : nullptr;
      const uint32_t col = half == 0 ? C::T_DV : C::T_DK;
#pragma unroll
      for (int c = 0; c < HD / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(tmem + lane_base + col + c * 32, r);
        if (to_acc) {
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
  } else {
    set_max_regs<C::DRAIN_REGS, C::LAUNCH_REGS>();
    // ------------------------------------------------------- dQ warpgroup
    // Thread i of the warpgroup holds query row q0 + i of the dQ tile (TMEM lane = row).
    // The whole tile is loaded into registers and its columns released to
    // dP^T(t+1) at once; then, 32 head-dim columns at a time, each warp
    // writes its 32 rows to its own 128-byte-swizzled staging box (one
    // 16-byte vector per store) and adds the box to the f32 accumulator with
    // a TMA tensor reduce-add, which also drops rows past N. The four warps
    // run independently: while the TMA unit reads one warp's box at the rate
    // the L2 takes the reductions, the other warps fill theirs.
    const int dw = warp & 3;  // rows 32 dw .. 32 dw + 31 of the tile
    const uint32_t lane_base = (dw * 32u) << 16;
    const uint32_t box = sDQ + dw * C::DQ_BOX_BYTES;
    uint8_t* stage_row = gbase + (box - base) + lane * 128;
    bool ok = true;
    for (int t = 0; t < steps; ++t) {
      int bhq, q0;
      step_tile(t, bhq, q0);
      ok = warp_wait(smem_u32(&bar_dqfull), t & 1, wc) && ok;
      uint32_t rr[HD / 32][32];
      if (ok) {
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < HD / 32; ++c) tmem_ld32_async(tmem + lane_base + C::T_DP + c * 32, rr[c]);
        tmem_wait_ld32(rr[0]);
#pragma unroll
        for (int c = 1; c < HD / 32; ++c) tmem_tie32(rr[c]);
        tc_fence_before();
        mbar_arrive(smem_u32(&bar_dqfree));  // the tile is in registers
      }
#pragma unroll
      for (int c = 0; c < HD / 32; ++c) {
        if (lane == 0) bulk_wait_group_read<0>();  // this warp's last reduce has read its box
        __syncwarp();
        if (ok) {
#pragma unroll
          for (int u = 0; u < 8; ++u)
            *reinterpret_cast<uint4*>(stage_row + ((u ^ (lane & 7)) * 16)) =
                make_uint4(rr[c][4 * u], rr[c][4 * u + 1], rr[c][4 * u + 2], rr[c][4 * u + 3]);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0 && ok) {
          int qy, qz;
          q_yz(bhq, q0 + 32 * dw, qy, qz);
          tma_reduce_add_3d(&tm_dq, box, c * 32, qy, qz);
          bulk_commit_group();
        }
      }
    }
    if (lane == 0) bulk_wait_all();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 13) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace fa
