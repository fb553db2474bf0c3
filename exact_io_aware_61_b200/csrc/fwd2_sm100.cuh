// fwd2_sm100.cuh -- bf16 attention forward with two query tiles per CTA
// (head dimensions 64 and 128).
//
// Same method as fwd_sm100.cuh (tiled pass, online softmax with a lazy
// rescale of the running output, O = o / l once at the end), arranged so the
// tensor core is never idle waiting on one softmax:
//   * a CTA owns 256 query rows = two 128-row tiles of one (batch, head);
//     both tiles read the same K/V tiles, halving shared-memory fills per
//     FLOP;
//   * each tile has its own softmax warpgroup and its own S and O in TMEM
//     (S0 | S1 | O0 | O1 = 512 columns at d = 128), and the MMA issuer
//     alternates PV0(j), S0(j+1), PV1(j), S1(j+1), so one warpgroup's
//     softmax runs while the other tile's MMAs execute;
//   * the softmax reads a whole 128-column score row with one TMEM load and
//     reduces it with short trees (three-input max, packed f32x2 FMA/add).
// Warps: 0-3 softmax tile 0, 4-7 softmax tile 1, 8 TMA producer, 9 TMEM
// allocator and MMA issuer, 10-11 idle. The block launches with 168
// registers per thread; the two softmax warpgroups then take 216 each and the
// third warpgroup keeps 72 (128 x (216 + 216 + 72) = 384 x 168). The host
// launches the kernel only if its register count is exactly 168, since a
// split above the launch allocation would wait forever.
#pragma once

#include <cuda.h>
#include "sm100_ptx.cuh"

namespace fa {

template <int HD>
struct Fwd2Cfg {
  static constexpr int BM = 128;  // rows per query tile
  static constexpr int BN = 128;  // keys per key tile
  // K and V ring depths. K runs one tile ahead of V (S(j+1) is issued right
  // after P(j)V(j)), so at d = 128 it gets the extra stage that fits.
  static constexpr int KST = HD == 64 ? 4 : 3;
  static constexpr int VST = HD == 64 ? 4 : 2;
  static constexpr int Q_TILE_BYTES = BM * HD * 2;
  static constexpr int KV_BYTES = BN * HD * 2;
  static constexpr int SMEM_BYTES = 1024 + 2 * Q_TILE_BYTES + (KST + VST) * KV_BYTES;
  static constexpr int THREADS = 384;
  static constexpr int LAUNCH_REGS = 168;  // the split below assumes exactly this
  static constexpr int SOFTMAX_REGS = 216;
  static constexpr int OTHER_REGS = 72;
  static_assert(128 * (2 * SOFTMAX_REGS + OTHER_REGS) <= THREADS * LAUNCH_REGS, "register split exceeds launch");
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t TMEM_O = 256;  // O0 at 256, O1 at 256 + HD
  // d = 64 leaves room for P in its own columns (P0 at 384, P1 at 448), so
  // S(j+1) can be computed as soon as the softmax has read S(j) instead of
  // after P(j)V(j); at d = 128 P overwrites S.
  static constexpr bool SEP_P = HD == 64;
  static constexpr uint32_t TMEM_P = 384;
  static constexpr float RESCALE_THRESHOLD = 8.0f;
  static constexpr int HEAD_GROUP = 8;  // heads scheduled together (K/V stay in L2)
  // Roles of the third warpgroup. Warp w runs on SM sub-partition w % 4,
  // which it shares with softmax warps w % 4 and w % 4 + 4.
  static constexpr int PRODUCER_WARP = 8;
  static constexpr int MMA_WARP = 9;
};

struct Fwd2Params {
  __nv_bfloat16* o;
  float* lse;
  int N, Hq, Hkv, BH, num_pairs;
  float scale_log2;
  int causal;
  unsigned long long timeout_ns;
  // Packed variable-length batches (the VARLEN kernel only): sequence s owns
  // query tokens cu_q[s] .. cu_q[s+1]-1 and key tokens cu_k[s] .. cu_k[s+1]-1
  // of Q [total_q][Hq][d] and K, V [total_k][Hkv][d]; O is laid out like Q and
  // LSE is [total_q][Hq]. num_pairs covers max_seqlen_q.
  const int* cu_q;
  const int* cu_k;
  int batch, total_q, total_k, max_seqlen_q;
  // Causal diagonal moved by diag_shift keys: query i (at key position
  // k_len - q_len + i) sees key j iff j <= k_len - q_len + i + diag_shift.
  // Negative shifts leave rows with no visible key: O = 0, LSE = -inf.
  int diag_shift;
};


// ---------------------------------------------------------------- helpers

FA_DEV float max3f(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// One 32-lane x 128-column TMEM load (one column per register), waited.
FA_DEV void tmem_ld128(uint32_t taddr, uint32_t (&r)[128]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x128.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, "
      "%32, %33, %34, %35, %36, %37, %38, %39, %40, %41, %42, %43, %44, %45, %46, %47, "
      "%48, %49, %50, %51, %52, %53, %54, %55, %56, %57, %58, %59, %60, %61, %62, %63, "
      "%64, %65, %66, %67, %68, %69, %70, %71, %72, %73, %74, %75, %76, %77, %78, %79, "
      "%80, %81, %82, %83, %84, %85, %86, %87, %88, %89, %90, %91, %92, %93, %94, %95, "
      "%96, %97, %98, %99, %100, %101, %102, %103, %104, %105, %106, %107, %108, %109, %110, %111, "
      "%112, %113, %114, %115, %116, %117, %118, %119, %120, %121, %122, %123, %124, %125, %126, %127}, [%128];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]),
        "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]),
        "=r"(r[40]), "=r"(r[41]), "=r"(r[42]), "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]),
        "=r"(r[48]), "=r"(r[49]), "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]),
        "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]), "=r"(r[62]), "=r"(r[63]),
        "=r"(r[64]), "=r"(r[65]), "=r"(r[66]), "=r"(r[67]), "=r"(r[68]), "=r"(r[69]), "=r"(r[70]), "=r"(r[71]),
        "=r"(r[72]), "=r"(r[73]), "=r"(r[74]), "=r"(r[75]), "=r"(r[76]), "=r"(r[77]), "=r"(r[78]), "=r"(r[79]),
        "=r"(r[80]), "=r"(r[81]), "=r"(r[82]), "=r"(r[83]), "=r"(r[84]), "=r"(r[85]), "=r"(r[86]), "=r"(r[87]),
        "=r"(r[88]), "=r"(r[89]), "=r"(r[90]), "=r"(r[91]), "=r"(r[92]), "=r"(r[93]), "=r"(r[94]), "=r"(r[95]),
        "=r"(r[96]), "=r"(r[97]), "=r"(r[98]), "=r"(r[99]), "=r"(r[100]), "=r"(r[101]), "=r"(r[102]),
        "=r"(r[103]), "=r"(r[104]), "=r"(r[105]), "=r"(r[106]), "=r"(r[107]), "=r"(r[108]), "=r"(r[109]),
        "=r"(r[110]), "=r"(r[111]), "=r"(r[112]), "=r"(r[113]), "=r"(r[114]), "=r"(r[115]), "=r"(r[116]),
        "=r"(r[117]), "=r"(r[118]), "=r"(r[119]), "=r"(r[120]), "=r"(r[121]), "=r"(r[122]), "=r"(r[123]),
        "=r"(r[124]), "=r"(r[125]), "=r"(r[126]), "=r"(r[127])
      : "r"(taddr)
      : "memory");
}

// ------------------------------------------------------------------ kernel

// VARLEN: packed variable-length batches (see Fwd2Params); the tensor maps
// are then rank-3 views {d, heads, tokens} with a {64, 1, 128} box, which
// lands in shared memory exactly like the dense {64, 128, 1} box, so only the
// coordinates, the per-sequence lengths and the output addressing change.
template <int HD, bool VARLEN = false>
// 12 warps: 3 per SM sub-partition, 16384 / 96 -> 168 registers each at launch.
__global__ void __launch_bounds__(384, 1)
    fa_fwd_bf16_2tile_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                             const __grid_constant__ CUtensorMap tm_v, const Fwd2Params p) {
  using C = Fwd2Cfg<HD>;
  constexpr int KST = C::KST, VST = C::VST;
  constexpr int KCH = HD / 64;

  extern __shared__ uint8_t smem_raw[];
  __shared__ uint64_t bar_q, bar_kfull[KST], bar_kempty[KST], bar_vfull[VST], bar_vempty[VST];
  __shared__ uint64_t bar_sfull[2], bar_pfull[2], bar_odone[2], bar_sfree[2], bar_drain;
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;

  const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
  const uint32_t sQ = base;  // tile t at sQ + t * Q_TILE_BYTES
  const uint32_t sK = sQ + 2 * C::Q_TILE_BYTES;
  const uint32_t sV = sK + KST * C::KV_BYTES;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // Work item: groups of HEAD_GROUP heads; inside a group the heaviest
  // (last) tile pairs of every head start first.
  const int bid = blockIdx.x;
  // Dense: groups of HEAD_GROUP heads, heaviest tile pairs of every head
  // first. Varlen: every (sequence, head) of the batch at one tile pair
  // index, pair indices from the last (heaviest when causal) down; CTAs past
  // their sequence's length leave at once.
  int pair, bh, hq, bh_kv;
  int q_len, k_len, q_tok = 0, k_tok = 0;
  if constexpr (VARLEN) {
    const int per_pair = p.batch * p.Hq;
    pair = p.num_pairs - 1 - bid / per_pair;
    const int rem = bid - (bid / per_pair) * per_pair;
    const int sq = rem / p.Hq;
    hq = rem - sq * p.Hq;
    bh = sq;
    bh_kv = hq / (p.Hq / p.Hkv);
    q_tok = p.cu_q[sq];
    k_tok = p.cu_k[sq];
    q_len = p.cu_q[sq + 1] - q_tok;
    k_len = p.cu_k[sq + 1] - k_tok;
    const bool bad = q_tok < 0 || k_tok < 0 || q_len < 0 || k_len < q_len || q_len > p.max_seqlen_q ||
                     q_tok + q_len > p.total_q || k_tok + k_len > p.total_k;
    if (bad) {
      if (threadIdx.x == 0) atomicCAS(&g_status, 0, kStatusInvalid);
      return;
    }
    if (pair * 2 * C::BM >= q_len) return;  // no rows of this sequence here
  } else {
    const int per_group = C::HEAD_GROUP * p.num_pairs;
    const int g = bid / per_group;
    const int heads_in_group = min(C::HEAD_GROUP, p.BH - g * C::HEAD_GROUP);
    const int r = bid - g * per_group;
    pair = p.num_pairs - 1 - r / heads_in_group;
    bh = g * C::HEAD_GROUP + r % heads_in_group;
    const int b = bh / p.Hq;
    hq = bh - b * p.Hq;
    bh_kv = b * p.Hkv + hq / (p.Hq / p.Hkv);
    q_len = k_len = p.N;
  }
  // query i of the (sequence's) tile sees keys up to kv_off + i: the last
  // positions when a sequence has fewer queries than keys, moved by the shift
  const int kv_off = k_len - q_len + p.diag_shift;
  const int q0 = pair * 2 * C::BM;
  const int n_kv_total = (k_len + C::BN - 1) / C::BN;
  int n_t[2];
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    const int qs = q0 + t * C::BM;
    const int last_key = kv_off + qs + C::BM - 1;  // causal: the last key any row of the tile sees
    n_t[t] = qs >= q_len ? 0 : !p.causal ? n_kv_total : last_key < 0 ? 0 : min(last_key / C::BN + 1, n_kv_total);
  }
  const int n_max = max(n_t[0], n_t[1]);
  if (n_max == 0) {
    // causal with a negative shift: no row of either tile sees a key
    if (warp < 8) {
      const int row = q0 + (warp >> 2) * C::BM + (threadIdx.x & 127);
      if (row < q_len) {
        const size_t o_index = VARLEN ? static_cast<size_t>(q_tok + row) * p.Hq + hq : static_cast<size_t>(bh) * p.N + row;
        uint4* dst = reinterpret_cast<uint4*>(p.o + o_index * HD);
#pragma unroll
        for (int i = 0; i < HD / 8; ++i) dst[i] = make_uint4(0u, 0u, 0u, 0u);
        p.lse[o_index] = -INFINITY;
      }
    }
    return;
  }
  // TMA coordinates (y, z) of query row 0 and of key row 0
  const int qy = VARLEN ? hq : 0, qz = VARLEN ? q_tok : bh;
  const int ky = VARLEN ? bh_kv : 0, kz = VARLEN ? k_tok : bh_kv;

  WaitCtl wc{&abort_flag, p.timeout_ns};

  if (threadIdx.x == 0) {
    abort_flag = 0;
    mbar_init(smem_u32(&bar_q), 1);
    for (int s = 0; s < KST; ++s) {
      mbar_init(smem_u32(&bar_kfull[s]), 1);
      mbar_init(smem_u32(&bar_kempty[s]), 1);
    }
    for (int s = 0; s < VST; ++s) {
      mbar_init(smem_u32(&bar_vfull[s]), 1);
      mbar_init(smem_u32(&bar_vempty[s]), 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(smem_u32(&bar_sfull[t]), 1);
      mbar_init(smem_u32(&bar_pfull[t]), 128);
      mbar_init(smem_u32(&bar_odone[t]), 1);
      mbar_init(smem_u32(&bar_sfree[t]), 128);
    }
    mbar_init(smem_u32(&bar_drain), 1);
    fence_mbar_init();
  }
  if (warp == C::MMA_WARP) {
    tmem_alloc(smem_u32(&tmem_slot), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;

  if (warp >= 8) {
    set_max_regs<C::OTHER_REGS, C::LAUNCH_REGS>();
  }
  if (warp >= 8 && warp != C::PRODUCER_WARP && warp != C::MMA_WARP) {
    // idle warps of the third warpgroup
  } else if (warp == C::PRODUCER_WARP) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      prefetch_tmap(&tm_q);
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_v);
      const int live_tiles = n_t[1] > 0 ? 2 : 1;
      mbar_arrive_expect_tx(smem_u32(&bar_q), live_tiles * C::Q_TILE_BYTES);
      for (int t = 0; t < live_tiles; ++t)
        for (int c = 0; c < KCH; ++c)
          tma_load_3d(sQ + t * C::Q_TILE_BYTES + c * (C::BM * 128), &tm_q, smem_u32(&bar_q), c * 64,
                      VARLEN ? qy : q0 + t * C::BM, VARLEN ? qz + q0 + t * C::BM : qz);
      // order K(0), K(1), V(0), K(2), V(1), ...: K one tile ahead of V
      int k_issued = 0, v_issued = 0;
      for (int i = 0; i <= n_max; ++i) {
        if (i < n_max) {
          const int s = i % KST;
          if (!mbar_wait(smem_u32(&bar_kempty[s]), ((i / KST) & 1) ^ 1, wc)) break;
          mbar_arrive_expect_tx(smem_u32(&bar_kfull[s]), C::KV_BYTES);
          for (int c = 0; c < KCH; ++c)
            tma_load_3d(sK + s * C::KV_BYTES + c * (C::BN * 128), &tm_k, smem_u32(&bar_kfull[s]), c * 64,
                        VARLEN ? ky : i * C::BN, VARLEN ? kz + i * C::BN : kz);
          k_issued = i + 1;
        }
        if (i >= 1) {
          const int j = i - 1, s = j % VST;
          if (!mbar_wait(smem_u32(&bar_vempty[s]), ((j / VST) & 1) ^ 1, wc)) break;
          mbar_arrive_expect_tx(smem_u32(&bar_vfull[s]), C::KV_BYTES);
          for (int c = 0; c < KCH; ++c)
            tma_load_3d(sV + s * C::KV_BYTES + c * (C::BN * 128), &tm_v, smem_u32(&bar_vfull[s]), c * 64,
                        VARLEN ? ky : j * C::BN, VARLEN ? kz + j * C::BN : kz);
          v_issued = j + 1;
        }
      }
      // leave no copy in flight into shared memory (a bounded wait elsewhere
      // may have given up before these stages were consumed)
      (void)mbar_wait_drain(smem_u32(&bar_q), 0, p.timeout_ns);
      for (int i = max(0, k_issued - KST); i < k_issued; ++i)
        (void)mbar_wait_drain(smem_u32(&bar_kfull[i % KST]), (i / KST) & 1, p.timeout_ns);
      for (int j = max(0, v_issued - VST); j < v_issued; ++j)
        (void)mbar_wait_drain(smem_u32(&bar_vfull[j % VST]), (j / VST) & 1, p.timeout_ns);
    }
  } else if (warp == C::MMA_WARP) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(128, 128, false, false);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(128, HD, false, true);
      auto issue_s = [&](int t, int j) {
        const uint32_t kb = sK + (j % KST) * C::KV_BYTES;
        const uint32_t qb = sQ + t * C::Q_TILE_BYTES;
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) {
          const uint32_t off = (kk >> 2) * (128 * 128) + (kk & 3) * 32;
          mma_bf16_ss(tmem + t * 128, sdesc_sw128(qb + off, 16, 1024), sdesc_sw128(kb + off, 16, 1024), idesc_qk,
                      kk > 0);
        }
        mma_commit(smem_u32(&bar_sfull[t]));
      };
      bool ok = mbar_wait(smem_u32(&bar_q), 0, wc) && mbar_wait(smem_u32(&bar_kfull[0]), 0, wc);
      if (ok) {
        tc_fence_after();
        for (int t = 0; t < 2; ++t)
          if (n_t[t] > 0) issue_s(t, 0);
        mma_commit(smem_u32(&bar_kempty[0]));
      }
      for (int j = 0; ok && j < n_max; ++j) {
        const int s = j % VST;
        bool v_ready = false, k_next_ready = false;
        if constexpr (!C::SEP_P) {
          // V(j) and K(j+1) were loaded at least a key tile ago (their stages
          // were released by earlier iterations): wait for them here, while the
          // softmax still works on S(j), not between a tile's P and its MMAs
          if (!mbar_wait(smem_u32(&bar_vfull[s]), (j / VST) & 1, wc)) break;
          v_ready = true;
          if (j + 1 < n_max) {
            if (!mbar_wait(smem_u32(&bar_kfull[(j + 1) % KST]), ((j + 1) / KST) & 1, wc)) break;
            k_next_ready = true;
          }
          tc_fence_after();
        }
        if constexpr (C::SEP_P) {
          // S(j+1) of each tile as soon as its softmax has read S(j); P(j)
          // has its own columns, so it does not wait for P(j)V(j)
          for (int t = 0; t < 2 && ok; ++t) {
            if (j + 1 >= n_t[t]) continue;
            if (!mbar_wait(smem_u32(&bar_sfree[t]), j & 1, wc)) { ok = false; break; }
            if (!k_next_ready) {
              if (!mbar_wait(smem_u32(&bar_kfull[(j + 1) % KST]), ((j + 1) / KST) & 1, wc)) { ok = false; break; }
              k_next_ready = true;
            }
            tc_fence_after();
            issue_s(t, j + 1);
          }
          if (!ok) break;
          if (k_next_ready) mma_commit(smem_u32(&bar_kempty[(j + 1) % KST]));
        }
        for (int t = 0; t < 2 && ok; ++t) {
          if (j >= n_t[t]) continue;
          if (!mbar_wait(smem_u32(&bar_pfull[t]), j & 1, wc)) { ok = false; break; }
          if (!v_ready) {
            if (!mbar_wait(smem_u32(&bar_vfull[s]), (j / VST) & 1, wc)) { ok = false; break; }
            v_ready = true;
          }
          tc_fence_after();
          const uint32_t vb = sV + s * C::KV_BYTES;
          const uint32_t pa = tmem + (C::SEP_P ? C::TMEM_P + t * 64 : t * 128);
#pragma unroll
          for (int kk = 0; kk < C::BN / 16; ++kk)
            mma_bf16_ts(tmem + C::TMEM_O + t * HD, pa + kk * 8, sdesc_sw128(vb + kk * 2048, C::BN * 128, 1024),
                        idesc_pv, (j > 0 || kk > 0));
          mma_commit(smem_u32(&bar_odone[t]));
          if (!C::SEP_P && j + 1 < n_t[t]) {
            if (!k_next_ready) {
              if (!mbar_wait(smem_u32(&bar_kfull[(j + 1) % KST]), ((j + 1) / KST) & 1, wc)) { ok = false; break; }
              k_next_ready = true;
              tc_fence_after();
            }
            issue_s(t, j + 1);
          }
        }
        if (!ok) break;
        mma_commit(smem_u32(&bar_vempty[s]));
        if (!C::SEP_P && k_next_ready) mma_commit(smem_u32(&bar_kempty[(j + 1) % KST]));
      }
      // no MMA may be in flight when tensor memory is released
      mma_commit(smem_u32(&bar_drain));
      (void)mbar_wait_drain(smem_u32(&bar_drain), 0, p.timeout_ns);
    }
  } else {
    // ------------------------------------------------------------- softmax
    set_max_regs<C::SOFTMAX_REGS, C::LAUNCH_REGS>();
    const int t = warp >> 2;                      // query tile of this warpgroup
    const int row = q0 + t * C::BM + (threadIdx.x & 127);
    const uint32_t lane_base = ((warp & 3) * 32u) << 16;
    const uint32_t s_addr = tmem + lane_base + t * 128;
    const uint32_t o_addr = tmem + lane_base + C::TMEM_O + t * HD;
    const int n = n_t[t];
    const uint64_t c2 = pack2(p.scale_log2, p.scale_log2);
    float m_ref = -INFINITY;
    float l = 0.f;
    bool ok = true;
    for (int j = 0; j < n; ++j) {
      if (!warp_wait(smem_u32(&bar_sfull[t]), j & 1, wc)) { ok = false; break; }
      tc_fence_after();
      uint32_t sr[128];
      tmem_ld128(s_addr, sr);
      if constexpr (C::SEP_P) {  // S(j) is in registers: its columns may take S(j+1)
        tc_fence_before();
        mbar_arrive(smem_u32(&bar_sfree[t]));
      }
      const int key0 = j * C::BN;
      if ((p.causal && key0 + C::BN > kv_off + q0 + t * C::BM) || key0 + C::BN > k_len) {
        const int lim = min(p.causal ? kv_off + row + 1 : k_len, k_len) - key0;
#pragma unroll
        for (int c = 0; c < 128; ++c)
          if (c >= lim) sr[c] = __float_as_uint(-INFINITY);
      }
      // row max: eight independent three-input chains, then a short tree
      float mk[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) mk[k] = __uint_as_float(sr[k]);
#pragma unroll
      for (int c = 8; c < 128; c += 16) {
#pragma unroll
        for (int k = 0; k < 8; ++k) mk[k] = max3f(mk[k], __uint_as_float(sr[c + k]), __uint_as_float(sr[c + 8 + k]));
      }
      const float mx = max3f(max3f(mk[0], mk[1], mk[2]), max3f(mk[3], mk[4], mk[5]), fmaxf(mk[6], mk[7])) *
                       p.scale_log2;
      // Raise the reference maximum only when this tile's maximum exceeds it
      // by more than the threshold (decided per warp); the running output is
      // rescaled below, after P is stored, while the score row is dead.
      bool rescale = false;
      float alpha = 1.f;
      if (j == 0) {
        m_ref = mx;
      } else if (__any_sync(0xffffffffu, mx > m_ref + C::RESCALE_THRESHOLD)) {
        const float m_new = fmaxf(m_ref, mx);
        alpha = m_new == -INFINITY ? 1.f : ex2_approx(m_ref - m_new);
        m_ref = m_new;
        rescale = true;
      }
      // p = 2^(s * scale * log2 e - m), packed to bf16 over the S columns; a
      // row that sees no key (m = -inf) takes m = 0, so its p are all 0
      const float m_use = m_ref == -INFINITY ? 0.f : m_ref;
      const uint64_t negm2 = pack2(-m_use, -m_use);
      uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
      uint32_t pk[64];
#pragma unroll
      for (int c = 0; c < 64; ++c) {
        float x0, x1;
        unpack2(ffma2(pack2(__uint_as_float(sr[2 * c]), __uint_as_float(sr[2 * c + 1])), c2, negm2), x0, x1);
        const float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
        acc[c & 3] = fadd2(acc[c & 3], pack2(p0, p1));
        pk[c] = pack_bf16x2(p0, p1);
      }
      float s0, s1;
      unpack2(fadd2(fadd2(acc[0], acc[1]), fadd2(acc[2], acc[3])), s0, s1);
      l = l * alpha + (s0 + s1);
      if constexpr (C::SEP_P) {
        // P(j) goes to its own columns, which P(j-1)V(j-1) reads: wait for it
        if (j > 0) {
          if (!warp_wait(smem_u32(&bar_odone[t]), (j - 1) & 1, wc)) { ok = false; break; }
          tc_fence_after();
        }
      }
      {
        uint32_t h0[32], h1[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          h0[i] = pk[i];
          h1[i] = pk[32 + i];
        }
        const uint32_t p_addr = C::SEP_P ? tmem + lane_base + C::TMEM_P + t * 64 : s_addr;
        tmem_st32(p_addr, h0);
        tmem_st32(p_addr + 32, h1);
      }
      if (rescale) {
        // o was last written by P_{j-1} V_{j-1}: wait for it (done above when
        // P has its own columns), then scale by alpha
        if (!C::SEP_P && !warp_wait(smem_u32(&bar_odone[t]), (j - 1) & 1, wc)) { ok = false; break; }
        tc_fence_after();
        const uint64_t a2 = pack2(alpha, alpha);
#pragma unroll
        for (int c = 0; c < HD / 32; ++c) {
          uint32_t orr[32];
          tmem_ld32(o_addr + c * 32, orr);
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            float lo, hi;
            unpack2(fmul2(pack2(__uint_as_float(orr[2 * i]), __uint_as_float(orr[2 * i + 1])), a2), lo, hi);
            orr[2 * i] = __float_as_uint(lo);
            orr[2 * i + 1] = __float_as_uint(hi);
          }
          tmem_st32(o_addr + c * 32, orr);
        }
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(smem_u32(&bar_pfull[t]));
    }
    if (n > 0 && ok && warp_wait(smem_u32(&bar_odone[t]), (n - 1) & 1, wc)) {
      tc_fence_after();
      const float inv_l = l > 0.f ? 1.f / l : 0.f;  // l = 0: the row saw no key
      const bool live = row < q_len;
      const size_t o_index = VARLEN ? static_cast<size_t>(q_tok + (live ? row : 0)) * p.Hq + hq
                                    : static_cast<size_t>(bh) * p.N + (live ? row : 0);
      __nv_bfloat16* orow = p.o + o_index * HD;
#pragma unroll
      for (int c = 0; c < HD / 32; ++c) {
        uint32_t orr[32];
        tmem_ld32(o_addr + c * 32, orr);
        uint4 w[4];
        uint32_t* wp = reinterpret_cast<uint32_t*>(w);
#pragma unroll
        for (int i = 0; i < 16; ++i)
          wp[i] = pack_bf16x2(__uint_as_float(orr[2 * i]) * inv_l, __uint_as_float(orr[2 * i + 1]) * inv_l);
        if (live) {
          uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
          for (int i = 0; i < 4; ++i) dst[i] = w[i];
        }
      }
      if (live) p.lse[o_index] = l > 0.f ? (m_ref + __log2f(l)) * 0.69314718055994530942f : -INFINITY;
    } else if (n == 0 && ok && row < q_len) {
      // causal with a negative shift: no row of this tile sees a key
      const size_t o_index = VARLEN ? static_cast<size_t>(q_tok + row) * p.Hq + hq : static_cast<size_t>(bh) * p.N + row;
      uint4* dst = reinterpret_cast<uint4*>(p.o + o_index * HD);
#pragma unroll
      for (int i = 0; i < HD / 8; ++i) dst[i] = make_uint4(0u, 0u, 0u, 0u);
      p.lse[o_index] = -INFINITY;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == C::MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace fa
