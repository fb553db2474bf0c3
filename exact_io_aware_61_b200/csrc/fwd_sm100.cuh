// fwd_sm100.cuh -- fused exact-attention forward for bf16 on sm_100a.
//
// One CTA owns one tile of 128 query rows of one (batch, query head) and
// streams the key/value tiles of its KV head through shared memory
// (fanfani.net "FlashAttention", "Do not materialize the matrix": load a
// block of queries and a block of keys and values, use the small block of
// scores, discard it). Per key tile j:
//   S_j  = Q K_j^T            tcgen05.mma, bf16 x bf16 -> f32 in TMEM
//   mask (causal diagonal tile, keys past N)
//   online softmax            running max m, normaliser l, rescale of the
//                             running output by 2^(m_old - m_new)
//                             ("A pinch of math"; mentria.ai "The trick: keep
//                             a running max, and rebase as you go.")
//   P_j (bf16) -> TMEM, aliasing S_j
//   O  += P_j V_j             tcgen05.mma with A read from TMEM
// and at the end O = o / l once and LSE = m + ln l.
//
// Roles (192 threads):
//   warps 0-3  softmax: thread t owns query row t = TMEM lane t
//   warp 4     TMA producer (lane 0): Q once, K/V ring
//   warp 5     TMEM allocator + MMA issuer (lane 0)
// TMEM columns: S buffers at 0 and 128 (double-buffered so S_{j+1} is
// computed while the softmax works on S_j), O accumulator at 256..256+d.
//
// The running maximum is kept in base-2 units of the scaled score
// (s * scale * log2 e). It is only raised when a tile's maximum exceeds it by
// more than 8 (a factor 256): o and l are always relative to the same
// reference, so O = o / l is unchanged, and p stays <= 256.
#pragma once

#include <cuda.h>
#include "sm100_ptx.cuh"

namespace fa {

// DECODE: the KV-cache configuration (one CTA per KV head and key split):
// deeper K/V rings, since the whole CTA is a stream of K and V.
template <int HD, bool DECODE = false>
struct FwdCfg {
  static constexpr int BM = 128;  // query rows per CTA
  static constexpr int BN = 128;  // keys per tile
  static constexpr int STAGES = DECODE ? (HD == 64 ? 6 : (HD == 128 ? 3 : 1)) : (HD == 64 ? 4 : (HD == 128 ? 2 : 1));
  static constexpr int Q_BYTES = BM * HD * 2;
  static constexpr int KV_BYTES = BN * HD * 2;
  static constexpr int SMEM_BYTES = 1024 + Q_BYTES + 2 * STAGES * KV_BYTES;
  static constexpr int THREADS = 192;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t TMEM_O = 256;
  static constexpr float RESCALE_THRESHOLD = 8.0f;
};

struct FwdParams {
  __nv_bfloat16* o;
  float* lse;
  int N, Hq, Hkv, num_q_tiles;
  float scale_log2;  // scale * log2(e)
  int causal;
  unsigned long long timeout_ns;
  // causal: query i sees key j iff j <= i + diag_shift; a row that sees no
  // key gets O = 0, LSE = -inf
  int diag_shift;
  // DECODE kernel: N is the number of cached keys Nk; the R = (Hq / Hkv) * Nq
  // query rows of KV head bh_kv are rows bh_kv * R .. bh_kv * R + R - 1 of Q
  // viewed as [B * Hq * Nq][d] (query heads of a group, then queries), and row
  // r is the query at position Nk - Nq + (r mod Nq). CTA (bh_kv, split s)
  // takes key tiles [s * split_tiles, min((s + 1) * split_tiles, tiles)) and
  // writes that split's normalised O and LSE to part s of o, lse laid out as
  // [splits][rows_total = B * Hkv * R][d] and [splits][rows_total].
  int R, Nq, splits, split_tiles, rows_total;
};

template <int HD, bool DECODE = false>
__global__ void __launch_bounds__(192, 1)
    fa_fwd_bf16_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v, const FwdParams p) {
  using C = FwdCfg<HD, DECODE>;
  constexpr int ST = C::STAGES;
  constexpr int KCH = HD / 64;  // 64-column (128-byte) chunks per row

  extern __shared__ uint8_t smem_raw[];
  __shared__ uint64_t bar_q, bar_kfull[ST], bar_kempty[ST], bar_vfull[ST], bar_vempty[ST];
  __shared__ uint64_t bar_sfull[2], bar_pfull[2], bar_odone, bar_drain;
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;

  const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
  const uint32_t sQ = base;
  const uint32_t sK = sQ + C::Q_BYTES;
  const uint32_t sV = sK + ST * C::KV_BYTES;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // 1-D grid, head-major: consecutive CTAs share a KV head (its K/V tiles stay
  // in L2), and within a head the longest (last) query tiles start first.
  // DECODE: consecutive CTAs are the key splits of one KV head.
  const int n_kv_total = (p.N + C::BN - 1) / C::BN;
  int bh, bh_kv, q0, n_kv, j0 = 0;
  size_t out_base = 0;  // DECODE: first output row of this CTA
  if constexpr (DECODE) {
    bh_kv = static_cast<int>(blockIdx.x) / p.splits;
    const int split = static_cast<int>(blockIdx.x) - bh_kv * p.splits;
    j0 = split * p.split_tiles;
    n_kv = min(n_kv_total, j0 + p.split_tiles) - j0;  // >= 1: the host sizes the splits
    bh = bh_kv;
    q0 = bh_kv * p.R;
    out_base = static_cast<size_t>(split) * p.rows_total + static_cast<size_t>(bh_kv) * p.R;
  } else {
    bh = static_cast<int>(blockIdx.x) / p.num_q_tiles;
    const int qt = p.num_q_tiles - 1 - (static_cast<int>(blockIdx.x) - bh * p.num_q_tiles);
    const int b = bh / p.Hq;
    const int hq = bh - b * p.Hq;
    bh_kv = b * p.Hkv + hq / (p.Hq / p.Hkv);
    q0 = qt * C::BM;
    const int last_key = q0 + C::BM - 1 + p.diag_shift;  // causal: the last key any row of the tile sees
    n_kv = !p.causal ? n_kv_total : last_key < 0 ? 0 : min(last_key / C::BN + 1, n_kv_total);
  }
  if (!DECODE && n_kv == 0) {
    // causal with a negative shift: no row of the tile sees a key
    const int row = q0 + threadIdx.x;
    if (threadIdx.x < C::BM && row < p.N) {
      uint4* dst = reinterpret_cast<uint4*>(p.o + (static_cast<size_t>(bh) * p.N + row) * HD);
#pragma unroll
      for (int i = 0; i < HD / 8; ++i) dst[i] = make_uint4(0u, 0u, 0u, 0u);
      p.lse[static_cast<size_t>(bh) * p.N + row] = -INFINITY;
    }
    return;
  }

  WaitCtl wc{&abort_flag, p.timeout_ns};

  if (threadIdx.x == 0) {
    abort_flag = 0;
    mbar_init(smem_u32(&bar_q), 1);
    for (int s = 0; s < ST; ++s) {
      mbar_init(smem_u32(&bar_kfull[s]), 1);
      mbar_init(smem_u32(&bar_kempty[s]), 1);
      mbar_init(smem_u32(&bar_vfull[s]), 1);
      mbar_init(smem_u32(&bar_vempty[s]), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(smem_u32(&bar_sfull[s]), 1);
      mbar_init(smem_u32(&bar_pfull[s]), 128);
    }
    mbar_init(smem_u32(&bar_odone), 1);
    mbar_init(smem_u32(&bar_drain), 1);
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
      prefetch_tmap(&tm_q);
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_v);
      mbar_arrive_expect_tx(smem_u32(&bar_q), C::Q_BYTES);
      for (int c = 0; c < KCH; ++c)
        tma_load_3d(sQ + c * (C::BM * 128), &tm_q, smem_u32(&bar_q), c * 64, q0, DECODE ? 0 : bh);
      int k_issued = 0, v_issued = 0;
      for (int j = 0; j < n_kv; ++j) {
        const int s = j % ST;
        const uint32_t ph = (j / ST) & 1;
        if (!mbar_wait(smem_u32(&bar_kempty[s]), ph ^ 1, wc)) break;
        mbar_arrive_expect_tx(smem_u32(&bar_kfull[s]), C::KV_BYTES);
        for (int c = 0; c < KCH; ++c)
          tma_load_3d(sK + s * C::KV_BYTES + c * (C::BN * 128), &tm_k, smem_u32(&bar_kfull[s]), c * 64,
                      (j0 + j) * C::BN, bh_kv);
        k_issued = j + 1;
        if (!mbar_wait(smem_u32(&bar_vempty[s]), ph ^ 1, wc)) break;
        mbar_arrive_expect_tx(smem_u32(&bar_vfull[s]), C::KV_BYTES);
        for (int c = 0; c < KCH; ++c)
          tma_load_3d(sV + s * C::KV_BYTES + c * (C::BN * 128), &tm_v, smem_u32(&bar_vfull[s]), c * 64,
                      (j0 + j) * C::BN, bh_kv);
        v_issued = j + 1;
      }
      // leave no copy in flight into shared memory
      (void)mbar_wait_drain(smem_u32(&bar_q), 0, p.timeout_ns);
      for (int j = max(0, k_issued - ST); j < k_issued; ++j)
        (void)mbar_wait_drain(smem_u32(&bar_kfull[j % ST]), (j / ST) & 1, p.timeout_ns);
      for (int j = max(0, v_issued - ST); j < v_issued; ++j)
        (void)mbar_wait_drain(smem_u32(&bar_vfull[j % ST]), (j / ST) & 1, p.timeout_ns);
    }
  } else if (warp == 5) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(128, 128, false, false);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(128, HD, false, true);
      bool ok = mbar_wait(smem_u32(&bar_q), 0, wc);
      for (int j = 0; ok && j <= n_kv; ++j) {
        if (j < n_kv) {
          const int s = j % ST;
          if (!mbar_wait(smem_u32(&bar_kfull[s]), (j / ST) & 1, wc)) break;
          tc_fence_after();
          const uint32_t d_s = tmem + (j & 1) * 128;
          const uint32_t kbase = sK + s * C::KV_BYTES;
#pragma unroll
          for (int kk = 0; kk < HD / 16; ++kk) {
            const uint32_t off = (kk >> 2) * (128 * 128) + (kk & 3) * 32;
            mma_bf16_ss(d_s, sdesc_sw128(sQ + off, 16, 1024), sdesc_sw128(kbase + off, 16, 1024), idesc_qk,
                        kk > 0);
          }
          mma_commit(smem_u32(&bar_kempty[s]));
          mma_commit(smem_u32(&bar_sfull[j & 1]));
        }
        if (j > 0) {
          const int jj = j - 1;
          const int s = jj % ST;
          if (!mbar_wait(smem_u32(&bar_pfull[jj & 1]), (jj >> 1) & 1, wc)) break;
          if (!mbar_wait(smem_u32(&bar_vfull[s]), (jj / ST) & 1, wc)) break;
          tc_fence_after();
          const uint32_t p_tmem = tmem + (jj & 1) * 128;
          const uint32_t vbase = sV + s * C::KV_BYTES;
#pragma unroll
          for (int kk = 0; kk < C::BN / 16; ++kk) {
            mma_bf16_ts(tmem + C::TMEM_O, p_tmem + kk * 8, sdesc_sw128(vbase + kk * 2048, C::BN * 128, 1024),
                        idesc_pv, (jj > 0 || kk > 0));
          }
          mma_commit(smem_u32(&bar_vempty[s]));
          mma_commit(smem_u32(&bar_odone));
        }
      }
      // no MMA may be in flight when tensor memory is released
      mma_commit(smem_u32(&bar_drain));
      (void)mbar_wait_drain(smem_u32(&bar_drain), 0, p.timeout_ns);
    }
  } else {
    // ------------------------------------------------------------- softmax
    const int row = q0 + threadIdx.x;                 // this thread's query
    const uint32_t lane_base = (warp * 32u) << 16;    // TMEM lane field
    // DECODE: the row's query sits at key position Nk - Nq + (r mod Nq); the
    // causal limit of every row is at least Nk - Nq + 1 keys
    const int dec_lim = !p.causal ? p.N : p.N - p.Nq + (DECODE ? static_cast<int>(threadIdx.x) % p.Nq : 0) + 1;
    const int dec_first = !p.causal ? p.N : p.N - p.Nq + 1;
    float m_ref = -INFINITY;
    float l = 0.f;
    bool ok = true;
    for (int j = 0; j < n_kv; ++j) {
      const int slot = j & 1;
      if (!warp_wait(smem_u32(&bar_sfull[slot]), (j >> 1) & 1, wc)) { ok = false; break; }
      tc_fence_after();
      const uint32_t s_addr = tmem + lane_base + slot * 128;
      float s[128];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t r[32];
        tmem_ld32(s_addr + c * 32, r);
#pragma unroll
        for (int i = 0; i < 32; ++i) s[c * 32 + i] = __uint_as_float(r[i]);
      }
      const int key0 = (j0 + j) * C::BN;
      const bool diag = DECODE ? key0 + C::BN > dec_first : p.causal && (key0 + C::BN > q0 + p.diag_shift);
      if (diag || key0 + C::BN > p.N) {
        // keys [key0, key0 + lim) visible
        const int lim = (DECODE ? dec_lim : min(p.causal ? row + p.diag_shift + 1 : p.N, p.N)) - key0;
#pragma unroll
        for (int c = 0; c < 128; ++c)
          if (c >= lim) s[c] = -INFINITY;
      }
      float mx = s[0];
#pragma unroll
      for (int c = 1; c < 128; ++c) mx = fmaxf(mx, s[c]);
      mx *= p.scale_log2;
      if (j == 0) {
        m_ref = mx;
      } else {
        const bool need = mx > m_ref + C::RESCALE_THRESHOLD;
        if (__any_sync(0xffffffffu, need)) {
          const float m_new = fmaxf(m_ref, mx);
          const float alpha = m_new == -INFINITY ? 1.f : ex2_approx(m_ref - m_new);
          // o was last written by P_{j-1} V_{j-1}; wait for it, then rescale.
          if (!warp_wait(smem_u32(&bar_odone), (j - 1) & 1, wc)) { ok = false; break; }
          tc_fence_after();
#pragma unroll
          for (int c = 0; c < HD / 32; ++c) {
            uint32_t r[32];
            const uint32_t o_addr = tmem + lane_base + C::TMEM_O + c * 32;
            tmem_ld32(o_addr, r);
#pragma unroll
            for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
            tmem_st32(o_addr, r);
          }
          l *= alpha;
          m_ref = m_new;
        }
      }
      const float neg_m = m_ref == -INFINITY ? 0.f : -m_ref;  // a row that sees no key: every p = 0
      float sum = 0.f;
      uint32_t pk[64];
#pragma unroll
      for (int c = 0; c < 64; ++c) {
        const float p0 = ex2_approx(fmaf(s[2 * c], p.scale_log2, neg_m));
        const float p1 = ex2_approx(fmaf(s[2 * c + 1], p.scale_log2, neg_m));
        sum += p0 + p1;
        pk[c] = pack_bf16x2(p0, p1);
      }
      l += sum;
      {
        uint32_t r0[32], r1[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) { r0[i] = pk[i]; r1[i] = pk[32 + i]; }
        tmem_st32(s_addr, r0);
        tmem_st32(s_addr + 32, r1);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(smem_u32(&bar_pfull[slot]));
    }
    if (ok && warp_wait(smem_u32(&bar_odone), (n_kv - 1) & 1, wc)) {
      tc_fence_after();
      const float inv_l = l > 0.f ? 1.f / l : 0.f;  // l = 0: the row saw no key
      const bool live = DECODE ? static_cast<int>(threadIdx.x) < p.R : row < p.N;
      const size_t o_row = DECODE ? out_base + (live ? threadIdx.x : 0) : static_cast<size_t>(bh) * p.N + (live ? row : 0);
      __nv_bfloat16* orow = p.o + o_row * HD;
#pragma unroll
      for (int c = 0; c < HD / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(tmem + lane_base + C::TMEM_O + c * 32, r);  // whole warp, converged
        uint4 w[4];
        uint32_t* wp = reinterpret_cast<uint32_t*>(w);
#pragma unroll
        for (int i = 0; i < 16; ++i)
          wp[i] = pack_bf16x2(__uint_as_float(r[2 * i]) * inv_l, __uint_as_float(r[2 * i + 1]) * inv_l);
        if (live) {
          uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
          for (int i = 0; i < 4; ++i) dst[i] = w[i];
        }
      }
      if (live) p.lse[o_row] = l > 0.f ? (m_ref + __log2f(l)) * 0.69314718055994530942f : -INFINITY;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace fa
