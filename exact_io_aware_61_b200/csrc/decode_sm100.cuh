// decode_sm100.cuh -- attention of a few new queries against a long KV cache
// (bf16, head dimension 64, 128 or 256), split over the keys.
//
// Nq queries sit at the last Nq of Nk key positions (query i at Nk - Nq + i;
// with the causal mask it sees keys up to there). The work is memory-bound:
// every key and value is read once and used by only the g * Nq query rows of
// its KV head (g = Hq / Hkv), a handful of FLOPs per byte, so the kernel keeps
// the HBM stream busy rather than the tensor cores:
//   * one CTA per (batch, KV head, key split) holds all R = g * Nq query rows
//     of the group (R <= 64) in shared memory, so K and V cross HBM once;
//   * 64-key K and V tiles arrive by TMA (128-byte swizzle, double-buffered);
//   * scores and P V are f32 FMAs on the CUDA cores; the online softmax of
//     each row runs over the split's tiles (fanfani.net "FlashAttention",
//     "A pinch of math: making the softmax work in pieces");
//   * each split writes its state (m, l, unnormalised o) per row, and a second
//     kernel merges the splits with the same rescale rule and writes O, LSE.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include "sm100_ptx.cuh"

namespace fa {

template <int HD, int RB>
struct DecodeCfg {
  // RB: query rows per CTA rounded up to 4, 8, 16, 32 or 64 (loops run exactly
  // that deep; no work is issued for rows that cannot exist)
  static constexpr int BK = 64;        // keys per tile
  static constexpr int THREADS = 256;  // 8 warps
  static constexpr int STAGES = 2;
  static constexpr int TILE_BYTES = BK * HD * 2;  // one K or V tile
  static constexpr int Q_BYTES = RB * HD * 4;
  static constexpr int P_BYTES = RB * BK * 4;
  static constexpr int SMEM_BYTES = 1024 + 2 * STAGES * TILE_BYTES + Q_BYTES + P_BYTES + RB * 4;
  // scores: thread = key (64) x row group (4); rows rg, rg + 4, ...
  static constexpr int SROWS = RB / 4;
  // P V: thread = (column chunk of 8, row, key subset); KS key subsets of a
  // tile when there are more threads than (row, chunk) pairs, else PROWS rows
  // per thread
  static constexpr int CHUNKS = HD / 8;
  static constexpr int PAIRS = RB * CHUNKS;
  static constexpr int KS = PAIRS >= THREADS ? 1 : THREADS / PAIRS;
  static constexpr int PROWS = PAIRS >= THREADS ? PAIRS / THREADS : 1;
  static constexpr int ROW_STRIDE = THREADS / CHUNKS;  // when PROWS > 1
  // two CTAs per SM (128 registers) unless the row bucket needs more registers
  static constexpr int MIN_BLOCKS = RB >= 64 ? 1 : 2;
  static_assert(RB % 4 == 0 && RB <= 64, "row bucket");
  static_assert(KS == 1 || PROWS == 1, "either key subsets or several rows per thread");
  static_assert(BK % KS == 0, "key subsets divide the tile");
};

struct DecodeParams {
  const __nv_bfloat16* q;  // [B][Hq][Nq][d]
  float* part_o;           // [B*Hkv][S][R][d]   unnormalised o of each split
  float* part_ml;          // [B*Hkv][S][R][2]   (m in log2 units, l)
  int Hq, Hkv, Nq, Nk, R, S, L;  // R = g*Nq rows; S splits of L keys (L a multiple of 64)
  float scale_log2;
  int causal;
  unsigned long long timeout_ns;
};

// 16-byte chunk `c` (8 bf16 along d) of key row `j` of a tile loaded by TMA as
// 64-column boxes of 64 rows x 128 bytes with the 128-byte swizzle.
template <int HD>
FA_DEV uint32_t swz_chunk(uint32_t tile, int j, int c) {
  return tile + (c >> 3) * (64 * 128) + j * 128 + (((c & 7) ^ (j & 7)) << 4);
}

FA_DEV void bf16x8_to_f32(const uint4 w, float (&f)[8]) {
  const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = bf16_lo(u[i]);
    f[2 * i + 1] = bf16_hi(u[i]);
  }
}

template <int HD, int RB>
__global__ void __launch_bounds__(256, (DecodeCfg<HD, RB>::MIN_BLOCKS))
    fa_decode_split_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                           const DecodeParams p) {
  using C = DecodeCfg<HD, RB>;
  constexpr int BK = C::BK, ST = C::STAGES, KS = C::KS, PROWS = C::PROWS;

  extern __shared__ uint8_t smem_raw[];
  __shared__ uint64_t bar_full[ST];
  __shared__ int abort_flag;

  const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
  uint8_t* const gbase = smem_raw + (base - smem_u32(smem_raw));
  const uint32_t sK = base;                        // stage s at sK + s * TILE
  const uint32_t sV = sK + ST * C::TILE_BYTES;
  float* const sQ = reinterpret_cast<float*>(gbase + 2 * ST * C::TILE_BYTES);  // [RB][HD]
  float* const sP = sQ + RB * HD;                                            // [RB][BK]
  float* const sAlpha = sP + RB * BK;                                        // [RB]

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int bhkv = blockIdx.y, split = blockIdx.x;
  const int b = bhkv / p.Hkv, hkv = bhkv - b * p.Hkv;
  const int g = p.Hq / p.Hkv;
  const int R = p.R;
  const int k_begin = split * p.L;
  const int k_end = min(k_begin + p.L, p.Nk);
  const int n_tiles = (k_end - k_begin + BK - 1) / BK;
  WaitCtl wc{&abort_flag, p.timeout_ns};

  if (tid == 0) {
    abort_flag = 0;
    for (int s = 0; s < ST; ++s) mbar_init(smem_u32(&bar_full[s]), 1);
    fence_mbar_init();
  }
  // query rows r = hh * Nq + i (head hkv * g + hh, query i) -> f32 in shared
  // memory; rows R .. RB-1 are zero
  for (int e = tid; e < RB * (HD / 8); e += C::THREADS) {
    const int r = e / (HD / 8), c = e - r * (HD / 8);
    float f[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    if (r < R) {
      const int hh = r / p.Nq, i = r - hh * p.Nq;
      const size_t row = (static_cast<size_t>(b) * p.Hq + hkv * g + hh) * p.Nq + i;
      bf16x8_to_f32(reinterpret_cast<const uint4*>(p.q + row * HD)[c], f);
    }
    float4* dst = reinterpret_cast<float4*>(sQ + r * HD + 8 * c);
    dst[0] = make_float4(f[0], f[1], f[2], f[3]);
    dst[1] = make_float4(f[4], f[5], f[6], f[7]);
  }
  __syncthreads();
  auto issue = [&](int t) {
    const int s = t % ST;
    const uint32_t bar = smem_u32(&bar_full[s]);
    mbar_arrive_expect_tx(bar, 2 * C::TILE_BYTES);
    for (int c = 0; c < HD / 64; ++c) {
      tma_load_3d(sK + s * C::TILE_BYTES + c * (64 * 128), &tm_k, bar, c * 64, k_begin + t * BK, bhkv);
      tma_load_3d(sV + s * C::TILE_BYTES + c * (64 * 128), &tm_v, bar, c * 64, k_begin + t * BK, bhkv);
    }
  };
  int issued = 0;  // tiles whose loads thread 0 has issued
  if (tid == 0) {
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
    for (int t = 0; t < min(ST, n_tiles); ++t) issue(t);
    issued = min(ST, n_tiles);
  }

  // score phase: thread = key (warp & 1) * 32 + lane, rows rg + 4 k
  const int key = (warp & 1) * 32 + lane;
  const int rg = warp >> 1;
  // softmax phase: warp w owns rows w, w + 8, ... (state replicated in its lanes)
  constexpr int MROWS = (RB + 7) / 8;
  float m_run[MROWS], l_run[MROWS];
#pragma unroll
  for (int k = 0; k < MROWS; ++k) {
    m_run[k] = -INFINITY;
    l_run[k] = 0.f;
  }
  // P V phase: columns 8 cc .. + 7; with key subsets, row pr and keys
  // ks, ks + KS, ...; else rows pr + ROW_STRIDE k
  const int cc = tid % C::CHUNKS;
  const int pr = KS > 1 ? (tid / C::CHUNKS) % RB : tid / C::CHUNKS;
  const int ks = KS > 1 ? tid / (C::CHUNKS * RB) : 0;
  uint64_t acc[PROWS][4];  // packed f32 pairs: columns (2x, 2x + 1)
#pragma unroll
  for (int k = 0; k < PROWS; ++k)
#pragma unroll
    for (int x = 0; x < 4; ++x) acc[k][x] = 0ull;

  bool ok = true;
  for (int t = 0; t < n_tiles; ++t) {
    const int s = t % ST;
    ok = ok && mbar_wait(smem_u32(&bar_full[s]), (t / ST) & 1, wc);
    const uint32_t kt = sK + s * C::TILE_BYTES, vt = sV + s * C::TILE_BYTES;
    const int kg = k_begin + t * BK + key;  // this thread's key position
    if (ok) {
      uint64_t dot2[C::SROWS];  // packed partial dot products (even, odd columns)
#pragma unroll
      for (int k = 0; k < C::SROWS; ++k) dot2[k] = 0ull;
#pragma unroll 4
      for (int c = 0; c < HD / 8; ++c) {
        uint4 w;
        asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                     : "=r"(w.x), "=r"(w.y), "=r"(w.z), "=r"(w.w)
                     : "r"(swz_chunk<HD>(kt, key, c)));
        const uint64_t k01 = pack2(bf16_lo(w.x), bf16_hi(w.x)), k23 = pack2(bf16_lo(w.y), bf16_hi(w.y));
        const uint64_t k45 = pack2(bf16_lo(w.z), bf16_hi(w.z)), k67 = pack2(bf16_lo(w.w), bf16_hi(w.w));
#pragma unroll
        for (int k = 0; k < C::SROWS; ++k) {
          const float4* qr = reinterpret_cast<const float4*>(sQ + (rg + 4 * k) * HD + 8 * c);
          const float4 qa = qr[0], qb = qr[1];
          dot2[k] = ffma2(pack2(qa.x, qa.y), k01, dot2[k]);
          dot2[k] = ffma2(pack2(qa.z, qa.w), k23, dot2[k]);
          dot2[k] = ffma2(pack2(qb.x, qb.y), k45, dot2[k]);
          dot2[k] = ffma2(pack2(qb.z, qb.w), k67, dot2[k]);
        }
      }
#pragma unroll
      for (int k = 0; k < C::SROWS; ++k) {
        const int r = rg + 4 * k;
        const int pos = p.Nk - p.Nq + (r % p.Nq);
        const bool vis = r < R && kg < k_end && (!p.causal || kg <= pos);
        float d0, d1;
        unpack2(dot2[k], d0, d1);
        sP[r * BK + key] = vis ? (d0 + d1) * p.scale_log2 : -INFINITY;
      }
    }
    __syncthreads();
    if (ok) {
      // online softmax per row: p = 2^(s - m_new), alpha = 2^(m_old - m_new)
#pragma unroll
      for (int k = 0; k < MROWS; ++k) {
        const int r = warp + 8 * k;
        if (r < RB) {
          const float s0 = sP[r * BK + lane], s1 = sP[r * BK + 32 + lane];
          float mt = fmaxf(s0, s1);
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, o));
          const float m_new = fmaxf(m_run[k], mt);
          const float m_use = m_new == -INFINITY ? 0.f : m_new;  // a row with nothing visible yet
          const float alpha = m_run[k] == -INFINITY ? 0.f : ex2_approx(m_run[k] - m_use);
          const float p0 = ex2_approx(s0 - m_use), p1 = ex2_approx(s1 - m_use);
          sP[r * BK + lane] = p0;
          sP[r * BK + 32 + lane] = p1;
          float ps = p0 + p1;
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, o);
          l_run[k] = l_run[k] * alpha + ps;
          m_run[k] = m_new;
          if (lane == 0) sAlpha[r] = alpha;
        }
      }
    }
    __syncthreads();
    if (ok) {
      // o = alpha o + P V over this thread's keys of the tile
#pragma unroll
      for (int k = 0; k < PROWS; ++k) {
        const float a = sAlpha[pr + C::ROW_STRIDE * k * (PROWS > 1)];
        const uint64_t a2 = pack2(a, a);
#pragma unroll
        for (int x = 0; x < 4; ++x) acc[k][x] = fmul2(acc[k][x], a2);
      }
#pragma unroll 4
      for (int jj = 0; jj < BK / KS; ++jj) {
        const int j = ks + KS * jj;
        uint4 w;
        asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                     : "=r"(w.x), "=r"(w.y), "=r"(w.z), "=r"(w.w)
                     : "r"(swz_chunk<HD>(vt, j, cc)));
        const uint64_t v2[4] = {pack2(bf16_lo(w.x), bf16_hi(w.x)), pack2(bf16_lo(w.y), bf16_hi(w.y)),
                                pack2(bf16_lo(w.z), bf16_hi(w.z)), pack2(bf16_lo(w.w), bf16_hi(w.w))};
#pragma unroll
        for (int k = 0; k < PROWS; ++k) {
          const float pj = sP[(pr + C::ROW_STRIDE * k * (PROWS > 1)) * BK + j];
          const uint64_t p2 = pack2(pj, pj);
#pragma unroll
          for (int x = 0; x < 4; ++x) acc[k][x] = ffma2(p2, v2[x], acc[k][x]);
        }
      }
    }
    __syncthreads();  // stage s and the P buffer are free again
    if (tid == 0 && ok && t + ST < n_tiles) {
      issue(t + ST);
      issued = t + ST + 1;
    }
  }
  // leave no copy in flight into shared memory (the stages are reused below,
  // and a bounded wait may have given up before they were consumed)
  if (tid == 0)
    for (int t = max(0, issued - ST); t < issued; ++t)
      (void)mbar_wait_drain(smem_u32(&bar_full[t % ST]), (t / ST) & 1, p.timeout_ns);
  __syncthreads();

  // this split's state; with key subsets, their sums are added first (the
  // subsets of a row share its max and rescale factors, so their sums add)
  const size_t part = static_cast<size_t>(bhkv) * p.S + split;
  if (KS > 1) {
    float* red = reinterpret_cast<float*>(gbase);  // the K/V stages are free now
    if (ks > 0) {
      uint64_t* dst = reinterpret_cast<uint64_t*>(red + ((ks - 1) * RB * C::CHUNKS + pr * C::CHUNKS + cc) * 8);
#pragma unroll
      for (int x = 0; x < 4; ++x) dst[x] = acc[0][x];
    }
    __syncthreads();
    if (ks == 0) {
      for (int q2 = 1; q2 < KS; ++q2) {
        const uint64_t* src =
            reinterpret_cast<const uint64_t*>(red + ((q2 - 1) * RB * C::CHUNKS + pr * C::CHUNKS + cc) * 8);
#pragma unroll
        for (int x = 0; x < 4; ++x) acc[0][x] = fadd2(acc[0][x], src[x]);
      }
    }
  }
  if (ok && ks == 0) {
#pragma unroll
    for (int k = 0; k < PROWS; ++k) {
      const int r = pr + C::ROW_STRIDE * k * (PROWS > 1);
      if (r < R) {
        uint64_t* dst = reinterpret_cast<uint64_t*>(p.part_o + (part * R + r) * HD + 8 * cc);
#pragma unroll
        for (int x = 0; x < 4; ++x) dst[x] = acc[k][x];
      }
    }
  }
  if (ok && lane == 0) {
#pragma unroll
    for (int k = 0; k < MROWS; ++k) {
      const int r = warp + 8 * k;
      if (r < R) reinterpret_cast<float2*>(p.part_ml)[part * R + r] = make_float2(m_run[k], l_run[k]);
    }
  }
}

struct DecodeMergeParams {
  const float* part_o;
  const float* part_ml;
  __nv_bfloat16* o;  // [B][Hq][Nq][d]
  float* lse;        // [B][Hq][Nq]
  int Hq, Hkv, Nq, R, S, rows;  // rows = B * Hkv * R
};

// One warp per query row: M = max_s m_s, w_s = 2^(m_s - M),
// O = sum_s w_s o_s / sum_s w_s l_s, LSE = (M + log2 L) ln 2.
template <int HD>
__global__ void __launch_bounds__(256) fa_decode_merge_kernel(const DecodeMergeParams p) {
  const int row = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= p.rows) return;
  const int bhkv = row / p.R, r = row - bhkv * p.R;
  const int b = bhkv / p.Hkv, hkv = bhkv - b * p.Hkv;
  const int g = p.Hq / p.Hkv, hh = r / p.Nq, i = r - hh * p.Nq;
  const size_t out_row = (static_cast<size_t>(b) * p.Hq + hkv * g + hh) * p.Nq + i;
  const float2* ml = reinterpret_cast<const float2*>(p.part_ml);
  float M = -INFINITY;
  for (int s = lane; s < p.S; s += 32) M = fmaxf(M, ml[(static_cast<size_t>(bhkv) * p.S + s) * p.R + r].x);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  const float M_use = M == -INFINITY ? 0.f : M;
  float L = 0.f;
  float acc[HD / 32];
#pragma unroll
  for (int x = 0; x < HD / 32; ++x) acc[x] = 0.f;
  for (int s = 0; s < p.S; ++s) {
    const size_t part = static_cast<size_t>(bhkv) * p.S + s;
    const float2 st = ml[part * p.R + r];
    const float w = st.x == -INFINITY ? 0.f : ex2_approx(st.x - M_use);
    L = fmaf(w, st.y, L);
    const float* po = p.part_o + (part * p.R + r) * HD;
#pragma unroll
    for (int x = 0; x < HD / 32; ++x) acc[x] = fmaf(w, po[lane + 32 * x], acc[x]);
  }
  const float inv = L > 0.f ? 1.f / L : 0.f;
  __nv_bfloat16* orow = p.o + out_row * HD;
#pragma unroll
  for (int x = 0; x < HD / 32; ++x) orow[lane + 32 * x] = __float2bfloat16_rn(acc[x] * inv);
  if (lane == 0) p.lse[out_row] = L > 0.f ? (M + __log2f(L)) * 0.69314718055994530942f : -INFINITY;
}

}  // namespace fa
