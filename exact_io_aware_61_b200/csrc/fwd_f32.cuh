// fwd_f32.cuh -- exact-attention forward in float32 on the CUDA cores.
//
// The same tiled pass and online-softmax recurrence as the bf16 kernel
// (fanfani.net "FlashAttention", "A pinch of math: making the softmax work in
// pieces"), in plain fp32 FMA arithmetic: tf32 tensor cores round the inputs
// to 10 mantissa bits, too coarse for 1e-5 agreement with an fp64 result.
//
// A block of 128 threads (4 warps) owns 16 query rows of one (batch, query
// head); warp w handles rows 4w..4w+3. Keys and values stream through shared
// memory 32 at a time. For each row, lane l scores key l of the tile, the
// warp reduces max and sum with shuffles, and lane l accumulates output
// columns l, l+32, ... with the running rescale exp(m_old - m_new).
#pragma once

#include "sm100_ptx.cuh"

namespace fa {

struct FwdF32Params {
  const float* q;
  const float* k;
  const float* v;
  float* o;
  float* lse;
  int N, Hq, Hkv;
  float scale;
  int causal;
};

template <int HD>
__global__ void __launch_bounds__(128) fa_fwd_f32_kernel(const FwdF32Params p) {
  constexpr int ROWS = 16, KT = 32, CPL = HD / 32;  // columns per lane
  extern __shared__ float sm_f32[];
  float* sQ = sm_f32;                // [ROWS][HD]
  float* sK = sQ + ROWS * HD;        // [KT][HD + 1]
  float* sV = sK + KT * (HD + 1);    // [KT][HD]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int blocks_per_head = (p.N + ROWS - 1) / ROWS;  // 1-D grid, head-major
  const size_t bh = blockIdx.x / blocks_per_head;
  const int r0 = static_cast<int>(blockIdx.x % blocks_per_head) * ROWS;
  const int b = static_cast<int>(bh / p.Hq);
  const int hq = static_cast<int>(bh % p.Hq);
  const size_t bh_kv = static_cast<size_t>(b) * p.Hkv + hq / (p.Hq / p.Hkv);
  const float* qg = p.q + bh * p.N * HD;
  const float* kg = p.k + bh_kv * p.N * HD;
  const float* vg = p.v + bh_kv * p.N * HD;

  for (int i = threadIdx.x; i < ROWS * HD; i += 128) {
    const int r = i / HD, c = i % HD;
    sQ[i] = (r0 + r < p.N) ? qg[static_cast<size_t>(r0 + r) * HD + c] : 0.f;
  }

  float m[4], l[4], acc[4][CPL];
#pragma unroll
  for (int rr = 0; rr < 4; ++rr) {
    m[rr] = -INFINITY;
    l[rr] = 0.f;
#pragma unroll
    for (int t = 0; t < CPL; ++t) acc[rr][t] = 0.f;
  }

  const int key_end = p.causal ? min(p.N, r0 + ROWS) : p.N;
  for (int kt0 = 0; kt0 < key_end; kt0 += KT) {
    __syncthreads();
    for (int i = threadIdx.x; i < KT * HD; i += 128) {
      const int r = i / HD, c = i % HD;
      const bool in = kt0 + r < p.N;
      sK[r * (HD + 1) + c] = in ? kg[static_cast<size_t>(kt0 + r) * HD + c] : 0.f;
      sV[r * HD + c] = in ? vg[static_cast<size_t>(kt0 + r) * HD + c] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int rr = 0; rr < 4; ++rr) {
      const int lr = warp * 4 + rr;
      const int row = r0 + lr;
      const int key = kt0 + lane;
      float s = 0.f;
#pragma unroll 8
      for (int c = 0; c < HD; ++c) s = fmaf(sQ[lr * HD + c], sK[lane * (HD + 1) + c], s);
      s *= p.scale;
      const bool vis = row < p.N && key < p.N && (!p.causal || key <= row);
      if (!vis) s = -INFINITY;
      float mt = s;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, off));
      const float m_new = fmaxf(m[rr], mt);
      if (m_new == -INFINITY) continue;  // nothing visible yet for this row (uniform in the warp)
      const float alpha = (m[rr] == -INFINITY) ? 0.f : expf(m[rr] - m_new);
      const float pr = vis ? expf(s - m_new) : 0.f;
      float ps = pr;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, off);
      l[rr] = alpha * l[rr] + ps;
      float add[CPL];
#pragma unroll
      for (int t = 0; t < CPL; ++t) add[t] = 0.f;
#pragma unroll 4
      for (int kk = 0; kk < KT; ++kk) {
        const float pk = __shfl_sync(0xffffffffu, pr, kk);
#pragma unroll
        for (int t = 0; t < CPL; ++t) add[t] = fmaf(pk, sV[kk * HD + lane + 32 * t], add[t]);
      }
#pragma unroll
      for (int t = 0; t < CPL; ++t) acc[rr][t] = fmaf(alpha, acc[rr][t], add[t]);
      m[rr] = m_new;
    }
  }

#pragma unroll
  for (int rr = 0; rr < 4; ++rr) {
    const int row = r0 + warp * 4 + rr;
    if (row >= p.N) continue;
    const float inv = l[rr] > 0.f ? 1.f / l[rr] : 0.f;
    float* orow = p.o + (bh * p.N + row) * HD;
#pragma unroll
    for (int t = 0; t < CPL; ++t) orow[lane + 32 * t] = acc[rr][t] * inv;
    if (lane == 0) p.lse[bh * p.N + row] = l[rr] > 0.f ? m[rr] + logf(l[rr]) : -INFINITY;
  }
}

template <int HD>
constexpr int fwd_f32_smem_bytes() {
  return static_cast<int>(sizeof(float)) * (16 * HD + 32 * (HD + 1) + 32 * HD);
}

}  // namespace fa
