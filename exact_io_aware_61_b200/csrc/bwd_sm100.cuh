// bwd_sm100.cuh -- the memory-bound stages around the backward main kernel
// (bwd2_sm100.cuh):
//   fa_bwd_prep_kernel   D = rowsum(dO * O) and LSE * log2(e) into
//                        128-row-padded workspace rows (+inf / 0 in the
//                        padding, so padded queries get zero weight), and
//                        zeroing of the f32 dQ accumulator
//   fa_bwd_dq_kernel     f32 accumulator -> bf16 (dQ; dK, dV when the
//                        backward splits a group's heads over CTAs)
//   fa_zero_f32_kernel   zero an f32 accumulator
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

// First workspace row of sequence s in the variable-length backward:
// 4 ceil(cu_q[s] / 4) + 4 s. Multiples of 4 (16 bytes of f32), and each
// sequence's rows end before the next one's start (the gap covers the round
// up); a head's row holds ws_seq_base(total_q, batch) + 128 floats, so the
// last sequence's 128-row tiles stay inside it.
FA_DEV int ws_seq_base(int cu_q_s, int s) { return ((cu_q_s + 3) & ~3) + 4 * s; }

struct BwdPrepVarlenParams {
  const __nv_bfloat16* o;   // [total_q][Hq][d]
  const __nv_bfloat16* dO;
  const float* lse;         // [total_q][Hq]
  float* ws_delta;          // [Hq][Npad]
  float* ws_lse2;           // [Hq][Npad]
  float* dq_acc;            // [total_q][Hq][d]
  const int* cu_q;
  int batch, Hq, Npad, total_q;
};

// Variable-length preprocess: every workspace row of every head is written,
// a row inside a sequence with D and LSE * log2(e) (and its dQ accumulator
// row zeroed), a row of the padding between sequences with 0 and +inf. The
// sequence of a row is found by bisection over the (monotone) sequence bases.
// 8 threads per row, 32 rows per block; grid (Npad / 32) * Hq.
template <int HD>
__global__ void __launch_bounds__(256) fa_bwd_prep_varlen_kernel(const BwdPrepVarlenParams p) {
  constexpr int PER = HD / 8;
  const int blocks_per_head = p.Npad / 32;
  const int h = static_cast<int>(blockIdx.x) / blocks_per_head;
  const int sub = threadIdx.x & 7;
  const int w = (static_cast<int>(blockIdx.x) - h * blocks_per_head) * 32 + (threadIdx.x >> 3);
  // largest s with ws_seq_base(cu_q[s], s) <= w (base of sequence 0 is 0)
  int lo = 0, hi = p.batch - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (ws_seq_base(__ldg(p.cu_q + mid), mid) <= w) lo = mid;
    else hi = mid - 1;
  }
  const int tok0 = __ldg(p.cu_q + lo);
  const int i = w - ws_seq_base(tok0, lo);
  // (offsets that break the sizes are reported by the main kernel; here they
  // only must not lead outside the tensors)
  const bool live = i < __ldg(p.cu_q + lo + 1) - tok0 && tok0 >= 0 && tok0 + i < p.total_q;
  const size_t row = static_cast<size_t>(tok0 + (live ? i : 0)) * p.Hq + h;
  float acc = 0.f;
  if (live) {
    const size_t off = row * HD + sub * PER;
    const uint4* o4 = reinterpret_cast<const uint4*>(p.o + off);
    const uint4* d4 = reinterpret_cast<const uint4*>(p.dO + off);
    float4* z4 = reinterpret_cast<float4*>(p.dq_acc + off);
#pragma unroll
    for (int j = 0; j < PER / 8; ++j) {
      const uint4 a = o4[j], g = d4[j];
      const uint32_t av[4] = {a.x, a.y, a.z, a.w};
      const uint32_t gv[4] = {g.x, g.y, g.z, g.w};
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        acc = fmaf(bf16_lo(av[t]), bf16_lo(gv[t]), acc);
        acc = fmaf(bf16_hi(av[t]), bf16_hi(gv[t]), acc);
      }
      z4[2 * j] = make_float4(0.f, 0.f, 0.f, 0.f);
      z4[2 * j + 1] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }
  acc += __shfl_xor_sync(0xffffffffu, acc, 1);
  acc += __shfl_xor_sync(0xffffffffu, acc, 2);
  acc += __shfl_xor_sync(0xffffffffu, acc, 4);
  if (sub == 0) {
    const size_t wi = static_cast<size_t>(h) * p.Npad + w;
    p.ws_delta[wi] = live ? acc : 0.f;
    p.ws_lse2[wi] = live ? p.lse[row] * 1.4426950408889634f : INFINITY;
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

// Grid-stride zeroing of n4 float4s.
__global__ void __launch_bounds__(256) fa_zero_f32_kernel(float* __restrict__ p, size_t n4) {
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n4;
       i += static_cast<size_t>(gridDim.x) * blockDim.x)
    reinterpret_cast<float4*>(p)[i] = make_float4(0.f, 0.f, 0.f, 0.f);
}

}  // namespace fa
