// Merge of normalised partial attention outputs over disjoint key sets.
//
// Part p holds, for every query row, the output O_p of the softmax over its
// own keys and that softmax's log-sum-exp LSE_p. With M = max_p LSE_p the
// merged result is
//   L = sum_p exp(LSE_p - M),   O = sum_p exp(LSE_p - M) O_p / L,
//   LSE = M + ln L,
// the rescale rule that carries the running (m, l, o) state from one key block
// to the next (fanfani.net, "FlashAttention", section "A pinch of math: making
// the softmax work in pieces"), applied to states whose o is already divided
// by l: (O_p, LSE_p) is the state m = LSE_p, l = 1, o = O_p. A part with
// LSE_p = -inf saw no key and adds nothing; a row whose parts all have
// -inf gets O = 0, LSE = -inf.
//
// Memory-bound: each row reads parts x (2 d + 4) bytes and writes 2 d + 4.
// A row is handled by d / 8 consecutive threads, each owning 8 columns
// (one 16-byte load per part); the LSE values of a row are read by all of
// its threads from the same addresses (one transaction per part).
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "sm100_ptx.cuh"

namespace fa {

struct MergeCfg {
  static constexpr int THREADS = 256;
  static constexpr int MIN_BLOCKS = 8;  // 2048 resident threads per SM (32 registers each)
};

// Read-only global loads kept in program order (volatile), so that a batch of
// them is in flight before the first is used.
FA_DEV uint4 ld_nc_v4(const void* ptr) {
  uint4 r;
  asm volatile("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(ptr));
  return r;
}

FA_DEV float ld_nc_f32(const float* ptr) {
  float r;
  asm volatile("ld.global.nc.f32 %0, [%1];" : "=f"(r) : "l"(ptr));
  return r;
}

// UNROLL: parts whose loads are in flight together (4 or 8, the host picks
// the smaller when it covers every part)
template <int HD, int UNROLL>
__global__ void __launch_bounds__(MergeCfg::THREADS, MergeCfg::MIN_BLOCKS)
    fa_merge_partials_kernel(const __nv_bfloat16* __restrict__ o_parts, const float* __restrict__ lse_parts,
                             int n_parts, long long rows, __nv_bfloat16* __restrict__ o, float* __restrict__ lse) {
  constexpr int TPR = HD / 8;  // threads per row
  constexpr float kLog2e = 1.4426950408889634f;
  constexpr float kLn2 = 0.69314718055994530942f;
  const long long first = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) / TPR;
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x / TPR;
  const int c8 = (threadIdx.x % TPR) * 8;
  for (long long row = first; row < rows; row += stride) {
    // pass 1: the row's largest LSE (all loads independent, the row's threads
    // read the same addresses)
    float M = -INFINITY;
    for (int q0 = 0; q0 < n_parts; q0 += UNROLL) {
      float lq[UNROLL];
#pragma unroll
      for (int u = 0; u < UNROLL; ++u)
        lq[u] = ld_nc_f32(lse_parts + static_cast<long long>(min(q0 + u, n_parts - 1)) * rows + row);
#pragma unroll
      for (int u = 0; u < UNROLL; ++u) asm volatile("" : "+f"(lq[u]));
#pragma unroll
      for (int u = 0; u < UNROLL; ++u) M = fmaxf(M, lq[u]);  // a repeated last part changes no max
    }
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.f;
    float L = 0.f;
    if (M != -INFINITY) {
      const float m2 = M * kLog2e;
      // pass 2: UNROLL parts at a time, every load issued before any is used;
      // past the last part the index is clamped (a valid address) and the
      // weight is 0, and a part with LSE = -inf weighs 0 whatever its O holds
      for (int q0 = 0; q0 < n_parts; q0 += UNROLL) {
        float lq[UNROLL];
        uint4 x[UNROLL];
#pragma unroll
        for (int u = 0; u < UNROLL; ++u) {
          const long long idx = static_cast<long long>(min(q0 + u, n_parts - 1)) * rows + row;
          lq[u] = ld_nc_f32(lse_parts + idx);
          x[u] = ld_nc_v4(o_parts + idx * HD + c8);
        }
        // every use below depends on these (empty, ordered) statements, which
        // come after the last load: the batch is issued before it is waited on
#pragma unroll
        for (int u = 0; u < UNROLL; ++u)
          asm volatile("" : "+r"(x[u].x), "+r"(x[u].y), "+r"(x[u].z), "+r"(x[u].w), "+f"(lq[u]));
#pragma unroll
        for (int u = 0; u < UNROLL; ++u) {
          const bool use = q0 + u < n_parts && lq[u] != -INFINITY;
          const float w = use ? ex2_approx(fmaf(lq[u], kLog2e, -m2)) : 0.f;
          L += w;
          const uint32_t xs[4] = {x[u].x, x[u].y, x[u].z, x[u].w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&xs[i]));
            if (!use) f = make_float2(0.f, 0.f);
            acc[2 * i] = fmaf(w, f.x, acc[2 * i]);
            acc[2 * i + 1] = fmaf(w, f.y, acc[2 * i + 1]);
          }
        }
      }
    }
    const float inv = L > 0.f ? 1.f / L : 0.f;
    uint32_t out[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) out[i] = pack_bf16x2(acc[2 * i] * inv, acc[2 * i + 1] * inv);
    *reinterpret_cast<uint4*>(o + row * HD + c8) = make_uint4(out[0], out[1], out[2], out[3]);
    if (c8 == 0) lse[row] = L > 0.f ? M + __log2f(L) * kLn2 : -INFINITY;
  }
}

}  // namespace fa
