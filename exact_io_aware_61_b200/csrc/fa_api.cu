// fa_api.cu -- the C ABI declared in include/fa.h: argument checks, TMA
// tensor maps, kernel selection and launches. One translation unit holds
// every kernel so that they share the device status word.

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <cstdint>
#include <initializer_list>
#include <mutex>
#include <utility>

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "fa.h"
#include "sm100_ptx.cuh"
#include "fwd_sm100.cuh"
#include "fwd2_sm100.cuh"
#include "fwd_f32.cuh"
#include "bwd_sm100.cuh"
#include "bwd2_sm100.cuh"
#include "bwd256_sm100.cuh"
#include "merge_sm100.cuh"

namespace {

constexpr long long kDefaultTimeoutNs = 2000000000LL;
std::atomic<long long> g_timeout_ns{kDefaultTimeoutNs};

// Waits only on a barrier nothing arrives at: the bounded wait must run out.
__global__ void fa_selftest_wait_kernel(unsigned long long timeout_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    fa::mbar_init(fa::smem_u32(&bar), 1);
    fa::fence_mbar_init();
  }
  __syncthreads();
  fa::WaitCtl wc{&abort_flag, timeout_ns};
  if (threadIdx.x == 0) (void)fa::mbar_wait(fa::smem_u32(&bar), 0, wc);
}

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

// The kernels are built for sm_100a only: CC 10.0.
int check_device(int* dev_out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return FA_ERR_CUDA;
  int major = 0, minor = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
    return FA_ERR_CUDA;
  if (major != 10 || minor != 0) return FA_ERR_UNSUPPORTED;
  *dev_out = dev;
  return FA_OK;
}

// Every configuration's dynamic shared memory fits the 227 KB (232,448 bytes)
// a block can opt into, with 1 KB left for its static barriers.
constexpr int kMaxDynamicSmem = 232448 - 1024;
static_assert(fa::Fwd2Cfg<64>::SMEM_BYTES <= kMaxDynamicSmem && fa::Fwd2Cfg<128>::SMEM_BYTES <= kMaxDynamicSmem,
              "two-tile forward shared memory");
static_assert(fa::FwdCfg<256>::SMEM_BYTES <= kMaxDynamicSmem && fa::FwdCfg<64, true>::SMEM_BYTES <= kMaxDynamicSmem &&
                  fa::FwdCfg<128, true>::SMEM_BYTES <= kMaxDynamicSmem &&
                  fa::FwdCfg<256, true>::SMEM_BYTES <= kMaxDynamicSmem,
              "one-tile forward shared memory");
static_assert(fa::Bwd2Cfg<64>::SMEM_BYTES <= kMaxDynamicSmem && fa::Bwd2Cfg<128>::SMEM_BYTES <= kMaxDynamicSmem,
              "backward shared memory");
static_assert(fa::Bwd256Cfg::SMEM_BYTES <= kMaxDynamicSmem, "d = 256 backward shared memory");

// Opt every kernel into its dynamic shared memory, once per device.
int prepare_kernels(int dev) {
  static std::mutex mu;
  static bool done[128] = {};
  if (dev < 0 || dev >= 128) return FA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(mu);
  if (done[dev]) return FA_OK;
  cudaError_t e = cudaSuccess;
  auto set = [&](const void* fn, int bytes) {
    if (e == cudaSuccess) e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  };
  set(reinterpret_cast<const void*>(&fa::fa_fwd_bf16_2tile_kernel<64>), fa::Fwd2Cfg<64>::SMEM_BYTES);
  set(reinterpret_cast<const void*>(&fa::fa_fwd_bf16_2tile_kernel<128>), fa::Fwd2Cfg<128>::SMEM_BYTES);
  set(reinterpret_cast<const void*>(&fa::fa_fwd_bf16_2tile_kernel<64, true>), fa::Fwd2Cfg<64>::SMEM_BYTES);
  set(reinterpret_cast<const void*>(&fa::fa_fwd_bf16_2tile_kernel<128, true>), fa::Fwd2Cfg<128>::SMEM_BYTES);
  set(reinterpret_cast<const void*>(&fa::fa_fwd_bf16_kernel<256>), fa::FwdCfg<256>::SMEM_BYTES);
  set(reinterpret_cast<const void*>(&fa::fa_fwd_bf16_kernel<64, true>), fa::FwdCfg<64, true>::SMEM_BYTES);
  set(reinterpret_cast<const void*>(&fa::fa_fwd_bf16_kernel<128, true>), fa::FwdCfg<128, true>::SMEM_BYTES);
  set(reinterpret_cast<const void*>(&fa::fa_fwd_f32_kernel<64>), fa::fwd_f32_smem_bytes<64>());
  set(reinterpret_cast<const void*>(&fa::fa_fwd_f32_kernel<128>), fa::fwd_f32_smem_bytes<128>());
  set(reinterpret_cast<const void*>(&fa::fa_fwd_f32_kernel<256>), fa::fwd_f32_smem_bytes<256>());
  set(reinterpret_cast<const void*>(&fa::fa_fwd_bf16_kernel<256, true>), fa::FwdCfg<256, true>::SMEM_BYTES);
  set(reinterpret_cast<const void*>(&fa::fa_bwd2_main_kernel<64>), fa::Bwd2Cfg<64>::SMEM_BYTES);
  set(reinterpret_cast<const void*>(&fa::fa_bwd2_main_kernel<128>), fa::Bwd2Cfg<128>::SMEM_BYTES);
  set(reinterpret_cast<const void*>(&fa::fa_bwd2_main_kernel<64, true>), fa::Bwd2Cfg<64>::SMEM_BYTES);
  set(reinterpret_cast<const void*>(&fa::fa_bwd2_main_kernel<128, true>), fa::Bwd2Cfg<128>::SMEM_BYTES);
  set(reinterpret_cast<const void*>(&fa::fa_bwd2_main_kernel<64, false, true>), fa::Bwd2Cfg<64>::SMEM_BYTES);
  set(reinterpret_cast<const void*>(&fa::fa_bwd2_main_kernel<128, false, true>), fa::Bwd2Cfg<128>::SMEM_BYTES);
  set(reinterpret_cast<const void*>(&fa::fa_bwd256_main_kernel), fa::Bwd256Cfg::SMEM_BYTES);
  if (e != cudaSuccess) return FA_ERR_CUDA;
  done[dev] = true;
  return FA_OK;
}

// Rank-3 tiled map over a dense [outer][rows][inner] tensor with a
// (box_inner x box_rows x 1) box and 128-byte swizzle; out-of-bounds reads
// fill zeros, out-of-bounds writes are dropped.
int make_map(CUtensorMap* map, const void* ptr, CUtensorMapDataType type, uint64_t elem_bytes, uint64_t inner,
             uint64_t rows, uint64_t outer, uint32_t box_inner, uint32_t box_rows) {
  auto encode = tensor_map_encoder();
  if (!encode) return FA_ERR_CUDA;
  const cuuint64_t dims[3] = {inner, rows, outer};
  const cuuint64_t strides[2] = {inner * elem_bytes, inner * rows * elem_bytes};
  const cuuint32_t box[3] = {box_inner, box_rows, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = encode(map, type, 3, const_cast<void*>(ptr), dims, strides, box, estr,
                            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? FA_OK : FA_ERR_CUDA;
}

// Rank-3 tiled map over a dense [d2][d1][d0] tensor with a (b0 x b1 x b2) box
// and 128-byte swizzle; out-of-bounds reads fill zeros.
int make_map3(CUtensorMap* map, const void* ptr, CUtensorMapDataType type, uint64_t elem_bytes, uint64_t d0,
              uint64_t d1, uint64_t d2, uint32_t b0, uint32_t b1, uint32_t b2) {
  auto encode = tensor_map_encoder();
  if (!encode) return FA_ERR_CUDA;
  const cuuint64_t dims[3] = {d0, d1, d2};
  const cuuint64_t strides[2] = {d0 * elem_bytes, d0 * d1 * elem_bytes};
  const cuuint32_t box[3] = {b0, b1, b2};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = encode(map, type, 3, const_cast<void*>(ptr), dims, strides, box, estr,
                            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? FA_OK : FA_ERR_CUDA;
}

bool aligned16(const void* p) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Shared shape checks. Returns FA_OK, or the error to report.
int check_shape(int B, int Hq, int Hkv, int N, int d, float scale, int causal, int dtype) {
  if (B < 0 || N < 0 || Hq < 1 || Hkv < 1 || d < 1) return FA_ERR_INVALID;
  if (Hq % Hkv != 0) return FA_ERR_INVALID;
  if (causal != 0 && causal != 1) return FA_ERR_INVALID;
  if (dtype != FA_BF16 && dtype != FA_F32) return FA_ERR_INVALID;
  if (!std::isfinite(scale)) return FA_ERR_INVALID;
  if (d != 64 && d != 128 && d != 256) return FA_ERR_UNSUPPORTED;
  // TMA coordinates and tile indices are 32-bit.
  if (static_cast<long long>(B) * Hq > INT32_MAX / 2 || N > INT32_MAX - 256) return FA_ERR_INVALID;
  return FA_OK;
}

unsigned long long timeout_now() { return static_cast<unsigned long long>(g_timeout_ns.load()); }

bool verbose() {
  static const bool v = [] {
    const char* e = std::getenv("FA_VERBOSE");
    return e != nullptr && e[0] != '\0' && e[0] != '0';
  }();
  return v;
}

// Status of the launch just made; with FA_VERBOSE set, a failure is described
// on stderr together with the kernel's resource attributes.
int launch_status(const void* kernel = nullptr) {
  const cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess) return FA_OK;
  if (verbose()) {
    std::fprintf(stderr, "fa: launch failed: %s\n", cudaGetErrorString(e));
    cudaFuncAttributes a;
    if (kernel != nullptr && cudaFuncGetAttributes(&a, kernel) == cudaSuccess)
      std::fprintf(stderr, "fa: kernel regs=%d maxThreads=%d staticSmem=%zu maxDynSmem=%d localBytes=%zu\n",
                   a.numRegs, a.maxThreadsPerBlock, a.sharedSizeBytes, a.maxDynamicSharedSizeBytes,
                   a.localSizeBytes);
  }
  return FA_ERR_CUDA;
}

template <int HD>
int make_qkv_maps(CUtensorMap* mq, CUtensorMap* mk, CUtensorMap* mv, const void* q, const void* k, const void* v,
                  int B, int Hq, int Hkv, int N) {
  int rc = make_map(mq, q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, HD, N, static_cast<uint64_t>(B) * Hq, 64, 128);
  if (rc == FA_OK)
    rc = make_map(mk, k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, HD, N, static_cast<uint64_t>(B) * Hkv, 64, 128);
  if (rc == FA_OK)
    rc = make_map(mv, v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, HD, N, static_cast<uint64_t>(B) * Hkv, 64, 128);
  return rc;
}

// d = 256: one 128-row query tile per CTA (S double-buffered in TMEM).
int launch_fwd_bf16_d256(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv,
                         int N, float scale, int causal, cudaStream_t stream, int diag_shift = 0) {
  using C = fa::FwdCfg<256>;
  CUtensorMap mq, mk, mv;
  int rc = make_qkv_maps<256>(&mq, &mk, &mv, q, k, v, B, Hq, Hkv, N);
  if (rc != FA_OK) return rc;
  fa::FwdParams p{};
  p.o = static_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  p.N = N;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.num_q_tiles = (N + C::BM - 1) / C::BM;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.causal = causal;
  p.timeout_ns = timeout_now();
  p.diag_shift = diag_shift;
  const long long blocks = static_cast<long long>(p.num_q_tiles) * B * Hq;
  if (blocks > INT32_MAX) return FA_ERR_INVALID;
  fa::fa_fwd_bf16_kernel<256><<<static_cast<unsigned>(blocks), C::THREADS, C::SMEM_BYTES, stream>>>(mq, mk, mv, p);
  return launch_status();
}

// d = 64, 128: two 128-row query tiles per CTA.
template <int HD>
int launch_fwd_bf16_2tile(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv,
                          int N, float scale, int causal, cudaStream_t stream, int diag_shift = 0) {
  using C = fa::Fwd2Cfg<HD>;
  CUtensorMap mq, mk, mv;
  int rc = make_qkv_maps<HD>(&mq, &mk, &mv, q, k, v, B, Hq, Hkv, N);
  if (rc != FA_OK) return rc;
  fa::Fwd2Params p{};
  p.diag_shift = diag_shift;
  p.o = static_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  p.N = N;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.BH = B * Hq;
  p.num_pairs = (N + 2 * C::BM - 1) / (2 * C::BM);
  p.scale_log2 = scale * 1.4426950408889634f;
  p.causal = causal;
  p.timeout_ns = timeout_now();
  const long long blocks = static_cast<long long>(p.num_pairs) * B * Hq;
  if (blocks > INT32_MAX) return FA_ERR_INVALID;
  // The kernel redistributes registers between its warpgroups (setmaxnreg);
  // the split adds up to exactly LAUNCH_REGS per thread, so refuse to launch
  // a build whose register count differs rather than risk a wait that never
  // ends.
  cudaFuncAttributes attr;
  if (cudaFuncGetAttributes(&attr, reinterpret_cast<const void*>(&fa::fa_fwd_bf16_2tile_kernel<HD>)) != cudaSuccess)
    return FA_ERR_CUDA;
  if (attr.numRegs != C::LAUNCH_REGS) {
    if (verbose()) std::fprintf(stderr, "fa: 2-tile forward built with %d registers, expected %d\n", attr.numRegs,
                                C::LAUNCH_REGS);
    return FA_ERR_UNSUPPORTED;
  }
  fa::fa_fwd_bf16_2tile_kernel<HD><<<static_cast<unsigned>(blocks), C::THREADS, C::SMEM_BYTES, stream>>>(mq, mk, mv,
                                                                                                          p);
  return launch_status(reinterpret_cast<const void*>(&fa::fa_fwd_bf16_2tile_kernel<HD>));
}

// Packed variable-length batch, d = 64 or 128: grid = tile pairs of the
// longest sequence x sequences x heads.
template <int HD>
int launch_fwd_varlen(const void* q, const void* k, const void* v, void* o, float* lse, const int* cu_q,
                      const int* cu_k, int batch, int max_seqlen_q, int total_q, int total_k, int Hq, int Hkv,
                      float scale, int causal, cudaStream_t stream) {
  using C = fa::Fwd2Cfg<HD>;
  CUtensorMap mq, mk, mv;
  int rc = make_map3(&mq, q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, HD, Hq, total_q, 64, 1, 128);
  if (rc == FA_OK) rc = make_map3(&mk, k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, HD, Hkv, total_k, 64, 1, 128);
  if (rc == FA_OK) rc = make_map3(&mv, v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, HD, Hkv, total_k, 64, 1, 128);
  if (rc != FA_OK) return rc;
  fa::Fwd2Params p{};
  p.o = static_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  p.N = 0;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.BH = batch * Hq;
  p.num_pairs = (max_seqlen_q + 2 * C::BM - 1) / (2 * C::BM);
  p.scale_log2 = scale * 1.4426950408889634f;
  p.causal = causal;
  p.timeout_ns = timeout_now();
  p.cu_q = cu_q;
  p.cu_k = cu_k;
  p.batch = batch;
  p.total_q = total_q;
  p.total_k = total_k;
  p.max_seqlen_q = max_seqlen_q;
  const long long blocks = static_cast<long long>(p.num_pairs) * batch * Hq;
  if (blocks > INT32_MAX) return FA_ERR_INVALID;
  cudaFuncAttributes attr;
  if (cudaFuncGetAttributes(&attr, reinterpret_cast<const void*>(&fa::fa_fwd_bf16_2tile_kernel<HD, true>)) !=
      cudaSuccess)
    return FA_ERR_CUDA;
  if (attr.numRegs != C::LAUNCH_REGS) return FA_ERR_UNSUPPORTED;  // the register split needs exactly this
  fa::fa_fwd_bf16_2tile_kernel<HD, true><<<static_cast<unsigned>(blocks), C::THREADS, C::SMEM_BYTES, stream>>>(
      mq, mk, mv, p);
  return launch_status(reinterpret_cast<const void*>(&fa::fa_fwd_bf16_2tile_kernel<HD, true>));
}

// The merge's grid: grid-stride over rows with exactly the blocks that are
// resident at once (a second, partial wave would leave its blocks a full share
// of rows). Planned before any launch, since it queries the runtime.
struct MergePlan {
  int unroll;  // parts whose loads are in flight together: 4 or 8
  unsigned blocks;
};

template <int HD>
int plan_merge(int n_parts, long long rows, int num_sms, MergePlan* mp) {
  mp->unroll = n_parts <= 4 ? 4 : 8;
  const long long want = (rows * (HD / 8) + fa::MergeCfg::THREADS - 1) / fa::MergeCfg::THREADS;
  int per_sm = 0;
  const cudaError_t e =
      mp->unroll == 4
          ? cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fa::fa_merge_partials_kernel<HD, 4>,
                                                          fa::MergeCfg::THREADS, 0)
          : cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fa::fa_merge_partials_kernel<HD, 8>,
                                                          fa::MergeCfg::THREADS, 0);
  if (e != cudaSuccess || per_sm < 1) return FA_ERR_CUDA;
  mp->blocks = static_cast<unsigned>(std::min<long long>(want, static_cast<long long>(per_sm) * num_sms));
  return FA_OK;
}

template <int HD>
int launch_merge(const MergePlan& mp, const void* o_parts, const float* lse_parts, int n_parts, long long rows,
                 void* o, float* lse, cudaStream_t stream) {
  const auto* src = static_cast<const __nv_bfloat16*>(o_parts);
  auto* dst = static_cast<__nv_bfloat16*>(o);
  if (mp.unroll == 4)
    fa::fa_merge_partials_kernel<HD, 4><<<mp.blocks, fa::MergeCfg::THREADS, 0, stream>>>(src, lse_parts, n_parts,
                                                                                        rows, dst, lse);
  else
    fa::fa_merge_partials_kernel<HD, 8><<<mp.blocks, fa::MergeCfg::THREADS, 0, stream>>>(src, lse_parts, n_parts,
                                                                                        rows, dst, lse);
  return launch_status();
}

int num_sms_of(int dev, int* num_sms) {
  return cudaDeviceGetAttribute(num_sms, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

template <int HD>
int launch_fwd_f32(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv, int N,
                   float scale, int causal, cudaStream_t stream) {
  fa::FwdF32Params p;
  p.q = static_cast<const float*>(q);
  p.k = static_cast<const float*>(k);
  p.v = static_cast<const float*>(v);
  p.o = static_cast<float*>(o);
  p.lse = lse;
  p.N = N;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.scale = scale;
  p.causal = causal;
  const long long blocks = static_cast<long long>((N + 15) / 16) * B * Hq;
  if (blocks > INT32_MAX) return FA_ERR_INVALID;
  fa::fa_fwd_f32_kernel<HD><<<static_cast<unsigned>(blocks), 128, fa::fwd_f32_smem_bytes<HD>(), stream>>>(p);
  return launch_status();
}

size_t padded_rows(int N) { return (static_cast<size_t>(N) + 127) / 128 * 128; }

// How many CTAs share the query heads of one (KV head, key tile) in the
// backward: 1 unless B * Hkv * (key tiles) is below 592 (4 CTAs per SM of a
// 148-SM part), then the smallest divisor of the group size that reaches it,
// or the group size. Key tiles hold 128 keys (64 at d = 256). A pure function
// of the shape, so the workspace size does not depend on the device.
int bwd_key_tile(int d) { return d == 256 ? 64 : 128; }

int bwd_head_split(int B, int Hq, int Hkv, int N, int d = 128) {
  const int tile = bwd_key_tile(d);
  const long long ctas = static_cast<long long>(B) * Hkv * ((static_cast<long long>(N) + tile - 1) / tile);
  const int g = Hq / Hkv;
  for (int s = 1; s <= g; ++s)
    if (g % s == 0 && ctas * s >= 592) return s;
  return g;
}

// Workspace carve-up, all f32: D [B*Hq][Npad], LSE*log2(e) [B*Hq][Npad],
// dQ accumulator [B*Hq][N][d]; when the backward splits a group's heads over
// CTAs, also dK and dV accumulators [B*Hkv][N][d].
struct BwdWorkspace {
  float* delta;
  float* lse2;
  float* dq_acc;
  float* dk_acc;  // null without a split
  float* dv_acc;
};

size_t bwd_workspace_bytes(int B, int Hq, int Hkv, int N, int d) {
  const size_t rows_q = static_cast<size_t>(B) * Hq;
  const size_t kv_acc = bwd_head_split(B, Hq, Hkv, N, d) > 1 ? 2 * static_cast<size_t>(B) * Hkv * N * d : 0;
  return sizeof(float) * (2 * rows_q * padded_rows(N) + rows_q * static_cast<size_t>(N) * d + kv_acc);
}

BwdWorkspace carve(void* ws, int B, int Hq, int Hkv, int N, int d) {
  const size_t npad = padded_rows(N);
  const size_t rows_q = static_cast<size_t>(B) * Hq;
  const size_t kv_elems = static_cast<size_t>(B) * Hkv * static_cast<size_t>(N) * d;
  BwdWorkspace w;
  w.delta = static_cast<float*>(ws);
  w.lse2 = w.delta + rows_q * npad;
  w.dq_acc = w.lse2 + rows_q * npad;
  const bool split = bwd_head_split(B, Hq, Hkv, N, d) > 1;
  w.dk_acc = split ? w.dq_acc + rows_q * static_cast<size_t>(N) * d : nullptr;
  w.dv_acc = split ? w.dk_acc + kv_elems : nullptr;
  return w;
}

unsigned grid_stride_blocks(size_t n4) {
  const size_t want = (n4 + 255) / 256;
  return static_cast<unsigned>(want < 148 * 16 ? want : 148 * 16);
}

// Everything the backward's launches need, built (tensor maps encoded, grid
// sizes and the main kernel's register count checked) before the first of
// them is queued, so that every error return of a backward entry point other
// than a failed launch comes before any kernel runs.
struct BwdPlan {
  cudaStream_t stream;
  BwdWorkspace w;
  size_t kv_elems, q_elems;
  int split;
  fa::BwdPrepParams pp;
  unsigned prep_blocks;
  CUtensorMap mq, mk, mv, mdo, mdq;
  fa::Bwd2Params mp;
  fa::Bwd256Params mp256;
  unsigned main_blocks;
  __nv_bfloat16* dq;
  __nv_bfloat16* dk;
  __nv_bfloat16* dv;
  bool partial;  // the main stage is fa_bwd_partial's (shifted diagonal, dK/dV added into caller f32)
};

// stages: bit 0 prep, bit 1 main, bit 2 dQ conversion. Pointers a stage does not use may be null.
template <int HD>
int plan_bwd(BwdPlan* pl, unsigned stages, const void* q, const void* k, const void* v, const void* o,
             const float* lse, const void* dO, void* dq, void* dk, void* dv, void* ws, int B, int Hq, int Hkv,
             int N, float scale, int causal, cudaStream_t stream, int diag_shift = 0, float* dk_acc = nullptr,
             float* dv_acc = nullptr) {
  using C = fa::Bwd2Cfg<HD == 256 ? 128 : HD>;
  pl->stream = stream;
  pl->partial = dk_acc != nullptr;
  pl->w = carve(ws, B, Hq, Hkv, N, HD);
  pl->kv_elems = static_cast<size_t>(B) * Hkv * static_cast<size_t>(N) * HD;
  pl->q_elems = static_cast<size_t>(B) * Hq * static_cast<size_t>(N) * HD;
  pl->split = bwd_head_split(B, Hq, Hkv, N, HD);
  pl->dq = static_cast<__nv_bfloat16*>(dq);
  pl->dk = static_cast<__nv_bfloat16*>(dk);
  pl->dv = static_cast<__nv_bfloat16*>(dv);
  const size_t npad = padded_rows(N);
  const uint64_t rows_q = static_cast<uint64_t>(B) * Hq, rows_kv = static_cast<uint64_t>(B) * Hkv;
  if (stages & 1u) {
    fa::BwdPrepParams& pp = pl->pp;
    pp.o = static_cast<const __nv_bfloat16*>(o);
    pp.dO = static_cast<const __nv_bfloat16*>(dO);
    pp.lse = lse;
    pp.ws_delta = pl->w.delta;
    pp.ws_lse2 = pl->w.lse2;
    pp.dq_acc = pl->w.dq_acc;
    pp.N = N;
    pp.Npad = static_cast<int>(npad);
    const long long blocks = static_cast<long long>(npad / 32) * B * Hq;
    if (blocks > INT32_MAX) return FA_ERR_INVALID;
    pl->prep_blocks = static_cast<unsigned>(blocks);
  }
  if ((stages & 2u) && HD == 256) {
    // the kernel redistributes registers between warpgroups (setmaxnreg)
    // assuming exactly LAUNCH_REGS per thread at launch: refuse another count
    cudaFuncAttributes attr;
    if (cudaFuncGetAttributes(&attr, reinterpret_cast<const void*>(&fa::fa_bwd256_main_kernel)) != cudaSuccess)
      return FA_ERR_CUDA;
    if (attr.numRegs != fa::Bwd256Cfg::LAUNCH_REGS) return FA_ERR_UNSUPPORTED;
    // 64-key tiles: K and V boxes of 64 rows, Q and dO boxes of 128
    int rc = make_map(&pl->mq, q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, HD, N, rows_q, 64, 128);
    if (rc == FA_OK) rc = make_map(&pl->mk, k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, HD, N, rows_kv, 64, 64);
    if (rc == FA_OK) rc = make_map(&pl->mv, v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, HD, N, rows_kv, 64, 64);
    if (rc == FA_OK) rc = make_map(&pl->mdo, dO, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, HD, N, rows_q, 64, 128);
    if (rc != FA_OK) return rc;
    fa::Bwd256Params& mp = pl->mp256;
    mp.ws_delta = pl->w.delta;
    mp.ws_lse2 = pl->w.lse2;
    mp.dq_acc = pl->w.dq_acc;
    mp.dk = pl->dk;
    mp.dv = pl->dv;
    mp.dk_acc = pl->w.dk_acc;
    mp.dv_acc = pl->w.dv_acc;
    mp.N = N;
    mp.Npad = static_cast<int>(npad);
    mp.Hq = Hq;
    mp.Hkv = Hkv;
    mp.num_tiles = (N + fa::Bwd256Cfg::BK - 1) / fa::Bwd256Cfg::BK;
    mp.head_split = pl->split;
    mp.BHkv = B * Hkv;
    mp.scale_log2 = scale * 1.4426950408889634f;
    mp.scale = scale;
    mp.causal = causal;
    mp.timeout_ns = timeout_now();
    const long long blocks = static_cast<long long>(mp.num_tiles) * B * Hkv * pl->split;
    if (blocks > INT32_MAX) return FA_ERR_INVALID;
    pl->main_blocks = static_cast<unsigned>(blocks);
  } else if (stages & 2u) {
    // The kernel redistributes registers between warpgroups (setmaxnreg) on
    // the assumption of exactly LAUNCH_REGS per thread at launch; a build
    // with another count would wait for ever, so it is refused here.
    cudaFuncAttributes attr;
    const void* kernel = pl->partial
                             ? reinterpret_cast<const void*>(&fa::fa_bwd2_main_kernel<HD == 256 ? 128 : HD, false, true>)
                             : reinterpret_cast<const void*>(&fa::fa_bwd2_main_kernel<HD == 256 ? 128 : HD>);
    if (cudaFuncGetAttributes(&attr, kernel) != cudaSuccess) return FA_ERR_CUDA;
    if (attr.numRegs != C::LAUNCH_REGS) {
      if (verbose()) std::fprintf(stderr, "fa: backward built with %d registers, expected %d\n", attr.numRegs,
                                  C::LAUNCH_REGS);
      return FA_ERR_UNSUPPORTED;
    }
    int rc = make_map(&pl->mq, q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, HD, N, rows_q, 64, 128);
    if (rc == FA_OK) rc = make_map(&pl->mk, k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, HD, N, rows_kv, 64, 128);
    if (rc == FA_OK) rc = make_map(&pl->mv, v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, HD, N, rows_kv, 64, 128);
    if (rc == FA_OK) rc = make_map(&pl->mdo, dO, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, HD, N, rows_q, 64, 128);
    if (rc == FA_OK)
      rc = make_map(&pl->mdq, pl->w.dq_acc, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, HD, N, rows_q, 32,
                    fa::Bwd2Cfg<HD>::DQ_BOX_ROWS);
    if (rc != FA_OK) return rc;
    fa::Bwd2Params& mp = pl->mp;
    mp.ws_delta = pl->w.delta;
    mp.ws_lse2 = pl->w.lse2;
    mp.dq_acc = pl->w.dq_acc;
    mp.dk = pl->dk;
    mp.dv = pl->dv;
    mp.dk_acc = pl->w.dk_acc;
    mp.dv_acc = pl->w.dv_acc;
    mp.head_split = pl->split;
    mp.BHkv = B * Hkv;
    mp.N = N;
    mp.Npad = static_cast<int>(npad);
    mp.Hq = Hq;
    mp.Hkv = Hkv;
    mp.num_tiles = static_cast<int>(npad / 128);
    mp.scale_log2 = scale * 1.4426950408889634f;
    mp.scale = scale;
    mp.causal = causal;
    mp.timeout_ns = timeout_now();
    mp.diag_shift = diag_shift;
    if (pl->partial) {
      mp.dk_acc = dk_acc;
      mp.dv_acc = dv_acc;
    }
    const long long blocks = static_cast<long long>(mp.num_tiles) * B * Hkv * pl->split;
    if (blocks > INT32_MAX) return FA_ERR_INVALID;
    pl->main_blocks = static_cast<unsigned>(blocks);
  }
  return FA_OK;
}

template <int HD>
int launch_bwd_stages(const BwdPlan& pl, unsigned stages) {
  using C = fa::Bwd2Cfg<HD == 256 ? 128 : HD>;
  if (stages & 1u) {
    fa::fa_bwd_prep_kernel<HD><<<pl.prep_blocks, 256, 0, pl.stream>>>(pl.pp);
    if (launch_status() != FA_OK) return FA_ERR_CUDA;
  }
  if (stages & 2u) {
    if (pl.split > 1 && !pl.partial) {  // zero the f32 dK and dV accumulators (contiguous)
      fa::fa_zero_f32_kernel<<<grid_stride_blocks(pl.kv_elems / 2), 256, 0, pl.stream>>>(pl.w.dk_acc,
                                                                                        pl.kv_elems / 2);
      if (launch_status() != FA_OK) return FA_ERR_CUDA;
    }
    if constexpr (HD == 256) {
      fa::fa_bwd256_main_kernel<<<pl.main_blocks, fa::Bwd256Cfg::THREADS, fa::Bwd256Cfg::SMEM_BYTES, pl.stream>>>(
          pl.mq, pl.mk, pl.mv, pl.mdo, pl.mp256);
      if (launch_status(reinterpret_cast<const void*>(&fa::fa_bwd256_main_kernel)) != FA_OK) return FA_ERR_CUDA;
    } else if (pl.partial) {
      fa::fa_bwd2_main_kernel<HD, false, true><<<pl.main_blocks, C::THREADS, C::SMEM_BYTES, pl.stream>>>(
          pl.mq, pl.mk, pl.mv, pl.mdo, pl.mdq, pl.mp);
      if (launch_status(reinterpret_cast<const void*>(&fa::fa_bwd2_main_kernel<HD, false, true>)) != FA_OK)
        return FA_ERR_CUDA;
      return FA_OK;  // dK, dV stay in the caller's f32 accumulators
    } else {
      fa::fa_bwd2_main_kernel<HD><<<pl.main_blocks, C::THREADS, C::SMEM_BYTES, pl.stream>>>(pl.mq, pl.mk, pl.mv,
                                                                                            pl.mdo, pl.mdq, pl.mp);
      if (launch_status(reinterpret_cast<const void*>(&fa::fa_bwd2_main_kernel<HD>)) != FA_OK) return FA_ERR_CUDA;
    }
    if (pl.split > 1) {
      const size_t n4 = pl.kv_elems / 4;
      fa::fa_bwd_dq_kernel<<<grid_stride_blocks(n4), 256, 0, pl.stream>>>(pl.w.dk_acc, pl.dk, n4);
      if (launch_status() != FA_OK) return FA_ERR_CUDA;
      fa::fa_bwd_dq_kernel<<<grid_stride_blocks(n4), 256, 0, pl.stream>>>(pl.w.dv_acc, pl.dv, n4);
      if (launch_status() != FA_OK) return FA_ERR_CUDA;
    }
  }
  if (stages & 4u) {
    const size_t n4 = pl.q_elems / 4;
    fa::fa_bwd_dq_kernel<<<grid_stride_blocks(n4), 256, 0, pl.stream>>>(pl.w.dq_acc, pl.dq, n4);
    if (launch_status() != FA_OK) return FA_ERR_CUDA;
  }
  return FA_OK;
}

// ------------------------------------------------- variable-length backward
//
// Workspace, all f32: D and LSE * log2(e) [Hq][Npad] with Npad covering every
// sequence's rows from ws_seq_base(cu_q[s], s) plus a 128-row tail; the dQ
// accumulator [total_q][Hq][d]; with a head split, dK and dV accumulators
// [total_k][Hkv][d]. The split estimate counts the key tiles of total_k.
size_t bwd_varlen_npad(int batch, int total_q) {
  const size_t rows = ((static_cast<size_t>(total_q) + 3) & ~static_cast<size_t>(3)) + 4 * static_cast<size_t>(batch) + 128;
  return (rows + 127) / 128 * 128;
}

int bwd_varlen_head_split(int total_k, int Hq, int Hkv) { return bwd_head_split(1, Hq, Hkv, total_k); }

size_t bwd_varlen_workspace_bytes(int batch, int total_q, int total_k, int Hq, int Hkv, int d) {
  const size_t kv_acc =
      bwd_varlen_head_split(total_k, Hq, Hkv) > 1 ? 2 * static_cast<size_t>(total_k) * Hkv * d : 0;
  return sizeof(float) * (2 * static_cast<size_t>(Hq) * bwd_varlen_npad(batch, total_q) +
                          static_cast<size_t>(total_q) * Hq * d + kv_acc);
}

template <int HD>
int run_bwd_varlen(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dO,
                   void* dq, void* dk, void* dv, const int* cu_q, const int* cu_k, int batch, int max_seqlen_q,
                   int max_seqlen_k, int total_q, int total_k, int Hq, int Hkv, float scale, int causal, void* ws,
                   cudaStream_t stream) {
  using C = fa::Bwd2Cfg<HD>;
  // plan everything before the first launch
  cudaFuncAttributes attr;
  if (cudaFuncGetAttributes(&attr, reinterpret_cast<const void*>(&fa::fa_bwd2_main_kernel<HD, true>)) != cudaSuccess)
    return FA_ERR_CUDA;
  if (attr.numRegs != C::LAUNCH_REGS) return FA_ERR_UNSUPPORTED;  // the register split needs exactly this
  const size_t npad = bwd_varlen_npad(batch, total_q);
  const int split = bwd_varlen_head_split(total_k, Hq, Hkv);
  const size_t q_elems = static_cast<size_t>(total_q) * Hq * HD;
  const size_t kv_elems = static_cast<size_t>(total_k) * Hkv * HD;
  float* delta = static_cast<float*>(ws);
  float* lse2 = delta + static_cast<size_t>(Hq) * npad;
  float* dq_acc = lse2 + static_cast<size_t>(Hq) * npad;
  float* dk_acc = split > 1 ? dq_acc + q_elems : nullptr;
  float* dv_acc = split > 1 ? dk_acc + kv_elems : nullptr;
  CUtensorMap mq, mk, mv, mdo, mdq;
  int rc = make_map3(&mq, q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, HD, Hq, total_q, 64, 1, 128);
  if (rc == FA_OK) rc = make_map3(&mk, k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, HD, Hkv, total_k, 64, 1, 128);
  if (rc == FA_OK) rc = make_map3(&mv, v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, HD, Hkv, total_k, 64, 1, 128);
  if (rc == FA_OK) rc = make_map3(&mdo, dO, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, HD, Hq, total_q, 64, 1, 128);
  if (rc == FA_OK)
    rc = make_map3(&mdq, dq_acc, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, HD, Hq, total_q, 32, 1, fa::Bwd2Cfg<HD>::DQ_BOX_ROWS);
  if (rc != FA_OK) return rc;
  fa::BwdPrepVarlenParams pp;
  pp.o = static_cast<const __nv_bfloat16*>(o);
  pp.dO = static_cast<const __nv_bfloat16*>(dO);
  pp.lse = lse;
  pp.ws_delta = delta;
  pp.ws_lse2 = lse2;
  pp.dq_acc = dq_acc;
  pp.cu_q = cu_q;
  pp.batch = batch;
  pp.Hq = Hq;
  pp.Npad = static_cast<int>(npad);
  pp.total_q = total_q;
  const long long prep_blocks = static_cast<long long>(npad / 32) * Hq;
  fa::Bwd2Params mp{};
  mp.ws_delta = delta;
  mp.ws_lse2 = lse2;
  mp.dq_acc = dq_acc;
  mp.dk = static_cast<__nv_bfloat16*>(dk);
  mp.dv = static_cast<__nv_bfloat16*>(dv);
  mp.dk_acc = dk_acc;
  mp.dv_acc = dv_acc;
  mp.head_split = split;
  mp.BHkv = batch * Hkv;
  mp.N = 0;
  mp.Npad = static_cast<int>(npad);
  mp.Hq = Hq;
  mp.Hkv = Hkv;
  mp.num_tiles = (max_seqlen_k + 127) / 128;
  mp.scale_log2 = scale * 1.4426950408889634f;
  mp.scale = scale;
  mp.causal = causal;
  mp.timeout_ns = timeout_now();
  mp.cu_q = cu_q;
  mp.cu_k = cu_k;
  mp.batch = batch;
  mp.total_q = total_q;
  mp.total_k = total_k;
  mp.max_seqlen_q = max_seqlen_q;
  mp.max_seqlen_k = max_seqlen_k;
  const long long main_blocks = static_cast<long long>(mp.num_tiles) * batch * Hkv * split;
  if (prep_blocks > INT32_MAX || main_blocks > INT32_MAX || npad > static_cast<size_t>(INT32_MAX))
    return FA_ERR_INVALID;
  // launches
  fa::fa_bwd_prep_varlen_kernel<HD><<<static_cast<unsigned>(prep_blocks), 256, 0, stream>>>(pp);
  if (launch_status() != FA_OK) return FA_ERR_CUDA;
  if (split > 1) {  // zero the f32 dK and dV accumulators (contiguous)
    fa::fa_zero_f32_kernel<<<grid_stride_blocks(kv_elems / 2), 256, 0, stream>>>(dk_acc, kv_elems / 2);
    if (launch_status() != FA_OK) return FA_ERR_CUDA;
  }
  fa::fa_bwd2_main_kernel<HD, true><<<static_cast<unsigned>(main_blocks), C::THREADS, C::SMEM_BYTES, stream>>>(
      mq, mk, mv, mdo, mdq, mp);
  if (launch_status(reinterpret_cast<const void*>(&fa::fa_bwd2_main_kernel<HD, true>)) != FA_OK) return FA_ERR_CUDA;
  if (split > 1) {
    fa::fa_bwd_dq_kernel<<<grid_stride_blocks(kv_elems / 4), 256, 0, stream>>>(dk_acc, mp.dk, kv_elems / 4);
    if (launch_status() != FA_OK) return FA_ERR_CUDA;
    fa::fa_bwd_dq_kernel<<<grid_stride_blocks(kv_elems / 4), 256, 0, stream>>>(dv_acc, mp.dv, kv_elems / 4);
    if (launch_status() != FA_OK) return FA_ERR_CUDA;
  }
  fa::fa_bwd_dq_kernel<<<grid_stride_blocks(q_elems / 4), 256, 0, stream>>>(dq_acc, static_cast<__nv_bfloat16*>(dq),
                                                                           q_elems / 4);
  if (launch_status() != FA_OK) return FA_ERR_CUDA;
  return FA_OK;
}

// Validation of fa_fwd_kvcache's sizes: FA_OK, or the error to report.
int check_kvcache_shape(int B, int Hq, int Hkv, int Nq, int Nk, int d, float scale, int causal, int dtype) {
  if (B < 0 || Hq < 1 || Hkv < 1 || Nq < 1 || Nk < Nq || d < 1) return FA_ERR_INVALID;
  if (Hq % Hkv != 0 || (causal != 0 && causal != 1) || !std::isfinite(scale)) return FA_ERR_INVALID;
  if (dtype != FA_BF16 && dtype != FA_F32) return FA_ERR_INVALID;
  if (static_cast<long long>(B) * Hq > INT32_MAX / 2 || Nk > INT32_MAX - 256) return FA_ERR_INVALID;
  if (dtype != FA_BF16 || (d != 64 && d != 128 && d != 256)) return FA_ERR_UNSUPPORTED;
  // query rows per KV head: one 128-row MMA tile
  if (static_cast<long long>(Hq / Hkv) * Nq > 128) return FA_ERR_UNSUPPORTED;
  return FA_OK;
}

// KV-cache forward on the tensor cores: one CTA per (batch,
// KV head, key split), one CTA per SM (its K/V ring fills shared memory and
// it allocates all of TMEM). The split count minimises the estimated time,
// waves x (tiles per split + a fixed cost of about two tiles per CTA); a
// pure function of the sizes.
struct DecodeTcPlan {
  int S, split_tiles;
};

DecodeTcPlan decode_tc_plan(int B, int Hkv, int Nk) {
  const long long pairs = static_cast<long long>(B) * Hkv;
  const int tiles = (Nk + 127) / 128;
  DecodeTcPlan best{1, tiles};
  double best_cost = 1e300;
  for (int s = 1; s <= std::min(tiles, 128); ++s) {
    const int per = (tiles + s - 1) / s;
    const int used = (tiles + per - 1) / per;  // splits actually needed at that size
    const double waves = static_cast<double>((pairs * used + 147) / 148);
    const double cost = waves * (per + 2.0);
    if (cost < best_cost - 1e-9) {
      best_cost = cost;
      best = DecodeTcPlan{used, per};
    }
  }
  return best;
}

size_t kvcache_workspace_bytes(int B, int Hq, int Hkv, int Nq, int Nk, int d) {
  // split parts of O (bf16) and LSE (f32) for the merge; none with one split
  const DecodeTcPlan tp = decode_tc_plan(B, Hkv, Nk);
  if (tp.S == 1) return 0;
  return static_cast<size_t>(tp.S) * B * Hq * Nq * (2 * static_cast<size_t>(d) + 4);
}

template <int HD>
int launch_decode_tc(const void* q, const void* k, const void* v, void* o, float* lse, void* ws, int B, int Hq,
                     int Hkv, int Nq, int Nk, float scale, int causal, cudaStream_t stream) {
  using C = fa::FwdCfg<HD, true>;
  const DecodeTcPlan tp = decode_tc_plan(B, Hkv, Nk);
  const int R = (Hq / Hkv) * Nq;
  const long long rows_total = static_cast<long long>(B) * Hq * Nq;
  const long long blocks = static_cast<long long>(B) * Hkv * tp.S;
  if (blocks > INT32_MAX || rows_total > INT32_MAX) return FA_ERR_INVALID;
  CUtensorMap mq, mk, mv;
  // Q as [B * Hq * Nq][d]: a KV head's R rows are contiguous
  int rc = make_map(&mq, q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, HD, static_cast<uint64_t>(rows_total), 1, 64, 128);
  if (rc == FA_OK) rc = make_map(&mk, k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, HD, Nk, static_cast<uint64_t>(B) * Hkv, 64, 128);
  if (rc == FA_OK) rc = make_map(&mv, v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, HD, Nk, static_cast<uint64_t>(B) * Hkv, 64, 128);
  if (rc != FA_OK) return rc;
  fa::FwdParams p{};
  __nv_bfloat16* o_part = static_cast<__nv_bfloat16*>(o);
  float* lse_part = lse;
  if (tp.S > 1) {  // split parts in the workspace, merged below
    o_part = static_cast<__nv_bfloat16*>(ws);
    lse_part = reinterpret_cast<float*>(static_cast<char*>(ws) + static_cast<size_t>(tp.S) * rows_total * HD * 2);
  }
  p.o = o_part;
  p.lse = lse_part;
  p.N = Nk;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.causal = causal;
  p.timeout_ns = timeout_now();
  p.R = R;
  p.Nq = Nq;
  p.splits = tp.S;
  p.split_tiles = tp.split_tiles;
  p.rows_total = static_cast<int>(rows_total);
  MergePlan mplan{};
  if (tp.S > 1) {  // everything that can fail short of a launch, before the first launch
    int dev = 0, num_sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || num_sms_of(dev, &num_sms) != FA_OK) return FA_ERR_CUDA;
    if ((rc = plan_merge<HD>(tp.S, rows_total, num_sms, &mplan)) != FA_OK) return rc;
  }
  fa::fa_fwd_bf16_kernel<HD, true><<<static_cast<unsigned>(blocks), C::THREADS, C::SMEM_BYTES, stream>>>(mq, mk, mv, p);
  if (launch_status(reinterpret_cast<const void*>(&fa::fa_fwd_bf16_kernel<HD, true>)) != FA_OK) return FA_ERR_CUDA;
  if (tp.S == 1) return FA_OK;
  return launch_merge<HD>(mplan, o_part, lse_part, tp.S, rows_total, o, lse, stream);
}

// Checks shared by the backward entry points. `ptrs` must all be 16-byte aligned and non-null.
int check_bwd(std::initializer_list<const void*> ptrs, void* workspace, size_t workspace_bytes, int B, int Hq,
              int Hkv, int N, int d, float scale, int causal, int dtype, int* dev) {
  int rc = check_shape(B, Hq, Hkv, N, d, scale, causal, dtype);
  if (rc != FA_OK) return rc;
  if (dtype != FA_BF16) return FA_ERR_UNSUPPORTED;
  if (B == 0 || N == 0) return -1;  // empty: nothing to launch
  for (const void* p : ptrs)
    if (!aligned16(p)) return FA_ERR_INVALID;
  if (workspace == nullptr || workspace_bytes < bwd_workspace_bytes(B, Hq, Hkv, N, d)) return FA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return FA_ERR_INVALID;
  if ((rc = check_device(dev)) != FA_OK) return rc;
  return prepare_kernels(*dev);
}

}  // namespace

extern "C" {

const char* fa_status_string(int status) {
  switch (status) {
    case FA_OK: return "FA_OK";
    case FA_ERR_INVALID: return "FA_ERR_INVALID: invalid argument";
    case FA_ERR_UNSUPPORTED: return "FA_ERR_UNSUPPORTED: not implemented for these arguments or this device";
    case FA_ERR_CUDA: return "FA_ERR_CUDA: a CUDA call failed";
    case FA_ERR_TIMEOUT: return "FA_ERR_TIMEOUT: a device-side bounded wait ran out";
    case FA_ERR_WORKSPACE: return "FA_ERR_WORKSPACE: workspace missing or too small";
    default: return "unknown fa_status";
  }
}

void fa_set_wait_timeout_ns(long long timeout_ns) {
  g_timeout_ns.store(timeout_ns > 0 ? timeout_ns : kDefaultTimeoutNs);
}

int fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv, int N, int d,
           float scale, int causal, int dtype, fa_stream_t stream) {
  int rc = check_shape(B, Hq, Hkv, N, d, scale, causal, dtype);
  if (rc != FA_OK) return rc;
  if (B == 0 || N == 0) return FA_OK;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse)) return FA_ERR_INVALID;
  int dev = 0;
  if ((rc = check_device(&dev)) != FA_OK) return rc;
  if ((rc = prepare_kernels(dev)) != FA_OK) return rc;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (dtype == FA_BF16) {
    switch (d) {
      case 64: return launch_fwd_bf16_2tile<64>(q, k, v, o, lse, B, Hq, Hkv, N, scale, causal, s);
      case 128: return launch_fwd_bf16_2tile<128>(q, k, v, o, lse, B, Hq, Hkv, N, scale, causal, s);
      default: return launch_fwd_bf16_d256(q, k, v, o, lse, B, Hq, Hkv, N, scale, causal, s);
    }
  }
  switch (d) {
    case 64: return launch_fwd_f32<64>(q, k, v, o, lse, B, Hq, Hkv, N, scale, causal, s);
    case 128: return launch_fwd_f32<128>(q, k, v, o, lse, B, Hq, Hkv, N, scale, causal, s);
    default: return launch_fwd_f32<256>(q, k, v, o, lse, B, Hq, Hkv, N, scale, causal, s);
  }
}

int fa_fwd_varlen(const void* q, const void* k, const void* v, void* o, float* lse, const int* cu_seqlens_q,
                  const int* cu_seqlens_k, int batch, int max_seqlen_q, int total_q, int total_k, int Hq, int Hkv,
                  int d, float scale, int causal, int dtype, fa_stream_t stream) {
  if (batch < 0 || max_seqlen_q < 0 || total_q < 0 || total_k < 0 || Hq < 1 || Hkv < 1 || d < 1)
    return FA_ERR_INVALID;
  if (Hq % Hkv != 0 || (causal != 0 && causal != 1) || !std::isfinite(scale)) return FA_ERR_INVALID;
  if (dtype != FA_BF16 && dtype != FA_F32) return FA_ERR_INVALID;
  if (dtype != FA_BF16 || (d != 64 && d != 128)) return FA_ERR_UNSUPPORTED;
  if (batch == 0 || max_seqlen_q == 0 || total_q == 0) return FA_OK;
  if (total_k < 1 || max_seqlen_q > total_q || static_cast<long long>(total_q) * Hq > INT32_MAX / 2 ||
      static_cast<long long>(total_k) * Hkv > INT32_MAX / 2)
    return FA_ERR_INVALID;
  for (const void* ptr : {q, k, v, static_cast<const void*>(o), static_cast<const void*>(lse)})
    if (!aligned16(ptr)) return FA_ERR_INVALID;
  for (const int* cu : {cu_seqlens_q, cu_seqlens_k})
    if (cu == nullptr || (reinterpret_cast<uintptr_t>(cu) & 3u) != 0) return FA_ERR_INVALID;
  int dev = 0;
  int rc = check_device(&dev);
  if (rc != FA_OK) return rc;
  if ((rc = prepare_kernels(dev)) != FA_OK) return rc;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  return d == 64 ? launch_fwd_varlen<64>(q, k, v, o, lse, cu_seqlens_q, cu_seqlens_k, batch, max_seqlen_q, total_q,
                                         total_k, Hq, Hkv, scale, causal, s)
                 : launch_fwd_varlen<128>(q, k, v, o, lse, cu_seqlens_q, cu_seqlens_k, batch, max_seqlen_q,
                                          total_q, total_k, Hq, Hkv, scale, causal, s);
}

int fa_fwd_partial(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv, int N,
                   int d, float scale, int causal, int diag_offset, int dtype, fa_stream_t stream) {
  int rc = check_shape(B, Hq, Hkv, N, d, scale, causal, dtype);
  if (rc != FA_OK) return rc;
  if (dtype != FA_BF16) return FA_ERR_UNSUPPORTED;
  if (B == 0 || N == 0) return FA_OK;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse)) return FA_ERR_INVALID;
  // offsets beyond +-N change nothing; clamping keeps the kernel's index sums in range
  const int shift = causal ? std::max(-N, std::min(N, diag_offset)) : 0;
  int dev = 0;
  if ((rc = check_device(&dev)) != FA_OK) return rc;
  if ((rc = prepare_kernels(dev)) != FA_OK) return rc;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  switch (d) {
    case 64: return launch_fwd_bf16_2tile<64>(q, k, v, o, lse, B, Hq, Hkv, N, scale, causal, s, shift);
    case 128: return launch_fwd_bf16_2tile<128>(q, k, v, o, lse, B, Hq, Hkv, N, scale, causal, s, shift);
    default: return launch_fwd_bf16_d256(q, k, v, o, lse, B, Hq, Hkv, N, scale, causal, s, shift);
  }
}

int fa_merge_partials(const void* o_parts, const float* lse_parts, int n_parts, long long rows, void* o, float* lse,
                      int d, int dtype, fa_stream_t stream) {
  if (n_parts < 1 || rows < 0 || (d != 64 && d != 128 && d != 256)) return FA_ERR_INVALID;
  if (dtype != FA_BF16 && dtype != FA_F32) return FA_ERR_INVALID;
  if (dtype != FA_BF16) return FA_ERR_UNSUPPORTED;
  if (rows == 0) return FA_OK;
  if (rows > (1LL << 40) / n_parts) return FA_ERR_INVALID;
  for (const void* ptr : {o_parts, static_cast<const void*>(lse_parts), static_cast<const void*>(o),
                          static_cast<const void*>(lse)})
    if (!aligned16(ptr)) return FA_ERR_INVALID;
  // the output may not overlap the inputs (every thread reads all parts of
  // its columns before writing, but the LSE of a row is read by all of its
  // threads and written by one)
  const auto lo = [](const void* ptr) { return reinterpret_cast<uintptr_t>(ptr); };
  const uintptr_t in0 = lo(o_parts), in1 = in0 + static_cast<uintptr_t>(n_parts) * rows * d * 2;
  const uintptr_t l0 = lo(lse_parts), l1 = l0 + static_cast<uintptr_t>(n_parts) * rows * 4;
  const uintptr_t out0 = lo(o), out1 = out0 + static_cast<uintptr_t>(rows) * d * 2;
  const uintptr_t lo0 = lo(lse), lo1 = lo0 + static_cast<uintptr_t>(rows) * 4;
  for (const auto& a : {std::make_pair(out0, out1), std::make_pair(lo0, lo1)})
    for (const auto& b : {std::make_pair(in0, in1), std::make_pair(l0, l1)})
      if (a.first < b.second && b.first < a.second) return FA_ERR_INVALID;
  int dev = 0;
  int rc = check_device(&dev);
  if (rc != FA_OK) return rc;
  if ((rc = prepare_kernels(dev)) != FA_OK) return rc;
  int num_sms = 0;
  if ((rc = num_sms_of(dev, &num_sms)) != FA_OK) return rc;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  MergePlan mp{};
  switch (d) {
    case 64:
      if ((rc = plan_merge<64>(n_parts, rows, num_sms, &mp)) != FA_OK) return rc;
      return launch_merge<64>(mp, o_parts, lse_parts, n_parts, rows, o, lse, s);
    case 128:
      if ((rc = plan_merge<128>(n_parts, rows, num_sms, &mp)) != FA_OK) return rc;
      return launch_merge<128>(mp, o_parts, lse_parts, n_parts, rows, o, lse, s);
    default:
      if ((rc = plan_merge<256>(n_parts, rows, num_sms, &mp)) != FA_OK) return rc;
      return launch_merge<256>(mp, o_parts, lse_parts, n_parts, rows, o, lse, s);
  }
}

int fa_bwd_partial(const void* q, const void* k, const void* v, const void* dO, float* dk_acc, float* dv_acc,
                   void* workspace, size_t workspace_bytes, int B, int Hq, int Hkv, int N, int d, float scale,
                   int causal, int diag_offset, int dtype, fa_stream_t stream) {
  int rc = check_shape(B, Hq, Hkv, N, d, scale, causal, dtype);
  if (rc != FA_OK) return rc;
  if (dtype != FA_BF16 || (d != 64 && d != 128)) return FA_ERR_UNSUPPORTED;
  int dev = 0;
  rc = check_bwd({q, k, v, dO, dk_acc, dv_acc}, workspace, workspace_bytes, B, Hq, Hkv, N, d, scale, causal, dtype,
                 &dev);
  if (rc != FA_OK) return rc < 0 ? FA_OK : rc;
  // offsets beyond +-N change nothing; clamping keeps the kernel's index sums in range
  const int shift = causal ? std::max(-N, std::min(N, diag_offset)) : 0;
  BwdPlan pl;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (d == 64) {
    if ((rc = plan_bwd<64>(&pl, 2u, q, k, v, nullptr, nullptr, dO, nullptr, nullptr, nullptr, workspace, B, Hq, Hkv, N,
                           scale, causal, s, shift, dk_acc, dv_acc)) != FA_OK)
      return rc;
    return launch_bwd_stages<64>(pl, 2u);
  }
  if ((rc = plan_bwd<128>(&pl, 2u, q, k, v, nullptr, nullptr, dO, nullptr, nullptr, nullptr, workspace, B, Hq, Hkv, N,
                          scale, causal, s, shift, dk_acc, dv_acc)) != FA_OK)
    return rc;
  return launch_bwd_stages<128>(pl, 2u);
}

int fa_f32_to_bf16(const float* src, void* dst, size_t n, fa_stream_t stream) {
  if (n == 0) return FA_OK;
  if (n % 4 != 0 || !aligned16(src) || !aligned16(dst)) return FA_ERR_INVALID;
  int dev = 0;
  int rc = check_device(&dev);
  if (rc != FA_OK) return rc;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  fa::fa_bwd_dq_kernel<<<grid_stride_blocks(n / 4), 256, 0, s>>>(src, static_cast<__nv_bfloat16*>(dst), n / 4);
  return launch_status();
}

size_t fa_bwd_varlen_workspace_size(int batch, int total_q, int total_k, int Hq, int Hkv, int d) {
  if (batch < 0 || total_q < 0 || total_k < 0 || Hq < 1 || Hkv < 1 || d < 1 || Hq % Hkv != 0) return 0;
  return bwd_varlen_workspace_bytes(batch, total_q, total_k, Hq, Hkv, d);
}

int fa_bwd_varlen(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dO,
                  void* dq, void* dk, void* dv, const int* cu_seqlens_q, const int* cu_seqlens_k, int batch,
                  int max_seqlen_q, int max_seqlen_k, int total_q, int total_k, int Hq, int Hkv, int d, float scale,
                  int causal, void* workspace, size_t workspace_bytes, int dtype, fa_stream_t stream) {
  if (batch < 0 || max_seqlen_q < 0 || max_seqlen_k < 0 || total_q < 0 || total_k < 0 || Hq < 1 || Hkv < 1 ||
      d < 1)
    return FA_ERR_INVALID;
  if (Hq % Hkv != 0 || (causal != 0 && causal != 1) || !std::isfinite(scale)) return FA_ERR_INVALID;
  if (dtype != FA_BF16 && dtype != FA_F32) return FA_ERR_INVALID;
  if (dtype != FA_BF16 || (d != 64 && d != 128)) return FA_ERR_UNSUPPORTED;
  if (batch == 0 || total_k == 0) return FA_OK;
  if (total_q == 0) {
    // no queries at all: every key's gradient is zero
    if (!aligned16(dk) || !aligned16(dv)) return FA_ERR_INVALID;
    int dev = 0;
    int rc = check_device(&dev);
    if (rc != FA_OK) return rc;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const size_t n4 = static_cast<size_t>(total_k) * Hkv * d / 8;  // bf16 elements, 8 per 16 bytes
    fa::fa_zero_f32_kernel<<<grid_stride_blocks(n4), 256, 0, s>>>(static_cast<float*>(dk), n4);
    if (launch_status() != FA_OK) return FA_ERR_CUDA;
    fa::fa_zero_f32_kernel<<<grid_stride_blocks(n4), 256, 0, s>>>(static_cast<float*>(dv), n4);
    return launch_status();
  }
  if (max_seqlen_q > total_q || max_seqlen_k > total_k || max_seqlen_k < 1 ||
      static_cast<long long>(total_q) * Hq > INT32_MAX / 2 || static_cast<long long>(total_k) * Hkv > INT32_MAX / 2 ||
      total_q > INT32_MAX - 4 * batch - 256)
    return FA_ERR_INVALID;
  for (const void* ptr : std::initializer_list<const void*>{q, k, v, o, lse, dO, dq, dk, dv})
    if (!aligned16(ptr)) return FA_ERR_INVALID;
  for (const int* cu : {cu_seqlens_q, cu_seqlens_k})
    if (cu == nullptr || (reinterpret_cast<uintptr_t>(cu) & 3u) != 0) return FA_ERR_INVALID;
  if (workspace == nullptr || !aligned16(workspace) ||
      workspace_bytes < bwd_varlen_workspace_bytes(batch, total_q, total_k, Hq, Hkv, d))
    return FA_ERR_WORKSPACE;
  int dev = 0;
  int rc = check_device(&dev);
  if (rc != FA_OK) return rc;
  if ((rc = prepare_kernels(dev)) != FA_OK) return rc;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  return d == 64 ? run_bwd_varlen<64>(q, k, v, o, lse, dO, dq, dk, dv, cu_seqlens_q, cu_seqlens_k, batch,
                                      max_seqlen_q, max_seqlen_k, total_q, total_k, Hq, Hkv, scale, causal,
                                      workspace, s)
                 : run_bwd_varlen<128>(q, k, v, o, lse, dO, dq, dk, dv, cu_seqlens_q, cu_seqlens_k, batch,
                                       max_seqlen_q, max_seqlen_k, total_q, total_k, Hq, Hkv, scale, causal,
                                       workspace, s);
}

size_t fa_bwd_workspace_size(int B, int Hq, int Hkv, int N, int d) {
  if (B < 0 || N < 0 || Hq < 1 || Hkv < 1 || d < 1 || Hq % Hkv != 0) return 0;
  return bwd_workspace_bytes(B, Hq, Hkv, N, d);
}

}  // extern "C"

namespace {

// Validate, plan every launch of the requested stages, then launch them in
// stream order. Errors other than a failed launch are returned before any
// kernel is queued.
int run_bwd(unsigned stages, std::initializer_list<const void*> ptrs, const void* q, const void* k, const void* v,
            const void* o, const float* lse, const void* dO, void* dq, void* dk, void* dv, void* ws,
            size_t ws_bytes, int B, int Hq, int Hkv, int N, int d, float scale, int causal, int dtype,
            fa_stream_t stream) {
  int dev = 0;
  int rc = check_bwd(ptrs, ws, ws_bytes, B, Hq, Hkv, N, d, scale, causal, dtype, &dev);
  if (rc != FA_OK) return rc < 0 ? FA_OK : rc;
  BwdPlan pl;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (d == 64) {
    if ((rc = plan_bwd<64>(&pl, stages, q, k, v, o, lse, dO, dq, dk, dv, ws, B, Hq, Hkv, N, scale, causal, s)) !=
        FA_OK)
      return rc;
    return launch_bwd_stages<64>(pl, stages);
  }
  if (d == 256) {
    if ((rc = plan_bwd<256>(&pl, stages, q, k, v, o, lse, dO, dq, dk, dv, ws, B, Hq, Hkv, N, scale, causal, s)) !=
        FA_OK)
      return rc;
    return launch_bwd_stages<256>(pl, stages);
  }
  if ((rc = plan_bwd<128>(&pl, stages, q, k, v, o, lse, dO, dq, dk, dv, ws, B, Hq, Hkv, N, scale, causal, s)) !=
      FA_OK)
    return rc;
  return launch_bwd_stages<128>(pl, stages);
}

}  // namespace

extern "C" {

int fa_bwd_prep(const void* o, const float* lse, const void* dO, void* workspace, size_t workspace_bytes, int B,
                int Hq, int Hkv, int N, int d, int dtype, fa_stream_t stream) {
  return run_bwd(1u, {o, lse, dO}, nullptr, nullptr, nullptr, o, lse, dO, nullptr, nullptr, nullptr, workspace,
                 workspace_bytes, B, Hq, Hkv, N, d, 1.0f, 0, dtype, stream);
}

int fa_bwd_main(const void* q, const void* k, const void* v, const void* dO, void* dk, void* dv, void* workspace,
                size_t workspace_bytes, int B, int Hq, int Hkv, int N, int d, float scale, int causal, int dtype,
                fa_stream_t stream) {
  return run_bwd(2u, {q, k, v, dO, dk, dv}, q, k, v, nullptr, nullptr, dO, nullptr, dk, dv, workspace,
                 workspace_bytes, B, Hq, Hkv, N, d, scale, causal, dtype, stream);
}

int fa_bwd_dq(void* dq, void* workspace, size_t workspace_bytes, int B, int Hq, int Hkv, int N, int d, int dtype,
              fa_stream_t stream) {
  return run_bwd(4u, {dq}, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, dq, nullptr, nullptr, workspace,
                 workspace_bytes, B, Hq, Hkv, N, d, 1.0f, 0, dtype, stream);
}

int fa_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dO, void* dq,
           void* dk, void* dv, void* workspace, size_t workspace_bytes, int B, int Hq, int Hkv, int N, int d,
           float scale, int causal, int dtype, fa_stream_t stream) {
  return run_bwd(7u, {q, k, v, o, lse, dO, dq, dk, dv}, q, k, v, o, lse, dO, dq, dk, dv, workspace,
                 workspace_bytes, B, Hq, Hkv, N, d, scale, causal, dtype, stream);
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Backward without caller-provided workspace.
//
// Some callers cannot allocate device memory at the point where they run the
// backward: code inside a region where the allocator must not be touched
// (a caching allocator that is locked, a pre-planned memory arena, a runtime
// that forbids cudaMalloc after start-up), or plain C callers with no
// allocator of their own. For them the scratch lives in a fixed array in
// device memory that the library owns: every GPU that loads the library
// holds it until the process exits.
namespace {

constexpr size_t kNoAllocScratchBytes = FA_NOALLOC_SCRATCH_BYTES;
static __device__ __align__(256) unsigned char g_noalloc_scratch[FA_NOALLOC_SCRATCH_BYTES];

// Device address of g_noalloc_scratch on the current device, looked up once
// per device with that device current (the first fa_bwd_noalloc call on the
// device does it). In host code the array's name is only a host-side
// stand-in, never a device address. The address is kept for the life of the
// process, so a device reset after the first call is not supported.
int noalloc_scratch(int dev, void** out) {
  static std::mutex mu;
  static void* addr[128] = {};
  if (dev < 0 || dev >= 128) return FA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(mu);
  if (addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return FA_ERR_CUDA;
    addr[dev] = p;
  }
  *out = addr[dev];
  return FA_OK;
}

}  // namespace

extern "C" {

int fa_bwd_noalloc(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dO,
                   void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int N, int d, float scale, int causal,
                   int dtype, fa_stream_t stream) {
  int rc = check_shape(B, Hq, Hkv, N, d, scale, causal, dtype);
  if (rc != FA_OK) return rc;
  if (dtype != FA_BF16) return FA_ERR_UNSUPPORTED;
  if (B == 0 || N == 0) return FA_OK;
  if (bwd_workspace_bytes(B, Hq, Hkv, N, d) > kNoAllocScratchBytes) return FA_ERR_WORKSPACE;
  int dev = 0;
  if ((rc = check_device(&dev)) != FA_OK) return rc;
  void* scratch = nullptr;
  if ((rc = noalloc_scratch(dev, &scratch)) != FA_OK) return rc;
  // Every scratch byte this problem reads is rewritten first (D, LSE and the
  // dQ accumulator by the prep kernel; the dK/dV accumulators, when the
  // group's heads are split, by a zeroing kernel before the main kernel), so
  // what an earlier call left in the array does not matter.
  return run_bwd(7u, {q, k, v, o, lse, dO, dq, dk, dv}, q, k, v, o, lse, dO, dq, dk, dv, scratch,
                 kNoAllocScratchBytes, B, Hq, Hkv, N, d, scale, causal, dtype, stream);
}

size_t fa_fwd_kvcache_workspace_size(int B, int Hq, int Hkv, int Nq, int Nk, int d) {
  if (check_kvcache_shape(B, Hq, Hkv, Nq, Nk, d, 1.0f, 0, FA_BF16) == FA_ERR_INVALID) return 0;
  return kvcache_workspace_bytes(B, Hq, Hkv, Nq, Nk, d);
}

int fa_fwd_kvcache(const void* q, const void* k, const void* v, void* o, float* lse, void* workspace,
                   size_t workspace_bytes, int B, int Hq, int Hkv, int Nq, int Nk, int d, float scale, int causal,
                   int dtype, fa_stream_t stream) {
  int rc = check_kvcache_shape(B, Hq, Hkv, Nq, Nk, d, scale, causal, dtype);
  if (rc != FA_OK) return rc;
  if (B == 0) return FA_OK;
  for (const void* ptr : {q, k, v, static_cast<const void*>(o), static_cast<const void*>(lse)})
    if (!aligned16(ptr)) return FA_ERR_INVALID;
  const size_t need = kvcache_workspace_bytes(B, Hq, Hkv, Nq, Nk, d);
  if (need > 0 && (workspace == nullptr || workspace_bytes < need)) return FA_ERR_WORKSPACE;
  if (need > 0 && !aligned16(workspace)) return FA_ERR_INVALID;
  int dev = 0;
  if ((rc = check_device(&dev)) != FA_OK) return rc;
  if ((rc = prepare_kernels(dev)) != FA_OK) return rc;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  switch (d) {
    case 64: return launch_decode_tc<64>(q, k, v, o, lse, workspace, B, Hq, Hkv, Nq, Nk, scale, causal, s);
    case 128: return launch_decode_tc<128>(q, k, v, o, lse, workspace, B, Hq, Hkv, Nq, Nk, scale, causal, s);
    default: return launch_decode_tc<256>(q, k, v, o, lse, workspace, B, Hq, Hkv, Nq, Nk, scale, causal, s);
  }
}

int fa_last_device_status(fa_stream_t stream) {
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return FA_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, fa::g_status, sizeof(int)) != cudaSuccess) return FA_ERR_CUDA;
  const int zero = 0;
  if (cudaMemcpyToSymbol(fa::g_status, &zero, sizeof(int)) != cudaSuccess) return FA_ERR_CUDA;
  return v;
}

int fa_selftest_wait_timeout(long long timeout_ns, fa_stream_t stream) {
  if (timeout_ns <= 0 || timeout_ns > 10000000000LL) return FA_ERR_INVALID;
  int dev = 0;
  int rc = check_device(&dev);
  if (rc != FA_OK) return rc;
  fa_selftest_wait_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      static_cast<unsigned long long>(timeout_ns));
  return launch_status();
}

}  // extern "C"
