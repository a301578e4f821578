// common.cuh -- shared device helpers of the CSA / HCA CUDA library (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "csa.h"

namespace csa {

// ----------------------------------------------------------------- launch --
// Every launcher bumps this counter (exported through csa_kernel_launches).
void count_launch(int n = 1);

// Kernel kinds for the profiler (csa_profile_*).
enum KernelKind {
  KK_PACK = 0, KK_GEMM, KK_FOLD, KK_WINDOW, KK_SCORES, KK_TOPK, KK_ATTN,
  KK_COMBINE, KK_PLAN, KK_TOPK_HIST, KK_TOPK_SELECT, KK_TOPK_FINAL, KK_DIAG, KK_COUNT
};
// Bracket one launch: begin() before it, end() after it, same stream.
int prof_begin(int kind, cudaStream_t st);
void prof_end(int slot, cudaStream_t st);

// Launch one kernel with profiling brackets and the launch counter.
#define CSA_LAUNCH(kind, st, ...)            \
  do {                                       \
    int csa_slot_ = ::csa::prof_begin(kind, st); \
    __VA_ARGS__;                             \
    ::csa::prof_end(csa_slot_, st);          \
    ::csa::count_launch();                   \
  } while (0)

// Programmatic dependent launch: a kernel launched with it may be scheduled
// while the previous kernel of the stream still runs; it calls pdl_wait()
// before it reads anything earlier stream work wrote (a no-op otherwise).
// A kernel calls pdl_trigger() to let its dependent be scheduled early.
constexpr bool kPdlAttend = true;   // attention after the top-k
constexpr bool kPdlTopk = false;    // top-k select after the scorer (measured slower)
constexpr bool kPdlCombine = false; // slice combine after the attention (no gain)
constexpr bool kPdlAppend = true;   // decode compressor: finish after the projection
// launch with the programmatic-dependent attribute when `pdl` is set
template <typename... KArgs, typename... Args>
inline cudaError_t launch_maybe_pdl(bool pdl, void (*kern)(KArgs...), dim3 grid, dim3 block,
                                    size_t smem, cudaStream_t st, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, args...);
}
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Host-side caches (csa_abi.cu): SM count of the current device; a kernel's
// dynamic shared-memory limit set once per (kernel, device, size); its
// resident CTAs per SM queried once per (kernel, device, threads, size).
int sm_count();
bool set_kernel_smem(const void* kern, int smem);
int kernel_occupancy(const void* kern, int threads, int smem);

// Device error word of the current GPU (set with atomicOr from kernels).
unsigned int* device_error_word();

inline csa_status last_launch_status() {
  return cudaGetLastError() == cudaSuccess ? CSA_OK : CSA_ERR_CUDA;
}

__host__ __device__ inline size_t align_up(size_t x, size_t a) {
  return (x + a - 1) / a * a;
}

// ------------------------------------------------------------ conversions --
__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

// OCP E4M3 code -> value (exact in fp32), through CUDA's conversion.
__device__ __forceinline__ float e4m3_to_f32(uint8_t code) {
  __half_raw h = __nv_cvt_fp8_to_halfraw((__nv_fp8_storage_t)code, __NV_E4M3);
  return __half2float(__half(h));
}
// value -> OCP E4M3 code, round to nearest even, saturating to +-448.
__device__ __forceinline__ uint8_t f32_to_e4m3(float x) {
  return (uint8_t)__nv_cvt_float_to_fp8(x, __NV_SATFINITE, __NV_E4M3);
}

// Order-preserving map of an fp32 score to uint32 (larger score -> larger key).
__device__ __forceinline__ uint32_t score_key(float s) {
  uint32_t u = __float_as_uint(s);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// ------------------------------------------------------------------- RoPE --
// Angle of pair p at position pos: pos * base^(-2p/rope_dims), in double so
// that positions up to 2^20 and beyond keep full fp32 accuracy after sincos.
__device__ __forceinline__ void rope_cs(double pos, int p, int rope_dims,
                                        double base, float* cs, float* sn) {
  double theta = pow(base, -2.0 * (double)p / (double)rope_dims);
  double s, c;
  sincos(pos * theta, &s, &c);
  *cs = (float)c;
  *sn = (float)s;
}

// Decode compressor: fold one (C, z) pair into an open entry's running
// softmax (largest logit, denominator, weighted sum of C); `fresh` starts
// the entry.
__device__ __forceinline__ void running_softmax_step(float& mx, float& den, float& num, float C,
                                                     float z, bool fresh) {
  if (fresh) {
    mx = z; den = 1.f; num = C;
    return;
  }
  const float m0 = mx, m1 = fmaxf(m0, z);
  const float s0 = expf(m0 - m1), s1 = expf(z - m1);
  mx = m1;
  den = fmaf(den, s0, s1);
  num = fmaf(num, s0, s1 * C);
}
__device__ __forceinline__ void running_softmax_add(float* mx, float* den, float* num, float C,
                                                    float z, bool fresh) {
  float m = fresh ? 0.f : *mx, d = fresh ? 0.f : *den, n = fresh ? 0.f : *num;
  running_softmax_step(m, d, n, C, z, fresh);
  *mx = m; *den = d; *num = n;
}

// ------------------------------------------------------------ reductions --
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Block-wide reduction (sum or max) for blockDim.x a multiple of 32;
// `red` needs 32 floats of shared memory.  Every thread gets the result.
template <bool kMax>
__device__ float block_reduce(float v, float* red) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int nw = blockDim.x >> 5;
  v = kMax ? warp_max(v) : warp_sum(v);
  __syncthreads();
  if (lane == 0) red[wid] = v;
  __syncthreads();
  float r = lane < nw ? red[lane] : (kMax ? -INFINITY : 0.0f);
  r = kMax ? warp_max(r) : warp_sum(r);
  return r;
}

// Block-wide exclusive scan of unsigned counts (blockDim.x <= 1024, multiple
// of 32).  `sh` needs 33 unsigned of shared memory.  Returns the exclusive
// prefix; *total receives the block total.
__device__ __forceinline__ unsigned block_exclusive_scan(unsigned v, unsigned* sh,
                                                         unsigned* total) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int nw = blockDim.x >> 5;
  unsigned x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    unsigned y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  __syncthreads();
  if (lane == 31) sh[wid] = x;
  __syncthreads();
  if (wid == 0) {
    unsigned s = lane < nw ? sh[lane] : 0u;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      unsigned y = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += y;
    }
    if (lane < nw) sh[lane] = s;  // inclusive over warps
    if (lane == 31) sh[32] = s;
  }
  __syncthreads();
  unsigned before = wid > 0 ? sh[wid - 1] : 0u;
  *total = sh[32];
  return before + x - v;
}

// Visible compressed entries for a query at t0: floor((t0+1)/m) clamped.
__host__ __device__ __forceinline__ int n_visible(int t0, int m, int N) {
  if (t0 < 0) return 0;
  long long v = ((long long)t0 + 1) / m;
  return (int)(v < N ? v : N);
}

}  // namespace csa
