// gemm_tc.cu -- the compressor projection P = H * Wpacked^T on the 5th-
// generation tensor cores ("DeepSeekV4技术报告阅读笔记" eq. 9-10 and 20-21: all
// of C^a, C^b, Z^a, Z^b and the indexer's four matrices in one product).
//
// bf16 inputs, both K-major (H rows and packed weight rows are contiguous
// along d), fp32 accumulation in TMEM, fp32 output [M][N].  128 x 256 output
// tiles, 64-deep K stages fed by TMA in the 128-byte swizzle layout; a
// persistent grid walks the tiles.  Warp 0 loads, warp 1 owns TMEM and
// issues the MMAs (4 per K stage), warps 2-5 drain the two TMEM accumulators
// and store; every wait is bounded.
#include <cuda.h>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace csa {

using namespace sm100;

constexpr int kGm = 128, kGn = 256, kGk = 64;
constexpr int kGStages = 4;
constexpr int kGAStage = kGm * kGk * 2;  // 16 KB
constexpr int kGBStage = kGn * kGk * 2;  // 32 KB
constexpr int kGThreads = 192;

struct GemmArgs {
  float* C;
  unsigned* err;
  int M, N, K, tiles_n, tiles;
};

__global__ void __launch_bounds__(kGThreads, 1)
    gemm_bf16_tc(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                 GemmArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* sA = sm;
  uint8_t* sB = sA + kGStages * kGAStage;
  uint64_t* bars = (uint64_t*)(sB + kGStages * kGBStage);
  uint64_t* full = bars;
  uint64_t* empty = bars + kGStages;
  uint64_t* tfull = bars + 2 * kGStages;
  uint64_t* tempty = tfull + 2;
  uint32_t* tbase_sm = (uint32_t*)(tempty + 2);
  volatile int* abort_sm = (volatile int*)(tbase_sm + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < kGStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], 4);
    }
    *abort_sm = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tbase_sm, 512);
    tmem_relinquish();
  }
  if (threadIdx.x == 32) {
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tbase_sm;
  const int KB = (a.K + kGk - 1) / kGk;

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------------------ loads --
    int kn = 0;
    for (int tile = blockIdx.x; tile < a.tiles; tile += gridDim.x) {
      const int m0 = (tile / a.tiles_n) * kGm, n0 = (tile % a.tiles_n) * kGn;
      bool ok = true;
      for (int kb = 0; kb < KB; ++kb, ++kn) {
        const int s = kn % kGStages;
        if (!mbar_wait(&empty[s], ((kn / kGStages) & 1) ^ 1, abort_sm)) { ok = false; break; }
        mbar_expect_tx(&full[s], kGAStage + kGBStage);
        tma_load_2d(sA + s * kGAStage, &tmA, &full[s], kb * kGk, m0);
        tma_load_2d(sB + s * kGBStage, &tmB, &full[s], kb * kGk, n0);
      }
      if (!ok) break;
    }
  } else if (warp == 1 && lane == 0) {
    // ------------------------------------------------------------- MMA --
    const uint32_t idesc = idesc_bf16(kGm, kGn);
    int kn = 0, an = 0;
    for (int tile = blockIdx.x; tile < a.tiles; tile += gridDim.x, ++an) {
      const int acc = an & 1;
      if (!mbar_wait(&tempty[acc], ((an >> 1) & 1) ^ 1, abort_sm)) break;
      tc_fence_after();
      const uint32_t d = tbase + acc * kGn;
      bool ok = true;
      for (int kb = 0; kb < KB; ++kb, ++kn) {
        const int s = kn % kGStages;
        if (!mbar_wait(&full[s], (kn / kGStages) & 1, abort_sm)) { ok = false; break; }
        tc_fence_after();
        const uint32_t ab = smem_u32(sA + s * kGAStage), bb = smem_u32(sB + s * kGBStage);
#pragma unroll
        for (int j = 0; j < 4; ++j)
          mma_bf16(d, sdesc_k_sw128(ab + j * 32), sdesc_k_sw128(bb + j * 32), idesc,
                   (kb | j) != 0);
        mma_commit(&empty[s]);
      }
      if (!ok) break;
      mma_commit(&tfull[acc]);
    }
  } else if (warp >= 2) {
    // -------------------------------------------------------- epilogue --
    const int quad = warp & 3;
    int an = 0;
    for (int tile = blockIdx.x; tile < a.tiles; tile += gridDim.x, ++an) {
      const int acc = an & 1;
      if (!mbar_wait(&tfull[acc], (an >> 1) & 1, abort_sm)) break;
      tc_fence_after();
      const int m0 = (tile / a.tiles_n) * kGm, n0 = (tile % a.tiles_n) * kGn;
      const int row = m0 + quad * 32 + lane;
      const uint32_t trow = tbase + ((uint32_t)(quad * 32) << 16) + acc * kGn;
      float* dst = a.C + (size_t)row * a.N + n0;
      for (int c0 = 0; c0 < kGn; c0 += 64) {
        float v[4][16];
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) tmem_ld16(trow + c0 + q4 * 16, v[q4]);
        tmem_wait_ld();
        if (row < a.M) {
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4)
#pragma unroll
            for (int u = 0; u < 16; u += 4) {
              const int col = c0 + q4 * 16 + u;
              if (n0 + col + 3 < a.N)
                *reinterpret_cast<float4*>(dst + col) =
                    make_float4(v[q4][u], v[q4][u + 1], v[q4][u + 2], v[q4][u + 3]);
              else
                for (int x = 0; x < 4; ++x)
                  if (n0 + col + x < a.N) dst[col + x] = v[q4][u + x];
            }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[acc]);
    }
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (*abort_sm) {
    if (threadIdx.x == 0) atomicOr(a.err, CSA_DEV_TIMEOUT);
    const uint64_t t0 = globaltimer();
    while (globaltimer() - t0 < 200000ull) __nanosleep(1000);
  }
  if (warp == 1) tmem_dealloc(tbase, 512);
}

bool make_tmap_bf16(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols,
                    uint32_t box_rows);
bool tma_available();

bool gemm_tc_supported(int M, int N, int K) {
  return M > 0 && N > 0 && K > 0 && K % 8 == 0 && N % 4 == 0 && tma_available();
}

// C[M][N] = A[M][K] * B[N][K]^T (bf16, K-major), fp32 out.
csa_status launch_gemm_tc(const void* A, const void* B, float* C, int M, int N, int K,
                          cudaStream_t st) {
  CUtensorMap tmA, tmB;
  if (!make_tmap_bf16(&tmA, A, (uint64_t)M, (uint64_t)K, kGm)) return CSA_ERR_CUDA;
  if (!make_tmap_bf16(&tmB, B, (uint64_t)N, (uint64_t)K, kGn)) return CSA_ERR_CUDA;
  GemmArgs a{C, device_error_word(), M, N, K, (N + kGn - 1) / kGn, 0};
  if (a.err == nullptr) return CSA_ERR_CUDA;
  a.tiles = ((M + kGm - 1) / kGm) * a.tiles_n;
  const int smem = 1024 + kGStages * (kGAStage + kGBStage) + 256;
  if (!set_kernel_smem((const void*)gemm_bf16_tc, smem)) return CSA_ERR_CUDA;
  const int sms = sm_count();
  const int grid = a.tiles < sms ? a.tiles : sms;
  CSA_LAUNCH(KK_GEMM, st, gemm_bf16_tc<<<grid, kGThreads, smem, st>>>(tmA, tmB, a));
  return last_launch_status();
}

}  // namespace csa
