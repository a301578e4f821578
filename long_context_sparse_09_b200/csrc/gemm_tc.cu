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
      // (the warp leaves together: the loop holds warp collectives)
      if (!__all_sync(0xffffffffu, mbar_wait(&tfull[acc], (an >> 1) & 1, abort_sm))) break;
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


// ------------------------------------------- GEMM with the fold epilogue --
// The compressor projection with the per-channel softmax over the 2m slots
// and the fold in the epilogue ("DeepSeekV4技术报告阅读笔记" eq. 11-12 and
// 22-23): the fp32 product never reaches HBM.
//
// An output tile is 128 token rows x 256 columns, the columns of one block
// of channels gathered from the packed weights by four 64-row TMA boxes:
// CSA [C^a | C^b | Z^a | Z^b] of 64 channels (main entries, then the
// indexer's), HCA [C | Z] of 128 channels.  CSA tiles overlap by m rows, so
// that an entry's b window (the m rows before its a window) is in the same
// tile: tile j of a sequence starts at row j*E*m - m and yields entries
// j*E .. j*E + E - 1 with E = (128 - m) / m; HCA tiles hold E = 128 / m
// whole entries.  The epilogue stages 8 channels of the four (two) parts at
// a time in shared memory ([part][channel][row]) and folds: for CSA one
// thread per (entry, channel), for HCA m/8 threads per (entry, channel),
// each over 8 rows, reduced with shuffles.  It writes the folded entries
// before their norm (fp32 F [B*nE][c + c_I], indexer channels after the
// main ones) and, from the main C^a columns, each token's C^a row (fp32
// [B*T][c], the source of the window rows).
constexpr int kFStages = 4;
constexpr int kFChunk = 8;  // channels staged per pass
constexpr int kFSmem = 1024 + kFStages * (kGAStage + kGBStage) + 4 * kFChunk * 128 * 4 + 256;

struct GemmFoldArgs {
  const float* bias;  // [m][nb]
  float* F;           // [B*nE][c + cI]
  float* Ca;          // [B*T][c]
  unsigned* err;
  int B, T, m, overlap, c, cI, nb;
  int col_Ca, col_Cb, col_Za, col_Zb, col_CIa, col_CIb, col_ZIa, col_ZIb;
  int b_Ba, b_Bb, b_BIa, b_BIb;
  int E;             // entries per tile
  int mt_per_seq;    // row tiles per sequence
  int nt;            // column tiles
  int tiles, K;
};

// rows of the packed weights the four 64-row boxes of column tile n load,
// and the tile's parts: 0 main, 1 indexer (CSA); the tile's first channel
struct FoldTile {
  int rows[4];
  int indexer, ch0, nch;
};

__device__ __forceinline__ FoldTile fold_tile(const GemmFoldArgs& a, int n) {
  FoldTile f;
  if (a.overlap) {
    const int nbc = a.c / 64;
    f.indexer = n >= nbc;
    f.ch0 = (f.indexer ? n - nbc : n) * 64;
    f.nch = 64;
    f.rows[0] = (f.indexer ? a.col_CIa : a.col_Ca) + f.ch0;
    f.rows[1] = (f.indexer ? a.col_CIb : a.col_Cb) + f.ch0;
    f.rows[2] = (f.indexer ? a.col_ZIa : a.col_Za) + f.ch0;
    f.rows[3] = (f.indexer ? a.col_ZIb : a.col_Zb) + f.ch0;
  } else {
    f.indexer = 0;
    f.ch0 = n * 128;
    f.nch = 128;
    f.rows[0] = a.col_Ca + f.ch0;
    f.rows[1] = a.col_Ca + f.ch0 + 64;
    f.rows[2] = a.col_Za + f.ch0;
    f.rows[3] = a.col_Za + f.ch0 + 64;
  }
  return f;
}

__global__ void __launch_bounds__(kGThreads, 1)
    gemm_fold_tc(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                 GemmFoldArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* sA = sm;
  uint8_t* sB = sA + kFStages * kGAStage;
  float* stg = (float*)(sB + kFStages * kGBStage);  // [4 parts][kFChunk][128 rows]
  uint64_t* bars = (uint64_t*)(stg + 4 * kFChunk * 128);
  uint64_t* full = bars;
  uint64_t* empty = bars + kFStages;
  uint64_t* tfull = bars + 2 * kFStages;
  uint64_t* tempty = tfull + 2;
  uint32_t* tbase_sm = (uint32_t*)(tempty + 2);
  volatile int* abort_sm = (volatile int*)(tbase_sm + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < kFStages; ++i) {
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
  const int stride = a.E * a.m;       // token rows a tile advances
  const int lead = a.overlap ? a.m : 0;  // rows before the tile's first entry

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------------------ loads --
    int kn = 0;
    for (int tile = blockIdx.x; tile < a.tiles; tile += gridDim.x) {
      const int mt = tile / a.nt, n = tile % a.nt;
      const int b = mt / a.mt_per_seq, j = mt % a.mt_per_seq;
      const int r0 = b * a.T + j * stride - lead;  // may be negative: zero fill
      const FoldTile f = fold_tile(a, n);
      bool ok = true;
      for (int kb = 0; kb < KB; ++kb, ++kn) {
        const int s = kn % kFStages;
        if (!mbar_wait(&empty[s], ((kn / kFStages) & 1) ^ 1, abort_sm)) { ok = false; break; }
        mbar_expect_tx(&full[s], kGAStage + kGBStage);
        tma_load_2d(sA + s * kGAStage, &tmA, &full[s], kb * kGk, r0);
#pragma unroll
        for (int q = 0; q < 4; ++q)
          tma_load_2d(sB + s * kGBStage + q * (kGBStage / 4), &tmB, &full[s], kb * kGk,
                      f.rows[q]);
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
        const int s = kn % kFStages;
        if (!mbar_wait(&full[s], (kn / kFStages) & 1, abort_sm)) { ok = false; break; }
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
    // ------------------------------------------------- fold epilogue --
    // After a wait gives up, a warp keeps walking its tiles without work so
    // that all four epilogue warps take the same named barriers.
    const int quad = warp & 3;
    const int rho = quad * 32 + lane;   // the tile row (TMEM lane) this thread drains
    const int et = threadIdx.x - 64;    // 0..127
    const int nF = a.c + a.cI;
    const int nE = a.T / a.m;
    int an = 0;
    bool dead = false;
    for (int tile = blockIdx.x; tile < a.tiles; tile += gridDim.x, ++an) {
      const int acc = an & 1;
      if (!dead) dead = !__all_sync(0xffffffffu, mbar_wait(&tfull[acc], (an >> 1) & 1, abort_sm));
      tc_fence_after();
      const int mt = tile / a.nt, n = tile % a.nt;
      const int b = mt / a.mt_per_seq, j = mt % a.mt_per_seq;
      const int e0 = j * a.E;                 // first entry of the tile
      const int tok0 = j * stride - lead;     // token (within the sequence) of row 0
      const FoldTile f = fold_tile(a, n);
      const uint32_t trow = tbase + ((uint32_t)(quad * 32) << 16) + acc * kGn;
      const int bA = f.indexer ? a.b_BIa : a.b_Ba, bB = f.indexer ? a.b_BIb : a.b_Bb;
      const int fcol = (f.indexer ? a.c : 0) + f.ch0;  // column of channel 0 in F
      // parts of the tile: CSA C^a, C^b, Z^a, Z^b at column 64 q; HCA C at
      // columns [0, 128), Z at [128, 256)
      for (int c0 = 0; c0 < f.nch; c0 += kFChunk) {
        // ---- stage 8 channels of every part: [part][ch][row]
        int colq[4];
        if (a.overlap) {
          colq[0] = c0; colq[1] = 64 + c0; colq[2] = 128 + c0; colq[3] = 192 + c0;
        } else {
          colq[0] = c0; colq[1] = c0; colq[2] = 128 + c0; colq[3] = 128 + c0;
        }
        float v[4][kFChunk];
        if (!dead) {
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint32_t r[8];
            asm volatile(
                "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
                  "=r"(r[6]), "=r"(r[7])
                : "r"(trow + colq[q]));
#pragma unroll
            for (int u = 0; u < kFChunk; ++u) v[q][u] = __uint_as_float(r[u]);
          }
          tmem_wait_ld();
        }
        named_bar(3, 128);  // the previous chunk's staged values are consumed
#pragma unroll
        for (int q = 0; q < 4; ++q)
#pragma unroll
          for (int u = 0; u < kFChunk; ++u) stg[(q * kFChunk + u) * 128 + rho] = v[q][u];
        // the token's C^a row (main channels; HCA: C) for the window rows
        const int tok = tok0 + rho;
        if (!dead && !f.indexer && rho >= lead && tok < a.T) {
          float* dst = a.Ca + ((size_t)b * a.T + tok) * a.c + f.ch0 + c0;
          *reinterpret_cast<float4*>(dst) = make_float4(v[0][0], v[0][1], v[0][2], v[0][3]);
          *reinterpret_cast<float4*>(dst + 4) = make_float4(v[0][4], v[0][5], v[0][6], v[0][7]);
        }
        named_bar(3, 128);
        if (dead) continue;
        // ---- fold
        if (a.overlap) {
          // one thread per (entry, channel): a rows lead + m u + r, b rows m u + r
          for (int it = et; it < a.E * kFChunk; it += 128) {
            const int u = it / kFChunk, ch = it % kFChunk;
            const int e = e0 + u;
            if (e >= nE) continue;
            const bool use_b = e > 0;
            const float* za = stg + (2 * kFChunk + ch) * 128 + lead + a.m * u;
            const float* zb = stg + (3 * kFChunk + ch) * 128 + a.m * u;
            const float* ca = stg + (0 * kFChunk + ch) * 128 + lead + a.m * u;
            const float* cb = stg + (1 * kFChunk + ch) * 128 + a.m * u;
            const float* ba = a.bias + bA + f.ch0 + c0 + ch;
            const float* bb = a.bias + bB + f.ch0 + c0 + ch;
            float mx = -INFINITY;
            for (int r = 0; r < a.m; ++r) {
              mx = fmaxf(mx, za[r] + ba[(size_t)r * a.nb]);
              if (use_b) mx = fmaxf(mx, zb[r] + bb[(size_t)r * a.nb]);
            }
            float den = 0.f, num = 0.f;
            for (int r = 0; r < a.m; ++r) {
              const float ea = expf(za[r] + ba[(size_t)r * a.nb] - mx);
              den += ea;
              num = fmaf(ea, ca[r], num);
              if (use_b) {
                const float eb = expf(zb[r] + bb[(size_t)r * a.nb] - mx);
                den += eb;
                num = fmaf(eb, cb[r], num);
              }
            }
            a.F[((size_t)b * nE + e) * nF + fcol + c0 + ch] = num / den;
          }
        } else {
          // m / 8 threads per (entry, channel), 8 rows each, shuffle-reduced
          const int G = a.m >= 8 ? a.m / 8 : 1;  // a power of two, <= 16
          const int per = a.m / G;
          for (int it0 = 0; it0 < a.E * kFChunk * G; it0 += 128) {
            const int it = it0 + et;
            const bool act = it < a.E * kFChunk * G;
            const int item = it / G, g = it % G;
            const int u = item / kFChunk, ch = item % kFChunk;
            const int e = e0 + u;
            const bool live = act && e < nE;
            const float* z = stg + (2 * kFChunk + ch) * 128 + a.m * u + g * per;
            const float* cv = stg + (0 * kFChunk + ch) * 128 + a.m * u + g * per;
            const float* bz = a.bias + bA + f.ch0 + c0 + ch;
            float mx = -INFINITY;
            if (live)
              for (int r = 0; r < per; ++r) mx = fmaxf(mx, z[r] + bz[(size_t)(g * per + r) * a.nb]);
            for (int o = 1; o < G; o <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
            float den = 0.f, num = 0.f;
            if (live)
              for (int r = 0; r < per; ++r) {
                const float ez = expf(z[r] + bz[(size_t)(g * per + r) * a.nb] - mx);
                den += ez;
                num = fmaf(ez, cv[r], num);
              }
            for (int o = 1; o < G; o <<= 1) {
              den += __shfl_xor_sync(0xffffffffu, den, o);
              num += __shfl_xor_sync(0xffffffffu, num, o);
            }
            if (live && g == 0) a.F[((size_t)b * nE + e) * nF + fcol + c0 + ch] = num / den;
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

// The fold epilogue covers CSA with m | 128 and m <= 64 (channels in
// blocks of 64) and HCA with m | 128 (channels in blocks of 128).
bool gemm_fold_supported(const csa_params& p, int d) {
  if (p.act != CSA_BF16 || d % 8 != 0 || !tma_available()) return false;
  if (p.m < 1 || 128 % p.m != 0) return false;
  if (p.overlap) return p.m <= 64 && p.c % 64 == 0 && p.c_I % 64 == 0 && p.c_I > 0;
  return p.c % 128 == 0;
}

size_t gemm_fold_ws_bytes(const csa_params& p, int B, int T) {
  const size_t nE = (size_t)(T / p.m);
  return align_up((size_t)B * nE * (p.c + (p.overlap ? p.c_I : 0)) * 4, 256) +
         align_up((size_t)B * T * p.c * 4, 256);
}

csa_status launch_gemm_fold(const csa_params& p, const PackLayout& L, int B, int T, int d,
                            const void* H, const void* packed, const float* bias, float* F,
                            float* Ca, cudaStream_t st) {
  CUtensorMap tmA, tmB;
  if (!make_tmap_bf16(&tmA, H, (uint64_t)B * T, (uint64_t)d, kGm)) return CSA_ERR_CUDA;
  if (!make_tmap_bf16(&tmB, packed, (uint64_t)L.ncols, (uint64_t)d, 64)) return CSA_ERR_CUDA;
  GemmFoldArgs a{};
  a.bias = bias; a.F = F; a.Ca = Ca; a.err = device_error_word();
  if (a.err == nullptr) return CSA_ERR_CUDA;
  a.B = B; a.T = T; a.m = p.m; a.overlap = p.overlap; a.c = p.c;
  a.cI = p.overlap ? p.c_I : 0; a.nb = L.nb;
  a.col_Ca = L.col_Ca; a.col_Cb = L.col_Cb; a.col_Za = L.col_Za; a.col_Zb = L.col_Zb;
  a.col_CIa = L.col_CIa; a.col_CIb = L.col_CIb; a.col_ZIa = L.col_ZIa; a.col_ZIb = L.col_ZIb;
  a.b_Ba = L.b_Ba; a.b_Bb = L.b_Bb; a.b_BIa = L.b_BIa; a.b_BIb = L.b_BIb;
  a.E = p.overlap ? (kGm - p.m) / p.m : kGm / p.m;
  const int nE = T / p.m;
  // every token row is drained as C^a once, so the tiles cover all T tokens
  const int stride = a.E * p.m;
  a.mt_per_seq = (T + stride - 1) / stride;
  if (a.mt_per_seq < 1) a.mt_per_seq = 1;
  (void)nE;
  a.nt = p.overlap ? p.c / 64 + p.c_I / 64 : p.c / 128;
  a.tiles = B * a.mt_per_seq * a.nt;
  a.K = d;
  if (!set_kernel_smem((const void*)gemm_fold_tc, kFSmem)) return CSA_ERR_CUDA;
  const int sms = sm_count();
  const int grid = a.tiles < sms ? a.tiles : sms;
  CSA_LAUNCH(KK_GEMM, st, gemm_fold_tc<<<grid, kGThreads, kFSmem, st>>>(tmA, tmB, a));
  return last_launch_status();
}

}  // namespace csa
