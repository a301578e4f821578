// append_tc.cu -- the decode-time compressor's projection on the 5th-
// generation tensor cores ("DeepSeekV4技术报告阅读笔记" eq. 9-12 and 20-23 for
// one new token per sequence; the running-softmax state of the open entries
// is the one csa_decode_append keeps, see compress.cu).
//
// D[128][16] = Wtile[128][d] . H[16][d]^T: the M side is one block of 64
// channels of one part (a or b window, main or indexer) as its 64 C rows and
// its 64 Z rows, the N side up to 16 tokens (rows past B are TMA zero fill).
// d is split over the CTAs of a cluster (one slice of k-blocks each); the
// weights stream by TMA in the 128-byte swizzle (the only HBM traffic), one
// thread issues the MMAs into a 16-column fp32 TMEM accumulator, and the
// epilogue stages it in shared memory.  The slices are summed in a fixed
// order through distributed shared memory, and each CTA of the cluster folds
// its share of the (channel, token) pairs into the state.  Every wait is
// bounded.
#include <cuda.h>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace csa {

using namespace sm100;

constexpr int kApN = 16;                    // tokens (MMA N)
constexpr int kApStages = 5;  // 101 KB of shared memory: two CTAs fit an SM
constexpr int kApA = 128 * 64 * 2;          // 16 KB: 64 C rows + 64 Z rows x 64 k
constexpr int kApB = kApN * 64 * 2;         // 2 KB: 16 token rows x 64 k
constexpr int kApStage = kApA + kApB;       // a multiple of 1024
constexpr int kApThreads = 192;             // warp 0 TMA, 1 MMA, 2-5 epilogue
constexpr int kApMaxSplit = 8;              // portable cluster size
constexpr int kApSmem = 1024 + kApStages * kApStage + 128 * kApN * 4 + 256;

struct ApArgs {
  PackLayout L;
  const float* bias;
  const int32_t* tpos;
  float* state;
  unsigned* err;
  size_t per_seq;
  int nb, KB, kbs, nsplit, m, overlap, c, cI;
};

__global__ void __launch_bounds__(kApThreads, 1)
    append_project_tc(const __grid_constant__ CUtensorMap tmW,
                      const __grid_constant__ CUtensorMap tmH, ApArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  float* dtile = (float*)(sm + kApStages * kApStage);  // [128 rows][16 tokens]
  uint64_t* bars = (uint64_t*)(dtile + 128 * kApN);
  uint64_t* full = bars;
  uint64_t* empty = bars + kApStages;
  uint64_t* tfull = bars + 2 * kApStages;
  uint32_t* tbase_sm = (uint32_t*)(tfull + 1);
  volatile int* abort_sm = (volatile int*)(tbase_sm + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int split = (int)cluster_ctarank();
  const int tile = blockIdx.x / a.nsplit;

  // tile -> part (0 a main, 1 b main, 2 a indexer, 3 b indexer) and block
  const int nbc = (a.c + 63) / 64, nbi = (a.cI + 63) / 64;
  int part, blk;
  if (tile < nbc) {
    part = 0; blk = tile;
  } else if (tile < 2 * nbc) {
    part = 1; blk = tile - nbc;
  } else if (tile < 2 * nbc + nbi) {
    part = 2; blk = tile - 2 * nbc;
  } else {
    part = 3; blk = tile - 2 * nbc - nbi;
  }
  const PackLayout& L = a.L;
  const int colC0 = part == 0 ? L.col_Ca : part == 1 ? L.col_Cb : part == 2 ? L.col_CIa : L.col_CIb;
  const int colZ0 = part == 0 ? L.col_Za : part == 1 ? L.col_Zb : part == 2 ? L.col_ZIa : L.col_ZIb;
  const int colB0 = part == 0 ? L.b_Ba : part == 1 ? L.b_Bb : part == 2 ? L.b_BIa : L.b_BIb;
  const int nchan = part < 2 ? a.c : a.cI;
  const int sch0 = part < 2 ? 0 : a.c;  // state channel of the part's channel 0
  const bool partb = part == 1 || part == 3;
  const int ch0 = blk * 64;
  const int nvalid = nchan - ch0 < 64 ? nchan - ch0 : 64;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kApStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    mbar_init(tfull, 1);
    *abort_sm = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tbase_sm, 32);
    tmem_relinquish();
  }
  if (threadIdx.x == 32) {
    prefetch_tmap(&tmW);
    prefetch_tmap(&tmH);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // launched as a programmatic dependent: the set-up above overlaps the
  // previous kernel; h and the state are touched only after this
  pdl_wait();
  const uint32_t tbase = *tbase_sm;
  const int kb0 = split * a.kbs;
  const int kb1 = kb0 + a.kbs < a.KB ? kb0 + a.kbs : a.KB;

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------------------ loads --
    const uint64_t pol = l2_evict_first_policy();  // weights are read once
    for (int kb = kb0, i = 0; kb < kb1; ++kb, ++i) {
      const int s = i % kApStages;
      if (!mbar_wait(&empty[s], ((i / kApStages) & 1) ^ 1, abort_sm)) break;
      uint8_t* st = sm + s * kApStage;
      mbar_expect_tx(&full[s], kApStage);
      tma_load_2d_hint(st, &tmW, &full[s], kb * 64, colC0 + ch0, pol);
      tma_load_2d_hint(st + kApA / 2, &tmW, &full[s], kb * 64, colZ0 + ch0, pol);
      tma_load_2d(st + kApA, &tmH, &full[s], kb * 64, 0);
    }
  } else if (warp == 1 && lane == 0) {
    // ------------------------------------------------------------- MMA --
    const uint32_t idesc = idesc_bf16(128, kApN);
    bool ok = true;
    for (int kb = kb0, i = 0; kb < kb1; ++kb, ++i) {
      const int s = i % kApStages;
      if (!mbar_wait(&full[s], (i / kApStages) & 1, abort_sm)) { ok = false; break; }
      tc_fence_after();
      const uint32_t ab = smem_u32(sm + s * kApStage), bb = ab + kApA;
#pragma unroll
      for (int j = 0; j < 4; ++j)
        mma_bf16(tbase, sdesc_k_sw128(ab + j * 32), sdesc_k_sw128(bb + j * 32), idesc,
                 (i | j) != 0);
      mma_commit(&empty[s]);
    }
    if (ok) mma_commit(tfull);
  } else if (warp >= 2) {
    // ------------------------------------------- epilogue: TMEM -> smem --
    const int quad = warp & 3;  // TMEM lanes 32 quad .. 32 quad + 31
    if (mbar_wait(tfull, 0, abort_sm)) {
      tc_fence_after();
      float v[16];
      tmem_ld16(tbase + ((uint32_t)(quad * 32) << 16), v);
      tmem_wait_ld();
      float4* dst = reinterpret_cast<float4*>(dtile + (quad * 32 + lane) * kApN);
#pragma unroll
      for (int u = 0; u < 4; ++u) dst[u] = make_float4(v[4 * u], v[4 * u + 1], v[4 * u + 2], v[4 * u + 3]);
    }
  }
  __syncwarp();
  tc_fence_before();
  cluster_sync_all();  // every slice's tile is staged
  pdl_trigger();       // the finishing kernel may start its launch

  // --------------------------- sum of the slices and the state update --
  // CTA `split` takes channels [c_lo, c_hi) of the block, all tokens
  if (!*abort_sm) {
    const int per = (64 + a.nsplit - 1) / a.nsplit;
    const int c_lo = split * per;
    const int c_hi = c_lo + per < nvalid ? c_lo + per : nvalid;
    const int nitems = c_hi > c_lo ? (c_hi - c_lo) * a.nb : 0;
    const int nch = a.c + a.cI;
    const int S = a.overlap ? 2 : 1;
    const uint32_t dbase = smem_u32(dtile);
    for (int it = threadIdx.x; it < nitems; it += kApThreads) {
      const int ch = c_lo + it / a.nb, b = it % a.nb;
      // every slice's pair is loaded first, then summed in slice order
      float cs[kApMaxSplit], zs[kApMaxSplit];
#pragma unroll
      for (int r = 0; r < kApMaxSplit; ++r) {
        cs[r] = zs[r] = 0.f;
        if (r < a.nsplit) {
          const uint32_t rb = mapa_shared(dbase, (uint32_t)r);
          cs[r] = ld_dsmem_f32(rb + (uint32_t)((ch * kApN + b) * 4));
          zs[r] = ld_dsmem_f32(rb + (uint32_t)(((64 + ch) * kApN + b) * 4));
        }
      }
      float C = 0.f, Z = 0.f;
#pragma unroll
      for (int r = 0; r < kApMaxSplit; ++r) {
        C += cs[r];
        Z += zs[r];
      }
      const int t = a.tpos[b];
      const int j = t / a.m, rr = t % a.m;
      float* st = a.state + (size_t)b * a.per_seq;
      const int gch = ch0 + ch;  // channel within the part
      if (part == 0) st[gch] = C;  // C^a_t: the window row's source
      const int entry = partb ? j + 1 : j;
      const bool fresh = rr == 0 && (partb || !a.overlap || j == 0);
      float* slot = st + a.c + (size_t)(entry % S) * 3 * nch;
      const int sch = sch0 + gch;
      running_softmax_add(slot + sch, slot + nch + sch, slot + 2 * nch + sch, C,
                          Z + a.bias[rr * L.nb + colB0 + gch], fresh);
    }
  }
  cluster_sync_all();  // no CTA leaves while its tile may still be read
  if (*abort_sm) {
    if (threadIdx.x == 0) atomicOr(a.err, CSA_DEV_TIMEOUT);
    const uint64_t t0 = globaltimer();
    while (globaltimer() - t0 < 200000ull) __nanosleep(1000);
  }
  if (warp == 1) tmem_dealloc(tbase, 32);
}

bool make_tmap_bf16(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols,
                    uint32_t box_rows);
bool tma_available();

bool append_tc_supported(const csa_params& p, int nb) {
  return p.act == CSA_BF16 && nb >= 1 && nb <= kApN && tma_available();
}

static int ap_max_active_clusters(int csize) {
  static int cache[64][kApMaxSplit + 1];
  static bool have[64][kApMaxSplit + 1];
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64 || csize < 1 || csize > kApMaxSplit) return 0;
  if (!have[dev][csize]) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(csize * 148);
    cfg.blockDim = dim3(kApThreads);
    cfg.dynamicSmemBytes = (size_t)kApSmem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)csize;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, append_project_tc, &cfg) != cudaSuccess) {
      cudaGetLastError();
      n = 0;
    }
    cache[dev][csize] = n;
    have[dev][csize] = true;
  }
  return cache[dev][csize];
}

csa_status launch_append_project_tc(const csa_params& p, const PackLayout& L, int nb, int d,
                                    const void* H, const void* packed, const float* bias,
                                    const int32_t* t, float* state, int cI, size_t per_seq,
                                    cudaStream_t st) {
  CUtensorMap tmW, tmH;
  if (!make_tmap_bf16(&tmW, packed, (uint64_t)L.ncols, (uint64_t)d, 64)) return CSA_ERR_CUDA;
  if (!make_tmap_bf16(&tmH, H, (uint64_t)nb, (uint64_t)d, kApN)) return CSA_ERR_CUDA;
  if (!set_kernel_smem((const void*)append_project_tc, kApSmem)) return CSA_ERR_CUDA;
  ApArgs a;
  a.L = L;
  a.bias = bias;
  a.tpos = t;
  a.state = state;
  a.err = device_error_word();
  if (a.err == nullptr) return CSA_ERR_CUDA;
  a.per_seq = per_seq;
  a.nb = nb;
  a.m = p.m;
  a.overlap = p.overlap;
  a.c = p.c;
  a.cI = p.overlap ? cI : 0;
  const int nbc = (p.c + 63) / 64, nbi = (a.cI + 63) / 64;
  const int tiles = p.overlap ? 2 * nbc + 2 * nbi : nbc;
  a.KB = (d + 63) / 64;
  // slices of d: at most one CTA per SM (a second CTA on a few SMs would
  // make them the last to finish), at most a cluster of 8, no empty slice
  const int sms = sm_count();
  int ns = sms / tiles;
  if (ns > kApMaxSplit) ns = kApMaxSplit;
  if (ns > a.KB) ns = a.KB;
  if (ns < 1) ns = 1;
  while (ns > 1 && ap_max_active_clusters(ns) < 1) --ns;
  a.kbs = (a.KB + ns - 1) / ns;
  a.nsplit = (a.KB + a.kbs - 1) / a.kbs;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(tiles * a.nsplit);
  cfg.blockDim = dim3(kApThreads);
  cfg.dynamicSmemBytes = (size_t)kApSmem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)a.nsplit;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cudaLaunchAttribute attrs[2] = {attr[0], {}};
  attrs[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attrs[1].val.programmaticStreamSerializationAllowed = kPdlAppend ? 1 : 0;
  cfg.attrs = attrs;
  cfg.numAttrs = 2;
  CSA_LAUNCH(KK_GEMM, st, cudaLaunchKernelEx(&cfg, append_project_tc, tmW, tmH, a));
  return last_launch_status();
}

}  // namespace csa
