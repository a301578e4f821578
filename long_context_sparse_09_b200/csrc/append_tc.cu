// append_tc.cu -- projections of a few tokens on the 5th-generation tensor
// cores: the decode-time compressor's ("DeepSeekV4技术报告阅读笔记" eq. 9-12
// and 20-23 for one new token per sequence; the running-softmax state of the
// open entries is the one csa_decode_append keeps, see compress.cu) and the
// grouped output projection (same notes 2.3.3; PaperTrace 2.2).
//
// D[128][16] = Wtile[128][d] . H[16][d]^T: the M side is one block of 64
// channels of one part (a or b window, main or indexer) as its 64 C rows and
// its 64 Z rows, the N side up to 16 tokens (rows past B are TMA zero fill).
// d is split over the CTAs of a cluster (one slice of k-blocks each); the
// weights stream by TMA in the 128-byte swizzle (the only HBM traffic), one
// thread issues the MMAs into a 16-column fp32 TMEM accumulator, and the
// epilogue stages it in shared memory.  The slices are summed in a fixed
// order through distributed shared memory, and each CTA of the cluster folds
// its share of the (channel, token) pairs into the state.  The output
// projection uses the same body with 128 consecutive output features as M
// and a plain bf16 store of its share of the (feature, token) pairs.  Every
// wait is bounded.
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
constexpr int kApPrefetch = 16;             // k-blocks a CTA pulls into L2 up front
constexpr int kApSmem = 1024 + kApStages * kApStage + 128 * kApN * 4 + 256;

struct ApArgs {
  PackLayout L;
  const uint8_t* dec = nullptr;  // tile-major weight blocks (compressor), or null
  const float* bias;
  const int32_t* tpos;
  float* state;
  unsigned* err;
  size_t per_seq;
  int nb, KB, kbs, nsplit, m, overlap, c, cI;
  // plain-store form: features f < fsplit go to out[b * ld_out + f],
  // features fsplit <= f < nfeat to out2[b * ld_out2 + f - fsplit], each as
  // bf16 or, with out_f32 / out2_f32 set, as fp32; the tile of features
  // f0.. reads the tokens' columns from (f0 / rows_per_group) * x_per_group on
  void* out;
  void* out2;
  int ld_out, ld_out2, fsplit, out_f32, out2_f32;
  int nfeat, rows_per_group, x_per_group;
};

// The compressor tile `tile` (64 channels of one part: 0 a main, 1 b main,
// 2 a indexer, 3 b indexer) -> its first C row and first Z row in the packed
// [ncols][d] weights, the part, its first channel and its valid channels.
struct ApTile {
  int rowA0, rowB0, part, ch0, nvalid;
};
__host__ __device__ inline ApTile ap_tile(const PackLayout& L, int c, int cI, int tile) {
  const int nbc = (c + 63) / 64, nbi = (cI + 63) / 64;
  ApTile t;
  int blk;
  if (tile < nbc) {
    t.part = 0; blk = tile;
  } else if (tile < 2 * nbc) {
    t.part = 1; blk = tile - nbc;
  } else if (tile < 2 * nbc + nbi) {
    t.part = 2; blk = tile - 2 * nbc;
  } else {
    t.part = 3; blk = tile - 2 * nbc - nbi;
  }
  const int colC0 = t.part == 0 ? L.col_Ca : t.part == 1 ? L.col_Cb : t.part == 2 ? L.col_CIa : L.col_CIb;
  const int colZ0 = t.part == 0 ? L.col_Za : t.part == 1 ? L.col_Zb : t.part == 2 ? L.col_ZIa : L.col_ZIb;
  const int nchan = t.part < 2 ? c : cI;
  t.ch0 = blk * 64;
  t.nvalid = nchan - t.ch0 < 64 ? nchan - t.ch0 : 64;
  t.rowA0 = colC0 + t.ch0;
  t.rowB0 = colZ0 + t.ch0;
  return t;
}

__device__ __forceinline__ void store_feature(void* base, int f32, size_t i, float v) {
  if (f32)
    reinterpret_cast<float*>(base)[i] = v;
  else
    reinterpret_cast<__nv_bfloat16*>(base)[i] = __float2bfloat16_rn(v);
}

// kMode 0: the compressor projection and state update; 1: a plain store.
template <int kMode>
__device__ __forceinline__ void skinny_body(const CUtensorMap* tmW, const CUtensorMap* tmH,
                                            const ApArgs& a) {
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

  // tile -> the two 64-row boxes of weights, the tokens' column offset and,
  // for the compressor, part (0 a main, 1 b main, 2 a indexer, 3 b indexer)
  int rowA0, rowB0, xoff = 0;
  int part = 0, colB0 = 0, nvalid = 128, sch0 = 0, ch0 = 0;
  bool partb = false;
  const PackLayout& L = a.L;
  if constexpr (kMode == 0) {
    const ApTile tt = ap_tile(L, a.c, a.cI, tile);
    part = tt.part;
    colB0 = part == 0 ? L.b_Ba : part == 1 ? L.b_Bb : part == 2 ? L.b_BIa : L.b_BIb;
    sch0 = part < 2 ? 0 : a.c;  // state channel of the part's channel 0
    partb = part == 1 || part == 3;
    ch0 = tt.ch0;
    nvalid = tt.nvalid;
    rowA0 = tt.rowA0;
    rowB0 = tt.rowB0;
  } else {
    const int f0 = tile * 128;
    rowA0 = f0;
    rowB0 = f0 + 64;
    xoff = (f0 / a.rows_per_group) * a.x_per_group;
    nvalid = a.nfeat - f0 < 128 ? a.nfeat - f0 : 128;
  }

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
    prefetch_tmap(tmW);
    prefetch_tmap(tmH);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const int kb0 = split * a.kbs;
  const int kb1 = kb0 + a.kbs < a.KB ? kb0 + a.kbs : a.KB;
  if (kMode == 0 && threadIdx.x == 0 && a.dec != nullptr) {
    // The weights do not come from the previous kernel: the first k-blocks
    // of this CTA's range are pulled into L2 while it finishes (a prefetch
    // only fills L2, where later writes would land anyway).  The plain-store
    // form streams more weights than L2 holds and does not prefetch.
    const int npre = kb1 - kb0 < kApPrefetch ? kb1 - kb0 : kApPrefetch;
    for (int i = 0; i < npre; ++i)
      bulk_prefetch_l2(a.dec + ((size_t)tile * a.KB + kb0 + i) * kApA, kApA);
  }
  // launched as a programmatic dependent: the set-up above overlaps the
  // previous kernel; h and the state are touched only after this
  pdl_wait();
  const uint32_t tbase = *tbase_sm;

  // Items of the state update: the (channel, token) pairs of this CTA's
  // share of the block, handed out from thread 64 on so that the two
  // issuing lanes take none while there are at most 128.  Each epilogue
  // thread loads its first item's position, bias and state while the
  // weights stream.
  int c_lo = 0, nitems = 0;
  if (kMode == 0) {
    const int per = (64 + a.nsplit - 1) / a.nsplit;
    c_lo = split * per;
    const int c_hi = c_lo + per < nvalid ? c_lo + per : nvalid;
    nitems = c_hi > c_lo ? (c_hi - c_lo) * a.nb : 0;
  }
  const int me = (threadIdx.x + 128) % kApThreads;
  const int nch = a.c + a.cI;
  const int S = a.overlap ? 2 : 1;
  // state of item `it`: its slot triple, bias and whether it starts the entry
  struct ApItem {
    float* slot;  // running max; denominator at + nch, weighted sum at + 2 nch
    float* src;   // C^a_t of the window row (part a main), else null
    float mx, den, num, zb;
    bool fresh;
  };
  auto item_state = [&](int it) {
    ApItem q;
    const int ch = c_lo + it / a.nb, b = it % a.nb;
    const int t = a.tpos[b];
    const int j = t / a.m, rr = t % a.m;
    float* st = a.state + (size_t)b * a.per_seq;
    const int gch = ch0 + ch;  // channel within the part
    q.src = part == 0 ? st + gch : nullptr;
    const int entry = partb ? j + 1 : j;
    q.fresh = rr == 0 && (partb || !a.overlap || j == 0);
    q.slot = st + a.c + (size_t)(entry % S) * 3 * nch + sch0 + gch;
    q.zb = a.bias[rr * L.nb + colB0 + gch];
    q.mx = q.den = q.num = 0.f;
    if (!q.fresh) {
      q.mx = q.slot[0];
      q.den = q.slot[nch];
      q.num = q.slot[2 * nch];
    }
    return q;
  };
  ApItem pre{};
  const bool have_pre = kMode == 0 && warp >= 2 && me < nitems;
  if (have_pre) pre = item_state(me);

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------------------ loads --
    const uint64_t pol = l2_evict_first_policy();  // weights are read once
    for (int kb = kb0, i = 0; kb < kb1; ++kb, ++i) {
      const int s = i % kApStages;
      if (!mbar_wait(&empty[s], ((i / kApStages) & 1) ^ 1, abort_sm)) break;
      uint8_t* st = sm + s * kApStage;
      mbar_expect_tx(&full[s], kApStage);
      if (kMode == 0 && a.dec != nullptr) {  // one contiguous pre-swizzled block
        bulk_load_hint(st, a.dec + ((size_t)tile * a.KB + kb) * kApA, kApA, &full[s], pol);
      } else {
        tma_load_2d_hint(st, tmW, &full[s], kb * 64, rowA0, pol);
        tma_load_2d_hint(st + kApA / 2, tmW, &full[s], kb * 64, rowB0, pol);
      }
      tma_load_2d(st + kApA, tmH, &full[s], xoff + kb * 64, 0);
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
    if (__all_sync(0xffffffffu, mbar_wait(tfull, 0, abort_sm))) {  // warp-uniform: tcgen05.ld follows
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
  if (kMode == 0 && !*abort_sm) {
    const uint32_t dbase = smem_u32(dtile);
    for (int it = me; it < nitems; it += kApThreads) {
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
      const ApItem q = (it == me && have_pre) ? pre : item_state(it);
      if (q.src != nullptr) *q.src = C;  // C^a_t: the window row's source
      float mx = q.mx, den = q.den, num = q.num;
      running_softmax_step(mx, den, num, C, Z + q.zb, q.fresh);
      q.slot[0] = mx;
      q.slot[nch] = den;
      q.slot[2 * nch] = num;
    }
  }
  // ------------------------------ sum of the slices and the plain store --
  // CTA `split` takes rows [r_lo, r_hi) of the tile, all tokens
  if (kMode == 1 && !*abort_sm) {
    const int per = (128 + a.nsplit - 1) / a.nsplit;
    const int r_lo = split * per;
    const int r_hi = r_lo + per < nvalid ? r_lo + per : nvalid;
    const int nitems = r_hi > r_lo ? (r_hi - r_lo) * a.nb : 0;
    const uint32_t dbase = smem_u32(dtile);
    for (int it = threadIdx.x; it < nitems; it += kApThreads) {
      const int row = r_lo + it / a.nb, b = it % a.nb;
      float vs[kApMaxSplit];
#pragma unroll
      for (int r = 0; r < kApMaxSplit; ++r)
        vs[r] = r < a.nsplit
                    ? ld_dsmem_f32(mapa_shared(dbase, (uint32_t)r) + (uint32_t)((row * kApN + b) * 4))
                    : 0.f;
      float v = 0.f;
#pragma unroll
      for (int r = 0; r < kApMaxSplit; ++r) v += vs[r];
      const int f = tile * 128 + row;
      if (f < a.fsplit)
        store_feature(a.out, a.out_f32, (size_t)b * a.ld_out + f, v);
      else
        store_feature(a.out2, a.out2_f32, (size_t)b * a.ld_out2 + (f - a.fsplit), v);
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

__global__ void __launch_bounds__(kApThreads, 1)
    append_project_tc(const __grid_constant__ CUtensorMap tmW,
                      const __grid_constant__ CUtensorMap tmH, ApArgs a) {
  skinny_body<0>(&tmW, &tmH, a);
}

__global__ void __launch_bounds__(kApThreads, 1)
    out_proj_tc(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                ApArgs a) {
  skinny_body<1>(&tmW, &tmX, a);
}

bool make_tmap_bf16(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols,
                    uint32_t box_rows);
bool tma_available();

bool append_tc_supported(const csa_params& p, int nb) {
  return p.act == CSA_BF16 && nb >= 1 && nb <= kApN && tma_available();
}

// kern 0: append_project_tc, 1: out_proj_tc (same resources)
static int ap_max_active_clusters(int csize, int kern = 0) {
  static int cache[64][2][kApMaxSplit + 1];
  static bool have[64][2][kApMaxSplit + 1];
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64 || csize < 1 || csize > kApMaxSplit) return 0;
  if (!have[dev][kern][csize]) {
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
    const cudaError_t e = kern == 0 ? cudaOccupancyMaxActiveClusters(&n, append_project_tc, &cfg)
                                    : cudaOccupancyMaxActiveClusters(&n, out_proj_tc, &cfg);
    if (e != cudaSuccess) {
      cudaGetLastError();
      n = 0;
    }
    cache[dev][kern][csize] = n;
    have[dev][kern][csize] = true;
  }
  return cache[dev][kern][csize];
}

// slices of d for `tiles` output tiles and KB k-blocks: at most one CTA per
// SM, at most a cluster of 8, no empty slice; sets a.kbs and a.nsplit
static void plan_slices(ApArgs& a, int tiles, int kern) {
  const int sms = sm_count();
  int ns = sms / tiles;
  if (ns > kApMaxSplit) ns = kApMaxSplit;
  if (ns > a.KB) ns = a.KB;
  if (ns < 1) ns = 1;
  while (ns > 1 && ap_max_active_clusters(ns, kern) < 1) --ns;
  a.kbs = (a.KB + ns - 1) / ns;
  a.nsplit = (a.KB + a.kbs - 1) / a.kbs;
}

template <typename Kern>
static csa_status launch_skinny(Kern kern, int tiles, const CUtensorMap& tmW,
                                const CUtensorMap& tmX, const ApArgs& a, cudaStream_t st) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(tiles * a.nsplit);
  cfg.blockDim = dim3(kApThreads);
  cfg.dynamicSmemBytes = (size_t)kApSmem;
  cfg.stream = st;
  cudaLaunchAttribute attrs[2];
  attrs[0].id = cudaLaunchAttributeClusterDimension;
  attrs[0].val.clusterDim.x = (unsigned)a.nsplit;
  attrs[0].val.clusterDim.y = 1;
  attrs[0].val.clusterDim.z = 1;
  attrs[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attrs[1].val.programmaticStreamSerializationAllowed = kPdlAppend ? 1 : 0;
  cfg.attrs = attrs;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kern, tmW, tmX, a) == cudaSuccess ? CSA_OK : CSA_ERR_CUDA;
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
  a.dec = nullptr;  // set below once the tile count is known
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
  if (L.dec_tiles == tiles && L.dec_kb == a.KB)
    a.dec = (const uint8_t*)packed + L.dec_off;
  // (a second CTA on a few SMs would make them the last to finish)
  plan_slices(a, tiles, 0);
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

// One 16 KB block per (tile, k-block), block index tile * KB + kb: the
// tile's 64 C rows, then its 64 Z rows, columns 64 kb .. 64 kb + 63, laid out
// as the 128-byte swizzle puts them in shared memory (row r's 16-byte chunk j
// at 128 r + 16 (j ^ r % 8)), so that one bulk copy fills a stage.  Channels
// past the part's end and columns past d are zero.
__global__ void __launch_bounds__(256) pack_dec_tiles(const __nv_bfloat16* __restrict__ W,
                                                      int d, int ncols, PackLayout L, int c,
                                                      int cI, int KB, uint8_t* __restrict__ dst) {
  const int tile = blockIdx.x / KB, kb = blockIdx.x % KB;
  const ApTile tt = ap_tile(L, c, cI, tile);
  uint8_t* blk = dst + (size_t)blockIdx.x * kDecBlockBytes;
  const unsigned short* Wb = reinterpret_cast<const unsigned short*>(W);
  for (int i = threadIdx.x; i < 1024; i += blockDim.x) {
    const int r = i >> 3, j = i & 7, rr = r & 63;
    const int row = (r < 64 ? tt.rowA0 : tt.rowB0) + rr;
    const int k0 = kb * 64 + j * 8;
    uint32_t v[4] = {0u, 0u, 0u, 0u};
    if (rr < tt.nvalid && row < ncols) {
      const unsigned short* src = Wb + (size_t)row * d;
#pragma unroll
      for (int e = 0; e < 8; ++e)
        if (k0 + e < d) v[e >> 1] |= (uint32_t)src[k0 + e] << (16 * (e & 1));
    }
    *reinterpret_cast<uint4*>(blk + r * 128 + ((j ^ (r & 7)) << 4)) =
        make_uint4(v[0], v[1], v[2], v[3]);
  }
}

csa_status launch_pack_dec_tiles(const csa_params& p, const PackLayout& L, int d, void* packed,
                                 cudaStream_t st) {
  if (p.act != CSA_BF16 || L.dec_tiles <= 0) return CSA_OK;
  const int cI = p.overlap ? p.c_I : 0;
  CSA_LAUNCH(KK_PACK, st,
             pack_dec_tiles<<<L.dec_tiles * L.dec_kb, 256, 0, st>>>(
                 (const __nv_bfloat16*)packed, d, L.ncols, L, p.c, cI, L.dec_kb,
                 (uint8_t*)packed + L.dec_off));
  return last_launch_status();
}

// ------------------------------------------- grouped output projection --
// Packed weights: W^G transposed to K-major rows ([g d_g][c n_h / g]: row
// i d_g + j is column j of W^G_i), then, 256-byte aligned, W^O transposed
// ([d][g d_g]).

static size_t op_wo_offset(int n_h, int c, int g, int d_g) {
  return align_up((size_t)g * d_g * (size_t)(c * (n_h / g)) * 2, 256);
}

size_t out_proj_packed_bytes(int n_h, int c, int g, int d_g, int d) {
  return op_wo_offset(n_h, c, g, d_g) + align_up((size_t)d * g * d_g * 2, 256);
}

size_t out_proj_ws_bytes(int R, int g, int d_g) {
  return align_up((size_t)R * g * d_g * 2, 256);
}

// dst[(row0 + j) * K + k] = src[k * width + j] for k < K, j < width (a
// 32 x 32-tiled transpose of one row-major [K][width] matrix)
__global__ void transpose_bf16(const __nv_bfloat16* __restrict__ src, int K, int width,
                               __nv_bfloat16* __restrict__ dst, size_t row0) {
  __shared__ __nv_bfloat16 tile[32][33];
  const int k0 = blockIdx.y * 32, j0 = blockIdx.x * 32;
  for (int r = threadIdx.y; r < 32; r += 8) {
    const int k = k0 + r, j = j0 + threadIdx.x;
    if (k < K && j < width) tile[r][threadIdx.x] = src[(size_t)k * width + j];
  }
  __syncthreads();
  for (int r = threadIdx.y; r < 32; r += 8) {
    const int j = j0 + r, k = k0 + threadIdx.x;
    if (k < K && j < width) dst[(row0 + j) * (size_t)K + k] = tile[threadIdx.x][r];
  }
}

csa_status launch_out_proj_pack(int n_h, int c, int g, int d_g, int d, const void* WG,
                                const void* WO, void* packed, cudaStream_t st) {
  const int Kg = c * (n_h / g);
  __nv_bfloat16* dst = (__nv_bfloat16*)packed;
  const __nv_bfloat16* wg = (const __nv_bfloat16*)WG;
  for (int i = 0; i < g; ++i) {
    const dim3 grid((d_g + 31) / 32, (Kg + 31) / 32);
    CSA_LAUNCH(KK_GEMM, st, transpose_bf16<<<grid, dim3(32, 8), 0, st>>>(
        wg + (size_t)i * Kg * d_g, Kg, d_g, dst, (size_t)i * d_g));
  }
  __nv_bfloat16* wo = (__nv_bfloat16*)((char*)packed + op_wo_offset(n_h, c, g, d_g));
  const dim3 grid((d + 31) / 32, (g * d_g + 31) / 32);
  CSA_LAUNCH(KK_GEMM, st, transpose_bf16<<<grid, dim3(32, 8), 0, st>>>(
      (const __nv_bfloat16*)WO, g * d_g, d, wo, 0));
  return last_launch_status();
}

// Y = group products of O (bf16), out = Y W^O, 16 tokens a pair of launches
csa_status launch_out_proj(int R, int n_h, int c, int g, int d_g, int d, const void* O,
                           const void* packed, void* out, void* ws, cudaStream_t st) {
  if (!tma_available()) return CSA_ERR_UNSUPPORTED;
  if (!set_kernel_smem((const void*)out_proj_tc, kApSmem)) return CSA_ERR_CUDA;
  unsigned* err = device_error_word();
  if (err == nullptr) return CSA_ERR_CUDA;
  const int Kg = c * (n_h / g), GD = g * d_g;
  const __nv_bfloat16* o = (const __nv_bfloat16*)O;
  const __nv_bfloat16* wg = (const __nv_bfloat16*)packed;
  const __nv_bfloat16* wo =
      (const __nv_bfloat16*)((const char*)packed + op_wo_offset(n_h, c, g, d_g));
  __nv_bfloat16* y = (__nv_bfloat16*)ws;
  __nv_bfloat16* res = (__nv_bfloat16*)out;
  for (int b0 = 0; b0 < R; b0 += kApN) {
    const int nb = R - b0 < kApN ? R - b0 : kApN;
    ApArgs a = {};
    a.err = err;
    a.nb = nb;
    // group products: features i d_g + j read the tokens' columns i Kg..
    CUtensorMap tmW, tmX;
    if (!make_tmap_bf16(&tmW, wg, (uint64_t)GD, (uint64_t)Kg, 64)) return CSA_ERR_CUDA;
    if (!make_tmap_bf16(&tmX, o + (size_t)b0 * n_h * c, (uint64_t)nb, (uint64_t)n_h * c, kApN))
      return CSA_ERR_CUDA;
    a.out = y + (size_t)b0 * GD;
    a.ld_out = GD;
    a.nfeat = GD;
    a.fsplit = GD;
    a.rows_per_group = d_g;
    a.x_per_group = Kg;
    a.KB = Kg / 64;
    const int tiles1 = GD / 128;
    plan_slices(a, tiles1, 1);
    csa_status s;
    CSA_LAUNCH(KK_GEMM, st, s = launch_skinny(out_proj_tc, tiles1, tmW, tmX, a, st));
    if (s != CSA_OK) return s;
    // the output projection of the (bf16) group outputs
    if (!make_tmap_bf16(&tmW, wo, (uint64_t)d, (uint64_t)GD, 64)) return CSA_ERR_CUDA;
    if (!make_tmap_bf16(&tmX, y + (size_t)b0 * GD, (uint64_t)nb, (uint64_t)GD, kApN))
      return CSA_ERR_CUDA;
    a.out = res + (size_t)b0 * d;
    a.ld_out = d;
    a.nfeat = d;
    a.fsplit = d;
    a.rows_per_group = 1 << 30;  // one group
    a.x_per_group = 0;
    a.KB = (GD + 63) / 64;
    const int tiles2 = (d + 127) / 128;
    plan_slices(a, tiles2, 1);
    CSA_LAUNCH(KK_GEMM, st, s = launch_skinny(out_proj_tc, tiles2, tmW, tmX, a, st));
    if (s != CSA_OK) return s;
  }
  return last_launch_status();
}

// ------------------------------------------------ query-side projections --
// "DeepSeekV4技术报告阅读笔记" eq. 13-15 and 18, 2.5.1-2.5.2.  Packed weights:
// stage 1 K-major rows [d_c + n_hI][d] (W^{DQ} transposed, then W^w
// transposed), then, 256-byte aligned, stage 2 K-major rows
// [n_h c + n_hI c_I][d_c] (W^{UQ} transposed, then W^{IUQ} transposed).
// Each stage's rows are padded with zero rows to a multiple of 128, so that
// every 64-row weight box lies inside its tensor map.

struct QpLayout {
  size_t off2 = 0, total = 0;
  int n1 = 0, n2 = 0;    // features of the two stages
  int n1p = 0, n2p = 0;  // rows after padding
};

static QpLayout qp_layout(const csa_params& p, int d, int d_c) {
  QpLayout L;
  L.n1 = d_c + p.n_hI;
  L.n2 = p.n_h * p.c + p.n_hI * p.c_I;
  L.n1p = (int)align_up((size_t)L.n1, 128);
  L.n2p = (int)align_up((size_t)L.n2, 128);
  L.off2 = align_up((size_t)L.n1p * d * 2, 256);
  L.total = L.off2 + align_up((size_t)L.n2p * d_c * 2, 256);
  return L;
}

size_t query_proj_packed_bytes(const csa_params& p, int d, int d_c) {
  return qp_layout(p, d, d_c).total;
}

size_t query_proj_ws_bytes(const csa_params& p, int R) {
  return align_up((size_t)R * p.n_h * p.c * 4, 256);
}

csa_status launch_query_proj_pack(const csa_params& p, int d, int d_c, const void* WDQ,
                                  const void* Ww, const void* WUQ, const void* WIUQ,
                                  void* packed, cudaStream_t st) {
  const QpLayout L = qp_layout(p, d, d_c);
  __nv_bfloat16* s1 = (__nv_bfloat16*)packed;
  __nv_bfloat16* s2 = (__nv_bfloat16*)((char*)packed + L.off2);
  auto tr = [&](const void* src, int K, int width, __nv_bfloat16* dst, size_t row0) {
    const dim3 grid((width + 31) / 32, (K + 31) / 32);
    CSA_LAUNCH(KK_GEMM, st, transpose_bf16<<<grid, dim3(32, 8), 0, st>>>(
        (const __nv_bfloat16*)src, K, width, dst, row0));
  };
  if (cudaMemsetAsync(packed, 0, L.total, st) != cudaSuccess) return CSA_ERR_CUDA;  // pad rows
  tr(WDQ, d, d_c, s1, 0);
  tr(Ww, d, p.n_hI, s1, (size_t)d_c);
  tr(WUQ, d_c, p.n_h * p.c, s2, 0);
  tr(WIUQ, d_c, p.n_hI * p.c_I, s2, (size_t)p.n_h * p.c);
  return last_launch_status();
}

// Per (token, head) of q: RMSNorm over the c values (unit gain, 2.5.1) and
// RoPE at the token's position on the last rope_dims (interleaved pairs,
// 2.5.2), stored as bf16.  One warp per (token, head).
__global__ void __launch_bounds__(256) query_finish(const float* __restrict__ qraw,
                                                    const int32_t* __restrict__ pos, int R,
                                                    int n_h, int c, int rope_dims, float eps,
                                                    double base,
                                                    __nv_bfloat16* __restrict__ q) {
  pdl_wait();
  const int warp = (int)((blockIdx.x * (size_t)blockDim.x + threadIdx.x) >> 5);
  const int lane = threadIdx.x & 31;
  if (warp >= R * n_h) return;
  const int r = warp / n_h;
  const float* x = qraw + (size_t)warp * c;
  float ss = 0.f;
  for (int j = lane * 4; j < c; j += 128) {
    const float4 v = *reinterpret_cast<const float4*>(x + j);
    ss = fmaf(v.x, v.x, fmaf(v.y, v.y, fmaf(v.z, v.z, fmaf(v.w, v.w, ss))));
  }
  ss = warp_sum(ss);
  const float inv = rsqrtf(ss / (float)c + eps);
  const int r0 = c - rope_dims;
  const double t = (double)pos[r];
  __nv_bfloat16* out = q + (size_t)warp * c;
  for (int j = lane * 2; j < c; j += 64) {
    float a = x[j] * inv, b = x[j + 1] * inv;
    if (j >= r0) {
      float cs, sn;
      rope_cs(t, (j - r0) >> 1, rope_dims, base, &cs, &sn);
      const float a2 = a * cs - b * sn, b2 = a * sn + b * cs;
      a = a2;
      b = b2;
    }
    *reinterpret_cast<__nv_bfloat162*>(out + j) = __floats2bfloat162_rn(a, b);
  }
}

// c^Q, w (stage 1) and q, q^I (stage 2 and the finish), 16 tokens a triple
// of launches
csa_status launch_query_proj(const csa_params& p, int R, int d, int d_c, const void* H,
                             const int32_t* pos, const void* packed, void* cQ, void* q,
                             void* qI, float* w, void* ws, cudaStream_t st) {
  if (!tma_available()) return CSA_ERR_UNSUPPORTED;
  if (!set_kernel_smem((const void*)out_proj_tc, kApSmem)) return CSA_ERR_CUDA;
  unsigned* err = device_error_word();
  if (err == nullptr) return CSA_ERR_CUDA;
  const QpLayout L = qp_layout(p, d, d_c);
  const __nv_bfloat16* w1 = (const __nv_bfloat16*)packed;
  const __nv_bfloat16* w2 = (const __nv_bfloat16*)((const char*)packed + L.off2);
  const __nv_bfloat16* h = (const __nv_bfloat16*)H;
  __nv_bfloat16* cq = (__nv_bfloat16*)cQ;
  float* qraw = (float*)ws;
  const int nq = p.n_h * p.c;
  for (int b0 = 0; b0 < R; b0 += kApN) {
    const int nb = R - b0 < kApN ? R - b0 : kApN;
    ApArgs a = {};
    a.err = err;
    a.nb = nb;
    a.rows_per_group = 1 << 30;  // one group: every tile reads the tokens from column 0
    CUtensorMap tmW, tmX;
    // stage 1: [c^Q | w] = h [W^{DQ} | W^w]
    if (!make_tmap_bf16(&tmW, w1, (uint64_t)L.n1p, (uint64_t)d, 64)) return CSA_ERR_CUDA;
    if (!make_tmap_bf16(&tmX, h + (size_t)b0 * d, (uint64_t)nb, (uint64_t)d, kApN))
      return CSA_ERR_CUDA;
    a.out = cq + (size_t)b0 * d_c;
    a.ld_out = d_c;
    a.out_f32 = 0;
    a.out2 = w + (size_t)b0 * p.n_hI;
    a.ld_out2 = p.n_hI;
    a.out2_f32 = 1;
    a.fsplit = d_c;
    a.nfeat = L.n1;
    a.KB = d / 64;
    const int tiles1 = (L.n1 + 127) / 128;
    plan_slices(a, tiles1, 1);
    csa_status s;
    CSA_LAUNCH(KK_GEMM, st, s = launch_skinny(out_proj_tc, tiles1, tmW, tmX, a, st));
    if (s != CSA_OK) return s;
    // stage 2: [q (fp32, before the norm) | q^I] = c^Q [W^{UQ} | W^{IUQ}]
    if (!make_tmap_bf16(&tmW, w2, (uint64_t)L.n2p, (uint64_t)d_c, 64)) return CSA_ERR_CUDA;
    if (!make_tmap_bf16(&tmX, cq + (size_t)b0 * d_c, (uint64_t)nb, (uint64_t)d_c, kApN))
      return CSA_ERR_CUDA;
    a.out = qraw + (size_t)b0 * nq;
    a.ld_out = nq;
    a.out_f32 = 1;
    a.out2 = (__nv_bfloat16*)qI + (size_t)b0 * p.n_hI * p.c_I;
    a.ld_out2 = p.n_hI * p.c_I;
    a.out2_f32 = 0;
    a.fsplit = nq;
    a.nfeat = L.n2;
    a.KB = d_c / 64;
    const int tiles2 = (L.n2 + 127) / 128;
    plan_slices(a, tiles2, 1);
    CSA_LAUNCH(KK_GEMM, st, s = launch_skinny(out_proj_tc, tiles2, tmW, tmX, a, st));
    if (s != CSA_OK) return s;
    // per-head RMSNorm and RoPE of q
    const int warps = nb * p.n_h;
    cudaError_t e = cudaSuccess;
    CSA_LAUNCH(KK_FOLD, st,
               e = launch_maybe_pdl(kPdlAppend, query_finish, dim3((warps + 7) / 8), dim3(256),
                                    (size_t)0, st, (const float*)(qraw + (size_t)b0 * nq),
                                    pos + b0, nb, p.n_h, p.c, p.rope_dims, p.rms_eps,
                                    (double)p.rope_base,
                                    (__nv_bfloat16*)q + (size_t)b0 * nq));
    if (e != cudaSuccess) return CSA_ERR_CUDA;
  }
  return last_launch_status();
}

}  // namespace csa
