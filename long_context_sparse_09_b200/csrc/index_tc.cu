// index_tc.cu -- Lightning-Indexer scores on the 5th-generation tensor cores
// ("DeepSeekV4技术报告阅读笔记" eq. 16; "02 · DeepSeek-V4: 压缩注意力撑起 1M 上下文"
// section 2.2).
//
// One product per (entry tile, query group): D[128 entries][G*n_hI] =
// K^I_tile[128][c_I] * Q_group[G*n_hI][c_I]^T, bf16 in, fp32 in TMEM.  The
// entries are the MMA's M dimension so that each TMEM lane -- one epilogue
// thread -- holds one entry's dot products with every head of the group's
// queries; ReLU, the head weights w and the sum over heads then run in
// registers with no cross-thread reduction.
//
// Warp roles (per CTA): warp 0 issues TMA loads of K^I tiles (and of the
// query group's q^I when it changes), warp 1 allocates TMEM and issues the
// MMAs, the remaining warps drain TMEM, apply the score epilogue and store
// fp32 scores.  K^I tiles go through a ring of smem stages, accumulators
// through two TMEM buffers, so loads, MMAs and epilogues overlap.  Every
// wait is bounded; a timeout sets CSA_DEV_TIMEOUT and the CTA winds down.
//
// Work: the flat list of (query group, entry tile) pairs over each group's
// visible tiles (a plan kernel computes per-group tile counts and their
// prefix sum on the device), split evenly over a persistent grid.
#include <cuda.h>

#include <algorithm>

#include "common.cuh"
#include "index_common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace csa {

using namespace sm100;

struct IdxTcArgs {
  const int32_t* q_pos;
  const float* w;
  const int* prefix;  // [ngroups + 1] exclusive prefix of tiles per group, or null:
                      // each CTA computes it (ngroups <= kInlineGroups)
  float* scores;      // [R][N]
  unsigned* err;
  unsigned* ghist;    // [R][4096] key histograms for the top-k (G == 1), or null
  int Q, N, m, nhI, ngroups;
  int stream_keys;    // every key tile is read by one group only: read it evict-first
};

constexpr int kMaxAcc = 8;  // TMEM accumulator ring depth (bounded by 512 columns)
constexpr int kKBlockBytes = kTileM * 128;  // 128 rows x 64 bf16

template <int G, int KB, int S, int NE, int NQ = 2>
struct IdxTcCfg {
  static constexpr int kStageBytes = KB * kKBlockBytes;
  static constexpr int kThreads = 64 + 32 * NE;
};

// Per-group visible tile counts and their exclusive prefix (CTA 0), and
// zeroing of the top-k bookkeeping words (every CTA, a strided share).
__global__ void __launch_bounds__(1024) index_plan(const int32_t* __restrict__ q_pos, int G,
                                                   int ngroups, int m, int N,
                                                   int* __restrict__ prefix,
                                                   unsigned* __restrict__ zero_words,
                                                   size_t nzero) {
  __shared__ unsigned sh[33];
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < nzero;
       i += (size_t)gridDim.x * blockDim.x)
    zero_words[i] = 0u;
  if (blockIdx.x != 0) return;
  unsigned running = 0;
  for (int base = 0; base < ngroups; base += blockDim.x) {
    const int g = base + threadIdx.x;
    unsigned tiles = 0;
    if (g < ngroups) {
      int nv = 0;
      for (int i = 0; i < G; ++i) nv = max(nv, n_visible(q_pos[g * G + i], m, N));
      tiles = (unsigned)((nv + kTileM - 1) / kTileM);
    }
    unsigned total;
    unsigned ex = block_exclusive_scan(tiles, sh, &total);
    if (g < ngroups) prefix[g] = (int)(running + ex);
    running += total;
  }
  if (threadIdx.x == 0) prefix[ngroups] = (int)running;
}

template <int G, int KB, int S, int NE, int NQ>
__global__ void __launch_bounds__(IdxTcCfg<G, KB, S, NE, NQ>::kThreads, 1)
    index_scores_tc(const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmQ, IdxTcArgs a) {
  using Cfg = IdxTcCfg<G, KB, S, NE, NQ>;
  // one query per group and two warps per TMEM lane quadrant: the two
  // epilogue warp groups take alternate tiles
  constexpr bool kAlt = G == 1 && NE == 8;
  const int NROWS = G * a.nhI;  // MMA N: the group's query heads
  const int NCOL = NROWS;       // TMEM columns per accumulator
  const int qslot_bytes = KB * NROWS * 128;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* kst = smem;                                  // S stages
  uint8_t* qsl = kst + S * Cfg::kStageBytes;            // NQ query slots
  uint64_t* bars = (uint64_t*)(qsl + NQ * qslot_bytes);  // barriers
  uint64_t* kfull = bars;
  uint64_t* kempty = bars + S;
  uint64_t* qfull = bars + 2 * S;
  uint64_t* qempty = qfull + 2;
  uint64_t* tfull = qempty + 2;
  uint64_t* tempty = tfull + kMaxAcc;
  uint32_t* tbase_sm = (uint32_t*)(tempty + kMaxAcc);
  volatile int* abort_sm = (volatile int*)(tbase_sm + 1);
  unsigned* shist = (unsigned*)((uint8_t*)bars + 512);  // [kHistBins] when G == 1
  int* s_prefix = (int*)((uint8_t*)bars + 512 + (G == 1 ? kHistBins * 4 : 0));  // [65]
  float* s_w = (float*)(s_prefix + 80);  // [G * 64] head weights of the group (G > 1)

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // as many TMEM accumulators as fit (up to 8): more products in flight
  // hide the latency of each tile's chain of dependent MMAs
  int nacc = 512 / NCOL;
  if (nacc > kMaxAcc) nacc = kMaxAcc;
  const int ncols_alloc = 512;

  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) {
      mbar_init(&kfull[i], 1);
      mbar_init(&kempty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&qfull[i], 1);
      mbar_init(&qempty[i], 1);
    }
    for (int i = 0; i < kMaxAcc; ++i) {
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], kAlt ? 4 : NE);
    }
    *abort_sm = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tbase_sm, ncols_alloc);
    tmem_relinquish();
  }
  if (threadIdx.x == 32) {
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmQ);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tbase_sm;

  if (a.prefix == nullptr) {
    // tiles of each group (threads 0..63) and their prefix: two warp scans
    if (threadIdx.x < kInlineGroups) {
      const int g = threadIdx.x;
      int tiles = 0;
      if (g < a.ngroups) {
        int nv = 0;
        for (int i = 0; i < G; ++i) nv = max(nv, n_visible(__ldg(a.q_pos + g * G + i), a.m, a.N));
        tiles = (nv + kTileM - 1) / kTileM;
      }
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, tiles, o);
        if (lane >= o) tiles += y;
      }
      s_prefix[g + 1] = tiles;
      if (g == 0) s_prefix[0] = 0;
    }
    __syncthreads();
    if (threadIdx.x >= 32 && threadIdx.x < kInlineGroups) s_prefix[threadIdx.x + 1] += s_prefix[32];
    __syncthreads();
  }
  const int* prefix = a.prefix ? a.prefix : s_prefix;
  const int total = prefix[a.ngroups];
  const int start = (int)((long long)total * blockIdx.x / gridDim.x);
  const int count = (int)((long long)total * (blockIdx.x + 1) / gridDim.x) - start;

  if (count > 0) {
    if (warp == 0 && lane == 0) {
      // ------------------------------------------------------- producer --
      TileCursor cur;
      cur.init(prefix, a.ngroups, start, count);
      const uint64_t pol = l2_evict_first_policy();
      int kn = 0, qn = 0;
      for (int i = 0; i < count; ++i) {
        if (cur.first(i)) {
          const int slot = qn % NQ;
          if (!mbar_wait(&qempty[slot], ((qn / NQ) & 1) ^ 1, abort_sm)) break;
          mbar_expect_tx(&qfull[slot], (uint32_t)qslot_bytes);
          uint8_t* dst = qsl + slot * qslot_bytes;
          for (int kb = 0; kb < KB; ++kb)
            tma_load_2d(dst + kb * NROWS * 128, &tmQ, &qfull[slot], kb * 64,
                        cur.g * G * a.nhI);
          ++qn;
        }
        const int s = kn % S;
        if (!mbar_wait(&kempty[s], ((kn / S) & 1) ^ 1, abort_sm)) break;
        mbar_expect_tx(&kfull[s], (uint32_t)Cfg::kStageBytes);
        const int b = (cur.g * G) / a.Q;
        const int row = b * a.N + cur.t * kTileM;
        for (int kb = 0; kb < KB; ++kb) {
          uint8_t* dst = kst + s * Cfg::kStageBytes + kb * kKBlockBytes;
          if (a.stream_keys)
            tma_load_2d_hint(dst, &tmK, &kfull[s], kb * 64, row, pol);
          else
            tma_load_2d(dst, &tmK, &kfull[s], kb * 64, row);
        }
        ++kn;
        cur.next(prefix, a.ngroups);
      }
    } else if (warp == 1 && lane == 0) {
      // ------------------------------------------------------------ MMA --
      TileCursor cur;
      cur.init(prefix, a.ngroups, start, count);
      const uint32_t idesc = idesc_bf16(kTileM, NROWS);
      int kn = 0, qn = 0, an = 0;
      for (int i = 0; i < count; ++i) {
        const bool first = cur.first(i), last = cur.last(prefix);
        const int slot = qn % NQ;
        if (first && !mbar_wait(&qfull[slot], (qn / NQ) & 1, abort_sm)) break;
        const int s = kn % S;
        if (!mbar_wait(&kfull[s], (kn / S) & 1, abort_sm)) break;
        const int acc = an % nacc;
        if (!mbar_wait(&tempty[acc], ((an / nacc) & 1) ^ 1, abort_sm)) break;
        tc_fence_after();
        const uint32_t abase = smem_u32(kst + s * Cfg::kStageBytes);
        const uint32_t bbase = smem_u32(qsl + slot * qslot_bytes);
        const uint32_t d = tbase + acc * NCOL;
#pragma unroll
        for (int kb = 0; kb < KB; ++kb)
#pragma unroll
          for (int j = 0; j < 4; ++j)
            mma_bf16(d, sdesc_k_sw128(abase + kb * kKBlockBytes + j * 32),
                     sdesc_k_sw128(bbase + kb * NROWS * 128 + j * 32), idesc,
                     (kb | j) != 0);
        mma_commit(&kempty[s]);
        mma_commit(&tfull[acc]);
        if (last) {
          mma_commit(&qempty[slot]);
          ++qn;
        }
        ++kn;
        ++an;
        cur.next(prefix, a.ngroups);
      }
    } else if (warp >= 2) {
      // ------------------------------------------------------- epilogue --
      const int e = warp - 2;
      const int quad = warp & 3;         // TMEM lane quadrant of this warp
      const int nq_mine = (NE == 4 || kAlt) ? G : G / 2;
      const int q0 = (NE == 4 || kAlt) ? 0 : (e >> 2) * (G / 2);
      const int alt = e >> 2;  // kAlt: this warp group's tile parity
      const bool hist = G == 1 && a.ghist != nullptr;
      const int et = threadIdx.x - 64;  // 0 .. 32*NE-1
      if (hist) {
        for (int i = et; i < kHistBins; i += 32 * NE) shist[i] = 0u;
        named_bar(2, 32 * NE);
      }
      TileCursor cur;
      cur.init(prefix, a.ngroups, start, count);
      int an = 0, hist_r = cur.g;
      // after a wait gives up the warp keeps walking the list without work,
      // so that every epilogue warp takes the same named barriers
      bool dead = false;
      float wreg[G == 1 ? 64 : 1];
      int w_r = -1;
      constexpr int NQM = (NE == 4 || kAlt) ? G : G / 2;  // queries of this warp
      int nvq[NQM];  // visible entries of those queries (current group)
      int grp_r = -1;
      for (int i = 0; i < count; ++i) {
        if (cur.g != grp_r) {  // group changed: its visible counts (and weights)
#pragma unroll
          for (int qq = 0; qq < NQM; ++qq)
            nvq[qq] = n_visible(__ldg(a.q_pos + cur.g * G + q0 + qq), a.m, a.N);
          if (G > 1 && a.nhI == 64) {
            named_bar(2, 32 * NE);  // every epilogue warp is done with the old weights
            for (int j = et; j < G * 64; j += 32 * NE) s_w[j] = __ldg(a.w + (size_t)cur.g * G * 64 + j);
            named_bar(2, 32 * NE);
          }
          grp_r = cur.g;
        }
        if (hist && cur.g != hist_r) {  // query changed: flush its histogram
          named_bar(2, 32 * NE);
          for (int bin = et; bin < kHistBins; bin += 32 * NE) {
            const unsigned c = shist[bin];
            if (c) {
              atomicAdd(&a.ghist[(size_t)hist_r * kHistBins + bin], c);
              shist[bin] = 0u;
            }
          }
          named_bar(2, 32 * NE);
          hist_r = cur.g;
        }
        if (kAlt && (an & 1) != alt) {  // the other warp group's tile
          ++an;
          cur.next(prefix, a.ngroups);
          continue;
        }
        const int acc = an % nacc;
        if (!dead) dead = !__all_sync(0xffffffffu, mbar_wait(&tfull[acc], (an / nacc) & 1, abort_sm));
        if (dead) {
          ++an;
          cur.next(prefix, a.ngroups);
          continue;
        }
        tc_fence_after();
        const int s = cur.t * kTileM + quad * 32 + lane;
        float sc[G];
#pragma unroll
        for (int qi = 0; qi < G; ++qi) sc[qi] = 0.f;
        const uint32_t trow = tbase + ((uint32_t)(quad * 32) << 16) + acc * NCOL;
        if (G == 1 && a.nhI == 64) {
          // one query per group: its 64 head weights stay in registers
          if (cur.g != w_r) {
            const float4* w4 = reinterpret_cast<const float4*>(a.w + (size_t)cur.g * 64);
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              const float4 t = __ldg(w4 + j);
              wreg[4 * j] = t.x; wreg[4 * j + 1] = t.y; wreg[4 * j + 2] = t.z; wreg[4 * j + 3] = t.w;
            }
            w_r = cur.g;
          }
          float v[4][16];
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) tmem_ld16(trow + q4 * 16, v[q4]);
          tmem_wait_ld();
          float part[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4)
#pragma unroll
            for (int j = 0; j < 16; ++j)
              part[q4] = fmaf(wreg[16 * q4 + j], fmaxf(v[q4][j], 0.f), part[q4]);
          sc[0] = (part[0] + part[1]) + (part[2] + part[3]);
        } else if (a.nhI == 64) {
          // 64 heads per query: weights of the group in shared memory
#pragma unroll
          for (int qq = 0; qq < NQM; ++qq) {
            const int qi = q0 + qq;
            float v[4][16];
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) tmem_ld16(trow + qi * 64 + q4 * 16, v[q4]);
            tmem_wait_ld();
            const float4* w4 = reinterpret_cast<const float4*>(s_w + qi * 64);
            float part[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4)
#pragma unroll
              for (int j4 = 0; j4 < 4; ++j4) {
                const float4 ww = w4[q4 * 4 + j4];
                part[q4] = fmaf(ww.x, fmaxf(v[q4][4 * j4 + 0], 0.f), part[q4]);
                part[q4] = fmaf(ww.y, fmaxf(v[q4][4 * j4 + 1], 0.f), part[q4]);
                part[q4] = fmaf(ww.z, fmaxf(v[q4][4 * j4 + 2], 0.f), part[q4]);
                part[q4] = fmaf(ww.w, fmaxf(v[q4][4 * j4 + 3], 0.f), part[q4]);
              }
            sc[qq] = (part[0] + part[1]) + (part[2] + part[3]);
          }
        } else {
        for (int qq = 0; qq < nq_mine; ++qq) {
          const int qi = q0 + qq;
          const float* wr = a.w + (size_t)(cur.g * G + qi) * a.nhI;
          // four independent partial sums over the heads (16 heads per
          // TMEM load); all loads of a 64-head block issued before one wait
          float part[4] = {0.f, 0.f, 0.f, 0.f};
          for (int c0 = 0; c0 < a.nhI; c0 += 64) {
            const int nb = min(64, a.nhI - c0) / 16;
            float v[4][16];
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4)
              if (q4 < nb) tmem_ld16(trow + qi * a.nhI + c0 + q4 * 16, v[q4]);
            tmem_wait_ld();
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
              if (q4 >= nb) continue;
              const float4* w4 = reinterpret_cast<const float4*>(wr + c0 + q4 * 16);
#pragma unroll
              for (int j4 = 0; j4 < 4; ++j4) {
                const float4 ww = __ldg(w4 + j4);
                part[q4] = fmaf(ww.x, fmaxf(v[q4][4 * j4 + 0], 0.f), part[q4]);
                part[q4] = fmaf(ww.y, fmaxf(v[q4][4 * j4 + 1], 0.f), part[q4]);
                part[q4] = fmaf(ww.z, fmaxf(v[q4][4 * j4 + 2], 0.f), part[q4]);
                part[q4] = fmaf(ww.w, fmaxf(v[q4][4 * j4 + 3], 0.f), part[q4]);
              }
            }
          }
          sc[qq] = (part[0] + part[1]) + (part[2] + part[3]);
        }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&tempty[acc]);
#pragma unroll
        for (int qq = 0; qq < NQM; ++qq) {
          const int r = cur.g * G + q0 + qq;
          if (s < nvq[qq]) {
            a.scores[(size_t)r * a.N + s] = sc[qq];
            if (hist) atomicAdd(&shist[score_key(sc[qq]) >> 20], 1u);
          }
        }
        ++an;
        cur.next(prefix, a.ngroups);
      }
      if (hist) {  // flush the last query's histogram
        named_bar(2, 32 * NE);
        for (int bin = et; bin < kHistBins; bin += 32 * NE) {
          const unsigned c = shist[bin];
          if (c) atomicAdd(&a.ghist[(size_t)hist_r * kHistBins + bin], c);
        }
      }
    }
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (*abort_sm) {
    if (threadIdx.x == 0) atomicOr(a.err, CSA_DEV_TIMEOUT);
    // let tensor-core work already issued drain before TMEM is released
    const uint64_t t0 = globaltimer();
    while (globaltimer() - t0 < 200000ull) __nanosleep(1000);
  }
  pdl_trigger();  // the top-k kernel may be scheduled as this grid retires
  if (warp == 1) tmem_dealloc(tbase, ncols_alloc);
}

// ------------------------------------------------------------------ host --
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = (EncodeTiledFn)p;
  }
  return fn;
}

// Encoded tensor maps are cached per host thread (direct-mapped on the
// pointer and shape): a decode step re-encodes the same maps every call.
namespace {
struct TmapKey {
  const void* base;
  uint64_t rows, cols;
  uint32_t box_rows, dtype;
  bool operator==(const TmapKey& o) const {
    return base == o.base && rows == o.rows && cols == o.cols && box_rows == o.box_rows &&
           dtype == o.dtype;
  }
};
struct TmapEntry {
  TmapKey key;
  CUtensorMap map;
  bool valid;
};
constexpr int kTmapCache = 64;
thread_local TmapEntry t_tmaps[kTmapCache];
TmapEntry& tmap_slot(const TmapKey& k) {
  uint64_t h = (uint64_t)(uintptr_t)k.base * 0x9E3779B97F4A7C15ull;
  h ^= (k.rows * 31 + k.cols) * 0xC2B2AE3D27D4EB4Full + k.box_rows * 131 + k.dtype;
  return t_tmaps[(h >> 40) % kTmapCache];
}
}  // namespace

static bool encode_bf16(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols,
                        uint32_t box_rows);
static bool encode_f32(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols,
                       uint32_t box_rows);

bool make_tmap_bf16(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols,
                    uint32_t box_rows) {
  const TmapKey k{base, rows, cols, box_rows, 2};
  TmapEntry& e = tmap_slot(k);
  if (e.valid && e.key == k) {
    *m = e.map;
    return true;
  }
  if (!encode_bf16(m, base, rows, cols, box_rows)) return false;
  e = TmapEntry{k, *m, true};
  return true;
}

bool make_tmap_f32(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols,
                   uint32_t box_rows) {
  const TmapKey k{base, rows, cols, box_rows, 4};
  TmapEntry& e = tmap_slot(k);
  if (e.valid && e.key == k) {
    *m = e.map;
    return true;
  }
  if (!encode_f32(m, base, rows, cols, box_rows)) return false;
  e = TmapEntry{k, *m, true};
  return true;
}

// 2-D bf16 tensor [rows][cols] (cols contiguous), boxes of 64 x box_rows with
// the 128-byte swizzle.
static bool encode_bf16(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols,
                        uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t es[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
            es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// fp32 rows of `cols` floats; boxes of 32 columns (128 bytes) x box_rows rows
static bool encode_f32(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols,
                       uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 4};
  cuuint32_t box[2] = {32, box_rows};
  cuuint32_t es[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(base), dims, strides, box,
            es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2-D byte tensor [rows][cols] (cols contiguous, a multiple of 16), boxes
// of box_cols x box_rows, without swizzle or (box_cols = 64) in the 64-byte
// swizzle.
bool make_tmap_u8(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols,
                  uint32_t box_cols, uint32_t box_rows, bool swizzle64) {
  const TmapKey k{base, rows, cols, box_rows, swizzle64 ? 65u : 1u};
  TmapEntry& e = tmap_slot(k);
  if (e.valid && e.key == k) {
    *m = e.map;
    return true;
  }
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t es[2] = {1, 1};
  if (fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, es,
         CU_TENSOR_MAP_INTERLEAVE_NONE,
         swizzle64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_NONE,
         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return false;
  e = TmapEntry{k, *m, true};
  return true;
}

bool tma_available() { return encode_fn() != nullptr; }

bool index_tc_supported(const csa_params& p) {
  return p.act == CSA_BF16 && (p.c_I == 64 || p.c_I == 128) && p.n_hI % 16 == 0 &&
         p.n_hI <= 64 && encode_fn() != nullptr;
}

int index_tc_group(const csa_params& p, int Q) {
  int G = 1;
  for (int g : {4, 2})
    if (Q % g == 0 && g * p.n_hI <= 256) { G = g; break; }
  return G;
}

size_t index_tc_plan_bytes(int ngroups) { return align_up((size_t)(ngroups + 1) * 4, 256); }

template <int G, int KB, int S, int NE, int NQ = 2>
static csa_status launch_tc_t(const CUtensorMap& tmK, const CUtensorMap& tmQ,
                              const IdxTcArgs& a, cudaStream_t st) {
  using Cfg = IdxTcCfg<G, KB, S, NE, NQ>;
  const int NROWS = G * a.nhI;
  size_t smem = 1024 + (size_t)S * Cfg::kStageBytes + NQ * (size_t)KB * NROWS * 128 + 512 +
                (G == 1 ? kHistBins * 4 : 0) + 80 * 4 + G * 64 * 4;
  auto kern = index_scores_tc<G, KB, S, NE, NQ>;
  if (!set_kernel_smem((const void*)kern, (int)smem)) return CSA_ERR_CUDA;
  const int sms = sm_count();
  const int occ = kernel_occupancy((const void*)kern, Cfg::kThreads, (int)smem);
  if (occ < 1) return CSA_ERR_UNSUPPORTED;
  const int grid = sms * occ;
  CSA_LAUNCH(KK_SCORES, st, kern<<<grid, Cfg::kThreads, smem, st>>>(tmK, tmQ, a));
  return last_launch_status();
}

csa_status launch_index_scores_tc(const csa_params& p, int B, int Q, const int32_t* q_pos,
                                  const void* qI, const float* w, const void* kI, int N,
                                  float* scores, int* plan, unsigned* zero_words, size_t nzero,
                                  unsigned* ghist, bool* hist_done, cudaStream_t st) {
  const int R = B * Q;
  const int G = index_tc_group(p, Q);
  const int ngroups = R / G;
  const bool inline_plan = ngroups <= kInlineGroups;
  if (nzero && cudaMemsetAsync(zero_words, 0, nzero * 4, st) != cudaSuccess) return CSA_ERR_CUDA;
  if (!inline_plan)
    CSA_LAUNCH(KK_PLAN, st, index_plan<<<1, 1024, 0, st>>>(q_pos, G, ngroups, p.m, N, plan,
                                                           nullptr, 0));
  *hist_done = false;
  if (N == 0) return last_launch_status();
  CUtensorMap tmK, tmQ;
  if (!make_tmap_bf16(&tmK, kI, (uint64_t)B * N, p.c_I, kTileM)) return CSA_ERR_CUDA;
  if (!make_tmap_bf16(&tmQ, qI, (uint64_t)R * p.n_hI, p.c_I, G * p.n_hI)) return CSA_ERR_CUDA;
  IdxTcArgs a{q_pos, w, inline_plan ? nullptr : plan, scores, device_error_word(), G == 1 ? ghist : nullptr,
              Q, N, p.m, p.n_hI, ngroups, Q == G ? 1 : 0};
  if (a.err == nullptr) return CSA_ERR_CUDA;
  *hist_done = a.ghist != nullptr;
  const bool k2 = p.c_I == 128;
  if (G == 1) return k2 ? launch_tc_t<1, 2, 6, 8, 1>(tmK, tmQ, a, st) : launch_tc_t<1, 1, 8, 4>(tmK, tmQ, a, st);
  if (G == 2) return k2 ? launch_tc_t<2, 2, 4, 4>(tmK, tmQ, a, st) : launch_tc_t<2, 1, 6, 4>(tmK, tmQ, a, st);
  return k2 ? launch_tc_t<4, 2, 2, 8>(tmK, tmQ, a, st) : launch_tc_t<4, 1, 4, 8>(tmK, tmQ, a, st);
}

}  // namespace csa
