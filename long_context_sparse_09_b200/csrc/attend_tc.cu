// attend_tc.cu -- shared-KV MQA with window and sink on the 5th-generation
// tensor cores ("DeepSeekV4技术报告阅读笔记" eq. 19 / 26 / 27, sections
// 2.5.2-2.5.3; "02 · DeepSeek-V4: 压缩注意力撑起 1M 上下文" sections 2.4-2.5).
//
// A CTA owns (query, block of 64 heads, slice of the query's key list).  The
// 64 heads are the MMA's M dimension: S = Q K^T (M = 64 heads, N = 64 keys,
// K = 512 dims) and O += P V (M = 64 heads, N = dims, K = 64 keys).  An M = 64
// accumulator fills half of every 32-lane TMEM sub-partition, so O (64 x 512
// fp32) lives as two halves -- dims 0-255 in the upper half-lanes, dims
// 256-511 in the lower half-lanes, 256 columns -- and the two S buffers of a
// double-buffered key tile sit in the remaining columns, one per half.  Each
// softmax thread therefore owns one head's row: the max, exp and sum are
// in-thread.  The running max is kept "lazily": O is rescaled only when a
// tile raises it by more than 8 (e^8 headroom in fp32).
//
// One smem key tile [64 keys][512] bf16 in the 128-byte swizzle layout is
// both the K-major B operand of Q K^T and the MN-major B operand of P V.
// Keys are gathered (top-k indices, window rows) by four loader warps with
// 16-byte loads; FP8-mixed rows are widened to bf16 exactly (E4M3 codes are
// bf16 values) and their per-row scale is applied in fp32: logit =
// scale_j * (q . codes_j) + q_rope . rope_j, and P V uses p_j * scale_j for
// the FP8 dims and p_j for the RoPE dims.
//
// Warps: 0-3 gather keys, 4 loads Q by TMA / owns TMEM / issues MMAs, 5-8 run
// the softmax and the epilogue (sink, normalisation, R_{-t0}, store).
#include <cuda.h>

#include <cstring>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace csa {

using namespace sm100;

struct AttnTcArgs {
  const int32_t* q_pos;
  const int32_t* idx;
  const uint8_t* ckv;
  const float* ckv_scale;
  const uint8_t* win;
  const float* win_scale;
  const int32_t* win_pos0;
  const float* sink;
  __nv_bfloat16* out;
  float* ws_o;   // split partials [nsplit][R][n_h][512] (global combine)
  float* ws_ml;  // their (max, sum) [nsplit][R][n_h][2]
  unsigned* err;
  int Q, N, W, n_h, m, topk, n_win, nsplit, keys_per_split, dense, R, hblocks;
  int items;               // (query, head block, key slice) work items of the launch
  int R_rows_c, R_rows_w;  // total rows of the cache / window tensors (out of range)
  int box_rows;            // rows of one output box: min(64, n_h)
  int cluster;             // the key slices of a (query, head block) form a cluster
  float scale2;  // softmax scale times log2(e): the softmax runs in base 2
  double base;
};

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kMasked = -1e30f;  // logit of an absent key (exp2 -> 0)

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

constexpr int kAtThreads = 288;   // 9 warps
constexpr int kQBytes = 64 * 1024;
constexpr int kPBytes = 8 * 1024;
constexpr float kLazyRescale = 8.0f;  // log2 units: rescale when the max grows 256x
constexpr int kMaxSlices = 8;         // key slices of one (query, head block): one cluster
constexpr bool kAsyncGather = true;   // bf16 selected rows by cp.async (else via registers)

// KT keys per tile, NS key-tile stages: FP8-mixed caches use 64-key tiles in
// 2 stages (its P needs two buffers per parity), bf16 caches 48-key tiles in
// 3 stages (a tile can load while the two before it are in use).
template <bool FP8, int KT, int NS>
struct AtLayout {
  static constexpr int NP = FP8 ? 2 : 1;  // P buffers per tile parity
  static constexpr int KSTAGE = KT * 1024;  // a key tile: 8 k-blocks of KT rows x 128 B
  static constexpr int q = 0;
  static constexpr int k = kQBytes;
  static constexpr int p = k + NS * KSTAGE;
  static constexpr int meta = p + 2 * NP * kPBytes;
  static constexpr int bars = meta + 896;  // key scales [NS][64] fp32, masks [NS] u64
  static constexpr int total = bars + 256;
};

__device__ __forceinline__ uint4 zero4() { return make_uint4(0u, 0u, 0u, 0u); }

__device__ __forceinline__ void st_shared16(uint8_t* p, uint4 v) {
  *reinterpret_cast<uint4*>(p) = v;
}

__device__ __forceinline__ uint32_t pack_bf16(float x, float y) {
  __nv_bfloat162 h = __floats2bfloat162_rn(x, y);
  return *reinterpret_cast<uint32_t*>(&h);
}

// 16 E4M3 codes -> 16 bf16 (exact), as two 16-byte chunks
__device__ __forceinline__ void widen_e4m3(uint4 raw, uint4& lo, uint4& hi) {
  const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
  uint32_t o[8];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t x = w[i];
    o[2 * i] = pack_bf16(e4m3_to_f32(x & 0xFF), e4m3_to_f32((x >> 8) & 0xFF));
    o[2 * i + 1] = pack_bf16(e4m3_to_f32((x >> 16) & 0xFF), e4m3_to_f32(x >> 24));
  }
  lo = make_uint4(o[0], o[1], o[2], o[3]);
  hi = make_uint4(o[4], o[5], o[6], o[7]);
}

// Key-row tensor maps (bf16 caches): boxes of 64 columns x 64 rows for
// contiguous key runs, and of 64 x 1 rows for gathers of selected rows; and
// the map of the fp32 split partials [S*R*n_h][512] in 128-byte boxes of
// box_rows rows.
struct KeyMaps {
  CUtensorMap c_box, c_row, w_box, w_row, o_ws;
};

template <bool FP8, int KT, int NS>
__global__ void __launch_bounds__(kAtThreads, 1)
    attend_tc(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ KeyMaps km,
              AttnTcArgs a) {
  using L = AtLayout<FP8, KT, NS>;
  static_assert(KT % 16 == 0 && KT <= 64 && (!FP8 || KT == 64), "key tile");
  constexpr int KBS = KT * 128;  // k-block stride of a key tile
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* sQ = sm + L::q;
  uint8_t* sK = sm + L::k;
  uint8_t* sP = sm + L::p;
  float* meta_scale = (float*)(sm + L::meta);                        // [NS][64]
  unsigned long long* meta_mask = (unsigned long long*)(sm + L::meta + 768);  // [NS]
  uint64_t* bars = (uint64_t*)(sm + L::bars);
  uint64_t* qfull = bars;
  uint64_t* kfull = bars + 1;       // [NS]
  uint64_t* kempty = kfull + NS;    // [NS]
  uint64_t* sfull = kempty + NS;    // [2]
  uint64_t* sfree = sfull + 2;      // [2]
  uint64_t* pfull = sfree + 2;      // [2]
  uint64_t* pvdone = pfull + 2;     // [2]
  uint64_t* oempty = pvdone + 2;    // O read out by the previous item's output
  uint32_t* tbase_sm = (uint32_t*)(oempty + 1);
  volatile int* abort_sm = (volatile int*)(tbase_sm + 1);
  int& valid_sm = *(int*)(tbase_sm + 2);  // the slice had keys (cluster combine)
  volatile int* stop_sm = (volatile int*)(tbase_sm + 3);  // a loader's wait gave up
  volatile int* ostop_sm = (volatile int*)(tbase_sm + 4);  // an output thread's wait gave up
  // slice max (base 2) and sum per head for the cluster combine; written
  // after the last tile, when the per-tile key scales are no longer read
  float2* ml_sm = (float2*)meta_scale;  // [64]
  __shared__ const uint8_t* row_sm[KT];
  __shared__ float rope_tab[64];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(qfull, 1);
    for (int i = 0; i < NS; ++i) {
      mbar_init(&kfull[i], 128);
      mbar_init(&kempty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sfull[i], 1);
      mbar_init(&sfree[i], 4);
      mbar_init(&pfull[i], 4);
      mbar_init(&pvdone[i], 1);
    }
    mbar_init(oempty, 4);
    *abort_sm = 0;
    *stop_sm = 0;
    *ostop_sm = 0;
    fence_mbar_init();
  }
  if (warp == 4) {
    tmem_alloc(tbase_sm, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tbase_sm;
  const size_t rb = FP8 ? 576 : 1024;  // stored row bytes
  // the set-up above may overlap the previous kernel; inputs are read below
  pdl_wait();
  // A CTA takes items blockIdx.x, + gridDim.x, ...: one item when the key
  // list of a query is split into slices (the slices are combined after the
  // item); with one slice per query the grid is one CTA per SM and every
  // role runs on into the next query (its gathers, Q load and first
  // S = Q K^T overlap the current query's output).  g counts the key tiles
  // of the CTA: stage g % NS, S / P buffer g & 1, and the barrier phases.
  struct ItemInfo {
    int r, hb, sp, b, t0, nv, lo, n_main, j_begin, j_end, ntiles;
  };
  auto item_info = [&](int item) {
    ItemInfo I;
    const int per_r = a.hblocks * a.nsplit;
    I.r = item / per_r;
    I.hb = (item % per_r) / a.nsplit;
    I.sp = item % a.nsplit;
    I.b = I.r / a.Q;
    I.t0 = a.q_pos[I.r];
    I.nv = n_visible(I.t0, a.m, a.N);
    I.lo = I.t0 - a.n_win + 1 > 0 ? I.t0 - a.n_win + 1 : 0;
    const int nwin_q = (a.n_win > 0 && I.t0 >= 0) ? I.t0 - I.lo + 1 : 0;
    I.n_main = a.dense ? I.nv : a.topk;
    const int nk = I.n_main + nwin_q;
    I.j_begin = I.sp * a.keys_per_split;
    I.j_end = min(nk, I.j_begin + a.keys_per_split);
    I.ntiles = I.j_end > I.j_begin ? (I.j_end - I.j_begin + KT - 1) / KT : 0;
    return I;
  };

  {
    if (warp < 4) {
     if constexpr (!FP8) {
      // ----------------------------------------------------- key loads (bf16) --
      // Contiguous 64-key runs (HCA entries, window rows) come in as TMA
      // boxes; selected rows are gathered with 16-byte loads, 16 in flight
      // per thread, and stored into the swizzled tile.
      const int t = threadIdx.x;
      __shared__ int s_mode, s_row0;
      int g = 0;
      bool quit = false;
      for (int item = blockIdx.x; !quit && item < a.items; item += gridDim.x) {
        const ItemInfo I = item_info(item);
        const int b = I.b, r = I.r, nv = I.nv, lo = I.lo, n_main = I.n_main, j_end = I.j_end;
        const int wp0 = a.win ? a.win_pos0[b] : 0;
        const uint8_t* ckv = a.ckv + (size_t)b * a.N * rb;
        const uint8_t* win = a.win + (size_t)b * a.W * rb;
        // the selected index of this thread's key in the next tile is loaded
        // one tile ahead (its latency hides behind the current tile's copies)
        auto sel_index = [&](int j) -> int {
          return (t < KT && !a.dense && j < j_end && j < n_main)
                     ? __ldg(a.idx + (size_t)r * a.topk + j) : 0;
        };
        int e_next = sel_index(I.j_begin + t);
        for (int i = 0; i < I.ntiles; ++i, ++g) {
          const int s = g % NS;
          // the loop holds named barriers: a wait that gives up raises a flag
          // that every loader reads after the next barrier, so all 128 leave
          // at the same point
          if (!mbar_wait(&kempty[s], ((g / NS) & 1) ^ 1, abort_sm)) *stop_sm = 1;
          const int j0 = I.j_begin + i * KT;
          const int e_sel = e_next;
          e_next = sel_index(j0 + KT + t);
          if (t < 64) {  // warps 0-1: key t of the tile (t < KT)
            const int j = j0 + t;
            int valid = 0;
            const int inwin = j >= n_main;
            const uint8_t* row = nullptr;
            if (t < KT && j < j_end) {
              if (j < n_main) {
                const int e = a.dense ? j : e_sel;
                if (e >= 0) {
                  if (e < nv) {
                    valid = 1;
                    row = ckv + (size_t)e * rb;
                  } else {
                    atomicOr(a.err, CSA_DEV_BAD_INDEX);
                  }
                }
              } else {
                const int wr = lo + (j - n_main) - wp0;
                if (a.win != nullptr && wr >= 0 && wr < a.W) {
                  valid = 1;
                  row = win + (size_t)wr * rb;
                } else {
                  atomicOr(a.err, CSA_DEV_BAD_WINDOW);
                }
              }
            }
            if (t < KT) {
              row_sm[t] = row;
              meta_scale[s * 64 + t] = 1.f;
            }
            const unsigned vb = __ballot_sync(0xffffffffu, valid);
            if ((t & 31) == 0) reinterpret_cast<unsigned*>(&meta_mask[s])[t >> 5] = vb;
            (void)inwin;
          }
          named_bar(1, 128);
          if (*stop_sm) {
            quit = true;
            break;
          }
          if (t == 0) {
            // whole tile contiguous in one tensor? (entries: dense; window)
            bool ent = true, wnd = true;
            for (int u = 0; u < KT; ++u) {
              const int j = j0 + u;
              if (j >= n_main) ent = false; else wnd = false;
            }
            s_mode = (a.dense && ent) ? 1 : (wnd ? 2 : 0);
            s_row0 = s_mode == 1 ? b * a.N + j0 : b * a.W + lo + (j0 - n_main) - wp0;
          }
          named_bar(1, 128);
          uint8_t* dstK = sK + s * L::KSTAGE;
          const int mode = s_mode;
          if (mode != 0) {
            if (t == 0) mbar_expect_tx(&kfull[s], (uint32_t)L::KSTAGE);
            __syncwarp();
            if (t < 8)
              tma_load_2d(dstK + t * KBS, mode == 1 ? &km.c_box : &km.w_box, &kfull[s], t * 64,
                          s_row0);
            if (t != 0) mbar_arrive(&kfull[s]);
          } else if (kAsyncGather) {
            // selected rows: 32 asynchronous 16-byte copies per thread straight
            // into the swizzled tile (absent rows are zero-filled); the barrier
            // completes when they land, so the next tile's copies can follow
#pragma unroll 8
            for (int u = 0; u < KT / 2; ++u) {
              const int idx = u * 128 + t;
              const int key = idx >> 6, ch = idx & 63;
              const int kb = ch >> 3, c = ch & 7;
              const uint8_t* src = row_sm[key];
              cp_async16(dstK + kb * KBS + key * 128 + ((c ^ (key & 7)) << 4),
                         src ? src + ch * 16 : a.ckv, src ? 16u : 0u);
            }
            cp_async_arrive(&kfull[s]);
          } else {
#pragma unroll 1
            for (int it0 = 0; it0 < KT / 2; it0 += 16) {
              uint4 v[16];
#pragma unroll
              for (int u = 0; u < 16; ++u) {
                const int idx = (it0 + u) * 128 + t;
                const int key = idx >> 6, ch = idx & 63;
                const uint8_t* src = it0 + u < KT / 2 ? row_sm[key] : nullptr;
                v[u] = src ? __ldg(reinterpret_cast<const uint4*>(src + ch * 16)) : zero4();
              }
#pragma unroll
              for (int u = 0; u < 16; ++u) {
                if (it0 + u >= KT / 2) continue;
                const int idx = (it0 + u) * 128 + t;
                const int key = idx >> 6, ch = idx & 63;
                const int kb = ch >> 3, c = ch & 7;
                st_shared16(dstK + kb * KBS + key * 128 + ((c ^ (key & 7)) << 4), v[u]);
              }
            }
            fence_proxy_async_smem();
            mbar_arrive(&kfull[s]);
          }
          named_bar(1, 128);  // row_sm and the mode are rewritten by the next tile
        }
      }
     } else {
      // ------------------------------------------- key gather (FP8-mixed) --
      const int t = threadIdx.x;
      int g = 0;
      bool quit = false;
      for (int item = blockIdx.x; !quit && item < a.items; item += gridDim.x) {
        const ItemInfo I = item_info(item);
        const int b = I.b, r = I.r, nv = I.nv, lo = I.lo, n_main = I.n_main, j_end = I.j_end;
        const uint8_t* ckv = a.ckv + (size_t)b * a.N * rb;
        const uint8_t* win = a.win + (size_t)b * a.W * rb;
        const int wp0 = a.win ? a.win_pos0[b] : 0;
        for (int i = 0; i < I.ntiles; ++i, ++g) {
          const int s = g % NS;
          if (!mbar_wait(&kempty[s], ((g / NS) & 1) ^ 1, abort_sm)) *stop_sm = 1;
          float sc_reg = 1.f;
          if (t < KT) {
            const int j = I.j_begin + i * KT + t;
            int valid = 0;
            const uint8_t* row = nullptr;
            float sc = 1.f;
            if (j < j_end) {
              if (j < n_main) {
                const int e = a.dense ? j : a.idx[(size_t)r * a.topk + j];
                if (e >= 0) {
                  if (e < nv) {
                    valid = 1;
                    row = ckv + (size_t)e * rb;
                    sc = a.ckv_scale[(size_t)b * a.N + e];
                  } else {
                    atomicOr(a.err, CSA_DEV_BAD_INDEX);
                  }
                }
              } else {
                const int wr = lo + (j - n_main) - wp0;
                if (a.win != nullptr && wr >= 0 && wr < a.W) {
                  valid = 1;
                  row = win + (size_t)wr * rb;
                  sc = a.win_scale[(size_t)b * a.W + wr];
                } else {
                  atomicOr(a.err, CSA_DEV_BAD_WINDOW);
                }
              }
            }
            row_sm[t] = valid ? row : nullptr;
            sc_reg = sc;  // in flight with the row loads below
            const unsigned bits = __ballot_sync(0xffffffffu, valid);
            if ((t & 31) == 0) reinterpret_cast<unsigned*>(&meta_mask[s])[t >> 5] = bits;
          }
          named_bar(1, 128);
          if (*stop_sm) {
            quit = true;
            break;
          }
          uint8_t* dstK = sK + s * L::KSTAGE;
          // all 18 loads in flight, then widen and store
          uint4 v[18];
#pragma unroll
          for (int u = 0; u < 18; ++u) {
            const int idx = u * 128 + t;
            const int key = idx / 36, ch = idx % 36;
            const uint8_t* src = row_sm[key];
            v[u] = src ? __ldg(reinterpret_cast<const uint4*>(src + ch * 16)) : zero4();
          }
#pragma unroll
          for (int u = 0; u < 18; ++u) {
            const int idx = u * 128 + t;
            const int key = idx / 36, ch = idx % 36;
            uint8_t* rowp = dstK + key * 128;
            const int sw = key & 7;
            if (ch < 28) {
              uint4 lo4, hi4;
              widen_e4m3(v[u], lo4, hi4);
              const int d0 = 2 * ch;  // destination chunk of dims 16ch..16ch+7
              const int kb = d0 >> 3, c0 = d0 & 7;
              st_shared16(rowp + kb * KBS + ((c0 ^ sw) << 4), lo4);
              st_shared16(rowp + kb * KBS + (((c0 + 1) ^ sw) << 4), hi4);
            } else {
              const int c = ch - 28;  // dims 448 + 8c .. : K-block 7
              st_shared16(rowp + 7 * KBS + ((c ^ sw) << 4), v[u]);
            }
          }
          if (t < KT) meta_scale[s * 64 + t] = sc_reg;
          fence_proxy_async_smem();
          mbar_arrive(&kfull[s]);
          named_bar(1, 128);  // row_sm is rewritten by the next tile
        }
      }
     }
    } else if (warp == 4) {
      // ------------------------------------------------------------- MMA --
      if (lane == 0) {
        // queries and outputs are touched once: keep the cached keys in L2
        const uint64_t qo_pol = l2_evict_first_policy();
        const uint32_t idesc_qk = idesc_bf16(64, KT, false);
        const uint32_t qb = smem_u32(sQ);
        // S(g) = Q K(g)^T into S buffer g&1 (waits for the tile and the buffer)
        auto issue_qk = [&](int i) -> bool {
          const int s = i % NS, bb = i & 1;
          if (!mbar_wait(&kfull[s], (i / NS) & 1, abort_sm)) return false;
          fence_proxy_async_smem();  // cp.async-written tile -> tensor-core reads
          if (!mbar_wait(&sfree[bb], ((i >> 1) & 1) ^ 1, abort_sm)) return false;
          tc_fence_after();
          const uint32_t sacc = tbase + ((uint32_t)(16 * bb) << 16) + 256;
          const uint32_t kbase = smem_u32(sK + s * L::KSTAGE);
#pragma unroll
          for (int kb = 0; kb < 8; ++kb) {
            const bool rope_blk = FP8 && kb == 7;
            const uint32_t d = rope_blk ? sacc + 64 : sacc;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const bool first = j == 0 && (kb == 0 || rope_blk);
              mma_bf16(d, sdesc_k_sw128(qb + kb * 8192 + j * 32),
                       sdesc_k_sw128(kbase + kb * KBS + j * 32), idesc_qk, first ? 0u : 1u);
            }
          }
          mma_commit(&sfull[bb]);
          return true;
        };
        int g = 0, qn = 0;  // key tiles and queries (Q loads) so far
        bool ok = true;
        for (int item = blockIdx.x; ok && item < a.items; item += gridDim.x) {
          const ItemInfo I = item_info(item);
          const int ntiles = I.ntiles;
          if (ntiles == 0) continue;
          // Q is rewritten once the previous query's last S = Q K^T is done
          if (g > 0 && !mbar_wait(&sfull[(g - 1) & 1], ((g - 1) >> 1) & 1, abort_sm)) break;
          mbar_expect_tx(qfull, kQBytes);
          for (int kb = 0; kb < 8; ++kb)
            tma_load_2d_hint(sQ + kb * 8192, &tmQ, qfull, kb * 64, I.r * a.n_h + I.hb * 64,
                             qo_pol);
          if (!mbar_wait(qfull, qn & 1, abort_sm) || !issue_qk(g)) break;
          for (int i = 0; i < ntiles; ++i) {
            const int gi = g + i, s = gi % NS, bb = gi & 1;
            // QK(i+1) early only if its tile and S buffer are already there;
            // P V(i) must not wait behind a late tile
            bool qk_next = false;
            if (i + 1 < ntiles && mbar_test_wait(&kfull[(gi + 1) % NS], ((gi + 1) / NS) & 1) &&
                mbar_test_wait(&sfree[(gi + 1) & 1], (((gi + 1) >> 1) & 1) ^ 1)) {
              if (!issue_qk(gi + 1)) {
                ok = false;
                break;
              }
              qk_next = true;
            }
            if (!mbar_wait(&pfull[bb], (gi >> 1) & 1, abort_sm)) {
              ok = false;
              break;
            }
            // the first P V overwrites O: the previous query's output must have
            // read it out of TMEM
            if (i == 0 && qn > 0 && !mbar_wait(oempty, (qn - 1) & 1, abort_sm)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t kbase = smem_u32(sK + s * L::KSTAGE);
            const uint32_t pb = smem_u32(sP + bb * L::NP * kPBytes);
#pragma unroll
            for (int j = 0; j < KT / 16; ++j) {
              const uint32_t acc = (i > 0 || j > 0) ? 1u : 0u;
              const uint32_t vb = kbase + j * 2048;  // 16 keys of the tile
              if constexpr (!FP8) {
                mma_bf16(tbase, sdesc_k_sw128(pb + j * 32), sdesc_mn_sw128(vb, KBS, 1024),
                         idesc_bf16(64, 256, true), acc);
                mma_bf16(tbase + (16u << 16), sdesc_k_sw128(pb + j * 32),
                         sdesc_mn_sw128(vb + 4 * KBS, KBS, 1024), idesc_bf16(64, 256, true), acc);
              } else {
                const uint32_t ps = pb, p1 = pb + kPBytes;  // p*scale, p
                mma_bf16(tbase, sdesc_k_sw128(ps + j * 32), sdesc_mn_sw128(vb, KBS, 1024),
                         idesc_bf16(64, 256, true), acc);
                mma_bf16(tbase + (16u << 16), sdesc_k_sw128(ps + j * 32),
                         sdesc_mn_sw128(vb + 4 * KBS, KBS, 1024), idesc_bf16(64, 192, true), acc);
                mma_bf16(tbase + (16u << 16) + 192, sdesc_k_sw128(p1 + j * 32),
                         sdesc_mn_sw128(vb + 7 * KBS, KBS, 1024), idesc_bf16(64, 64, true), acc);
              }
            }
            mma_commit(&kempty[s]);
            mma_commit(&pvdone[bb]);
            if (i + 1 < ntiles && !qk_next && !issue_qk(gi + 1)) {
              ok = false;
              break;
            }
          }
          g += ntiles;
          ++qn;
        }
      }
    } else if (warp >= 5) {
      // ------------------------------------------------- softmax / output --
      const int quad = warp & 3;
      const int half = lane >> 4;
      const int hl = quad * 16 + (lane & 15);  // head within the block
      const uint32_t trow = tbase + ((uint32_t)(quad * 32) << 16);
      int g = 0;
      for (int item = blockIdx.x; item < a.items; item += gridDim.x) {
        const ItemInfo I = item_info(item);
        const int r = I.r, sp = I.sp, t0 = I.t0, ntiles = I.ntiles;
        const int head = I.hb * 64 + hl;
        if (ntiles == 0) {
          // no keys in this slice: all weight on the sink (or an empty slice)
          if (a.nsplit > 1 && a.cluster) {
            if (half == 0) ml_sm[hl] = make_float2(-INFINITY, 0.f);
          } else if (head < a.n_h) {
            if (a.nsplit == 1) {
              __nv_bfloat16* dst = a.out + ((size_t)r * a.n_h + head) * 512 + half * 256;
              for (int c0 = 0; c0 < 256; c0 += 8) *reinterpret_cast<uint4*>(dst + c0) = zero4();
            } else {
              const size_t slot = ((size_t)sp * a.R + r) * a.n_h + head;
              float* dst = a.ws_o + slot * 512 + half * 256;
              for (int c0 = 0; c0 < 256; c0 += 4)
                *reinterpret_cast<float4*>(dst + c0) = make_float4(0.f, 0.f, 0.f, 0.f);
              if (half == 0) {
                a.ws_ml[slot * 2] = -INFINITY;
                a.ws_ml[slot * 2 + 1] = 0.f;
              }
            }
          }
          continue;
        }
        float m_used = kMasked, l = 0.f;  // running max (base 2) and sum
        bool ok = true;
        for (int i = 0; i < ntiles; ++i) {
          const int gi = g + i;
          const int bb = gi & 1, s = gi % NS;  // S / P buffer, key stage
          const bool mine = half == bb;
          // (every lane of the warp takes the same exit: the loop holds warp
          // collectives)
          if (!__all_sync(0xffffffffu, mbar_wait(&sfull[bb], (gi >> 1) & 1, abort_sm))) {
            ok = false;
            break;
          }
          tc_fence_after();
          float sv[KT];
#pragma unroll
          for (int c = 0; c < KT / 16; ++c) {
            float v[16];
            tmem_ld16(trow + 256 + c * 16, v);
#pragma unroll
            for (int u = 0; u < 16; ++u) sv[c * 16 + u] = v[u];
          }
          if constexpr (FP8) {  // logit = scale_j * (q . codes_j) + q_rope . rope_j, 16 keys at a time
            tmem_wait_ld();
            const float* scl0 = meta_scale + s * 64;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              float v[16];
              tmem_ld16(trow + 320 + c * 16, v);
              tmem_wait_ld();
#pragma unroll
              for (int u = 0; u < 16; ++u) sv[c * 16 + u] = fmaf(scl0[c * 16 + u], sv[c * 16 + u], v[u]);
            }
          }
          tmem_wait_ld();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&sfree[bb]);
          // logits in base-2 units; absent keys get a huge negative logit
          const unsigned long long vmask = meta_mask[s];
          const float* scl = meta_scale + s * 64;
          float mq[4] = {kMasked, kMasked, kMasked, kMasked};  // four short chains
#pragma unroll
          for (int j = 0; j < KT; ++j) {
            const float z = ((vmask >> j) & 1ull) ? a.scale2 * sv[j] : kMasked;
            sv[j] = z;
            mq[j & 3] = fmaxf(mq[j & 3], z);
          }
          const float mt = fmaxf(fmaxf(mq[0], mq[1]), fmaxf(mq[2], mq[3]));
          float alpha = 1.f;
          int resc = 0;
          if (mt > 0.5f * kMasked) {  // the tile has a present key
            if (m_used == kMasked) {
              m_used = mt;
            } else if (mt > m_used + kLazyRescale) {
              alpha = fast_exp2(m_used - mt);
              m_used = mt;
              resc = 1;
            }
          }
          const int src = mine ? lane : (lane ^ 16);
          m_used = __shfl_sync(0xffffffffu, m_used, src);
          alpha = __shfl_sync(0xffffffffu, alpha, src);
          resc = __shfl_sync(0xffffffffu, resc, src);
          if (__any_sync(0xffffffffu, resc)) {
            // O must not be in flight: wait for the previous tile's P V (a
            // rescale needs a present key in an earlier tile of this item)
            if (!__all_sync(0xffffffffu,
                            mbar_wait(&pvdone[(gi - 1) & 1], ((gi - 1) >> 1) & 1, abort_sm))) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t orow = trow + ((uint32_t)(16 * half) << 16);
            for (int c0 = 0; c0 < 256; c0 += 16) {
              float v[16];
              tmem_ld16(orow + c0, v);
              tmem_wait_ld();
#pragma unroll
              for (int u = 0; u < 16; ++u) v[u] *= alpha;
              tmem_st16(orow + c0, v);
            }
            tmem_wait_st();
            tc_fence_before();
          }
          float ls[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int j = 0; j < KT; ++j) {
            const float p = sv[j] > 0.5f * kMasked ? fast_exp2(sv[j] - m_used) : 0.f;
            ls[j & 3] += p;
            sv[j] = p;
          }
          const float lsum = (ls[0] + ls[1]) + (ls[2] + ls[3]);
          l = l * alpha + lsum;
          l = __shfl_sync(0xffffffffu, l, src);
          // P buffer bb was read by the P V of tile gi-2
          if (gi >= 2 &&
              !__all_sync(0xffffffffu, mbar_wait(&pvdone[bb], ((gi - 2) >> 1) & 1, abort_sm))) {
            ok = false;
            break;
          }
          if (mine) {
            uint8_t* prow = sP + bb * L::NP * kPBytes + hl * 128;
#pragma unroll
            for (int c = 0; c < KT / 8; ++c) {
              const int off = ((c ^ (hl & 7)) << 4);
              const float* x = sv + 8 * c;
              const uint4 w1 = make_uint4(pack_bf16(x[0], x[1]), pack_bf16(x[2], x[3]),
                                          pack_bf16(x[4], x[5]), pack_bf16(x[6], x[7]));
              if constexpr (FP8) {
                const float* y = scl + 8 * c;
                const uint4 ws = make_uint4(pack_bf16(x[0] * y[0], x[1] * y[1]),
                                            pack_bf16(x[2] * y[2], x[3] * y[3]),
                                            pack_bf16(x[4] * y[4], x[5] * y[5]),
                                            pack_bf16(x[6] * y[6], x[7] * y[7]));
                st_shared16(prow + off, ws);
                st_shared16(prow + kPBytes + off, w1);
              } else {
                st_shared16(prow + off, w1);
              }
            }
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(&pfull[bb]);
        }
        // ---------------------------------------------------------- output --
        // One slice (nsplit == 1): O rows are normalised with the sink,
        // de-rotated and stored as bf16 straight from registers (the key
        // stages already hold the next query's keys); O is released to the
        // next query's first P V once read.  Several slices in a cluster: the
        // running max and sum go to shared memory and the cluster combines the
        // slices below.  Several slices without a cluster: fp32 partials,
        // staged in the idle key buffers and written by TMA stores, and (max,
        // sum) go to the workspace for attend_combine.
        // (every softmax thread reaches the named barriers below, also after a
        // timed-out wait, so that none of them waits for ever)
        const int glast = g + ntiles - 1;
        g += ntiles;
        const bool fin = ok && mbar_wait(&pvdone[glast & 1], (glast >> 1) & 1, abort_sm);
        tc_fence_after();
        const bool any = m_used > 0.5f * kMasked;
        const uint32_t orow = trow + ((uint32_t)(16 * half) << 16);
        const int brows = a.box_rows;
        const int dim0 = half * 256;
        if (a.nsplit > 1 && a.cluster) {
          named_bar(2, 128);  // every softmax thread is done with the key scales
          if (half == 0) ml_sm[hl] = fin ? make_float2(any ? m_used : -INFINITY, l)
                                         : make_float2(-INFINITY, 0.f);
        } else if (a.nsplit > 1) {
          const bool store = fin && hl < brows;  // head < n_h
          named_bar(2, 128);
          uint8_t* stage = sK;  // 2 x 64 KB, free once the last P V is done
          const int box_bytes = brows * 128;
          const int sw = hl & 7;
          for (int c0 = 0; c0 < 256; c0 += 64) {
            float v[64];
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4)
              tmem_ld16(orow + c0 + q4 * 16, *reinterpret_cast<float(*)[16]>(v + q4 * 16));
            tmem_wait_ld();
            if (!store) continue;
            const int d0 = dim0 + c0;
#pragma unroll
            for (int h2 = 0; h2 < 2; ++h2) {
              uint8_t* rowp = stage + ((d0 >> 5) + h2) * box_bytes + hl * 128;
#pragma unroll
              for (int cc = 0; cc < 8; ++cc) {
                const float* x = v + 32 * h2 + 4 * cc;
                *reinterpret_cast<float4*>(rowp + ((cc ^ sw) << 4)) =
                    make_float4(x[0], x[1], x[2], x[3]);
              }
            }
          }
          fence_proxy_async_smem();
          named_bar(2, 128);
          if (threadIdx.x == 160 && fin) {
            const int row0 = (sp * a.R + r) * a.n_h + I.hb * 64;
            for (int bx = 0; bx < 16; ++bx)
              tma_store_2d(&km.o_ws, stage + bx * box_bytes, bx * 32, row0);
            bulk_commit();
            bulk_wait_read();
          }
          if (hl < brows && half == 0) {  // natural-log max for the combine
            const size_t slot = ((size_t)sp * a.R + r) * a.n_h + head;
            a.ws_ml[slot * 2] = (fin && any) ? m_used * kLn2 : -INFINITY;
            a.ws_ml[slot * 2 + 1] = fin ? l : 0.f;
          }
        } else {
          if (warp == 5) {  // R_{-t0} of the 32 RoPE pairs
            float cs, sn;
            rope_cs(-(double)t0, lane, 64, a.base, &cs, &sn);
            rope_tab[2 * lane] = cs;
            rope_tab[2 * lane + 1] = sn;
          }
          const float zs = hl < brows ? a.sink[head] * kLog2e : 0.f;
          const float M = fmaxf(any ? m_used : zs, zs);
          const float em = any ? fast_exp2(m_used - M) : 0.f;
          const float f = em / (l * em + fast_exp2(zs - M));
          if (!fin) *ostop_sm = 1;
          named_bar(2, 128);  // the RoPE table is written; the stop flag is final
          const bool quit = *ostop_sm;
          const bool store = fin && hl < brows;  // head < n_h
          __nv_bfloat16* orow_g = a.out + ((size_t)r * a.n_h + head) * 512;
          for (int c0 = 0; c0 < 256; c0 += 64) {
            float v[64];
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4)
              tmem_ld16(orow + c0 + q4 * 16, *reinterpret_cast<float(*)[16]>(v + q4 * 16));
            tmem_wait_ld();
            if (c0 == 192) {  // O is in registers: the next query's P V may start
              tc_fence_before();
              __syncwarp();
              if (lane == 0) mbar_arrive(oempty);
            }
            if (!store) continue;
            const int d0 = dim0 + c0;
#pragma unroll
            for (int u = 0; u < 64; ++u) v[u] *= f;
            if (d0 >= 448) {  // RoPE dims
#pragma unroll
              for (int u = 0; u < 64; u += 2) {
                const float cs = rope_tab[u], sn = rope_tab[u + 1];
                const float x0 = v[u], x1 = v[u + 1];
                v[u] = x0 * cs - x1 * sn;
                v[u + 1] = x0 * sn + x1 * cs;
              }
            }
            uint4* dst = reinterpret_cast<uint4*>(orow_g + d0);
#pragma unroll
            for (int cc = 0; cc < 8; ++cc) {
              const float* x = v + 8 * cc;
              __stcs(dst + cc, make_uint4(pack_bf16(x[0], x[1]), pack_bf16(x[2], x[3]),
                                          pack_bf16(x[4], x[5]), pack_bf16(x[6], x[7])));
            }
          }
          named_bar(2, 128);  // the RoPE table and the stop flag are reused
          if (quit) break;
        }
      }
    }
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (a.nsplit > 1 && a.cluster) {
    // --------------------------------------------- slice combine (cluster) --
    // The CTAs of the cluster hold the key slices of one (query, head
    // block), CTA rank = slice.  Each CTA weighs its O by its share of the
    // softmax (running maxima and sums read from every CTA through
    // distributed shared memory, sink included), stages it in its idle key
    // buffers, and CTA c sums heads [h0, h1) over the cluster, applies
    // R_{-t0} and stores bf16 O.
    const ItemInfo I0 = item_info(blockIdx.x);  // one item per CTA in a cluster
    const int ntiles = I0.ntiles, t0 = I0.t0, sp = I0.sp, hb = I0.hb, r = I0.r;
    const int S = a.nsplit;
    const int brows = a.box_rows;
    if (threadIdx.x == 0) valid_sm = (ntiles > 0 && !*abort_sm) ? 1 : 0;
    if (warp == 4) {  // R_{-t0} of the 32 RoPE pairs
      float cs, sn;
      rope_cs(-(double)t0, lane, 64, a.base, &cs, &sn);
      rope_tab[2 * lane] = cs;
      rope_tab[2 * lane + 1] = sn;
    }
    __syncwarp();
    cluster_sync_all();  // maxima, sums and flags of every slice are visible
    unsigned live = 0;   // slices that hold keys (and did not time out)
    for (int p = 0; p < S; ++p) {
      int vp;
      asm volatile("ld.shared::cluster.u32 %0, [%1];"
                   : "=r"(vp)
                   : "r"(mapa_shared(smem_u32(&valid_sm), p))
                   : "memory");
      live |= (vp ? 1u : 0u) << p;
    }
    uint8_t* stage = sK;  // [64 heads][512] fp32, 16-byte chunks swizzled by head
    if (warp >= 5 && ((live >> sp) & 1u)) {
      const int quad = warp & 3, half = lane >> 4;
      const int hl = quad * 16 + (lane & 15);
      const bool hv = hl < brows;  // head < n_h
      const float zs = hv ? a.sink[hb * 64 + hl] * kLog2e : 0.f;
      const uint32_t mla = smem_u32(&ml_sm[hl]);
      float2 mlp[kMaxSlices];
      float M = zs;
#pragma unroll
      for (int p = 0; p < kMaxSlices; ++p) {
        mlp[p] = (p < S && ((live >> p) & 1u)) ? ld_dsmem_f2(mapa_shared(mla, p))
                                               : make_float2(-INFINITY, 0.f);
        M = fmaxf(M, mlp[p].x);
      }
      float den = fast_exp2(zs - M);
#pragma unroll
      for (int p = 0; p < kMaxSlices; ++p)
        den += mlp[p].x > -INFINITY ? mlp[p].y * fast_exp2(mlp[p].x - M) : 0.f;
      const float2 mine = ml_sm[hl];
      const float f = mine.x > -INFINITY ? fast_exp2(mine.x - M) / den : 0.f;
      const uint32_t orow = tbase + ((uint32_t)(quad * 32 + 16 * half) << 16);
      uint8_t* rowp = stage + hl * 2048;
      for (int c0 = 0; c0 < 256; c0 += 64) {
        float v[64];
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4)
          tmem_ld16(orow + c0 + q4 * 16, *reinterpret_cast<float(*)[16]>(v + q4 * 16));
        tmem_wait_ld();
#pragma unroll
        for (int cc = 0; cc < 16; ++cc) {  // 16-byte chunk of dims half*256 + c0 + 4cc
          const int ch = (half * 256 + c0) / 4 + cc;
          const int off = (ch >> 3) * 128 + (((ch & 7) ^ (hl & 7)) << 4);
          *reinterpret_cast<float4*>(rowp + off) =
              make_float4(v[4 * cc] * f, v[4 * cc + 1] * f, v[4 * cc + 2] * f, v[4 * cc + 3] * f);
        }
      }
    }
    tc_fence_before();
    __syncwarp();
    cluster_sync_all();  // weighted slices are staged
    {
      const int hper = (brows + S - 1) / S;
      const int h0 = sp * hper, h1 = min(brows, h0 + hper);
      const uint32_t sbase = smem_u32(stage);
      for (int it = threadIdx.x; it < (h1 - h0) * 128; it += kAtThreads) {
        const int h = h0 + (it >> 7), ch = it & 127;  // 16-byte chunk: dims 4ch .. 4ch+3
        const uint32_t off = sbase + h * 2048 + (ch >> 3) * 128 + (((ch & 7) ^ (h & 7)) << 4);
        float4 x[kMaxSlices];  // all peers' chunks in flight, then the sum
#pragma unroll
        for (int p = 0; p < kMaxSlices; ++p)
          x[p] = (p < S && ((live >> p) & 1u)) ? ld_dsmem_f4(mapa_shared(off, p))
                                               : make_float4(0.f, 0.f, 0.f, 0.f);
        float4 acc = x[0];
#pragma unroll
        for (int p = 1; p < kMaxSlices; ++p) {
          acc.x += x[p].x; acc.y += x[p].y; acc.z += x[p].z; acc.w += x[p].w;
        }
        const int d = ch * 4;
        if (d >= 448) {  // RoPE dims: pairs (d, d+1), (d+2, d+3)
          const int pr = (d - 448) >> 1;
          const float c0 = rope_tab[2 * pr], s0 = rope_tab[2 * pr + 1];
          const float c1 = rope_tab[2 * pr + 2], s1 = rope_tab[2 * pr + 3];
          const float x0 = acc.x, x1 = acc.y, x2 = acc.z, x3 = acc.w;
          acc.x = x0 * c0 - x1 * s0;
          acc.y = x0 * s0 + x1 * c0;
          acc.z = x2 * c1 - x3 * s1;
          acc.w = x2 * s1 + x3 * c1;
        }
        __nv_bfloat16* dst = a.out + ((size_t)r * a.n_h + hb * 64 + h) * 512 + d;
        *reinterpret_cast<uint2*>(dst) = make_uint2(pack_bf16(acc.x, acc.y), pack_bf16(acc.z, acc.w));
      }
    }
    __syncwarp();
    cluster_sync_all();  // no CTA leaves while its staged slice is read
    tc_fence_after();
  }
  if (*abort_sm) {
    if (threadIdx.x == 0) atomicOr(a.err, CSA_DEV_TIMEOUT);
    const uint64_t t0w = globaltimer();
    while (globaltimer() - t0w < 200000ull) __nanosleep(1000);
  }
  pdl_trigger();  // the slice combine may be scheduled as this grid retires
  if (warp == 4) tmem_dealloc(tbase, 512);
}

// ------------------------------------------------------------------ host --
bool make_tmap_bf16(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols,
                    uint32_t box_rows);
bool make_tmap_f32(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols,
                   uint32_t box_rows);
bool tma_available();

bool attend_tc_supported(const csa_params& p) {
  return p.act == CSA_BF16 && (p.kv == CSA_BF16 || p.kv == CSA_KV_FP8MIX) && p.c == 512 &&
         p.rope_dims == 64 && p.n_h % 16 == 0 && (p.n_h <= 64 || p.n_h % 64 == 0) &&
         tma_available();
}

// Key slices per (query, head block): at most one wave of CTAs (148 SMs, one
// CTA each).  Up to kMaxSlices slices are launched as a cluster and combined
// in the kernel; more slices write partials for attend_combine.
// keys per tile of the kernel instance that serves these parameters
constexpr int kKtFp8 = 64, kNsFp8 = 2;   // FP8-mixed cache
constexpr int kKtBf16 = 48, kNsBf16 = 3;  // bf16 cache
static int tile_keys(const csa_params& p) { return p.kv == CSA_KV_FP8MIX ? kKtFp8 : kKtBf16; }

template <bool FP8, int KT, int NS>
static int max_active_clusters_t(int csize) {
  const int smem = AtLayout<FP8, KT, NS>::total + 1024;
  if (!set_kernel_smem((const void*)attend_tc<FP8, KT, NS>, smem)) return 0;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(csize * 148);
  cfg.blockDim = dim3(kAtThreads);
  cfg.dynamicSmemBytes = (size_t)smem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)csize;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, attend_tc<FP8, KT, NS>, &cfg) != cudaSuccess) {
    cudaGetLastError();
    n = 0;
  }
  return n;
}

// clusters of `csize` attention CTAs that fit on the current GPU at once
static int max_active_clusters(bool fp8, int csize) {
  static int cache[64][2][kMaxSlices + 1];
  static bool have[64][2][kMaxSlices + 1];
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64 || csize < 1 || csize > kMaxSlices) return 0;
  if (!have[dev][fp8][csize]) {
    cache[dev][fp8][csize] = fp8 ? max_active_clusters_t<true, kKtFp8, kNsFp8>(csize)
                                 : max_active_clusters_t<false, kKtBf16, kNsBf16>(csize);
    have[dev][fp8][csize] = true;
  }
  return cache[dev][fp8][csize];
}

// most key slices per (query, head block); a build may lower it
#ifndef CSA_ATTN_MAX_SPLIT
#define CSA_ATTN_MAX_SPLIT 256
#endif

void attend_tc_plan(const csa_params& p, int R, int N, bool dense, int* nsplit, int* kps,
                    int* cluster) {
  const int hbn = (p.n_h + 63) / 64;
  const int base = R * hbn;
  const int nk_max = (dense ? N : p.topk) + p.n_win;
  const int KT = tile_keys(p);
  const int ntiles = (nk_max + KT - 1) / KT;
  int s = base >= 148 ? 1 : 148 / base;
  if (s > ntiles) s = ntiles;
  if (s > CSA_ATTN_MAX_SPLIT) s = CSA_ATTN_MAX_SPLIT;
  if (s < 1) s = 1;
  int k = (nk_max + s - 1) / s;
  k = (k + KT - 1) / KT * KT;
  if (k < KT) k = KT;
  *kps = k;
  *nsplit = nk_max > 0 ? (nk_max + k - 1) / k : 1;
  // clusters only if all of them fit on the GPU at once (clusters of CTAs
  // this large are placed whole within a GPC: 16 clusters of 8 took two waves)
  *cluster = *nsplit > 1 && *nsplit <= kMaxSlices &&
             base <= max_active_clusters(p.kv == CSA_KV_FP8MIX, *nsplit);
}

// one CTA per (query, head block, key slice); the slices of one (query, head
// block) are launched as a cluster
template <bool FP8, int KT, int NS>
static cudaError_t launch_attend_kernel(unsigned items, int smem, int cluster, cudaStream_t st,
                                        const CUtensorMap& tmQ, const KeyMaps& km,
                                        const AttnTcArgs& a) {
  if (!set_kernel_smem((const void*)attend_tc<FP8, KT, NS>, smem)) return cudaErrorInvalidValue;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(items);
  cfg.blockDim = dim3(kAtThreads);
  cfg.dynamicSmemBytes = (size_t)smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  unsigned na = 0;
  if (cluster > 1) {
    attr[na].id = cudaLaunchAttributeClusterDimension;
    attr[na].val.clusterDim.x = (unsigned)cluster;
    attr[na].val.clusterDim.y = 1;
    attr[na].val.clusterDim.z = 1;
    ++na;
  }
  if (kPdlAttend) {
    attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  return cudaLaunchKernelEx(&cfg, attend_tc<FP8, KT, NS>, tmQ, km, a);
}

csa_status launch_attend_tc(const csa_params& p, bool dense, int B, int Q,
                            const int32_t* q_pos, const void* q, const int32_t* idx,
                            const void* ckv, const float* ckv_scale, int N, const void* win,
                            const float* win_scale, int W, const int32_t* win_pos0,
                            const float* sink, void* out, float* ws_o, float* ws_ml,
                            int nsplit, int kps, int cluster, cudaStream_t st) {
  const int R = B * Q;
  const int hbn = (p.n_h + 63) / 64;
  CUtensorMap tmQ;
  if (!make_tmap_bf16(&tmQ, q, (uint64_t)R * p.n_h, 512, 64)) return CSA_ERR_CUDA;
  AttnTcArgs a{};
  a.q_pos = q_pos; a.idx = idx; a.ckv = (const uint8_t*)ckv; a.ckv_scale = ckv_scale;
  a.win = (const uint8_t*)win; a.win_scale = win_scale; a.win_pos0 = win_pos0; a.sink = sink;
  a.out = (__nv_bfloat16*)out; a.ws_o = ws_o; a.ws_ml = ws_ml; a.err = device_error_word();
  a.cluster = cluster;
  a.Q = Q; a.N = N; a.W = W; a.n_h = p.n_h; a.m = p.m; a.topk = p.topk; a.n_win = p.n_win;
  a.nsplit = nsplit; a.keys_per_split = kps; a.dense = dense ? 1 : 0; a.R = R; a.hblocks = hbn;
  a.scale2 = p.softmax_scale * kLog2e; a.base = (double)p.rope_base;
  if (a.err == nullptr) return CSA_ERR_CUDA;
  const long long items = (long long)R * hbn * nsplit;
  a.items = (int)items;
  // one slice per query: a persistent grid of one CTA per SM walks the items
  const long long grid = (nsplit == 1 && !cluster && items > sm_count()) ? sm_count() : items;
  KeyMaps km;
  memset(&km, 0, sizeof(km));
  a.R_rows_c = B * N;
  a.R_rows_w = B * W;
  if (p.kv == CSA_BF16) {
    // a tensor map needs at least one row: an empty cache / window borrows
    // the other's memory (its rows are never used)
    const void* cbase = N > 0 ? ckv : win;
    const void* wbase = (W > 0 && win) ? win : ckv;
    const uint64_t crows = N > 0 ? (uint64_t)B * N : (uint64_t)B * W;
    const uint64_t wrows = (W > 0 && win) ? (uint64_t)B * W : (uint64_t)B * N;
    if (crows == 0 || wrows == 0) return CSA_ERR_UNSUPPORTED;
    if (!make_tmap_bf16(&km.c_box, cbase, crows, 512, kKtBf16) ||
        !make_tmap_bf16(&km.c_row, cbase, crows, 512, 1) ||
        !make_tmap_bf16(&km.w_box, wbase, wrows, 512, kKtBf16) ||
        !make_tmap_bf16(&km.w_row, wbase, wrows, 512, 1))
      return CSA_ERR_CUDA;
    a.R_rows_c = (int)crows;
    a.R_rows_w = (int)wrows;
  }
  a.box_rows = p.n_h < 64 ? p.n_h : 64;
  if (nsplit > 1 && !cluster &&
      !make_tmap_f32(&km.o_ws, ws_o, (uint64_t)nsplit * R * p.n_h, 512, (uint32_t)a.box_rows))
    return CSA_ERR_CUDA;
  if (nsplit < 1 || (cluster && nsplit > kMaxSlices)) return CSA_ERR_UNSUPPORTED;
  const int cl = cluster ? nsplit : 1;
  cudaError_t e;
  if (p.kv == CSA_KV_FP8MIX)
    CSA_LAUNCH(KK_ATTN, st,
               e = launch_attend_kernel<true, kKtFp8, kNsFp8>(
                   (unsigned)grid, AtLayout<true, kKtFp8, kNsFp8>::total + 1024,
                                              cl, st, tmQ, km, a));
  else
    CSA_LAUNCH(KK_ATTN, st,
               e = launch_attend_kernel<false, kKtBf16, kNsBf16>(
                   (unsigned)grid, AtLayout<false, kKtBf16, kNsBf16>::total + 1024,
                                               cl, st, tmQ, km, a));
  return e == cudaSuccess ? CSA_OK : CSA_ERR_CUDA;
}

}  // namespace csa
