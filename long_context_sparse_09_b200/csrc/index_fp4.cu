// index_fp4.cu -- Lightning-Indexer scores with the QK path in MXFP4 and the
// scores in bf16 ("02 · DeepSeek-V4: 压缩注意力撑起 1M 上下文" section 3.3), and
// the quantiser of indexer keys into that format.
//
// Key cache format (MXFP4, OCP Microscaling): per row of c_I = 128 values,
// 64 bytes of E2M1 codes (element 2j in the low nibble of byte j, 2j+1 in the
// high nibble) in one plane, and 4 E8M0 scale bytes (2^(s - 127) for each
// block of 32 consecutive values) in a second plane.  A block's scale is
// 2^(floor(log2 max|x|) - 2) and its elements are x / scale rounded to the
// nearest E2M1 value (ties to even, saturating at 6).
//
// Scorer, per 128-entry tile: the codes (8 KB) arrive by TMA and their scale
// words by 4-byte cp.async into a ring of shared-memory stages; four dequant
// warps, one thread per entry, turn each E2M1 pair into an f16 pair with the
// hardware conversion, multiply by the block's 2^e (exact) and store the row
// straight into tensor memory as the MMA's A operand -- the 32 KB of f16 keys
// never touch shared memory, which holds only the codes and the query.  The
// MMA warp computes D[128 entries][n_hI] = K^I_tile q^T with A from TMEM and
// the query (q^I rounded to MXFP4 per head and block, same f16 form) from
// shared memory; the products and their sums are exact in the fp32
// accumulator for these operands.  Eight epilogue warps (two groups taking
// alternate tiles) apply ReLU, w and the head sum in fp32 and round the score
// to bf16; the scores go to the fp32 workspace the top-k reads.
#include <cuda.h>

#include "common.cuh"
#include "index_common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace csa {

using namespace sm100;

constexpr int kF4CI = 128;                           // indexer key width of this path
constexpr int kF4CodeBytes = kF4CI / 2;              // 64 B of codes per entry
constexpr int kF4Blocks = kF4CI / 32;                // 4 scale bytes per entry
constexpr int kF4SC = 8;                             // code stages
constexpr int kF4SA = 4;                             // f16 key stages in TMEM
constexpr int kF4Acc = 4;                            // accumulators in TMEM
constexpr int kF4CodeTile = kTileM * kF4CodeBytes;   // 8 KB
constexpr int kF4ScaleTile = kTileM * kF4Blocks;     // 512 B
constexpr int kF4QSlot = 64 * kF4CI * 2;             // 16 KB: up to 64 heads x 128 f16
constexpr int kF4Threads = 448;  // warp 0 loads, 1 MMA, 2-5 dequant, 6-13 epilogue
constexpr int kF4ColA = kF4Acc * 64;                 // TMEM columns of the key stages
// block exponents whose E2M1 values are exact f16 numbers: 6 * 2^13 <= 65504
// and 0.5 * 2^-23 is a multiple of the smallest f16 subnormal 2^-24
constexpr int kF4ExpLo = -23, kF4ExpHi = 13;

struct IdxF4Args {
  const int32_t* q_pos;
  const __nv_bfloat16* qI;  // [R][n_hI][128]
  const float* w;           // [R][n_hI]
  const uint8_t* kscale;    // [B*N][4] E8M0
  const int* prefix;        // [ngroups + 1] tiles per query, or null (computed inline)
  float* scores;            // [R][N]
  unsigned* err;
  unsigned* ghist;          // [R][4096] key histograms for the multi-CTA top-k, or null
  long long rows;           // B*N
  int Q, N, m, nhI, ngroups, stream_keys;
};

// ------------------------------------------------------------- helpers --
// 4-byte global -> shared copy; src_bytes = 0 writes zeros without reading.
__device__ __forceinline__ void cp_async4(void* dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(smem_u32(dst)), "l"(src),
               "r"(src_bytes)
               : "memory");
}

// Eight E2M1 codes (one 32-bit word, element 2j in the low nibble of byte j)
// -> four f16 pairs (low half = the even element), by the hardware
// conversion.
__device__ __forceinline__ void e2m1x8_to_f16x8(uint32_t w, uint32_t& o0, uint32_t& o1,
                                                uint32_t& o2, uint32_t& o3) {
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t"
      "cvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
      "cvt.rn.f16x2.e2m1x2 %2, b2;\n\t"
      "cvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
      : "=r"(o0), "=r"(o1), "=r"(o2), "=r"(o3)
      : "r"(w));
}

__device__ __forceinline__ uint32_t mul_f16x2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// f16 bit pattern of 2^e, kF4ExpLo <= e <= kF4ExpHi (subnormal below 2^-14)
__device__ __forceinline__ uint32_t f16_pow2_bits(int e) {
  return e >= -14 ? (uint32_t)(e + 15) << 10 : 1u << (e + 24);
}

// 2^k as a float, -149 <= k <= 127 (exact; subnormal below 2^-126).
__device__ __forceinline__ float pow2f(int k) {
  return k >= -126 ? __int_as_float((k + 127) << 23) : __int_as_float(1 << (k + 149));
}

// The E2M1 value nearest to a = |x| / scale in [0, 8): the grid step is 0.5
// below 2, 1 below 4 and 2 above; ties go to the even multiple of the step
// (the even mantissa); 6 is the largest value.  (Scaling by the inverse
// step and back is exact: both are powers of two.)
__device__ __forceinline__ float e2m1_round(float a) {
  const float inv = a < 2.f ? 2.f : (a < 4.f ? 1.f : 0.5f);
  const float step = a < 2.f ? 0.5f : (a < 4.f ? 1.f : 2.f);
  return fminf(rintf(a * inv) * step, 6.f);
}

// MXFP4 block exponent of a block whose largest magnitude is amax:
// floor(log2 amax) - 2, or -127 for an all-zero block.
__device__ __forceinline__ int mx_block_exp(float amax) {
  if (!(amax > 0.f)) return -127;
  int ex;
  frexpf(amax, &ex);  // amax = f 2^ex, f in [0.5, 1)
  const int e = ex - 3;
  return e < -127 ? -127 : (e > 127 ? 127 : e);
}

// D[tmem] (+)= A[tmem] * B[smem desc]^T, f16 inputs, fp32 accumulate.
__device__ __forceinline__ void mma_f16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc,
                                           uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Instruction descriptor of kind::f16 with f16 A and B, fp32 D, both K-major.
__host__ __device__ constexpr uint32_t idesc_f16(int M, int N) {
  return (1u << 4) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// ------------------------------------------------------------- scorer --
__global__ void __launch_bounds__(kF4Threads, 1)
    index_scores_fp4(const __grid_constant__ CUtensorMap tmC, IdxF4Args a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* qsl = smem;                              // 2 query slots
  uint8_t* cst = qsl + 2 * kF4QSlot;                // kF4SC code stages
  uint8_t* sst = cst + kF4SC * kF4CodeTile;         // kF4SC scale stages
  uint64_t* bars = (uint64_t*)(sst + kF4SC * kF4ScaleTile);
  uint64_t* cfull = bars;
  uint64_t* cempty = cfull + kF4SC;
  uint64_t* afull = cempty + kF4SC;
  uint64_t* aempty = afull + kF4SA;
  uint64_t* qfull = aempty + kF4SA;
  uint64_t* qempty = qfull + 2;
  uint64_t* tfull = qempty + 2;
  uint64_t* tempty = tfull + kF4Acc;
  uint32_t* tbase_sm = (uint32_t*)(tempty + kF4Acc);
  volatile int* abort_sm = (volatile int*)(tbase_sm + 1);
  unsigned* shist = (unsigned*)((uint8_t*)bars + 512);  // [kHistBins]
  int* s_prefix = (int*)(shist + kHistBins);            // [kInlineGroups + 1]
  float* s_w = (float*)(s_prefix + 80);                 // [2][64] head weights per slot

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nhI = a.nhI;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kF4SC; ++i) {
      mbar_init(&cfull[i], 1 + 32);  // the TMA's expect_tx + 32 lanes' cp.async
      mbar_init(&cempty[i], 4);      // the four dequant warps
    }
    for (int i = 0; i < kF4SA; ++i) {
      mbar_init(&afull[i], 4);
      mbar_init(&aempty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&qfull[i], 128);  // every dequant thread
      mbar_init(&qempty[i], 1 + 8);  // the MMA's commit + the eight epilogue warps
    }
    for (int i = 0; i < kF4Acc; ++i) {
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], 4);  // the epilogue warp group of the tile
    }
    *abort_sm = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tbase_sm, 512);
    tmem_relinquish();
  }
  if (threadIdx.x == 32) prefetch_tmap(&tmC);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tbase_sm;

  if (a.prefix == nullptr) {  // tiles of each query (threads 0..63) and their prefix
    if (threadIdx.x < kInlineGroups) {
      const int g = threadIdx.x;
      int tiles = 0;
      if (g < a.ngroups) tiles = (n_visible(__ldg(a.q_pos + g), a.m, a.N) + kTileM - 1) / kTileM;
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
    if (warp == 0) {
      // ----------------------------------------------------------- loads --
      TileCursor cur;
      cur.init(prefix, a.ngroups, start, count);
      const uint64_t pol = l2_evict_first_policy();
      for (int i = 0; i < count; ++i) {
        const int s = i % kF4SC;
        if (!mbar_wait(&cempty[s], ((i / kF4SC) & 1) ^ 1, abort_sm)) break;
        const long long row0 = (long long)(cur.g / a.Q) * a.N + (long long)cur.t * kTileM;
        if (lane == 0) {
          mbar_expect_tx(&cfull[s], (uint32_t)kF4CodeTile);
          if (a.stream_keys)
            tma_load_2d_hint(cst + s * kF4CodeTile, &tmC, &cfull[s], 0, (int)row0, pol);
          else
            tma_load_2d(cst + s * kF4CodeTile, &tmC, &cfull[s], 0, (int)row0);
        }
        // the scale words of rows 4 lane .. 4 lane + 3 (zeros past the cache)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const long long row = row0 + lane * 4 + j;
          const bool in = row < a.rows;
          cp_async4(sst + s * kF4ScaleTile + (lane * 4 + j) * 4, a.kscale + (in ? row : 0) * 4,
                    in ? 4u : 0u);
        }
        cp_async_arrive(&cfull[s]);
        cur.next(prefix, a.ngroups);
      }
    } else if (warp == 1 && lane == 0) {
      // ------------------------------------------------------------ MMA --
      TileCursor cur;
      cur.init(prefix, a.ngroups, start, count);
      const uint32_t idesc = idesc_f16(kTileM, nhI);
      int qn = 0;
      for (int i = 0; i < count; ++i) {
        const bool first = cur.first(i), last = cur.last(prefix);
        const int slot = qn & 1;
        if (first && !mbar_wait(&qfull[slot], (qn >> 1) & 1, abort_sm)) break;
        const int sa = i % kF4SA;
        if (!mbar_wait(&afull[sa], (i / kF4SA) & 1, abort_sm)) break;
        const int acc = i % kF4Acc;
        if (!mbar_wait(&tempty[acc], ((i / kF4Acc) & 1) ^ 1, abort_sm)) break;
        tc_fence_after();
        const uint32_t d = tbase + acc * 64;
        const uint32_t at = tbase + kF4ColA + sa * 64;
        const uint32_t bbase = smem_u32(qsl + slot * kF4QSlot);
#pragma unroll
        for (int j = 0; j < 8; ++j)  // K = 16 per product: 8 TMEM columns of f16 pairs
          mma_f16_ts(d, at + 8 * j, sdesc_k_sw128(bbase + (j >> 2) * nhI * 128 + (j & 3) * 32),
                     idesc, j != 0);
        mma_commit(&aempty[sa]);
        mma_commit(&tfull[acc]);
        if (last) {
          mma_commit(&qempty[slot]);
          ++qn;
        }
        cur.next(prefix, a.ngroups);
      }
    } else if (warp >= 2 && warp < 6) {
      // ------------------------------------------------------- dequant --
      const int quad = warp & 3;          // TMEM lane quadrant
      const int row = quad * 32 + lane;   // the entry of the tile this thread converts
      const int dt = threadIdx.x - 64;    // 0..127
      // the code tile arrives in the 64-byte swizzle: 16-byte chunk c of row r
      // sits at chunk c ^ ((r >> 1) & 3), so 8 consecutive rows reading the
      // same chunk hit 8 different bank groups
      const int swz = (row >> 1) & 3;
      TileCursor cur;
      cur.init(prefix, a.ngroups, start, count);
      int qn = 0;
      bool range_err = false;
      for (int i = 0; i < count; ++i) {
        if (cur.first(i)) {
          // the query of this group: q^I rounded to MXFP4 per head and block
          // of 32, as exact f16 values in the 128-byte swizzled K-major slot
          const int slot = qn & 1;
          // (the warp leaves together: the loop holds warp collectives)
          if (!__all_sync(0xffffffffu, mbar_wait(&qempty[slot], ((qn >> 1) & 1) ^ 1, abort_sm)))
            break;
          uint8_t* qs = qsl + slot * kF4QSlot;
          const int r = cur.g;
          for (int it = dt; it < nhI * kF4Blocks; it += 128) {
            const int h = it >> 2, blk = it & 3;
            const uint4* src = reinterpret_cast<const uint4*>(
                a.qI + ((size_t)r * nhI + h) * kF4CI + blk * 32);
            float x[32];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const uint4 v = __ldg(src + u);
              const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                x[8 * u + 2 * k] = __uint_as_float(wv[k] << 16);
                x[8 * u + 2 * k + 1] = __uint_as_float(wv[k] & 0xFFFF0000u);
              }
            }
            float amax = 0.f;
#pragma unroll
            for (int k = 0; k < 32; ++k) amax = fmaxf(amax, fabsf(x[k]));
            int e = mx_block_exp(amax);
            if (amax > 0.f && (e < kF4ExpLo || e > kF4ExpHi)) {
              range_err = true;
              e = e < kF4ExpLo ? kF4ExpLo : kF4ExpHi;
            }
            const int ed = amax > 0.f ? e : 0;
            const float down = pow2f(-ed), up = pow2f(ed);
            uint32_t hv[16];
#pragma unroll
            for (int k = 0; k < 16; ++k) {
              float v2[2];
#pragma unroll
              for (int z = 0; z < 2; ++z) {
                const float xv = x[2 * k + z];
                const float qv = e2m1_round(fabsf(xv) * down);
                v2[z] = (xv < 0.f && qv > 0.f ? -qv : qv) * up;
              }
              const __half2 hh = __floats2half2_rn(v2[0], v2[1]);
              hv[k] = *reinterpret_cast<const uint32_t*>(&hh);
            }
            const int kb = blk >> 1;
            uint8_t* dst = qs + kb * nhI * 128 + (h >> 3) * 1024 + (h & 7) * 128;
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const int chunk = (blk & 1) * 4 + u;
              *reinterpret_cast<uint4*>(dst + ((chunk ^ (h & 7)) << 4)) =
                  make_uint4(hv[4 * u], hv[4 * u + 1], hv[4 * u + 2], hv[4 * u + 3]);
            }
          }
          if (dt < nhI) s_w[slot * 64 + dt] = __ldg(a.w + (size_t)r * nhI + dt);
          fence_proxy_async_smem();
          mbar_arrive(&qfull[slot]);
          ++qn;
        }
        const int s = i % kF4SC;
        if (!__all_sync(0xffffffffu, mbar_wait(&cfull[s], (i / kF4SC) & 1, abort_sm))) break;
        const int sa = i % kF4SA;
        if (!__all_sync(0xffffffffu, mbar_wait(&aempty[sa], ((i / kF4SA) & 1) ^ 1, abort_sm)))
          break;
        tc_fence_after();
        const uint8_t* crow = cst + s * kF4CodeTile + row * kF4CodeBytes;
        const uint32_t sw = *reinterpret_cast<const uint32_t*>(sst + s * kF4ScaleTile + row * 4);
        const uint32_t ta = tbase + ((uint32_t)(quad * 32) << 16) + kF4ColA + sa * 64;
        // block c of the row -> TMEM columns 16c .. 16c+15 (the column of a
        // tcgen05.st is the same for every lane of the warp)
#pragma unroll
        for (int c = 0; c < kF4Blocks; ++c) {
          const uint4 q = *reinterpret_cast<const uint4*>(crow + ((c ^ swz) << 4));
          int e = (int)((sw >> (8 * c)) & 0xFFu) - 127;
          if (e < kF4ExpLo || e > kF4ExpHi) {
            if (q.x | q.y | q.z | q.w) range_err = true;
            e = e < kF4ExpLo ? kF4ExpLo : kF4ExpHi;
          }
          const uint32_t sb = f16_pow2_bits(e);
          const uint32_t s2 = sb | (sb << 16);
          const uint32_t qw[4] = {q.x, q.y, q.z, q.w};
          float v[16];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            uint32_t o0, o1, o2, o3;
            e2m1x8_to_f16x8(qw[u], o0, o1, o2, o3);
            v[4 * u] = __uint_as_float(mul_f16x2(o0, s2));
            v[4 * u + 1] = __uint_as_float(mul_f16x2(o1, s2));
            v[4 * u + 2] = __uint_as_float(mul_f16x2(o2, s2));
            v[4 * u + 3] = __uint_as_float(mul_f16x2(o3, s2));
          }
          tmem_st16(ta + 16 * c, v);  // columns 16c .. 16c+15: values 32c .. 32c+31
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&cempty[s]);
          mbar_arrive(&afull[sa]);
        }
        cur.next(prefix, a.ngroups);
      }
      if (range_err) atomicOr(a.err, CSA_DEV_RANGE);
    } else if (warp >= 6) {
      // ------------------------------------------------------- epilogue --
      const int e8 = warp - 6;
      const int quad = warp & 3;
      const int alt = e8 >> 2;  // this warp group's tile parity
      const int et = threadIdx.x - 192;  // 0..255
      const bool hist = a.ghist != nullptr;
      if (hist) {
        for (int k = et; k < kHistBins; k += 256) shist[k] = 0u;
        named_bar(2, 256);
      }
      // After a wait gives up the warp keeps walking the list without work,
      // so that all eight warps take the same named barriers.
      TileCursor cur;
      cur.init(prefix, a.ngroups, start, count);
      int qn = 0, hist_r = cur.g, nv = 0;
      bool dead = false;
      for (int i = 0; i < count; ++i) {
        const bool first = cur.first(i), last = cur.last(prefix);
        const int slot = qn & 1;
        if (first) {
          if (!dead) dead = !__all_sync(0xffffffffu, mbar_wait(&qfull[slot], (qn >> 1) & 1, abort_sm));
          nv = n_visible(__ldg(a.q_pos + cur.g), a.m, a.N);
        }
        if (hist && cur.g != hist_r) {  // query changed: flush its histogram
          named_bar(2, 256);
          for (int bin = et; bin < kHistBins; bin += 256) {
            const unsigned c = shist[bin];
            if (c) {
              atomicAdd(&a.ghist[(size_t)hist_r * kHistBins + bin], c);
              shist[bin] = 0u;
            }
          }
          named_bar(2, 256);
          hist_r = cur.g;
        }
        if ((i & 1) == alt && !dead)
          dead = !__all_sync(0xffffffffu, mbar_wait(&tfull[i % kF4Acc], (i / kF4Acc) & 1, abort_sm));
        if ((i & 1) == alt && !dead) {
          const int acc = i % kF4Acc;
          tc_fence_after();
          const uint32_t trow = tbase + ((uint32_t)(quad * 32) << 16) + acc * 64;
          const float4* w4 = reinterpret_cast<const float4*>(s_w + slot * 64);
          float part[4] = {0.f, 0.f, 0.f, 0.f};
          float v[4][16];
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4)
            if (q4 * 16 < nhI) tmem_ld16(trow + q4 * 16, v[q4]);
          tmem_wait_ld();
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            if (q4 * 16 >= nhI) continue;
#pragma unroll
            for (int j4 = 0; j4 < 4; ++j4) {
              const float4 ww = w4[q4 * 4 + j4];
              part[q4] = fmaf(ww.x, fmaxf(v[q4][4 * j4 + 0], 0.f), part[q4]);
              part[q4] = fmaf(ww.y, fmaxf(v[q4][4 * j4 + 1], 0.f), part[q4]);
              part[q4] = fmaf(ww.z, fmaxf(v[q4][4 * j4 + 2], 0.f), part[q4]);
              part[q4] = fmaf(ww.w, fmaxf(v[q4][4 * j4 + 3], 0.f), part[q4]);
            }
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&tempty[acc]);
          // the score in bf16 (held in the fp32 workspace)
          const float sc =
              __bfloat162float(__float2bfloat16_rn((part[0] + part[1]) + (part[2] + part[3])));
          const int s = cur.t * kTileM + quad * 32 + lane;
          if (s < nv) {
            a.scores[(size_t)cur.g * a.N + s] = sc;
            if (hist) atomicAdd(&shist[score_key(sc) >> 20], 1u);
          }
        }
        if (last) {  // done with the slot's head weights
          __syncwarp();
          if (lane == 0) mbar_arrive(&qempty[slot]);
          ++qn;
        }
        cur.next(prefix, a.ngroups);
      }
      if (hist) {  // flush the last query's histogram
        named_bar(2, 256);
        for (int bin = et; bin < kHistBins; bin += 256) {
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
    // let asynchronous work already issued drain before TMEM is released
    const uint64_t t0 = globaltimer();
    while (globaltimer() - t0 < 200000ull) __nanosleep(1000);
  }
  if (warp == 1) tmem_dealloc(tbase, 512);
}

// ----------------------------------------------------------- quantiser --
// One thread per block of 32 values of a bf16 row: scale exponent and E2M1
// codes (the rule of the scorer's query side), written as 16 code bytes and
// one E8M0 byte.
__global__ void __launch_bounds__(256) mxfp4_quantize_rows(const __nv_bfloat16* __restrict__ x,
                                                           long long nblocks,
                                                           uint8_t* __restrict__ codes,
                                                           uint8_t* __restrict__ scales) {
  const long long bi = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (bi >= nblocks) return;
  const uint4* src = reinterpret_cast<const uint4*>(x + bi * 32);
  float v[32];
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const uint4 q = src[u];
    const uint32_t wv[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      v[8 * u + 2 * k] = __uint_as_float(wv[k] << 16);
      v[8 * u + 2 * k + 1] = __uint_as_float(wv[k] & 0xFFFF0000u);
    }
  }
  float amax = 0.f;
#pragma unroll
  for (int k = 0; k < 32; ++k) amax = fmaxf(amax, fabsf(v[k]));
  const int e = mx_block_exp(amax);
  const float down = pow2f(-e);
  uint32_t out[4] = {0u, 0u, 0u, 0u};
#pragma unroll
  for (int k = 0; k < 32; ++k) {
    const float qv = e2m1_round(fabsf(v[k]) * down);
    // magnitude code of qv: 0, 0.5, 1, 1.5 -> 0..3; 2, 3 -> 4, 5; 4, 6 -> 6, 7
    const uint32_t mag = qv < 2.f ? (uint32_t)(qv * 2.f)
                                  : (qv < 4.f ? (uint32_t)qv + 2u : (qv == 4.f ? 6u : 7u));
    const uint32_t code = mag | (v[k] < 0.f && qv > 0.f ? 8u : 0u);
    out[k >> 3] |= code << (4 * (k & 7));
  }
  reinterpret_cast<uint4*>(codes)[bi] = make_uint4(out[0], out[1], out[2], out[3]);
  scales[bi] = (uint8_t)(e + 127);
}

// --------------------------------------------------------------- host --
__global__ void index_plan(const int32_t* q_pos, int G, int ngroups, int m, int N, int* prefix,
                           unsigned* zero_words, size_t nzero);
bool make_tmap_u8(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols,
                  uint32_t box_cols, uint32_t box_rows, bool swizzle64);
bool tma_available();

csa_status launch_mxfp4_quantize(long long rows, int width, const void* x, void* codes,
                                 void* scales, cudaStream_t st) {
  const long long nblocks = rows * (width / 32);
  if (nblocks == 0) return CSA_OK;
  const unsigned grid = (unsigned)((nblocks + 255) / 256);
  CSA_LAUNCH(KK_PACK, st, mxfp4_quantize_rows<<<grid, 256, 0, st>>>(
                              (const __nv_bfloat16*)x, nblocks, (uint8_t*)codes,
                              (uint8_t*)scales));
  return last_launch_status();
}

bool index_fp4_supported(const csa_params& p) {
  return p.act == CSA_BF16 && p.c_I == kF4CI && p.n_hI % 16 == 0 && p.n_hI >= 16 &&
         p.n_hI <= 64 && tma_available();
}

static size_t fp4_smem_bytes() {
  return 1024 + 2 * (size_t)kF4QSlot + (size_t)kF4SC * (kF4CodeTile + kF4ScaleTile) + 512 +
         kHistBins * 4 + 80 * 4 + 2 * 64 * 4;
}

csa_status launch_index_scores_fp4(const csa_params& p, int B, int Q, const int32_t* q_pos,
                                   const void* qI, const float* w, const void* kcodes,
                                   const void* kscales, int N, float* scores, int* plan,
                                   unsigned* ghist, cudaStream_t st) {
  const int R = B * Q;
  const bool inline_plan = R <= kInlineGroups;
  if (!inline_plan)
    CSA_LAUNCH(KK_PLAN, st, index_plan<<<1, 1024, 0, st>>>(q_pos, 1, R, p.m, N, plan, nullptr, 0));
  if (N == 0) return last_launch_status();
  CUtensorMap tmC;
  if (!make_tmap_u8(&tmC, kcodes, (uint64_t)B * N, kF4CodeBytes, kF4CodeBytes, kTileM, true))
    return CSA_ERR_CUDA;
  IdxF4Args a{q_pos, (const __nv_bfloat16*)qI, w, (const uint8_t*)kscales,
              inline_plan ? nullptr : plan, scores, device_error_word(), ghist,
              (long long)B * N, Q, N, p.m, p.n_hI, R, Q == 1 ? 1 : 0};
  if (a.err == nullptr) return CSA_ERR_CUDA;
  const size_t smem = fp4_smem_bytes();
  if (!set_kernel_smem((const void*)index_scores_fp4, (int)smem)) return CSA_ERR_CUDA;
  const int occ = kernel_occupancy((const void*)index_scores_fp4, kF4Threads, (int)smem);
  if (occ < 1) return CSA_ERR_UNSUPPORTED;
  const int grid = sm_count() * occ;
  CSA_LAUNCH(KK_SCORES, st, index_scores_fp4<<<grid, kF4Threads, smem, st>>>(tmC, a));
  return last_launch_status();
}

}  // namespace csa
