// compress.cu -- CSA / HCA KV compression ("DeepSeekV4技术报告阅读笔记" eq. 9-12
// and 20-23; RMSNorm and partial RoPE of section 2.5.1-2.5.2; the FP8/BF16
// entry format of "02 · DeepSeek-V4: 压缩注意力撑起 1M 上下文" section 2.5).
//
// Path: (1) projection GEMM P = H * Wpacked^T into an fp32 workspace
// [B*T][ncols] (columns C^a | C^b | Z^a | Z^b | indexer C^a | C^b | Z^a | Z^b),
// (2) one CTA per entry folds its 2m rows with a per-channel softmax, applies
// RMSNorm + RoPE and stores the entry (bf16 / fp32 / FP8-mixed) and its
// indexer key, (3) one CTA per token writes the window row.
#include <cstdio>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace csa {

static int esize(int dt) { return dt == CSA_F32 ? 4 : 2; }

PackLayout pack_layout(const csa_params& p, int d) {
  PackLayout L;
  const int c = p.c, ci = p.c_I;
  if (p.overlap) {
    L.col_Ca = 0; L.col_Cb = c; L.col_Za = 2 * c; L.col_Zb = 3 * c;
    L.col_CIa = 4 * c; L.col_CIb = 4 * c + ci;
    L.col_ZIa = 4 * c + 2 * ci; L.col_ZIb = 4 * c + 3 * ci;
    L.ncols = 4 * c + 4 * ci;
    L.nb = 2 * c + 2 * ci;
    L.b_Ba = 0; L.b_Bb = c; L.b_BIa = 2 * c; L.b_BIb = 2 * c + ci;
  } else {
    L.col_Ca = 0; L.col_Za = c;
    L.ncols = 2 * c;
    L.nb = c;
    L.b_Ba = 0;
  }
  L.bias_off = align_up((size_t)L.ncols * d * esize(p.act), 256);
  L.total = L.bias_off + align_up((size_t)p.m * L.nb * 4, 256);
  if (p.act == CSA_BF16) {  // tile-major copy for the decode projection
    L.dec_tiles = (c + 63) / 64 + (p.overlap ? (c + 63) / 64 + 2 * ((ci + 63) / 64) : 0);
    L.dec_kb = (d + 63) / 64;
    L.dec_off = align_up(L.total, 1024);
    L.total = L.dec_off + (size_t)L.dec_tiles * L.dec_kb * kDecBlockBytes;
  }
  return L;
}

// ------------------------------------------------------------------ pack --
// dst[(col0 + j) * d + k] = W[k * width + j]  (a 32x32-tiled transpose)
template <typename T>
__global__ void pack_transpose(const T* __restrict__ W, int d, int width,
                               T* __restrict__ dst, int col0) {
  __shared__ T tile[32][33];
  const int k0 = blockIdx.y * 32, j0 = blockIdx.x * 32;
  for (int r = threadIdx.y; r < 32; r += 8) {
    int k = k0 + r, j = j0 + threadIdx.x;
    if (k < d && j < width) tile[r][threadIdx.x] = W[(size_t)k * width + j];
  }
  __syncthreads();
  for (int r = threadIdx.y; r < 32; r += 8) {
    int j = j0 + r, k = k0 + threadIdx.x;
    if (k < d && j < width) dst[(size_t)(col0 + j) * d + k] = tile[threadIdx.x][r];
  }
}

__global__ void pack_bias(const float* __restrict__ Bsrc, int m, int width,
                          float* __restrict__ dst, int nb, int col0) {
  int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < m * width) {
    int r = i / width, j = i % width;
    dst[(size_t)r * nb + col0 + j] = Bsrc[i];
  }
}

csa_status launch_pack(const csa_params& p, int d, const void* const W[8],
                       const float* const Bias[4], void* packed, cudaStream_t st) {
  PackLayout L = pack_layout(p, d);
  const int cols[8] = {L.col_Ca, L.col_Cb, L.col_Za, L.col_Zb,
                       L.col_CIa, L.col_CIb, L.col_ZIa, L.col_ZIb};
  const int widths[8] = {p.c, p.c, p.c, p.c, p.c_I, p.c_I, p.c_I, p.c_I};
  // argument order: Wkv_a, Wkv_b, Wz_a, Wz_b, WIkv_a, WIkv_b, WIz_a, WIz_b
  for (int t = 0; t < 8; ++t) {
    int col = cols[t];
    if (col < 0) continue;
    int width = widths[t];
    dim3 grid((width + 31) / 32, (d + 31) / 32), block(32, 8);
    if (p.act == CSA_F32)
      CSA_LAUNCH(KK_PACK, st, pack_transpose<float><<<grid, block, 0, st>>>(
                                  (const float*)W[t], d, width, (float*)packed, col));
    else
      CSA_LAUNCH(KK_PACK, st, pack_transpose<__nv_bfloat16><<<grid, block, 0, st>>>(
                                  (const __nv_bfloat16*)W[t], d, width,
                                  (__nv_bfloat16*)packed, col));
  }
  float* bias = (float*)((char*)packed + L.bias_off);
  const int bcols[4] = {L.b_Ba, L.b_Bb, L.b_BIa, L.b_BIb};
  const int bw[4] = {p.c, p.c, p.c_I, p.c_I};
  for (int t = 0; t < 4; ++t) {
    if (bcols[t] < 0) continue;
    int n = p.m * bw[t];
    CSA_LAUNCH(KK_PACK, st, pack_bias<<<(n + 255) / 256, 256, 0, st>>>(
                                Bias[t], p.m, bw[t], bias, L.nb, bcols[t]));
  }
  if (L.dec_tiles > 0) {
    const csa_status s = launch_pack_dec_tiles(p, L, d, packed, st);
    if (s != CSA_OK) return s;
  }
  return last_launch_status();
}

// ------------------------------------------------------------------ GEMM --
// C[M][N] (fp32) = A[M][K] * Bm[N][K]^T, fp32 accumulation in k order.
// 64x64 tile per 256-thread CTA, 4x4 outputs per thread.
template <typename T>
__global__ void __launch_bounds__(256) gemm_nt_simt(const T* __restrict__ A,
                                                    const T* __restrict__ Bm,
                                                    float* __restrict__ C, int M,
                                                    int N, int K) {
  __shared__ float As[16][64 + 4];
  __shared__ float Bs[16][64 + 4];
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const int m0 = blockIdx.y * 64, n0 = blockIdx.x * 64;
  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
  for (int k0 = 0; k0 < K; k0 += 16) {
    for (int i = threadIdx.x; i < 64 * 16; i += 256) {
      int r = i >> 4, kk = i & 15;
      int gk = k0 + kk;
      int gm = m0 + r, gn = n0 + r;
      As[kk][r] = (gm < M && gk < K) ? to_f32(A[(size_t)gm * K + gk]) : 0.f;
      Bs[kk][r] = (gn < N && gk < K) ? to_f32(Bm[(size_t)gn * K + gk]) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < 16; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = Bs[kk][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    int gm = m0 + ty * 4 + i;
    if (gm >= M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      int gn = n0 + tx * 4 + j;
      if (gn < N) C[(size_t)gm * N + gn] = acc[i][j];
    }
  }
}

// ------------------------------------------------------------ fold / store --
// One channel of entry i: softmax over the a rows m*i..m*i+m-1 (logit Z^a +
// B^a) and, when overlapping and i > 0, the b rows m*(i-1)..m*i-1 (Z^b + B^b);
// returns sum S * C over the same rows.
__device__ float fold_channel(const float* __restrict__ Pb, int ncols, int m,
                              int i, bool use_b, int cCa, int cZa, int cCb,
                              int cZb, const float* __restrict__ bias, int nb,
                              int bA, int bB, int ch) {
  float mx = -INFINITY;
  for (int r = 0; r < m; ++r) {
    float z = Pb[(size_t)(m * i + r) * ncols + cZa + ch] + bias[r * nb + bA + ch];
    mx = fmaxf(mx, z);
  }
  if (use_b)
    for (int r = 0; r < m; ++r) {
      float z = Pb[(size_t)(m * (i - 1) + r) * ncols + cZb + ch] + bias[r * nb + bB + ch];
      mx = fmaxf(mx, z);
    }
  float den = 0.f, num = 0.f;
  for (int r = 0; r < m; ++r) {
    size_t row = (size_t)(m * i + r) * ncols;
    float e = expf(Pb[row + cZa + ch] + bias[r * nb + bA + ch] - mx);
    den += e;
    num = fmaf(e, Pb[row + cCa + ch], num);
  }
  if (use_b)
    for (int r = 0; r < m; ++r) {
      size_t row = (size_t)(m * (i - 1) + r) * ncols;
      float e = expf(Pb[row + cZb + ch] + bias[r * nb + bB + ch] - mx);
      den += e;
      num = fmaf(e, Pb[row + cCb + ch], num);
    }
  return num / den;
}

// RMSNorm (unit gain) and RoPE at `pos` of the row held in shared xs[c].
__device__ void norm_rope_shared(float* xs, int c, int rd, float eps, double pos,
                                 double base, float* red) {
  float ss = 0.f;
  for (int ch = threadIdx.x; ch < c; ch += blockDim.x) ss = fmaf(xs[ch], xs[ch], ss);
  ss = block_reduce<false>(ss, red);
  float inv = 1.0f / sqrtf(ss / (float)c + eps);
  __syncthreads();
  for (int ch = threadIdx.x; ch < c; ch += blockDim.x) xs[ch] *= inv;
  __syncthreads();
  for (int pp = threadIdx.x; pp < rd / 2; pp += blockDim.x) {
    float cs, sn;
    rope_cs(pos, pp, rd, base, &cs, &sn);
    int j = c - rd + 2 * pp;
    float x0 = xs[j], x1 = xs[j + 1];
    xs[j] = x0 * cs - x1 * sn;
    xs[j + 1] = x0 * sn + x1 * cs;
  }
  __syncthreads();
}

// Store the row xs[c] in KV format kKV (0 f32, 1 bf16, 2 fp8-mixed).
template <int kKV>
__device__ void store_kv_row(const float* xs, int c, int rd, void* dst,
                             float* dst_scale, float* red) {
  if (kKV == CSA_F32) {
    for (int ch = threadIdx.x; ch < c; ch += blockDim.x) ((float*)dst)[ch] = xs[ch];
  } else if (kKV == CSA_BF16) {
    for (int ch = threadIdx.x; ch < c; ch += blockDim.x)
      ((__nv_bfloat16*)dst)[ch] = __float2bfloat16_rn(xs[ch]);
  } else {
    const int nf = c - rd;
    float amax = 0.f;
    for (int ch = threadIdx.x; ch < nf; ch += blockDim.x) amax = fmaxf(amax, fabsf(xs[ch]));
    amax = block_reduce<true>(amax, red);
    float s = amax > 0.f ? amax / 448.0f : 1.0f;
    uint8_t* codes = (uint8_t*)dst;
    for (int ch = threadIdx.x; ch < nf; ch += blockDim.x) codes[ch] = f32_to_e4m3(xs[ch] / s);
    __nv_bfloat16* rope = (__nv_bfloat16*)(codes + nf);
    for (int ch = nf + threadIdx.x; ch < c; ch += blockDim.x)
      rope[ch - nf] = __float2bfloat16_rn(xs[ch]);
    if (threadIdx.x == 0) *dst_scale = s;
  }
}

__host__ __device__ inline size_t kv_row_bytes(int kv, int c, int rd) {
  return kv == CSA_F32 ? (size_t)4 * c : kv == CSA_BF16 ? (size_t)2 * c : (size_t)(c - rd) + 2 * rd;
}

template <typename TA, int kKV>
__global__ void __launch_bounds__(256) fold_entries(
    const float* __restrict__ P, int ncols, const float* __restrict__ bias, int nb,
    PackLayout L, int B, int T, int nE, int m, int overlap, int c, int rd,
    int cI, float eps, double base, void* __restrict__ ckv,
    float* __restrict__ ckv_scale, TA* __restrict__ kI) {
  extern __shared__ float xs[];  // c floats
  __shared__ float red[32];
  const int b = blockIdx.x / nE, i = blockIdx.x % nE;
  const float* Pb = P + (size_t)b * T * ncols;
  const bool use_b = overlap && i > 0;
  for (int ch = threadIdx.x; ch < c; ch += blockDim.x)
    xs[ch] = fold_channel(Pb, ncols, m, i, use_b, L.col_Ca, L.col_Za, L.col_Cb,
                          L.col_Zb, bias, nb, L.b_Ba, L.b_Bb, ch);
  __syncthreads();
  norm_rope_shared(xs, c, rd, eps, (double)m * i, base, red);
  const size_t rowb = kv_row_bytes(kKV, c, rd);
  const size_t e = (size_t)b * nE + i;
  store_kv_row<kKV>(xs, c, rd, (char*)ckv + e * rowb,
                    ckv_scale ? ckv_scale + e : nullptr, red);
  if (kI != nullptr)
    for (int ch = threadIdx.x; ch < cI; ch += blockDim.x)
      kI[e * cI + ch] = from_f32<TA>(fold_channel(Pb, ncols, m, i, use_b, L.col_CIa,
                                                  L.col_ZIa, L.col_CIb, L.col_ZIb, bias,
                                                  nb, L.b_BIa, L.b_BIb, ch));
}

// The entries folded by the GEMM's epilogue (F [B*nE][c + cI] fp32, main
// channels then indexer channels): RMSNorm + RoPE at m*i and the store of
// the entry; the indexer key rounded to the activation dtype.
template <typename TA, int kKV>
__global__ void __launch_bounds__(256) finish_entries(
    const float* __restrict__ F, int nE, int c, int cI, int m, int rd, float eps,
    double base, void* __restrict__ ckv, float* __restrict__ ckv_scale, TA* __restrict__ kI) {
  extern __shared__ float xs[];  // c floats
  __shared__ float red[32];
  const size_t e = blockIdx.x;
  const int i = (int)(e % nE);
  const float* src = F + e * (size_t)(c + cI);
  for (int ch = threadIdx.x; ch < c; ch += blockDim.x) xs[ch] = src[ch];
  __syncthreads();
  norm_rope_shared(xs, c, rd, eps, (double)m * i, base, red);
  const size_t rowb = kv_row_bytes(kKV, c, rd);
  store_kv_row<kKV>(xs, c, rd, (char*)ckv + e * rowb, ckv_scale ? ckv_scale + e : nullptr, red);
  if (kI != nullptr)
    for (int ch = threadIdx.x; ch < cI; ch += blockDim.x) kI[e * cI + ch] = from_f32<TA>(src[c + ch]);
}

template <int kKV>
__global__ void __launch_bounds__(256) window_rows(const float* __restrict__ P,
                                                  int ncols, int colC, int T, int c,
                                                  int rd, float eps, double base,
                                                  void* __restrict__ win,
                                                  float* __restrict__ win_scale) {
  extern __shared__ float xs[];
  __shared__ float red[32];
  const size_t row = blockIdx.x;  // b*T + j
  const int j = (int)(row % T);
  for (int ch = threadIdx.x; ch < c; ch += blockDim.x) xs[ch] = P[row * ncols + colC + ch];
  __syncthreads();
  norm_rope_shared(xs, c, rd, eps, (double)j, base, red);
  const size_t rowb = kv_row_bytes(kKV, c, rd);
  store_kv_row<kKV>(xs, c, rd, (char*)win + row * rowb,
                    win_scale ? win_scale + row : nullptr, red);
}

bool gemm_tc_supported(int M, int N, int K);
csa_status launch_gemm_tc(const void* A, const void* B, float* C, int M, int N, int K,
                          cudaStream_t st);
bool gemm_fold_supported(const csa_params& p, int d);
size_t gemm_fold_ws_bytes(const csa_params& p, int B, int T);
csa_status launch_gemm_fold(const csa_params& p, const PackLayout& L, int B, int T, int d,
                            const void* H, const void* packed, const float* bias, float* F,
                            float* Ca, cudaStream_t st);

// bf16 projections whose shapes the fold epilogue covers skip the fp32
// product: the workspace holds the folded entries and the C^a rows
size_t compress_ws_bytes(const csa_params& p, int B, int T, int d) {
  if (gemm_fold_supported(p, d)) return gemm_fold_ws_bytes(p, B, T);
  PackLayout L = pack_layout(p, d);
  return align_up((size_t)B * T * L.ncols * sizeof(float), 256);
}

template <typename TA, int kKV>
static void launch_finish(const csa_params& p, const float* F, const float* Ca, int B, int T,
                          int nE, void* ckv, float* ckv_scale, void* kI, void* win,
                          float* win_scale, cudaStream_t st) {
  size_t smem = (size_t)p.c * sizeof(float);
  if (nE > 0)
    CSA_LAUNCH(KK_FOLD, st, finish_entries<TA, kKV><<<B * nE, 256, smem, st>>>(
        F, nE, p.c, p.overlap ? p.c_I : 0, p.m, p.rope_dims, p.rms_eps, (double)p.rope_base,
        ckv, ckv_scale, (TA*)kI));
  if (win != nullptr)
    CSA_LAUNCH(KK_WINDOW, st, window_rows<kKV><<<B * T, 256, smem, st>>>(
        Ca, p.c, 0, T, p.c, p.rope_dims, p.rms_eps, (double)p.rope_base, win, win_scale));
}

template <typename TA, int kKV>
static void launch_fold(const csa_params& p, const PackLayout& L, const float* P,
                        const float* bias, int B, int T, int nE, void* ckv,
                        float* ckv_scale, void* kI, void* win, float* win_scale,
                        cudaStream_t st) {
  size_t smem = (size_t)p.c * sizeof(float);
  if (nE > 0) {
    CSA_LAUNCH(KK_FOLD, st, fold_entries<TA, kKV><<<B * nE, 256, smem, st>>>(
        P, L.ncols, bias, L.nb, L, B, T, nE, p.m, p.overlap, p.c, p.rope_dims, p.c_I,
        p.rms_eps, (double)p.rope_base, ckv, ckv_scale, (TA*)kI));
  }
  if (win != nullptr) {
    CSA_LAUNCH(KK_WINDOW, st, window_rows<kKV><<<B * T, 256, smem, st>>>(
        P, L.ncols, L.col_Ca, T, p.c, p.rope_dims, p.rms_eps, (double)p.rope_base, win,
        win_scale));
  }
}

csa_status launch_compress(const csa_params& p, int B, int T, int d,
                           const void* H, const void* packed, void* ckv,
                           float* ckv_scale, void* kI, void* win,
                           float* win_scale, void* ws, cudaStream_t st) {
  PackLayout L = pack_layout(p, d);
  const int M = B * T;
  float* P = (float*)ws;
  dim3 grid((L.ncols + 63) / 64, (M + 63) / 64);
  if (gemm_fold_supported(p, d)) {
    // the projection with the softmax and fold in its epilogue, then the
    // norm, RoPE and store of the entries and the window rows
    const float* bias = (const float*)((const char*)packed + L.bias_off);
    const int nE = T / p.m;
    float* F = (float*)ws;
    float* Ca = (float*)((char*)ws + align_up((size_t)B * nE * (p.c + (p.overlap ? p.c_I : 0)) * 4, 256));
    csa_status s = launch_gemm_fold(p, L, B, T, d, H, packed, bias, F, Ca, st);
    if (s != CSA_OK) return s;
    if (p.kv == CSA_F32)
      launch_finish<__nv_bfloat16, CSA_F32>(p, F, Ca, B, T, nE, ckv, ckv_scale, kI, win, win_scale, st);
    else if (p.kv == CSA_BF16)
      launch_finish<__nv_bfloat16, CSA_BF16>(p, F, Ca, B, T, nE, ckv, ckv_scale, kI, win, win_scale, st);
    else
      launch_finish<__nv_bfloat16, CSA_KV_FP8MIX>(p, F, Ca, B, T, nE, ckv, ckv_scale, kI, win, win_scale, st);
    return last_launch_status();
  }
  if (p.act == CSA_BF16 && gemm_tc_supported(M, L.ncols, d)) {
    csa_status s = launch_gemm_tc(H, packed, P, M, L.ncols, d, st);
    if (s != CSA_OK) return s;
  } else if (p.act == CSA_F32)
    CSA_LAUNCH(KK_GEMM, st, gemm_nt_simt<float><<<grid, 256, 0, st>>>(
        (const float*)H, (const float*)packed, P, M, L.ncols, d));
  else
    CSA_LAUNCH(KK_GEMM, st, gemm_nt_simt<__nv_bfloat16><<<grid, 256, 0, st>>>(
        (const __nv_bfloat16*)H, (const __nv_bfloat16*)packed, P, M, L.ncols, d));
  const float* bias = (const float*)((const char*)packed + L.bias_off);
  const int nE = T / p.m;
  if (p.act == CSA_F32) {
    if (p.kv == CSA_F32)
      launch_fold<float, CSA_F32>(p, L, P, bias, B, T, nE, ckv, ckv_scale, kI, win, win_scale, st);
    else if (p.kv == CSA_BF16)
      launch_fold<float, CSA_BF16>(p, L, P, bias, B, T, nE, ckv, ckv_scale, kI, win, win_scale, st);
    else
      launch_fold<float, CSA_KV_FP8MIX>(p, L, P, bias, B, T, nE, ckv, ckv_scale, kI, win, win_scale, st);
  } else {
    if (p.kv == CSA_F32)
      launch_fold<__nv_bfloat16, CSA_F32>(p, L, P, bias, B, T, nE, ckv, ckv_scale, kI, win, win_scale, st);
    else if (p.kv == CSA_BF16)
      launch_fold<__nv_bfloat16, CSA_BF16>(p, L, P, bias, B, T, nE, ckv, ckv_scale, kI, win, win_scale, st);
    else
      launch_fold<__nv_bfloat16, CSA_KV_FP8MIX>(p, L, P, bias, B, T, nE, ckv, ckv_scale, kI, win, win_scale, st);
  }
  return last_launch_status();
}

// ------------------------------------------------------ decode: append --
// One new token per sequence.  The softmax of an entry's fold is kept as a
// running state instead of the rows it spans: per channel the largest logit
// seen so far, the sum of exp(logit - largest) and the sum of that weight
// times C, rescaled when a larger logit arrives.  Token t of block j = t / m
// (row r = t % m) adds its a part (C^a, Z^a + B^a[r]) to entry j and, when
// the windows overlap, its b part (C^b, Z^b + B^b[r]) to entry j + 1.  When t
// closes block j (r == m-1) entry j is complete: num / den per channel, then
// RMSNorm and RoPE at m*j and the same storage as the prefill.  The window
// row of token t (RMSNorm + RoPE(t) of C^a_t, or C_t) is written every step;
// when the W window rows are full the last n_win - 1 of them move to the
// front and win_pos0 advances, so W >= 2 (n_win - 1) rows per sequence
// suffice for any length.  Each token costs O(c) state work; nothing scales
// with m.
//
// State of one sequence (fp32): xrow[c] (C^a of the current token), then S
// slots (S = 2 with overlap: entries j and j+1 are open at once; S = 1
// without), each mx[nch] den[nch] num[nch] with nch = c + c_I (c without
// indexer).  Entry i lives in slot i % S.

struct AppendState {
  int c, cI, nch, S;
  size_t per_seq;  // floats per sequence
};

static AppendState append_state(const csa_params& p) {
  AppendState A;
  A.c = p.c;
  A.cI = p.overlap ? p.c_I : 0;
  A.nch = A.c + A.cI;
  A.S = p.overlap ? 2 : 1;
  A.per_seq = (size_t)A.c + (size_t)A.S * 3 * A.nch;
  return A;
}

// A CTA owns 4 pairs, pair q = blockIdx.x*4 + p: the C and Z columns of one
// channel of one part (a or b; main or indexer), computed for kB tokens (B
// rounded up to a power of two; the rows past B are zeros and their results
// are dropped).  d is walked in chunks of kChunk elements through a
// kStages-deep cp.async pipeline in shared memory: each stage holds the
// chunk of the CTA's 8 weight rows (the only HBM stream) and of the kB rows
// of h, so several chunks are in flight while one is used.  Warps 2p and
// 2p+1 take the even and odd halves of each chunk of pair p; the halves are
// summed through shared memory and lane 0 of warp 2p updates the state.
template <typename TA>
struct AppendProj {
  static constexpr int V = 16 / sizeof(TA);      // elements per 16-byte piece
  static constexpr int kPieces = 64;             // 16-byte pieces per row of a chunk
  static constexpr int kChunk = kPieces * V;     // elements of d per chunk
  static constexpr int kStages = 3;
  static constexpr int kThreads = 256;
  __host__ __device__ static size_t stage_elems(int kB) { return (size_t)(8 + kB) * kChunk; }
  static size_t smem(int kB) { return kStages * stage_elems(kB) * sizeof(TA); }
};

template <typename TA, int kB>
__global__ void __launch_bounds__(256) append_project(
    const TA* __restrict__ H, const TA* __restrict__ Wp, int B, int d, PackLayout L,
    const float* __restrict__ bias, int m, int overlap, int c, int cI,
    const int32_t* __restrict__ tpos, float* __restrict__ state, size_t per_seq) {
  using K = AppendProj<TA>;
  constexpr int V = K::V, kPieces = K::kPieces, kChunk = K::kChunk, kStages = K::kStages;
  extern __shared__ __align__(16) unsigned char append_smem[];
  __shared__ float half_sum[4][kB][2];
  // stage s: rows 0..7 the weight rows (row 2p the C row of pair p, 2p+1 its
  // Z row), rows 8..8+kB-1 the rows of h; each row kChunk elements
  TA* sm = reinterpret_cast<TA*>(append_smem);
  constexpr size_t stage = (size_t)(8 + kB) * kChunk;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int pp = warp >> 1, half = warp & 1;
  const int q = blockIdx.x * 4 + pp;
  // pair q -> (C column, Z column, bias column, state channel, part b?)
  int colC = 0, colZ = 0, colB = 0, sch = 0;
  bool partb = false, active = true;
  if (q < c) {
    colC = L.col_Ca + q; colZ = L.col_Za + q; colB = L.b_Ba + q; sch = q;
  } else if (!overlap) {
    active = false;
  } else if (q < 2 * c) {
    const int ch = q - c;
    colC = L.col_Cb + ch; colZ = L.col_Zb + ch; colB = L.b_Bb + ch; sch = ch; partb = true;
  } else if (q < 2 * c + cI) {
    const int ch = q - 2 * c;
    colC = L.col_CIa + ch; colZ = L.col_ZIa + ch; colB = L.b_BIa + ch; sch = c + ch;
  } else if (q < 2 * c + 2 * cI) {
    const int ch = q - 2 * c - cI;
    colC = L.col_CIb + ch; colZ = L.col_ZIb + ch; colB = L.b_BIb + ch; sch = c + ch;
    partb = true;
  } else {
    active = false;  // still takes part in the copies and barriers
  }
  // warp w copies weight row w: the C (even w) or Z (odd w) row of pair w/2
  const TA* wrow = Wp + (size_t)(half ? colZ : colC) * d;
  const int nchunk = (d + kChunk - 1) / kChunk;
  // chunk ci into stage ci % kStages (zeros past d and past B); one group
  auto load_chunk = [&](int ci) {
    TA* st0 = sm + (size_t)(ci % kStages) * stage;
    const int k0 = ci * kChunk;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int piece = lane + 32 * h;
      const int k = k0 + piece * V;
      const bool ok = active && k < d;
      sm100::cp_async16(st0 + (size_t)warp * kChunk + piece * V,
                        ok ? (const void*)(wrow + k) : (const void*)Wp, ok ? 16u : 0u);
    }
#pragma unroll
    for (int i = threadIdx.x; i < kB * kPieces; i += K::kThreads) {
      const int b = i / kPieces, piece = i - b * kPieces;
      const int k = k0 + piece * V;
      const bool ok = b < B && k < d;
      sm100::cp_async16(st0 + (size_t)(8 + b) * kChunk + piece * V,
                        ok ? (const void*)(H + (size_t)b * d + k) : (const void*)H,
                        ok ? 16u : 0u);
    }
  };
#pragma unroll
  for (int s = 0; s < kStages - 1; ++s) {
    if (s < nchunk) load_chunk(s);
    sm100::cp_async_commit();  // (empty groups keep the count uniform)
  }
  float accC[kB], accZ[kB];
#pragma unroll
  for (int b = 0; b < kB; ++b) accC[b] = accZ[b] = 0.f;
  const int e0 = (lane + 32 * half) * V;  // this warp's piece of every chunk
  for (int ci = 0; ci < nchunk; ++ci) {
    sm100::cp_async_wait<kStages - 2>();  // chunk ci has landed (this thread's part)
    __syncthreads();  // ... every thread's part; stage (ci-1) % kStages is free
    if (ci + kStages - 1 < nchunk) load_chunk(ci + kStages - 1);
    sm100::cp_async_commit();
    if (active) {  // (past d the pieces are zeros)
      const TA* st0 = sm + (size_t)(ci % kStages) * stage;
      const uint4 rc = *reinterpret_cast<const uint4*>(st0 + (size_t)(2 * pp) * kChunk + e0);
      const uint4 rz = *reinterpret_cast<const uint4*>(st0 + (size_t)(2 * pp + 1) * kChunk + e0);
      uint4 hr[kB];
#pragma unroll
      for (int b = 0; b < kB; ++b)
        hr[b] = *reinterpret_cast<const uint4*>(st0 + (size_t)(8 + b) * kChunk + e0);
      const TA* cv = reinterpret_cast<const TA*>(&rc);
      const TA* zv = reinterpret_cast<const TA*>(&rz);
#pragma unroll
      for (int e = 0; e < V; ++e) {
        const float wc = to_f32(cv[e]), wz = to_f32(zv[e]);
#pragma unroll
        for (int b = 0; b < kB; ++b) {
          const float hx = to_f32(reinterpret_cast<const TA*>(&hr[b])[e]);
          accC[b] = fmaf(hx, wc, accC[b]);
          accZ[b] = fmaf(hx, wz, accZ[b]);
        }
      }
    }
  }
  sm100::cp_async_wait<0>();  // (only empty groups remain)
#pragma unroll
  for (int b = 0; b < kB; ++b) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      accC[b] += __shfl_xor_sync(0xffffffffu, accC[b], o);
      accZ[b] += __shfl_xor_sync(0xffffffffu, accZ[b], o);
    }
  }
  if (half == 1 && lane == 0)
#pragma unroll
    for (int b = 0; b < kB; ++b) {
      half_sum[pp][b][0] = accC[b];
      half_sum[pp][b][1] = accZ[b];
    }
  __syncthreads();
  if (!active || half == 1 || lane != 0) return;
  const int nch = c + cI;
  const int S = overlap ? 2 : 1;
#pragma unroll
  for (int b = 0; b < kB; ++b) {
    if (b >= B) break;
    const float vC = accC[b] + half_sum[pp][b][0];
    const float vZ = accZ[b] + half_sum[pp][b][1];
    const int t = tpos[b];
    const int j = t / m, r = t % m;
    float* st = state + (size_t)b * per_seq;
    if (q < c) st[q] = vC;  // C^a_t: the window row's source
    // entry j (a part) or j + 1 (b part); a fresh entry starts at row 0
    const int entry = partb ? j + 1 : j;
    const bool fresh = r == 0 && (partb || !overlap || j == 0);
    float* slot = st + c + (size_t)(entry % S) * 3 * nch;
    running_softmax_add(slot + sch, slot + nch + sch, slot + 2 * nch + sch, vC,
                        vZ + bias[r * L.nb + colB], fresh);
  }
}

// dst[0..n) = src[0..n) by the whole block (non-overlapping ranges), in the
// widest words both addresses and n allow.
__device__ void block_copy_bytes(char* dst, const char* src, size_t n) {
  const uintptr_t al = (uintptr_t)dst | (uintptr_t)src | (uintptr_t)n;
  if ((al & 15u) == 0) {
    for (size_t i = threadIdx.x; i < n / 16; i += blockDim.x)
      reinterpret_cast<uint4*>(dst)[i] = reinterpret_cast<const uint4*>(src)[i];
  } else if ((al & 3u) == 0) {
    for (size_t i = threadIdx.x; i < n / 4; i += blockDim.x)
      reinterpret_cast<uint32_t*>(dst)[i] = reinterpret_cast<const uint32_t*>(src)[i];
  } else {
    for (size_t i = threadIdx.x; i < n; i += blockDim.x) dst[i] = src[i];
  }
}

// blockIdx.y: 0 the entry closed by token t (if any), 1 its indexer key,
// 2 the window row of token t (rolling the window first when its rows are
// full).
template <typename TA, int kKV>
__global__ void __launch_bounds__(256) append_finish(
    const float* __restrict__ state, size_t per_seq, const int32_t* __restrict__ tpos, int m,
    int overlap, int c, int rd, int cI, float eps, double base, void* __restrict__ ckv,
    float* __restrict__ ckv_scale, int N, TA* __restrict__ kI, void* __restrict__ win,
    float* __restrict__ win_scale, int32_t* __restrict__ win_pos0, int W, int n_win,
    unsigned* __restrict__ err) {
  extern __shared__ float xs[];  // c floats
  __shared__ float red[32];
  pdl_wait();     // launched as a programmatic dependent of the projection
  pdl_trigger();  // a following dependent may set up meanwhile (it waits for us)
  const int b = blockIdx.x, part = blockIdx.y;
  const int t = tpos[b];
  const float* st = state + (size_t)b * per_seq;
  const size_t rowb = kv_row_bytes(kKV, c, rd);
  if (part == 2) {  // window row of token t
    if (win == nullptr) return;
    int wr = t - win_pos0[b];
    const int keep = n_win > 1 ? n_win - 1 : 0;  // earlier rows the window still needs
    if (wr == W && W >= 2 * keep && W > 0) {
      // the rows are full: roll the window.  Rows W-keep..W-1 (positions
      // t-keep..t-1) move to rows 0..keep-1 (the ranges do not overlap) and
      // row 0 becomes position t - keep.
      char* wb = (char*)win + (size_t)b * W * rowb;
      block_copy_bytes(wb, wb + (size_t)(W - keep) * rowb, (size_t)keep * rowb);
      if (win_scale != nullptr)
        for (int i = threadIdx.x; i < keep; i += blockDim.x)
          win_scale[(size_t)b * W + i] = win_scale[(size_t)b * W + W - keep + i];
      __syncthreads();  // every thread has read win_pos0 and copied its share
      if (threadIdx.x == 0) win_pos0[b] = t - keep;
      wr = keep;
    }
    if (wr < 0 || wr >= W) {
      if (threadIdx.x == 0) atomicOr(err, CSA_DEV_BAD_WINDOW);
      return;
    }
    for (int ch = threadIdx.x; ch < c; ch += blockDim.x) xs[ch] = st[ch];
    __syncthreads();
    norm_rope_shared(xs, c, rd, eps, (double)t, base, red);
    const size_t e = (size_t)b * W + wr;
    store_kv_row<kKV>(xs, c, rd, (char*)win + e * rowb, win_scale ? win_scale + e : nullptr,
                      red);
    return;
  }
  if (t % m != m - 1) return;  // no block closed by this token
  const int i = t / m;
  if (i >= N) {
    if (threadIdx.x == 0) atomicOr(err, CSA_DEV_BAD_INDEX);
    return;
  }
  const int nch = c + (overlap ? cI : 0);
  const float* slot = st + c + (size_t)(overlap ? i % 2 : 0) * 3 * nch;
  const size_t e = (size_t)b * N + i;
  if (part == 0) {
    for (int ch = threadIdx.x; ch < c; ch += blockDim.x)
      xs[ch] = slot[2 * nch + ch] / slot[nch + ch];
    __syncthreads();
    norm_rope_shared(xs, c, rd, eps, (double)m * i, base, red);
    store_kv_row<kKV>(xs, c, rd, (char*)ckv + e * rowb, ckv_scale ? ckv_scale + e : nullptr,
                      red);
  } else if (kI != nullptr && overlap) {
    for (int ch = threadIdx.x; ch < cI; ch += blockDim.x)
      kI[e * cI + ch] = from_f32<TA>(slot[2 * nch + c + ch] / slot[nch + c + ch]);
  }
}

constexpr int kAppendMaxB = 16;  // tokens per launch of append_project

size_t decode_tail_bytes(const csa_params& p, int B, int d) {
  (void)d;
  return (size_t)B * append_state(p).per_seq * sizeof(float);
}

template <typename TA, int kB>
static csa_status launch_append_project_kb(const csa_params& p, const PackLayout& L, int nb,
                                           int d, const TA* H, const TA* packed,
                                           const float* bias, const int32_t* t, float* sb,
                                           const AppendState& A, dim3 grid, cudaStream_t st) {
  const size_t smem = AppendProj<TA>::smem(kB);
  if (!set_kernel_smem((const void*)append_project<TA, kB>, (int)smem)) return CSA_ERR_CUDA;
  CSA_LAUNCH(KK_GEMM, st, append_project<TA, kB><<<grid, AppendProj<TA>::kThreads, smem, st>>>(
      H, packed, nb, d, L, bias, p.m, p.overlap, A.c, A.cI, t, sb, A.per_seq));
  return CSA_OK;
}

// kB = nb rounded up to a power of two (nb <= kAppendMaxB)
template <typename TA>
static csa_status launch_append_project(const csa_params& p, const PackLayout& L, int nb, int d,
                                        const TA* H, const TA* packed, const float* bias,
                                        const int32_t* t, float* sb, const AppendState& A,
                                        dim3 grid, cudaStream_t st) {
  if (nb <= 1) return launch_append_project_kb<TA, 1>(p, L, nb, d, H, packed, bias, t, sb, A, grid, st);
  if (nb <= 2) return launch_append_project_kb<TA, 2>(p, L, nb, d, H, packed, bias, t, sb, A, grid, st);
  if (nb <= 4) return launch_append_project_kb<TA, 4>(p, L, nb, d, H, packed, bias, t, sb, A, grid, st);
  if (nb <= 8) return launch_append_project_kb<TA, 8>(p, L, nb, d, H, packed, bias, t, sb, A, grid, st);
  return launch_append_project_kb<TA, 16>(p, L, nb, d, H, packed, bias, t, sb, A, grid, st);
}

template <typename TA, int kKV>
static void launch_append_finish(const csa_params& p, const AppendState& A, int B,
                                 const float* state, const int32_t* t, void* ckv,
                                 float* ckv_scale, int N, void* kI, void* win, float* win_scale,
                                 int32_t* win_pos0, int W, cudaStream_t st) {
  const size_t smem = (size_t)p.c * sizeof(float);
  cudaError_t e = cudaSuccess;
  CSA_LAUNCH(KK_FOLD, st,
             e = launch_maybe_pdl(kPdlAppend, append_finish<TA, kKV>, dim3(B, 3), dim3(256), smem,
                                  st, (const float*)state, A.per_seq, t, p.m, p.overlap, p.c,
                                  p.rope_dims, A.cI, p.rms_eps, (double)p.rope_base, ckv,
                                  ckv_scale, N, (TA*)kI, win, win_scale, win_pos0, W, p.n_win,
                                  device_error_word()));
  (void)e;  // a failed launch is reported by last_launch_status()
}

csa_status launch_decode_append(const csa_params& p, int B, int d, const void* H,
                                const int32_t* t, const void* packed, float* tail, void* ckv,
                                float* ckv_scale, int N, void* kI, void* win, float* win_scale,
                                int32_t* win_pos0, int W, cudaStream_t st) {
  const PackLayout L = pack_layout(p, d);
  const AppendState A = append_state(p);
  const float* bias = (const float*)((const char*)packed + L.bias_off);
  if (device_error_word() == nullptr) return CSA_ERR_CUDA;
  const int npairs = L.ncols / 2;
  const dim3 grid((npairs + 3) / 4);
  for (int b0 = 0; b0 < B; b0 += kAppendMaxB) {  // the projections, kAppendMaxB tokens a launch
    const int nb = B - b0 < kAppendMaxB ? B - b0 : kAppendMaxB;
    float* sb = tail + (size_t)b0 * A.per_seq;
    if (append_tc_supported(p, nb)) {  // bf16: the tensor-core projection
      const csa_status s = launch_append_project_tc(
          p, L, nb, d, (const __nv_bfloat16*)H + (size_t)b0 * d, packed, bias, t + b0, sb,
          A.cI, A.per_seq, st);
      if (s != CSA_OK) return s;
      continue;
    }
    const csa_status s = p.act == CSA_F32
        ? launch_append_project<float>(p, L, nb, d, (const float*)H + (size_t)b0 * d,
                                       (const float*)packed, bias, t + b0, sb, A, grid, st)
        : launch_append_project<__nv_bfloat16>(p, L, nb, d,
                                               (const __nv_bfloat16*)H + (size_t)b0 * d,
                                               (const __nv_bfloat16*)packed, bias, t + b0, sb,
                                               A, grid, st);
    if (s != CSA_OK) return s;
  }
  if (p.act == CSA_F32) {
    if (p.kv == CSA_F32)
      launch_append_finish<float, CSA_F32>(p, A, B, tail, t, ckv, ckv_scale, N, kI, win, win_scale, win_pos0, W, st);
    else if (p.kv == CSA_BF16)
      launch_append_finish<float, CSA_BF16>(p, A, B, tail, t, ckv, ckv_scale, N, kI, win, win_scale, win_pos0, W, st);
    else
      launch_append_finish<float, CSA_KV_FP8MIX>(p, A, B, tail, t, ckv, ckv_scale, N, kI, win, win_scale, win_pos0, W, st);
  } else {
    if (p.kv == CSA_F32)
      launch_append_finish<__nv_bfloat16, CSA_F32>(p, A, B, tail, t, ckv, ckv_scale, N, kI, win, win_scale, win_pos0, W, st);
    else if (p.kv == CSA_BF16)
      launch_append_finish<__nv_bfloat16, CSA_BF16>(p, A, B, tail, t, ckv, ckv_scale, N, kI, win, win_scale, win_pos0, W, st);
    else
      launch_append_finish<__nv_bfloat16, CSA_KV_FP8MIX>(p, A, B, tail, t, ckv, ckv_scale, N, kI, win, win_scale, win_pos0, W, st);
  }
  return last_launch_status();
}

}  // namespace csa
