// index_topk.cu -- Lightning-Indexer scores and top-k selection
// ("DeepSeekV4技术报告阅读笔记" eq. 16-17; "02 · DeepSeek-V4: 压缩注意力撑起 1M
// 上下文" section 2.2: 64 indexer heads of width 128, top-k 512 / 1024).
//
// Scores I[r][s] = sum_h w[r][h] * ReLU(qI[r][h] . kI[b][s]) are written to an
// fp32 workspace [B*Q][N] for the visible entries s < floor((t0+1)/m); a
// radix-select kernel then keeps the top k of each query (ties -> lower s)
// and writes them in ascending index order.
#include "common.cuh"
#include "kernels.h"

namespace csa {

// ---------------------------------------------------------- SIMT scorer --
// One thread per (query, entry); the query's heads live in shared memory.
template <typename T, int NH>
__global__ void __launch_bounds__(256) index_scores_simt(
    const int32_t* __restrict__ q_pos, const T* __restrict__ qI,
    const float* __restrict__ w, const T* __restrict__ kI, int Q, int N, int m,
    int nhI, int cI, float* __restrict__ scores) {
  extern __shared__ float qs[];  // [NH][cI] then ws[NH]
  float* ws = qs + NH * cI;
  const int r = blockIdx.x;
  const int b = r / Q;
  const int nv = n_visible(q_pos[r], m, N);
  const int s0 = blockIdx.y * blockDim.x;
  if (s0 >= nv) return;
  for (int i = threadIdx.x; i < NH * cI; i += blockDim.x) {
    int h = i / cI;
    qs[i] = h < nhI ? to_f32(qI[((size_t)r * nhI + h) * cI + (i % cI)]) : 0.f;
  }
  for (int h = threadIdx.x; h < NH; h += blockDim.x) ws[h] = h < nhI ? w[(size_t)r * nhI + h] : 0.f;
  __syncthreads();
  const int s = s0 + threadIdx.x;
  if (s >= nv) return;
  const T* k = kI + ((size_t)b * N + s) * cI;
  float acc[NH];
#pragma unroll
  for (int h = 0; h < NH; ++h) acc[h] = 0.f;
  for (int e0 = 0; e0 < cI; e0 += 8) {
    float kv[8];
    if (sizeof(T) == 2) {
      uint4 raw = *reinterpret_cast<const uint4*>(k + e0);
      const __nv_bfloat16* hb = reinterpret_cast<const __nv_bfloat16*>(&raw);
#pragma unroll
      for (int j = 0; j < 8; ++j) kv[j] = __bfloat162float(hb[j]);
    } else {
      float4 a = *reinterpret_cast<const float4*>(k + e0);
      float4 c = *reinterpret_cast<const float4*>(k + e0 + 4);
      kv[0] = a.x; kv[1] = a.y; kv[2] = a.z; kv[3] = a.w;
      kv[4] = c.x; kv[5] = c.y; kv[6] = c.z; kv[7] = c.w;
    }
#pragma unroll
    for (int h = 0; h < NH; ++h) {
      const float4 q0 = *reinterpret_cast<const float4*>(qs + h * cI + e0);
      const float4 q1 = *reinterpret_cast<const float4*>(qs + h * cI + e0 + 4);
      float a = acc[h];
      a = fmaf(q0.x, kv[0], a); a = fmaf(q0.y, kv[1], a);
      a = fmaf(q0.z, kv[2], a); a = fmaf(q0.w, kv[3], a);
      a = fmaf(q1.x, kv[4], a); a = fmaf(q1.y, kv[5], a);
      a = fmaf(q1.z, kv[6], a); a = fmaf(q1.w, kv[7], a);
      acc[h] = a;
    }
  }
  float sc = 0.f;
#pragma unroll
  for (int h = 0; h < NH; ++h) sc = fmaf(ws[h], fmaxf(acc[h], 0.f), sc);
  scores[(size_t)r * N + s] = sc;
}

// ------------------------------------------------------------ radix top-k --
// One 1024-thread CTA per query.  Three digit passes (11, 11, 10 bits) over
// the order-preserving keys find the k-th largest key K; the output takes
// every entry with key > K and the lowest-index entries with key == K.
constexpr int kTopkThreads = 1024;

__global__ void __launch_bounds__(kTopkThreads) topk_radix(
    const float* __restrict__ scores, int N, const int32_t* __restrict__ q_pos,
    int m, int k, int32_t* __restrict__ idx_out, float* __restrict__ score_out) {
  __shared__ unsigned hist[2048];
  __shared__ unsigned scan_sh[33];
  __shared__ unsigned s_digit, s_remaining;
  const int r = blockIdx.x;
  const int nv = n_visible(q_pos[r], m, N);
  const float* sc = scores + (size_t)r * N;
  int32_t* out = idx_out + (size_t)r * k;
  float* sout = score_out ? score_out + (size_t)r * k : nullptr;
  if (nv <= k) {
    for (int j = threadIdx.x; j < k; j += blockDim.x) {
      out[j] = j < nv ? j : -1;
      if (sout) sout[j] = j < nv ? sc[j] : -INFINITY;
    }
    return;
  }
  unsigned prefix = 0, mask = 0;
  unsigned remaining = (unsigned)k;  // rank of the wanted key among those matching prefix
  const int shifts[3] = {21, 10, 0};
  const int widths[3] = {11, 11, 10};
  for (int pass = 0; pass < 3; ++pass) {
    const int shift = shifts[pass];
    const unsigned dmask = (1u << widths[pass]) - 1u;
    for (int i = threadIdx.x; i < 2048; i += blockDim.x) hist[i] = 0;
    __syncthreads();
    for (int s = threadIdx.x; s < nv; s += blockDim.x) {
      unsigned key = score_key(sc[s]);
      if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & dmask], 1u);
    }
    __syncthreads();
    // suffix sums: thread t owns bins 2t and 2t+1; scan in descending order
    const int t = threadIdx.x;
    const int rt = kTopkThreads - 1 - t;  // rt-th thread holds bins 2rt, 2rt+1
    unsigned h_hi = hist[2 * rt + 1], h_lo = hist[2 * rt];
    unsigned total;
    unsigned above = block_exclusive_scan(h_hi + h_lo, scan_sh, &total);
    // `above` = keys in bins > 2rt+1
    if (above < remaining && above + h_hi >= remaining) {
      s_digit = 2 * rt + 1;
      s_remaining = remaining - above;
    } else if (above + h_hi < remaining && above + h_hi + h_lo >= remaining) {
      s_digit = 2 * rt;
      s_remaining = remaining - above - h_hi;
    }
    __syncthreads();
    prefix |= s_digit << shift;
    mask |= dmask << shift;
    remaining = s_remaining;
    __syncthreads();
  }
  // prefix = K (exact key of the k-th largest); `remaining` keys equal to K
  // are taken, lowest index first.
  const unsigned K = prefix;
  unsigned eq_before = 0, sel_before = 0;
  for (int base = 0; base < nv; base += blockDim.x) {
    const int s = base + threadIdx.x;
    unsigned key = s < nv ? score_key(sc[s]) : 0u;
    bool gt = s < nv && key > K;
    bool eq = s < nv && key == K;
    unsigned eq_tot, sel_tot;
    unsigned eq_rank = block_exclusive_scan(eq ? 1u : 0u, scan_sh, &eq_tot);
    bool sel = gt || (eq && eq_before + eq_rank < remaining);
    unsigned pos = block_exclusive_scan(sel ? 1u : 0u, scan_sh, &sel_tot);
    if (sel) {
      out[sel_before + pos] = s;
      if (sout) sout[sel_before + pos] = sc[s];
    }
    eq_before += eq_tot;
    sel_before += sel_tot;
  }
}

size_t index_topk_ws_bytes(const csa_params& p, int B, int Q, int N) {
  return align_up((size_t)B * Q * N * sizeof(float), 256);
}

template <typename T>
static void launch_scores(const csa_params& p, int B, int Q, const int32_t* q_pos,
                          const void* qI, const float* w, const void* kI, int N,
                          float* scores, cudaStream_t st) {
  const int R = B * Q;
  if (N == 0) return;
  dim3 grid(R, (N + 255) / 256);
  int nh = p.n_hI <= 4 ? 4 : p.n_hI <= 8 ? 8 : p.n_hI <= 16 ? 16 : p.n_hI <= 32 ? 32 : 64;
  size_t smem = ((size_t)nh * p.c_I + nh) * sizeof(float);
#define CSA_SCORES(NH)                                                          \
  do {                                                                          \
    cudaFuncSetAttribute(index_scores_simt<T, NH>,                              \
                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem); \
    CSA_LAUNCH(KK_SCORES, st, index_scores_simt<T, NH><<<grid, 256, smem, st>>>( \
        q_pos, (const T*)qI, w, (const T*)kI, Q, N, p.m, p.n_hI, p.c_I, scores)); \
  } while (0)
  switch (nh) {
    case 4: CSA_SCORES(4); break;
    case 8: CSA_SCORES(8); break;
    case 16: CSA_SCORES(16); break;
    case 32: CSA_SCORES(32); break;
    default: CSA_SCORES(64); break;
  }
#undef CSA_SCORES
}

csa_status launch_index_topk(const csa_params& p, int B, int Q,
                             const int32_t* q_pos, const void* qI,
                             const float* w, const void* kI, int N,
                             int32_t* idx_out, float* score_out, void* ws,
                             cudaStream_t st) {
  float* scores = (float*)ws;
  if (p.act == CSA_F32)
    launch_scores<float>(p, B, Q, q_pos, qI, w, kI, N, scores, st);
  else
    launch_scores<__nv_bfloat16>(p, B, Q, q_pos, qI, w, kI, N, scores, st);
  CSA_LAUNCH(KK_TOPK, st, topk_radix<<<B * Q, kTopkThreads, 0, st>>>(
                              scores, N, q_pos, p.m, p.topk, idx_out, score_out));
  return last_launch_status();
}

}  // namespace csa
