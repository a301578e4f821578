// attend.cu -- shared-KV multi-query attention over the selected compressed
// entries (CSA) or all visible entries (HCA) plus the sliding window, in one
// softmax with a per-head sink, then R_{-t0} on the RoPE dims of the output
// ("DeepSeekV4技术报告阅读笔记" eq. 19, 26, 27, sections 2.5.2-2.5.3;
// "02 · DeepSeek-V4: 压缩注意力撑起 1M 上下文" section 2.4).
//
// SIMT path: a CTA owns (query, block of HB heads, split of the key list).
// Key tiles of 16 rows are dequantised into shared memory once and used by
// all HB heads (the single KV head is shared); logits and the online softmax
// run per head in 16-lane groups.  With more than one split, partial
// (max, sum, o) go to a workspace and a second kernel combines them in split
// order (deterministic), adds the sink and de-rotates.
#include "common.cuh"
#include "kernels.h"

namespace csa {

constexpr int kKT = 16;  // keys per tile

struct AttnArgs {
  const int32_t* q_pos;
  const void* q;
  const int32_t* idx;
  const void* ckv;
  const float* ckv_scale;
  const void* win;
  const float* win_scale;
  const int32_t* win_pos0;
  const float* sink;
  void* out;
  float* ws_o;  // [S][R][n_h][c]
  float* ws_ml; // [S][R][n_h][2]
  unsigned* err;
  int Q, N, W, n_h, c, rd, m, topk, n_win, nsplit, keys_per_split;
  int dense;
  float scale;
  double base;
};

__host__ __device__ inline size_t row_bytes(int kv, int c, int rd) {
  return kv == CSA_F32 ? (size_t)4 * c : kv == CSA_BF16 ? (size_t)2 * c : (size_t)(c - rd) + 2 * rd;
}

// Load 16-byte chunk `ch` of a stored row into fp32 shared memory.
template <int kKV>
__device__ __forceinline__ void load_chunk(const uint8_t* row, float scale, int ch,
                                           int c, int rd, float* dst) {
  const uint4 raw = *reinterpret_cast<const uint4*>(row + (size_t)ch * 16);
  if (kKV == CSA_F32) {
    const float* f = reinterpret_cast<const float*>(&raw);
    *reinterpret_cast<float4*>(dst + ch * 4) = make_float4(f[0], f[1], f[2], f[3]);
  } else if (kKV == CSA_BF16) {
    const __nv_bfloat16* h = reinterpret_cast<const __nv_bfloat16*>(&raw);
#pragma unroll
    for (int j = 0; j < 8; ++j) dst[ch * 8 + j] = __bfloat162float(h[j]);
  } else {
    const int nf = c - rd;
    const int nfc = nf / 16;  // code chunks
    if (ch < nfc) {
      const uint8_t* b = reinterpret_cast<const uint8_t*>(&raw);
#pragma unroll
      for (int j = 0; j < 16; ++j) dst[ch * 16 + j] = e4m3_to_f32(b[j]) * scale;
    } else {
      const __nv_bfloat16* h = reinterpret_cast<const __nv_bfloat16*>(&raw);
      const int e0 = nf + (ch - nfc) * 8;
#pragma unroll
      for (int j = 0; j < 8; ++j) dst[e0 + j] = __bfloat162float(h[j]);
    }
  }
}

// Apply R_{-t0} to dims e..e+3 (two pairs) if they lie in the RoPE range.
__device__ __forceinline__ void derotate4(float4& o, int e, int c, int rd, int t0,
                                          double base) {
  if (e < c - rd) return;
  const int p0 = (e - (c - rd)) >> 1;
  float cs, sn;
  rope_cs(-(double)t0, p0, rd, base, &cs, &sn);
  float x0 = o.x, x1 = o.y;
  o.x = x0 * cs - x1 * sn;
  o.y = x0 * sn + x1 * cs;
  rope_cs(-(double)t0, p0 + 1, rd, base, &cs, &sn);
  x0 = o.z; x1 = o.w;
  o.z = x0 * cs - x1 * sn;
  o.w = x0 * sn + x1 * cs;
}

template <typename T>
__device__ __forceinline__ void store4(T* dst, float4 v) {
  dst[0] = from_f32<T>(v.x); dst[1] = from_f32<T>(v.y);
  dst[2] = from_f32<T>(v.z); dst[3] = from_f32<T>(v.w);
}

template <typename T, int kKV, int CV4>
__global__ void attend_simt(AttnArgs a) {
  const int HB = blockDim.x / 16;
  const int c = a.c, cp = c + 4;
  extern __shared__ float sm[];
  float* qs = sm;                    // [HB][cp]
  float* ks = qs + HB * cp;          // [kKT][cp]
  float* ps = ks + kKT * cp;         // [HB][kKT]
  int* kvalid = reinterpret_cast<int*>(ps + HB * kKT);  // [kKT]

  const int r = blockIdx.x, hb = blockIdx.y, split = blockIdx.z;
  const int b = r / a.Q;
  const int t0 = a.q_pos[r];
  const int nv = n_visible(t0, a.m, a.N);
  const int lo = t0 - a.n_win + 1 > 0 ? t0 - a.n_win + 1 : 0;
  const int nwin_q = (a.n_win > 0 && t0 >= 0) ? t0 - lo + 1 : 0;
  const int n_main = a.dense ? nv : a.topk;
  const int nk = n_main + nwin_q;
  const int j_begin = split * a.keys_per_split;
  const int j_end = min(nk, j_begin + a.keys_per_split);

  const int tid = threadIdx.x;
  const int h = tid >> 4, g = tid & 15;
  const int head = hb * HB + h;

  // queries of this head block, pre-scaled by the softmax scale
  const T* qsrc = reinterpret_cast<const T*>(a.q) + ((size_t)r * a.n_h + hb * HB) * c;
  for (int i = tid; i < HB * c; i += blockDim.x)
    qs[(i / c) * cp + (i % c)] = to_f32(qsrc[i]) * a.scale;

  const size_t rb = row_bytes(kKV, c, a.rd);
  const int chunks = (int)(rb / 16);
  const uint8_t* ckv = reinterpret_cast<const uint8_t*>(a.ckv) + (size_t)b * a.N * rb;
  const uint8_t* win = reinterpret_cast<const uint8_t*>(a.win) + (size_t)b * a.W * rb;
  const int wp0 = a.win ? a.win_pos0[b] : 0;

  float m_run = -INFINITY, l_run = 0.f;
  float4 o[CV4];
#pragma unroll
  for (int i = 0; i < CV4; ++i) o[i] = make_float4(0.f, 0.f, 0.f, 0.f);

  __shared__ const uint8_t* s_row[kKT];
  __shared__ float s_sc[kKT];
  for (int j0 = j_begin; j0 < j_end; j0 += kKT) {
    __syncthreads();  // previous tile fully consumed
    // resolve the tile's key rows
    if (tid < kKT) {
      int j = j0 + tid;
      int valid = 0;
      const uint8_t* row = nullptr;
      float sc = 1.f;
      if (j < j_end) {
        if (j < n_main) {
          int s = a.dense ? j : a.idx[(size_t)r * a.topk + j];
          if (s >= 0) {
            if (s < nv) {
              valid = 1;
              row = ckv + (size_t)s * rb;
              if (kKV == CSA_KV_FP8MIX) sc = a.ckv_scale[(size_t)b * a.N + s];
            } else {
              atomicOr(a.err, CSA_DEV_BAD_INDEX);
            }
          }
        } else {
          int wr = lo + (j - n_main) - wp0;
          if (a.win != nullptr && wr >= 0 && wr < a.W) {
            valid = 1;
            row = win + (size_t)wr * rb;
            if (kKV == CSA_KV_FP8MIX) sc = a.win_scale[(size_t)b * a.W + wr];
          } else {
            atomicOr(a.err, CSA_DEV_BAD_WINDOW);
          }
        }
      }
      kvalid[tid] = valid;
      s_row[tid] = row;
      s_sc[tid] = sc;
    }
    __syncthreads();
    for (int i = tid; i < kKT * chunks; i += blockDim.x) {
      int jj = i / chunks, ch = i % chunks;
      if (kvalid[jj]) {
        load_chunk<kKV>(s_row[jj], s_sc[jj], ch, c, a.rd, ks + jj * cp);
      } else {
        for (int e = ch * c / chunks; e < (ch + 1) * c / chunks; ++e) ks[jj * cp + e] = 0.f;
      }
    }
    __syncthreads();
    // logits: thread (h, g) scores key g for head h
    float z = -INFINITY;
    if (kvalid[g]) {
      const float4* qv = reinterpret_cast<const float4*>(qs + h * cp);
      const float4* kv = reinterpret_cast<const float4*>(ks + g * cp);
      float acc = 0.f;
      for (int e4 = 0; e4 < c / 4; ++e4) {
        float4 x = qv[e4], y = kv[e4];
        acc = fmaf(x.x, y.x, acc); acc = fmaf(x.y, y.y, acc);
        acc = fmaf(x.z, y.z, acc); acc = fmaf(x.w, y.w, acc);
      }
      z = acc;
    }
    float tmax = z;
#pragma unroll
    for (int off = 8; off > 0; off >>= 1) tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, off));
    const float new_m = fmaxf(m_run, tmax);
    float p, alpha;
    if (new_m == -INFINITY) {
      p = 0.f;
      alpha = 1.f;
    } else {
      p = expf(z - new_m);
      alpha = expf(m_run - new_m);
    }
    float psum = p;
#pragma unroll
    for (int off = 8; off > 0; off >>= 1) psum += __shfl_xor_sync(0xffffffffu, psum, off);
    l_run = l_run * alpha + psum;
    m_run = new_m;
    ps[h * kKT + g] = p;
    __syncthreads();
    // o = alpha * o + sum_j p_j v_j  (thread owns dims 4*(g + 16 i) .. +3)
#pragma unroll
    for (int i = 0; i < CV4; ++i) {
      o[i].x *= alpha; o[i].y *= alpha; o[i].z *= alpha; o[i].w *= alpha;
    }
    for (int j = 0; j < kKT; ++j) {
      const float pj = ps[h * kKT + j];
      const float4* vr = reinterpret_cast<const float4*>(ks + j * cp);
#pragma unroll
      for (int i = 0; i < CV4; ++i) {
        float4 v = vr[g + 16 * i];
        o[i].x = fmaf(pj, v.x, o[i].x); o[i].y = fmaf(pj, v.y, o[i].y);
        o[i].z = fmaf(pj, v.z, o[i].z); o[i].w = fmaf(pj, v.w, o[i].w);
      }
    }
  }

  if (a.nsplit == 1) {
    const float zs = a.sink[head];
    const float M = fmaxf(m_run, zs);
    const float em = expf(m_run - M);
    const float den = l_run * em + expf(zs - M);
    const float f = em / den;
    T* dst = reinterpret_cast<T*>(a.out) + ((size_t)r * a.n_h + head) * c;
#pragma unroll
    for (int i = 0; i < CV4; ++i) {
      int e = 4 * (g + 16 * i);
      float4 v = make_float4(o[i].x * f, o[i].y * f, o[i].z * f, o[i].w * f);
      derotate4(v, e, c, a.rd, t0, a.base);
      store4<T>(dst + e, v);
    }
  } else {
    const size_t R = gridDim.x;
    const size_t slot = ((size_t)split * R + r) * a.n_h + head;
    float* dst = a.ws_o + slot * c;
#pragma unroll
    for (int i = 0; i < CV4; ++i) reinterpret_cast<float4*>(dst)[g + 16 * i] = o[i];
    if (g == 0) {
      a.ws_ml[slot * 2] = m_run;
      a.ws_ml[slot * 2 + 1] = l_run;
    }
  }
}

// Fixed-order combine of the splits, sink, normalisation, R_{-t0}, store.
// One CTA per (query, head): the split weights exp(m_s - M) are formed once
// in shared memory, then each thread sums its 4 dims over the splits with
// the loads issued back to back.
template <typename T>
__global__ void __launch_bounds__(128) attend_combine(AttnArgs a) {
  __shared__ float wsp[256];
  __shared__ float s_den;
  pdl_wait();  // partials of the attention kernel
  const int r = blockIdx.x, head = blockIdx.y;
  const size_t R = gridDim.x;
  const int c = a.c;
  const int S = a.nsplit;
  const float zs = a.sink[head];
  // R_{-t0} of this thread's first four dims, started before the partials
  // arrive (c = 4 blockDim.x covers every dim in one pass)
  const int t0 = a.q_pos[r];
  const int e_first = 4 * threadIdx.x;
  float rc0 = 1.f, rs0 = 0.f, rc1 = 1.f, rs1 = 0.f;
  const bool rope_now = e_first < c && e_first >= c - a.rd;
  if (rope_now) {
    const int p0 = (e_first - (c - a.rd)) >> 1;
    rope_cs(-(double)t0, p0, a.rd, a.base, &rc0, &rs0);
    rope_cs(-(double)t0, p0 + 1, a.rd, a.base, &rc1, &rs1);
  }
  // split maxima and sums (S <= 256)
  float mloc = -INFINITY;
  for (int s = threadIdx.x; s < S; s += blockDim.x)
    mloc = fmaxf(mloc, a.ws_ml[(((size_t)s * R + r) * a.n_h + head) * 2]);
  __shared__ float red[32];
  const float M = fmaxf(block_reduce<true>(mloc, red), zs);
  float dloc = 0.f;
  for (int s = threadIdx.x; s < S; s += blockDim.x) {
    const size_t slot = ((size_t)s * R + r) * a.n_h + head;
    const float wgt = expf(a.ws_ml[slot * 2] - M);
    wsp[s] = wgt;
    dloc += a.ws_ml[slot * 2 + 1] * wgt;
  }
  const float dsum = block_reduce<false>(dloc, red);
  if (threadIdx.x == 0) s_den = dsum + expf(zs - M);
  __syncthreads();
  const float inv = 1.0f / s_den;
  T* dst = reinterpret_cast<T*>(a.out) + ((size_t)r * a.n_h + head) * c;
  const size_t stride = R * a.n_h * (size_t)c / 4;  // float4 stride between splits
  for (int e = 4 * threadIdx.x; e < c; e += 4 * blockDim.x) {
    const float4* src = reinterpret_cast<const float4*>(a.ws_o + ((size_t)r * a.n_h + head) * c) + e / 4;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    int s = 0;
    for (; s + 8 <= S; s += 8) {  // eight partials in flight
      float4 v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) v[u] = __ldcg(src + (size_t)(s + u) * stride);
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const float f = wsp[s + u];
        acc.x = fmaf(f, v[u].x, acc.x); acc.y = fmaf(f, v[u].y, acc.y);
        acc.z = fmaf(f, v[u].z, acc.z); acc.w = fmaf(f, v[u].w, acc.w);
      }
    }
    for (; s < S; ++s) {
      const float4 v = src[(size_t)s * stride];
      const float f = wsp[s];
      acc.x = fmaf(f, v.x, acc.x); acc.y = fmaf(f, v.y, acc.y);
      acc.z = fmaf(f, v.z, acc.z); acc.w = fmaf(f, v.w, acc.w);
    }
    acc.x *= inv; acc.y *= inv; acc.z *= inv; acc.w *= inv;
    if (e == e_first && rope_now) {  // the factors computed at the start
      float x0 = acc.x, x1 = acc.y;
      acc.x = x0 * rc0 - x1 * rs0;
      acc.y = x0 * rs0 + x1 * rc0;
      x0 = acc.z; x1 = acc.w;
      acc.z = x0 * rc1 - x1 * rs1;
      acc.w = x0 * rs1 + x1 * rc1;
    } else {
      derotate4(acc, e, c, a.rd, t0, a.base);
    }
    store4<T>(dst + e, acc);
  }
}

static int head_block(int n_h) { return n_h >= 16 ? 16 : n_h; }

bool attend_tc_supported(const csa_params& p);
void attend_tc_plan(const csa_params& p, int R, int N, bool dense, int* nsplit, int* kps,
                    int* cluster);
csa_status launch_attend_tc(const csa_params& p, bool dense, int B, int Q,
                            const int32_t* q_pos, const void* q, const int32_t* idx,
                            const void* ckv, const float* ckv_scale, int N, const void* win,
                            const float* win_scale, int W, const int32_t* win_pos0,
                            const float* sink, void* out, float* ws_o, float* ws_ml,
                            int nsplit, int kps, int cluster, cudaStream_t st);

static void split_plan(const csa_params& p, int R, int N, bool dense, int* nsplit,
                       int* kps) {
  if (attend_tc_supported(p)) {
    int cluster = 0;
    attend_tc_plan(p, R, N, dense, nsplit, kps, &cluster);
    return;
  }
  const int HB = head_block(p.n_h);
  const int base_ctas = R * (p.n_h / HB);
  const int nk_max = (dense ? N : p.topk) + p.n_win;
  const int want = 148 * 4;
  int s = 1;
  if (base_ctas < want) s = (want + base_ctas - 1) / base_ctas;
  if (s > 256) s = 256;  // the combine keeps <= 256 split weights in shared memory
  int max_s = (nk_max + kKT - 1) / kKT;
  if (s > max_s) s = max_s;
  if (s < 1) s = 1;
  int k = (nk_max + s - 1) / s;
  k = (k + kKT - 1) / kKT * kKT;
  if (k < kKT) k = kKT;
  *nsplit = (nk_max + k - 1) / k;
  if (*nsplit < 1) *nsplit = 1;
  *kps = k;
}


size_t attend_ws_bytes(const csa_params& p, int B, int Q, int N, bool dense) {
  int ns, kps;
  split_plan(p, B * Q, N, dense, &ns, &kps);
  if (ns <= 1) return 0;
  size_t R = (size_t)B * Q;
  return align_up((size_t)ns * R * p.n_h * p.c * 4, 256) +
         align_up((size_t)ns * R * p.n_h * 2 * 4, 256);
}

template <typename T, int kKV, int CV4>
static void launch_attn_t(const AttnArgs& a, int R, cudaStream_t st) {
  const int HB = head_block(a.n_h);
  const int cp = a.c + 4;
  size_t smem = ((size_t)HB * cp + kKT * cp + HB * kKT + kKT) * sizeof(float);
  cudaFuncSetAttribute(attend_simt<T, kKV, CV4>,
                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  dim3 grid(R, a.n_h / HB, a.nsplit);
  CSA_LAUNCH(KK_ATTN, st, attend_simt<T, kKV, CV4><<<grid, HB * 16, smem, st>>>(a));
  if (a.nsplit > 1)
    CSA_LAUNCH(KK_COMBINE, st, attend_combine<T><<<dim3(R, a.n_h), 128, 0, st>>>(a));
}

template <typename T, int kKV>
static csa_status launch_attn_c(const AttnArgs& a, int R, cudaStream_t st) {
  switch (a.c) {
    case 64: launch_attn_t<T, kKV, 1>(a, R, st); break;
    case 128: launch_attn_t<T, kKV, 2>(a, R, st); break;
    case 256: launch_attn_t<T, kKV, 4>(a, R, st); break;
    case 512: launch_attn_t<T, kKV, 8>(a, R, st); break;
    default: return CSA_ERR_UNSUPPORTED;
  }
  return last_launch_status();
}

csa_status launch_attend(const csa_params& p, bool dense, int B, int Q,
                         const int32_t* q_pos, const void* q,
                         const int32_t* idx, const void* ckv,
                         const float* ckv_scale, int N, const void* win,
                         const float* win_scale, int W,
                         const int32_t* win_pos0, const float* sink, void* out,
                         void* ws, cudaStream_t st) {
  const int R = B * Q;
  AttnArgs a{};
  a.q_pos = q_pos; a.q = q; a.idx = idx; a.ckv = ckv; a.ckv_scale = ckv_scale;
  a.win = win; a.win_scale = win_scale; a.win_pos0 = win_pos0; a.sink = sink;
  a.out = out; a.err = device_error_word();
  a.Q = Q; a.N = N; a.W = W; a.n_h = p.n_h; a.c = p.c; a.rd = p.rope_dims; a.m = p.m;
  a.topk = p.topk; a.n_win = p.n_win; a.dense = dense ? 1 : 0;
  a.scale = p.softmax_scale; a.base = (double)p.rope_base;
  split_plan(p, R, N, dense, &a.nsplit, &a.keys_per_split);
  if (a.nsplit > 1) {
    a.ws_o = (float*)ws;
    a.ws_ml = (float*)((char*)ws + align_up((size_t)a.nsplit * R * p.n_h * p.c * 4, 256));
  }
  if (attend_tc_supported(p)) {
    // up to 8 key slices of a (query, head block) are combined inside the
    // kernel (one cluster each); more slices are combined by attend_combine
    int cluster = 0, ns = 0, kps = 0;
    attend_tc_plan(p, R, N, dense, &ns, &kps, &cluster);  // the split of a.nsplit
    csa_status s = launch_attend_tc(p, dense, B, Q, q_pos, q, idx, ckv, ckv_scale, N, win,
                                    win_scale, W, win_pos0, sink, out, a.ws_o, a.ws_ml,
                                    a.nsplit, a.keys_per_split, cluster, st);
    if (s != CSA_OK || a.nsplit <= 1 || cluster) return s;
    cudaError_t e = cudaSuccess;
    CSA_LAUNCH(KK_COMBINE, st,
               e = launch_maybe_pdl(kPdlCombine, attend_combine<__nv_bfloat16>, dim3(R, a.n_h),
                                    dim3(128), 0, st, a));
    return e == cudaSuccess ? CSA_OK : CSA_ERR_CUDA;
  }
  if (p.act == CSA_F32) {
    if (p.kv == CSA_F32) return launch_attn_c<float, CSA_F32>(a, R, st);
    if (p.kv == CSA_BF16) return launch_attn_c<float, CSA_BF16>(a, R, st);
    return launch_attn_c<float, CSA_KV_FP8MIX>(a, R, st);
  }
  if (p.kv == CSA_F32) return launch_attn_c<__nv_bfloat16, CSA_F32>(a, R, st);
  if (p.kv == CSA_BF16) return launch_attn_c<__nv_bfloat16, CSA_BF16>(a, R, st);
  return launch_attn_c<__nv_bfloat16, CSA_KV_FP8MIX>(a, R, st);
}

}  // namespace csa
