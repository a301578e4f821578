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
// Block-wide exact top-k of one query's scores sc[0..nv) (nv > k), 1024
// threads.  Three digit passes (11, 11, 10 bits) over the order-preserving
// keys find the k-th largest key K; the output takes every entry with key > K
// and the lowest-index entries with key == K, in ascending index order.
constexpr int kTopkThreads = 1024;

struct RadixShared {
  unsigned hist[2048];
  unsigned scan[33];
  unsigned digit, remaining;
};

__device__ void radix_select_block(const float* __restrict__ sc, int nv, int k,
                                   int32_t* __restrict__ out, float* __restrict__ sout,
                                   RadixShared& sh) {
  unsigned prefix = 0, mask = 0;
  unsigned remaining = (unsigned)k;  // rank of the wanted key among those matching prefix
  const int shifts[3] = {21, 10, 0};
  const int widths[3] = {11, 11, 10};
  for (int pass = 0; pass < 3; ++pass) {
    const int shift = shifts[pass];
    const unsigned dmask = (1u << widths[pass]) - 1u;
    for (int i = threadIdx.x; i < 2048; i += blockDim.x) sh.hist[i] = 0;
    __syncthreads();
    for (int s = threadIdx.x; s < nv; s += blockDim.x) {
      unsigned key = score_key(sc[s]);
      if ((key & mask) == prefix) atomicAdd(&sh.hist[(key >> shift) & dmask], 1u);
    }
    __syncthreads();
    // thread t owns bins 2rt, 2rt+1 with rt = 1023 - t, so the exclusive scan
    // over t counts the keys in higher bins
    const int rt = kTopkThreads - 1 - threadIdx.x;
    unsigned h_hi = sh.hist[2 * rt + 1], h_lo = sh.hist[2 * rt];
    unsigned total;
    unsigned above = block_exclusive_scan(h_hi + h_lo, sh.scan, &total);
    if (above < remaining && above + h_hi >= remaining) {
      sh.digit = 2 * rt + 1;
      sh.remaining = remaining - above;
    } else if (above + h_hi < remaining && above + h_hi + h_lo >= remaining) {
      sh.digit = 2 * rt;
      sh.remaining = remaining - above - h_hi;
    }
    __syncthreads();
    prefix |= sh.digit << shift;
    mask |= dmask << shift;
    remaining = sh.remaining;
    __syncthreads();
  }
  const unsigned K = prefix;
  unsigned eq_before = 0, sel_before = 0;
  for (int base = 0; base < nv; base += blockDim.x) {
    const int s = base + threadIdx.x;
    unsigned key = s < nv ? score_key(sc[s]) : 0u;
    bool gt = s < nv && key > K;
    bool eq = s < nv && key == K;
    unsigned eq_tot, sel_tot;
    unsigned eq_rank = block_exclusive_scan(eq ? 1u : 0u, sh.scan, &eq_tot);
    bool sel = gt || (eq && eq_before + eq_rank < remaining);
    unsigned pos = block_exclusive_scan(sel ? 1u : 0u, sh.scan, &sel_tot);
    if (sel) {
      out[sel_before + pos] = s;
      if (sout) sout[sel_before + pos] = sc[s];
    }
    eq_before += eq_tot;
    sel_before += sel_tot;
  }
}

__device__ __forceinline__ void write_all_visible(const float* sc, int nv, int k, int32_t* out,
                                                  float* sout) {
  for (int j = threadIdx.x; j < k; j += blockDim.x) {
    out[j] = j < nv ? j : -1;
    if (sout) sout[j] = j < nv ? sc[j] : -INFINITY;
  }
}

// Top-k of one query with at most kFastMax visible entries, all in one
// pass of loads (1024 threads x 8 consecutive entries in registers): a
// histogram of the top 12 key bits gives the bin T of the k-th key; the keys
// of bin T are listed and a two-digit radix select over their low 20 bits
// gives the exact k-th key K; one scan of (key > K, key == K) counts then
// places every selected entry in index order, the lowest indices first
// among keys equal to K.  Returns false, before writing any output, when bin
// T holds more than kFastCand keys.
constexpr int kFastMax = 8192;
constexpr int kFastCand = 2048;
struct FastTopkSmem {
  unsigned hist[4096];
  uint2 cand[kFastCand];
};

__device__ bool topk_block_fast(const float* __restrict__ sc, int nv, int k,
                                int32_t* __restrict__ out, float* __restrict__ sout,
                                FastTopkSmem& F, RadixShared& sh) {
  __shared__ unsigned s_nc;
  __shared__ int sT;
  __shared__ unsigned sAbove;
  const int t = threadIdx.x;
  const int sb = t * 8;
  float v[8];
  if ((((uintptr_t)sc) & 15) == 0 && sb + 8 <= nv) {
    const float4 a0 = __ldg(reinterpret_cast<const float4*>(sc + sb));
    const float4 a1 = __ldg(reinterpret_cast<const float4*>(sc + sb + 4));
    v[0] = a0.x; v[1] = a0.y; v[2] = a0.z; v[3] = a0.w;
    v[4] = a1.x; v[5] = a1.y; v[6] = a1.z; v[7] = a1.w;
  } else {
#pragma unroll
    for (int u = 0; u < 8; ++u) v[u] = sb + u < nv ? __ldg(sc + sb + u) : 0.f;
  }
  unsigned key[8];
#pragma unroll
  for (int u = 0; u < 8; ++u) key[u] = score_key(v[u]);
#pragma unroll
  for (int j = 0; j < 4; ++j) F.hist[4 * t + j] = 0;
  if (t == 0) s_nc = 0;
  __syncthreads();
#pragma unroll
  for (int u = 0; u < 8; ++u)
    if (sb + u < nv) atomicAdd(&F.hist[key[u] >> 20], 1u);
  __syncthreads();
  // bin T of the k-th key: thread t owns bins 4(1023 - t) .. +3
  {
    const int rt = 1023 - t;
    unsigned c[4], sum = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      c[j] = F.hist[4 * rt + j];
      sum += c[j];
    }
    unsigned tot;
    unsigned above = block_exclusive_scan(sum, sh.scan, &tot);
#pragma unroll
    for (int j = 3; j >= 0; --j) {
      if (above < (unsigned)k && above + c[j] >= (unsigned)k) {
        sT = 4 * rt + j;
        sAbove = above;
      }
      above += c[j];
    }
  }
  __syncthreads();
  const int T = sT;
  const unsigned above = sAbove;
#pragma unroll
  for (int u = 0; u < 8; ++u)
    if (sb + u < nv && (int)(key[u] >> 20) == T) {
      const unsigned p = atomicAdd(&s_nc, 1u);
      if (p < (unsigned)kFastCand) F.cand[p] = make_uint2(key[u], 0u);
    }
  __syncthreads();
  const unsigned nc = s_nc;
  if (nc > (unsigned)kFastCand) return false;
  // exact k-th key among the candidates (keys only: ties are settled below)
  unsigned remaining = (unsigned)k - above;
  unsigned prefix = (unsigned)T << 20, mask = 0xFFF00000u;
  for (int pass = 0; pass < 2; ++pass) {
    const int shift = pass == 0 ? 10 : 0;
    sh.hist[t] = 0;
    __syncthreads();
    for (unsigned j = t; j < nc; j += 1024) {
      const unsigned kk = F.cand[j].x;
      if ((kk & mask) == prefix) atomicAdd(&sh.hist[(kk >> shift) & 1023u], 1u);
    }
    __syncthreads();
    const int bin = 1023 - t;
    const unsigned hc = sh.hist[bin];
    unsigned tot;
    const unsigned higher = block_exclusive_scan(hc, sh.scan, &tot);
    if (higher < remaining && higher + hc >= remaining) {
      sh.digit = (unsigned)bin;
      sh.remaining = remaining - higher;
    }
    __syncthreads();
    prefix |= sh.digit << shift;
    mask |= 1023u << shift;
    remaining = sh.remaining;
  }
  const unsigned K = prefix;
  // one scan of (key > K, key == K) counts: positions in index order
  unsigned ngt = 0, neq = 0;
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    const bool vis = sb + u < nv;
    ngt += (vis && key[u] > K) ? 1u : 0u;
    neq += (vis && key[u] == K) ? 1u : 0u;
  }
  unsigned tge;
  const unsigned x = block_exclusive_scan((ngt << 16) | neq, sh.scan, &tge);
  unsigned bg = x >> 16, be = x & 0xFFFFu;
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    if (sb + u >= nv) continue;
    int pos = -1;
    if (key[u] > K) {
      pos = (int)(bg + min(be, remaining));
      ++bg;
    } else if (key[u] == K) {
      if (be < remaining) pos = (int)(bg + be);
      ++be;
    }
    if (pos >= 0 && pos < k) {
      out[pos] = sb + u;
      if (sout) sout[pos] = v[u];
    }
  }
  return true;
}

// One CTA per query (used when there are many queries).
__global__ void __launch_bounds__(kTopkThreads, 2) topk_radix(
    const float* __restrict__ scores, int N, const int32_t* __restrict__ q_pos,
    int m, int k, int32_t* __restrict__ idx_out, float* __restrict__ score_out) {
  extern __shared__ __align__(16) uint8_t topk_fast_smem[];
  __shared__ RadixShared sh;
  __shared__ int s_ok;
  const int r = blockIdx.x;
  const int nv = n_visible(q_pos[r], m, N);
  const float* sc = scores + (size_t)r * N;
  int32_t* out = idx_out + (size_t)r * k;
  float* sout = score_out ? score_out + (size_t)r * k : nullptr;
  if (nv <= k) {
    write_all_visible(sc, nv, k, out, sout);
    return;
  }
  if (nv <= kFastMax) {
    const bool ok = topk_block_fast(sc, nv, k, out, sout,
                                    *reinterpret_cast<FastTopkSmem*>(topk_fast_smem), sh);
    if (threadIdx.x == 0) s_ok = ok;
    __syncthreads();
    if (s_ok) return;
  }
  radix_select_block(sc, nv, k, out, sout, sh);
}

// ------------------------------------------------- multi-CTA top-k (few q) --
// For a handful of queries with long visible ranges (decode).  (1) The top 12
// key bits of every visible score are histogrammed (by the tensor-core
// scorer's epilogue, or by topk_hist).  (2) Every CTA of the select pass
// takes a chunk of one query's scores (8 consecutive entries per thread),
// finds the bin T that holds the k-th largest key, and writes, in index
// order, the entries of higher bins ("above") and the (key, index) pairs of
// bin T ("candidates") to its chunk's slots, with their counts.  (3) The last
// CTA of the query gathers both lists in index order, finds the exact k-th
// key among the candidates (radix select over the low 20 key bits), keeps the
// candidates above it and, of those equal to it, the lowest indices, and
// merges the two ascending lists into the output.  A chunk or query whose
// candidates overflow the slots falls back to the exact block-wide select.
constexpr int kBins = 4096;
constexpr int kChunk = 8192;     // entries per CTA in (1) and (2)
constexpr int kPer = kChunk / 1024;
constexpr int kMaxChunks = 512;  // chunks of one query (counts fit one packed scan)
constexpr int kCandCap = 4096;   // candidates per query in (3)
constexpr int kAboveCap = 4096;  // largest k of this path
constexpr int kLocalCap = 2048;  // candidate slots per chunk

struct MultiTopkWs {
  unsigned* ghist;  // [R][kBins]
  unsigned* done;   // [R] CTAs of the select pass that have finished
  uint2* ccnt;      // [R][nch] (above, candidates) per chunk
  int* above;       // [R][nch][k] above entries of each chunk, ascending
  uint2* cand;      // [R][nch][kLocalCap] (key, index) of each chunk, ascending
};

// dynamic shared memory of topk_select_final (finalize)
struct SelectSmem {
  int a[kAboveCap];       // above entries of the query, ascending
  uint2 c[kCandCap];      // candidates of the query, ascending by index
  int cs[kAboveCap];      // chosen candidates, ascending
  unsigned oa[kMaxChunks + 1], oc[kMaxChunks + 1];  // chunk offsets
};

__global__ void __launch_bounds__(1024) topk_hist(const float* __restrict__ scores, int N,
                                                  const int32_t* __restrict__ q_pos, int m,
                                                  int k, unsigned* __restrict__ ghist) {
  __shared__ unsigned h[kBins];
  const int r = blockIdx.x;
  const int nv = n_visible(q_pos[r], m, N);
  if (nv <= k) return;
  const int s0 = blockIdx.y * kChunk;
  if (s0 >= nv) return;
  const int s1 = min(nv, s0 + kChunk);
  for (int i = threadIdx.x; i < kBins; i += blockDim.x) h[i] = 0;
  __syncthreads();
  const float* sc = scores + (size_t)r * N;
  for (int s = s0 + threadIdx.x; s < s1; s += blockDim.x) atomicAdd(&h[score_key(sc[s]) >> 20], 1u);
  __syncthreads();
  for (int i = threadIdx.x; i < kBins; i += blockDim.x)
    if (h[i]) atomicAdd(&ghist[(size_t)r * kBins + i], h[i]);
}

// Bin holding the k-th largest key and the number of keys in higher bins
// (1024 threads, 4 bins each).
__device__ void find_threshold_bin(const unsigned* __restrict__ gh, unsigned k, unsigned* scan,
                                   int* T_out, unsigned* above_out, int* sT, unsigned* sAbove) {
  const int rt = 1023 - (int)threadIdx.x;  // bins 4rt .. 4rt+3
  unsigned c[4];
  unsigned sum = 0;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    c[j] = __ldcg(gh + 4 * rt + j);
    sum += c[j];
  }
  unsigned total;
  unsigned above = block_exclusive_scan(sum, scan, &total);
#pragma unroll
  for (int j = 3; j >= 0; --j) {
    if (above < k && above + c[j] >= k) {
      *sT = 4 * rt + j;
      *sAbove = above;
    }
    above += c[j];
  }
  __syncthreads();
  *T_out = *sT;
  *above_out = *sAbove;
}

// first position in the ascending list v[0..n) whose value is >= x
template <typename F>
__device__ __forceinline__ unsigned lower_bound(unsigned n, int x, F at) {
  unsigned lo = 0, hi = n;
  while (lo < hi) {
    const unsigned mid = (lo + hi) >> 1;
    if (at(mid) < x) lo = mid + 1; else hi = mid;
  }
  return lo;
}

// Exact completion of one query's selection (1024 threads).  Returns false,
// before writing any output, when the candidates do not fit (the caller then
// runs the exact block-wide select).
__device__ bool finalize_query(const float* __restrict__ sc, int k, int r, int nch, int T,
                               unsigned above, const MultiTopkWs& ws, int32_t* __restrict__ out,
                               float* __restrict__ sout, SelectSmem& S, RadixShared& sh) {
  const int t = threadIdx.x;
  // chunk counts -> offsets of each chunk's lists in the query's lists
  uint2 cc = make_uint2(0u, 0u);
  if (t < nch) cc = __ldcg(ws.ccnt + (size_t)r * nch + t);
  // a chunk whose candidates filled its slots takes the exact select
  const int bad = __syncthreads_or(t < nch && cc.y >= (unsigned)kLocalCap);
  // one scan of both counts: above entries < k <= 4096 in bits 20..31,
  // candidates (< kLocalCap per chunk, kMaxChunks chunks: < 2^20) below
  const unsigned cy = min(cc.y, (unsigned)kLocalCap - 1u);
  unsigned tot2;
  const unsigned x2 = block_exclusive_scan((min(cc.x, 4095u) << 20) | cy, sh.scan, &tot2);
  const unsigned xa = x2 >> 20, xc = x2 & 0xFFFFFu;
  unsigned na = tot2 >> 20, ncand = tot2 & 0xFFFFFu;
  if (t < nch) {
    S.oa[t] = xa;
    S.oc[t] = xc;
  }
  if (t == 0) {
    S.oa[nch] = na;
    S.oc[nch] = ncand;
  }
  __syncthreads();
  if (bad || na != above || ncand > (unsigned)kCandCap) return false;
  // gather both lists in index order (chunk c's slice follows chunk c-1's)
  auto chunk_of = [&](const unsigned* off, unsigned j) {
    unsigned lo = 0, hi = (unsigned)nch - 1;  // last c with off[c] <= j
    while (lo < hi) {
      const unsigned mid = (lo + hi + 1) >> 1;
      if (off[mid] <= j) lo = mid; else hi = mid - 1;
    }
    return lo;
  };
  for (unsigned j = t; j < na; j += 1024) {
    const unsigned c = chunk_of(S.oa, j);
    S.a[j] = __ldcg(ws.above + ((size_t)r * nch + c) * k + (j - S.oa[c]));
  }
  for (unsigned j = t; j < ncand; j += 1024) {
    const unsigned c = chunk_of(S.oc, j);
    S.c[j] = __ldcg(ws.cand + ((size_t)r * nch + c) * kLocalCap + (j - S.oc[c]));
  }
  __syncthreads();
  // radix select of the remaining-th largest key among the candidates: two
  // 10-bit digits below the 12 bits of bin T
  unsigned remaining = (unsigned)k - above;  // 1 <= remaining <= ncand
  unsigned prefix = (unsigned)T << 20, mask = 0xFFF00000u;
  for (int pass = 0; pass < 2; ++pass) {
    const int shift = pass == 0 ? 10 : 0;
    sh.hist[t] = 0;
    __syncthreads();
    for (unsigned j = t; j < ncand; j += 1024) {
      const unsigned key = S.c[j].x;
      if ((key & mask) == prefix) atomicAdd(&sh.hist[(key >> shift) & 1023u], 1u);
    }
    __syncthreads();
    const int bin = 1023 - t;  // the scan over t counts the higher bins
    const unsigned hc = sh.hist[bin];
    unsigned tot;
    const unsigned higher = block_exclusive_scan(hc, sh.scan, &tot);
    if (higher < remaining && higher + hc >= remaining) {
      sh.digit = (unsigned)bin;
      sh.remaining = remaining - higher;
    }
    __syncthreads();
    prefix |= sh.digit << shift;
    mask |= 1023u << shift;
    remaining = sh.remaining;
  }
  const unsigned K = prefix;  // exact key of the k-th largest score
  // candidates kept: keys above K, and the `remaining` lowest indices with
  // key K.  Thread t owns the four consecutive candidates 4t .. 4t+3; one
  // scan of (greater, equal) counts gives every kept candidate its place.
  unsigned kgt = 0, keq = 0;
  uint2 cv[4];
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const unsigned j = 4u * t + u;
    cv[u] = j < ncand ? S.c[j] : make_uint2(0u, 0u);
    kgt += (j < ncand && cv[u].x > K) ? 1u : 0u;
    keq += (j < ncand && cv[u].x == K) ? 1u : 0u;
  }
  unsigned tge;
  const unsigned xge = block_exclusive_scan((kgt << 16) | keq, sh.scan, &tge);
  unsigned ngt = xge >> 16, neq = xge & 0xFFFFu;  // before this thread's candidates
  const unsigned nkeep = (tge >> 16) + min(tge & 0xFFFFu, remaining);
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const unsigned j = 4u * t + u;
    if (j >= ncand) continue;
    if (cv[u].x > K) {
      S.cs[ngt + min(neq, remaining)] = (int)cv[u].y;
      ++ngt;
    } else if (cv[u].x == K) {
      if (neq < remaining) S.cs[ngt + neq] = (int)cv[u].y;
      ++neq;
    }
  }
  __syncthreads();
  // merge the two ascending lists: position = own rank + rank in the other
  for (unsigned j = t; j < na; j += 1024) {
    const int s = S.a[j];
    const unsigned pos = j + lower_bound(nkeep, s, [&](unsigned i) { return S.cs[i]; });
    if (pos < (unsigned)k) {
      out[pos] = s;
      if (sout) sout[pos] = sc[s];
    }
  }
  for (unsigned j = t; j < nkeep; j += 1024) {
    const int s = S.cs[j];
    const unsigned pos = j + lower_bound(na, s, [&](unsigned i) { return S.a[i]; });
    if (pos < (unsigned)k) {
      out[pos] = s;
      if (sout) sout[pos] = sc[s];
    }
  }
  return true;
}

// Selection pass over a chunk of one query's scores; the last CTA of the
// query to finish completes the query (threadfence + counter).
__global__ void __launch_bounds__(1024) topk_select_final(
    const float* __restrict__ scores, int N, const int32_t* __restrict__ q_pos, int m, int k,
    MultiTopkWs ws, int32_t* __restrict__ idx_out, float* __restrict__ score_out) {
  extern __shared__ __align__(16) uint8_t topk_smem[];
  SelectSmem& S = *reinterpret_cast<SelectSmem*>(topk_smem);
  __shared__ RadixShared sh;
  __shared__ int sT;
  __shared__ unsigned sAbove;
  __shared__ int s_last, s_exact;
  pdl_trigger();  // the attention kernel may take the SMs this grid frees
  pdl_wait();     // scores and histograms of the scoring kernel
  const int r = blockIdx.x, c = blockIdx.y, nch = gridDim.y;
  const int nv = n_visible(q_pos[r], m, N);
  const float* sc = scores + (size_t)r * N;
  int32_t* out = idx_out + (size_t)r * k;
  float* sout = score_out ? score_out + (size_t)r * k : nullptr;
  int T = 0;
  unsigned above = 0;
  if (nv > k) {
    // this thread's 8 consecutive scores first (in flight while the
    // threshold is found)
    const int sb = c * kChunk + (int)threadIdx.x * kPer;
    float v[kPer];
    if ((N & 3) == 0 && sb + kPer <= nv) {  // two 16-byte loads
      const float4 a0 = __ldcg(reinterpret_cast<const float4*>(sc + sb));
      const float4 a1 = __ldcg(reinterpret_cast<const float4*>(sc + sb + 4));
      v[0] = a0.x; v[1] = a0.y; v[2] = a0.z; v[3] = a0.w;
      v[4] = a1.x; v[5] = a1.y; v[6] = a1.z; v[7] = a1.w;
    } else {
#pragma unroll
      for (int u = 0; u < kPer; ++u) v[u] = sb + u < nv ? __ldcg(sc + sb + u) : 0.f;
    }
    find_threshold_bin(ws.ghist + (size_t)r * kBins, (unsigned)k, sh.scan, &T, &above, &sT,
                       &sAbove);
    unsigned na = 0, nc = 0;
    unsigned key[kPer];
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
      key[u] = score_key(v[u]);
      const int bin = (int)(key[u] >> 20);
      const bool vis = sb + u < nv;
      na += (vis && bin > T) ? 1u : 0u;
      nc += (vis && bin == T) ? 1u : 0u;
    }
    // one scan of both counts (each total <= kChunk < 2^16)
    unsigned tot;
    const unsigned x = block_exclusive_scan(na | (nc << 16), sh.scan, &tot);
    unsigned pa = x & 0xFFFFu, pc = x >> 16;
    int* ab = ws.above + ((size_t)r * nch + c) * k;
    uint2* cd = ws.cand + ((size_t)r * nch + c) * kLocalCap;
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
      if (sb + u >= nv) continue;
      const int bin = (int)(key[u] >> 20);
      if (bin > T) {
        if (pa < (unsigned)k) ab[pa] = sb + u;  // a chunk holds fewer than k
        ++pa;
      } else if (bin == T) {
        if (pc < (unsigned)kLocalCap) cd[pc] = make_uint2(key[u], (unsigned)(sb + u));
        ++pc;
      }
    }
    if (threadIdx.x == 0) ws.ccnt[(size_t)r * nch + c] = make_uint2(tot & 0xFFFFu, tot >> 16);
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    const unsigned prev = atomicAdd(&ws.done[r], 1u);
    s_last = prev == (unsigned)nch - 1;
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  if (nv <= k) {
    write_all_visible(sc, nv, k, out, sout);
    return;
  }
  const bool ok = finalize_query(sc, k, r, nch, T, above, ws, out, sout, S, sh);
  if (threadIdx.x == 0) s_exact = !ok;
  __syncthreads();
  if (s_exact) radix_select_block(sc, nv, k, out, sout, sh);
}

// ------------------------------------------------------------------ host --
bool index_tc_supported(const csa_params& p);
int index_tc_group(const csa_params& p, int Q);
csa_status launch_index_scores_tc(const csa_params& p, int B, int Q, const int32_t* q_pos,
                                  const void* qI, const float* w, const void* kI, int N,
                                  float* scores, int* plan, unsigned* zero_words, size_t nzero,
                                  unsigned* ghist, bool* hist_done, cudaStream_t st);
__global__ void index_plan(const int32_t* q_pos, int G, int ngroups, int m, int N, int* prefix,
                           unsigned* zero_words, size_t nzero);

bool index_fp4_supported(const csa_params& p);
csa_status launch_index_scores_fp4(const csa_params& p, int B, int Q, const int32_t* q_pos,
                                   const void* qI, const float* w, const void* kcodes,
                                   const void* kscales, int N, float* scores, int* plan,
                                   unsigned* ghist, cudaStream_t st);

static bool use_multi_topk(int R, int N, int k) {
  return R <= 64 && N >= 4096 && k <= kAboveCap && (N + kChunk - 1) / kChunk <= kMaxChunks;
}

struct IdxWsLayout {
  size_t scores = 0, plan = 0, ghist = 0, done = 0, ccnt = 0, above = 0, cand = 0, total = 0;
};

static IdxWsLayout idx_ws_layout(const csa_params& p, int B, int Q, int N) {
  IdxWsLayout L;
  const size_t R = (size_t)B * Q;
  size_t off = align_up(R * N * sizeof(float), 256);
  L.plan = off;
  off += align_up((R + 1) * sizeof(int), 256);
  if (use_multi_topk((int)R, N, p.topk)) {
    const size_t nch = (N + kChunk - 1) / kChunk;
    L.ghist = off;  // ghist and done are contiguous (zeroed together)
    off += R * kBins * 4;
    L.done = off;
    off = align_up(off + R * 4, 256);
    L.ccnt = off;
    off += align_up(R * nch * sizeof(uint2), 256);
    L.above = off;
    off += align_up(R * nch * p.topk * sizeof(int), 256);
    L.cand = off;
    off += align_up(R * nch * kLocalCap * sizeof(uint2), 256);
  }
  L.total = off;
  return L;
}

size_t index_topk_ws_bytes(const csa_params& p, int B, int Q, int N) {
  return idx_ws_layout(p, B, Q, N).total;
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
                             cudaStream_t st, const Mxfp4Keys* fp4) {
  const IdxWsLayout L = idx_ws_layout(p, B, Q, N);
  const int R = B * Q;
  char* base = (char*)ws;
  float* scores = (float*)base;
  int* plan = (int*)(base + L.plan);
  const bool multi = use_multi_topk(R, N, p.topk);
  MultiTopkWs mw{};
  size_t nzero = 0;
  if (multi) {
    mw = MultiTopkWs{(unsigned*)(base + L.ghist), (unsigned*)(base + L.done),
                     (uint2*)(base + L.ccnt), (int*)(base + L.above), (uint2*)(base + L.cand)};
    nzero = (L.ccnt - L.ghist) / 4;  // ghist and done
  }
  bool hist_done = false;
  if (fp4 != nullptr) {
    if (!index_fp4_supported(p)) return CSA_ERR_UNSUPPORTED;
    if (multi && cudaMemsetAsync(mw.ghist, 0, nzero * 4, st) != cudaSuccess) return CSA_ERR_CUDA;
    csa_status s = launch_index_scores_fp4(p, B, Q, q_pos, qI, w, fp4->codes, fp4->scales, N,
                                           scores, plan, multi ? mw.ghist : nullptr, st);
    if (s != CSA_OK) return s;
    hist_done = multi && N > 0;
  } else if (index_tc_supported(p)) {
    csa_status s = launch_index_scores_tc(p, B, Q, q_pos, qI, w, kI, N, scores, plan, mw.ghist,
                                          nzero, multi ? mw.ghist : nullptr, &hist_done, st);
    if (s != CSA_OK) return s;
  } else {
    if (multi && cudaMemsetAsync(mw.ghist, 0, nzero * 4, st) != cudaSuccess) return CSA_ERR_CUDA;
    if (p.act == CSA_F32)
      launch_scores<float>(p, B, Q, q_pos, qI, w, kI, N, scores, st);
    else
      launch_scores<__nv_bfloat16>(p, B, Q, q_pos, qI, w, kI, N, scores, st);
  }
  if (multi) {
    dim3 grid(R, (N + kChunk - 1) / kChunk);
    if (!hist_done)
      CSA_LAUNCH(KK_TOPK_HIST, st, topk_hist<<<grid, 1024, 0, st>>>(scores, N, q_pos, p.m, p.topk,
                                                                    mw.ghist));
    const int smem = (int)sizeof(SelectSmem);
    if (!set_kernel_smem((const void*)topk_select_final, smem)) return CSA_ERR_CUDA;
    cudaError_t e = cudaSuccess;
    CSA_LAUNCH(KK_TOPK_SELECT, st,
               e = launch_maybe_pdl(kPdlTopk && hist_done, topk_select_final, grid, dim3(1024),
                                    (size_t)smem, st, (const float*)scores, N, q_pos, p.m,
                                    p.topk, mw, idx_out, score_out));
    if (e != cudaSuccess) return CSA_ERR_CUDA;
  } else {
    const int smem = (int)sizeof(FastTopkSmem);
    if (!set_kernel_smem((const void*)topk_radix, smem)) return CSA_ERR_CUDA;
    CSA_LAUNCH(KK_TOPK, st, topk_radix<<<R, kTopkThreads, smem, st>>>(scores, N, q_pos, p.m,
                                                                      p.topk, idx_out, score_out));
  }
  return last_launch_status();
}

}  // namespace csa
