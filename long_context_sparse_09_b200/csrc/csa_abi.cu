// csa_abi.cu -- the extern "C" entry points of include/csa.h: argument
// validation (synchronous, before any launch), workspace sizing, the device
// error word and the launch counter.
#include <atomic>
#include <cstdint>
#include <mutex>
#include <vector>

#include "common.cuh"
#include "kernels.h"

namespace csa {

static std::atomic<uint64_t> g_launches{0};
void count_launch(int n) { g_launches.fetch_add((uint64_t)n, std::memory_order_relaxed); }

__device__ unsigned int g_dev_error;

// ------------------------------------------------------------- profiler --
struct ProfRec {
  int kind;
  cudaEvent_t a, b;
};
static std::mutex g_prof_mu;
static std::atomic<bool> g_prof_on{false};
static std::vector<ProfRec> g_prof_recs;
static std::vector<ProfRec> g_prof_free;

// Events recorded while `st` is being captured into a CUDA graph must be
// external event nodes to be recorded at each replay.
static void prof_record(cudaEvent_t e, cudaStream_t st) {
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(st, &cs) == cudaSuccess && cs == cudaStreamCaptureStatusActive)
    cudaEventRecordWithFlags(e, st, cudaEventRecordExternal);
  else
    cudaEventRecord(e, st);
}

int prof_begin(int kind, cudaStream_t st) {
  if (!g_prof_on.load(std::memory_order_relaxed)) return -1;
  std::lock_guard<std::mutex> lk(g_prof_mu);
  ProfRec r{kind, nullptr, nullptr};
  if (!g_prof_free.empty()) {
    r.a = g_prof_free.back().a;
    r.b = g_prof_free.back().b;
    g_prof_free.pop_back();
  } else if (cudaEventCreate(&r.a) != cudaSuccess || cudaEventCreate(&r.b) != cudaSuccess) {
    return -1;
  }
  prof_record(r.a, st);
  g_prof_recs.push_back(r);
  return (int)g_prof_recs.size() - 1;
}

void prof_end(int slot, cudaStream_t st) {
  if (slot < 0) return;
  std::lock_guard<std::mutex> lk(g_prof_mu);
  if (slot < (int)g_prof_recs.size()) prof_record(g_prof_recs[slot].b, st);
}

static const char* kKindNames[KK_COUNT] = {
    "pack_weights", "compress_gemm", "compress_fold", "compress_window", "index_scores",
    "topk_radix", "attend", "attend_combine", "index_plan", "topk_hist", "topk_select",
    "topk_final", "diag_bounded_wait"};

unsigned int* device_error_word() {
  // cudaGetSymbolAddress is per device; cache one address per device index.
  static unsigned int* addr[64] = {nullptr};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return nullptr;
  if (addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_dev_error) != cudaSuccess) return nullptr;
    addr[dev] = (unsigned int*)p;
  }
  return addr[dev];
}

// ---------------------------------------------------- per-device launch caches
// Kernel attributes and device properties persist for the process, so they
// are set / queried once per (kernel, device) instead of on every call.
namespace {
struct KernelFacts {
  const void* kern;
  int dev, smem, threads;
  int occupancy;  // resident CTAs per SM at (threads, smem); -1: not asked yet
};
std::mutex g_facts_mu;
std::vector<KernelFacts> g_facts;
KernelFacts* find_facts(const void* kern, int dev, int smem, int threads) {
  for (auto& f : g_facts)
    if (f.kern == kern && f.dev == dev && f.smem == smem && f.threads == threads) return &f;
  return nullptr;
}
}  // namespace

int current_device() {
  int dev = 0;
  cudaGetDevice(&dev);
  return dev;
}

int sm_count() {
  static int cnt[64] = {0};
  const int dev = current_device();
  if (dev < 0 || dev >= 64) return 0;
  if (cnt[dev] == 0) cudaDeviceGetAttribute(&cnt[dev], cudaDevAttrMultiProcessorCount, dev);
  return cnt[dev];
}

bool set_kernel_smem(const void* kern, int smem) {
  const int dev = current_device();
  std::lock_guard<std::mutex> lk(g_facts_mu);
  if (find_facts(kern, dev, smem, 0)) return true;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return false;
  g_facts.push_back({kern, dev, smem, 0, -1});
  return true;
}

int kernel_occupancy(const void* kern, int threads, int smem) {
  const int dev = current_device();
  std::lock_guard<std::mutex> lk(g_facts_mu);
  if (KernelFacts* f = find_facts(kern, dev, smem, threads)) return f->occupancy;
  int occ = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, threads, smem) != cudaSuccess)
    occ = 0;
  g_facts.push_back({kern, dev, smem, threads, occ});
  return occ;
}

static bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

static csa_status check_params(const csa_params* p, bool need_indexer) {
  if (p == nullptr) return CSA_ERR_ARG;
  if (p->m <= 0 || p->c <= 0 || p->n_h <= 0 || p->n_win < 0) return CSA_ERR_SHAPE;
  if (p->rope_dims < 0 || p->rope_dims > p->c || (p->rope_dims & 1)) return CSA_ERR_SHAPE;
  if (p->overlap != 0 && p->overlap != 1) return CSA_ERR_ARG;
  if (p->act != CSA_F32 && p->act != CSA_BF16) return CSA_ERR_DTYPE;
  if (p->kv != CSA_F32 && p->kv != CSA_BF16 && p->kv != CSA_KV_FP8MIX) return CSA_ERR_DTYPE;
  if (p->kv == CSA_KV_FP8MIX && ((p->c - p->rope_dims) % 16 != 0 || p->rope_dims % 8 != 0))
    return CSA_ERR_SHAPE;
  if (!(p->rope_base > 0.f) || !(p->rms_eps >= 0.f)) return CSA_ERR_ARG;
  if (need_indexer) {
    if (p->c_I <= 0 || p->n_hI <= 0 || p->topk <= 0) return CSA_ERR_SHAPE;
  }
  return CSA_OK;
}

static cudaStream_t S(csa_stream_t s) { return (cudaStream_t)s; }

}  // namespace csa

using namespace csa;

extern "C" {

int csa_abi_version(void) { return 1; }

void csa_profile_enable(int on) { g_prof_on.store(on != 0); }

int csa_profile_kernel_count(void) { return KK_COUNT; }

const char* csa_profile_kernel_name(int kind) {
  return (kind >= 0 && kind < KK_COUNT) ? kKindNames[kind] : "";
}

csa_status csa_profile_collect(double* total_ms, uint64_t* launches) {
  if (!total_ms || !launches) return CSA_ERR_ARG;
  std::lock_guard<std::mutex> lk(g_prof_mu);
  for (int k = 0; k < KK_COUNT; ++k) {
    total_ms[k] = 0.0;
    launches[k] = 0;
  }
  csa_status st = CSA_OK;
  for (const ProfRec& r : g_prof_recs) {
    float ms = 0.f;
    if (cudaEventSynchronize(r.b) != cudaSuccess || cudaEventElapsedTime(&ms, r.a, r.b) != cudaSuccess)
      st = CSA_ERR_CUDA;
    total_ms[r.kind] += ms;
    launches[r.kind] += 1;
    g_prof_free.push_back(r);
  }
  g_prof_recs.clear();
  return st;
}

uint64_t csa_kernel_launches(void) { return g_launches.load(); }

const char* csa_status_string(csa_status s) {
  switch (s) {
    case CSA_OK: return "ok";
    case CSA_ERR_ARG: return "invalid argument";
    case CSA_ERR_SHAPE: return "invalid or unsupported shape";
    case CSA_ERR_ALIGN: return "pointer not 16-byte aligned";
    case CSA_ERR_DTYPE: return "unsupported dtype";
    case CSA_ERR_CUDA: return "CUDA error";
    case CSA_ERR_TIMEOUT: return "device wait timed out";
    case CSA_ERR_UNSUPPORTED: return "unsupported by this build";
    case CSA_ERR_WORKSPACE: return "workspace too small";
  }
  return "unknown status";
}

csa_status csa_device_status(csa_stream_t stream, uint32_t* flags) {
  if (flags == nullptr) return CSA_ERR_ARG;
  unsigned int* w = device_error_word();
  if (w == nullptr) return CSA_ERR_CUDA;
  unsigned int v = 0;
  if (cudaMemcpyAsync(&v, w, sizeof v, cudaMemcpyDeviceToHost, S(stream)) != cudaSuccess)
    return CSA_ERR_CUDA;
  if (cudaMemsetAsync(w, 0, sizeof v, S(stream)) != cudaSuccess) return CSA_ERR_CUDA;
  if (cudaStreamSynchronize(S(stream)) != cudaSuccess) return CSA_ERR_CUDA;
  *flags = v;
  return CSA_OK;
}

// ------------------------------------------------------------------ pack --
size_t csa_packed_weight_bytes(const csa_params* p, int d) {
  if (check_params(p, p && p->overlap == 1) != CSA_OK || d <= 0) return 0;
  return pack_layout(*p, d).total;
}

csa_status csa_pack_weights(const csa_params* p, int d, const void* Wkv_a,
                            const void* Wkv_b, const void* Wz_a, const void* Wz_b,
                            const void* WIkv_a, const void* WIkv_b,
                            const void* WIz_a, const void* WIz_b, const float* B_a,
                            const float* B_b, const float* BI_a, const float* BI_b,
                            void* packed, csa_stream_t stream) {
  csa_status st = check_params(p, p && p->overlap == 1);
  if (st != CSA_OK) return st;
  if (d <= 0) return CSA_ERR_SHAPE;
  if (!Wkv_a || !Wz_a || !B_a || !packed) return CSA_ERR_ARG;
  if (p->overlap) {
    if (!Wkv_b || !Wz_b || !B_b || !WIkv_a || !WIkv_b || !WIz_a || !WIz_b || !BI_a || !BI_b)
      return CSA_ERR_ARG;
  } else if (Wkv_b || Wz_b || B_b || WIkv_a || WIkv_b || WIz_a || WIz_b || BI_a || BI_b) {
    return CSA_ERR_ARG;
  }
  if (!aligned16(packed)) return CSA_ERR_ALIGN;
  const void* W[8] = {Wkv_a, Wkv_b, Wz_a, Wz_b, WIkv_a, WIkv_b, WIz_a, WIz_b};
  const float* Bs[4] = {B_a, B_b, BI_a, BI_b};
  return launch_pack(*p, d, W, Bs, packed, S(stream));
}

// ------------------------------------------- grouped output projection --
static csa_status check_out_proj(int n_h, int c, int g, int d_g, int d) {
  if (n_h <= 0 || c <= 0 || g <= 0 || d_g <= 0 || d <= 0) return CSA_ERR_SHAPE;
  if (n_h % g != 0) return CSA_ERR_SHAPE;
  if ((c * (n_h / g)) % 64 != 0 || d_g % 128 != 0) return CSA_ERR_SHAPE;
  return CSA_OK;
}

size_t csa_out_proj_packed_bytes(int n_h, int c, int g, int d_g, int d) {
  if (check_out_proj(n_h, c, g, d_g, d) != CSA_OK) return 0;
  return out_proj_packed_bytes(n_h, c, g, d_g, d);
}

csa_status csa_out_proj_pack(int n_h, int c, int g, int d_g, int d, const void* WG,
                             const void* WO, void* packed, csa_stream_t stream) {
  csa_status st = check_out_proj(n_h, c, g, d_g, d);
  if (st != CSA_OK) return st;
  if (!WG || !WO || !packed) return CSA_ERR_ARG;
  if (!aligned16(packed)) return CSA_ERR_ALIGN;
  return launch_out_proj_pack(n_h, c, g, d_g, d, WG, WO, packed, S(stream));
}

size_t csa_out_proj_workspace_bytes(int R, int n_h, int c, int g, int d_g, int d) {
  if (R <= 0 || check_out_proj(n_h, c, g, d_g, d) != CSA_OK) return 0;
  return out_proj_ws_bytes(R, g, d_g);
}

csa_status csa_out_proj(int R, int n_h, int c, int g, int d_g, int d, const void* O,
                        const void* packed, void* out, void* workspace, size_t ws_bytes,
                        csa_stream_t stream) {
  csa_status st = check_out_proj(n_h, c, g, d_g, d);
  if (st != CSA_OK) return st;
  if (R <= 0) return CSA_ERR_SHAPE;
  if (!O || !packed || !out) return CSA_ERR_ARG;
  if (!aligned16(O) || !aligned16(packed) || !aligned16(out)) return CSA_ERR_ALIGN;
  if (workspace == nullptr || ws_bytes < out_proj_ws_bytes(R, g, d_g)) return CSA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return CSA_ERR_ALIGN;
  return launch_out_proj(R, n_h, c, g, d_g, d, O, packed, out, workspace, S(stream));
}

// ------------------------------------------------- query-side projections --
static csa_status check_query_proj(const csa_params* p, int d, int d_c) {
  csa_status st = check_params(p, true);
  if (st != CSA_OK) return st;
  if (d <= 0 || d_c <= 0) return CSA_ERR_SHAPE;
  if (p->act != CSA_BF16) return CSA_ERR_UNSUPPORTED;
  if (d % 64 != 0 || d_c % 64 != 0 || p->c % 4 != 0) return CSA_ERR_SHAPE;
  return CSA_OK;
}

size_t csa_query_proj_packed_bytes(const csa_params* p, int d, int d_c) {
  if (check_query_proj(p, d, d_c) != CSA_OK) return 0;
  return query_proj_packed_bytes(*p, d, d_c);
}

csa_status csa_query_proj_pack(const csa_params* p, int d, int d_c, const void* WDQ,
                               const void* Ww, const void* WUQ, const void* WIUQ, void* packed,
                               csa_stream_t stream) {
  csa_status st = check_query_proj(p, d, d_c);
  if (st != CSA_OK) return st;
  if (!WDQ || !Ww || !WUQ || !WIUQ || !packed) return CSA_ERR_ARG;
  if (!aligned16(packed)) return CSA_ERR_ALIGN;
  return launch_query_proj_pack(*p, d, d_c, WDQ, Ww, WUQ, WIUQ, packed, S(stream));
}

size_t csa_query_proj_workspace_bytes(const csa_params* p, int R, int d, int d_c) {
  if (R <= 0 || check_query_proj(p, d, d_c) != CSA_OK) return 0;
  return query_proj_ws_bytes(*p, R);
}

csa_status csa_query_proj(const csa_params* p, int R, int d, int d_c, const void* H,
                          const int32_t* pos, const void* packed, void* cQ, void* q, void* qI,
                          float* w, void* workspace, size_t ws_bytes, csa_stream_t stream) {
  csa_status st = check_query_proj(p, d, d_c);
  if (st != CSA_OK) return st;
  if (R <= 0) return CSA_ERR_SHAPE;
  if (!H || !pos || !packed || !cQ || !q || !qI || !w) return CSA_ERR_ARG;
  if (!aligned16(H) || !aligned16(packed) || !aligned16(cQ) || !aligned16(q) ||
      !aligned16(qI) || !aligned16(w))
    return CSA_ERR_ALIGN;
  if (workspace == nullptr || ws_bytes < query_proj_ws_bytes(*p, R)) return CSA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return CSA_ERR_ALIGN;
  return launch_query_proj(*p, R, d, d_c, H, pos, packed, cQ, q, qI, w, workspace, S(stream));
}

// -------------------------------------------------------------- compress --
size_t csa_compress_workspace_bytes(const csa_params* p, int B, int T, int d) {
  if (check_params(p, p && p->overlap == 1) != CSA_OK || B <= 0 || T <= 0 || d <= 0) return 0;
  return compress_ws_bytes(*p, B, T, d);
}

static csa_status compress_common(const csa_params* p, bool csa_variant, int B, int T,
                                  int d, const void* H, const void* packed, void* ckv,
                                  float* ckv_scale, void* kI, void* win, float* win_scale,
                                  void* workspace, size_t ws_bytes, csa_stream_t stream) {
  csa_status st = check_params(p, csa_variant);
  if (st != CSA_OK) return st;
  if ((p->overlap == 1) != csa_variant) return CSA_ERR_ARG;
  if (B <= 0 || T <= 0 || d <= 0) return CSA_ERR_SHAPE;
  if (!H || !packed) return CSA_ERR_ARG;
  const int nE = T / p->m;
  if (nE > 0 && !ckv) return CSA_ERR_ARG;
  if (csa_variant && nE > 0 && !kI) return CSA_ERR_ARG;
  if (!csa_variant && kI) return CSA_ERR_ARG;
  const bool fp8 = p->kv == CSA_KV_FP8MIX;
  if (fp8 && nE > 0 && !ckv_scale) return CSA_ERR_ARG;
  if (fp8 && win && !win_scale) return CSA_ERR_ARG;
  if (!fp8 && (ckv_scale || win_scale)) return CSA_ERR_ARG;
  if (!aligned16(H) || !aligned16(packed) || (ckv && !aligned16(ckv)) || (win && !aligned16(win)))
    return CSA_ERR_ALIGN;
  const size_t need = compress_ws_bytes(*p, B, T, d);
  if (need > 0 && (workspace == nullptr || ws_bytes < need)) return CSA_ERR_WORKSPACE;
  return launch_compress(*p, B, T, d, H, packed, ckv, ckv_scale, kI, win, win_scale,
                         workspace, S(stream));
}

size_t csa_decode_tail_bytes(const csa_params* p, int B, int d) {
  if (check_params(p, p && p->overlap == 1) != CSA_OK || B <= 0 || d <= 0) return 0;
  return decode_tail_bytes(*p, B, d);
}

static csa_status append_common(const csa_params* p, bool csa_variant, int B, int d,
                                const void* H, const int32_t* t, const void* packed,
                                float* tail, void* ckv, float* ckv_scale, int N, void* kI,
                                void* win, float* win_scale, int32_t* win_pos0, int W,
                                csa_stream_t stream) {
  csa_status st = check_params(p, csa_variant);
  if (st != CSA_OK) return st;
  if ((p->overlap == 1) != csa_variant) return CSA_ERR_ARG;
  if (B <= 0 || d <= 0 || N < 0 || W < 0) return CSA_ERR_SHAPE;
  if (d % (p->act == CSA_F32 ? 4 : 8) != 0) return CSA_ERR_SHAPE;
  if (!H || !t || !packed || !tail || !ckv) return CSA_ERR_ARG;
  if (csa_variant != (kI != nullptr)) return CSA_ERR_ARG;
  const bool fp8 = p->kv == CSA_KV_FP8MIX;
  if (fp8 && !ckv_scale) return CSA_ERR_ARG;
  if (win && (!win_pos0 || (fp8 && !win_scale))) return CSA_ERR_ARG;
  if (!fp8 && (ckv_scale || win_scale)) return CSA_ERR_ARG;
  if (!aligned16(H) || !aligned16(packed) || !aligned16(tail)) return CSA_ERR_ALIGN;
  return launch_decode_append(*p, B, d, H, t, packed, tail, ckv, ckv_scale, N, kI, win,
                              win_scale, win_pos0, W, S(stream));
}

csa_status csa_decode_append(const csa_params* p, int B, int d, const void* H,
                             const int32_t* t, const void* packed, float* tail, void* ckv,
                             float* ckv_scale, int N, void* kI, void* win, float* win_scale,
                             int32_t* win_pos0, int W, csa_stream_t stream) {
  return append_common(p, true, B, d, H, t, packed, tail, ckv, ckv_scale, N, kI, win,
                       win_scale, win_pos0, W, stream);
}

csa_status hca_decode_append(const csa_params* p, int B, int d, const void* H,
                             const int32_t* t, const void* packed, float* tail, void* ckv,
                             float* ckv_scale, int N, void* win, float* win_scale,
                             int32_t* win_pos0, int W, csa_stream_t stream) {
  return append_common(p, false, B, d, H, t, packed, tail, ckv, ckv_scale, N, nullptr, win,
                       win_scale, win_pos0, W, stream);
}

csa_status csa_compress(const csa_params* p, int B, int T, int d, const void* H,
                        const void* packed, void* ckv, float* ckv_scale, void* kI,
                        void* win, float* win_scale, void* workspace, size_t ws_bytes,
                        csa_stream_t stream) {
  return compress_common(p, true, B, T, d, H, packed, ckv, ckv_scale, kI, win, win_scale,
                         workspace, ws_bytes, stream);
}

csa_status hca_compress(const csa_params* p, int B, int T, int d, const void* H,
                        const void* packed, void* ckv, float* ckv_scale, void* win,
                        float* win_scale, void* workspace, size_t ws_bytes,
                        csa_stream_t stream) {
  return compress_common(p, false, B, T, d, H, packed, ckv, ckv_scale, nullptr, win,
                         win_scale, workspace, ws_bytes, stream);
}

// ---------------------------------------------------------- index / top-k --
size_t csa_index_topk_workspace_bytes(const csa_params* p, int B, int Q, int N) {
  if (check_params(p, true) != CSA_OK || B <= 0 || Q <= 0 || N < 0) return 0;
  return index_topk_ws_bytes(*p, B, Q, N);
}

csa_status csa_index_topk(const csa_params* p, int B, int Q, const int32_t* q_pos,
                          const void* qI, const float* w, const void* kI, int N,
                          int32_t* idx_out, float* score_out, void* workspace,
                          size_t ws_bytes, csa_stream_t stream) {
  csa_status st = check_params(p, true);
  if (st != CSA_OK) return st;
  if (B <= 0 || Q <= 0 || N < 0) return CSA_ERR_SHAPE;
  if (p->c_I % 8 != 0 || p->n_hI > 64) return CSA_ERR_UNSUPPORTED;
  if (!q_pos || !qI || !w || !idx_out || (N > 0 && !kI)) return CSA_ERR_ARG;
  if (!aligned16(qI) || (kI && !aligned16(kI)) || !aligned16(w)) return CSA_ERR_ALIGN;
  const size_t need = index_topk_ws_bytes(*p, B, Q, N);
  if (need > 0 && (workspace == nullptr || ws_bytes < need)) return CSA_ERR_WORKSPACE;
  return launch_index_topk(*p, B, Q, q_pos, qI, w, kI, N, idx_out, score_out, workspace,
                           S(stream));
}

// ------------------------------------------------------ MXFP4 indexer --
csa_status csa_mxfp4_quantize(int rows, int width, const void* x, void* codes, void* scales,
                              csa_stream_t stream) {
  if (rows < 0 || width <= 0 || width % 32 != 0) return CSA_ERR_SHAPE;
  if (rows == 0) return CSA_OK;
  if (!x || !codes || !scales) return CSA_ERR_ARG;
  if (!aligned16(x) || !aligned16(codes)) return CSA_ERR_ALIGN;
  return launch_mxfp4_quantize(rows, width, x, codes, scales, S(stream));
}

csa_status csa_index_topk_mxfp4(const csa_params* p, int B, int Q, const int32_t* q_pos,
                                const void* qI, const float* w, const void* kI_codes,
                                const void* kI_scales, int N, int32_t* idx_out,
                                float* score_out, void* workspace, size_t ws_bytes,
                                csa_stream_t stream) {
  csa_status st = check_params(p, true);
  if (st != CSA_OK) return st;
  if (B <= 0 || Q <= 0 || N < 0) return CSA_ERR_SHAPE;
  if (!index_fp4_supported(*p)) return CSA_ERR_UNSUPPORTED;
  if (!q_pos || !qI || !w || !idx_out || (N > 0 && (!kI_codes || !kI_scales))) return CSA_ERR_ARG;
  if (!aligned16(qI) || !aligned16(w) || (kI_codes && !aligned16(kI_codes)) ||
      (kI_scales && ((uintptr_t)kI_scales & 3u)))
    return CSA_ERR_ALIGN;
  const size_t need = index_topk_ws_bytes(*p, B, Q, N);
  if (need > 0 && (workspace == nullptr || ws_bytes < need)) return CSA_ERR_WORKSPACE;
  const Mxfp4Keys keys{kI_codes, kI_scales};
  return launch_index_topk(*p, B, Q, q_pos, qI, w, nullptr, N, idx_out, score_out, workspace,
                           S(stream), &keys);
}

// ---------------------------------------------------------------- attend --
size_t csa_attend_workspace_bytes(const csa_params* p, int B, int Q, int N) {
  if (check_params(p, false) != CSA_OK || B <= 0 || Q <= 0 || N < 0) return 0;
  return attend_ws_bytes(*p, B, Q, N, p->overlap == 0);
}

static csa_status attend_common(const csa_params* p, bool dense, int B, int Q,
                                const int32_t* q_pos, const void* q, const int32_t* idx,
                                const void* ckv, const float* ckv_scale, int N,
                                const void* win, const float* win_scale, int W,
                                const int32_t* win_pos0, const float* sink, void* out,
                                void* workspace, size_t ws_bytes, csa_stream_t stream) {
  csa_status st = check_params(p, false);
  if (st != CSA_OK) return st;
  if (B <= 0 || Q <= 0 || N < 0 || W < 0) return CSA_ERR_SHAPE;
  if (!dense && p->topk <= 0) return CSA_ERR_SHAPE;
  if (p->n_h % 2 != 0 || (p->n_h > 16 && p->n_h % 16 != 0)) return CSA_ERR_UNSUPPORTED;
  if (p->c != 64 && p->c != 128 && p->c != 256 && p->c != 512) return CSA_ERR_UNSUPPORTED;
  if (!q_pos || !q || !sink || !out) return CSA_ERR_ARG;
  if (!dense && !idx) return CSA_ERR_ARG;
  if (N > 0 && !ckv) return CSA_ERR_ARG;
  if (p->n_win > 0 && (!win || !win_pos0 || W <= 0)) return CSA_ERR_ARG;
  const bool fp8 = p->kv == CSA_KV_FP8MIX;
  if (fp8 && ((N > 0 && !ckv_scale) || (p->n_win > 0 && !win_scale))) return CSA_ERR_ARG;
  if (!aligned16(q) || (ckv && !aligned16(ckv)) || (win && !aligned16(win)) || !aligned16(out))
    return CSA_ERR_ALIGN;
  const size_t need = attend_ws_bytes(*p, B, Q, N, dense);
  if (need > 0 && (workspace == nullptr || ws_bytes < need)) return CSA_ERR_WORKSPACE;
  if (device_error_word() == nullptr) return CSA_ERR_CUDA;
  return launch_attend(*p, dense, B, Q, q_pos, q, idx, ckv, ckv_scale, N, win, win_scale, W,
                       win_pos0, sink, out, workspace, S(stream));
}

csa_status csa_attend(const csa_params* p, int B, int Q, const int32_t* q_pos,
                      const void* q, const int32_t* idx, const void* ckv,
                      const float* ckv_scale, int N, const void* win,
                      const float* win_scale, int W, const int32_t* win_pos0,
                      const float* sink, void* out, void* workspace, size_t ws_bytes,
                      csa_stream_t stream) {
  if (p && p->overlap != 1) return CSA_ERR_ARG;
  return attend_common(p, false, B, Q, q_pos, q, idx, ckv, ckv_scale, N, win, win_scale, W,
                       win_pos0, sink, out, workspace, ws_bytes, stream);
}

csa_status hca_attend(const csa_params* p, int B, int Q, const int32_t* q_pos,
                      const void* q, const void* ckv, const float* ckv_scale, int N,
                      const void* win, const float* win_scale, int W,
                      const int32_t* win_pos0, const float* sink, void* out,
                      void* workspace, size_t ws_bytes, csa_stream_t stream) {
  if (p && p->overlap != 0) return CSA_ERR_ARG;
  return attend_common(p, true, B, Q, q_pos, q, nullptr, ckv, ckv_scale, N, win, win_scale,
                       W, win_pos0, sink, out, workspace, ws_bytes, stream);
}

}  // extern "C"
