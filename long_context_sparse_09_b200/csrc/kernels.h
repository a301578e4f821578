// kernels.h -- host-side launchers of the CSA / HCA kernels (internal).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "csa.h"

namespace csa {

// Packed compressor weights: [ncols][d] act dtype (K-major rows, one per GEMM
// output column), then fp32 biases [m][nb] at bias_off, then (bf16 only) at
// dec_off the same weights again as the decode projection streams them: per
// (tile of 64 channels of one part, k-block of 64) one contiguous 16 KB block
// of its 64 C rows and 64 Z rows, already in the 128-byte swizzle of shared
// memory ([dec_tiles][dec_kb][16 KB]).
struct PackLayout {
  int ncols = 0;
  int col_Ca = -1, col_Cb = -1, col_Za = -1, col_Zb = -1;
  int col_CIa = -1, col_CIb = -1, col_ZIa = -1, col_ZIb = -1;
  int nb = 0;
  int b_Ba = -1, b_Bb = -1, b_BIa = -1, b_BIb = -1;
  size_t bias_off = 0;
  size_t dec_off = 0;
  int dec_tiles = 0, dec_kb = 0;
  size_t total = 0;
};
PackLayout pack_layout(const csa_params& p, int d);

csa_status launch_pack(const csa_params& p, int d, const void* const W[8],
                       const float* const Bias[4], void* packed, cudaStream_t st);

size_t compress_ws_bytes(const csa_params& p, int B, int T, int d);
csa_status launch_compress(const csa_params& p, int B, int T, int d,
                           const void* H, const void* packed, void* ckv,
                           float* ckv_scale, void* kI, void* win,
                           float* win_scale, void* ws, cudaStream_t st);

size_t decode_tail_bytes(const csa_params& p, int B, int d);
// grouped output projection (bf16; tensor cores, 16 tokens a pair of launches)
size_t out_proj_packed_bytes(int n_h, int c, int g, int d_g, int d);
size_t out_proj_ws_bytes(int R, int g, int d_g);
csa_status launch_out_proj_pack(int n_h, int c, int g, int d_g, int d, const void* WG,
                                const void* WO, void* packed, cudaStream_t st);
csa_status launch_out_proj(int R, int n_h, int c, int g, int d_g, int d, const void* O,
                           const void* packed, void* out, void* ws, cudaStream_t st);
// query-side projections (bf16; tensor cores, 16 tokens a triple of launches)
size_t query_proj_packed_bytes(const csa_params& p, int d, int d_c);
size_t query_proj_ws_bytes(const csa_params& p, int R);
csa_status launch_query_proj_pack(const csa_params& p, int d, int d_c, const void* WDQ,
                                  const void* Ww, const void* WUQ, const void* WIUQ,
                                  void* packed, cudaStream_t st);
csa_status launch_query_proj(const csa_params& p, int R, int d, int d_c, const void* H,
                             const int32_t* pos, const void* packed, void* cQ, void* q,
                             void* qI, float* w, void* ws, cudaStream_t st);
// decode append, tensor-core projection (bf16, at most 16 tokens a launch)
bool append_tc_supported(const csa_params& p, int nb);
constexpr size_t kDecBlockBytes = 16384;  // one tile-major weight block
csa_status launch_pack_dec_tiles(const csa_params& p, const PackLayout& L, int d, void* packed,
                                 cudaStream_t st);
csa_status launch_append_project_tc(const csa_params& p, const PackLayout& L, int nb, int d,
                                    const void* H, const void* packed, const float* bias,
                                    const int32_t* t, float* state, int cI, size_t per_seq,
                                    cudaStream_t st);
csa_status launch_decode_append(const csa_params& p, int B, int d, const void* H,
                                const int32_t* t, const void* packed, float* tail, void* ckv,
                                float* ckv_scale, int N, void* kI, void* win, float* win_scale,
                                int32_t* win_pos0, int W, cudaStream_t st);

size_t index_topk_ws_bytes(const csa_params& p, int B, int Q, int N);
// indexer keys in MXFP4: E2M1 codes [B*N][c_I/2] and E8M0 scales [B*N][c_I/32]
struct Mxfp4Keys {
  const void* codes;
  const void* scales;
};
// scores from bf16 keys (kI), or from MXFP4 keys (fp4 != null, kI unused)
csa_status launch_index_topk(const csa_params& p, int B, int Q,
                             const int32_t* q_pos, const void* qI,
                             const float* w, const void* kI, int N,
                             int32_t* idx_out, float* score_out, void* ws,
                             cudaStream_t st, const Mxfp4Keys* fp4 = nullptr);
bool index_fp4_supported(const csa_params& p);
csa_status launch_mxfp4_quantize(long long rows, int width, const void* x, void* codes,
                                 void* scales, cudaStream_t st);

size_t attend_ws_bytes(const csa_params& p, int B, int Q, int N, bool dense);
csa_status launch_attend(const csa_params& p, bool dense, int B, int Q,
                         const int32_t* q_pos, const void* q,
                         const int32_t* idx, const void* ckv,
                         const float* ckv_scale, int N, const void* win,
                         const float* win_scale, int W,
                         const int32_t* win_pos0, const float* sink, void* out,
                         void* ws, cudaStream_t st);

}  // namespace csa
