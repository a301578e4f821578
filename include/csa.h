/*
 * csa.h -- C ABI of the B200 (sm_100a) CSA / HCA forward pass.
 *
 * The operations are those of DeepSeek-V4's Compressed Sparse Attention and
 * Heavily Compressed Attention as described in "DeepSeekV4技术报告阅读笔记"
 * (zouxinn.github.io; cited below as [N] with its section / equation numbers)
 * and "02 · DeepSeek-V4: 压缩注意力撑起 1M 上下文" (PaperTrace; cited as [P]):
 * compression (prefill, and one token at a time for decode), indexer scores
 * and top-k, the shared-KV attention with window and sink, and the grouped
 * output projection that follows it.
 *
 * Conventions for every call
 *   - All tensor arguments are DEVICE pointers to caller-owned memory, laid
 *     out row-major with the last dimension contiguous, as stated per
 *     argument.  The library allocates nothing and keeps no device state
 *     besides one error word per GPU (and the fixed scratch array of
 *     csa_index_topk_noalloc).
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *     stream) and runs asynchronously; outputs are valid once the stream has
 *     reached the call.
 *   - Argument errors are reported synchronously by the return value before
 *     anything is launched.  Errors found on the device (an index or window
 *     row out of range, a bounded wait that ran out) set bits in the device
 *     error word, which
 *     csa_device_status() reads; the offending element is skipped, never
 *     dereferenced.
 *   - Queries are numbered r = b*Q + j for sequence b < B and query j < Q.
 *     Positions are 0-based token positions within the sequence.
 *   - A compressed entry s covers tokens m*s .. m*s+m-1 (its a-window) and is
 *     visible to a query at position t0 iff s < floor((t0+1)/m) ([N] 2.3.2,
 *     read as "only complete blocks").
 *   - KV formats: CSA_F32 / CSA_BF16 rows of c values; CSA_KV_FP8MIX rows of
 *     (c - rope_dims) OCP E4M3 codes followed by rope_dims bf16 values
 *     ((c - rope_dims) + 2*rope_dims bytes per row) plus one fp32 scale per
 *     row in a separate plane: value_j = e4m3(code_j) * scale ([P] 2.5: RoPE
 *     dims in BF16, the rest in FP8).
 */
#ifndef CSA_H
#define CSA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* csa_stream_t; /* same type as cudaStream_t */

typedef enum {
  CSA_OK = 0,
  CSA_ERR_ARG = 1,         /* null pointer or bad scalar argument */
  CSA_ERR_SHAPE = 2,       /* inconsistent or unsupported sizes */
  CSA_ERR_ALIGN = 3,       /* pointer not 16-byte aligned */
  CSA_ERR_DTYPE = 4,       /* unsupported dtype / KV format combination */
  CSA_ERR_CUDA = 5,        /* a CUDA launch or query failed */
  CSA_ERR_TIMEOUT = 6,     /* a bounded device-side wait ran out */
  CSA_ERR_UNSUPPORTED = 7, /* valid request this build does not implement */
  CSA_ERR_WORKSPACE = 8    /* workspace missing or smaller than required */
} csa_status;

typedef enum { CSA_F32 = 0, CSA_BF16 = 1, CSA_KV_FP8MIX = 2 } csa_dtype;

/* Device error-word bits (csa_device_status). */
#define CSA_DEV_BAD_INDEX 0x1u  /* a top-k index >= the visible entries */
#define CSA_DEV_BAD_WINDOW 0x2u /* a window token outside the window rows */
#define CSA_DEV_TIMEOUT 0x4u    /* a bounded wait gave up */
#define CSA_DEV_RANGE 0x8u      /* an MXFP4 block exponent outside [-23, 13] (the
                                   MXFP4 indexer's exact range); that block was
                                   scored with its exponent clamped */

typedef struct {
  int m;          /* tokens per compressed entry (CSA m, HCA m') */
  int overlap;    /* 1: CSA two-window compressor [N] eq. 11-12;
                     0: HCA single window [N] eq. 22-23 */
  int c;          /* entry width (key = value width) */
  int rope_dims;  /* RoPE on the last rope_dims of c (even, <= c) */
  int c_I;        /* indexer key width (CSA only) */
  int n_hI;       /* indexer heads (CSA only) */
  int n_h;        /* query heads sharing the one KV head */
  int topk;       /* entries selected per query (CSA only) */
  int n_win;      /* sliding-window tokens, >= 0 */
  float rope_base;     /* RoPE base: pair p turns by pos * base^(-2p/rope_dims) */
  float rms_eps;       /* RMSNorm eps (unit gain) */
  float softmax_scale; /* logit scale of q.k (the sink logit is not scaled) */
  int act;        /* csa_dtype of H, weights, q, q^I: CSA_F32 or CSA_BF16 */
  int kv;         /* csa_dtype of the entry / window caches */
} csa_params;

/* ---------------------------------------------------------------------------
 * Compressor weights.  [N] eq. 9-10 (CSA: W^{aKV}, W^{bKV}, W^{aZ}, W^{bZ}
 * in R^{d x c}, and the same four at width c_I for the indexer keys, [N]
 * 2.3.2 / [P] 2.2) and eq. 20-21 (HCA: W^{KV}, W^Z); position biases
 * B^a, B^b in R^{m x c} ([N] eq. 11; the page prints "m x b", read as m x c).
 *
 * csa_pack_weights copies the caller's matrices (act dtype, [d][width] each,
 * as in C = H W) and fp32 biases ([m][width]) into one packed buffer of
 * csa_packed_weight_bytes() bytes, in the layout csa_compress reads.  For
 * HCA (overlap = 0) pass the single branch as *_a and NULL for every *_b and
 * indexer argument.  The packed buffer is caller-owned and may be reused for
 * any number of csa_compress calls with the same params and d.
 * ------------------------------------------------------------------------- */
size_t csa_packed_weight_bytes(const csa_params* p, int d);
csa_status csa_pack_weights(const csa_params* p, int d,
                            const void* Wkv_a, const void* Wkv_b,
                            const void* Wz_a, const void* Wz_b,
                            const void* WIkv_a, const void* WIkv_b,
                            const void* WIz_a, const void* WIz_b,
                            const float* B_a, const float* B_b,
                            const float* BI_a, const float* BI_b,
                            void* packed, csa_stream_t stream);

/* ---------------------------------------------------------------------------
 * csa_compress: overlapped two-window compression of B sequences of T tokens
 * ([N] eq. 9-12, [P] 2.1), followed by RMSNorm (unit gain, [N] 2.5.1) and
 * RoPE at position m*i on the last rope_dims ([N] 2.5.2; the entry position
 * is read as the first token of its a-window) of each entry i.
 *   H        [B][T][d]            act dtype
 *   packed   from csa_pack_weights
 *   ckv      [B][T/m][row]        kv format: compressed entries (T/m = floor)
 *   ckv_scale[B][T/m] fp32        CSA_KV_FP8MIX only, else NULL
 *   kI       [B][T/m][c_I]        act dtype: indexer keys (same compressor
 *                                 at width c_I, no norm, no RoPE)
 *   win      [B][T][row]          kv format: per-token window rows, RMSNorm +
 *                                 RoPE(position j) of C^a_j = h_j W^{aKV}
 *                                 (the uncompressed KV of the window branch,
 *                                 [N] 2.5.3); NULL to skip
 *   win_scale[B][T] fp32          CSA_KV_FP8MIX with win != NULL, else NULL
 *   workspace / ws_bytes          >= csa_compress_workspace_bytes()
 * hca_compress is the same with overlap = 0 ([N] eq. 20-23, [P] 2.3) and no
 * indexer keys (kI must be NULL); its window rows use C_j = h_j W^{KV}.
 * ------------------------------------------------------------------------- */
size_t csa_compress_workspace_bytes(const csa_params* p, int B, int T, int d);
csa_status csa_compress(const csa_params* p, int B, int T, int d,
                        const void* H, const void* packed,
                        void* ckv, float* ckv_scale, void* kI,
                        void* win, float* win_scale,
                        void* workspace, size_t ws_bytes, csa_stream_t stream);
csa_status hca_compress(const csa_params* p, int B, int T, int d,
                        const void* H, const void* packed,
                        void* ckv, float* ckv_scale,
                        void* win, float* win_scale,
                        void* workspace, size_t ws_bytes, csa_stream_t stream);

/* ---------------------------------------------------------------------------
 * csa_decode_append: the compressor one token at a time (decode; the same
 * arithmetic as csa_compress, [N] eq. 9-12, 2.5.1-2.5.3, up to the order of
 * the softmax sums).  For each sequence b the new token h_b at position t[b]
 * (tokens 0..t[b]-1 appended before) is projected with the packed weights and
 * folded into the running softmax of the entries it belongs to (entry
 * t[b] / m, and entry t[b] / m + 1 through its b window): per channel the
 * largest logit so far, the sum of exp(logit - largest) and the weighted sum
 * of C, rescaled when a larger logit arrives.  When t[b] closes block
 * i = t[b] / m (t[b] % m == m-1) entry i is num / den per channel, normalised,
 * rotated at m*i and stored as ckv[b][i] and kI[b][i]; the window row of the
 * token (RMSNorm + RoPE(t[b]) of C^a_t) is stored as win[b][t[b]-win_pos0[b]].
 *   H        [B][d]               act dtype, d a multiple of 8 (bf16) or 4
 *   t        [B] int32            positions of the new tokens
 *   packed   from csa_pack_weights (same d)
 *   tail     csa_decode_tail_bytes(p, B, d) bytes, fp32: caller-owned state
 *            between calls, per sequence c floats (C^a of the last token)
 *            then 2 slots (1 for HCA) of 3 x (c + c_I) floats (c for HCA);
 *            entry i uses slot i % 2.  It needs no initialisation: a slot is
 *            restarted by the first token that reaches its entry.
 *   ckv      [B][N][row], ckv_scale [B][N] (CSA_KV_FP8MIX, else NULL)
 *   kI       [B][N][c_I]          act dtype
 *   win      [B][W][row], win_scale [B][W] (CSA_KV_FP8MIX, else NULL),
 *            win_pos0 [B] int32   position of window row 0 (device; read and
 *                                 updated); NULL win skips the window row
 * The window rolls: when token t[b] would land on row W (the rows are full)
 * and W >= 2 (n_win - 1), rows W-n_win+1..W-1 move to rows 0..n_win-2,
 * win_pos0[b] becomes t[b] - (n_win - 1) and the token's row is n_win - 1.
 * So W = 2 n_win rows per sequence hold the window for any length, and the
 * attention calls read the same win / win_pos0.
 * An entry index >= N or a window row outside [0, W) that cannot be rolled
 * is skipped and raises CSA_DEV_BAD_INDEX / CSA_DEV_BAD_WINDOW in the device
 * error word.
 * hca_decode_append is the same with overlap = 0 ([N] eq. 20-23, one open
 * entry) and no indexer keys.
 * ------------------------------------------------------------------------- */
size_t csa_decode_tail_bytes(const csa_params* p, int B, int d);
csa_status csa_decode_append(const csa_params* p, int B, int d, const void* H,
                             const int32_t* t, const void* packed, float* tail,
                             void* ckv, float* ckv_scale, int N, void* kI,
                             void* win, float* win_scale, int32_t* win_pos0,
                             int W, csa_stream_t stream);
csa_status hca_decode_append(const csa_params* p, int B, int d, const void* H,
                             const int32_t* t, const void* packed, float* tail,
                             void* ckv, float* ckv_scale, int N,
                             void* win, float* win_scale, int32_t* win_pos0,
                             int W, csa_stream_t stream);

/* ---------------------------------------------------------------------------
 * csa_out_proj: the grouped output projection that follows the attention
 * ([N] 2.3.3 "Grouped Output Projection"; [P] 2.2).  The n_h head outputs
 * of a token (csa_attend's out row, [n_h][c]) are cut into g groups of n_h/g
 * consecutive heads; group i (c n_h/g values) times W^G_i gives d_g values
 * (stored as bf16: Y); the g d_g values times W^O give the d outputs.
 * bf16 only; 16 tokens per pair of tensor-core launches (weights streamed
 * once per 16 tokens: the decode form).
 *   WG  [g][c n_h/g][d_g] bf16, WO [g d_g][d] bf16 (row-major, x W form)
 *   packed  csa_out_proj_packed_bytes(...) bytes from csa_out_proj_pack
 *           (W^G and W^O transposed to K-major rows)
 *   O   [R][n_h][c] bf16    out [R][d] bf16
 *   workspace  csa_out_proj_workspace_bytes(...) bytes (Y, [R][g d_g] bf16)
 * Shapes: n_h % g == 0, (c n_h / g) % 64 == 0, d_g % 128 == 0; otherwise
 * CSA_ERR_SHAPE (and 0 from the size queries).  Pointers 16-byte aligned.
 * ------------------------------------------------------------------------- */
size_t csa_out_proj_packed_bytes(int n_h, int c, int g, int d_g, int d);
csa_status csa_out_proj_pack(int n_h, int c, int g, int d_g, int d, const void* WG,
                             const void* WO, void* packed, csa_stream_t stream);
size_t csa_out_proj_workspace_bytes(int R, int n_h, int c, int g, int d_g, int d);
csa_status csa_out_proj(int R, int n_h, int c, int g, int d_g, int d, const void* O,
                        const void* packed, void* out, void* workspace, size_t ws_bytes,
                        csa_stream_t stream);

/* ---------------------------------------------------------------------------
 * csa_query_proj: the query side of the layer for R tokens ([N] eq. 13-15
 * and 18, 2.5.1-2.5.2), the projections that feed csa_index_topk and
 * csa_attend:
 *   c^Q = h W^{DQ}                 (eq. 13, d -> d_c; the low-rank latent,
 *                                   stored bf16 and read back as bf16)
 *   w   = h W^w                    (eq. 15, n_hI fp32 head weights)
 *   q^I = c^Q W^{IUQ}              (eq. 14, n_hI heads of c_I; no norm, no
 *                                   RoPE, like the indexer keys)
 *   q   = RoPE_t(RMSNorm(c^Q W^{UQ})) per head (eq. 18; unit-gain RMSNorm
 *                                   over each head's c values, RoPE at the
 *                                   token's position t on the last
 *                                   rope_dims, interleaved pairs)
 * bf16 only (tensor cores; CSA_ERR_UNSUPPORTED otherwise); 16 tokens a
 * triple of launches (weights streamed once per 16 tokens: the decode form).
 *   WDQ [d][d_c], Ww [d][n_hI], WUQ [d_c][n_h c], WIUQ [d_c][n_hI c_I] bf16
 *       (row-major, x W form) -> packed, csa_query_proj_packed_bytes() bytes
 *       from csa_query_proj_pack (K-major rows, zero-padded)
 *   H   [R][d] bf16, pos [R] int32 token positions
 *   cQ  [R][d_c] bf16, q [R][n_h][c] bf16, qI [R][n_hI][c_I] bf16,
 *   w   [R][n_hI] fp32            outputs (caller-owned)
 *   workspace  csa_query_proj_workspace_bytes() bytes (q before its norm,
 *              fp32)
 * Shapes: d % 64 == 0, d_c % 64 == 0, c % 4 == 0; pointers 16-byte
 * aligned.  Argument errors as for every call.
 * ------------------------------------------------------------------------- */
size_t csa_query_proj_packed_bytes(const csa_params* p, int d, int d_c);
csa_status csa_query_proj_pack(const csa_params* p, int d, int d_c, const void* WDQ,
                               const void* Ww, const void* WUQ, const void* WIUQ,
                               void* packed, csa_stream_t stream);
size_t csa_query_proj_workspace_bytes(const csa_params* p, int R, int d, int d_c);
csa_status csa_query_proj(const csa_params* p, int R, int d, int d_c, const void* H,
                          const int32_t* pos, const void* packed, void* cQ, void* q,
                          void* qI, float* w, void* workspace, size_t ws_bytes,
                          csa_stream_t stream);

/* ---------------------------------------------------------------------------
 * csa_index_topk: Lightning-Indexer scores and top-k selection ([N] eq. 16-17,
 * [P] 2.2):  I[r][s] = sum_h w[r][h] * ReLU(qI[r][h] . kI[b][s])  for every
 * visible s, then the topk largest.  Ties are broken towards the lower index.
 *   q_pos    [B*Q] int32          query positions t0
 *   qI       [B*Q][n_hI][c_I]     act dtype
 *   w        [B*Q][n_hI] fp32     head weights
 *   kI       [B][N][c_I]          act dtype: indexer-key cache
 *   idx_out  [B*Q][topk] int32    selected entries in ascending order, -1
 *                                 padded when fewer than topk are visible
 *   score_out[B*Q][topk] fp32     score of each selected entry (nullable)
 *   workspace / ws_bytes          >= csa_index_topk_workspace_bytes()
 * Scores are computed from the stored values with fp32 accumulation.
 * ------------------------------------------------------------------------- */
size_t csa_index_topk_workspace_bytes(const csa_params* p, int B, int Q, int N);
csa_status csa_index_topk(const csa_params* p, int B, int Q,
                          const int32_t* q_pos, const void* qI, const float* w,
                          const void* kI, int N, int32_t* idx_out,
                          float* score_out, void* workspace, size_t ws_bytes,
                          csa_stream_t stream);

/* csa_index_topk_noalloc: csa_index_topk for callers that cannot allocate
 * device memory or pass a workspace -- e.g. plugins of a host framework that
 * owns all device memory, or latency-critical loops where an allocation would
 * synchronise the device.  The pages have no counterpart: this is a library
 * convenience, not part of the method.
 *   Same arguments and results as csa_index_topk, without the workspace.
 *   The scratch is one fixed 16 MiB device array inside the library; it
 *   occupies that memory on every GPU that loads the library until the
 *   process exits.  A request fits when csa_index_topk_workspace_bytes(p, B,
 *   Q, N) -- the workspace csa_index_topk would take: 4 B*Q*N bytes of fp32
 *   scores, the tile plan and, for a few long queries, the multi-CTA top-k
 *   lists -- is at most 16 MiB (16,777,216 bytes); the 1M-context decode of
 *   4 sequences needs about 6.6 MiB.  A request that needs more returns
 *   CSA_ERR_WORKSPACE before anything is launched.
 *   The first call on a device looks up the array's device address (with
 *   that device current); make that first call before any stream capture.
 *   Every call on a device shares the same array: calls whose kernels can
 *   overlap on the GPU (different streams without ordering between them)
 *   race on it and give undefined results.  Nothing in it needs to start at
 *   zero; it keeps the last call's contents.
 *   Calls no cudaMalloc, cudaFree or other allocating routine. */
csa_status csa_index_topk_noalloc(const csa_params* p, int B, int Q,
                                  const int32_t* q_pos, const void* qI,
                                  const float* w, const void* kI, int N,
                                  int32_t* idx_out, float* score_out,
                                  csa_stream_t stream);

/* ---------------------------------------------------------------------------
 * MXFP4 indexer ("02 · DeepSeek-V4: 压缩注意力撑起 1M 上下文" 3.3: the
 * indexer's QK path in FP4 with bf16 scores).  Format (OCP Microscaling
 * MXFP4): a row of `width` values is cut into blocks of 32 consecutive
 * values; a block's scale is 2^e with e = floor(log2 max|x|) - 2 (-127 for
 * an all-zero block), stored as one E8M0 byte e + 127; each value is
 * x / 2^e rounded to the nearest E2M1 value (0, 0.5, 1, 1.5, 2, 3, 4, 6;
 * ties to the even mantissa; saturating at 6), stored as a 4-bit code (bit
 * 3 the sign), value 2j in the low nibble of byte j.
 *
 * csa_mxfp4_quantize: x [rows][width] bf16 -> codes [rows][width/2] bytes,
 *   scales [rows][width/32] bytes.  width % 32 == 0; x and codes 16-byte
 *   aligned.
 * csa_index_topk_mxfp4: csa_index_topk with the keys in MXFP4 (kI_codes
 *   [B][N][c_I/2], kI_scales [B][N][c_I/32]) and q^I (bf16, as in
 *   csa_index_topk) rounded to MXFP4 per head and block inside the call.
 *   The score of an entry is sum_h w_h ReLU(q^I_h . K^I_s) of the rounded
 *   values, accumulated in fp32 and rounded to bf16 (returned as fp32
 *   values); ties are broken towards the lower index as in csa_index_topk.
 *   Requires act = CSA_BF16, c_I = 128, n_hI a multiple of 16 up to 64
 *   (else CSA_ERR_UNSUPPORTED).  Block exponents must lie in [-23, 13]
 *   (block maxima in [2^-21, 2^16)) for exact products; a block outside
 *   that range with a nonzero code raises CSA_DEV_RANGE.  Workspace:
 *   csa_index_topk_workspace_bytes().
 * ------------------------------------------------------------------------- */
csa_status csa_mxfp4_quantize(int rows, int width, const void* x, void* codes, void* scales,
                              csa_stream_t stream);
csa_status csa_index_topk_mxfp4(const csa_params* p, int B, int Q, const int32_t* q_pos,
                                const void* qI, const float* w, const void* kI_codes,
                                const void* kI_scales, int N, int32_t* idx_out,
                                float* score_out, void* workspace, size_t ws_bytes,
                                csa_stream_t stream);

/* ---------------------------------------------------------------------------
 * csa_attend: shared-KV multi-query attention of each query over its
 * selected entries and its last n_win tokens, in ONE softmax whose
 * denominator also holds exp(z'_h) ([N] eq. 19, 2.5.3, eq. 27; [P] 2.4),
 * followed by R_{-t0} on the last rope_dims of each head's output ([N]
 * 2.5.2).  logits = softmax_scale * q_h . key; key = value = the stored row.
 *   q_pos    [B*Q] int32           query positions t0
 *   q        [B*Q][n_h][c]         act dtype, already normalised and rotated
 *   idx      [B*Q][topk] int32     entries to attend (-1 = unused slot)
 *   ckv      [B][N][row], ckv_scale [B][N] (FP8MIX only, else NULL)
 *   win      [B][W][row], win_scale [B][W] (FP8MIX only, else NULL): row w
 *            of sequence b holds token win_pos0[b] + w; the query attends
 *            tokens max(0, t0-n_win+1) .. t0, which must all be present
 *   win_pos0 [B] int32
 *   sink     [n_h] fp32            sink logits z'_h
 *   out      [B*Q][n_h][c]         act dtype
 *   workspace / ws_bytes           >= csa_attend_workspace_bytes()
 * hca_attend: the same over ALL visible entries s < floor((t0+1)/m) (no
 * selection, [N] eq. 26, [P] 2.3) plus the window.
 * ------------------------------------------------------------------------- */
size_t csa_attend_workspace_bytes(const csa_params* p, int B, int Q, int N);
csa_status csa_attend(const csa_params* p, int B, int Q, const int32_t* q_pos,
                      const void* q, const int32_t* idx,
                      const void* ckv, const float* ckv_scale, int N,
                      const void* win, const float* win_scale, int W,
                      const int32_t* win_pos0, const float* sink, void* out,
                      void* workspace, size_t ws_bytes, csa_stream_t stream);
csa_status hca_attend(const csa_params* p, int B, int Q, const int32_t* q_pos,
                      const void* q, const void* ckv, const float* ckv_scale,
                      int N, const void* win, const float* win_scale, int W,
                      const int32_t* win_pos0, const float* sink, void* out,
                      void* workspace, size_t ws_bytes, csa_stream_t stream);

/* ---------------------------------------------------------------------------
 * Status and diagnostics.
 * csa_device_status waits for `stream`, returns the device error word of the
 * current GPU in *flags (CSA_DEV_* bits, 0 = clean) and clears it.
 * csa_kernel_launches returns how many kernels this library has launched in
 * this process (all GPUs), a counter for benchmarks.
 * ------------------------------------------------------------------------- */
csa_status csa_device_status(csa_stream_t stream, uint32_t* flags);

/* csa_diag_bounded_wait: runs, on purpose, the failure path of the bounded
 * device-side wait that every kernel of the library uses (no page
 * counterpart: a diagnostic of the library).  One CTA holds a TMEM
 * allocation and waits on an mbarrier with a limit of limit_ns
 * (0 < limit_ns <= 2e9, the kernels' own limit); with arrive = 0 nothing
 * arrives, the wait gives up, CSA_DEV_TIMEOUT is set in the device error
 * word and the CTA winds down like the library's kernels (TMEM freed, kernel
 * returns); with arrive = 1 a second warp arrives after limit_ns / 10 and
 * the wait completes.  waited_ns (device pointer, nullable) receives the
 * time spent waiting.  CSA_ERR_ARG for a limit out of range or arrive not
 * 0/1. */
csa_status csa_diag_bounded_wait(uint64_t limit_ns, int arrive, uint64_t* waited_ns,
                                 csa_stream_t stream);
const char* csa_status_string(csa_status s);
uint64_t csa_kernel_launches(void);
int csa_abi_version(void);

/* ---------------------------------------------------------------------------
 * Per-kernel device-time profiling.  While enabled, every kernel launch of
 * the library is bracketed by two CUDA events on its stream (a few us of host
 * time per launch, nothing on the device timeline).  csa_profile_collect
 * waits for the recorded events, writes for each kernel kind k <
 * csa_profile_kernel_count() the summed device time in ms and the number of
 * launches since the previous collect (arrays of that length, caller-owned),
 * and starts a new collection.  Kind names come from csa_profile_kernel_name.
 * ------------------------------------------------------------------------- */
void csa_profile_enable(int on);
int csa_profile_kernel_count(void);
const char* csa_profile_kernel_name(int kind);
csa_status csa_profile_collect(double* total_ms, uint64_t* launches);

#ifdef __cplusplus
}
#endif
#endif /* CSA_H */
