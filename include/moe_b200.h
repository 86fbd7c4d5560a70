/*
 * moe_b200.h -- C ABI of a single-GPU Mixture-of-Experts expert layer for NVIDIA B200 (sm_100a).
 *
 * What the layer computes follows "Olmo-core 3" as the three news pages describe it:
 *   - each token activates k of E experts (noticiarioia.com, "Mudanca de arquitetura e ganhos de
 *     desempenho"; unite.ai, intro);
 *   - routing metadata stays on the GPU so the host enqueues work without waiting for copies back
 *     (bytechap.com, "Como funciona"; unite.ai, "Parallelismo, precisione e tecniche di memoria");
 *   - routed rows are written straight into each expert's contiguous input buffer ("row-wise"
 *     expert parallelism; same two sections);
 *   - one device-scheduled grouped GEMM runs all experts without host synchronisation (unite.ai,
 *     same section);
 *   - MXFP8 operands are supported (unite.ai, same section; noticiarioia.com, "Otimizacoes e
 *     testes em escala de trilhoes").
 * The formulas the pages leave open are fixed as follows (per token t):
 *   l_t = W_r x_t (+ bias); S_t = top-k experts of l_t, equal scores to the lower expert id, slots in
 *   descending score order; g_t,j = softmax(l_t)[S_j] renormalised over S_t;
 *   out_t = sum_j g_t,j W2_e (silu(W1_e x_t) * W3_e x_t), e = S_t,j, W13_e = [W1_e ; W3_e].
 *
 * Conventions shared by every entry point
 *   - All pointers are DEVICE pointers unless the argument says "host". The caller allocates and
 *     owns every buffer; the library never allocates, frees, synchronises the host or copies device
 *     to host (moe_get_error is the one explicit, caller-requested exception).
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream). All work is
 *     enqueued asynchronously on it; results are valid once that stream reaches this point.
 *   - Tensors are dense row-major. Weights use the [out, in] convention: W_r [E,d], W13 [E,2F,d]
 *     (rows 0..F-1 gate W1, rows F..2F-1 up W3), W2 [E,d,F].
 *   - "act" dtype is fp32 when cfg->dtype == MOE_DTYPE_FP32 and bf16 otherwise. Router scores,
 *     gates and gate gradients are always fp32; index arrays are int32.
 *   - Routed-row buffers have moe_max_rows(cfg) rows: T*k + (A-1)*E rounded up to a multiple of A,
 *     where A, the group alignment, is 32 rows (128 in MXFP8 mode, whose scales move in 128-row
 *     chunks). Each expert's group starts on an A-row boundary (poff) and its pad rows are kept at
 *     zero by the kernels that write the buffer.
 *   - Every function returns MOE_OK (0) or a negative MOE_ERR_* code. Arguments are validated on the
 *     host before anything is enqueued; on an error nothing is enqueued.
 *   - Device-side problems (an expert id outside [0,E), counts that do not add up to T*k, a
 *     non-finite router score, a bounded wait that ran out) set bits of a sticky int32 flag that
 *     lives in the first bytes of the workspace; kernels that detect them skip the offending
 *     accesses and return instead of trapping or spinning. Read it with moe_get_error.
 *   - Calls are stateless and re-entrant; two calls may share a workspace only if they are ordered
 *     on the same stream.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* ---- status codes ---------------------------------------------------------------------------- */
#define MOE_OK 0
#define MOE_ERR_INVALID_ARG (-1) /* null pointer, bad size, bad enum value */
#define MOE_ERR_UNSUPPORTED (-2) /* valid request outside what this build implements */
#define MOE_ERR_WORKSPACE (-3)   /* workspace missing or smaller than moe_workspace_size() */
#define MOE_ERR_CUDA (-4)        /* a CUDA runtime/driver call failed (launch, tensor map) */

/* ---- device error flag bits (moe_get_error) --------------------------------------------------- */
#define MOE_DEVERR_ROUTING 1u  /* expert id out of range or sum(counts) != T*k */
#define MOE_DEVERR_TIMEOUT 2u  /* a bounded pipeline wait ran out; the kernel returned early */
#define MOE_DEVERR_NONFINITE 4u/* a router score was NaN or infinite */

/* ---- configuration ----------------------------------------------------------------------------- */
enum moe_dtype {
  MOE_DTYPE_FP32 = 0,  /* fp32 storage, GEMMs on tf32 tensor cores, fp32 accumulate */
  MOE_DTYPE_BF16 = 1,  /* bf16 storage, fp32 accumulate */
  MOE_DTYPE_MXFP8 = 2  /* bf16 storage, GEMM operands E4M3 + one UE8M0 scale per 32 along K */
};

typedef struct {
  int T;      /* tokens, >= 1 */
  int d;      /* model width, multiple of 64 */
  int F;      /* expert hidden width, multiple of 128 */
  int E;      /* experts, 1..256 */
  int k;      /* experts per token, 1..min(E, 8) */
  int dtype;  /* enum moe_dtype */
  int renorm; /* 1: gates renormalised over the chosen k (required by the backward pass) */
} moe_config_t;

/* Rows of every routed-row buffer: T*k + (A-1)*E rounded up to A (A = 32, or 128 in MXFP8 mode).
 * Returns 0 for an invalid config. */
MOE_API int64_t moe_max_rows(const moe_config_t* cfg);

/* Bytes of scratch the layer-level calls need (routing histograms, router-gradient scratch incl.
 * the router weight gradient's fp32 partials, and the sticky error flag). The first call on a fresh workspace must be preceded by moe_clear_error (or a
 * zero fill of the buffer) so that the flag starts at 0. Returns MOE_ERR_INVALID_ARG on a bad cfg. */
MOE_API int moe_workspace_size(const moe_config_t* cfg, size_t* bytes /* host */);

/* Copy the sticky device error flag to *flags (host) -- synchronises with `stream`. */
MOE_API int moe_get_error(const void* ws, uint32_t* flags /* host */, void* stream);
/* Reset the sticky device error flag to 0 (asynchronous on `stream`). */
MOE_API int moe_clear_error(void* ws, void* stream);

/* ---- routing ------------------------------------------------------------------------------------ */

/* Router scores l = x W_r^T (+ bias), fp32 [T,E]. x: act [T,d]; W_r: act [E,d]; bias: fp32 [E] or
 * NULL (a constant input with no gradient). Tensor-core GEMM with fp32 accumulation. */
MOE_API int moe_router_logits(const moe_config_t* cfg, const void* x, const void* W_r, const float* bias,
                      float* logits, void* ws, size_t ws_bytes, void* stream);

/* Top-k selection and gates (bytechap.com, "Detalles clave": routing scores pick the experts).
 * logits: fp32 [T,E]; bias: fp32 [E] added before selection and softmax, or NULL.
 * idx: int32 [T,k] out -- the k largest scores, equal scores to the lower id, descending order.
 * gates: fp32 [T,k] out -- softmax probabilities of the chosen experts, renormalised over the k
 * chosen when cfg->renorm. A non-finite score sets MOE_DEVERR_NONFINITE. */
MOE_API int moe_route_topk(const moe_config_t* cfg, const float* logits, const float* bias, int32_t* idx,
                   float* gates, void* ws, size_t ws_bytes, void* stream);

/* GPU-resident routing metadata from idx (int32 [T,k]); no host synchronisation (bytechap.com,
 * "Como funciona"). Outputs (all int32):
 *   counts[E]      rows routed to each expert;
 *   offsets[E+1]   exclusive prefix sum of counts, offsets[E] = T*k;
 *   poff[E+1]      exclusive prefix sum of counts rounded up to the group alignment (32 rows,
 *                  128 for MXFP8 configs): expert e owns padded rows [poff[e], poff[e+1]) of every
 *                  routed-row buffer;
 *   perm[T*k]      position of entry t*k+j in the expert-sorted order, ascending token id within an
 *                  expert (a stable counting sort; deterministic, no atomics in the ordering);
 *   prow[T*k]      padded row of entry t*k+j: poff[e] + perm - offsets[e];
 *   row_token[max_rows]  entry t*k+j held by each padded row, -1 for pad rows and unused rows.
 * An expert id outside [0,E) sets MOE_DEVERR_ROUTING; such an entry gets no row (perm = prow = -1),
 * and dispatch, combine, combine_bwd and the token reduce skip every entry whose prow lies outside
 * [0, max_rows): nothing is read or written through it. */
MOE_API int moe_route_metadata(const moe_config_t* cfg, const int32_t* idx, int32_t* counts,
                       int32_t* offsets, int32_t* poff, int32_t* perm, int32_t* prow,
                       int32_t* row_token, void* ws, size_t ws_bytes, void* stream);

/* Allocation-free variant of moe_route_metadata (the pages have no counterpart; this is a service
 * for callers). Some callers cannot allocate device memory: an engine plugin handed only its input and
 * output tensors under a fixed memory plan, or a host runtime without a device allocator, cannot
 * provide the workspace moe_route_metadata needs for its per-chunk histograms. This entry point takes
 * the same inputs and outputs (same meaning, layout and results) and no workspace: its scratch is a
 * static device array inside the library of 65536 int32 (256 KB), held on every GPU that loads the
 * library until the process exits.
 *   - Limit: ceil(T/256) * E <= 65536 (e.g. T = 131072 at E = 128); larger requests return
 *     MOE_ERR_WORKSPACE and enqueue nothing.
 *   - The first call on a device looks up the scratch's device address (cudaGetSymbolAddress, with
 *     that device current), and so does the first call after the device's context has been
 *     re-created (cudaDeviceReset); make such a call before any stream capture.
 *   - Every call on a device shares the one array: calls that overlap on the GPU (other streams, other
 *     host threads) race and corrupt each other's results. Order them on one stream.
 *   - Nothing in the scratch needs clearing (each call writes all it reads). Device-side routing
 *     errors (expert ids outside [0,E)) are not reported, since there is no error flag; such entries
 *     get perm = prow = -1 as in moe_route_metadata. */
MOE_API int moe_route_metadata_noalloc(const moe_config_t* cfg, const int32_t* idx, int32_t* counts,
                                       int32_t* offsets, int32_t* poff, int32_t* perm, int32_t* prow,
                                       int32_t* row_token, void* stream);

/* ---- row-wise dispatch and combine --------------------------------------------------------------- */

/* Row-wise dispatch (unite.ai, "Parallelismo, precisione e tecniche di memoria": each routed token is
 * written directly into its expert's input buffer): x_perm[prow[t*k+j]] = x[t] for all j, and every
 * pad row [poff[e]+counts[e], poff[e+1]) is zeroed. x: act [T,d]; x_perm: act [max_rows,d] (bf16 in
 * MXFP8 mode, quantised afterwards with moe_quantize_mxfp8_rowcol). */
MOE_API int moe_dispatch(const moe_config_t* cfg, const void* x, const int32_t* prow, const int32_t* counts,
                 const int32_t* poff, void* x_perm, void* stream);

/* Gate-weighted combine (the pages are silent on the combine; this is the gate-weighted sum over the
 * token's k experts that the layer's definition gives): out[t] = sum_j gates[t,j] * y[prow[t*k+j]]
 * (fp32 accumulation, a gather:
 * deterministic, no atomics). y: act [max_rows,d]; out: act [T,d]. */
MOE_API int moe_combine(const moe_config_t* cfg, const void* y, const float* gates, const int32_t* prow,
                void* out, void* stream);

/* Backward of the combine (pages silent; the exact derivative of moe_combine):
 * dy[prow[t*k+j]] = gates[t,j] * dout[t]; dgates[t,j] = <dout[t], y[row]>.
 * Pad rows of dy are zeroed. When dlsel is non-NULL (learned router, renormalised gates) it also
 * writes dlsel[t,j] = g_j (dg_j - sum_i g_i dg_i), the score gradient of the chosen experts, and,
 * when dlogits is non-NULL, the dense score gradient dlogits[t,e] (act [T,E], zero for experts
 * not chosen). dout: act [T,d]; y: act [max_rows,d]; dy: act [max_rows,d]; dgates, dlsel: fp32 [T,k]. */
MOE_API int moe_combine_bwd(const moe_config_t* cfg, const void* dout, const void* y, const float* gates,
                    const int32_t* prow, const int32_t* idx, const int32_t* counts,
                    const int32_t* poff, void* dy, float* dgates, float* dlsel, void* dlogits,
                    void* stream);

/* Scatter-add of routed-row gradients back to tokens (pages silent; the exact derivative of the
 * dispatch), done as a deterministic gather-sum:
 * dx[t] = sum_j dx_perm[prow[t*k+j]] (+ sum_j dlsel[t,j] * W_r[idx[t,j]] when dlsel, idx and W_r
 * are all non-NULL: the router's input gradient). dx_perm: act [max_rows,d]; dx: act [T,d]. */
MOE_API int moe_token_reduce(const moe_config_t* cfg, const void* dx_perm, const int32_t* prow,
                     const float* dlsel, const int32_t* idx, const void* W_r, void* dx, void* stream);

/* ---- device-scheduled grouped GEMM (tcgen05 tensor cores, TMA, TMEM) ------------------------------ */

enum moe_gemm_op {
  /* h13 = X_e W13_e^T and a = silu(h13[:, :F]) * h13[:, F:] for every expert's rows.
   * A = x_perm act [max_rows,d]; B = W13 [E,2F,d]; C = h13 act [max_rows,2F]; C2 = a act [max_rows,F].
   * C may be NULL: only a is stored (the forward of a layer that recomputes h13 in its backward). */
  MOE_GEMM_FWD1_SWIGLU = 0,
  /* y = a_e W2_e^T.  A = a [max_rows,F]; B = W2 [E,d,F]; C = y [max_rows,d]. */
  MOE_GEMM_FWD2 = 1,
  /* da = dy_e W2_e, then the SwiGLU backward with the saved h13 (aux):
   * dh13[:, :F] = da * up * silu'(gate), dh13[:, F:] = da * silu(gate).
   * A = dy [max_rows,d]; B = W2 [E,d,F]; aux = h13 [max_rows,2F]; C = dh13 [max_rows,2F].
   * aux may be C itself (dh13 overwrites h13 in place: each element is read before it is written). */
  MOE_GEMM_DGRAD2_SWIGLU = 2,
  /* dx_perm = dh13_e W13_e.  A = dh13 [max_rows,2F]; B = W13 [E,2F,d]; C = dx_perm [max_rows,d]. */
  MOE_GEMM_DGRAD1 = 3,
  /* dW2_e = dy_e^T a_e over the expert's rows (zero for an expert with no rows).
   * A = dy [max_rows,d]; B = a [max_rows,F]; C = dW2 act [E,d,F]. */
  MOE_GEMM_WGRAD2 = 4,
  /* dW13_e = dh13_e^T x_perm_e.  A = dh13 [max_rows,2F]; B = x_perm [max_rows,d]; C = dW13 [E,2F,d]. */
  MOE_GEMM_WGRAD1 = 5
};

/* One launch runs every expert. The tile schedule is built on the device from counts/poff (as
 * produced by moe_route_metadata): a persistent grid of one CTA per SM walks the ragged tiles, so the
 * host never learns the group sizes. Row tiles past an expert's padded end are masked. Rows of the
 * routed buffers must keep the zero pad rows that dispatch / combine_bwd / this GEMM write. */
MOE_API int moe_grouped_gemm(const moe_config_t* cfg, int op, const void* A, const void* B, void* C, void* C2,
                     const void* aux, const int32_t* counts, const int32_t* poff, void* ws,
                     size_t ws_bytes, void* stream);

/* Router weight gradient dW_r = dlogits^T x (act [E,d]) from the dense score gradient written by
 * moe_combine_bwd (act [T,E]); a tensor-core GEMM contracting over tokens. When its output tiles are
 * too few to fill the GPU, the token range is split into chunks whose fp32 partial products go to
 * the workspace and are summed in a fixed order (deterministic). ws as for moe_workspace_size. */
MOE_API int moe_router_wgrad(const moe_config_t* cfg, const void* dlogits, const void* x, void* dW_r,
                     void* ws, size_t ws_bytes, void* stream);

/* ---- MXFP8 ----------------------------------------------------------------------------------------- */

/* MXFP8 quantisation of a bf16 matrix src [rows, cols] (row-major), per the OCP Microscaling (MX) v1.0
 * definitions (the pages only name the format: unite.ai, "Parallelismo, precisione e tecniche di
 * memoria"): per block of 32 elements, scale byte e+127 with e = clamp(floor(log2 amax) - 8, -127,
 * 127) (0 for an all-zero block) and E4M3 codes round-to-nearest-even(x / 2^e) saturated to +-448.
 * Codes q always keep the layout of src. Blocks and scale layouts by mode:
 *   MOE_QUANT_ROW        blocks along a row;    s [rows, cols/32]                       (cols % 32)
 *   MOE_QUANT_COL        blocks down a column;  s [cols, rows/32]              (rows % 32, cols % 8)
 *   MOE_QUANT_ROW_TILED  blocks along a row;    s tiled over (row, block)    (rows, cols % 128)
 *   MOE_QUANT_COL_TILED  blocks down a column;  s tiled over (column, block) (rows, cols % 128)
 *   MOE_QUANT_ROW_TILED_GATEUP  as ROW_TILED for stacks of [G gate rows; G up rows] (W13 with
 *                        G = F), rows remapped so each 64 gate + 64 up rows share chunks (G % 64);
 *                        a layout for 64 + 64-row fused tiles (the layer's grouped GEMM takes
 *                        128 + 128-row tiles and plain ROW_TILED W13 scales).
 * Tiled: the scale of (MN index i, K-block b) -- i = row for ROW modes, column for COL modes -- sits in
 * 512-byte chunk (i/128, b/4) (chunks of one i/128 consecutive), at byte (i%32)*16 + ((i%128)/32)*4 +
 * b%4: the layout the MXFP8 grouped GEMM streams. `G` is used by the GATEUP mode only.
 * src 16-byte aligned; q 16-byte (ROW modes) / 8-byte (COL modes) aligned. */
#define MOE_QUANT_ROW 0
#define MOE_QUANT_COL 1
#define MOE_QUANT_ROW_TILED 2
#define MOE_QUANT_COL_TILED 3
#define MOE_QUANT_ROW_TILED_GATEUP 4
MOE_API int moe_quantize_mxfp8(const void* src, int64_t rows, int cols, int mode, int64_t G, uint8_t* q,
                               uint8_t* s, void* stream);

/* Both tiled quantisations of one operand from a single read of src: MOE_QUANT_ROW_TILED into
 * (q_row, s_row) and MOE_QUANT_COL_TILED into (q_col, s_col), bit-identical to two moe_quantize_mxfp8
 * calls. For an activation that one GEMM contracts along its columns and another along its rows
 * (x_perm, a, dy, dh13 of the layer). rows % 128 == 0, cols % 128 == 0; src and q_col 16-byte
 * aligned, q_row 8-byte aligned; the four outputs must not overlap. */
MOE_API int moe_quantize_mxfp8_rowcol(const void* src, int64_t rows, int cols, uint8_t* q_row,
                                      uint8_t* s_row, uint8_t* q_col, uint8_t* s_col, void* stream);

/* One MXFP8 operand in both tiled orientations (caller-owned), for a routed-row activation [R, cols]
 * with R = moe_max_rows(cfg): row-block codes q_row [R, cols] + scales s_row (MOE_QUANT_ROW_TILED,
 * R*cols/32 bytes; 4-byte aligned) for the GEMM that contracts along the columns, and column-block
 * codes q_col [R, cols] + scales s_col (MOE_QUANT_COL_TILED over 32-row blocks of the expert groups,
 * cols*R/32 bytes) for the weight gradient that contracts over the expert's rows. Code arrays are
 * 16-byte aligned. */
typedef struct {
  uint8_t *q_row, *s_row, *q_col, *s_col;
} moe_mxfp8_operand_t;

/* Row-wise dispatch straight into MXFP8 expert buffers (unite.ai, "Parallelismo, precisione e
 * tecniche di memoria": tokens are written directly into their experts' buffers, and MXFP8 cuts the
 * expert data moved): the routed buffer x_perm[r] = x[row_token[r] / k] (zero for pad rows) is formed
 * and quantised in one pass -- no bf16 x_perm is written. Codes and scales are bit-identical to
 * moe_dispatch followed by moe_quantize_mxfp8_rowcol on rows [0, poff[E]); rows at or past poff[E] are
 * not written (no GEMM reads them). x: bf16 [T,d] (16-byte aligned); row_token, poff: from
 * moe_route_metadata; out: [R, d] operand. cfg->dtype must be MOE_DTYPE_MXFP8, d % 128 == 0. */
MOE_API int moe_dispatch_mxfp8(const moe_config_t* cfg, const void* x, const int32_t* row_token,
                               const int32_t* poff, const moe_mxfp8_operand_t* out, void* stream);

/* Backward of the combine straight into MXFP8 (the pages are silent on the backward's formulas; this
 * is the exact derivative of the combine): dy[r] = bf16(gates[n] * dout[n / k]) with n = row_token[r]
 * (zero for pad rows) is formed and quantised in one pass -- no bf16 dy is written -- and
 * dgates[n] = <dout[n / k], y[r]> (fp32, fixed summation order). Codes and scales are bit-identical to
 * quantising the bf16 dy that moe_combine_bwd writes. dout: bf16 [T,d]; y: bf16 [R,d]; gates, dgates:
 * fp32 [T,k]; dy: [R, d] operand. Score gradients of a learned router are not computed here
 * (moe_layer_bwd_mxfp8 adds them). cfg->dtype must be MOE_DTYPE_MXFP8, d % 128 == 0. */
MOE_API int moe_combine_bwd_mxfp8(const moe_config_t* cfg, const void* dout, const void* y,
                                  const float* gates, const int32_t* row_token, const int32_t* poff,
                                  float* dgates, const moe_mxfp8_operand_t* dy, void* stream);

/* The grouped GEMM of moe_grouped_gemm with MXFP8 operands (tcgen05 kind::mxf8f6f4.block_scale, fp32
 * accumulation, bf16 outputs). Each operand is E4M3 codes in the layout its bf16 counterpart has in
 * moe_grouped_gemm plus UE8M0 scales, tiled, along that GEMM's contraction axis:
 *   FWD1_SWIGLU   A = x_perm ROW_TILED [R,d]     B = W13 ROW_TILED [E*2F,d]
 *   FWD2          A = a      ROW_TILED [R,F]     B = W2  ROW_TILED [E*d,F]
 *   DGRAD2_SWIGLU A = dy     ROW_TILED [R,d]     B = W2  COL_TILED [E*d,F]
 *   DGRAD1        A = dh13   ROW_TILED [R,2F]    B = W13 COL_TILED [E*2F,d]
 *   WGRAD2        A = dy     COL_TILED [R,d]     B = a   COL_TILED [R,F]
 *   WGRAD1        A = dh13   COL_TILED [R,2F]    B = x_perm COL_TILED [R,d]
 * with R = moe_max_rows(cfg) (a multiple of 128 in MXFP8 mode; expert groups start on 128-row
 * boundaries, so the wgrads' contraction blocks never straddle two experts). aux (DGRAD2) is the bf16
 * h13. Requires cfg->dtype == MOE_DTYPE_MXFP8, d % 128 == 0. */
MOE_API int moe_grouped_gemm_mxfp8(const moe_config_t* cfg, int op, const uint8_t* Aq, const uint8_t* As,
                                   const uint8_t* Bq, const uint8_t* Bs, void* C, void* C2,
                                   const void* aux, const int32_t* counts, const int32_t* poff,
                                   void* ws, size_t ws_bytes, void* stream);

/* The two MXFP8 SwiGLU GEMMs with their activation output quantised in the epilogue (both tiled
 * orientations of its bf16 value; no bf16 copy of it is written). Operands as for
 * moe_grouped_gemm_mxfp8:
 *   MOE_GEMM_FWD1_SWIGLU   C = h13 bf16 [R,2F] (kept for the backward), out = a [R, F];
 *   MOE_GEMM_DGRAD2_SWIGLU aux = h13 bf16, C unused (may be NULL), out = dh13 [R, 2F].
 * Codes and scales are bit-identical to moe_quantize_mxfp8_rowcol of the bf16 output that
 * moe_grouped_gemm_mxfp8 writes for the same op. Other ops: MOE_ERR_INVALID_ARG. */
MOE_API int moe_grouped_gemm_mxfp8_quant(const moe_config_t* cfg, int op, const uint8_t* Aq,
                                         const uint8_t* As, const uint8_t* Bq, const uint8_t* Bs,
                                         void* C, const void* aux, const moe_mxfp8_operand_t* out,
                                         const int32_t* counts, const int32_t* poff, void* ws,
                                         size_t ws_bytes, void* stream);

/* ---- whole layer ------------------------------------------------------------------------------------ */

typedef struct {
  const void* W_r; /* act [E,d]; NULL when routing is given as input (saved->idx / saved->gates) */
  const void* W13; /* act [E,2F,d] */
  const void* W2;  /* act [E,d,F] */
} moe_weights_t;

/* Forward results kept for the backward pass. Caller-owned device buffers. */
typedef struct {
  float* logits;      /* fp32 [T,E] (learned router only, else may be NULL) */
  int32_t* idx;       /* [T,k]  output, or INPUT when W_r == NULL */
  float* gates;       /* [T,k]  output, or INPUT when W_r == NULL */
  int32_t* counts;    /* [E] */
  int32_t* offsets;   /* [E+1] */
  int32_t* poff;      /* [E+1] */
  int32_t* perm;      /* [T*k] */
  int32_t* prow;      /* [T*k] */
  int32_t* row_token; /* [max_rows] */
  void* x_perm;       /* act [max_rows,d] */
  void* h13;          /* act [max_rows,2F]; NULL selects activation recompute (bf16 / fp32 layer) */
  void* a;            /* act [max_rows,F]; with recompute, scratch between the two passes */
  void* y;            /* act [max_rows,d] */
} moe_saved_t;

/* Gradients (outputs) and backward scratch (caller-owned device buffers). */
typedef struct {
  void* dW_r;    /* act [E,d] (learned router only, else may be NULL) */
  void* dW13;    /* act [E,2F,d] */
  void* dW2;     /* act [E,d,F] */
  float* dgates; /* fp32 [T,k] */
  void* dy;      /* act [max_rows,d]   scratch */
  void* dh13;    /* act [max_rows,2F]  scratch */
  void* dx_perm; /* act [max_rows,d]   scratch */
} moe_grads_t;

/* Whole forward: [router scores -> top-k] -> metadata -> dispatch -> grouped GEMM1 + SwiGLU ->
 * grouped GEMM2 -> combine. x: act [T,d]; bias: fp32 [E] or NULL; out: act [T,d].
 * Activation recompute (the memory-for-throughput trade of unite.ai "Parallelismo, precisione e
 * tecniche di memoria"): with saved->h13 == NULL the forward stores no h13 and moe_layer_bwd recomputes h13 and
 * a with one more GEMM1, writing h13 into grads->dh13 (which the SwiGLU backward then overwrites)
 * and a into saved->a. The caller may reuse saved->a's memory between the two passes. Results are
 * bit-identical to the stored-activation path. */
MOE_API int moe_layer_fwd(const moe_config_t* cfg, const moe_weights_t* w, const void* x, const float* bias,
                  void* out, moe_saved_t* saved, void* ws, size_t ws_bytes, void* stream);

/* Whole backward given dout (act [T,d]): combine_bwd -> GEMM2 dgrad + SwiGLU bwd -> GEMM1 dgrad ->
 * token reduce (+ router input term) -> GEMM2 wgrad -> GEMM1 wgrad (-> router wgrad): the data path
 * first, each op reading what the one before it just wrote, then the weight gradients. x is the
 * forward input; dx (act [T,d]) is the caller's buffer. The selection is held fixed (no gradient
 * through the top-k choice). Requires cfg->renorm == 1 when the router is learned. */
MOE_API int moe_layer_bwd(const moe_config_t* cfg, const moe_weights_t* w, const moe_saved_t* saved,
                  const void* x, const void* dout, void* dx, moe_grads_t* g, void* ws,
                  size_t ws_bytes, void* stream);

/* ---- whole layer, MXFP8 ---------------------------------------------------------------------------------- */

/* Quantised copies of the expert weights (caller-owned; refresh after every weight update), scales
 * in the tiled layouts moe_grouped_gemm_mxfp8 reads (ROW_TILED / COL_TILED):
 *   W13q/W13s  ROW along d  [E*2F, d] / [E*2F, d/32]      (forward GEMM1)
 *   W13tq/W13ts COL along 2F [E*2F, d] / [d, E*2F/32]     (GEMM1 dgrad)
 *   W2q/W2s    ROW along F  [E*d, F] / [E*d, F/32]        (forward GEMM2)
 *   W2tq/W2ts  COL along d  [E*d, F] / [F, E*d/32]        (GEMM2 dgrad) */
typedef struct {
  uint8_t *W13q, *W13s, *W13tq, *W13ts;
  uint8_t *W2q, *W2s, *W2tq, *W2ts;
} moe_mxfp8_weights_t;

/* Quantised routed activations (caller-owned), R32 = moe_max_rows(cfg):
 *   x*: x_perm [R32, d]   a*: a [R32, F]   dy*: dy [R32, d]   dh*: dh13 [R32, 2F]
 *   ?q/?s ROW_TILED (codes [R32, cols], scales R32*cols/32 bytes);
 *   ?tq/?ts COL_TILED (codes [R32, cols], scales cols*R32/32 bytes).
 * Each activation exists only in these two quantised forms (see moe_layer_fwd_mxfp8). Kept from the
 * forward to the backward: the column forms xtq/xts and atq/ats (the weight gradients' operands).
 * xq/xs and aq/as are forward scratch, dy* and dh* backward scratch. */
typedef struct {
  uint8_t *xq, *xs, *xtq, *xts;
  uint8_t *aq, *as, *atq, *ats;
  uint8_t *dyq, *dys, *dytq, *dyts;
  uint8_t *dhq, *dhs, *dhtq, *dhts;
} moe_mxfp8_acts_t;

/* Fill every buffer of qw from the bf16 weights (4 quantisation launches). */
MOE_API int moe_quantize_weights_mxfp8(const moe_config_t* cfg, const moe_weights_t* w,
                                       const moe_mxfp8_weights_t* qw, void* stream);

/* moe_layer_fwd with MXFP8 expert GEMMs (cfg->dtype == MOE_DTYPE_MXFP8): the dispatch writes the
 * routed input only in its two quantised forms (moe_dispatch_mxfp8) and GEMM1's epilogue writes a only
 * in its two quantised forms (moe_grouped_gemm_mxfp8_quant); h13 and y are kept in bf16, SwiGLU and the
 * combine run on bf16 values. saved->x_perm and saved->a are not used (may be NULL). A learned router
 * runs in bf16. Needs all of qa's x* and a* buffers. */
MOE_API int moe_layer_fwd_mxfp8(const moe_config_t* cfg, const moe_weights_t* w,
                                const moe_mxfp8_weights_t* qw, const void* x, const float* bias,
                                void* out, moe_saved_t* saved, const moe_mxfp8_acts_t* qa, void* ws,
                                size_t ws_bytes, void* stream);

/* moe_layer_bwd with MXFP8 expert GEMMs (dgrad operands ROW/COL as listed above, wgrad operands COL
 * along the expert's rows, in 32-row blocks of its zero-padded group). Reads qa's column forms of x and
 * a as the forward left them; dy comes straight out of the combine backward and dh13 out of the
 * SwiGLU-backward epilogue in their two quantised forms only (moe_combine_bwd_mxfp8,
 * moe_grouped_gemm_mxfp8_quant). grads->dy and grads->dh13 are not used (may be NULL). */
MOE_API int moe_layer_bwd_mxfp8(const moe_config_t* cfg, const moe_weights_t* w,
                                const moe_mxfp8_weights_t* qw, const moe_saved_t* saved,
                                const moe_mxfp8_acts_t* qa, const void* x, const void* dout, void* dx,
                                moe_grads_t* g, void* ws, size_t ws_bytes, void* stream);

/* ---- expert parallelism across the GPUs of one node (bf16) --------------------------------------------
 *
 * Row-wise expert parallelism (unite.ai, "Parallelismo, precisione e tecniche di memoria": each routed
 * token row goes directly into the input buffer of the expert that owns it, then device-scheduled
 * grouped GEMMs run every GPU's local experts). G = world ranks, one GPU each (G <= 8, E % G == 0);
 * rank h owns the E/G consecutive experts [h*E/G, (h+1)*E/G). cfg is the per-rank config: T = this
 * rank's tokens, E = all experts. Per step:
 *   1. each rank: moe_route_metadata on its own idx (counts over all E experts, offsets, perm);
 *   2. the caller all-gathers the ranks' counts into all_counts [G][E] (int32, rank-major) with a
 *      collective on the stream (NCCL all_gather);
 *   3. each rank: moe_ep_layout -- every rank derives the same layout of every owner's routed-row
 *      buffers: local expert e's group starts at poff_loc[e] (32-aligned), and inside it the rows of
 *      source rank 0 come first, then rank 1, ...; each source's rows in its own token order;
 *   4. after a collective that orders the ranks (the owners' buffers are free), moe_ep_dispatch stores
 *      this rank's token rows into the owners' x_perm through peer pointers; each owner zeroes its pad
 *      rows with moe_ep_zero_pad;
 *   5. after a collective (every dispatch is done), each owner runs the grouped GEMMs on its local
 *      experts with cfg_loc = {T: G*T*k, k: 1, E: E/G} (so moe_max_rows(cfg_loc) == moe_ep_max_rows),
 *      counts_loc and poff_loc;
 *   6. after a collective, moe_ep_combine gathers the k expert outputs of each token from the owners.
 *   Backward: moe_ep_combine_bwd (dy stored into the owners, gate gradients), moe_ep_zero_pad of dy,
 *   a collective, the owners' dgrad / wgrad GEMMs, a collective, moe_ep_token_reduce.
 * Peer arguments ("*_peers") are HOST arrays of G device pointers, entry h = that buffer on rank h (a
 * peer mapping on a multi-GPU node, e.g. symmetric memory; any device pointers the GPU can reach).
 * Kernels never wait on another GPU: the caller's collectives order the phases. */

/* Rows of each owner's routed-row buffers: G*T*k + 31*E/G rounded up to 32 (every entry of every rank
 * could go to one owner). Returns 0 for an invalid config or world. */
MOE_API int64_t moe_ep_max_rows(const moe_config_t* cfg, int world);

/* Step 3. all_counts [G][E] int32; idx [T,k], perm and offsets from this rank's moe_route_metadata.
 * Outputs: src_base [E] (row, in the owner's buffers, of this rank's first entry for each expert),
 * counts_loc [E/G] and poff_loc [E/G + 1] (this rank as owner), dst_row [T*k] (each entry's row in its
 * owner's buffers; -1 for an expert id outside [0,E)). */
MOE_API int moe_ep_layout(const moe_config_t* cfg, int rank, int world, const int32_t* all_counts,
                          const int32_t* idx, const int32_t* perm, const int32_t* offsets,
                          int32_t* src_base, int32_t* counts_loc, int32_t* poff_loc, int32_t* dst_row,
                          void* stream);

/* Zero the owner's pad rows [poff_loc[e] + counts_loc[e], poff_loc[e+1]) of buf [moe_ep_max_rows, d]. */
MOE_API int moe_ep_zero_pad(const moe_config_t* cfg, int world, void* buf, const int32_t* counts_loc,
                            const int32_t* poff_loc, void* stream);

/* x_perm_owner[dst_row[t*k+j]] = x[t] (owner = idx[t,j] / (E/G)), peer stores. x: bf16 [T,d]. */
MOE_API int moe_ep_dispatch(const moe_config_t* cfg, int world, const void* x, const int32_t* idx,
                            const int32_t* dst_row, void* const* x_perm_peers, void* stream);

/* out[t] = sum_j gates[t,j] * y_owner[dst_row[t*k+j]] (fp32 accumulation), peer loads. */
MOE_API int moe_ep_combine(const moe_config_t* cfg, int world, void* const* y_peers, const float* gates,
                           const int32_t* idx, const int32_t* dst_row, void* out, void* stream);

/* dy_owner[row] = gates[t,j] * dout[t] (peer stores), dgates[t,j] = <dout[t], y_owner[row]> (peer
 * loads), row = dst_row[t*k+j]. A learned router's score gradients are not formed here. */
MOE_API int moe_ep_combine_bwd(const moe_config_t* cfg, int world, const void* dout, void* const* y_peers,
                               const float* gates, const int32_t* idx, const int32_t* dst_row,
                               void* const* dy_peers, float* dgates, void* stream);

/* dx[t] = sum_j dx_perm_owner[dst_row[t*k+j]], peer loads. */
MOE_API int moe_ep_token_reduce(const moe_config_t* cfg, int world, void* const* dx_perm_peers,
                                const int32_t* idx, const int32_t* dst_row, void* dx, void* stream);

/* ---- test support ------------------------------------------------------------------------------------- */

/* Launch one block whose thread waits on a pipeline barrier that nothing ever completes, with the
 * library's bounded wait and the given limit (ns). It must give up, set MOE_DEVERR_TIMEOUT in the
 * workspace flag and return; used to check the timeout path without hanging a GPU. */
MOE_API int moe_test_bounded_wait(void* ws, uint64_t limit_ns, void* stream);

/* Library version string (host). */
MOE_API const char* moe_version(void);

/* Number of kernels this library has enqueued in this process so far (host counter, diagnostics;
 * benchmarks read it before and after a timed region). */
MOE_API uint64_t moe_launch_count(void);

#ifdef __cplusplus
}
#endif
#endif /* MOE_B200_H */
