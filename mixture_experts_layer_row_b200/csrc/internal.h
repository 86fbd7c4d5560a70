// Internal declarations shared by the translation units of libmoe_b200 (not part of the C ABI).
#pragma once

#include "common.cuh"

namespace moe {

// Grouped GEMM epilogues and grouping modes.
// EPI_SWIGLU_FWD_Q / EPI_SWIGLU_BWD_Q (MXFP8 only): as the SwiGLU epilogues, but the activation they
// produce (a, or dh13) leaves as E4M3 codes quantised along rows and along 32-row column blocks, with
// tiled scales, instead of a bf16 copy (the forward still stores h13 in bf16).
enum {
  EPI_STORE = 0,
  EPI_SWIGLU_FWD = 1,
  EPI_SWIGLU_BWD = 2,
  EPI_STORE_F32_BIAS = 3,
  EPI_SWIGLU_FWD_Q = 4,
  EPI_SWIGLU_BWD_Q = 5
};
enum { GROUP_M = 0, GROUP_K = 1 };

// GK_WGRAD_SPLIT: single-group wgrad with the contraction split into chunks of ksplit rows, one fp32
// partial product per chunk (summed afterwards by launch_split_reduce).
// GK_FWD1_SWIGLU_Q / GK_DGRAD2_SWIGLU_Q (MXFP8): the SwiGLU GEMMs with the quantising epilogues.
enum GemmKind {
  GK_FWD1_SWIGLU,
  GK_FWD2,
  GK_DGRAD2_SWIGLU,
  GK_DGRAD1,
  GK_WGRAD,
  GK_ROUTER,
  GK_WGRAD_SPLIT,
  GK_FWD1_SWIGLU_Q,
  GK_DGRAD2_SWIGLU_Q
};

// A row-major 2-D operand as the TMA unit sees it.
struct GemmOperand {
  const void* ptr;
  int64_t rows, cols, ld;  // ld in elements
};

struct GemmParams {
  const int32_t* counts;  // [E] rows per group, or nullptr for one group
  const int32_t* poff;    // [E+1] 32-aligned group starts
  int E;
  int M;  // GROUP_K: output rows per group; single-group GROUP_M: rows
  int N;  // output columns (GROUP_M SwiGLU forward: F)
  int K;  // GROUP_M: contraction length; single-group GROUP_K: contraction rows
  int b_rows_per_group;  // rows of the weight operand's 2-D view per group
  void* C;
  int64_t ldc;
  void* C2;
  int64_t ldc2;
  const void* aux;
  int64_t ldaux;
  const float* bias;
  int F;
  // MXFP8 operands: UE8M0 scales in the tiled layout (512-byte chunks per 128 MN indices x 4
  // K-blocks); sA_ld / sB_ld = chunks per 128 MN indices (= K-blocks / 4 of that operand)
  const uint8_t* sA;
  const uint8_t* sB;
  int64_t sA_ld, sB_ld;
  uint32_t* err;
  uint64_t wait_limit_ns;
  // MN-major operands whose column count is a whole number of 128-byte blocks are loaded as one
  // 3-D box per stage (set by the launcher); otherwise as 32-row x 128-byte 2-D boxes.
  int a_box3d, b_box3d;
  // GROUP_K without groups: contraction rows per split (0 = one split); split s writes C rows
  // [s*c_group_rows, s*c_group_rows + M). c_group_rows (0 = M) is M rounded up to the 32-row store
  // box when M is not a multiple of 32, so a box never reaches into the next split's rows.
  int ksplit;
  int c_group_rows;
  // quantising epilogues: tiled scales of the row-block codes (K-blocks per row: q_kb_row) and of the
  // column-block codes (K-blocks per column: q_kb_col); the codes go out through tensor maps
  uint8_t* q_qr;  // row-block codes [A rows, output columns]
  uint8_t* q_qc;  // column-block codes, same layout
  uint8_t* q_sr;
  uint8_t* q_sc;
  int64_t q_kb_row, q_kb_col;
};

// Host-side count of kernels enqueued (every launcher adds the kernels it launched).
void count_launches(int n);

#define MOE_LAUNCH(call)                              \
  do {                                                \
    if ((call) != cudaSuccess) return MOE_ERR_CUDA;   \
  } while (0)

// Launch with programmatic dependent launch allowed (see pdl_enter): the kernel may be scheduled
// while the previous kernel in the stream finishes; it waits for that kernel before touching memory.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t s, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, args...);
}

// Host helpers for TMA descriptors (swizzle: 2 = 128B, 1 = 128B with 32-byte atoms, 0 = none).
bool make_tmap_nd(CUtensorMap* m, const void* ptr, int es, int rank, const uint64_t* dims,
                  const uint64_t* strides_bytes, const uint32_t* box, int swizzle);
bool make_tmap(CUtensorMap* m, const void* ptr, int es, int64_t rows, int64_t cols, int64_t ld,
               int box_cols, int box_rows, int swizzle);
// MN-major operand [rows, cols] (cols a multiple of 128 bytes) as a 3-D tensor
// (128-byte column block, row, column block), box = box_rows rows x nblk column blocks.
bool make_tmap_mn(CUtensorMap* m, const void* ptr, int es, int64_t rows, int64_t cols, int64_t ld,
                  int box_rows, int nblk, int swizzle);
int sm_count();

int launch_gemm(GemmKind kind, int es, int bn, const GemmOperand& A, const GemmOperand& B,
                const GemmParams& p, cudaStream_t s);
int launch_quantize(const void* src, int64_t rows, int cols, int mode, int64_t G, uint8_t* q,
                    uint8_t* s, cudaStream_t st);
int launch_quantize_rowcol(const void* src, int64_t rows, int cols, uint8_t* qr, uint8_t* sr,
                           uint8_t* qc, uint8_t* sc, cudaStream_t st);
// MXFP8 layer: row- and column-block quantisation of a routed-row operand built from token-order rows
// (rows with row_token < 0 are zero; 32-row blocks at or past *poff_end are skipped).
int launch_dispatch_quant(const void* x, const int32_t* row_token, const int32_t* poff_end, int k,
                          int64_t rows, int cols, uint8_t* qr, uint8_t* sr, uint8_t* qc, uint8_t* sc,
                          cudaStream_t st);
int launch_combine_bwd_quant(const void* dout, const void* y, const float* gates,
                             const int32_t* row_token, const int32_t* poff_end, int k, int64_t rows,
                             int cols, float* dgates, uint8_t* qr, uint8_t* sr, uint8_t* qc,
                             uint8_t* sc, cudaStream_t st);
int launch_bounded_wait_probe(uint32_t* err, uint64_t limit_ns, cudaStream_t s);
// out[i] = round_to_act(sum over s < nsplit of part[s*stride + i]) for i < n (fixed summation order).
int launch_split_reduce(const float* part, int nsplit, int64_t n, int64_t stride, void* out, bool bf16,
                        cudaStream_t s);

int launch_topk(const float* logits, const float* bias, int T, int E, int k, int renorm, int32_t* idx,
                float* gates, uint32_t* err, cudaStream_t s);
size_t metadata_ws_bytes(int T, int E);
// Group alignment of the routed-row buffers: 32 rows, 128 in MXFP8 mode (whole 128-row scale chunks).
inline int group_align(int dtype) { return dtype == MOE_DTYPE_MXFP8 ? 128 : 32; }
int launch_metadata(const int32_t* idx, int T, int E, int k, int align, int64_t max_rows,
                    int32_t* counts, int32_t* offsets, int32_t* poff, int32_t* perm, int32_t* prow,
                    int32_t* row_token, int32_t* hist_ws, uint32_t* err, cudaStream_t s);

// Row kernels: every padded row outside [0, max_rows) (such as the -1 the metadata writes for an
// invalid expert id) is skipped.
int launch_dispatch(const void* x, const int32_t* prow, const int32_t* counts, const int32_t* poff,
                    void* xp, int T, int k, int E, int row_bytes, int64_t max_rows, cudaStream_t s);
int launch_combine(const void* y, const float* gates, const int32_t* prow, void* out, int T, int k,
                   int row_bytes, bool bf16, int64_t max_rows, cudaStream_t s);
int launch_combine_bwd(const void* dout, const void* y, const float* gates, const int32_t* prow,
                       const int32_t* idx, const int32_t* counts, const int32_t* poff, void* dy,
                       float* dgates, float* dlsel, void* dlogits, int T, int k, int E, int row_bytes,
                       bool bf16, int64_t max_rows, cudaStream_t s);
// dlsel[t,j] = g_j (dg_j - sum_i g_i dg_i) and the dense score gradient dlogits [T,E] (act dtype).
int launch_score_grad(const float* gates, const float* dgates, const int32_t* idx, float* dlsel,
                      void* dlogits, int T, int k, int E, bool bf16, cudaStream_t s);
int launch_token_reduce(const void* dxp, const int32_t* prow, const float* dlsel, const int32_t* idx,
                        const void* Wr, void* dx, int T, int k, int E, int row_bytes, bool bf16,
                        int64_t max_rows, cudaStream_t s);

// Expert parallelism across the GPUs of one node (ep.cu). Up to kMaxEpRanks ranks.
constexpr int kMaxEpRanks = 8;
int launch_ep_layout(const int32_t* all_counts, int G, int E, int rank, const int32_t* idx,
                     const int32_t* perm, const int32_t* offsets, int64_t n_entries,
                     int32_t* src_base, int32_t* counts_loc, int32_t* poff_loc, int32_t* dst_row,
                     cudaStream_t s);
int launch_ep_zero_pad(void* buf, const int32_t* counts_loc, const int32_t* poff_loc, int EL,
                       int row_bytes, cudaStream_t s);
// op 0 dispatch (x -> peers_a), 1 combine (peers_a = y -> out), 2 combine backward (dout, peers_a = y,
// peers_b = dy, dgates), 3 token reduce (peers_a = dx_perm -> out)
int launch_ep_rows(int op, int G, int T, int k, int E, int row_bytes, int64_t max_rows,
                   const void* x_or_dout, void* const* peers_a, void* const* peers_b,
                   const float* gates, const int32_t* idx, const int32_t* dst_row, void* out,
                   float* dgates, cudaStream_t s);

}  // namespace moe
