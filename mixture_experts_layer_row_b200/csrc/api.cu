// C ABI of the MoE expert layer library: argument validation, workspace layout, and the forward /
// backward composition of the kernels. Every entry point validates on the host and enqueues nothing
// on an error; all work is asynchronous on the caller's stream; nothing here allocates.
#include <atomic>
#include <cstring>

#include "internal.h"

namespace moe {
static std::atomic<uint64_t> g_launches{0};
void count_launches(int n) { g_launches.fetch_add((uint64_t)n, std::memory_order_relaxed); }
}  // namespace moe

using namespace moe;

namespace {

constexpr uint64_t kWaitLimitNs = 1000ull * 1000ull * 1000ull;  // 1 s per pipeline wait

inline cudaStream_t S(void* s) { return reinterpret_cast<cudaStream_t>(s); }
inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline size_t round256(size_t b) { return (b + 255) & ~size_t(255); }

int check_cfg(const moe_config_t* c) {
  if (!c) return MOE_ERR_INVALID_ARG;
  if (c->T < 1 || c->d < 1 || c->F < 1 || c->E < 1 || c->k < 1) return MOE_ERR_INVALID_ARG;
  if (c->dtype != MOE_DTYPE_FP32 && c->dtype != MOE_DTYPE_BF16 && c->dtype != MOE_DTYPE_MXFP8)
    return MOE_ERR_INVALID_ARG;
  if (c->renorm != 0 && c->renorm != 1) return MOE_ERR_INVALID_ARG;
  if (c->k > c->E) return MOE_ERR_INVALID_ARG;
  if (c->E > 256 || c->k > 8) return MOE_ERR_UNSUPPORTED;
  if (c->d % 64 != 0 || c->F % 128 != 0) return MOE_ERR_UNSUPPORTED;
  const int64_t rows = (int64_t)c->T * c->k + 128ll * c->E + 128;
  if (rows >= (1ll << 31) - 256) return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

inline int es_of(const moe_config_t* c) { return c->dtype == MOE_DTYPE_FP32 ? 4 : 2; }
inline int64_t max_rows_of(const moe_config_t* c) {
  const int64_t a = group_align(c->dtype);
  return ((int64_t)c->T * c->k + (a - 1) * c->E + a - 1) / a * a;
}

// The router weight gradient dW_r = dlogits^T x has only ceil(E/128) x ceil(d/BN) output tiles, too
// few to fill the GPU, so its contraction over the T tokens is split into `n` chunks of `rows` rows
// (a multiple of 32, at least 256) that run as separate tiles; their fp32 partial products are then
// summed in a fixed order. Aim: about one tile per SM of a 148-SM part.
struct RouterSplit {
  int n, rows;
  int slab_rows;  // rows of one split's fp32 partial: E rounded up to the 32-row store box
};

RouterSplit router_split(const moe_config_t* c) {
  const int bn = c->d >= 256 ? 256 : 128;
  const int tiles = ((c->E + 127) / 128) * ((c->d + bn - 1) / bn);
  int n = (148 + tiles - 1) / tiles;
  const int max_n = c->T / 256;
  if (n > max_n) n = max_n;
  const int slab = (c->E + 31) / 32 * 32;
  if (n < 2) return {1, c->T, slab};
  int rows = (c->T + n - 1) / n;
  rows = (rows + 31) / 32 * 32;
  return {(c->T + rows - 1) / rows, rows, slab};
}

struct WsLayout {
  size_t head, hist, dlsel, dlogits, rpart, total;
};

WsLayout ws_layout(const moe_config_t* c) {
  WsLayout w;
  w.head = 0;
  w.hist = kWsHeadBytes;
  w.dlsel = w.hist + round256(metadata_ws_bytes(c->T, c->E));
  w.dlogits = w.dlsel + round256((size_t)c->T * c->k * sizeof(float));
  w.rpart = w.dlogits + round256((size_t)c->T * c->E * es_of(c));
  const RouterSplit rs = router_split(c);
  w.total = w.rpart + (rs.n > 1 ? round256((size_t)rs.n * rs.slab_rows * c->d * sizeof(float)) : 0);
  return w;
}

int check_ws(const moe_config_t* c, void* ws, size_t ws_bytes) {
  if (!ws) return MOE_ERR_WORKSPACE;
  if (!aligned16(ws)) return MOE_ERR_INVALID_ARG;
  if (ws_bytes < ws_layout(c).total) return MOE_ERR_WORKSPACE;
  return MOE_OK;
}

inline uint32_t* err_of(void* ws) { return reinterpret_cast<uint32_t*>(ws); }

#define MOE_TRY(expr)            \
  do {                           \
    const int _r = (expr);       \
    if (_r != MOE_OK) return _r; \
  } while (0)

#define MOE_REQUIRE(cond, code) \
  do {                          \
    if (!(cond)) return (code); \
  } while (0)

GemmParams base_params(const moe_config_t* c, void* ws) {
  GemmParams p;
  std::memset(&p, 0, sizeof(p));
  p.E = c->E;
  p.F = c->F;
  p.err = ws ? err_of(ws) : nullptr;
  p.wait_limit_ns = kWaitLimitNs;
  return p;
}

int gemm_op(const moe_config_t* c, int op, const void* A, const void* B, void* Cout, void* C2,
                 const void* aux, const int32_t* counts, const int32_t* poff, void* ws, cudaStream_t s) {
  const int es = es_of(c);
  const int64_t R = max_rows_of(c);
  const int d = c->d, F = c->F, E = c->E;
  GemmParams p = base_params(c, ws);
  p.counts = counts;
  p.poff = poff;
  p.C = Cout;
  GemmOperand a{A, 0, 0, 0}, b{B, 0, 0, 0};
  switch (op) {
    case MOE_GEMM_FWD1_SWIGLU:
      MOE_REQUIRE(C2, MOE_ERR_INVALID_ARG);
      a = {A, R, d, d};
      b = {B, (int64_t)E * 2 * F, d, d};
      p.K = d; p.N = F; p.b_rows_per_group = 2 * F; p.ldc = 2 * F; p.C2 = C2; p.ldc2 = F;
      return launch_gemm(GK_FWD1_SWIGLU, es, 256, a, b, p, s);
    case MOE_GEMM_FWD2:
      a = {A, R, F, F};
      b = {B, (int64_t)E * d, F, F};
      p.K = F; p.N = d; p.b_rows_per_group = d; p.ldc = d;
      return launch_gemm(GK_FWD2, es, d >= 256 ? 256 : 128, a, b, p, s);
    case MOE_GEMM_DGRAD2_SWIGLU:
      MOE_REQUIRE(aux, MOE_ERR_INVALID_ARG);
      MOE_REQUIRE(aligned16(aux), MOE_ERR_INVALID_ARG);
      a = {A, R, d, d};
      b = {B, (int64_t)E * d, F, F};
      p.K = d; p.N = F; p.b_rows_per_group = d; p.aux = aux; p.ldaux = 2 * F; p.ldc = 2 * F;
      return launch_gemm(GK_DGRAD2_SWIGLU, es, F >= 256 ? 256 : 128, a, b, p, s);
    case MOE_GEMM_DGRAD1:
      a = {A, R, 2 * F, 2 * F};
      b = {B, (int64_t)E * 2 * F, d, d};
      p.K = 2 * F; p.N = d; p.b_rows_per_group = 2 * F; p.ldc = d;
      return launch_gemm(GK_DGRAD1, es, d >= 256 ? 256 : 128, a, b, p, s);
    case MOE_GEMM_WGRAD2:
      a = {A, R, d, d};
      b = {B, R, F, F};
      p.M = d; p.N = F; p.ldc = F;
      return launch_gemm(GK_WGRAD, es, F >= 256 ? 256 : 128, a, b, p, s);
    case MOE_GEMM_WGRAD1:
      a = {A, R, 2 * F, 2 * F};
      b = {B, R, d, d};
      p.M = 2 * F; p.N = d; p.ldc = d;
      return launch_gemm(GK_WGRAD, es, d >= 256 ? 256 : 128, a, b, p, s);
    default:
      return MOE_ERR_INVALID_ARG;
  }
}

int64_t r32_of(const moe_config_t* c) { return max_rows_of(c); }

int gemm_op_mx(const moe_config_t* c, int op, const uint8_t* Aq, const uint8_t* As, const uint8_t* Bq,
               const uint8_t* Bs, void* Cout, void* C2, const void* aux, const int32_t* counts,
               const int32_t* poff, void* ws, cudaStream_t s) {
  const int64_t R = r32_of(c);
  const int d = c->d, F = c->F, E = c->E;
  GemmParams p = base_params(c, ws);
  p.counts = counts;
  p.poff = poff;
  p.C = Cout;
  p.sA = As;
  p.sB = Bs;
  GemmOperand a{Aq, 0, 0, 0}, b{Bq, 0, 0, 0};
  switch (op) {
    case MOE_GEMM_FWD1_SWIGLU:
      MOE_REQUIRE(C2, MOE_ERR_INVALID_ARG);
      a = {Aq, R, d, d};
      b = {Bq, (int64_t)E * 2 * F, d, d};
      p.K = d; p.N = F; p.b_rows_per_group = 2 * F; p.ldc = 2 * F; p.C2 = C2; p.ldc2 = F;
      p.sA_ld = d / 128; p.sB_ld = d / 128;
      return launch_gemm(GK_FWD1_SWIGLU, 1, 128, a, b, p, s);
    case MOE_GEMM_FWD2:
      a = {Aq, R, F, F};
      b = {Bq, (int64_t)E * d, F, F};
      p.K = F; p.N = d; p.b_rows_per_group = d; p.ldc = d;
      p.sA_ld = F / 128; p.sB_ld = F / 128;
      return launch_gemm(GK_FWD2, 1, 128, a, b, p, s);
    case MOE_GEMM_DGRAD2_SWIGLU:
      MOE_REQUIRE(aux && aligned16(aux), MOE_ERR_INVALID_ARG);
      a = {Aq, R, d, d};
      b = {Bq, (int64_t)E * d, F, F};
      p.K = d; p.N = F; p.b_rows_per_group = d; p.aux = aux; p.ldaux = 2 * F; p.ldc = 2 * F;
      p.sA_ld = d / 128; p.sB_ld = (int64_t)E * d / 128;
      return launch_gemm(GK_DGRAD2_SWIGLU, 1, 128, a, b, p, s);
    case MOE_GEMM_DGRAD1:
      a = {Aq, R, 2 * F, 2 * F};
      b = {Bq, (int64_t)E * 2 * F, d, d};
      p.K = 2 * F; p.N = d; p.b_rows_per_group = 2 * F; p.ldc = d;
      p.sA_ld = 2 * F / 128; p.sB_ld = (int64_t)E * 2 * F / 128;
      return launch_gemm(GK_DGRAD1, 1, 128, a, b, p, s);
    case MOE_GEMM_WGRAD2:
      a = {Aq, R, d, d};
      b = {Bq, R, F, F};
      p.M = d; p.N = F; p.ldc = F;
      p.sA_ld = R / 128; p.sB_ld = R / 128;
      return launch_gemm(GK_WGRAD, 1, 128, a, b, p, s);
    case MOE_GEMM_WGRAD1:
      a = {Aq, R, 2 * F, 2 * F};
      b = {Bq, R, d, d};
      p.M = 2 * F; p.N = d; p.ldc = d;
      p.sA_ld = R / 128; p.sB_ld = R / 128;
      return launch_gemm(GK_WGRAD, 1, 128, a, b, p, s);
    default:
      return MOE_ERR_INVALID_ARG;
  }
}

// The MXFP8 SwiGLU GEMMs whose activation output leaves quantised (row-block codes for the next
// GEMM, column-block codes for a weight gradient): FWD1_SWIGLU (C = h13, bf16; out = a) and
// DGRAD2_SWIGLU (aux = h13; out = dh13, no bf16 copy).
int gemm_op_mx_quant(const moe_config_t* c, int op, const uint8_t* Aq, const uint8_t* As,
                     const uint8_t* Bq, const uint8_t* Bs, void* Cout, const void* aux,
                     const moe_mxfp8_operand_t* out, const int32_t* counts, const int32_t* poff,
                     void* ws, cudaStream_t s) {
  const int64_t R = r32_of(c);
  const int d = c->d, F = c->F, E = c->E;
  GemmParams p = base_params(c, ws);
  p.counts = counts;
  p.poff = poff;
  p.C = Cout;
  p.sA = As;
  p.sB = Bs;
  p.q_qr = out->q_row;
  p.q_sr = out->s_row;
  p.q_qc = out->q_col;
  p.q_sc = out->s_col;
  p.q_kb_col = R / 32;
  GemmOperand a{Aq, 0, 0, 0}, b{Bq, 0, 0, 0};
  switch (op) {
    case MOE_GEMM_FWD1_SWIGLU:
      a = {Aq, R, d, d};
      b = {Bq, (int64_t)E * 2 * F, d, d};
      p.K = d; p.N = F; p.b_rows_per_group = 2 * F; p.ldc = 2 * F;
      p.sA_ld = d / 128; p.sB_ld = d / 128;
      p.q_kb_row = F / 32;
      return launch_gemm(GK_FWD1_SWIGLU_Q, 1, 128, a, b, p, s);
    case MOE_GEMM_DGRAD2_SWIGLU:
      MOE_REQUIRE(aux && aligned16(aux), MOE_ERR_INVALID_ARG);
      a = {Aq, R, d, d};
      b = {Bq, (int64_t)E * d, F, F};
      p.K = d; p.N = F; p.b_rows_per_group = d; p.aux = aux; p.ldaux = 2 * F; p.ldc = 2 * F;
      p.sA_ld = d / 128; p.sB_ld = (int64_t)E * d / 128;
      p.q_kb_row = 2 * F / 32;
      return launch_gemm(GK_DGRAD2_SWIGLU_Q, 1, 128, a, b, p, s);
    default:
      return MOE_ERR_INVALID_ARG;
  }
}

bool operand_ok(const moe_mxfp8_operand_t* o) {
  return o && o->q_row && o->s_row && o->q_col && o->s_col && aligned16(o->q_row) &&
         aligned16(o->q_col) && ((reinterpret_cast<uintptr_t>(o->s_row) & 3u) == 0);
}

int router_logits_impl(const moe_config_t* c, const void* x, const void* Wr, const float* bias,
                       float* logits, void* ws, cudaStream_t s) {
  GemmParams p = base_params(c, ws);
  p.counts = nullptr;
  p.M = c->T; p.K = c->d; p.N = c->E; p.b_rows_per_group = 0;
  p.C = logits; p.ldc = c->E; p.bias = bias;
  GemmOperand a{x, c->T, c->d, c->d}, b{Wr, c->E, c->d, c->d};
  return launch_gemm(GK_ROUTER, es_of(c), c->E <= 128 ? 128 : 256, a, b, p, s);
}

int router_wgrad_impl(const moe_config_t* c, const void* dlogits, const void* x, void* dWr, void* ws,
                      cudaStream_t s) {
  GemmParams p = base_params(c, ws);
  p.counts = nullptr;
  p.M = c->E; p.N = c->d; p.K = c->T;
  p.ldc = c->d;
  GemmOperand a{dlogits, c->T, c->E, c->E}, b{x, c->T, c->d, c->d};
  const int bn = c->d >= 256 ? 256 : 128;
  const RouterSplit rs = router_split(c);
  if (rs.n < 2) {
    p.C = dWr;
    return launch_gemm(GK_WGRAD, es_of(c), bn, a, b, p, s);
  }
  float* part = reinterpret_cast<float*>(static_cast<char*>(ws) + ws_layout(c).rpart);
  p.C = part;
  p.ksplit = rs.rows;
  p.c_group_rows = rs.slab_rows;
  MOE_TRY(launch_gemm(GK_WGRAD_SPLIT, es_of(c), bn, a, b, p, s));
  return launch_split_reduce(part, rs.n, (int64_t)c->E * c->d, (int64_t)rs.slab_rows * c->d, dWr,
                             es_of(c) == 2, s);
}

bool router_shape_ok(const moe_config_t* c) {
  // the dense score-gradient [T,E] is a TMA operand: its rows must be 16-byte multiples
  return ((size_t)c->E * es_of(c)) % 16 == 0;
}

}  // namespace

extern "C" {

const char* moe_version(void) { return "moe_b200 0.1 (sm_100a)"; }

uint64_t moe_launch_count(void) { return moe::g_launches.load(std::memory_order_relaxed); }

int64_t moe_max_rows(const moe_config_t* cfg) {
  if (check_cfg(cfg) != MOE_OK) return 0;
  return max_rows_of(cfg);
}

int moe_workspace_size(const moe_config_t* cfg, size_t* bytes) {
  MOE_TRY(check_cfg(cfg));
  MOE_REQUIRE(bytes, MOE_ERR_INVALID_ARG);
  *bytes = ws_layout(cfg).total;
  return MOE_OK;
}

int moe_get_error(const void* ws, uint32_t* flags, void* stream) {
  MOE_REQUIRE(ws && flags, MOE_ERR_INVALID_ARG);
  if (cudaMemcpyAsync(flags, ws, sizeof(uint32_t), cudaMemcpyDeviceToHost, S(stream)) != cudaSuccess)
    return MOE_ERR_CUDA;
  return cudaStreamSynchronize(S(stream)) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

int moe_clear_error(void* ws, void* stream) {
  MOE_REQUIRE(ws, MOE_ERR_INVALID_ARG);
  return cudaMemsetAsync(ws, 0, sizeof(uint32_t), S(stream)) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

int moe_router_logits(const moe_config_t* cfg, const void* x, const void* W_r, const float* bias,
                      float* logits, void* ws, size_t ws_bytes, void* stream) {
  MOE_TRY(check_cfg(cfg));
  MOE_TRY(check_ws(cfg, ws, ws_bytes));
  MOE_REQUIRE(cfg->dtype != MOE_DTYPE_MXFP8, MOE_ERR_UNSUPPORTED);
  MOE_REQUIRE(x && W_r && logits, MOE_ERR_INVALID_ARG);
  MOE_REQUIRE(aligned16(x) && aligned16(W_r) && aligned16(logits), MOE_ERR_INVALID_ARG);
  return router_logits_impl(cfg, x, W_r, bias, logits, ws, S(stream));
}

int moe_route_topk(const moe_config_t* cfg, const float* logits, const float* bias, int32_t* idx,
                   float* gates, void* ws, size_t ws_bytes, void* stream) {
  MOE_TRY(check_cfg(cfg));
  MOE_TRY(check_ws(cfg, ws, ws_bytes));
  MOE_REQUIRE(logits && idx && gates, MOE_ERR_INVALID_ARG);
  return launch_topk(logits, bias, cfg->T, cfg->E, cfg->k, cfg->renorm, idx, gates, err_of(ws),
                     S(stream));
}

int moe_route_metadata(const moe_config_t* cfg, const int32_t* idx, int32_t* counts,
                       int32_t* offsets, int32_t* poff, int32_t* perm, int32_t* prow,
                       int32_t* row_token, void* ws, size_t ws_bytes, void* stream) {
  MOE_TRY(check_cfg(cfg));
  MOE_TRY(check_ws(cfg, ws, ws_bytes));
  MOE_REQUIRE(idx && counts && offsets && poff && perm && prow && row_token, MOE_ERR_INVALID_ARG);
  const WsLayout L = ws_layout(cfg);
  int32_t* hist = reinterpret_cast<int32_t*>(static_cast<char*>(ws) + L.hist);
  return launch_metadata(idx, cfg->T, cfg->E, cfg->k, group_align(cfg->dtype), max_rows_of(cfg),
                         counts, offsets, poff, perm, prow, row_token, hist, err_of(ws), S(stream));
}

int moe_dispatch(const moe_config_t* cfg, const void* x, const int32_t* prow, const int32_t* counts,
                 const int32_t* poff, void* x_perm, void* stream) {
  MOE_TRY(check_cfg(cfg));
  MOE_REQUIRE(x && prow && counts && poff && x_perm, MOE_ERR_INVALID_ARG);
  MOE_REQUIRE(aligned16(x) && aligned16(x_perm), MOE_ERR_INVALID_ARG);
  return launch_dispatch(x, prow, counts, poff, x_perm, cfg->T, cfg->k, cfg->E, cfg->d * es_of(cfg),
                         max_rows_of(cfg), S(stream));
}

int moe_combine(const moe_config_t* cfg, const void* y, const float* gates, const int32_t* prow,
                void* out, void* stream) {
  MOE_TRY(check_cfg(cfg));
  MOE_REQUIRE(y && gates && prow && out, MOE_ERR_INVALID_ARG);
  MOE_REQUIRE(aligned16(y) && aligned16(out), MOE_ERR_INVALID_ARG);
  return launch_combine(y, gates, prow, out, cfg->T, cfg->k, cfg->d * es_of(cfg), es_of(cfg) == 2,
                        max_rows_of(cfg), S(stream));
}

int moe_combine_bwd(const moe_config_t* cfg, const void* dout, const void* y, const float* gates,
                    const int32_t* prow, const int32_t* idx, const int32_t* counts,
                    const int32_t* poff, void* dy, float* dgates, float* dlsel, void* dlogits,
                    void* stream) {
  MOE_TRY(check_cfg(cfg));
  MOE_REQUIRE(dout && y && gates && prow && counts && poff && dy && dgates, MOE_ERR_INVALID_ARG);
  MOE_REQUIRE(aligned16(dout) && aligned16(y) && aligned16(dy), MOE_ERR_INVALID_ARG);
  MOE_REQUIRE(!dlogits || (dlsel && idx), MOE_ERR_INVALID_ARG);
  MOE_REQUIRE(!dlsel || cfg->renorm == 1, MOE_ERR_UNSUPPORTED);
  return launch_combine_bwd(dout, y, gates, prow, idx, counts, poff, dy, dgates, dlsel, dlogits,
                            cfg->T, cfg->k, cfg->E, cfg->d * es_of(cfg), es_of(cfg) == 2,
                            max_rows_of(cfg), S(stream));
}

int moe_token_reduce(const moe_config_t* cfg, const void* dx_perm, const int32_t* prow,
                     const float* dlsel, const int32_t* idx, const void* W_r, void* dx, void* stream) {
  MOE_TRY(check_cfg(cfg));
  MOE_REQUIRE(dx_perm && prow && dx, MOE_ERR_INVALID_ARG);
  MOE_REQUIRE(aligned16(dx_perm) && aligned16(dx) && (!W_r || aligned16(W_r)), MOE_ERR_INVALID_ARG);
  return launch_token_reduce(dx_perm, prow, dlsel, idx, W_r, dx, cfg->T, cfg->k, cfg->E,
                             cfg->d * es_of(cfg), es_of(cfg) == 2, max_rows_of(cfg), S(stream));
}

int moe_grouped_gemm(const moe_config_t* cfg, int op, const void* A, const void* B, void* C, void* C2,
                     const void* aux, const int32_t* counts, const int32_t* poff, void* ws,
                     size_t ws_bytes, void* stream) {
  MOE_TRY(check_cfg(cfg));
  MOE_TRY(check_ws(cfg, ws, ws_bytes));
  MOE_REQUIRE(cfg->dtype != MOE_DTYPE_MXFP8, MOE_ERR_UNSUPPORTED);
  MOE_REQUIRE(A && B && (C || op == MOE_GEMM_FWD1_SWIGLU) && counts && poff, MOE_ERR_INVALID_ARG);
  MOE_REQUIRE(aligned16(A) && aligned16(B) && (!C || aligned16(C)) && (!C2 || aligned16(C2)),
              MOE_ERR_INVALID_ARG);
  return gemm_op(cfg, op, A, B, C, C2, aux, counts, poff, ws, S(stream));
}

int moe_quantize_mxfp8(const void* src, int64_t rows, int cols, int mode, int64_t G, uint8_t* q,
                       uint8_t* s, void* stream) {
  MOE_REQUIRE(src && q && s && rows >= 1 && cols >= 1, MOE_ERR_INVALID_ARG);
  MOE_REQUIRE(aligned16(src), MOE_ERR_INVALID_ARG);
  const bool q16 = aligned16(q), q8 = (reinterpret_cast<uintptr_t>(q) & 7u) == 0;
  switch (mode) {
    case MOE_QUANT_ROW: MOE_REQUIRE(cols % 32 == 0 && q16, MOE_ERR_INVALID_ARG); break;
    case MOE_QUANT_COL: MOE_REQUIRE(rows % 32 == 0 && cols % 8 == 0 && q8, MOE_ERR_INVALID_ARG); break;
    case MOE_QUANT_ROW_TILED: MOE_REQUIRE(rows % 128 == 0 && cols % 128 == 0 && q16, MOE_ERR_INVALID_ARG); break;
    case MOE_QUANT_COL_TILED: MOE_REQUIRE(rows % 128 == 0 && cols % 128 == 0 && q8, MOE_ERR_INVALID_ARG); break;
    case MOE_QUANT_ROW_TILED_GATEUP:
      MOE_REQUIRE(G >= 64 && G % 64 == 0 && rows % (2 * G) == 0 && cols % 128 == 0 && q16,
                  MOE_ERR_INVALID_ARG);
      break;
    default: return MOE_ERR_INVALID_ARG;
  }
  return launch_quantize(src, rows, cols, mode, G, q, s, S(stream));
}

int moe_quantize_mxfp8_rowcol(const void* src, int64_t rows, int cols, uint8_t* q_row, uint8_t* s_row,
                              uint8_t* q_col, uint8_t* s_col, void* stream) {
  MOE_REQUIRE(src && q_row && s_row && q_col && s_col && rows >= 1 && cols >= 1, MOE_ERR_INVALID_ARG);
  MOE_REQUIRE(rows % 128 == 0 && cols % 128 == 0, MOE_ERR_INVALID_ARG);
  const auto a8 = [](const void* q) { return (reinterpret_cast<uintptr_t>(q) & 7u) == 0; };
  MOE_REQUIRE(aligned16(src) && a8(q_row) && aligned16(q_col), MOE_ERR_INVALID_ARG);
  return launch_quantize_rowcol(src, rows, cols, q_row, s_row, q_col, s_col, S(stream));
}

int moe_grouped_gemm_mxfp8(const moe_config_t* cfg, int op, const uint8_t* Aq, const uint8_t* As,
                           const uint8_t* Bq, const uint8_t* Bs, void* C, void* C2, const void* aux,
                           const int32_t* counts, const int32_t* poff, void* ws, size_t ws_bytes,
                           void* stream) {
  MOE_TRY(check_cfg(cfg));
  MOE_TRY(check_ws(cfg, ws, ws_bytes));
  MOE_REQUIRE(cfg->dtype == MOE_DTYPE_MXFP8, MOE_ERR_INVALID_ARG);
  MOE_REQUIRE(cfg->d % 128 == 0, MOE_ERR_UNSUPPORTED);
  MOE_REQUIRE(Aq && As && Bq && Bs && C && counts && poff, MOE_ERR_INVALID_ARG);
  MOE_REQUIRE(aligned16(Aq) && aligned16(Bq) && aligned16(C) && (!C2 || aligned16(C2)),
              MOE_ERR_INVALID_ARG);
  return gemm_op_mx(cfg, op, Aq, As, Bq, Bs, C, C2, aux, counts, poff, ws, S(stream));
}

int moe_dispatch_mxfp8(const moe_config_t* cfg, const void* x, const int32_t* row_token,
                       const int32_t* poff, const moe_mxfp8_operand_t* out, void* stream) {
  MOE_TRY(check_cfg(cfg));
  MOE_REQUIRE(cfg->dtype == MOE_DTYPE_MXFP8, MOE_ERR_INVALID_ARG);
  MOE_REQUIRE(cfg->d % 128 == 0, MOE_ERR_UNSUPPORTED);
  MOE_REQUIRE(x && row_token && poff && operand_ok(out) && aligned16(x), MOE_ERR_INVALID_ARG);
  return launch_dispatch_quant(x, row_token, poff + cfg->E, cfg->k, max_rows_of(cfg), cfg->d,
                               out->q_row, out->s_row, out->q_col, out->s_col, S(stream));
}

int moe_combine_bwd_mxfp8(const moe_config_t* cfg, const void* dout, const void* y, const float* gates,
                          const int32_t* row_token, const int32_t* poff, float* dgates,
                          const moe_mxfp8_operand_t* dy, void* stream) {
  MOE_TRY(check_cfg(cfg));
  MOE_REQUIRE(cfg->dtype == MOE_DTYPE_MXFP8, MOE_ERR_INVALID_ARG);
  MOE_REQUIRE(cfg->d % 128 == 0, MOE_ERR_UNSUPPORTED);
  MOE_REQUIRE(dout && y && gates && row_token && poff && dgates && operand_ok(dy), MOE_ERR_INVALID_ARG);
  MOE_REQUIRE(aligned16(dout) && aligned16(y), MOE_ERR_INVALID_ARG);
  return launch_combine_bwd_quant(dout, y, gates, row_token, poff + cfg->E, cfg->k, max_rows_of(cfg),
                                  cfg->d, dgates, dy->q_row, dy->s_row, dy->q_col, dy->s_col,
                                  S(stream));
}

int moe_grouped_gemm_mxfp8_quant(const moe_config_t* cfg, int op, const uint8_t* Aq, const uint8_t* As,
                                 const uint8_t* Bq, const uint8_t* Bs, void* C, const void* aux,
                                 const moe_mxfp8_operand_t* out, const int32_t* counts,
                                 const int32_t* poff, void* ws, size_t ws_bytes, void* stream) {
  MOE_TRY(check_cfg(cfg));
  MOE_TRY(check_ws(cfg, ws, ws_bytes));
  MOE_REQUIRE(cfg->dtype == MOE_DTYPE_MXFP8, MOE_ERR_INVALID_ARG);
  MOE_REQUIRE(cfg->d % 128 == 0, MOE_ERR_UNSUPPORTED);
  MOE_REQUIRE(op == MOE_GEMM_FWD1_SWIGLU || op == MOE_GEMM_DGRAD2_SWIGLU, MOE_ERR_INVALID_ARG);
  MOE_REQUIRE(Aq && As && Bq && Bs && counts && poff && operand_ok(out), MOE_ERR_INVALID_ARG);
  MOE_REQUIRE(op != MOE_GEMM_FWD1_SWIGLU || (C && aligned16(C)), MOE_ERR_INVALID_ARG);
  MOE_REQUIRE(aligned16(Aq) && aligned16(Bq), MOE_ERR_INVALID_ARG);
  return gemm_op_mx_quant(cfg, op, Aq, As, Bq, Bs, op == MOE_GEMM_FWD1_SWIGLU ? C : nullptr, aux, out,
                          counts, poff, ws, S(stream));
}

int moe_router_wgrad(const moe_config_t* cfg, const void* dlogits, const void* x, void* dW_r, void* ws,
                     size_t ws_bytes, void* stream) {
  MOE_TRY(check_cfg(cfg));
  MOE_TRY(check_ws(cfg, ws, ws_bytes));
  MOE_REQUIRE(cfg->dtype != MOE_DTYPE_MXFP8, MOE_ERR_UNSUPPORTED);
  MOE_REQUIRE(dlogits && x && dW_r, MOE_ERR_INVALID_ARG);
  MOE_REQUIRE(aligned16(dlogits) && aligned16(x) && aligned16(dW_r), MOE_ERR_INVALID_ARG);
  MOE_REQUIRE(router_shape_ok(cfg), MOE_ERR_UNSUPPORTED);
  return router_wgrad_impl(cfg, dlogits, x, dW_r, ws, S(stream));
}

int moe_layer_fwd(const moe_config_t* cfg, const moe_weights_t* w, const void* x, const float* bias,
                  void* out, moe_saved_t* sv, void* ws, size_t ws_bytes, void* stream) {
  MOE_TRY(check_cfg(cfg));
  MOE_TRY(check_ws(cfg, ws, ws_bytes));
  MOE_REQUIRE(cfg->dtype != MOE_DTYPE_MXFP8, MOE_ERR_UNSUPPORTED);
  MOE_REQUIRE(w && sv && x && out && w->W13 && w->W2, MOE_ERR_INVALID_ARG);
  // sv->h13 == NULL selects activation recompute: h13 is not kept, the backward regenerates it
  MOE_REQUIRE(sv->idx && sv->gates && sv->counts && sv->offsets && sv->poff && sv->perm && sv->prow &&
                  sv->row_token && sv->x_perm && sv->a && sv->y,
              MOE_ERR_INVALID_ARG);
  MOE_REQUIRE(aligned16(x) && aligned16(out) && aligned16(w->W13) && aligned16(w->W2) &&
                  aligned16(sv->x_perm) && (!sv->h13 || aligned16(sv->h13)) && aligned16(sv->a) &&
                  aligned16(sv->y),
              MOE_ERR_INVALID_ARG);
  cudaStream_t s = S(stream);
  if (w->W_r) {
    MOE_REQUIRE(sv->logits && aligned16(w->W_r) && aligned16(sv->logits), MOE_ERR_INVALID_ARG);
    MOE_TRY(router_logits_impl(cfg, x, w->W_r, bias, sv->logits, ws, s));
    MOE_TRY(launch_topk(sv->logits, nullptr, cfg->T, cfg->E, cfg->k, cfg->renorm, sv->idx, sv->gates,
                        err_of(ws), s));
  }
  const WsLayout L = ws_layout(cfg);
  int32_t* hist = reinterpret_cast<int32_t*>(static_cast<char*>(ws) + L.hist);
  MOE_TRY(launch_metadata(sv->idx, cfg->T, cfg->E, cfg->k, group_align(cfg->dtype), max_rows_of(cfg),
                          sv->counts, sv->offsets, sv->poff, sv->perm, sv->prow, sv->row_token, hist,
                          err_of(ws), s));
  MOE_TRY(launch_dispatch(x, sv->prow, sv->counts, sv->poff, sv->x_perm, cfg->T, cfg->k, cfg->E,
                          cfg->d * es_of(cfg), max_rows_of(cfg), s));
  MOE_TRY(gemm_op(cfg, MOE_GEMM_FWD1_SWIGLU, sv->x_perm, w->W13, sv->h13, sv->a, nullptr, sv->counts,
                  sv->poff, ws, s));
  MOE_TRY(gemm_op(cfg, MOE_GEMM_FWD2, sv->a, w->W2, sv->y, nullptr, nullptr, sv->counts, sv->poff, ws,
                  s));
  return launch_combine(sv->y, sv->gates, sv->prow, out, cfg->T, cfg->k, cfg->d * es_of(cfg),
                        es_of(cfg) == 2, max_rows_of(cfg), s);
}

int moe_layer_bwd(const moe_config_t* cfg, const moe_weights_t* w, const moe_saved_t* sv,
                  const void* x, const void* dout, void* dx, moe_grads_t* g, void* ws,
                  size_t ws_bytes, void* stream) {
  MOE_TRY(check_cfg(cfg));
  MOE_TRY(check_ws(cfg, ws, ws_bytes));
  MOE_REQUIRE(cfg->dtype != MOE_DTYPE_MXFP8, MOE_ERR_UNSUPPORTED);
  MOE_REQUIRE(w && sv && g && x && dout && dx && w->W13 && w->W2, MOE_ERR_INVALID_ARG);
  MOE_REQUIRE(g->dW13 && g->dW2 && g->dgates && g->dy && g->dh13 && g->dx_perm, MOE_ERR_INVALID_ARG);
  MOE_REQUIRE(aligned16(dout) && aligned16(dx) && aligned16(g->dW13) && aligned16(g->dW2) &&
                  aligned16(g->dy) && aligned16(g->dh13) && aligned16(g->dx_perm),
              MOE_ERR_INVALID_ARG);
  const bool router = w->W_r != nullptr;
  if (router) {
    MOE_REQUIRE(cfg->renorm == 1, MOE_ERR_UNSUPPORTED);
    MOE_REQUIRE(router_shape_ok(cfg), MOE_ERR_UNSUPPORTED);
    MOE_REQUIRE(g->dW_r && aligned16(g->dW_r), MOE_ERR_INVALID_ARG);
  }
  cudaStream_t s = S(stream);
  const WsLayout L = ws_layout(cfg);
  float* dlsel = router ? reinterpret_cast<float*>(static_cast<char*>(ws) + L.dlsel) : nullptr;
  void* dlog = router ? static_cast<void*>(static_cast<char*>(ws) + L.dlogits) : nullptr;
  const int rb = cfg->d * es_of(cfg);
  const bool bf = es_of(cfg) == 2;
  MOE_TRY(launch_combine_bwd(dout, sv->y, sv->gates, sv->prow, sv->idx, sv->counts, sv->poff, g->dy,
                             g->dgates, dlsel, dlog, cfg->T, cfg->k, cfg->E, rb, bf, max_rows_of(cfg),
                             s));
  // Activation recompute (the forward kept no h13): GEMM1 regenerates h13 into the dh13 buffer and a
  // into saved->a; the SwiGLU-backward GEMM then overwrites h13 with dh13 in place (each element is
  // read and written by the same tile, the read first).
  const void* h13 = sv->h13;
  if (!h13) {
    MOE_TRY(gemm_op(cfg, MOE_GEMM_FWD1_SWIGLU, sv->x_perm, w->W13, g->dh13, sv->a, nullptr, sv->counts,
                    sv->poff, ws, s));
    h13 = g->dh13;
  }
  // The data path first (dgrad2 -> dgrad1 -> token reduce, each reading what the one before it just
  // wrote, partly still in L2), then the two weight gradients.
  MOE_TRY(gemm_op(cfg, MOE_GEMM_DGRAD2_SWIGLU, g->dy, w->W2, g->dh13, nullptr, h13, sv->counts,
                  sv->poff, ws, s));
  MOE_TRY(gemm_op(cfg, MOE_GEMM_DGRAD1, g->dh13, w->W13, g->dx_perm, nullptr, nullptr, sv->counts,
                  sv->poff, ws, s));
  MOE_TRY(launch_token_reduce(g->dx_perm, sv->prow, dlsel, router ? sv->idx : nullptr, w->W_r, dx,
                              cfg->T, cfg->k, cfg->E, rb, bf, max_rows_of(cfg), s));
  MOE_TRY(gemm_op(cfg, MOE_GEMM_WGRAD2, g->dy, sv->a, g->dW2, nullptr, nullptr, sv->counts, sv->poff,
                  ws, s));
  MOE_TRY(gemm_op(cfg, MOE_GEMM_WGRAD1, g->dh13, sv->x_perm, g->dW13, nullptr, nullptr, sv->counts,
                  sv->poff, ws, s));
  if (router) MOE_TRY(router_wgrad_impl(cfg, dlog, x, g->dW_r, ws, s));
  return MOE_OK;
}

int moe_quantize_weights_mxfp8(const moe_config_t* cfg, const moe_weights_t* w,
                               const moe_mxfp8_weights_t* qw, void* stream) {
  MOE_TRY(check_cfg(cfg));
  MOE_REQUIRE(cfg->dtype == MOE_DTYPE_MXFP8, MOE_ERR_INVALID_ARG);
  MOE_REQUIRE(w && qw && w->W13 && w->W2, MOE_ERR_INVALID_ARG);
  MOE_REQUIRE(qw->W13q && qw->W13s && qw->W13tq && qw->W13ts && qw->W2q && qw->W2s && qw->W2tq &&
                  qw->W2ts,
              MOE_ERR_INVALID_ARG);
  const int64_t E = cfg->E, d = cfg->d, F = cfg->F;
  cudaStream_t s = S(stream);
  MOE_TRY(moe_quantize_mxfp8(w->W13, E * 2 * F, (int)d, MOE_QUANT_ROW_TILED, 0, qw->W13q,
                             qw->W13s, s));
  MOE_TRY(moe_quantize_mxfp8(w->W13, E * 2 * F, (int)d, MOE_QUANT_COL_TILED, 0, qw->W13tq, qw->W13ts, s));
  MOE_TRY(moe_quantize_mxfp8(w->W2, E * d, (int)F, MOE_QUANT_ROW_TILED, 0, qw->W2q, qw->W2s, s));
  return moe_quantize_mxfp8(w->W2, E * d, (int)F, MOE_QUANT_COL_TILED, 0, qw->W2tq, qw->W2ts, s);
}

int moe_layer_fwd_mxfp8(const moe_config_t* cfg, const moe_weights_t* w, const moe_mxfp8_weights_t* qw,
                        const void* x, const float* bias, void* out, moe_saved_t* sv,
                        const moe_mxfp8_acts_t* qa, void* ws, size_t ws_bytes, void* stream) {
  MOE_TRY(check_cfg(cfg));
  MOE_TRY(check_ws(cfg, ws, ws_bytes));
  MOE_REQUIRE(cfg->dtype == MOE_DTYPE_MXFP8, MOE_ERR_INVALID_ARG);
  MOE_REQUIRE(cfg->d % 128 == 0, MOE_ERR_UNSUPPORTED);
  MOE_REQUIRE(w && qw && qa && sv && x && out, MOE_ERR_INVALID_ARG);
  MOE_REQUIRE(sv->idx && sv->gates && sv->counts && sv->offsets && sv->poff && sv->perm && sv->prow &&
                  sv->row_token && sv->h13 && sv->y,
              MOE_ERR_INVALID_ARG);
  const moe_mxfp8_operand_t xo{qa->xq, qa->xs, qa->xtq, qa->xts};
  const moe_mxfp8_operand_t ao{qa->aq, qa->as, qa->atq, qa->ats};
  MOE_REQUIRE(operand_ok(&xo) && operand_ok(&ao), MOE_ERR_INVALID_ARG);
  MOE_REQUIRE(aligned16(x) && aligned16(out) && aligned16(sv->h13) && aligned16(sv->y),
              MOE_ERR_INVALID_ARG);
  cudaStream_t s = S(stream);
  const int64_t R = max_rows_of(cfg);
  const int d = cfg->d;
  if (w->W_r) {
    MOE_REQUIRE(sv->logits && aligned16(w->W_r) && aligned16(sv->logits), MOE_ERR_INVALID_ARG);
    moe_config_t rc = *cfg;
    rc.dtype = MOE_DTYPE_BF16;  // the router GEMM runs in bf16
    MOE_TRY(router_logits_impl(&rc, x, w->W_r, bias, sv->logits, ws, s));
    MOE_TRY(launch_topk(sv->logits, nullptr, cfg->T, cfg->E, cfg->k, cfg->renorm, sv->idx, sv->gates,
                        err_of(ws), s));
  }
  const WsLayout L = ws_layout(cfg);
  int32_t* hist = reinterpret_cast<int32_t*>(static_cast<char*>(ws) + L.hist);
  MOE_TRY(launch_metadata(sv->idx, cfg->T, cfg->E, cfg->k, group_align(cfg->dtype), R, sv->counts,
                          sv->offsets, sv->poff, sv->perm, sv->prow, sv->row_token, hist, err_of(ws),
                          s));
  // row-wise dispatch straight into the quantised expert buffers (no bf16 x_perm)
  MOE_TRY(launch_dispatch_quant(x, sv->row_token, sv->poff + cfg->E, cfg->k, R, d, xo.q_row, xo.s_row,
                                xo.q_col, xo.s_col, s));
  // GEMM1 + SwiGLU: h13 in bf16 for the backward, a only as its two quantised forms
  MOE_TRY(gemm_op_mx_quant(cfg, MOE_GEMM_FWD1_SWIGLU, xo.q_row, xo.s_row, qw->W13q, qw->W13s, sv->h13,
                           nullptr, &ao, sv->counts, sv->poff, ws, s));
  MOE_TRY(gemm_op_mx(cfg, MOE_GEMM_FWD2, ao.q_row, ao.s_row, qw->W2q, qw->W2s, sv->y, nullptr, nullptr,
                     sv->counts, sv->poff, ws, s));
  return launch_combine(sv->y, sv->gates, sv->prow, out, cfg->T, cfg->k, d * 2, true, R, s);
}

int moe_layer_bwd_mxfp8(const moe_config_t* cfg, const moe_weights_t* w, const moe_mxfp8_weights_t* qw,
                        const moe_saved_t* sv, const moe_mxfp8_acts_t* qa, const void* x,
                        const void* dout, void* dx, moe_grads_t* g, void* ws, size_t ws_bytes,
                        void* stream) {
  MOE_TRY(check_cfg(cfg));
  MOE_TRY(check_ws(cfg, ws, ws_bytes));
  MOE_REQUIRE(cfg->dtype == MOE_DTYPE_MXFP8, MOE_ERR_INVALID_ARG);
  MOE_REQUIRE(cfg->d % 128 == 0, MOE_ERR_UNSUPPORTED);
  MOE_REQUIRE(w && qw && qa && sv && g && x && dout && dx, MOE_ERR_INVALID_ARG);
  MOE_REQUIRE(g->dW13 && g->dW2 && g->dgates && g->dx_perm, MOE_ERR_INVALID_ARG);
  const moe_mxfp8_operand_t dyo{qa->dyq, qa->dys, qa->dytq, qa->dyts};
  const moe_mxfp8_operand_t dho{qa->dhq, qa->dhs, qa->dhtq, qa->dhts};
  MOE_REQUIRE(operand_ok(&dyo) && operand_ok(&dho) && qa->xtq && qa->xts && qa->atq && qa->ats,
              MOE_ERR_INVALID_ARG);
  MOE_REQUIRE(aligned16(dout) && aligned16(dx) && aligned16(g->dW13) && aligned16(g->dW2) &&
                  aligned16(g->dx_perm) && aligned16(sv->h13) && aligned16(sv->y),
              MOE_ERR_INVALID_ARG);
  const bool router = w->W_r != nullptr;
  moe_config_t rc = *cfg;
  rc.dtype = MOE_DTYPE_BF16;
  if (router) {
    MOE_REQUIRE(cfg->renorm == 1, MOE_ERR_UNSUPPORTED);
    MOE_REQUIRE(router_shape_ok(&rc), MOE_ERR_UNSUPPORTED);
    MOE_REQUIRE(g->dW_r && aligned16(g->dW_r), MOE_ERR_INVALID_ARG);
  }
  cudaStream_t s = S(stream);
  const int64_t R = max_rows_of(cfg);
  const int d = cfg->d;
  const WsLayout L = ws_layout(cfg);
  float* dlsel = router ? reinterpret_cast<float*>(static_cast<char*>(ws) + L.dlsel) : nullptr;
  void* dlog = router ? static_cast<void*>(static_cast<char*>(ws) + L.dlogits) : nullptr;
  // combine backward straight into dy's quantised forms (no bf16 dy), and the gate gradients
  MOE_TRY(launch_combine_bwd_quant(dout, sv->y, sv->gates, sv->row_token, sv->poff + cfg->E, cfg->k, R,
                                   d, g->dgates, dyo.q_row, dyo.s_row, dyo.q_col, dyo.s_col, s));
  if (router)
    MOE_TRY(launch_score_grad(sv->gates, g->dgates, sv->idx, dlsel, dlog, cfg->T, cfg->k, cfg->E,
                              true, s));
  // GEMM2 dgrad + SwiGLU backward: dh13 only as its two quantised forms
  MOE_TRY(gemm_op_mx_quant(cfg, MOE_GEMM_DGRAD2_SWIGLU, dyo.q_row, dyo.s_row, qw->W2tq, qw->W2ts,
                           nullptr, sv->h13, &dho, sv->counts, sv->poff, ws, s));
  MOE_TRY(gemm_op_mx(cfg, MOE_GEMM_WGRAD2, dyo.q_col, dyo.s_col, qa->atq, qa->ats, g->dW2, nullptr,
                     nullptr, sv->counts, sv->poff, ws, s));
  MOE_TRY(gemm_op_mx(cfg, MOE_GEMM_DGRAD1, dho.q_row, dho.s_row, qw->W13tq, qw->W13ts, g->dx_perm,
                     nullptr, nullptr, sv->counts, sv->poff, ws, s));
  MOE_TRY(gemm_op_mx(cfg, MOE_GEMM_WGRAD1, dho.q_col, dho.s_col, qa->xtq, qa->xts, g->dW13, nullptr,
                     nullptr, sv->counts, sv->poff, ws, s));
  MOE_TRY(launch_token_reduce(g->dx_perm, sv->prow, dlsel, router ? sv->idx : nullptr, w->W_r, dx,
                              cfg->T, cfg->k, cfg->E, d * 2, true, R, s));
  if (router) MOE_TRY(router_wgrad_impl(&rc, dlog, x, g->dW_r, ws, s));
  return MOE_OK;
}

// ---- expert parallelism across the GPUs of one node ------------------------------------------------

namespace {
int check_ep(const moe_config_t* cfg, int world) {
  MOE_TRY(check_cfg(cfg));
  MOE_REQUIRE(world >= 1 && world <= kMaxEpRanks, MOE_ERR_INVALID_ARG);
  MOE_REQUIRE(cfg->E % world == 0, MOE_ERR_INVALID_ARG);
  MOE_REQUIRE(cfg->dtype == MOE_DTYPE_BF16, MOE_ERR_UNSUPPORTED);
  return MOE_OK;
}
int64_t ep_rows(const moe_config_t* c, int world) {
  const int64_t EL = c->E / world;
  return ((int64_t)world * c->T * c->k + 31 * EL + 31) / 32 * 32;
}
}  // namespace

int64_t moe_ep_max_rows(const moe_config_t* cfg, int world) {
  if (check_ep(cfg, world) != MOE_OK) return 0;
  const int64_t r = ep_rows(cfg, world);
  return r < (1ll << 31) - 256 ? r : 0;
}

int moe_ep_layout(const moe_config_t* cfg, int rank, int world, const int32_t* all_counts,
                  const int32_t* idx, const int32_t* perm, const int32_t* offsets, int32_t* src_base,
                  int32_t* counts_loc, int32_t* poff_loc, int32_t* dst_row, void* stream) {
  MOE_TRY(check_ep(cfg, world));
  MOE_REQUIRE(rank >= 0 && rank < world, MOE_ERR_INVALID_ARG);
  MOE_REQUIRE(all_counts && idx && perm && offsets && src_base && counts_loc && poff_loc && dst_row,
              MOE_ERR_INVALID_ARG);
  return launch_ep_layout(all_counts, world, cfg->E, rank, idx, perm, offsets,
                          (int64_t)cfg->T * cfg->k, src_base, counts_loc, poff_loc, dst_row, S(stream));
}

int moe_ep_zero_pad(const moe_config_t* cfg, int world, void* buf, const int32_t* counts_loc,
                    const int32_t* poff_loc, void* stream) {
  MOE_TRY(check_ep(cfg, world));
  MOE_REQUIRE(buf && counts_loc && poff_loc && aligned16(buf), MOE_ERR_INVALID_ARG);
  return launch_ep_zero_pad(buf, counts_loc, poff_loc, cfg->E / world, cfg->d * 2, S(stream));
}

int moe_ep_dispatch(const moe_config_t* cfg, int world, const void* x, const int32_t* idx,
                    const int32_t* dst_row, void* const* x_perm_peers, void* stream) {
  MOE_TRY(check_ep(cfg, world));
  MOE_REQUIRE(x && idx && dst_row && x_perm_peers && aligned16(x), MOE_ERR_INVALID_ARG);
  return launch_ep_rows(0, world, cfg->T, cfg->k, cfg->E, cfg->d * 2, ep_rows(cfg, world), x,
                        x_perm_peers, nullptr, nullptr, idx, dst_row, nullptr, nullptr, S(stream));
}

int moe_ep_combine(const moe_config_t* cfg, int world, void* const* y_peers, const float* gates,
                   const int32_t* idx, const int32_t* dst_row, void* out, void* stream) {
  MOE_TRY(check_ep(cfg, world));
  MOE_REQUIRE(y_peers && gates && idx && dst_row && out && aligned16(out), MOE_ERR_INVALID_ARG);
  return launch_ep_rows(1, world, cfg->T, cfg->k, cfg->E, cfg->d * 2, ep_rows(cfg, world), nullptr,
                        y_peers, nullptr, gates, idx, dst_row, out, nullptr, S(stream));
}

int moe_ep_combine_bwd(const moe_config_t* cfg, int world, const void* dout, void* const* y_peers,
                       const float* gates, const int32_t* idx, const int32_t* dst_row,
                       void* const* dy_peers, float* dgates, void* stream) {
  MOE_TRY(check_ep(cfg, world));
  MOE_REQUIRE(dout && y_peers && gates && idx && dst_row && dy_peers && dgates && aligned16(dout),
              MOE_ERR_INVALID_ARG);
  return launch_ep_rows(2, world, cfg->T, cfg->k, cfg->E, cfg->d * 2, ep_rows(cfg, world), dout,
                        y_peers, dy_peers, gates, idx, dst_row, nullptr, dgates, S(stream));
}

int moe_ep_token_reduce(const moe_config_t* cfg, int world, void* const* dx_perm_peers,
                        const int32_t* idx, const int32_t* dst_row, void* dx, void* stream) {
  MOE_TRY(check_ep(cfg, world));
  MOE_REQUIRE(dx_perm_peers && idx && dst_row && dx && aligned16(dx), MOE_ERR_INVALID_ARG);
  return launch_ep_rows(3, world, cfg->T, cfg->k, cfg->E, cfg->d * 2, ep_rows(cfg, world), nullptr,
                        dx_perm_peers, nullptr, nullptr, idx, dst_row, dx, nullptr, S(stream));
}

int moe_test_bounded_wait(void* ws, uint64_t limit_ns, void* stream) {
  MOE_REQUIRE(ws, MOE_ERR_INVALID_ARG);
  return launch_bounded_wait_probe(err_of(ws), limit_ns, S(stream));
}

}  // extern "C"
