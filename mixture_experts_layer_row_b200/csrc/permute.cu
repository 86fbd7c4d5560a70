// Row movement between token order and expert-grouped order, all HBM-bound and written as
// coalesced 16-byte vector loops (one warp per token, every lane moving 16-byte chunks of the row):
//   dispatch      x[t] -> x_perm[prow[t,j]] for j < k, read once and written k times ("row-wise"
//                 placement straight into each expert's contiguous input buffer: bytechap.com, "Como
//                 funciona"; unite.ai, "Parallelismo, precisione e tecniche di memoria"); pad rows 0.
//   combine       out[t] = sum_j g[t,j] y[prow[t,j]]  (a gather: deterministic, no atomics)
//   combine_bwd   dy[prow[t,j]] = g[t,j] dout[t];  dg[t,j] = <dout[t], y[prow[t,j]]> (+ score grads);
//                 its reads are staged in shared memory by bulk copies (three streams per token: the
//                 register-staged loop could not keep enough of them in flight)
//   token_reduce  dx[t] = sum_j dx_perm[prow[t,j]] (+ sum_j dl[t,j] W_r[idx[t,j]])
// Every routed-row pad row (the tail of each expert's 32-aligned group) is written as zero by
// dispatch and combine_bwd so the grouped GEMMs can run whole 32-row blocks. An entry whose padded row
// lies outside [0, max_rows) -- the -1 that the metadata writes for an expert id outside [0,E) -- is
// skipped by every kernel here: nothing is read or written through it.
#include "internal.h"

namespace moe {

namespace {

constexpr int kWarps = 8;  // warps per block = tokens per block
// combine backward with bulk-staged rows: staging per block, and the dynamic shared-memory ceiling
constexpr size_t kCbStageBudget = 60 * 1024;
constexpr size_t kCbSmemMax = 227 * 1024;
static_assert(kWarps * 8 <= 64, "one warp issues a block's routed-row copies, two slots per lane (k <= 8)");

// 16-byte vector <-> floats. BF16: 8 values per vector; FP32: 4.
template <bool BF16>
struct Vec;
template <>
struct Vec<true> {
  static constexpr int N = 8;
  __device__ static void unpack(const uint4& v, float (&f)[8]) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      f[2 * i] = bf16lo(w[i]);
      f[2 * i + 1] = bf16hi(w[i]);
    }
  }
  __device__ static uint4 pack(const float (&f)[8]) {
    return make_uint4(pack_bf16(f[0], f[1]), pack_bf16(f[2], f[3]), pack_bf16(f[4], f[5]),
                      pack_bf16(f[6], f[7]));
  }
};
template <>
struct Vec<false> {
  static constexpr int N = 4;
  __device__ static void unpack(const uint4& v, float (&f)[4]) {
    f[0] = __uint_as_float(v.x);
    f[1] = __uint_as_float(v.y);
    f[2] = __uint_as_float(v.z);
    f[3] = __uint_as_float(v.w);
  }
  __device__ static uint4 pack(const float (&f)[4]) {
    return make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]),
                      __float_as_uint(f[3]));
  }
};

// Padded row of slot `lane` of token t, or -1 when the slot is unused or its row is out of range.
__device__ __forceinline__ int slot_row(const int32_t* prow, int t, int k, int lane, int max_rows) {
  if (lane >= k) return -1;
  const int r = prow[(size_t)t * k + lane];
  return (r >= 0 && r < max_rows) ? r : -1;
}

// A load that is always issued: a slot without a row (-1) reads row 0 and gets zeros instead, so the
// k loads of a step stay unconditional (predicating them on the row was measured 30 % slower in
// combine).
__device__ __forceinline__ uint4 ldg_stream(const uint4* p);
__device__ __forceinline__ uint4 ldg_row(const uint4* base, int row, int vpr, int v) {
  uint4 w = ldg_stream(base + (size_t)(row < 0 ? 0 : row) * vpr + v);
  if (row < 0) w = make_uint4(0u, 0u, 0u, 0u);
  return w;
}

__device__ __forceinline__ uint4 ldg_stream(const uint4* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// Zero the pad rows [poff[e]+counts[e], poff[e+1]) of one expert; called by whole blocks.
__device__ __forceinline__ void zero_pad_rows(uint4* buf, int e, const int32_t* counts,
                                              const int32_t* poff, int vpr) {
  const int r0 = poff[e] + counts[e], r1 = poff[e + 1];
  const int64_t n = (int64_t)(r1 - r0) * vpr;
  uint4* base = buf + (size_t)r0 * vpr;
  for (int64_t i = threadIdx.x; i < n; i += blockDim.x) base[i] = make_uint4(0, 0, 0, 0);
}

__global__ void __launch_bounds__(kWarps * 32) dispatch_kernel(
    const uint4* __restrict__ x, const int32_t* __restrict__ prow, const int32_t* __restrict__ counts,
    const int32_t* __restrict__ poff, uint4* __restrict__ xp, int T, int k, int vpr, int tok_blocks,
    int max_rows) {
  pdl_enter();  // wait for the previous kernel before any global access
  if ((int)blockIdx.x >= tok_blocks) {
    zero_pad_rows(xp, blockIdx.x - tok_blocks, counts, poff, vpr);
    return;
  }
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * kWarps + (threadIdx.x >> 5);
  if (t >= T) return;
  const int myrow = slot_row(prow, t, k, lane, max_rows);
  int rows[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) rows[j] = __shfl_sync(0xffffffffu, myrow, j);
  const uint4* src = x + (size_t)t * vpr;
  // eight loads of the row in flight per lane before any of their k stores (the loads are the only
  // waits here; a 4-KB bf16 row is one batch): 32.9 -> 30.3 us against the interleaved loop
  constexpr int kBatch = 8;
  for (int v0 = lane; v0 < vpr; v0 += 32 * kBatch) {
    uint4 val[kBatch];
#pragma unroll
    for (int u = 0; u < kBatch; ++u)
      val[u] = (v0 + 32 * u < vpr) ? ldg_stream(src + v0 + 32 * u) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      if (v0 + 32 * u < vpr) {
#pragma unroll
        for (int j = 0; j < 8; ++j)
          if (j < k && rows[j] >= 0) xp[(size_t)rows[j] * vpr + v0 + 32 * u] = val[u];
      }
    }
  }
}

template <bool BF16>
__global__ void __launch_bounds__(kWarps * 32) combine_kernel(const uint4* __restrict__ y,
                                                              const float* __restrict__ gates,
                                                              const int32_t* __restrict__ prow,
                                                              uint4* __restrict__ out, int T, int k,
                                                              int vpr, int max_rows) {
  pdl_enter();  // wait for the previous kernel before any global access
  using V = Vec<BF16>;
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * kWarps + (threadIdx.x >> 5);
  if (t >= T) return;
  const int myrow = slot_row(prow, t, k, lane, max_rows);
  const float myg = lane < k ? gates[(size_t)t * k + lane] : 0.f;
  int rows[8];
  float g[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    rows[j] = __shfl_sync(0xffffffffu, myrow, j);
    g[j] = __shfl_sync(0xffffffffu, myg, j);
  }
#pragma unroll 2
  for (int v = lane; v < vpr; v += 32) {
    float acc[V::N];
#pragma unroll
    for (int i = 0; i < V::N; ++i) acc[i] = 0.f;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      if (j < k) {
        float f[V::N];
        V::unpack(ldg_row(y, rows[j], vpr, v), f);
#pragma unroll
        for (int i = 0; i < V::N; ++i) acc[i] = fmaf(g[j], f[i], acc[i]);
      }
    }
    out[(size_t)t * vpr + v] = V::pack(acc);
  }
}

// The end of a token's combine backward, once each lane holds its partial dot products with the k
// rows: dgates[t,j] = <dout[t], y[row_j]>, and for a learned router the score gradients dl_j =
// g_j (dg_j - sum_i g_i dg_i) and the dense row dlogits[t, e] (act dtype), zero except at the chosen
// experts.
template <bool BF16>
__device__ __forceinline__ void combine_bwd_finish(float (&dot)[8], const float (&g)[8], int t, int k,
                                                   int E, int lane, const int32_t* __restrict__ idx,
                                                   float* __restrict__ dgates, float* __restrict__ dlsel,
                                                   void* __restrict__ dlogits) {
#pragma unroll
  for (int j = 0; j < 8; ++j) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) dot[j] += __shfl_xor_sync(0xffffffffu, dot[j], off);
  }
  float s = 0.f;
#pragma unroll
  for (int j = 0; j < 8; ++j)
    if (j < k) s = fmaf(g[j], dot[j], s);
  float mydl = 0.f;
  int mye = -1;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    if (j < k && lane == j) {
      dgates[(size_t)t * k + j] = dot[j];
      mydl = g[j] * (dot[j] - s);
      if (dlsel) dlsel[(size_t)t * k + j] = mydl;
      mye = idx ? idx[(size_t)t * k + j] : -1;
    }
  }
  if (dlogits) {
    int ej[8];
    float dj[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      ej[j] = __shfl_sync(0xffffffffu, mye, j);
      dj[j] = __shfl_sync(0xffffffffu, mydl, j);
    }
    for (int e = lane; e < E; e += 32) {
      float val = 0.f;
#pragma unroll
      for (int j = 0; j < 8; ++j)
        if (j < k && ej[j] == e) val = dj[j];
      if (BF16)
        reinterpret_cast<__nv_bfloat16*>(dlogits)[(size_t)t * E + e] = __float2bfloat16_rn(val);
      else
        reinterpret_cast<float*>(dlogits)[(size_t)t * E + e] = val;
    }
  }
}

template <bool BF16>
// 64 registers at most: four blocks (32 warps) per SM keep enough loads in flight
__global__ void __launch_bounds__(kWarps * 32, 4) combine_bwd_kernel(
    const uint4* __restrict__ dout, const uint4* __restrict__ y, const float* __restrict__ gates,
    const int32_t* __restrict__ prow, const int32_t* __restrict__ idx,
    const int32_t* __restrict__ counts, const int32_t* __restrict__ poff, uint4* __restrict__ dy,
    float* __restrict__ dgates, float* __restrict__ dlsel, void* __restrict__ dlogits, int T, int k,
    int E, int vpr, int tok_blocks, int max_rows) {
  pdl_enter();  // wait for the previous kernel before any global access
  using V = Vec<BF16>;
  if ((int)blockIdx.x >= tok_blocks) {
    zero_pad_rows(dy, blockIdx.x - tok_blocks, counts, poff, vpr);
    return;
  }
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * kWarps + (threadIdx.x >> 5);
  if (t >= T) return;
  const int myrow = slot_row(prow, t, k, lane, max_rows);
  const float myg = lane < k ? gates[(size_t)t * k + lane] : 0.f;
  int rows[8];
  float g[8], dot[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    rows[j] = __shfl_sync(0xffffffffu, myrow, j);
    g[j] = __shfl_sync(0xffffffffu, myg, j);
    dot[j] = 0.f;
  }
#pragma unroll 1
  for (int v = lane; v < vpr; v += 32) {
    float fd[V::N];
    V::unpack(ldg_stream(dout + (size_t)t * vpr + v), fd);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      if (j < k) {
        float fy[V::N], o[V::N];
        V::unpack(ldg_row(y, rows[j], vpr, v), fy);
#pragma unroll
        for (int i = 0; i < V::N; ++i) {
          dot[j] = fmaf(fd[i], fy[i], dot[j]);
          o[i] = g[j] * fd[i];
        }
        if (rows[j] >= 0) dy[(size_t)rows[j] * vpr + v] = V::pack(o);
      }
    }
  }
  combine_bwd_finish<BF16>(dot, g, t, k, E, lane, idx, dgates, dlsel, dlogits);
}

// The same combine backward with the reads staged in shared memory by bulk copies. One thread of the
// block copies the block's dout rows (one copy: they are consecutive) and every routed y row of its
// tokens, all completing on one mbarrier; then one warp per token computes from shared memory. Data
// in flight no longer occupies registers (a register-staged 16-byte load holds four until it lands),
// so with three blocks per SM about twice as many bytes of the gather are in flight, and one block
// computes while the others' copies land (60 KB per block measured best: 62 us against 65 us for
// 100 KB and 81 us for 150 KB, e128 bf16 shapes).
template <bool BF16>
__global__ void __launch_bounds__(kWarps * 32) combine_bwd_bulk_kernel(
    const uint4* __restrict__ dout, const uint4* __restrict__ y, const float* __restrict__ gates,
    const int32_t* __restrict__ prow, const int32_t* __restrict__ idx,
    const int32_t* __restrict__ counts, const int32_t* __restrict__ poff, uint4* __restrict__ dy,
    float* __restrict__ dgates, float* __restrict__ dlsel, void* __restrict__ dlogits, int T, int k,
    int E, int vpr, int tok_blocks, int max_rows, int tpb) {
  pdl_enter();  // wait for the previous kernel before any global access
  using V = Vec<BF16>;
  if ((int)blockIdx.x >= tok_blocks) {
    zero_pad_rows(dy, blockIdx.x - tok_blocks, counts, poff, vpr);
    return;
  }
  extern __shared__ __align__(128) uint8_t cb_smem[];
  uint64_t* bar = reinterpret_cast<uint64_t*>(cb_smem);
  uint4* sdout = reinterpret_cast<uint4*>(cb_smem + 128);  // [tpb][vpr]
  uint4* sy = sdout + (size_t)tpb * vpr;                    // [tpb][k][vpr], slot-major per token
  const int t0 = blockIdx.x * tpb;
  const int nt = min(tpb, T - t0);
  const uint32_t rb = (uint32_t)vpr * 16u;
  if (threadIdx.x == 0) {
    mbar_init(bar, 1);
    fence_barrier_init();
  }
  __syncthreads();
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (w == 0) {
    // lane i owns routed slots i and i + 32 of the block (tpb * k <= 64): one parallel read of the
    // rows, a ballot for the byte count, and each lane issues its own copies once lane 0 has armed
    // the barrier
    const int ns = nt * k;
    int r0 = lane < ns ? prow[(size_t)t0 * k + lane] : -1;
    int r1 = lane + 32 < ns ? prow[(size_t)t0 * k + lane + 32] : -1;
    if (!(r0 >= 0 && r0 < max_rows)) r0 = -1;
    if (!(r1 >= 0 && r1 < max_rows)) r1 = -1;
    const int nvalid = __popc(__ballot_sync(0xffffffffu, r0 >= 0)) + __popc(__ballot_sync(0xffffffffu, r1 >= 0));
    if (lane == 0) {
      mbar_arrive_expect_tx(bar, (uint32_t)(nt + nvalid) * rb);
      bulk_load(sdout, dout + (size_t)t0 * vpr, (uint32_t)nt * rb, bar);
    }
    __syncwarp();
    if (r0 >= 0) bulk_load(sy + (size_t)lane * vpr, y + (size_t)r0 * vpr, rb, bar);
    if (r1 >= 0) bulk_load(sy + (size_t)(lane + 32) * vpr, y + (size_t)r1 * vpr, rb, bar);
  }
  // every copy lands unless the memory system fails; the wait is bounded all the same
  const bool ready = mbar_wait_bounded(bar, 0, 2000000000ull, nullptr, nullptr);
  if (w >= nt || !ready) return;
  const int t = t0 + w;
  const int myrow = slot_row(prow, t, k, lane, max_rows);
  const float myg = lane < k ? gates[(size_t)t * k + lane] : 0.f;
  int rows[8];
  float g[8], dot[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    rows[j] = __shfl_sync(0xffffffffu, myrow, j);
    g[j] = __shfl_sync(0xffffffffu, myg, j);
    dot[j] = 0.f;
  }
  const uint4* sd = sdout + (size_t)w * vpr;
  const uint4* sw = sy + (size_t)w * k * vpr;
#pragma unroll 1
  for (int v = lane; v < vpr; v += 32) {
    float fd[V::N];
    V::unpack(sd[v], fd);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      if (j < k && rows[j] >= 0) {
        float fy[V::N], o[V::N];
        V::unpack(sw[(size_t)j * vpr + v], fy);
#pragma unroll
        for (int i = 0; i < V::N; ++i) {
          dot[j] = fmaf(fd[i], fy[i], dot[j]);
          o[i] = g[j] * fd[i];
        }
        dy[(size_t)rows[j] * vpr + v] = V::pack(o);
      }
    }
  }
  combine_bwd_finish<BF16>(dot, g, t, k, E, lane, idx, dgates, dlsel, dlogits);
}

template <bool BF16>
__global__ void __launch_bounds__(kWarps * 32) token_reduce_kernel(
    const uint4* __restrict__ dxp, const int32_t* __restrict__ prow, const float* __restrict__ dlsel,
    const int32_t* __restrict__ idx, const uint4* __restrict__ Wr, uint4* __restrict__ dx, int T,
    int k, int E, int vpr, int max_rows) {
  pdl_enter();  // wait for the previous kernel before any global access
  using V = Vec<BF16>;
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * kWarps + (threadIdx.x >> 5);
  if (t >= T) return;
  const bool router = dlsel && idx && Wr;
  const int myrow = slot_row(prow, t, k, lane, max_rows);
  const float mydl = (router && lane < k) ? dlsel[(size_t)t * k + lane] : 0.f;
  int mye = (router && lane < k) ? idx[(size_t)t * k + lane] : 0;
  if (mye < 0 || mye >= E) mye = 0;
  int rows[8], es[8];
  float dl[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    rows[j] = __shfl_sync(0xffffffffu, myrow, j);
    dl[j] = __shfl_sync(0xffffffffu, mydl, j);
    es[j] = __shfl_sync(0xffffffffu, mye, j);
  }
#pragma unroll 2
  for (int v = lane; v < vpr; v += 32) {
    float acc[V::N];
#pragma unroll
    for (int i = 0; i < V::N; ++i) acc[i] = 0.f;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      if (j < k) {
        float f[V::N];
        V::unpack(ldg_row(dxp, rows[j], vpr, v), f);
#pragma unroll
        for (int i = 0; i < V::N; ++i) acc[i] += f[i];
        if (router) {
          V::unpack(Wr[(size_t)es[j] * vpr + v], f);
#pragma unroll
          for (int i = 0; i < V::N; ++i) acc[i] = fmaf(dl[j], f[i], acc[i]);
        }
      }
    }
    dx[(size_t)t * vpr + v] = V::pack(acc);
  }
}

// Score gradients of a learned router with renormalised gates, from the gate gradients: per token,
// dl_j = g_j (dg_j - sum_i g_i dg_i) for its k slots, and the dense row dlogits[t, e] (act dtype) that
// is zero except at the chosen experts. One warp per token. (combine_bwd_kernel computes the same on
// the way; the MXFP8 layer's fused combine backward leaves it to this kernel.)
template <bool BF16>
__global__ void __launch_bounds__(kWarps * 32) score_grad_kernel(const float* __restrict__ gates,
                                                                 const float* __restrict__ dgates,
                                                                 const int32_t* __restrict__ idx,
                                                                 float* __restrict__ dlsel,
                                                                 void* __restrict__ dlogits, int T,
                                                                 int k, int E) {
  pdl_enter();  // wait for the previous kernel before any global access
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * kWarps + (threadIdx.x >> 5);
  if (t >= T) return;
  const float g = lane < k ? gates[(size_t)t * k + lane] : 0.f;
  const float dg = lane < k ? dgates[(size_t)t * k + lane] : 0.f;
  float s = g * dg;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
  const float mydl = g * (dg - s);
  const int mye = lane < k ? idx[(size_t)t * k + lane] : -1;
  if (lane < k) dlsel[(size_t)t * k + lane] = mydl;
  int ej[8];
  float dj[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    ej[j] = __shfl_sync(0xffffffffu, mye, j);
    dj[j] = __shfl_sync(0xffffffffu, mydl, j);
  }
  for (int e = lane; e < E; e += 32) {
    float val = 0.f;
#pragma unroll
    for (int j = 0; j < 8; ++j)
      if (j < k && ej[j] == e) val = dj[j];
    if (BF16)
      reinterpret_cast<__nv_bfloat16*>(dlogits)[(size_t)t * E + e] = __float2bfloat16_rn(val);
    else
      reinterpret_cast<float*>(dlogits)[(size_t)t * E + e] = val;
  }
}

// Row bound passed to the kernels (row indices are int32).
inline int clamp_rows(int64_t max_rows) { return max_rows > INT32_MAX ? INT32_MAX : (int)max_rows; }

}  // namespace

int launch_dispatch(const void* x, const int32_t* prow, const int32_t* counts, const int32_t* poff,
                    void* xp, int T, int k, int E, int row_bytes, int64_t max_rows, cudaStream_t s) {
  const int vpr = row_bytes / 16;
  const int mr = clamp_rows(max_rows);
  const int tok_blocks = (T + kWarps - 1) / kWarps;
  MOE_LAUNCH(launch_pdl(dispatch_kernel, tok_blocks + E, kWarps * 32, 0, s, 
      static_cast<const uint4*>(x), prow, counts, poff, static_cast<uint4*>(xp), T, k, vpr,
      tok_blocks, mr));
  count_launches(1);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

int launch_combine(const void* y, const float* gates, const int32_t* prow, void* out, int T, int k,
                   int row_bytes, bool bf16, int64_t max_rows, cudaStream_t s) {
  const int vpr = row_bytes / 16;
  const int mr = clamp_rows(max_rows);
  const int blocks = (T + kWarps - 1) / kWarps;
  if (bf16)
    MOE_LAUNCH(launch_pdl(combine_kernel<true>, blocks, kWarps * 32, 0, s, static_cast<const uint4*>(y), gates, prow,
                                                        static_cast<uint4*>(out), T, k, vpr, mr));
  else
    MOE_LAUNCH(launch_pdl(combine_kernel<false>, blocks, kWarps * 32, 0, s, static_cast<const uint4*>(y), gates, prow,
                                                         static_cast<uint4*>(out), T, k, vpr, mr));
  count_launches(1);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

int launch_combine_bwd(const void* dout, const void* y, const float* gates, const int32_t* prow,
                       const int32_t* idx, const int32_t* counts, const int32_t* poff, void* dy,
                       float* dgates, float* dlsel, void* dlogits, int T, int k, int E, int row_bytes,
                       bool bf16, int64_t max_rows, cudaStream_t s) {
  const int vpr = row_bytes / 16;
  const int mr = clamp_rows(max_rows);
  // bulk-staged kernel: tokens per block sized for about 60 KB of staged rows (three blocks per SM)
  const size_t per_tok = (size_t)(1 + k) * row_bytes;
  const int tpb = (int)std::min<size_t>(kWarps, std::max<size_t>(1, kCbStageBudget / per_tok));
  const size_t smem = 128 + (size_t)tpb * per_tok;
  if (smem <= kCbSmemMax) {
    static bool attr_done[2][64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) dev = 0;
    if (!attr_done[bf16][dev]) {
      const cudaError_t e = bf16 ? cudaFuncSetAttribute(combine_bwd_bulk_kernel<true>,
                                                        cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                        (int)kCbSmemMax)
                                 : cudaFuncSetAttribute(combine_bwd_bulk_kernel<false>,
                                                        cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                        (int)kCbSmemMax);
      if (e != cudaSuccess) return MOE_ERR_CUDA;
      attr_done[bf16][dev] = true;
    }
    const int tb = (T + tpb - 1) / tpb;
    if (bf16)
      MOE_LAUNCH(launch_pdl(combine_bwd_bulk_kernel<true>, tb + E, kWarps * 32, smem, s,
          static_cast<const uint4*>(dout), static_cast<const uint4*>(y), gates, prow, idx, counts,
          poff, static_cast<uint4*>(dy), dgates, dlsel, dlogits, T, k, E, vpr, tb, mr, tpb));
    else
      MOE_LAUNCH(launch_pdl(combine_bwd_bulk_kernel<false>, tb + E, kWarps * 32, smem, s,
          static_cast<const uint4*>(dout), static_cast<const uint4*>(y), gates, prow, idx, counts,
          poff, static_cast<uint4*>(dy), dgates, dlsel, dlogits, T, k, E, vpr, tb, mr, tpb));
    count_launches(1);
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
  }
  // rows too wide to stage even one token: the register-staged kernel
  const int tok_blocks = (T + kWarps - 1) / kWarps;
  if (bf16)
    MOE_LAUNCH(launch_pdl(combine_bwd_kernel<true>, tok_blocks + E, kWarps * 32, 0, s, 
        static_cast<const uint4*>(dout), static_cast<const uint4*>(y), gates, prow, idx, counts,
        poff, static_cast<uint4*>(dy), dgates, dlsel, dlogits, T, k, E, vpr, tok_blocks, mr));
  else
    MOE_LAUNCH(launch_pdl(combine_bwd_kernel<false>, tok_blocks + E, kWarps * 32, 0, s, 
        static_cast<const uint4*>(dout), static_cast<const uint4*>(y), gates, prow, idx, counts,
        poff, static_cast<uint4*>(dy), dgates, dlsel, dlogits, T, k, E, vpr, tok_blocks, mr));
  count_launches(1);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

int launch_token_reduce(const void* dxp, const int32_t* prow, const float* dlsel, const int32_t* idx,
                        const void* Wr, void* dx, int T, int k, int E, int row_bytes, bool bf16,
                        int64_t max_rows, cudaStream_t s) {
  const int vpr = row_bytes / 16;
  const int mr = clamp_rows(max_rows);
  const int blocks = (T + kWarps - 1) / kWarps;
  if (bf16)
    MOE_LAUNCH(launch_pdl(token_reduce_kernel<true>, blocks, kWarps * 32, 0, s, 
        static_cast<const uint4*>(dxp), prow, dlsel, idx, static_cast<const uint4*>(Wr),
        static_cast<uint4*>(dx), T, k, E, vpr, mr));
  else
    MOE_LAUNCH(launch_pdl(token_reduce_kernel<false>, blocks, kWarps * 32, 0, s, 
        static_cast<const uint4*>(dxp), prow, dlsel, idx, static_cast<const uint4*>(Wr),
        static_cast<uint4*>(dx), T, k, E, vpr, mr));
  count_launches(1);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

int launch_score_grad(const float* gates, const float* dgates, const int32_t* idx, float* dlsel,
                      void* dlogits, int T, int k, int E, bool bf16, cudaStream_t s) {
  const int blocks = (T + kWarps - 1) / kWarps;
  if (bf16)
    MOE_LAUNCH(launch_pdl(score_grad_kernel<true>, blocks, kWarps * 32, 0, s, gates, dgates, idx, dlsel,
                          dlogits, T, k, E));
  else
    MOE_LAUNCH(launch_pdl(score_grad_kernel<false>, blocks, kWarps * 32, 0, s, gates, dgates, idx, dlsel,
                          dlogits, T, k, E));
  count_launches(1);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

}  // namespace moe
