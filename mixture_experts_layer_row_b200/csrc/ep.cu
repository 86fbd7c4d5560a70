// Row-wise expert parallelism across the GPUs of one node (the multi-GPU design of "Olmo-core 3":
// each routed token row is written directly into the input buffer of the expert that owns it, on
// whichever GPU holds that expert, and the device-scheduled grouped GEMM then runs each GPU's local
// experts -- unite.ai, "Parallelismo, precisione e tecniche di memoria"; bytechap.com, "Como funciona").
//
// G ranks, one GPU each; rank h owns the E/G consecutive experts [h*E/G, (h+1)*E/G). Every rank routes
// its own T tokens over all E experts, counts its entries per expert (moe_route_metadata), and the
// ranks all-gather those counts (one small collective, issued by the caller). From the gathered counts
// every rank computes the same layout of every owner's routed-row buffers:
//   - an owner's local expert e holds rows [poff[e], poff[e+1]) (starts 32-aligned, as on one GPU);
//   - inside the group the rows come source rank by source rank, and inside one source in that
//     source's token order (the single-GPU stable order of its own entries).
// The row kernels then move rows across GPUs with plain loads and stores through peer pointers (P2P
// over NVLink): dispatch stores x rows into the owners' buffers, combine and the token reduce load
// expert outputs / input gradients from them, the combine backward loads y and stores dy. No TMA, no
// multicast; nothing waits on another GPU inside a kernel (the caller orders the ranks with
// collectives between the phases).
#include "internal.h"

namespace moe {
namespace {

constexpr int kEpWarps = 8;

// Layout from the gathered counts all_counts[G][E]: one CTA of 256 threads (E <= 256).
//   src_base[e]   row (in the owner's buffers) of this rank's first entry for expert e;
//   owner view    counts_loc[E/G], poff_loc[E/G + 1] of this rank's local experts.
__global__ void __launch_bounds__(256) ep_layout_kernel(const int32_t* __restrict__ all_counts, int G,
                                                        int E, int rank, int32_t* __restrict__ src_base,
                                                        int32_t* __restrict__ counts_loc,
                                                        int32_t* __restrict__ poff_loc) {
  pdl_enter();  // wait for the previous kernel before any global access
  __shared__ int pad[256];
  const int EL = E / G;
  const int e = threadIdx.x;
  int total = 0, before = 0;
  if (e < E) {
    for (int s = 0; s < G; ++s) {
      const int c = all_counts[(size_t)s * E + e];
      if (s < rank) before += c;
      total += c;
    }
    pad[e] = (total + 31) / 32 * 32;
  }
  __syncthreads();
  if (e < E) {
    // exclusive prefix of the padded group sizes inside the owner's own experts
    const int h0 = (e / EL) * EL;
    int start = 0;
    for (int q = h0; q < e; ++q) start += pad[q];
    src_base[e] = start + before;
    if (e / EL == rank) {
      counts_loc[e - h0] = total;
      poff_loc[e - h0] = start;
      if (e - h0 == EL - 1) poff_loc[EL] = start + pad[e];
    }
  }
}

// dst_row[n] = src_base[e] + (perm[n] - offsets[e]) for e = idx[n]: the entry's row in its owner's
// buffers (perm / offsets: this rank's own single-GPU metadata). Entries with an invalid expert id
// get -1 (the row kernels skip them).
__global__ void ep_dst_row_kernel(const int32_t* __restrict__ idx, const int32_t* __restrict__ perm,
                                  const int32_t* __restrict__ offsets,
                                  const int32_t* __restrict__ src_base, int64_t n_entries, int E,
                                  int32_t* __restrict__ dst_row) {
  pdl_enter();
  const int64_t n = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (n >= n_entries) return;
  const int e = idx[n];
  const int p = perm[n];
  dst_row[n] = (e >= 0 && e < E && p >= 0) ? src_base[e] + (p - offsets[e]) : -1;
}

// Pad rows [poff[e] + counts[e], poff[e+1]) of the owner's local experts are zeroed by the owner
// (in its own memory); one CTA per local expert.
__global__ void __launch_bounds__(256) ep_zero_pad_kernel(uint4* __restrict__ buf,
                                                          const int32_t* __restrict__ counts,
                                                          const int32_t* __restrict__ poff, int vpr) {
  pdl_enter();
  const int e = blockIdx.x;
  const int r0 = poff[e] + counts[e], r1 = poff[e + 1];
  const int64_t n = (int64_t)(r1 - r0) * vpr;
  uint4* base = buf + (size_t)r0 * vpr;
  for (int64_t i = threadIdx.x; i < n; i += blockDim.x) base[i] = make_uint4(0, 0, 0, 0);
}

struct Peers {
  uint4* p[kMaxEpRanks];
};

// One warp per token; slot j's row lives on owner idx/EL at dst_row.
__device__ __forceinline__ void ep_slot(const int32_t* idx, const int32_t* dst_row, int t, int k,
                                        int lane, int E, int EL, int max_rows, int& owner, int& row) {
  owner = 0;
  row = -1;
  if (lane < k) {
    const int e = idx[(size_t)t * k + lane];
    const int r = dst_row[(size_t)t * k + lane];
    if (e >= 0 && e < E && r >= 0 && r < max_rows) {
      owner = e / EL;
      row = r;
    }
  }
}

__global__ void __launch_bounds__(kEpWarps * 32) ep_dispatch_kernel(
    const uint4* __restrict__ x, const int32_t* __restrict__ idx, const int32_t* __restrict__ dst_row,
    Peers xp, int T, int k, int E, int EL, int vpr, int max_rows) {
  pdl_enter();
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * kEpWarps + (threadIdx.x >> 5);
  if (t >= T) return;
  int myo, myr;
  ep_slot(idx, dst_row, t, k, lane, E, EL, max_rows, myo, myr);
  uint4* dst[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int o = __shfl_sync(0xffffffffu, myo, j), r = __shfl_sync(0xffffffffu, myr, j);
    dst[j] = r >= 0 ? xp.p[o] + (size_t)r * vpr : nullptr;
  }
  const uint4* src = x + (size_t)t * vpr;
#pragma unroll 4
  for (int v = lane; v < vpr; v += 32) {
    const uint4 val = src[v];
#pragma unroll
    for (int j = 0; j < 8; ++j)
      if (j < k && dst[j]) dst[j][v] = val;
  }
}

template <bool BF16>
__device__ __forceinline__ void unpack16(const uint4& w, float (&f)[8]) {
  const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = BF16 ? bf16lo(u[i]) : __uint_as_float(u[i]);
    f[2 * i + 1] = BF16 ? bf16hi(u[i]) : 0.f;
  }
}

// out[t] = sum_j g[t,j] y_owner[row]  (bf16 rows, fp32 accumulation; the peer loads of one step are
// all issued before the sums)
__global__ void __launch_bounds__(kEpWarps * 32) ep_combine_kernel(
    Peers y, const float* __restrict__ gates, const int32_t* __restrict__ idx,
    const int32_t* __restrict__ dst_row, uint4* __restrict__ out, int T, int k, int E, int EL, int vpr,
    int max_rows) {
  pdl_enter();
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * kEpWarps + (threadIdx.x >> 5);
  if (t >= T) return;
  int myo, myr;
  ep_slot(idx, dst_row, t, k, lane, E, EL, max_rows, myo, myr);
  const float myg = lane < k ? gates[(size_t)t * k + lane] : 0.f;
  const uint4* src[8];
  float g[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int o = __shfl_sync(0xffffffffu, myo, j), r = __shfl_sync(0xffffffffu, myr, j);
    src[j] = r >= 0 ? y.p[o] + (size_t)r * vpr : nullptr;
    g[j] = __shfl_sync(0xffffffffu, myg, j);
  }
  for (int v = lane; v < vpr; v += 32) {
    uint4 w[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) w[j] = (j < k && src[j]) ? src[j][v] : make_uint4(0u, 0u, 0u, 0u);
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      float f[8];
      unpack16<true>(w[j], f);
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] = fmaf(g[j], f[i], acc[i]);
    }
    out[(size_t)t * vpr + v] = make_uint4(pack_bf16(acc[0], acc[1]), pack_bf16(acc[2], acc[3]),
                                          pack_bf16(acc[4], acc[5]), pack_bf16(acc[6], acc[7]));
  }
}

// dy_owner[row] = g dout[t] (peer stores), dgates[t,j] = <dout[t], y_owner[row]> (peer loads).
__global__ void __launch_bounds__(kEpWarps * 32) ep_combine_bwd_kernel(
    const uint4* __restrict__ dout, Peers y, const float* __restrict__ gates,
    const int32_t* __restrict__ idx, const int32_t* __restrict__ dst_row, Peers dy,
    float* __restrict__ dgates, int T, int k, int E, int EL, int vpr, int max_rows) {
  pdl_enter();
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * kEpWarps + (threadIdx.x >> 5);
  if (t >= T) return;
  int myo, myr;
  ep_slot(idx, dst_row, t, k, lane, E, EL, max_rows, myo, myr);
  const float myg = lane < k ? gates[(size_t)t * k + lane] : 0.f;
  const uint4* ys[8];
  uint4* dys[8];
  float g[8], dot[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int o = __shfl_sync(0xffffffffu, myo, j), r = __shfl_sync(0xffffffffu, myr, j);
    ys[j] = r >= 0 ? y.p[o] + (size_t)r * vpr : nullptr;
    dys[j] = r >= 0 ? dy.p[o] + (size_t)r * vpr : nullptr;
    g[j] = __shfl_sync(0xffffffffu, myg, j);
    dot[j] = 0.f;
  }
  for (int v = lane; v < vpr; v += 32) {
    float fd[8];
    unpack16<true>(dout[(size_t)t * vpr + v], fd);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      if (j < k && ys[j]) {
        float fy[8], o[8];
        unpack16<true>(ys[j][v], fy);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          dot[j] = fmaf(fd[i], fy[i], dot[j]);
          o[i] = g[j] * fd[i];
        }
        dys[j][v] = make_uint4(pack_bf16(o[0], o[1]), pack_bf16(o[2], o[3]), pack_bf16(o[4], o[5]),
                               pack_bf16(o[6], o[7]));
      }
    }
  }
#pragma unroll
  for (int j = 0; j < 8; ++j) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) dot[j] += __shfl_xor_sync(0xffffffffu, dot[j], off);
    if (j < k && lane == j) dgates[(size_t)t * k + j] = dot[j];
  }
}

// dx[t] = sum_j dx_perm_owner[row]
__global__ void __launch_bounds__(kEpWarps * 32) ep_token_reduce_kernel(
    Peers dxp, const int32_t* __restrict__ idx, const int32_t* __restrict__ dst_row,
    uint4* __restrict__ dx, int T, int k, int E, int EL, int vpr, int max_rows) {
  pdl_enter();
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * kEpWarps + (threadIdx.x >> 5);
  if (t >= T) return;
  int myo, myr;
  ep_slot(idx, dst_row, t, k, lane, E, EL, max_rows, myo, myr);
  const uint4* src[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int o = __shfl_sync(0xffffffffu, myo, j), r = __shfl_sync(0xffffffffu, myr, j);
    src[j] = r >= 0 ? dxp.p[o] + (size_t)r * vpr : nullptr;
  }
  for (int v = lane; v < vpr; v += 32) {
    uint4 w[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) w[j] = (j < k && src[j]) ? src[j][v] : make_uint4(0u, 0u, 0u, 0u);
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      float f[8];
      unpack16<true>(w[j], f);
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] += f[i];
    }
    dx[(size_t)t * vpr + v] = make_uint4(pack_bf16(acc[0], acc[1]), pack_bf16(acc[2], acc[3]),
                                         pack_bf16(acc[4], acc[5]), pack_bf16(acc[6], acc[7]));
  }
}

bool peers_from(void* const* ptrs, int G, Peers* out) {
  if (!ptrs || G < 1 || G > kMaxEpRanks) return false;
  for (int h = 0; h < kMaxEpRanks; ++h) {
    out->p[h] = h < G ? static_cast<uint4*>(ptrs[h]) : nullptr;
    if (h < G && (!ptrs[h] || (reinterpret_cast<uintptr_t>(ptrs[h]) & 15u))) return false;
  }
  return true;
}

}  // namespace

int launch_ep_layout(const int32_t* all_counts, int G, int E, int rank, const int32_t* idx,
                     const int32_t* perm, const int32_t* offsets, int64_t n_entries,
                     int32_t* src_base, int32_t* counts_loc, int32_t* poff_loc, int32_t* dst_row,
                     cudaStream_t s) {
  MOE_LAUNCH(launch_pdl(ep_layout_kernel, 1, 256, 0, s, all_counts, G, E, rank, src_base, counts_loc,
                        poff_loc));
  const unsigned blocks = (unsigned)((n_entries + 255) / 256);
  MOE_LAUNCH(launch_pdl(ep_dst_row_kernel, blocks, 256, 0, s, idx, perm, offsets,
                        (const int32_t*)src_base, n_entries, E, dst_row));
  count_launches(2);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

int launch_ep_zero_pad(void* buf, const int32_t* counts_loc, const int32_t* poff_loc, int EL,
                       int row_bytes, cudaStream_t s) {
  MOE_LAUNCH(launch_pdl(ep_zero_pad_kernel, EL, 256, 0, s, static_cast<uint4*>(buf), counts_loc,
                        poff_loc, row_bytes / 16));
  count_launches(1);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

int launch_ep_rows(int op, int G, int T, int k, int E, int row_bytes, int64_t max_rows,
                   const void* x_or_dout, void* const* peers_a, void* const* peers_b,
                   const float* gates, const int32_t* idx, const int32_t* dst_row, void* out,
                   float* dgates, cudaStream_t s) {
  Peers pa, pb;
  if (!peers_from(peers_a, G, &pa)) return MOE_ERR_INVALID_ARG;
  if (op == 2 && !peers_from(peers_b, G, &pb)) return MOE_ERR_INVALID_ARG;
  const int vpr = row_bytes / 16, EL = E / G;
  const int mr = max_rows > INT32_MAX ? INT32_MAX : (int)max_rows;
  const unsigned blocks = (unsigned)((T + kEpWarps - 1) / kEpWarps);
  switch (op) {
    case 0:  // dispatch
      MOE_LAUNCH(launch_pdl(ep_dispatch_kernel, blocks, kEpWarps * 32, 0, s,
                            static_cast<const uint4*>(x_or_dout), idx, dst_row, pa, T, k, E, EL, vpr, mr));
      break;
    case 1:  // combine
      MOE_LAUNCH(launch_pdl(ep_combine_kernel, blocks, kEpWarps * 32, 0, s, pa, gates, idx, dst_row,
                            static_cast<uint4*>(out), T, k, E, EL, vpr, mr));
      break;
    case 2:  // combine backward
      MOE_LAUNCH(launch_pdl(ep_combine_bwd_kernel, blocks, kEpWarps * 32, 0, s,
                            static_cast<const uint4*>(x_or_dout), pa, gates, idx, dst_row, pb, dgates, T,
                            k, E, EL, vpr, mr));
      break;
    case 3:  // token reduce
      MOE_LAUNCH(launch_pdl(ep_token_reduce_kernel, blocks, kEpWarps * 32, 0, s, pa, idx, dst_row,
                            static_cast<uint4*>(out), T, k, E, EL, vpr, mr));
      break;
    default:
      return MOE_ERR_INVALID_ARG;
  }
  count_launches(1);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

}  // namespace moe
