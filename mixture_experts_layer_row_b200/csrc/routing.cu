// Routing on the GPU: top-k selection with gates, then the routing metadata (per-expert histogram,
// exclusive scans, stable permutation) computed entirely on the device so that the host never waits
// for a copy back ("GPU-resident routing", bytechap.com "Como funciona"; unite.ai "Parallelismo,
// precisione e tecniche di memoria").
//
// Top-k: one warp per token; each lane holds ceil(E/32) scores; k rounds of a warp-wide argmax with
// the order (score descending, expert id ascending), so equal scores go to the lower id.
// Metadata: three small kernels over chunks of 256 tokens:
//   1. per-chunk expert histogram (shared-memory counters; counts do not depend on arrival order);
//   2. one CTA turns the histograms into per-chunk bases (exclusive scan over chunks), counts,
//      offsets and aligned padded offsets (exclusive scans over experts), checks sum = T*k;
//   3. per chunk, the stable rank of every entry inside its expert: within a warp by
//      __match_any_sync + popc of the lower lanes, across warps and chunks by the scanned bases.
//      The order is ascending (token, slot): deterministic, no atomics decide it.
#include "internal.h"

namespace moe {

constexpr int kChunk = 256;  // tokens per metadata chunk (one CTA of 256 threads)

template <int VPL>
__global__ void __launch_bounds__(256) topk_kernel(const float* __restrict__ logits,
                                                   const float* __restrict__ bias, int T, int E, int k,
                                                   int renorm, int32_t* __restrict__ idx,
                                                   float* __restrict__ gates, uint32_t* err) {
  pdl_enter();  // wait for the previous kernel before any global access
  const int lane = threadIdx.x & 31;
  const int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (t >= T) return;
  float v[VPL];
  bool bad = false;
#pragma unroll
  for (int i = 0; i < VPL; ++i) {
    const int e = lane + 32 * i;
    float x = -INFINITY;
    if (e < E) {
      x = logits[(size_t)t * E + e];
      if (bias) x += bias[e];
      if (!isfinite(x)) {
        bad = true;
        x = -INFINITY;
      }
    }
    v[i] = x;
  }
  if (__any_sync(0xffffffffu, bad) && lane == 0) set_error(err, MOE_DEVERR_NONFINITE);
  uint32_t picked = 0;
  float sel_v[8];
  int sel_e[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    if (j >= k) break;
    float bv = -INFINITY;
    int be = 0x7fffffff;
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      const int e = lane + 32 * i;
      if (e < E && !((picked >> i) & 1u)) {
        if (v[i] > bv || (v[i] == bv && e < be)) {
          bv = v[i];
          be = e;
        }
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
      const int oe = __shfl_xor_sync(0xffffffffu, be, off);
      if (ov > bv || (ov == bv && oe < be)) {
        bv = ov;
        be = oe;
      }
    }
    if ((be & 31) == lane) picked |= 1u << (be >> 5);
    sel_v[j] = bv;
    sel_e[j] = be;
  }
  // gates: softmax of the chosen scores (renormalised), or full softmax probabilities
  const float m = sel_v[0];
  float denom = 0.f;
  if (renorm) {
#pragma unroll
    for (int j = 0; j < 8; ++j)
      if (j < k) denom += expf(sel_v[j] - m);
  } else {
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < VPL; ++i)
      if (lane + 32 * i < E) s += expf(v[i] - m);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    denom = s;
  }
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    if (j < k && lane == j) {
      idx[(size_t)t * k + j] = sel_e[j];
      gates[(size_t)t * k + j] = expf(sel_v[j] - m) / denom;
    }
  }
}

__global__ void __launch_bounds__(kChunk) hist_kernel(const int32_t* __restrict__ idx, int T, int E,
                                                      int k, int32_t* __restrict__ hist,
                                                      uint32_t* err) {
  pdl_enter();  // wait for the previous kernel before any global access
  __shared__ int h[256];
  for (int e = threadIdx.x; e < E; e += blockDim.x) h[e] = 0;
  __syncthreads();
  const int t = blockIdx.x * kChunk + threadIdx.x;
  bool bad = false;
  if (t < T) {
    for (int j = 0; j < k; ++j) {
      const int e = idx[(size_t)t * k + j];
      if (e < 0 || e >= E)
        bad = true;
      else
        atomicAdd(&h[e], 1);
    }
  }
  if (bad) set_error(err, MOE_DEVERR_ROUTING);
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) hist[(size_t)blockIdx.x * E + e] = h[e];
}

// Exclusive scan of `val` over the 256 threads of the block; returns the exclusive prefix and
// writes the block total to *total.
__device__ int block_exclusive_scan_256(int val, int* smem_warp, int* total) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  int inc = val;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int o = __shfl_up_sync(0xffffffffu, inc, off);
    if (lane >= off) inc += o;
  }
  if (lane == 31) smem_warp[w] = inc;
  __syncthreads();
  if (w == 0) {
    int s = lane < 8 ? smem_warp[lane] : 0;
    int si = s;
#pragma unroll
    for (int off = 1; off < 8; off <<= 1) {
      const int o = __shfl_up_sync(0xffffffffu, si, off);
      if (lane >= off) si += o;
    }
    if (lane < 8) smem_warp[8 + lane] = si - s;  // exclusive warp base
    if (lane == 7) smem_warp[16] = si;
  }
  __syncthreads();
  const int r = smem_warp[8 + w] + inc - val;
  *total = smem_warp[16];
  __syncthreads();
  return r;
}

__global__ void __launch_bounds__(256) scan_kernel(int32_t* __restrict__ hist, int nchunks, int T,
                                                   int E, int k, int align, int64_t max_rows,
                                                   int32_t* __restrict__ counts,
                                                   int32_t* __restrict__ offsets,
                                                   int32_t* __restrict__ poff,
                                                   int32_t* __restrict__ row_token, uint32_t* err) {
  pdl_enter();  // wait for the previous kernel before any global access
  __shared__ int sw[32];
  const int e = threadIdx.x;
  int run = 0;
  if (e < E) {
    // the expert's per-chunk counts in batches of 16 loads in flight (a loop that waited on each load
    // in turn took 12 us for 32 chunks), replaced in place by their exclusive prefix
    constexpr int kB = 16;
    for (int c0 = 0; c0 < nchunks; c0 += kB) {
      int v[kB];
#pragma unroll
      for (int u = 0; u < kB; ++u) v[u] = c0 + u < nchunks ? hist[(size_t)(c0 + u) * E + e] : 0;
#pragma unroll
      for (int u = 0; u < kB; ++u) {
        if (c0 + u < nchunks) {
          hist[(size_t)(c0 + u) * E + e] = run;
          run += v[u];
        }
      }
    }
  }
  const int cnt = e < E ? run : 0;
  const int pcnt = (cnt + align - 1) / align * align;
  int tot, ptot;
  const int off = block_exclusive_scan_256(cnt, sw, &tot);
  const int poffe = block_exclusive_scan_256(pcnt, sw, &ptot);
  if (e < E) {
    counts[e] = cnt;
    offsets[e] = off;
    poff[e] = poffe;
    for (int r = poffe + cnt; r < poffe + pcnt; ++r) row_token[r] = -1;
  }
  if (e == 0) {
    offsets[E] = tot;
    poff[E] = ptot;
    if (tot != T * k) set_error(err, MOE_DEVERR_ROUTING);
  }
  for (int64_t r = ptot + threadIdx.x; r < max_rows; r += blockDim.x) row_token[r] = -1;
}

__global__ void __launch_bounds__(kChunk) rank_kernel(const int32_t* __restrict__ idx, int T, int E,
                                                      int k, const int32_t* __restrict__ chunk_base,
                                                      const int32_t* __restrict__ offsets,
                                                      const int32_t* __restrict__ poff,
                                                      int32_t* __restrict__ perm,
                                                      int32_t* __restrict__ prow,
                                                      int32_t* __restrict__ row_token) {
  pdl_enter();  // wait for the previous kernel before any global access
  __shared__ int wcnt[kChunk / 32][256];
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  for (int i = threadIdx.x; i < (kChunk / 32) * 256; i += blockDim.x) (&wcnt[0][0])[i] = 0;
  __syncthreads();
  const int64_t total = (int64_t)T * k;
  const int64_t seg = ((int64_t)blockIdx.x * kChunk + 32 * w) * k;  // first entry of this warp
  int lrank[8], ex[8];
#pragma unroll
  for (int it = 0; it < 8; ++it) {
    ex[it] = -1;
    lrank[it] = 0;
    if (it >= k) continue;
    const int64_t n = seg + it * 32 + lane;
    int e = -1;
    if (n < total) {
      e = idx[n];
      if (e < 0 || e >= E) e = -1;
    }
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    const int leader = __ffs(peers) - 1;
    const int prior = __popc(peers & ((1u << lane) - 1u));
    const int base = e >= 0 ? wcnt[w][e] : 0;
    __syncwarp();
    if (lane == leader && e >= 0) wcnt[w][e] = base + __popc(peers);
    __syncwarp();
    ex[it] = e;
    lrank[it] = base + prior;
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int run = 0;
    for (int ww = 0; ww < kChunk / 32; ++ww) {
      const int v = wcnt[ww][e];
      wcnt[ww][e] = run;
      run += v;
    }
  }
  __syncthreads();
#pragma unroll
  for (int it = 0; it < 8; ++it) {
    if (it >= k) break;
    const int e = ex[it];
    const int64_t n = seg + it * 32 + lane;
    if (e < 0) {
      // an expert id outside [0,E) (flagged by the histogram): the entry has no row; -1 makes the row
      // kernels skip it instead of following a stale position
      if (n < total) perm[n] = prow[n] = -1;
      continue;
    }
    const int r = chunk_base[(size_t)blockIdx.x * E + e] + wcnt[w][e] + lrank[it];
    perm[n] = offsets[e] + r;
    const int pr = poff[e] + r;
    prow[n] = pr;
    row_token[pr] = (int32_t)n;
  }
}

int launch_topk(const float* logits, const float* bias, int T, int E, int k, int renorm,
                int32_t* idx, float* gates, uint32_t* err, cudaStream_t s) {
  const int threads = 256;
  const int blocks = (int)(((int64_t)T * 32 + threads - 1) / threads);
  const int vpl = (E + 31) / 32;
  switch (vpl) {
#define MOE_TOPK_CASE(V) \
  case V:                \
    MOE_LAUNCH(launch_pdl(topk_kernel<V>, blocks, threads, 0, s, logits, bias, T, E, k, renorm, idx, gates, err)); break;
    MOE_TOPK_CASE(1)
    MOE_TOPK_CASE(2)
    MOE_TOPK_CASE(3)
    MOE_TOPK_CASE(4)
    MOE_TOPK_CASE(5)
    MOE_TOPK_CASE(6)
    MOE_TOPK_CASE(7)
    MOE_TOPK_CASE(8)
#undef MOE_TOPK_CASE
    default:
      return MOE_ERR_UNSUPPORTED;
  }
  count_launches(1);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

size_t metadata_ws_bytes(int T, int E) {
  const size_t nchunks = (T + kChunk - 1) / kChunk;
  return nchunks * E * sizeof(int32_t);
}

int launch_metadata(const int32_t* idx, int T, int E, int k, int align, int64_t max_rows,
                    int32_t* counts, int32_t* offsets, int32_t* poff, int32_t* perm, int32_t* prow,
                    int32_t* row_token, int32_t* hist_ws, uint32_t* err, cudaStream_t s) {
  const int nchunks = (T + kChunk - 1) / kChunk;
  MOE_LAUNCH(launch_pdl(hist_kernel, nchunks, kChunk, 0, s, idx, T, E, k, hist_ws, err));
  MOE_LAUNCH(launch_pdl(scan_kernel, 1, 256, 0, s, hist_ws, nchunks, T, E, k, align, max_rows, counts, offsets, poff,
                                row_token, err));
  MOE_LAUNCH(launch_pdl(rank_kernel, nchunks, kChunk, 0, s, idx, T, E, k, hist_ws, offsets, poff, perm, prow, row_token));
  count_launches(3);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

}  // namespace moe
