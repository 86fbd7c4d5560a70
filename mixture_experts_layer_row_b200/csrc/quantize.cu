// MXFP8 quantisation: bf16 -> E4M3 codes + one UE8M0 scale per 32 elements along the contraction
// axis of the GEMM that consumes the operand (MXFP8 is the reduced-precision format of unite.ai,
// "Parallelismo, precisione e tecniche di memoria"; element and scale encodings per the OCP
// Microscaling Formats v1.0 specification):
//   block exponent e = floor(log2(amax)) - 8 (8 = E4M3's largest exponent), clamped to [-127, 127];
//   scale byte = e + 127; code = round-to-nearest-even(x * 2^-e) saturated to +-448;
//   an all-zero block gets scale byte 0 and zero codes.
// floor(log2) is read from the fp32 exponent bits (exact, subnormals included); the scaling by a power
// of two is exact in fp32, and the conversion is the hardware's cvt.rn.satfinite.e4m3x2.f32.
//
// Blocks run along rows (ROW: 32 consecutive elements of a row) or down columns (COL: 32 consecutive
// rows of a column); codes keep the source layout [rows, cols]. Scale layouts:
//   plain  ROW [rows, cols/32], COL [cols, rows/32];
//   tiled  the layout the MXFP8 grouped GEMM streams: for the scale of (MN index i, K-block b), with
//          i = row (ROW) or column (COL), 512-byte chunks per (128 MN indices, 4 K-blocks) at chunk
//          (i/128, b/4), byte (i%32)*16 + ((i%128)/32)*4 + b%4 inside -- exactly the rows that
//          tcgen05.cp 32x128b.warpx4 spreads over the four TMEM lane quadrants;
//   tiled gate/up  like tiled ROW for a stack of [gate; up] blocks of 2*G rows each, with the MN
//          index of row f of gate (up) remapped to 128*(f/64) + f%64 (+64), so that the 64 gate and
//          64 up rows of one fused GEMM1 tile share one chunk.
// Both kernels are HBM-bound streams with 16-byte loads.
#include "internal.h"

namespace moe {
namespace {

__device__ __forceinline__ int64_t scale_index(int layout, int64_t i, int64_t b, int64_t KB, int64_t G) {
  if (layout == 0) return i * KB + b;  // plain
  if (layout == 2) {                   // tiled gate/up: remap the row inside its [gate; up] stack
    const int64_t e = i / (2 * G), rr = i % (2 * G), f = rr % G, up = rr / G;
    i = e * 2 * G + (f / 64) * 128 + up * 64 + f % 64;
  }
  return tiled_sf_offset(i, b, KB);
}

__global__ void __launch_bounds__(256) quant_row_kernel(const uint4* __restrict__ src, int64_t nblocks,
                                                        int blocks_per_row, int layout, int64_t G,
                                                        uint4* __restrict__ q,
                                                        uint8_t* __restrict__ s) {
  pdl_enter();  // wait for the previous kernel before any global access
  const int64_t b = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= nblocks) return;
  uint4 w[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) w[i] = src[b * 4 + i];
  float v[32];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t u[4] = {w[i].x, w[i].y, w[i].z, w[i].w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      v[8 * i + 2 * j] = bf16lo(u[j]);
      v[8 * i + 2 * j + 1] = bf16hi(u[j]);
    }
  }
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(v[i]));
  uint8_t sb;
  const int e = block_exponent(amax, &sb);
  const float inv = exp2_exact(-e);
  uint32_t c[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint32_t lo = cvt_e4m3x2(v[4 * i] * inv, v[4 * i + 1] * inv);
    const uint32_t hi = cvt_e4m3x2(v[4 * i + 2] * inv, v[4 * i + 3] * inv);
    c[i] = amax > 0.f ? (lo | (hi << 16)) : 0u;
  }
  q[b * 2] = make_uint4(c[0], c[1], c[2], c[3]);
  q[b * 2 + 1] = make_uint4(c[4], c[5], c[6], c[7]);
  s[scale_index(layout, b / blocks_per_row, b % blocks_per_row, blocks_per_row, G)] = sb;
}

// One thread per (32-row block, 4 consecutive columns): the 32 8-byte row segments stay in registers
// between the block-maximum pass and the conversion, so the source is read once (a warp covers 128
// contiguous columns of each row).
__global__ void __launch_bounds__(128) quant_col_kernel(const uint2* __restrict__ src, int64_t rows,
                                                        int cols, int layout, uint32_t* __restrict__ q,
                                                        uint8_t* __restrict__ s) {
  pdl_enter();  // wait for the previous kernel before any global access
  const int groups = cols / 4;
  const int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t rblocks = rows / 32;
  if (t >= rblocks * groups) return;
  const int64_t rb = t / groups;
  const int cg = (int)(t % groups);
  const uint2* base = src + (rb * 32) * groups + cg;  // row stride = groups uint2
  uint2 w[32];
#pragma unroll
  for (int r = 0; r < 32; ++r) w[r] = base[(int64_t)r * groups];
  float amax[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int r = 0; r < 32; ++r) {
    amax[0] = fmaxf(amax[0], fabsf(bf16lo(w[r].x)));
    amax[1] = fmaxf(amax[1], fabsf(bf16hi(w[r].x)));
    amax[2] = fmaxf(amax[2], fabsf(bf16lo(w[r].y)));
    amax[3] = fmaxf(amax[3], fabsf(bf16hi(w[r].y)));
  }
  float inv[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    uint8_t sb;
    const int e = block_exponent(amax[j], &sb);
    inv[j] = amax[j] > 0.f ? exp2_exact(-e) : 0.f;
    s[scale_index(layout, (int64_t)cg * 4 + j, rb, rblocks, 0)] = sb;
  }
  const uint32_t keep = zero_block_mask(amax);
  uint32_t* qb = q + (rb * 32) * groups + cg;
#pragma unroll
  for (int r = 0; r < 32; ++r) {
    const uint32_t lo = cvt_e4m3x2(bf16lo(w[r].x) * inv[0], bf16hi(w[r].x) * inv[1]);
    const uint32_t hi = cvt_e4m3x2(bf16lo(w[r].y) * inv[2], bf16hi(w[r].y) * inv[3]);
    qb[(int64_t)r * groups] = (lo | (hi << 16)) & keep;
  }
}

// Both tiled quantisations of one operand in a single read. A CTA of 128 threads takes a 32-row x
// 128-column tile: coalesced 16-byte loads into registers and shared memory; row blocks (4 lanes hold
// one 32-column block) are converted from registers and stored as 8-byte groups; column blocks (one
// thread per column) are read back from shared memory, converted into a shared code tile and stored
// as 16-byte rows. Codes and scales are bit-identical to quant_row_kernel / quant_col_kernel with the
// tiled layout.
constexpr int kRcRows = 32, kRcCols = 128, kRcThreads = 128;

__global__ void __launch_bounds__(kRcThreads) quant_rowcol_kernel(const uint4* __restrict__ src,
                                                                  int64_t rows, int cols,
                                                                  uint2* __restrict__ qr,
                                                                  uint8_t* __restrict__ sr,
                                                                  uint4* __restrict__ qc,
                                                                  uint8_t* __restrict__ sc) {
  __shared__ __align__(16) uint4 tile[kRcRows * kRcCols / 8];      // bf16 [32][128]
  __shared__ __align__(16) uint8_t codes[kRcRows * kRcCols];        // column-block codes [32][128]
  pdl_enter();  // wait for the previous kernel before any global access
  const int ctiles = cols / kRcCols;
  const int64_t rb = blockIdx.x / ctiles;
  const int cb = (int)(blockIdx.x % ctiles);
  const int t = threadIdx.x;
  const int64_t row0 = rb * kRcRows;
  const int64_t w16 = cols / 8;  // 16-byte words per row
  const int c16 = t & 15;        // this thread's 16-byte column word inside the tile
  uint4 v[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = (t >> 4) + 8 * i;
    v[i] = src[(row0 + r) * w16 + cb * 16 + c16];
    tile[r * 16 + c16] = v[i];
  }
  // row blocks: lanes 4j..4j+3 hold the 32 columns of one block of one row
  const int kb = cols / 32;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = (t >> 4) + 8 * i;
    const uint32_t u[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
    float f[8];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      f[2 * j] = bf16lo(u[j]);
      f[2 * j + 1] = bf16hi(u[j]);
    }
    float m = 0.f;
#pragma unroll
    for (int j = 0; j < 8; ++j) m = fmaxf(m, fabsf(f[j]));
    m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
    m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
    uint8_t sb;
    const float ir = exp2_exact(-block_exponent(m, &sb));
    uint2 c;
    c.x = cvt_e4m3x2(f[0] * ir, f[1] * ir) | ((uint32_t)cvt_e4m3x2(f[2] * ir, f[3] * ir) << 16);
    c.y = cvt_e4m3x2(f[4] * ir, f[5] * ir) | ((uint32_t)cvt_e4m3x2(f[6] * ir, f[7] * ir) << 16);
    if (!(m > 0.f)) c = make_uint2(0u, 0u);
    qr[(row0 + r) * w16 + cb * 16 + c16] = c;
    if ((t & 3) == 0) sr[tiled_sf_offset(row0 + r, (int64_t)cb * 4 + (c16 >> 2), kb)] = sb;
  }
  __syncthreads();
  // column blocks: thread t owns column t of the tile (32 rows)
  {
    const __nv_bfloat16* tb = reinterpret_cast<const __nv_bfloat16*>(tile);
    float f[kRcRows];
    float amax = 0.f;
#pragma unroll
    for (int r = 0; r < kRcRows; ++r) {
      f[r] = __bfloat162float(tb[r * kRcCols + t]);
      amax = fmaxf(amax, fabsf(f[r]));
    }
    uint8_t sb;
    const int e = block_exponent(amax, &sb);
    const float inv = amax > 0.f ? exp2_exact(-e) : 0.f;
    sc[tiled_sf_offset((int64_t)cb * kRcCols + t, rb, rows / 32)] = sb;
#pragma unroll
    for (int r = 0; r < kRcRows; r += 2) {
      const uint32_t c2 = amax > 0.f ? cvt_e4m3x2(f[r] * inv, f[r + 1] * inv) : 0u;
      codes[r * kRcCols + t] = (uint8_t)(c2 & 0xFFu);
      codes[(r + 1) * kRcCols + t] = (uint8_t)(c2 >> 8);
    }
  }
  __syncthreads();
  const uint4* cw = reinterpret_cast<const uint4*>(codes);
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    const int idx = t + kRcThreads * j;  // 16-byte word of the code tile: 8 per row
    const int r = idx >> 3, c = idx & 7;
    qc[((row0 + r) * cols + (int64_t)cb * kRcCols) / 16 + c] = cw[idx];
  }
}

// Both tiled quantisations of an expert-grouped routed-row operand, built straight from token-order
// rows, so that no bf16 copy of the routed buffer is written (the MXFP8 layer's fused dispatch and
// fused combine backward):
//   GQ_X   padded row r holds x[t], t = row_token[r] / k                 (row-wise dispatch);
//   GQ_DY  padded row r holds dy = bf16(gates[n] * dout[t]), n = row_token[r], t = n / k (the combine
//          backward), and dgates[n] = <dout[t], y[r]> (fp32, fixed summation order) comes out on the
//          way;
// pad rows (row_token < 0) are zero. Each 32-row x 128-column tile is quantised exactly as
// quant_rowcol_kernel does (row blocks from registers, column blocks through shared memory), so codes
// and scales are bit-identical to quantising the bf16 routed buffer. Blocks at or past the used rows
// (poff[E]) are skipped: no GEMM reads them.
// One CTA per 32-row block walks the row's tiles and fetches the next tile's rows while it quantises
// the current one (GQ_DY's dot products run across the tiles; for GQ_X one CTA per tile was measured
// 15 % slower).
enum { GQ_X = 0, GQ_DY = 1 };

// Quantise the 32 x 128 tile held as v[4] (rows t/16 + 8i, 16-byte column word t%16) into the row and
// column forms; the shared buffers are free on entry and on exit.
__device__ __forceinline__ void quant_tile_32x128(const uint4 (&v)[4], uint4* tile, uint8_t* codes,
                                                  int64_t row0, int64_t rb, int cb, int cols,
                                                  int64_t rows, uint2* __restrict__ qr,
                                                  uint8_t* __restrict__ sr, uint4* __restrict__ qc,
                                                  uint8_t* __restrict__ sc) {
  const int t = threadIdx.x;
  const int c16 = t & 15;
  const int64_t w16 = cols / 8;
  const int kb = cols / 32;
#pragma unroll
  for (int i = 0; i < 4; ++i) tile[((t >> 4) + 8 * i) * 16 + c16] = v[i];
  // row blocks from registers: lanes 4j..4j+3 hold the 32 columns of one block of one row
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = (t >> 4) + 8 * i;
    const uint32_t u[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
    float f[8];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      f[2 * j] = bf16lo(u[j]);
      f[2 * j + 1] = bf16hi(u[j]);
    }
    float m = 0.f;
#pragma unroll
    for (int j = 0; j < 8; ++j) m = fmaxf(m, fabsf(f[j]));
    m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
    m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
    uint8_t sb;
    const float ir = exp2_exact(-block_exponent(m, &sb));
    uint2 c;
    c.x = cvt_e4m3x2(f[0] * ir, f[1] * ir) | ((uint32_t)cvt_e4m3x2(f[2] * ir, f[3] * ir) << 16);
    c.y = cvt_e4m3x2(f[4] * ir, f[5] * ir) | ((uint32_t)cvt_e4m3x2(f[6] * ir, f[7] * ir) << 16);
    if (!(m > 0.f)) c = make_uint2(0u, 0u);
    qr[(row0 + r) * w16 + cb * 16 + c16] = c;
    if ((t & 3) == 0) sr[tiled_sf_offset(row0 + r, (int64_t)cb * 4 + (c16 >> 2), kb)] = sb;
  }
  __syncthreads();
  // column blocks: thread t owns column t of the tile (32 rows)
  {
    const __nv_bfloat16* tb = reinterpret_cast<const __nv_bfloat16*>(tile);
    float f[kRcRows];
    float amax = 0.f;
#pragma unroll
    for (int r = 0; r < kRcRows; ++r) {
      f[r] = __bfloat162float(tb[r * kRcCols + t]);
      amax = fmaxf(amax, fabsf(f[r]));
    }
    uint8_t sb;
    const int e = block_exponent(amax, &sb);
    const float inv = amax > 0.f ? exp2_exact(-e) : 0.f;
    sc[tiled_sf_offset((int64_t)cb * kRcCols + t, rb, rows / 32)] = sb;
#pragma unroll
    for (int r = 0; r < kRcRows; r += 2) {
      const uint32_t c2 = amax > 0.f ? cvt_e4m3x2(f[r] * inv, f[r + 1] * inv) : 0u;
      codes[r * kRcCols + t] = (uint8_t)(c2 & 0xFFu);
      codes[(r + 1) * kRcCols + t] = (uint8_t)(c2 >> 8);
    }
  }
  __syncthreads();
  const uint4* cw = reinterpret_cast<const uint4*>(codes);
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    const int idx = t + kRcThreads * j;  // 16-byte word of the code tile: 8 per row
    const int r = idx >> 3, c = idx & 7;
    qc[((row0 + r) * cols + (int64_t)cb * kRcCols) / 16 + c] = cw[idx];
  }
  __syncthreads();  // the shared buffers are free again
}

template <int SRC>
__global__ void __launch_bounds__(kRcThreads) gather_quant_kernel(
    const uint4* __restrict__ tok, const int32_t* __restrict__ row_token,
    const int32_t* __restrict__ poff_end, int k, int64_t rows, int cols,
    const float* __restrict__ gates, const uint4* __restrict__ y, float* __restrict__ dgates,
    uint2* __restrict__ qr, uint8_t* __restrict__ sr, uint4* __restrict__ qc, uint8_t* __restrict__ sc) {
  __shared__ __align__(16) uint4 tile[kRcRows * kRcCols / 8];  // bf16 [32][128]
  __shared__ __align__(16) uint8_t codes[kRcRows * kRcCols];    // column-block codes [32][128]
  pdl_enter();  // wait for the previous kernel before any global access
  const int ctiles = cols / kRcCols;
  const int64_t rb = blockIdx.x;
  const int64_t row0 = rb * kRcRows;
  if (row0 >= *poff_end) return;
  const int t = threadIdx.x;
  const int c16 = t & 15;        // this thread's 16-byte column word inside a tile
  const int64_t w16 = cols / 8;  // 16-byte words per row
  // the four rows this thread loads: r = t/16 + 8i
  int64_t srow[4];
  int ent[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int n = row_token[row0 + (t >> 4) + 8 * i];
    ent[i] = n;
    srow[i] = n >= 0 ? (int64_t)(n / k) : -1;
  }
  if constexpr (SRC == GQ_X) {
    const uint4 z4 = make_uint4(0u, 0u, 0u, 0u);
    uint4 vn[4];  // the next tile's words
#pragma unroll
    for (int i = 0; i < 4; ++i) vn[i] = srow[i] >= 0 ? tok[srow[i] * w16 + c16] : z4;
    for (int cb = 0; cb < ctiles; ++cb) {
      uint4 v[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) v[i] = vn[i];
      if (cb + 1 < ctiles) {
#pragma unroll
        for (int i = 0; i < 4; ++i) vn[i] = srow[i] >= 0 ? tok[srow[i] * w16 + (cb + 1) * 16 + c16] : z4;
      }
      quant_tile_32x128(v, tile, codes, row0, rb, cb, cols, rows, qr, sr, qc, sc);
    }
  } else {
    float g[4], dot[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      g[i] = ent[i] >= 0 ? gates[ent[i]] : 0.f;
      dot[i] = 0.f;
    }
    const uint4 z4 = make_uint4(0u, 0u, 0u, 0u);
    uint4 dn[4], yn[4];  // the next tile's dout and y words
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      dn[i] = srow[i] >= 0 ? tok[srow[i] * w16 + c16] : z4;
      yn[i] = srow[i] >= 0 ? y[(row0 + (t >> 4) + 8 * i) * w16 + c16] : z4;
    }
    for (int cb = 0; cb < ctiles; ++cb) {
      uint4 dc[4], yc[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        dc[i] = dn[i];
        yc[i] = yn[i];
      }
      if (cb + 1 < ctiles) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          dn[i] = srow[i] >= 0 ? tok[srow[i] * w16 + (cb + 1) * 16 + c16] : z4;
          yn[i] = srow[i] >= 0 ? y[(row0 + (t >> 4) + 8 * i) * w16 + (cb + 1) * 16 + c16] : z4;
        }
      }
      uint4 v[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint32_t du[4] = {dc[i].x, dc[i].y, dc[i].z, dc[i].w};
        const uint32_t yu[4] = {yc[i].x, yc[i].y, yc[i].z, yc[i].w};
        uint32_t o[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float d0 = bf16lo(du[j]), d1 = bf16hi(du[j]);
          dot[i] = fmaf(d0, bf16lo(yu[j]), dot[i]);
          dot[i] = fmaf(d1, bf16hi(yu[j]), dot[i]);
          o[j] = pack_bf16(g[i] * d0, g[i] * d1);
        }
        v[i] = make_uint4(o[0], o[1], o[2], o[3]);
      }
      quant_tile_32x128(v, tile, codes, row0, rb, cb, cols, rows, qr, sr, qc, sc);
    }
    // the 16 threads that share a row hold its partial dot products over their columns
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float d = dot[i];
      d += __shfl_xor_sync(0xffffffffu, d, 1);
      d += __shfl_xor_sync(0xffffffffu, d, 2);
      d += __shfl_xor_sync(0xffffffffu, d, 4);
      d += __shfl_xor_sync(0xffffffffu, d, 8);
      if (c16 == 0 && ent[i] >= 0) dgates[ent[i]] = d;
    }
  }
}

}  // namespace

// Row-block and column-block tiled quantisations (MOE_QUANT_ROW_TILED into qr/sr, MOE_QUANT_COL_TILED
// into qc/sc) of one [rows, cols] operand in one pass; rows % 128 == 0, cols % 128 == 0.
int launch_quantize_rowcol(const void* src, int64_t rows, int cols, uint8_t* qr, uint8_t* sr,
                           uint8_t* qc, uint8_t* sc, cudaStream_t st) {
  const int64_t grid = (rows / kRcRows) * (cols / kRcCols);
  MOE_LAUNCH(launch_pdl(quant_rowcol_kernel, (unsigned)grid, kRcThreads, 0, st,
                        static_cast<const uint4*>(src), rows, cols, reinterpret_cast<uint2*>(qr), sr,
                        reinterpret_cast<uint4*>(qc), sc));
  count_launches(1);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

// MXFP8 dispatch: both tiled quantisations of the routed input built from x [T, cols] through
// row_token (rows = routed-row buffer rows, a multiple of 128; cols % 128 == 0).
int launch_dispatch_quant(const void* x, const int32_t* row_token, const int32_t* poff_end, int k,
                          int64_t rows, int cols, uint8_t* qr, uint8_t* sr, uint8_t* qc, uint8_t* sc,
                          cudaStream_t st) {
  MOE_LAUNCH(launch_pdl(gather_quant_kernel<GQ_X>, (unsigned)(rows / kRcRows), kRcThreads, 0, st,
                        static_cast<const uint4*>(x), row_token, poff_end, k, rows, cols,
                        (const float*)nullptr, (const uint4*)nullptr, (float*)nullptr,
                        reinterpret_cast<uint2*>(qr), sr, reinterpret_cast<uint4*>(qc), sc));
  count_launches(1);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

// MXFP8 combine backward: dy = bf16(g * dout) quantised both ways straight from dout [T, cols], and
// dgates[n] = <dout[t], y[row]>.
int launch_combine_bwd_quant(const void* dout, const void* y, const float* gates,
                             const int32_t* row_token, const int32_t* poff_end, int k, int64_t rows,
                             int cols, float* dgates, uint8_t* qr, uint8_t* sr, uint8_t* qc,
                             uint8_t* sc, cudaStream_t st) {
  MOE_LAUNCH(launch_pdl(gather_quant_kernel<GQ_DY>, (unsigned)(rows / kRcRows), kRcThreads, 0, st,
                        static_cast<const uint4*>(dout), row_token, poff_end, k, rows, cols, gates,
                        static_cast<const uint4*>(y), dgates, reinterpret_cast<uint2*>(qr), sr,
                        reinterpret_cast<uint4*>(qc), sc));
  count_launches(1);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

// mode: MOE_QUANT_ROW / COL / ROW_TILED / COL_TILED / ROW_TILED_GATEUP (G = gate rows per stack)
int launch_quantize(const void* src, int64_t rows, int cols, int mode, int64_t G, uint8_t* q,
                    uint8_t* s, cudaStream_t st) {
  const bool row = mode == MOE_QUANT_ROW || mode == MOE_QUANT_ROW_TILED ||
                   mode == MOE_QUANT_ROW_TILED_GATEUP;
  const int layout = (mode == MOE_QUANT_ROW || mode == MOE_QUANT_COL) ? 0
                     : (mode == MOE_QUANT_ROW_TILED_GATEUP)           ? 2
                                                                       : 1;
  if (row) {
    const int64_t nb = rows * (cols / 32);
    const int64_t grid = (nb + 255) / 256;
    MOE_LAUNCH(launch_pdl(quant_row_kernel, (unsigned)grid, 256, 0, st, static_cast<const uint4*>(src), nb, cols / 32,
                                                      layout, G, reinterpret_cast<uint4*>(q), s));
  } else {
    const int64_t nt = (rows / 32) * (cols / 4);
    const int64_t grid = (nt + 127) / 128;
    MOE_LAUNCH(launch_pdl(quant_col_kernel, (unsigned)grid, 128, 0, st, static_cast<const uint2*>(src), rows, cols,
                                                      layout, reinterpret_cast<uint32_t*>(q), s));
  }
  count_launches(1);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

}  // namespace moe
