// Device-scheduled grouped GEMM on the 5th-generation tensor cores (tcgen05), the one dense
// contraction of the MoE layer ("grouped GEMM combines many small expert computations",
// bytechap.com "Como funciona"; "device-scheduled grouped matrix multiplications that make expert
// parallelism completely synchronisation-free", unite.ai "Parallelismo, precisione e tecniche di
// memoria").
//
// Structure (one persistent CTA per SM, or CTA pair per two SMs; 192 threads each, 320 with eight
// epilogue warps):
//   warp 0      TMA producer: one elected thread streams A/B tiles into a STAGES-deep shared-memory
//               ring (128-byte swizzle), completion counted on a "full" mbarrier per stage;
//   warp 1      allocates TMEM; one thread issues tcgen05.mma (M=128, N=BN, fp32 accumulate) into
//               one of NACC TMEM accumulators and frees each ring stage with tcgen05.commit;
//   warps 2..5  epilogue: tcgen05.ld the finished accumulator (one row per thread), apply the fused
//               op (store, SwiGLU forward, SwiGLU backward, fp32 + bias) and store to global memory
//               (TMA stores of staged boxes; the SwiGLU forward's a and the quantised codes straight
//               from registers), while the MMA thread already fills the other accumulator (NACC = 2).
//               The 256-column MXFP8 tiles have one accumulator, their scale columns filling the rest
//               of TMEM; for the plain stores of those tiles eight epilogue warps (2..9) copy it into
//               registers and hand it back before converting and storing.
// The tile schedule is built on the device from the routing metadata (counts, padded offsets): the
// host never learns the group sizes. Two grouping modes:
//   GROUP_M  ragged rows per expert (forward and dgrad): tiles (expert, n-block, m-block), m fastest
//            so CTAs running at the same time share the expert's weight block through L2;
//   GROUP_K  ragged contraction per expert (wgrad): tiles (expert, m-block, n-block), the K loop runs
//            over the expert's 32-aligned row range in 32-row chunks (zero pad rows make the tail
//            exact); an expert with no rows writes a zero gradient. Without experts, the same mode
//            splits one long contraction into fixed chunks with one fp32 partial each (router dW_r).
// CTA pairs (PAIR, a cluster of two CTAs on neighbouring SMs): a tile covers 256 rows; each CTA
// loads its 128 rows of A and half of B's columns into its own shared memory (TMA with
// .cta_group::2, completing on the leader's barrier, no multicast), the leader's MMA thread issues
// tcgen05.mma.cta_group::2 (M=256) that reads both CTAs' shared memory and writes each CTA's 128
// accumulator rows into that CTA's TMEM, and its commits arrive on both CTAs' barriers. Each CTA's
// epilogue drains its own rows and releases the accumulator with a remote arrive on the leader.
// A pair tile with at most 128 of its group's rows left (an expert's ragged tail) runs as an M = 128
// pair MMA instead: each CTA holds 64 rows of A, and its accumulator keeps those 64 rows with output
// columns [0, BN/2) in TMEM lanes 0-63 and [BN/2, BN) in lanes 64-127, so no tensor work goes to
// rows past the group.
// Every mbarrier wait is bounded; on a timeout the CTA raises MOE_DEVERR_TIMEOUT, drains what it has
// in flight (bounded), frees TMEM and returns.
#include "internal.h"

namespace moe {

namespace {

constexpr int BM = 128;

constexpr int kSmemBudget = 232448;  // 227 KB of opt-in shared memory per CTA
constexpr int kCtrlBytes = 2048;      // mbarriers, TMEM slot, abort word, tile prefix [<=257 ints]

constexpr bool epi_swiglu_fwd(int e) { return e == EPI_SWIGLU_FWD || e == EPI_SWIGLU_FWD_Q; }
constexpr bool epi_swiglu_bwd(int e) { return e == EPI_SWIGLU_BWD || e == EPI_SWIGLU_BWD_Q; }
constexpr bool epi_quant(int e) { return e == EPI_SWIGLU_FWD_Q || e == EPI_SWIGLU_BWD_Q; }

template <int ES, bool A_MN, bool B_MN, int BN, int EPI, int MODE, bool PAIR>
struct Cfg {
  // PAIR: a cluster of two CTAs computes a 256-row tile with cta_group::2 MMAs; each CTA holds 128
  // rows of A, half of B's BN columns, and its 128 accumulator rows in its own tensor memory.
  static constexpr int TILE_M = PAIR ? 2 * BM : BM;  // output rows per tile
  static constexpr int TILE_N = BN;                  // accumulator columns per tile
  static constexpr int BN_CTA = PAIR ? BN / 2 : BN;  // rows of B (along N) held by one CTA
  static constexpr int EPR = 128 / ES;       // elements per 128-byte smem row
  // K elements per pipeline stage: one 128-byte row, except for the bf16 wgrads on CTA pairs (both
  // operands MN-major), whose short contractions take 128 rows per stage. Each stage costs the MMA
  // thread a barrier wait and a commit that the tensor pipe does not overlap, and a pair's halved
  // B share leaves room for three such stages.
  static constexpr int BK = (ES == 2 && MODE == GROUP_K && PAIR) ? 2 * EPR : EPR;
  static constexpr int UK = 32 / ES;         // K per tcgen05.mma (32 bytes)
  static constexpr int KSTEPS = BK / UK;     // MMAs per full stage (4)
  static constexpr int CHUNKS = BK / 32;     // 32-row K chunks per stage (MN-major operands)
  static constexpr int A_BYTES = BM * BK * ES;
  static constexpr int B_BYTES = BN_CTA * BK * ES;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  // output staging: each epilogue warp owns NBUF swizzled 32-row x 128-byte boxes
  static constexpr bool MX = (ES == 1);      // MXFP8 block-scaled (E4M3 operands, UE8M0 scales)
  static_assert(!(PAIR && MX), "block-scaled MMAs run on single CTAs");
  // epilogue warps: four (one per TMEM lane quadrant), or eight (two per quadrant, each taking half
  // of the accumulator columns) for the MXFP8 plain-store tiles of 256 columns (fwd2, dgrad1, wgrads),
  // which hold one accumulator (below). There each thread reads its 128 accumulator columns into
  // registers and hands the accumulator back before it converts and stores them, so the next tile's
  // MMAs overlap the stores. The stores go through a 2 KB transpose buffer per warp (plain
  // shared-memory stores and loads, whole 64-byte row segments to global memory) instead of TMA
  // staging boxes; for the wgrads that leaves room for a fourth pipeline stage, so a tile's short
  // contraction (512 routed rows at the MXFP8 shapes) is loaded while the previous tile computes.
  static constexpr int EPW = (ES == 1 && BN == 256 && !PAIR && EPI == EPI_STORE) ? 8 : 4;
  static constexpr bool EARLY = EPW == 8;
  static constexpr int THREADS = 64 + 32 * EPW;  // producer, MMA issuer, epilogue
  static constexpr int OES = (EPI == EPI_STORE_F32_BIAS) ? 4 : (MX ? 2 : ES);  // output element size
  static constexpr int OEPR = 128 / OES;     // output columns per staged box
  // accumulators in TMEM: two (the epilogue drains one while the MMA fills the other), or one for
  // MXFP8 tiles of 256 columns, whose per-stage scale columns leave no room for a second
  static constexpr int NACC = (MX && BN == 256) ? 1 : 2;
  static_assert(!epi_quant(EPI) || (MX && !PAIR), "quantising epilogues are MXFP8-only");
  // staging boxes per epilogue warp: SwiGLU forward h13 gate + up (a, or a's codes when quantising,
  // goes straight from registers to global memory); SwiGLU backward dh13 gate + up (quantising: none,
  // dh13's codes go straight to global memory); plain stores round robin over NBUF boxes, one where
  // a single accumulator makes the MMA wait for the epilogue (a deeper ring pays more there than a
  // second box).
  // The early-release wgrad epilogue uses no boxes (its transpose buffers are sized below).
  static constexpr int NBUF = (EPI == EPI_SWIGLU_FWD) ? 2
                              : (EPI == EPI_SWIGLU_FWD_Q) ? 2
                              : (EPI == EPI_SWIGLU_BWD_Q) ? 0
                              : (EPI == EPI_SWIGLU_BWD) ? 2
                              : (NACC == 1 ? 1 : 2);
  static constexpr int STAGING_BYTES = EARLY ? EPW * 2048 : EPW * NBUF * 4096;
  static_assert(!EARLY || (NACC == 1 && OES == 2 && EPI == EPI_STORE), "early release: bf16 stores");
  static_assert(STAGING_BYTES % (EPW * 1024) == 0, "per-warp staging: whole, 1 KB aligned slices");
  // MXFP8: per stage, one 512-byte scale chunk per 128 rows of A and of B (TMEM: 4 columns each)
  static constexpr int SF_BYTES = MX ? 512 + (BN / 128) * 512 : 0;
  static constexpr int SF_COLS = MX ? 4 + 4 * (BN / 128) : 0;
  static constexpr int STAGES_FIT =
      (kSmemBudget - kCtrlBytes - 1024 - STAGING_BYTES) / (STAGE_BYTES + SF_BYTES);
  static constexpr int STAGES = STAGES_FIT > 8 ? 8 : STAGES_FIT;
  static_assert(STAGES >= 2, "pipeline too shallow");
  static constexpr int TMEM_COLS = MX ? 512 : 2 * BN;  // accumulators (+ scale columns)
  static_assert(!MX || NACC * BN + STAGES * SF_COLS <= 512, "TMEM overflow");
  static constexpr int BN_OUT = epi_swiglu_fwd(EPI) ? BN / 2 : BN;  // output columns per tile
  static constexpr uint32_t IDESC =
      MX ? instr_desc_mx(A_MN, B_MN, BM, BN) : instr_desc(ES == 2 ? 1u : 2u, A_MN, B_MN, TILE_M, BN);
  // pair tail tile: M = 128 over the pair, HALF_M rows of A per CTA
  static constexpr int HALF_M = BM / 2;
  static constexpr uint32_t IDESC_HALF = PAIR ? instr_desc(ES == 2 ? 1u : 2u, A_MN, B_MN, BM, BN) : IDESC;
  // MN-major operands: 16-bit types use the plain 128B swizzle (8-row atoms of 1 KB); 32-bit (tf32)
  // operands need the 128B swizzle with 32-byte chunks (4-row atoms of 512 B).
  static constexpr uint32_t MN_LAYOUT = ES == 4 ? kLayoutSW128Atom32 : kLayoutSW128;
  static constexpr uint32_t MN_SBO = ES == 4 ? 512 : 1024;
  static constexpr size_t SMEM_BYTES =
      kCtrlBytes + 1024 /*alignment slack*/ + (size_t)STAGES * (STAGE_BYTES + SF_BYTES) +
      STAGING_BYTES;
  static_assert(SMEM_BYTES <= (size_t)kSmemBudget, "over the opt-in shared memory per CTA");
  static_assert(A_BYTES % 1024 == 0 && B_BYTES % 1024 == 0,
                "stage operands start on 1 KB boundaries (128-byte swizzle atoms)");
  static_assert(SF_BYTES % 16 == 0, "scale chunks are bulk-copied in 16-byte units");
  static_assert(TMEM_COLS >= 32 && TMEM_COLS <= 512 && (TMEM_COLS & (TMEM_COLS - 1)) == 0,
                "TMEM is allocated in powers of two from 32 to 512 columns");
};

// One tile of the device schedule. lo / hi are the group's row range as read from the routing
// metadata: GROUP_M the group's padded routed rows [lo, hi), GROUP_K its contraction rows [lo, hi).
// They are kept raw, so that a role can fetch the next tile's entry while it works on the current
// one and only use the loaded values a tile later (the loads then never stall the loop).
struct TileInfo {
  int e;   // group
  int m0;  // GROUP_M: first row relative to the group start; GROUP_K: first output row
  int n0;  // first output column
  int lo, hi;
};

template <int MODE>
__device__ __forceinline__ int ti_rows(const TileInfo& ti, const GemmParams& p) {
  return MODE == GROUP_M ? ti.hi - ti.lo : p.M;  // GROUP_M: padded rows of the group
}
__device__ __forceinline__ int ti_row_base(const TileInfo& ti) { return ti.lo; }  // GROUP_M
__device__ __forceinline__ int ti_kstart(const TileInfo& ti) { return ti.lo; }    // GROUP_K

// A pair tile with at most BM of its group's rows left runs as an M = 128 pair MMA (64 rows per CTA).
template <bool PAIR, int MODE>
__device__ __forceinline__ bool ti_half(const TileInfo& ti, const GemmParams& p) {
  if constexpr (PAIR && MODE == GROUP_M) return ti_rows<MODE>(ti, p) - ti.m0 <= BM;
  else return false;
}

// K stages of a tile: GROUP_M K/BK; GROUP_K the group's 32-row contraction chunks, CHUNKS per stage
template <class C, int MODE>
__device__ __forceinline__ int ti_nchunks(const TileInfo& ti, const GemmParams& p) {
  if constexpr (MODE == GROUP_M) return p.K / C::BK;
  else return (ti.hi - ti.lo + 31) / 32;
}

// GROUP_K: number of output groups (experts, contraction splits, or one)
__host__ __device__ __forceinline__ int k_groups(const GemmParams& p) {
  if (p.counts) return p.E;
  if (p.ksplit) return (p.K + p.ksplit - 1) / p.ksplit;
  return 1;
}

template <class C, int MODE>
__device__ __forceinline__ int num_kstages(const TileInfo& ti, const GemmParams& p) {
  if constexpr (MODE == GROUP_M) return ti_nchunks<C, MODE>(ti, p);
  else return (ti_nchunks<C, MODE>(ti, p) + C::CHUNKS - 1) / C::CHUNKS;
}

// GROUP_M: m-tiles of group e, from the shared-memory tile prefix (no global load)
__device__ __forceinline__ int prefix_m_tiles(const int* prefix, int e, int n_tiles) {
  return (prefix[e + 1] - prefix[e]) / n_tiles;
}

// The device tile schedule as every role of a CTA sees it. GROUP_M: prefix[e] = first tile of group
// e (inclusive scan of its tile counts). GROUP_K: prefix[e] = poff[e] (the groups' contraction row
// ranges, staged in shared memory) and a fixed m_tiles x n_tiles block of tiles per group, whose
// index is split by multiply-shift division.
struct Sched {
  const int* prefix;
  int n_tiles, m_tiles_fixed, total;
  FastDiv per_group, per_row;  // GROUP_K: divisors m_tiles_fixed * n_tiles and n_tiles
};

template <class C, int EPI, int MODE>
__device__ __forceinline__ void tile_info(int tile, const GemmParams& p, const Sched& sch, TileInfo& ti) {
  const int* prefix = sch.prefix;
  const int n_tiles = sch.n_tiles;
  if constexpr (MODE == GROUP_M) {
    int e = 0;
    if (p.counts) {
      int lo = 0, hi = p.E - 1;  // largest e with prefix[e] <= tile
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (prefix[mid] <= tile) lo = mid; else hi = mid - 1;
      }
      e = lo;
    }
    const int local = tile - prefix[e];
    const int mt = prefix_m_tiles(prefix, e, n_tiles);
    ti.e = e;
    ti.n0 = (local / mt) * C::BN_OUT;
    ti.m0 = (local % mt) * C::TILE_M;
    if (p.counts) {
      ti.lo = p.poff[e];
      ti.hi = p.poff[e + 1];
    } else {
      ti.lo = 0;
      ti.hi = p.M;
    }
  } else {
    const int e = sch.per_group.div(tile);
    const int local = tile - e * sch.per_group.d;
    const int mi = sch.per_row.div(local);
    ti.e = e;
    ti.m0 = mi * C::TILE_M;
    ti.n0 = (local - mi * n_tiles) * C::TILE_N;
    if (p.counts) {
      ti.lo = prefix[e];
      ti.hi = prefix[e + 1];
    } else if (p.ksplit) {
      ti.lo = e * p.ksplit;
      ti.hi = min(p.K, ti.lo + p.ksplit);
    } else {
      ti.lo = 0;
      ti.hi = p.K;
    }
  }
}

// Round an fp32 value to the output element type (bf16 for 2-byte outputs) and back.
template <int OES>
__device__ __forceinline__ float round_out(float v) {
  if constexpr (OES == 2) return __bfloat162float(__float2bfloat16_rn(v));
  else return v;
}

// SwiGLU helpers with the fast exponential and division intrinsics (bf16 outputs need ~8 bits).
__device__ __forceinline__ float silu_f(float g) { return __fdividef(g, 1.f + __expf(-g)); }

// Write 32 fp32 values of this thread's row into a staged box (row `lane`, 128 bytes, 128B swizzle:
// 16-byte chunk j of row r sits at chunk j ^ (r & 7)) as OES-byte elements, starting at chunk `ch0`.
template <int OES>
__device__ __forceinline__ void stage_row32(uint8_t* box, int lane, int ch0, const float* v) {
  uint8_t* row = box + lane * 128;
  if constexpr (OES == 2) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint4 w = make_uint4(pack_bf16(v[8 * q + 0], v[8 * q + 1]), pack_bf16(v[8 * q + 2], v[8 * q + 3]),
                                 pack_bf16(v[8 * q + 4], v[8 * q + 5]), pack_bf16(v[8 * q + 6], v[8 * q + 7]));
      st_shared_v4(row + (((ch0 + q) ^ (lane & 7)) << 4), w);
    }
  } else {
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const uint4 w = make_uint4(__float_as_uint(v[4 * q]), __float_as_uint(v[4 * q + 1]),
                                 __float_as_uint(v[4 * q + 2]), __float_as_uint(v[4 * q + 3]));
      st_shared_v4(row + (((ch0 + q) ^ (lane & 7)) << 4), w);
    }
  }
}

// Store 32 fp32 values of this thread's row to global memory as OES-byte elements (16-byte stores).
template <int OES>
__device__ __forceinline__ void store_row32_global(uint8_t* dst, const float* v) {
  uint4* d = reinterpret_cast<uint4*>(dst);
  if constexpr (OES == 2) {
#pragma unroll
    for (int q = 0; q < 4; ++q)
      d[q] = make_uint4(pack_bf16(v[8 * q + 0], v[8 * q + 1]), pack_bf16(v[8 * q + 2], v[8 * q + 3]),
                        pack_bf16(v[8 * q + 4], v[8 * q + 5]), pack_bf16(v[8 * q + 6], v[8 * q + 7]));
  } else {
#pragma unroll
    for (int q = 0; q < 8; ++q)
      d[q] = make_uint4(__float_as_uint(v[4 * q]), __float_as_uint(v[4 * q + 1]),
                        __float_as_uint(v[4 * q + 2]), __float_as_uint(v[4 * q + 3]));
  }
}

// Store 32 one-byte codes (8 words, column order) of this thread's row: one whole, aligned 32-byte
// sector of the [rows, cols] code array (the chunk's first column is a multiple of 32).
__device__ __forceinline__ void store_codes32(uint8_t* dst, const uint32_t (&c)[8]) {
  uint4* d = reinterpret_cast<uint4*>(dst);
  d[0] = make_uint4(c[0], c[1], c[2], c[3]);
  d[1] = make_uint4(c[4], c[5], c[6], c[7]);
}

// Hand a fully written box to the TMA unit: every lane fences its writes, lane 0 stores the box.
__device__ __forceinline__ void box_store(const CUtensorMap* map, const uint8_t* box, int lane, int c0,
                                          int c1) {
  fence_proxy_async_smem();
  __syncwarp();
  if (lane == 0) {
    tma_store_2d(map, box, c0, c1);
    bulk_commit();
  }
}

// 32 stored values (bf16 or fp32) as raw 16-byte words, and their unpacking to fp32.
template <int ES>
__device__ __forceinline__ void raw_load32(const void* src, uint4* w) {
  const uint4* s = reinterpret_cast<const uint4*>(src);
#pragma unroll
  for (int q = 0; q < 2 * ES; ++q) w[q] = s[q];
}
template <int ES>
__device__ __forceinline__ void unpack32(const uint4* w, float* v) {
  if constexpr (ES == 2) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      v[8 * q + 0] = bf16lo(w[q].x); v[8 * q + 1] = bf16hi(w[q].x);
      v[8 * q + 2] = bf16lo(w[q].y); v[8 * q + 3] = bf16hi(w[q].y);
      v[8 * q + 4] = bf16lo(w[q].z); v[8 * q + 5] = bf16hi(w[q].z);
      v[8 * q + 6] = bf16lo(w[q].w); v[8 * q + 7] = bf16hi(w[q].w);
    }
  } else {
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      v[4 * q] = __uint_as_float(w[q].x); v[4 * q + 1] = __uint_as_float(w[q].y);
      v[4 * q + 2] = __uint_as_float(w[q].z); v[4 * q + 3] = __uint_as_float(w[q].w);
    }
  }
}

template <int ES, bool A_MN, bool B_MN, int BN, int EPI, int MODE, bool PAIR>
__global__ void __launch_bounds__(Cfg<ES, A_MN, B_MN, BN, EPI, MODE, PAIR>::THREADS, 1)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmA,
                        const __grid_constant__ CUtensorMap tmB,
                        const __grid_constant__ CUtensorMap tmC,
                        const __grid_constant__ CUtensorMap tmX1,
                        const __grid_constant__ CUtensorMap tmX2, const GemmParams p) {
  // tmX1 / tmX2: pair tail tiles -- 64-row boxes of A / of B (SwiGLU forward)
  const CUtensorMap& tmA64 = tmX1;
  const CUtensorMap& tmB64 = tmX2;
  using C = Cfg<ES, A_MN, B_MN, BN, EPI, MODE, PAIR>;
  static_assert(MODE == GROUP_M || (A_MN && B_MN), "wgrad mode needs MN-major operands");
  extern __shared__ __align__(16) uint8_t smem_raw[];
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem_raw);  // control area first
  const uint32_t data_addr = smem_u32(smem_raw) + kCtrlBytes;
  uint8_t* smem = smem_raw + kCtrlBytes + (((data_addr + 1023u) & ~1023u) - data_addr);
  uint8_t* smA = smem;
  uint8_t* smB = smem + (size_t)C::STAGES * C::A_BYTES;
  uint8_t* stg = smB + (size_t)C::STAGES * C::B_BYTES;  // epilogue staging, 1 KB aligned
  uint8_t* sfs = stg + C::STAGING_BYTES;                  // MXFP8 scale chunks, per stage
  uint64_t* full = bars;
  uint64_t* empty = bars + C::STAGES;
  uint64_t* tfull = bars + 2 * C::STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* done = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  volatile int* abort_word = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* prefix = reinterpret_cast<int*>(tmem_slot + 2);  // [E+1]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // CTA pairs walk the tile list together: pair index = cluster index, rank 0 = leader
  const uint32_t rank = PAIR ? cluster_ctarank() : 0u;
  const int tile0 = PAIR ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;
  const int tstep = PAIR ? (int)(gridDim.x >> 1) : (int)gridDim.x;
  pdl_trigger();  // the next kernel may be scheduled as SMs free up

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      // single CTA: every epilogue thread arrives; pair: lane 0 of every epilogue warp of each CTA
      mbar_init(&tempty[b], PAIR ? 2 * C::EPW : C::EPW * 32);
    }
    mbar_init(done, 1);
    *abort_word = 0;
    if constexpr (PAIR) fence_barrier_init_cluster();
    else fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&tmA);
    prefetch_tensormap(&tmB);
    prefetch_tensormap(&tmC);
    if constexpr (PAIR && MODE == GROUP_M) {
      prefetch_tensormap(&tmA64);
      if constexpr (EPI == EPI_SWIGLU_FWD) prefetch_tensormap(&tmB64);
    }
  }
  if (warp == 1) {
    if constexpr (PAIR) {
      tmem_alloc_pair(tmem_slot, C::TMEM_COLS);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(tmem_slot, C::TMEM_COLS);
      tmem_relinquish();
    }
  }
  // Local setup above touches no global memory; wait here for the previous kernel in the stream
  // (the routing metadata and operands it wrote) before building the schedule from it.
  pdl_wait();

  // ---- device-side tile schedule ----
  int n_tiles, m_tiles_fixed = 0, total;
  if constexpr (MODE == GROUP_M) {
    n_tiles = (p.N + C::BN_OUT - 1) / C::BN_OUT;
    const int G = p.counts ? p.E : 1;
    for (int e = threadIdx.x; e < G; e += blockDim.x) {
      const int rows = p.counts ? (p.poff[e + 1] - p.poff[e]) : p.M;
      prefix[e + 1] = ((rows + C::TILE_M - 1) / C::TILE_M) * n_tiles;
    }
    __syncthreads();
    if (warp == 0) {  // inclusive scan of per-group tile counts, 8 groups per lane
      int loc[8], s = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int e = lane * 8 + i;
        loc[i] = e < G ? prefix[e + 1] : 0;
        s += loc[i];
      }
      int inc = s;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int o = __shfl_up_sync(0xffffffffu, inc, off);
        if (lane >= off) inc += o;
      }
      int run = inc - s;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int e = lane * 8 + i;
        run += loc[i];
        if (e < G) prefix[e + 1] = run;
      }
      if (lane == 0) prefix[0] = 0;
    }
    __syncthreads();
    total = prefix[p.counts ? p.E : 1];
  } else {
    n_tiles = (p.N + BN - 1) / BN;
    m_tiles_fixed = (p.M + C::TILE_M - 1) / C::TILE_M;
    total = k_groups(p) * m_tiles_fixed * n_tiles;
    if (p.counts)
      for (int e = threadIdx.x; e <= p.E; e += blockDim.x) prefix[e] = p.poff[e];
  }
  Sched sch;
  sch.prefix = prefix;
  sch.n_tiles = n_tiles;
  sch.m_tiles_fixed = m_tiles_fixed;
  sch.total = total;
  if constexpr (MODE == GROUP_K) {
    sch.per_group = FastDiv(max(1, m_tiles_fixed * n_tiles));
    sch.per_row = FastDiv(max(1, n_tiles));
  }

  tc_fence_before();
  __syncthreads();
  if constexpr (PAIR) cluster_sync();  // both CTAs' barriers exist before either signals the other
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // leader's barriers as shared::cluster addresses (pair: TMA completion and accumulator release)
  const uint32_t full_lead = PAIR ? cluster_addr(full, 0) : 0u;
  const uint32_t tempty_lead = PAIR ? cluster_addr(tempty, 0) : 0u;

  if (warp == 0) {
    // ===================== TMA producer =====================
    if (lane == 0 && PAIR) {
      // Both CTAs of a pair load their own halves (A rows m0 + 128*rank, B columns n0 +
      // BN/2*rank) into their own shared memory; every copy completes on the leader's full barrier,
      // which the leader arms with the bytes of both halves. A half past the group's rows is not
      // loaded (its accumulator rows are never stored).
      int it = 0;
      bool ok = true;
      TileInfo nxt;  // the next tile's entry is fetched a tile ahead
      if (tile0 < total) tile_info<C, EPI, MODE>(tile0, p, sch, nxt);
      for (int tile = tile0; tile < total && ok; tile += tstep) {
        const TileInfo ti = nxt;
        if (tile + tstep < total) tile_info<C, EPI, MODE>(tile + tstep, p, sch, nxt);
        const int nst = num_kstages<C, MODE>(ti, p);
        // tail tile (<= BM rows left): 64 rows of A per CTA for an M = 128 pair MMA
        const bool half = ti_half<PAIR, MODE>(ti, p);
        const int cta_rows = half ? C::HALF_M : BM;
        const uint32_t a_bytes = (uint32_t)cta_rows * C::BK * ES;
        const bool a0 = ti.m0 < ti_rows<MODE>(ti, p), a1 = ti.m0 + cta_rows < ti_rows<MODE>(ti, p);
        const bool mine = rank == 0 ? a0 : a1;
        const uint32_t tx = (a0 ? a_bytes : 0) + (a1 ? a_bytes : 0) + 2 * C::B_BYTES;
        const int m_cta = ti.m0 + (int)rank * cta_rows;
        const int n_cta = ti.n0 + (int)rank * C::BN_CTA;
        for (int ks = 0; ks < nst; ++ks, ++it) {
          const int s = it % C::STAGES;
          if (!mbar_wait_bounded(&empty[s], ((it / C::STAGES) & 1) ^ 1, p.wait_limit_ns, abort_word,
                                 p.err)) {
            ok = false;
            break;
          }
          uint8_t* a_dst = smA + (size_t)s * C::A_BYTES;
          uint8_t* b_dst = smB + (size_t)s * C::B_BYTES;
          const uint32_t fb = full_lead + 8u * (uint32_t)s;
          if (rank == 0) mbar_arrive_expect_tx(&full[s], tx);
          if constexpr (MODE == GROUP_M) {
            const int k0 = ks * C::BK;
            if (mine) tma_load_2d_pair(a_dst, half ? &tmA64 : &tmA, fb, k0, ti_row_base(ti) + m_cta);
            const int brow = ti.e * p.b_rows_per_group;
            if constexpr (B_MN) {
              tma_load_3d_pair(b_dst, &tmB, fb, 0, brow + k0, n_cta / C::EPR);
            } else if constexpr (epi_swiglu_fwd(EPI)) {
              if (!half) {
                // leader: the gate rows of the tile's outputs; peer: the matching up rows
                tma_load_2d_pair(b_dst, &tmB, fb, k0, brow + (rank ? p.F : 0) + ti.n0);
              } else {
                // M = 128: the accumulator's lanes 0-63 take B columns [0, BN/2) (the leader's half),
                // lanes 64-127 columns [BN/2, BN) (the peer's). Each CTA loads 64 gate rows and the
                // 64 matching up rows, so each lane holds gate and up for the same output columns.
                const int g0 = brow + ti.n0 + (int)rank * (BN / 4);
                tma_load_2d_pair(b_dst, &tmB64, fb, k0, g0);
                tma_load_2d_pair(b_dst + (BN / 4) * 128, &tmB64, fb, k0, g0 + p.F);
              }
            } else {
              tma_load_2d_pair(b_dst, &tmB, fb, k0, brow + n_cta);
            }
          } else {
            const int krow0 = ti_kstart(ti) + ks * C::CHUNKS * 32;
            if (mine) tma_load_3d_pair(a_dst, &tmA, fb, 0, krow0, m_cta / C::EPR);
            tma_load_3d_pair(b_dst, &tmB, fb, 0, krow0, n_cta / C::EPR);
          }
        }
      }
      // drain: the leader's MMAs have consumed every stage this CTA filled (so its copies have
      // landed) before the CTA exits
      for (int j = max(0, it - C::STAGES); j < it; ++j)
        mbar_wait_bounded(&empty[j % C::STAGES], (j / C::STAGES) & 1, p.wait_limit_ns, nullptr, p.err);
    } else if (lane == 0) {
      int it = 0;
      bool ok = true;
      TileInfo nxt;  // the next tile's entry is fetched a tile ahead
      if (tile0 < total) tile_info<C, EPI, MODE>(tile0, p, sch, nxt);
      for (int tile = tile0; tile < total && ok; tile += tstep) {
        const TileInfo ti = nxt;
        if (tile + tstep < total) tile_info<C, EPI, MODE>(tile + tstep, p, sch, nxt);
        const int nst = num_kstages<C, MODE>(ti, p);
        for (int ks = 0; ks < nst; ++ks, ++it) {
          const int s = it % C::STAGES;
          if (!mbar_wait_bounded(&empty[s], ((it / C::STAGES) & 1) ^ 1, p.wait_limit_ns, abort_word,
                                 p.err)) {
            ok = false;
            break;
          }
          uint8_t* a_dst = smA + (size_t)s * C::A_BYTES;
          uint8_t* b_dst = smB + (size_t)s * C::B_BYTES;
          const uint8_t* sf_a = nullptr;
          const uint8_t* sf_b = nullptr;
          uint8_t* sf_dst = nullptr;
          int64_t b_chunk_step = 0;
          if constexpr (C::MX) {
            // this stage's scales: one 512-byte chunk for the 128 rows of A, one per 128 of B
            uint8_t* sf = sfs + (size_t)s * C::SF_BYTES;
            int64_t amb, akq, bmb, bkq;
            if constexpr (MODE == GROUP_M) {
              amb = ((int64_t)ti_row_base(ti) + ti.m0) >> 7;
              akq = ks;
              if constexpr (B_MN) {
                bmb = ti.n0 >> 7;
                bkq = (int64_t)ti.e * (p.b_rows_per_group >> 7) + ks;
              } else if constexpr (epi_swiglu_fwd(EPI)) {
                bmb = ((int64_t)ti.e * p.b_rows_per_group + ti.n0) >> 7;  // gate rows n0..n0+BN/2-1
                bkq = ks;
              } else {
                bmb = ((int64_t)ti.e * p.b_rows_per_group + ti.n0) >> 7;
                bkq = ks;
              }
            } else {
              amb = ti.m0 >> 7;
              bmb = ti.n0 >> 7;
              akq = bkq = (ti_kstart(ti) >> 7) + ks;
            }
            sf_a = p.sA + (amb * p.sA_ld + akq) * 512;
            sf_b = p.sB + (bmb * p.sB_ld + bkq) * 512;
            // the tile's second 128 B rows: the next chunk row, or for the fused SwiGLU tile (gate
            // rows, then the up rows F further down W13) the chunk row F/128 further
            b_chunk_step = (epi_swiglu_fwd(EPI) ? (int64_t)(p.F >> 7) : 1) * p.sB_ld * 512;
            sf_dst = sf;
          }
          if constexpr (MODE == GROUP_M) {
            const int k0 = ks * C::BK;
            mbar_arrive_expect_tx(&full[s], C::STAGE_BYTES + C::SF_BYTES);
            if constexpr (C::MX) {
              bulk_load(sf_dst, sf_a, 512, &full[s]);
#pragma unroll
              for (int c = 0; c < BN / 128; ++c)  // B: one chunk per 128 rows of the tile
                bulk_load(sf_dst + 512 * (c + 1), sf_b + (int64_t)c * b_chunk_step, 512, &full[s]);
            }
            // A: K-major rows of the routed buffer (or the token matrix)
            tma_load_2d(a_dst, &tmA, &full[s], k0, ti_row_base(ti) + ti.m0);
            if constexpr (!B_MN) {
              const int brow = ti.e * p.b_rows_per_group;
              if constexpr (epi_swiglu_fwd(EPI)) {
                tma_load_2d(b_dst, &tmB, &full[s], k0, brow + ti.n0);                       // gate
                tma_load_2d(b_dst + (BN / 2) * 128, &tmB, &full[s], k0, brow + p.F + ti.n0);  // up
              } else {
                tma_load_2d(b_dst, &tmB, &full[s], k0, brow + ti.n0);
              }
            } else {
              // MN-major weight [E*K rows, N cols]: BN/EPR column blocks x BK rows
              const int krow = ti.e * p.b_rows_per_group + k0;
              if (p.b_box3d) {
                tma_load_3d(b_dst, &tmB, &full[s], 0, krow, ti.n0 / C::EPR);
              } else {
#pragma unroll
                for (int blk = 0; blk < BN / C::EPR; ++blk)
#pragma unroll
                  for (int ch = 0; ch < C::CHUNKS; ++ch)
                    tma_load_2d(b_dst + blk * (C::BK * 128) + ch * 4096, &tmB, &full[s],
                                ti.n0 + blk * C::EPR, krow + ch * 32);
              }
            }
          } else {
            // GROUP_K: both operands MN-major, contraction rows kstart + 32*chunk. A 3-D box always
            // brings BK rows; in the group's last stage the rows past its end (the next group's, or
            // zero fill past the tensor) land in shared memory but the MMA loop stops before them.
            const int c0 = ks * C::CHUNKS;
            const int nch = min(C::CHUNKS, ti_nchunks<C, MODE>(ti, p) - c0);
            const int krow0 = ti_kstart(ti) + c0 * 32;
            const uint32_t a_bytes = p.a_box3d ? C::A_BYTES : nch * 32 * 128 * (BM / C::EPR);
            const uint32_t b_bytes = p.b_box3d ? C::B_BYTES : nch * 32 * 128 * (BN / C::EPR);
            mbar_arrive_expect_tx(&full[s], a_bytes + b_bytes + C::SF_BYTES);
            if constexpr (C::MX) {
              bulk_load(sf_dst, sf_a, 512, &full[s]);
#pragma unroll
              for (int c = 0; c < BN / 128; ++c)  // B: one chunk per 128 rows of the tile
                bulk_load(sf_dst + 512 * (c + 1), sf_b + (int64_t)c * b_chunk_step, 512, &full[s]);
            }
            if (p.a_box3d) {
              tma_load_3d(a_dst, &tmA, &full[s], 0, krow0, ti.m0 / C::EPR);
            } else {
              for (int ch = 0; ch < nch; ++ch)
#pragma unroll
                for (int blk = 0; blk < BM / C::EPR; ++blk)
                  tma_load_2d(a_dst + blk * (C::BK * 128) + ch * 4096, &tmA, &full[s],
                              ti.m0 + blk * C::EPR, krow0 + ch * 32);
            }
            if (p.b_box3d) {
              tma_load_3d(b_dst, &tmB, &full[s], 0, krow0, ti.n0 / C::EPR);
            } else {
              for (int ch = 0; ch < nch; ++ch)
#pragma unroll
                for (int blk = 0; blk < BN / C::EPR; ++blk)
                  tma_load_2d(b_dst + blk * (C::BK * 128) + ch * 4096, &tmB, &full[s],
                              ti.n0 + blk * C::EPR, krow0 + ch * 32);
            }
          }
        }
      }
      // drain: every load this thread issued must have landed before the CTA exits
      for (int j = max(0, it - C::STAGES); j < it; ++j)
        mbar_wait_bounded(&full[j % C::STAGES], (j / C::STAGES) & 1, p.wait_limit_ns, nullptr, p.err);
    }
  } else if (warp == 1) {
    // ===================== MMA issuer =====================
    // (a pair's MMAs are issued by the leader alone; they read both CTAs' shared memory and write
    // both CTAs' tensor memory)
    if (lane == 0 && rank == 0) {
      int it = 0, local = 0;
      bool ok = true;
      bool issued = false;
      TileInfo nxt;  // the next tile's entry is fetched a tile ahead
      if (tile0 < total) tile_info<C, EPI, MODE>(tile0, p, sch, nxt);
      for (int tile = tile0; tile < total && ok; tile += tstep, ++local) {
        const TileInfo ti = nxt;
        if (tile + tstep < total) tile_info<C, EPI, MODE>(tile + tstep, p, sch, nxt);
        const int nst = num_kstages<C, MODE>(ti, p);
        const uint32_t idesc = ti_half<PAIR, MODE>(ti, p) ? C::IDESC_HALF : C::IDESC;
        const int buf = local % C::NACC;
        const uint32_t use = (uint32_t)(local / C::NACC) & 1u;  // parity of this buffer's use
        const bool drained =
            PAIR ? mbar_wait_bounded_cluster(&tempty[buf], use ^ 1u, p.wait_limit_ns, abort_word, p.err)
                 : mbar_wait_bounded(&tempty[buf], use ^ 1u, p.wait_limit_ns, abort_word, p.err);
        if (!drained) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + buf * BN;
        for (int ks = 0; ks < nst; ++ks, ++it) {
          const int s = it % C::STAGES;
          if (!mbar_wait_bounded(&full[s], (it / C::STAGES) & 1, p.wait_limit_ns, abort_word, p.err)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(smA + (size_t)s * C::A_BYTES);
          const uint32_t b_addr = smem_u32(smB + (size_t)s * C::B_BYTES);
          int nk = C::KSTEPS;
          if constexpr (MODE == GROUP_K) nk = min(C::CHUNKS, ti_nchunks<C, MODE>(ti, p) - ks * C::CHUNKS) * (32 / C::UK);
          uint32_t sf_col = 0;
          if constexpr (C::MX) {
            // this stage's scales: smem chunks -> TMEM columns after the accumulator(s)
            sf_col = tmem_base + C::NACC * BN + s * C::SF_COLS;
            const uint32_t sf_smem = smem_u32(sfs + (size_t)s * C::SF_BYTES);
#pragma unroll
            for (int c = 0; c < 1 + BN / 128; ++c)
              tmem_cp_32x128b_x4(sf_col + 4 * c, smem_desc(sf_smem + 512 * c, 16, 128, 0));
          }
          for (int kk = 0; kk < nk; ++kk) {
            uint64_t ad, bd;
            if constexpr (A_MN) ad = smem_desc(a_addr + kk * C::UK * 128, C::BK * 128, C::MN_SBO, C::MN_LAYOUT);
            else ad = smem_desc(a_addr + kk * 32, 16, 1024, kLayoutSW128);
            if constexpr (B_MN) bd = smem_desc(b_addr + kk * C::UK * 128, C::BK * 128, C::MN_SBO, C::MN_LAYOUT);
            else bd = smem_desc(b_addr + kk * 32, 16, 1024, kLayoutSW128);
            if constexpr (C::MX) {
              const uint32_t id = C::IDESC | ((uint32_t)kk << 29) | ((uint32_t)kk << 4);
              umma_mx(d_tmem, ad, bd, id, sf_col | ((uint32_t)kk << 30),
                      (sf_col + 4) | ((uint32_t)kk << 30), (ks > 0 || kk > 0) ? 1u : 0u);
            } else if constexpr (PAIR) {
              umma_pair<ES == 2 ? 0 : 1>(d_tmem, ad, bd, idesc, (ks > 0 || kk > 0) ? 1u : 0u);
            } else {
              umma<ES == 2 ? 0 : 1>(d_tmem, ad, bd, C::IDESC, (ks > 0 || kk > 0) ? 1u : 0u);
            }
            issued = true;
          }
          if constexpr (PAIR) umma_commit_pair(&empty[s], 0x3);  // frees the stage in both CTAs
          else umma_commit(&empty[s]);
        }
        if (!ok) break;
        if (nst > 0) {
          if constexpr (PAIR) umma_commit_pair(&tfull[buf], 0x3);
          else umma_commit(&tfull[buf]);
        } else {
          mbar_arrive(&tfull[buf]);
          if constexpr (PAIR) mbar_arrive_cluster(cluster_addr(&tfull[buf], 1));
        }
      }
      // all MMAs issued by this thread must be complete before TMEM is released
      if (issued) {
        if constexpr (PAIR) umma_commit_pair(done, 0x1);
        else umma_commit(done);
        mbar_wait_bounded(done, 0, p.wait_limit_ns, nullptr, p.err);
      }
    }
  } else if (warp >= 2 && warp < 2 + C::EPW) {
    // ===================== epilogue (warps 2..5) =====================
    // Each warp owns the 32 accumulator rows of its TMEM lane quadrant (one row per thread). It
    // stages 32-row x 128-byte boxes in swizzled shared memory and stores them with TMA. A warp's
    // slab of 32 rows is entirely inside or entirely outside its expert's 32-aligned group, so whole
    // slabs are skipped instead of masking rows; columns past N are clipped by the tensor bounds.
    const int q = warp & 3;               // TMEM lane quadrant this warp may access
    const int ew = warp - 2;              // epilogue warp index
    const int chalf = ew >> 2;            // eight epilogue warps: the accumulator column half
    uint8_t* wstg = stg + (size_t)ew * (C::STAGING_BYTES / C::EPW);  // this warp's staging
    int nb = 0;                           // next staging box (round robin)
    int local = 0;
    TileInfo nxt;  // the next tile's entry is fetched a tile ahead
    if (tile0 < total) tile_info<C, EPI, MODE>(tile0, p, sch, nxt);
    for (int tile = tile0; tile < total; tile += tstep, ++local) {
      const TileInfo ti = nxt;
      if (tile + tstep < total) tile_info<C, EPI, MODE>(tile + tstep, p, sch, nxt);
      const int nst = num_kstages<C, MODE>(ti, p);
      const int buf = local % C::NACC;
      int ok = 1;
      if (lane == 0)
        ok = mbar_wait_bounded(&tfull[buf], (uint32_t)(local / C::NACC) & 1u, p.wait_limit_ns,
                               abort_word, p.err);
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      tc_fence_after();
      const uint32_t t_row = tmem_base + ((uint32_t)(q * 32) << 16) + buf * BN + chalf * (BN / 2);
      // Full tile: this warp's 32 rows are rows q*32.. of the CTA's 128, over all BN accumulator
      // columns. Pair tail tile (M = 128): rows (q&1)*32.. of the CTA's 64, over the BN/2 accumulator
      // columns of its lane half, which hold output columns (q>>1)*BN/2 + [0, BN/2) of the tile.
      const bool half = ti_half<PAIR, MODE>(ti, p);
      const int slab = half ? ti.m0 + (int)rank * C::HALF_M + (q & 1) * 32
                            : ti.m0 + (int)rank * BM + q * 32;  // first tile row of this warp
      // output column half: the lane half of a pair tail tile, or this warp's half of the columns
      const int whalf = half ? (q >> 1) : chalf;
      const bool active = slab < ti_rows<MODE>(ti, p);         // warp-uniform
      int c1;                                                  // tensor row of this slab
      if constexpr (MODE == GROUP_K) c1 = ti.e * (p.c_group_rows ? p.c_group_rows : p.M) + slab;
      else c1 = ti_row_base(ti) + slab;
      // Every variant walks the accumulator in 32-column chunks and keeps the TMEM load of the next
      // chunk in flight while it converts and stages the current one; CPB chunks fill one box.
      constexpr int CPB = C::OEPR / 32;
      // quantising epilogues: the warp's 32 rows are one 32-row column block of the routed buffer
      const int64_t qrb = (int64_t)c1 >> 5;
      if constexpr (epi_swiglu_fwd(EPI)) {
        // Full tile: accumulator columns [0, BN/2) gate, [BN/2, BN) up, for output columns
        // n0 + [0, BN/2). Tail tile: [0, BN/4) gate, [BN/4, BN/2) up, for output columns
        // n0 + whalf*BN/4 + [0, BN/4).
        auto swiglu = [&](auto nch_c) {
          constexpr int NCH = decltype(nch_c)::value;  // 32-column chunks of output
          constexpr int UP = NCH * 32;                 // accumulator column of the first up value
          const int col0 = ti.n0 + whalf * UP;         // first output column of this warp
          uint32_t ga[32], ua[32], gb[32], ub[32];
          tmem_ld_32x32b_x32(t_row, ga);
          tmem_ld_32x32b_x32(t_row + UP, ua);
          uint8_t* bg = wstg;
          uint8_t* bu = wstg + 4096;
          uint32_t srow = 0;           // row-block scale bytes of four consecutive chunks
#pragma unroll
          for (int j = 0; j < NCH; ++j) {
            uint32_t(&rg)[32] = (j & 1) ? gb : ga;
            uint32_t(&ru)[32] = (j & 1) ? ub : ua;
            tmem_ld_wait_regs(rg);
            tmem_regs_after(ru);
            if (j + 1 < NCH) {
              tmem_ld_32x32b_x32(t_row + (j + 1) * 32, (j & 1) ? ga : gb);
              tmem_ld_32x32b_x32(t_row + UP + (j + 1) * 32, (j & 1) ? ua : ub);
            }
            if (j % CPB == 0) {
              if (lane == 0) bulk_wait_read<0>();
              __syncwarp();
            }
            float g[32], u[32], a[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              // round to the stored precision first: a is computed from the h13 that is kept
              g[i] = round_out<C::OES>(__uint_as_float(rg[i]));
              u[i] = round_out<C::OES>(__uint_as_float(ru[i]));
              a[i] = silu_f(g[i]) * u[i];
            }
            const int ch0 = ((j % CPB) * 32 * C::OES) >> 4;
            if (p.C) {  // h13 kept for the backward (absent: the backward recomputes it)
              stage_row32<C::OES>(bg, lane, ch0, g);
              stage_row32<C::OES>(bu, lane, ch0, u);
            }
            if constexpr (EPI == EPI_SWIGLU_FWD_Q) {
              // a as stored in bf16, quantised along the row (the next GEMM's contraction) and down
              // the warp's 32-row column block (the weight gradient's contraction)
#pragma unroll
              for (int i = 0; i < 32; ++i) a[i] = round_out<2>(a[i]);
              uint32_t cr[8], cc[8];
              srow |= (uint32_t)mx_row_block(a, cr) << (8 * (j & 3));
              const uint8_t scol = mx_col_blocks(a, lane, cc);
              const size_t off = (size_t)(c1 + lane) * (p.q_kb_row * 32) + col0 + j * 32;
              store_codes32(p.q_qr + off, cr);
              store_codes32(p.q_qc + off, cc);
              p.q_sc[tiled_sf_offset(col0 + j * 32 + lane, qrb, p.q_kb_col)] = scol;
            } else {
              // a straight from registers (the row's 32 values are 64 or 128 contiguous bytes): the
              // epilogue has time to spare behind the MMAs, and the box it no longer stages leaves
              // room for a sixth pipeline stage
              store_row32_global<C::OES>(static_cast<uint8_t*>(p.C2) +
                                             ((size_t)(c1 + lane) * p.ldc2 + col0 + j * 32) * C::OES, a);
            }
            if (j % CPB == CPB - 1 || j == NCH - 1) {
              const int c = col0 + (j / CPB) * C::OEPR;
              if (p.C) {
                box_store(&tmC, bg, lane, c, c1);
                box_store(&tmC, bu, lane, p.F + c, c1);
              }
            }
            if constexpr (EPI == EPI_SWIGLU_FWD_Q) {
              if ((j & 3) == 3) {  // the row's 4 scale bytes of 128 columns
                const int c = col0 + (j & ~3) * 32;
                *reinterpret_cast<uint32_t*>(p.q_sr + tiled_sf_offset(c1 + lane, c >> 5, p.q_kb_row)) = srow;
                srow = 0;
              }
            }
          }
        };
        if (active) {
          if (half) swiglu(std::integral_constant<int, BN / 4 / 32>{});
          else swiglu(std::integral_constant<int, BN / 2 / 32>{});
        }
      } else if constexpr (epi_swiglu_bwd(EPI)) {
        // dA chunk from TMEM; gate and up of the saved h13 for the same 32 columns from global
        // memory, both fetched one chunk ahead. Quantising: dh13 leaves as row-block and column-block
        // codes of its bf16 value (boxes: row codes gate / up, column codes gate / up).
        constexpr int NCH = BN / 32;
        constexpr int RW = 2 * C::OES;  // 16-byte words per 32 stored values
        const char* hrow = reinterpret_cast<const char*>(p.aux) +
                           ((size_t)ti_row_base(ti) + slab + lane) * p.ldaux * C::OES;
        if (active) {
          uint32_t da[32], db[32];
          uint4 gwa[RW], uwa[RW], gwb[RW], uwb[RW];
          tmem_ld_32x32b_x32(t_row, da);
          if (ti.n0 < p.N) {
            raw_load32<C::OES>(hrow + (size_t)ti.n0 * C::OES, gwa);
            raw_load32<C::OES>(hrow + (size_t)(p.F + ti.n0) * C::OES, uwa);
          }
          uint8_t* bg = wstg;
          uint8_t* bu = wstg + 4096;
          uint32_t srg = 0, sru = 0;  // quantising: row-block scale bytes of four consecutive chunks
#pragma unroll
          for (int j = 0; j < NCH; ++j) {
            uint32_t(&rd)[32] = (j & 1) ? db : da;
            const uint4* gw = (j & 1) ? gwb : gwa;
            const uint4* uw = (j & 1) ? uwb : uwa;
            const int col = ti.n0 + j * 32;
            const bool cols = col < p.N;  // warp-uniform; N is a multiple of the box width
            tmem_ld_wait_regs(rd);
            if (j + 1 < NCH) {
              tmem_ld_32x32b_x32(t_row + (j + 1) * 32, (j & 1) ? da : db);
              if (col + 32 < p.N) {
                raw_load32<C::OES>(hrow + (size_t)(col + 32) * C::OES, (j & 1) ? gwa : gwb);
                raw_load32<C::OES>(hrow + (size_t)(p.F + col + 32) * C::OES, (j & 1) ? uwa : uwb);
              }
            }
            if (cols) {
              if (EPI == EPI_SWIGLU_BWD && j % CPB == 0) {
                if (lane == 0) bulk_wait_read<0>();
                __syncwarp();
              }
              float g[32], u[32];
              unpack32<C::OES>(gw, g);
              unpack32<C::OES>(uw, u);
#pragma unroll
              for (int i = 0; i < 32; ++i) {
                const float dav = __uint_as_float(rd[i]);
                const float sg = __fdividef(1.f, 1.f + __expf(-g[i]));
                const float gi = g[i];
                g[i] = dav * u[i] * sg * (1.f + gi * (1.f - sg));  // d gate
                u[i] = dav * gi * sg;                              // d up
              }
              if constexpr (EPI == EPI_SWIGLU_BWD_Q) {
                uint32_t cr[8], cc[8];
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                  g[i] = round_out<2>(g[i]);
                  u[i] = round_out<2>(u[i]);
                }
                const size_t row_off = (size_t)(c1 + lane) * (p.q_kb_row * 32);
                srg |= (uint32_t)mx_row_block(g, cr) << (8 * (j & 3));
                uint8_t sc = mx_col_blocks(g, lane, cc);
                store_codes32(p.q_qr + row_off + col, cr);
                store_codes32(p.q_qc + row_off + col, cc);
                p.q_sc[tiled_sf_offset(col + lane, qrb, p.q_kb_col)] = sc;
                sru |= (uint32_t)mx_row_block(u, cr) << (8 * (j & 3));
                sc = mx_col_blocks(u, lane, cc);
                store_codes32(p.q_qr + row_off + p.F + col, cr);
                store_codes32(p.q_qc + row_off + p.F + col, cc);
                p.q_sc[tiled_sf_offset(p.F + col + lane, qrb, p.q_kb_col)] = sc;
                if ((j & 3) == 3) {
                  const int c = ti.n0 + (j & ~3) * 32;
                  *reinterpret_cast<uint32_t*>(p.q_sr + tiled_sf_offset(c1 + lane, c >> 5, p.q_kb_row)) = srg;
                  *reinterpret_cast<uint32_t*>(p.q_sr + tiled_sf_offset(c1 + lane, (p.F + c) >> 5, p.q_kb_row)) = sru;
                  srg = sru = 0;
                }
              } else {
                const int ch0 = ((j % CPB) * 32 * C::OES) >> 4;
                stage_row32<C::OES>(bg, lane, ch0, g);
                stage_row32<C::OES>(bu, lane, ch0, u);
                if (j % CPB == CPB - 1) {
                  const int c = (j / CPB) * C::OEPR;
                  box_store(&tmC, bg, lane, ti.n0 + c, c1);
                  box_store(&tmC, bu, lane, p.F + ti.n0 + c, c1);
                }
              }
            }
          }
        }
      } else {
        // plain store (act dtype), fp32 + bias (router scores), or a weight gradient (GROUP_K; an
        // expert without rows has nst == 0 and gets zeros). Tail tiles of a pair: BN/2 columns per
        // warp, output columns n0 + whalf*BN/2 + [0, BN/2).
        auto store = [&](auto nch_c) {
          constexpr int NCH = decltype(nch_c)::value;
          const int col0 = ti.n0 + whalf * (NCH * 32);
          const bool acc = nst > 0;
          uint32_t ra[32], rb[32];
          if (acc) tmem_ld_32x32b_x32(t_row, ra);
#pragma unroll
          for (int j = 0; j < NCH; ++j) {
            uint32_t(&rc)[32] = (j & 1) ? rb : ra;
            const int c = col0 + (j / CPB) * C::OEPR;  // first column of this chunk's box
            const bool cols = c < p.N;
            if (acc) {
              tmem_ld_wait_regs(rc);
              if (j + 1 < NCH) tmem_ld_32x32b_x32(t_row + (j + 1) * 32, (j & 1) ? ra : rb);
            }
            uint8_t* bx = wstg + nb * 4096;
            if (cols && j % CPB == 0) {
              if (lane == 0) bulk_wait_read<C::NBUF - 1>();
              __syncwarp();
            }
            float v[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] = acc ? __uint_as_float(rc[i]) : 0.f;
            if constexpr (EPI == EPI_STORE_F32_BIAS) {
              if (p.bias) {
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                  const int col = col0 + j * 32 + i;
                  if (col < p.N) v[i] += p.bias[col];
                }
              }
            }
            if (cols) {
              stage_row32<C::OES>(bx, lane, ((j % CPB) * 32 * C::OES) >> 4, v);
              if (j % CPB == CPB - 1 || j == NCH - 1) {
                box_store(&tmC, bx, lane, c, c1);
                nb = (nb + 1) % C::NBUF;
              }
            }
          }
        };
        if constexpr (C::EARLY) {
          constexpr int NCH = BN / 32 / (C::EPW / 4);  // this warp's 32-column chunks
          const bool acc = nst > 0 && active;
          uint32_t r[NCH][32];
          if (acc) {
#pragma unroll
            for (int j = 0; j < NCH; ++j) tmem_ld_32x32b_x32(t_row + j * 32, r[j]);
            tmem_ld_wait_regs(r[0]);
#pragma unroll
            for (int j = 1; j < NCH; ++j) tmem_regs_after(r[j]);
          }
          tc_fence_before();
          mbar_arrive(&tempty[buf]);  // the accumulator is free; the values are in registers
          if (active) {
            const int col0 = ti.n0 + whalf * (NCH * 32);
            uint8_t* out = static_cast<uint8_t*>(p.C);
            // 32 rows x 64 bytes; row r's 16-byte chunk q sits at chunk q ^ ((r >> 1) & 3), so both
            // the row-wise writes and the transposed reads below touch every bank once per 128 bytes
            uint8_t* tb = wstg;
#pragma unroll
            for (int j = 0; j < NCH; ++j) {
              const int col = col0 + j * 32;
              if (col >= p.N) continue;  // warp-uniform
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                float v[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) v[i] = acc ? __uint_as_float(r[j][8 * q + i]) : 0.f;
                st_shared_v4(tb + lane * 64 + ((q ^ ((lane >> 1) & 3)) << 4),
                             make_uint4(pack_bf16(v[0], v[1]), pack_bf16(v[2], v[3]), pack_bf16(v[4], v[5]),
                                        pack_bf16(v[6], v[7])));
              }
              __syncwarp();
              // each store instruction writes 8 whole 64-byte row segments: row 8i + lane/4,
              // 16-byte part lane%4
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                const int rr = 8 * i + (lane >> 2), sg = lane & 3;
                const uint4 w = ld_shared_v4(tb + rr * 64 + ((sg ^ ((rr >> 1) & 3)) << 4));
                *reinterpret_cast<uint4*>(out + ((size_t)(c1 + rr) * p.ldc + col) * 2 + sg * 16) = w;
              }
              __syncwarp();
            }
          }
        } else if (active) {
          if (half) store(std::integral_constant<int, BN / 2 / 32>{});
          else store(std::integral_constant<int, BN / 32 / (C::EPW / 4)>{});
        }
      }
      tc_fence_before();
      if constexpr (PAIR) {
        // the leader's MMA thread waits for every epilogue warp of both CTAs of the pair
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(tempty_lead + 8u * (uint32_t)buf);
      } else if constexpr (!C::EARLY) {
        mbar_arrive(&tempty[buf]);
      }
    }
    if (lane == 0) bulk_wait_all();  // every staged box written out before the CTA ends
  }

  tc_fence_before();
  __syncthreads();
  if constexpr (PAIR) cluster_sync();  // the peer's tensor memory stays allocated until both finish
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    if constexpr (PAIR) tmem_dealloc_pair(tmem_base, C::TMEM_COLS);
    else tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

// ------------------------------------------------------------------------------------------------
// host side: tensor maps and launch
// ------------------------------------------------------------------------------------------------

}  // namespace

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  return fn;
}

bool make_tmap_nd(CUtensorMap* m, const void* ptr, int es, int rank, const uint64_t* dims,
                  const uint64_t* strides_bytes, const uint32_t* box, int swizzle) {
  EncodeTiledFn fn = get_encode_fn();
  if (!fn || rank < 1 || rank > 5) return false;
  cuuint64_t d[5], st[4];
  cuuint32_t b[5], es1[5];
  for (int i = 0; i < rank; ++i) {
    d[i] = dims[i];
    b[i] = box[i];
    es1[i] = 1;
  }
  for (int i = 0; i + 1 < rank; ++i) st[i] = strides_bytes[i];
  const CUtensorMapSwizzle sw = swizzle == 2   ? CU_TENSOR_MAP_SWIZZLE_128B
                                : swizzle == 1 ? CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B
                                               : CU_TENSOR_MAP_SWIZZLE_NONE;
  const CUtensorMapDataType dt = es == 1   ? CU_TENSOR_MAP_DATA_TYPE_UINT8
                                 : es == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                           : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
  const CUresult r = fn(m, dt,
                        rank, const_cast<void*>(ptr), d, st, b, es1, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// MN-major operand as a 3-D tensor: (128-byte column block, row, column block), so that one box of
// box_rows rows x nblk column blocks lands in shared memory as nblk consecutive [box_rows x 128 B]
// blocks -- the MN-major layout the MMA descriptors expect. cols must be a multiple of 128 bytes.
bool make_tmap_mn(CUtensorMap* m, const void* ptr, int es, int64_t rows, int64_t cols, int64_t ld,
                  int box_rows, int nblk, int swizzle) {
  const int epr = 128 / es;
  if (cols % epr != 0) return false;
  const uint64_t dims[3] = {(uint64_t)epr, (uint64_t)rows, (uint64_t)(cols / epr)};
  const uint64_t strides[2] = {(uint64_t)(ld * es), 128};
  const uint32_t box[3] = {(uint32_t)epr, (uint32_t)box_rows, (uint32_t)nblk};
  return make_tmap_nd(m, ptr, es, 3, dims, strides, box, swizzle);
}

// 2-D row-major tensor [rows, cols] of `es`-byte elements, box [box_rows, box_cols]; swizzle as in
// make_tmap_nd (2: 128B, 1: 128B with 32-byte atoms, 0: none).
bool make_tmap(CUtensorMap* m, const void* ptr, int es, int64_t rows, int64_t cols, int64_t ld,
               int box_cols, int box_rows, int swizzle) {
  const uint64_t dims[2] = {(uint64_t)cols, (uint64_t)rows};
  const uint64_t strides[1] = {(uint64_t)(ld * es)};
  const uint32_t box[2] = {(uint32_t)box_cols, (uint32_t)box_rows};
  return make_tmap_nd(m, ptr, es, 2, dims, strides, box, swizzle);
}

int sm_count() {
  static int n[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) dev = 0;
  if (!n[dev]) cudaDeviceGetAttribute(&n[dev], cudaDevAttrMultiProcessorCount, dev);
  return n[dev] > 0 ? n[dev] : 148;
}

namespace {

template <int ES, bool A_MN, bool B_MN, int BN, int EPI, int MODE, bool PAIR>
int launch_impl(const GemmOperand& A, const GemmOperand& B, const GemmParams& p, cudaStream_t s) {
  using C = Cfg<ES, A_MN, B_MN, BN, EPI, MODE, PAIR>;
  auto kern = grouped_gemm_kernel<ES, A_MN, B_MN, BN, EPI, MODE, PAIR>;
  static bool attr_done[64] = {false};
  static int pair_slots[64] = {0};  // co-resident CTA pairs (clusters of 2) per device
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) dev = 0;
  if (!attr_done[dev]) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)C::SMEM_BYTES) != cudaSuccess)
      return MOE_ERR_CUDA;
    attr_done[dev] = true;
  }
  GemmParams q = p;
  CUtensorMap ta, tb;
  // A box: K-major -> [BM rows, EPR cols]; MN-major -> [BK rows, BM/EPR column blocks] as one 3-D
  // box when the columns are whole 128-byte blocks, else [32 rows, EPR cols] 2-D boxes (single
  // CTAs only). B likewise, with the BN_CTA rows (or columns) one CTA holds.
  const int mn_sw = ES == 4 ? 1 : 2;
  q.a_box3d = A_MN && (A.cols % C::EPR == 0);
  q.b_box3d = B_MN && (B.cols % C::EPR == 0);
  if (PAIR && ((A_MN && !q.a_box3d) || (B_MN && !q.b_box3d))) return MOE_ERR_UNSUPPORTED;
  if (q.a_box3d) {
    if (!make_tmap_mn(&ta, A.ptr, ES, A.rows, A.cols, A.ld, C::BK, BM / C::EPR, mn_sw)) return MOE_ERR_CUDA;
  } else if (!make_tmap(&ta, A.ptr, ES, A.rows, A.cols, A.ld, C::EPR, A_MN ? 32 : BM, A_MN ? mn_sw : 2)) {
    return MOE_ERR_CUDA;
  }
  if (q.b_box3d) {
    if (!make_tmap_mn(&tb, B.ptr, ES, B.rows, B.cols, B.ld, C::BK, C::BN_CTA / C::EPR, mn_sw))
      return MOE_ERR_CUDA;
  } else {
    const int b_box_rows = B_MN ? 32 : ((PAIR || !epi_swiglu_fwd(EPI)) ? C::BN_CTA : BN / 2);
    if (!make_tmap(&tb, B.ptr, ES, B.rows, B.cols, B.ld, C::EPR, b_box_rows, B_MN ? mn_sw : 2))
      return MOE_ERR_CUDA;
  }
  // outputs: 32-row x 128-byte boxes stored from the epilogue's swizzled staging
  CUtensorMap tc;
  const int64_t out_rows =
      (MODE == GROUP_K) ? (int64_t)k_groups(p) * (p.c_group_rows ? p.c_group_rows : p.M) : A.rows;
  const int64_t out_cols = (epi_swiglu_fwd(EPI) || epi_swiglu_bwd(EPI)) ? 2 * (int64_t)p.F : p.N;
  // SwiGLU forward: a [rows, F] is stored from registers with 16-byte stores
  if (EPI == EPI_SWIGLU_FWD &&
      (!p.C2 || (reinterpret_cast<uintptr_t>(p.C2) & 15) || (p.ldc2 * C::OES) % 16 != 0))
    return MOE_ERR_INVALID_ARG;
  // quantising epilogues: the codes [rows, F] (a) or [rows, 2F] (dh13) are stored from registers
  if (epi_quant(EPI) && (!p.q_qr || !p.q_qc || !p.q_sr || !p.q_sc)) return MOE_ERR_INVALID_ARG;
  if (p.C) {
    if (!make_tmap(&tc, p.C, C::OES, out_rows, out_cols, p.ldc, C::OEPR, 32, 2)) return MOE_ERR_CUDA;
  } else if (EPI == EPI_SWIGLU_BWD_Q) {
    tc = ta;  // dh13 leaves as codes only: tc is never used
  } else if (EPI == EPI_SWIGLU_FWD) {
    tc = ta;  // SwiGLU forward without h13: only a is stored, tc is never used
  } else {
    return MOE_ERR_INVALID_ARG;
  }
  // pair tail tiles (M = 128 over the pair): 64-row boxes of A, and of B for the SwiGLU forward,
  // whose tail tile loads 64 gate + 64 up rows per CTA
  CUtensorMap ta64 = ta, tb64 = tb;
  if (PAIR && MODE == GROUP_M) {
    if (!make_tmap(&ta64, A.ptr, ES, A.rows, A.cols, A.ld, C::EPR, C::HALF_M, 2)) return MOE_ERR_CUDA;
    if (EPI == EPI_SWIGLU_FWD &&
        !make_tmap(&tb64, B.ptr, ES, B.rows, B.cols, B.ld, C::EPR, BN / 4, 2))
      return MOE_ERR_CUDA;
  }
  // persistent grid: one CTA (pair) per SM (pair of SMs), capped by the tile count where the host
  // knows it (GROUP_K: fixed tiles per group)
  int64_t cap = 0;
  if (MODE == GROUP_K) {
    cap = (int64_t)k_groups(p) * ((p.M + C::TILE_M - 1) / C::TILE_M) * ((p.N + BN - 1) / BN);
    if (cap < 1) cap = 1;
  }
  if constexpr (PAIR) {
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute at[2];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = 2;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    at[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.blockDim = dim3(C::THREADS);
    cfg.dynamicSmemBytes = C::SMEM_BYTES;
    cfg.stream = s;
    cfg.attrs = at;
    cfg.numAttrs = 1;  // occupancy query: cluster shape only
    if (!pair_slots[dev]) {
      cfg.gridDim = dim3(2 * (sm_count() / 2));
      int n = 0;
      if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess || n < 1) return MOE_ERR_CUDA;
      pair_slots[dev] = n;
    }
    int64_t pairs = pair_slots[dev];
    if (cap > 0 && cap < pairs) pairs = cap;
    cfg.gridDim = dim3((unsigned)(2 * pairs));
    cfg.numAttrs = 2;  // cluster shape + programmatic dependent launch
    if (cudaLaunchKernelEx(&cfg, kern, ta, tb, tc, ta64, tb64, q) != cudaSuccess) return MOE_ERR_CUDA;
  } else {
    int64_t grid = sm_count();
    if (cap > 0 && cap < grid) grid = cap;
    MOE_LAUNCH(launch_pdl(kern, (unsigned)grid, C::THREADS, C::SMEM_BYTES, s, ta, tb, tc, ta64, tb64, q));
  }
  count_launches(1);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

}  // namespace

// Dispatch a GEMM request to its compiled variant. The caller (api.cu) has validated shapes.
// The ragged-row bf16 / tf32 GEMMs with light epilogues (fwd1 + SwiGLU, fwd2, dgrad1) run on CTA
// pairs: 256 x 256 tiles with cta_group::2 MMAs, so each weight tile is fetched once per 256 routed
// rows and each SM holds half of B. The bf16 expert wgrads run on pairs as well: each SM then loads
// half of the other operand's 256 columns, and the accumulator hand-back to the leader is one
// CTA-scope arrive per epilogue warp. The SwiGLU backward (whose epilogue a pair would couple: the
// MMA then waits for the slower CTA of the two), the router GEMMs and MXFP8 run on single CTAs with
// 128-row tiles.
int launch_gemm(GemmKind kind, int es, int bn, const GemmOperand& A, const GemmOperand& B,
                const GemmParams& p, cudaStream_t s) {
#define MOE_GEMM_CASES(ES_)                                                                        \
  switch (kind) {                                                                                  \
    case GK_FWD1_SWIGLU:                                                                           \
      return launch_impl<ES_, false, false, 256, EPI_SWIGLU_FWD, GROUP_M, true>(A, B, p, s);       \
    case GK_FWD2:                                                                                  \
      if (bn == 256) return launch_impl<ES_, false, false, 256, EPI_STORE, GROUP_M, true>(A, B, p, s);  \
      return launch_impl<ES_, false, false, 128, EPI_STORE, GROUP_M, false>(A, B, p, s);           \
    case GK_DGRAD2_SWIGLU:                                                                         \
      if (bn == 256)                                                                               \
        return launch_impl<ES_, false, true, 256, EPI_SWIGLU_BWD, GROUP_M, false>(A, B, p, s);     \
      return launch_impl<ES_, false, true, 128, EPI_SWIGLU_BWD, GROUP_M, false>(A, B, p, s);       \
    case GK_DGRAD1:                                                                                \
      if (bn == 256) return launch_impl<ES_, false, true, 256, EPI_STORE, GROUP_M, true>(A, B, p, s);  \
      return launch_impl<ES_, false, true, 128, EPI_STORE, GROUP_M, false>(A, B, p, s);            \
    case GK_WGRAD:                                                                                 \
      if (bn == 256 && ES_ == 2 && p.counts) /* bf16 expert wgrads: CTA pairs */                   \
        return launch_impl<ES_, true, true, 256, EPI_STORE, GROUP_K, ES_ == 2>(A, B, p, s);        \
      if (bn == 256) return launch_impl<ES_, true, true, 256, EPI_STORE, GROUP_K, false>(A, B, p, s); \
      return launch_impl<ES_, true, true, 128, EPI_STORE, GROUP_K, false>(A, B, p, s);             \
    case GK_ROUTER:                                                                                \
      if (bn == 256)                                                                               \
        return launch_impl<ES_, false, false, 256, EPI_STORE_F32_BIAS, GROUP_M, false>(A, B, p, s); \
      return launch_impl<ES_, false, false, 128, EPI_STORE_F32_BIAS, GROUP_M, false>(A, B, p, s);  \
    case GK_FWD1_SWIGLU_Q:                                                                         \
    case GK_DGRAD2_SWIGLU_Q:                                                                       \
      return MOE_ERR_UNSUPPORTED; /* quantising epilogues: MXFP8 only */                           \
    case GK_WGRAD_SPLIT:  /* fp32 partial products, no bias */                                     \
      if (bn == 256)                                                                               \
        return launch_impl<ES_, true, true, 256, EPI_STORE_F32_BIAS, GROUP_K, false>(A, B, p, s);  \
      return launch_impl<ES_, true, true, 128, EPI_STORE_F32_BIAS, GROUP_K, false>(A, B, p, s);    \
  }
  if (es == 2) {
    MOE_GEMM_CASES(2)
  } else if (es == 4) {
    MOE_GEMM_CASES(4)
  } else if (es == 1) {
    // MXFP8: 256-column tiles (twice the work per block-scaled MMA) with one accumulator, since the
    // per-stage scale columns leave no TMEM for a second; the SwiGLU forward tile is 128 gate + 128
    // up rows of W13 (F is a multiple of 128); fwd2, dgrad1 and the wgrads take wide tiles when N
    // is a multiple of 256 (every B scale chunk a tile reads then exists). The SwiGLU backward and
    // narrow cases use 128-column tiles with two accumulators.
    const bool wide = p.N % 256 == 0;
    switch (kind) {
      case GK_FWD1_SWIGLU: return launch_impl<1, false, false, 256, EPI_SWIGLU_FWD, GROUP_M, false>(A, B, p, s);
      case GK_FWD1_SWIGLU_Q: return launch_impl<1, false, false, 256, EPI_SWIGLU_FWD_Q, GROUP_M, false>(A, B, p, s);
      case GK_DGRAD2_SWIGLU_Q: return launch_impl<1, false, true, 128, EPI_SWIGLU_BWD_Q, GROUP_M, false>(A, B, p, s);
      case GK_FWD2:
        if (wide) return launch_impl<1, false, false, 256, EPI_STORE, GROUP_M, false>(A, B, p, s);
        return launch_impl<1, false, false, 128, EPI_STORE, GROUP_M, false>(A, B, p, s);
      case GK_DGRAD2_SWIGLU:  // epilogue-heavy: two accumulators overlap it with the next tile
        return launch_impl<1, false, true, 128, EPI_SWIGLU_BWD, GROUP_M, false>(A, B, p, s);
      case GK_DGRAD1:
        if (wide) return launch_impl<1, false, true, 256, EPI_STORE, GROUP_M, false>(A, B, p, s);
        return launch_impl<1, false, true, 128, EPI_STORE, GROUP_M, false>(A, B, p, s);
      case GK_WGRAD:
        if (wide) return launch_impl<1, true, true, 256, EPI_STORE, GROUP_K, false>(A, B, p, s);
        return launch_impl<1, true, true, 128, EPI_STORE, GROUP_K, false>(A, B, p, s);
      default: return MOE_ERR_UNSUPPORTED;
    }
  }
#undef MOE_GEMM_CASES
  return MOE_ERR_UNSUPPORTED;
}

// Sum of the split-contraction partials (fp32, fixed order), rounded to the output dtype.
__global__ void __launch_bounds__(256) split_reduce_kernel(const float4* __restrict__ part, int nsplit,
                                                           int64_t n4, int64_t stride4,
                                                           void* __restrict__ out, int bf16) {
  pdl_enter();  // wait for the previous kernel before any global access
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4;
       i += (int64_t)gridDim.x * blockDim.x) {
    float4 acc = part[i];
    for (int s = 1; s < nsplit; ++s) {
      const float4 v = part[(int64_t)s * stride4 + i];
      acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
    }
    if (bf16) reinterpret_cast<uint2*>(out)[i] = make_uint2(pack_bf16(acc.x, acc.y), pack_bf16(acc.z, acc.w));
    else reinterpret_cast<float4*>(out)[i] = acc;
  }
}

int launch_split_reduce(const float* part, int nsplit, int64_t n, int64_t stride, void* out, bool bf16,
                        cudaStream_t s) {
  if (n % 4 != 0 || stride % 4 != 0 || stride < n || nsplit < 1) return MOE_ERR_UNSUPPORTED;
  const int64_t n4 = n / 4;
  int64_t blocks = (n4 + 255) / 256;
  if (blocks > 4 * (int64_t)sm_count()) blocks = 4 * (int64_t)sm_count();
  MOE_LAUNCH(launch_pdl(split_reduce_kernel, (unsigned)blocks, 256, 0, s, reinterpret_cast<const float4*>(part), nsplit, n4,
                                                        stride / 4, out, bf16 ? 1 : 0));
  count_launches(1);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

// Bounded-wait self-test: wait on a barrier nobody arrives at.
__global__ void bounded_wait_probe_kernel(uint32_t* err, uint64_t limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_word;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_word = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait_bounded(&bar, 0, limit_ns, &abort_word, err);
}

int launch_bounded_wait_probe(uint32_t* err, uint64_t limit_ns, cudaStream_t s) {
  bounded_wait_probe_kernel<<<1, 32, 0, s>>>(err, limit_ns);
  count_launches(1);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

}  // namespace moe
