// Weight-major grouped expert GEMMs on the 5th-generation tensor cores (sm_100a): the
// expert's weight rows are the MMA's M side and the expert's tokens its N side.
//
// Expert FFN: "Hugging Face 图解 Mixture of Experts（MoE）原理、训练与推理权衡", section
// "什么是混合专家模型" (each expert is an FFN) and section "更多关于高效训练的内容"
// (experts receive uneven numbers of tokens; handle them without padding or drops).
//
// Why a second orientation.  The token-major kernels (ffn_tc.cu) give a CTA pair 256
// token rows of one expert; an expert with 41 rows still costs a 256-row tile of tensor
// work.  With many experts and skewed loads (most experts hold a few dozen rows, a few
// hold hundreds) that padding, not the weights, sets the time.  Here a tile is 256 output
// features (weight rows, 128 per CTA) x N tokens, N = the expert's rows rounded up to 32
// (at most NT): a 41-row expert pads to 64 columns.  Each tile streams its weight slab
// once; the token blocks of one weight slab are consecutive tiles, so CTAs running at the
// same time share the slab through L2.
//
//   MODE 0 (gate/up): A = W_gate[e] and W_up[e] rows f0 .. f0+255 (two M=256 MMAs per k
//       step into two accumulators, g in columns [0, 128), u in [128, 256)), B = N <= 128
//       rows of x_perm; the epilogue writes H[token][f] = silu(g) * u as bf16.
//   MODE 1 (down):    A = W_dn[e] rows n0 .. n0+255, B = N <= 256 rows of H; the epilogue
//       writes gate_of_row[token] * acc to the gated rows (bf16 or fp32).
//
// CTA pairs (cta_group::2): each CTA stages 128 weight rows and N/2 token rows per
// 64-wide k-block (TMA, 128-byte swizzle); the even CTA issues the MMAs; the accumulator
// rows (features) of each CTA land in its own TMEM.  Epilogue: a thread owns one feature
// (its TMEM lane) for 32 tokens per tcgen05.ld; a shared-memory turn-around writes whole
// 128-byte lines of token rows.  Two accumulators of 256 columns let the epilogue of one
// tile overlap the next tile's mainloop.  Every wait is bounded (MOE_DEVERR_PIPE_TIMEOUT,
// then an orderly exit).  No load uses cluster multicast.
#include "common.cuh"
#include "tc_prims.cuh"
#include "tile_sched.cuh"

namespace moe {
namespace {

constexpr int kWMaxE = 1024;
constexpr uint32_t kWTmemCols = 512;
constexpr int kWRows = 128;                     // weight rows per CTA (256 per pair)
constexpr int kWBlock = kWRows * BK * 2;       // 16 KB: one 128-row operand block
constexpr int kFp4PadRows = 2 * kWRows;        // zero rows after the prepared 4-bit scales
constexpr int kWXBox = 16;                      // token rows per TMA box: a tile loads only its n / 2 rows

template <int MODE>
struct WmCfg {
  static constexpr int NT = MODE == 0 ? 128 : 256;            // tokens per tile (MMA N at most)
  static constexpr int a_blocks = MODE == 0 ? 2 : 1;           // gate + up, or down
  static constexpr int b_bytes = (NT / 2) * BK * 2;            // this CTA's token rows per stage
  static constexpr int stage_bytes = a_blocks * kWBlock + b_bytes;
  static constexpr int stages = MODE == 0 ? 5 : 6;
  static constexpr int epi_warps = 4;
  static constexpr int threads = 64 + 32 * epi_warps;
  static constexpr int bars = stages * stage_bytes;
  static constexpr int nbars = 2 * stages + 4 + 1;   // full, empty, tfull[2], tempty[2], fin
  static constexpr int misc = bars + nbars * 8;
  static constexpr int tiles = misc + 16;
  static constexpr int sh32 = tiles + (kWMaxE + 1) * 4;
  static constexpr int stage = (sh32 + 32 * 4 + 127) / 128 * 128;
  static constexpr int end = stage + epi_warps * kStageWarpBytes;
  static constexpr size_t smem = end + 1024;
  static_assert(smem <= 232448, "shared memory per CTA");
  static_assert(stage_bytes % 1024 == 0, "stages must keep the 1024-byte swizzle alignment");
};

// Output feature tiles (256 per pair) per token block.
template <int MODE>
__host__ __device__ __forceinline__ int wm_m_tiles(int F, int d) {
  return MODE == 0 ? (F + 255) / 256 : (d + 255) / 256;
}

// MMA width for a tile of `rows` tokens: rows rounded up to 32, at most NT.
template <int MODE>
__device__ __forceinline__ int wm_n(int rows) {
  const int n = (rows + 31) / 32 * 32;
  return n < WmCfg<MODE>::NT ? n : WmCfg<MODE>::NT;
}

// The turn-around of the weight-major epilogue: thread `lane` holds output column col +
// lane for the 32 tokens row0 .. row0+31 (v[i] = token i).  It writes them as column lane
// of a 32 x 32 tile in shared memory, then the warp stores whole token rows (16 bytes per
// lane: 8 bf16 or 4 fp32 columns) -- rows past rows_valid and columns past ncols skipped.
template <typename OutT>
__device__ __forceinline__ void stage_store32_t(uint8_t* stage, const float (&v)[32], int lane, OutT* out,
                                                long long row0, int rows_valid, long long ld, int col, int ncols) {
  if constexpr (sizeof(OutT) == 4) {
#pragma unroll
    for (int i = 0; i < 32; ++i) *reinterpret_cast<float*>(stage + i * kStagePitchF32 + lane * 4) = v[i];
    __syncwarp();
    const int rs = lane >> 3, cv = lane & 7;       // 4 rows per pass, 8 x 16 B per row
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int r = i * 4 + rs;
      const float4 x = *reinterpret_cast<const float4*>(stage + r * kStagePitchF32 + cv * 16);
      if (r < rows_valid && col + cv * 4 + 4 <= ncols)
        *reinterpret_cast<float4*>(out + (row0 + r) * ld + col + cv * 4) = x;
    }
  } else {
#pragma unroll
    for (int i = 0; i < 32; ++i)
      *reinterpret_cast<__nv_bfloat16*>(stage + i * kStagePitchB16 + lane * 2) = __float2bfloat16_rn(v[i]);
    __syncwarp();
    const int rs = lane >> 2, cv = lane & 3;       // 8 rows per pass, 4 x 16 B per row
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int r = i * 8 + rs;
      const uint4 x = *reinterpret_cast<const uint4*>(stage + r * kStagePitchB16 + cv * 16);
      if (r < rows_valid && col + cv * 8 + 8 <= ncols)
        *reinterpret_cast<uint4*>(out + (row0 + r) * ld + col + cv * 8) = x;
    }
  }
  __syncwarp();
}

// Gate of the token in row c * 32 + lane of a weight-major tile (1 past the tile's rows, or
// without gates).
__device__ __forceinline__ float wm_gate(const float* __restrict__ gate_of_row, const TileCoord& tc, int c,
                                         int lane) {
  const int r = c * 32 + lane;
  return (gate_of_row && r < tc.rows) ? __ldg(gate_of_row + tc.row0 + r) : 1.f;
}

// One tile's epilogue for one warp: features col0 .. col0+31 (its TMEM lanes) of the tile's
// tokens, 32 tokens per tcgen05.ld.  wscale multiplies every accumulator (the 4-bit
// weights' per-tensor scale; 1 for bf16 weights).
//   MODE 0: H[token][f] = silu(wscale g) * (wscale u), bf16;
//   MODE 1: y[token][n] = gate_of_row[token] * wscale * acc.
// g0, g1 (MODE 1): this lane's gates of the tile's first two 32-token chunks, fetched by the
// caller before the accumulator was ready; later gates are fetched one chunk pair ahead.
template <int MODE, typename OutT>
__device__ __forceinline__ void wm_epilogue_tile(uint32_t taddr, uint8_t* stage, int lane, const TileCoord& tc,
                                                 int rank, int q, int d, int F, float wscale,
                                                 const float* __restrict__ gate_of_row, OutT* __restrict__ out,
                                                 float g0 = 1.f, float g1 = 1.f) {
  const int col0 = tc.n_tile * 256 + rank * kWRows + q * 32;   // this warp's first feature
  const int chunks = (tc.rows + 31) / 32;
  if constexpr (MODE == 0) {
#pragma unroll 1
    for (int c = 0; c < chunks; ++c) {
      const long long r0 = (long long)tc.row0 + c * 32;
      const int rv = min(32, tc.rows - c * 32);
      float h[32];
      uint32_t g[32], u[32];
      tmem_ld32(taddr + c * 32, g);
      tmem_ld32(taddr + 128 + c * 32, u);
      tmem_wait_ld();
      tmem_regs_ready(g);
      tmem_regs_ready(u);
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const float gi = __uint_as_float(g[i]) * wscale;
        // fast exp / divide: H is rounded to bf16 next, far coarser than their error
        h[i] = __fdividef(gi, 1.f + __expf(-gi)) * (__uint_as_float(u[i]) * wscale);
      }
      stage_store32_t<OutT>(stage, h, lane, out, r0, rv, F, col0, F);
    }
  } else {
    // two 32-token chunks per TMEM wait (the tile's mainloop is only K / 64 k-blocks)
    float ga = g0, gb = g1;
#pragma unroll 1
    for (int c = 0; c < chunks; c += 2) {
      const float na = wm_gate(gate_of_row, tc, c + 2, lane), nb = wm_gate(gate_of_row, tc, c + 3, lane);
      const bool two = c + 1 < chunks;                     // warp-uniform
      uint32_t v[32], vb[32];
      tmem_ld32(taddr + c * 32, v);
      if (two) tmem_ld32(taddr + (c + 1) * 32, vb);
      tmem_wait_ld();
      tmem_regs_ready(v);
      tmem_regs_ready(vb);
      float h[32];
      const float gs = ga * wscale;
#pragma unroll
      for (int i = 0; i < 32; ++i) h[i] = __uint_as_float(v[i]) * __shfl_sync(0xffffffffu, gs, i);
      stage_store32_t<OutT>(stage, h, lane, out, (long long)tc.row0 + c * 32, min(32, tc.rows - c * 32), d, col0,
                            d);
      if (two) {
        const float gsb = gb * wscale;
#pragma unroll
        for (int i = 0; i < 32; ++i) h[i] = __uint_as_float(vb[i]) * __shfl_sync(0xffffffffu, gsb, i);
        stage_store32_t<OutT>(stage, h, lane, out, (long long)tc.row0 + (c + 1) * 32,
                              min(32, tc.rows - (c + 1) * 32), d, col0, d);
      }
      ga = na;
      gb = nb;
    }
  }
}

// GATHER (gate/up only): the token rows come straight from x [n_tokens, d] through
// token_of_row (no permuted copy of x): TMA row gathers (four rows per instruction, one
// lane per four rows) land them in the same swizzled layout as the tiled loads, counted
// on the even CTA's `full` barrier with the weights' bytes; tmX maps x with a one-row box.
template <int MODE, typename OutT, bool GATHER = false>
__global__ void __launch_bounds__(WmCfg<MODE>::threads, 1)
grouped_gemm_wm_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                       const int32_t* __restrict__ offsets, int E, int K, int d, int F, long long rows_max,
                       const float* __restrict__ gate_of_row, OutT* __restrict__ out, int* err,
                       const int32_t* __restrict__ token_of_row = nullptr, int n_tokens = 0) {
  static_assert(!GATHER || MODE == 0, "the gathered form is the gate/up GEMM's");
  using C = WmCfg<MODE>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int* tile_start = reinterpret_cast<int*>(smem + C::tiles);
  int* sh32 = reinterpret_cast<int*>(smem + C::sh32);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::misc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::misc + 4);
  const uint32_t rank = cluster_ctarank();
  const int cid = (int)(blockIdx.x >> 1), ncl = (int)(gridDim.x >> 1);

  const int m_tiles = wm_m_tiles<MODE>(F, d);
  build_tile_starts(offsets, E, C::NT, m_tiles, rows_max, tile_start, sh32, err);
  const int total = tile_start[E];
  if (cid >= total) return;   // both CTAs of the pair see the same cid: uniform, nothing allocated

  const uint32_t bar_full = sb + C::bars;
  const uint32_t bar_empty = bar_full + 8 * C::stages;
  const uint32_t bar_tfull = bar_empty + 8 * C::stages;
  const uint32_t bar_tempty = bar_tfull + 16;
  const uint32_t bar_fin = bar_tempty + 16;
  auto a_blk = [&](int s, int a) { return sb + (uint32_t)(s * C::stage_bytes + a * kWBlock); };
  auto b_blk = [&](int s) { return sb + (uint32_t)(s * C::stage_bytes + C::a_blocks * kWBlock); };

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::stages; ++s) {
      mbar_init(bar_full + 8 * s, 1);
      mbar_init(bar_empty + 8 * s, 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(bar_tfull + 8 * a, 1);
      mbar_init(bar_tempty + 8 * a, 2 * 32 * C::epi_warps);
    }
    mbar_init(bar_fin, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(kWTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int KB = (K + BK - 1) / BK;

  if (GATHER && warp == 0) {
    // ------------------------------------------------------------ gathering producer (both CTAs)
    // Lane j < n / 8 owns rows 4j .. 4j+3 of this CTA's n / 2 token rows and fetches them
    // with one TMA row gather per k-block (rows past the group read token 0: their MMA
    // columns are never stored); lane 0 also loads the weight slab.
    int stage = 0;
    uint32_t phase = 0;
    int last_phase[C::stages];
#pragma unroll
    for (int s = 0; s < C::stages; ++s) last_phase[s] = -1;
    bool ok = true;
    for (int tile = cid; ok && tile < total; tile += ncl) {
      const TileCoord tc = tile_coord(tile_start, offsets, E, C::NT, tile);
      const int half = wm_n<MODE>(tc.rows) / 2;
      const int w_row = tc.e * 2 * F + tc.n_tile * 256 + (int)rank * kWRows;
      const bool mine = 4 * lane < half;
      const int r0 = (int)rank * half + 4 * lane;           // this lane's first row of the tile
      int t[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        int v = 0;
        if (mine && r0 + i < tc.rows) {
          v = __ldg(token_of_row + tc.row0 + r0 + i);
          if ((unsigned)v >= (unsigned)n_tokens) {
            record_error(err, MOE_DEVERR_ROW);
            v = 0;
          }
        }
        t[i] = v;
      }
      for (int kb = 0; kb < KB; ++kb) {
        const bool got = mbar_wait(bar_empty + 8 * stage, phase ^ 1u, abort_flag, err);
        if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
        const uint32_t full_c = map_to_rank(bar_full + 8 * stage, 0);
        if (lane == 0) {
          if (rank == 0)
            mbar_expect_tx(bar_full + 8 * stage, 2u * (uint32_t)(C::a_blocks * kWBlock + half * BK * 2));
          tma_load_2d_pair(a_blk(stage, 0), &tmW, full_c, kb * BK, w_row);
          tma_load_2d_pair(a_blk(stage, 1), &tmW, full_c, kb * BK, w_row + F);
          last_phase[stage] = (int)phase;
        }
        if (mine) tma_gather4_pair(b_blk(stage) + (uint32_t)(lane * 512), &tmX, full_c, kb * BK, t[0], t[1], t[2], t[3]);
        if (++stage == C::stages) { stage = 0; phase ^= 1u; }
      }
    }
    if (!ok && lane == 0 && rank == 0) {
      for (int s = 0; s < C::stages; ++s)
        if (last_phase[s] >= 0) mbar_wait_drain(bar_full + 8 * s, (uint32_t)last_phase[s], err);
    }
  } else if (warp == 0) {
    // ------------------------------------------------------------ TMA producer (both CTAs)
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int last_phase[C::stages];
#pragma unroll
      for (int s = 0; s < C::stages; ++s) last_phase[s] = -1;
      bool ok = true;
      for (int tile = cid; ok && tile < total; tile += ncl) {
        const TileCoord tc = tile_coord(tile_start, offsets, E, C::NT, tile);
        const int n = wm_n<MODE>(tc.rows);
        // this CTA's weight rows, and its half of the tile's tokens (columns [rank n/2, ...))
        const int w_row = MODE == 0 ? tc.e * 2 * F + tc.n_tile * 256 + (int)rank * kWRows
                                    : tc.e * d + tc.n_tile * 256 + (int)rank * kWRows;
        const int x_row = tc.row0 + (int)rank * (n / 2);
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait(bar_empty + 8 * stage, phase ^ 1u, abort_flag, err)) { ok = false; break; }
          if (rank == 0)
            mbar_expect_tx(bar_full + 8 * stage, 2u * (uint32_t)(C::a_blocks * kWBlock + (n / 2) * BK * 2));
          const uint32_t full_c = map_to_rank(bar_full + 8 * stage, 0);
          tma_load_2d_pair(a_blk(stage, 0), &tmW, full_c, kb * BK, w_row);
          if (MODE == 0) tma_load_2d_pair(a_blk(stage, 1), &tmW, full_c, kb * BK, w_row + F);
          for (int xb = 0; xb < n / 2; xb += kWXBox)      // n / 2 is a multiple of 16
            tma_load_2d_pair(b_blk(stage) + (uint32_t)(xb * BK * 2), &tmX, full_c, kb * BK, x_row + xb);
          last_phase[stage] = (int)phase;
          if (++stage == C::stages) { stage = 0; phase ^= 1u; }
        }
      }
      if (!ok && rank == 0) {
        for (int s = 0; s < C::stages; ++s)
          if (last_phase[s] >= 0) mbar_wait_drain(bar_full + 8 * s, (uint32_t)last_phase[s], err);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (even CTA)
    if (lane == 0 && rank == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      bool ok = true;
      for (int tile = cid; ok && tile < total; tile += ncl, ++it) {
        const int acc = it & 1;
        const uint32_t acc_phase = (uint32_t)(it >> 1) & 1u;
        const TileCoord tc = tile_coord(tile_start, offsets, E, C::NT, tile);
        const uint32_t idesc = make_idesc(2 * kWRows, wm_n<MODE>(tc.rows));
        if (!mbar_wait(bar_tempty + 8 * acc, acc_phase ^ 1u, abort_flag, err)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * 256);
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait(bar_full + 8 * stage, phase, abort_flag, err)) { ok = false; break; }
          tc_fence_after();
          const uint64_t bdesc = sw128_desc(b_blk(stage));
          const uint64_t adesc0 = sw128_desc(a_blk(stage, 0));
          const uint64_t adesc1 = sw128_desc(a_blk(stage, MODE == 0 ? 1 : 0));
#pragma unroll
          for (int kk = 0; kk < BK / UMMA_K; ++kk) {   // +32 bytes along K per step (>> 4 = 2)
            const uint32_t accumulate = (kb | kk) != 0 ? 1u : 0u;
            umma_bf16_pair(d_tmem, adesc0 + 2 * kk, bdesc + 2 * kk, idesc, accumulate);
            if (MODE == 0) umma_bf16_pair(d_tmem + 128, adesc1 + 2 * kk, bdesc + 2 * kk, idesc, accumulate);
          }
          umma_commit_pair_both(bar_empty + 8 * stage);
          if (++stage == C::stages) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        umma_commit_pair_both(bar_tfull + 8 * acc);
      }
      umma_commit_pair(bar_fin);
      mbar_wait_drain(bar_fin, 0, err);
    }
  } else {
    // ------------------------------------------------------------ epilogue (both CTAs)
    const int q = warp & 3;                                  // TMEM lane quarter of this warp
    uint8_t* stage = smem + C::stage + (warp - 2) * kStageWarpBytes;
    int it = 0;
    for (int tile = cid; tile < total; tile += ncl, ++it) {
      const TileCoord tc = tile_coord(tile_start, offsets, E, C::NT, tile);
      const int acc = it & 1;
      const uint32_t acc_phase = (uint32_t)(it >> 1) & 1u;
      // the first gates, fetched while the tile's MMAs still run
      const float g0 = MODE == 1 ? wm_gate(gate_of_row, tc, 0, lane) : 1.f;
      const float g1 = MODE == 1 ? wm_gate(gate_of_row, tc, 1, lane) : 1.f;
      const bool got = mbar_wait(bar_tfull + 8 * acc, acc_phase, abort_flag, err);
      if (!__all_sync(0xffffffffu, got)) break;
      __syncwarp();
      tc_fence_after();
      const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * 256);
      wm_epilogue_tile<MODE, OutT>(taddr, stage, lane, tc, (int)rank, q, d, F, 1.f, gate_of_row, out, g0, g1);
      tc_fence_before();
      mbar_arrive_remote(map_to_rank(bar_tempty + 8 * acc, 0));
    }
  }

  __syncthreads();
  cluster_sync();                                           // no remote arrive after a CTA exits
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(kWTmemCols) : "memory");
  }
}

// =====================================================================================
// 4-bit expert weights (weight-only): the same weight-major tiles, with each stage's
// weight blocks arriving as packed E2M1 codes (a quarter of the bytes) and expanded to
// bf16 in shared memory by eight converter warps before the MMAs read them.
//
// Handbook digest (agihunt.info), "已确认", bullet "量化与推理": routed experts in MXFP4
// (Kimi K3), NVFP4 training with key layers kept in BF16 (Nemotron 3).  The activations
// stay bf16, and a kind::f16 MMA multiplies bf16 by bf16, so the weights are expanded:
//   value = e2m1(code) * block scale, exact in bf16 (at most 2 significant bits times a
//   power of two (MXFP4, E8M0 scale) or times an E4M3 scale of at most 4 bits (NVFP4));
//   the NVFP4 per-expert fp32 tensor scale multiplies the fp32 accumulators.
// Weights: codes [rows, K/2] bytes as moe_quantize_fp4_host writes them (element 2j in the
// low nibble of byte j), loaded by TMA; scales in the k-block-major layout of
// moe_prepare_fp4_scales, [K/64][rows + 256][64/block] bytes, so the scales of one
// k-block of 128 rows are one contiguous 256- or 512-byte bulk copy (the 256 zero rows
// cover the blocks of the last tiles that start past the matrix, at most 127 rows past
// it).  K a multiple of 64.
//
// Per stage and CTA: the codes and scales of its weight rows and its token rows land by
// TMA and bulk copy on the CTA's own `packed` barrier.  The eight converter warps form four
// groups of two; group g decodes the stages g, g + 4, ..., so the four stages of the ring
// are decoded side by side (one group for every stage took 1.5x as long).  A converter
// thread owns two weight rows of its stages (all blocks and chunks of them).  It decodes
// each 32-bit word of codes (eight
// elements) in registers: shifts and masks place each code's bits in a bf16 (which reads
// as 2^-126 times the code's value, subnormal codes included), byte permutes put the
// pairs in order, and each bf16 pair is multiplied by 2^126, then by the block scale.  Each
// 16-byte chunk goes to the 128-byte-swizzled operand layout (chunk c of row r at
// r * 128 + ((c ^ (r & 7)) * 16)); then each thread's proxy fence, and one arrive per
// converter warp of the stage's group on the even CTA's `full` barrier (2 x 2 warps).
// `empty` (the MMAs' completion) frees the stage in both CTAs.
// =====================================================================================
template <int MODE>
struct Wm4Cfg {
  static constexpr int NT = WmCfg<MODE>::NT;
  static constexpr int a_blocks = WmCfg<MODE>::a_blocks;
  static constexpr int b_bytes = WmCfg<MODE>::b_bytes;
  static constexpr int packed_block = kWRows * BK / 2;          // 4 KB of codes per weight block
  static constexpr int scale_block = kWRows * 4;                // up to 4 scale bytes per row and k-block
  static constexpr int stage_bytes = a_blocks * kWBlock + b_bytes + a_blocks * (packed_block + scale_block);
  static constexpr int stage_pitch = (stage_bytes + 1023) / 1024 * 1024;
  static constexpr int stages = 4;
  // converter groups decoding stages side by side (one group per stage measured fastest:
  // 4.08 -> 2.74 ms for the MXFP4 gate/up of the stress layer with one group); a group
  // must see every phase of the stages it waits on, so the groups divide the stages
  static constexpr int cvt_groups = 4;
  static constexpr int epi_warps = 4, cvt_warps = 8;
  static constexpr int threads = 64 + 32 * (epi_warps + cvt_warps);
  static constexpr int bars = stages * stage_pitch;
  static constexpr int nbars = 3 * stages + 4 + 1;
  static constexpr int misc = bars + nbars * 8;
  static constexpr int tiles = (misc + 16 + 15) / 16 * 16;
  static constexpr int sh32 = tiles + (kWMaxE + 1) * 4;
  static constexpr int stage = (sh32 + 32 * 4 + 127) / 128 * 128;
  static constexpr int end = stage + epi_warps * kStageWarpBytes;
  static constexpr size_t smem = end + 1024;
  static_assert(smem <= 232448, "shared memory per CTA");
  static_assert((a_blocks * kWBlock + b_bytes) % 1024 == 0, "swizzle alignment");
  static_assert(cvt_warps % cvt_groups == 0 && kWRows % (cvt_warps * 32 / cvt_groups) == 0,
                "converter groups of whole warps, each thread the same number of weight rows");
  static_assert(stages % cvt_groups == 0, "a converter group waits only on the stages it has seen");
};

// bf16 of a block scale byte: E8M0 (2^(b - 127); b = 0 is 2^-127, a bf16 subnormal) or
// E4M3 (normal 2^(e-7) (1 + m/8), subnormal m 2^-9).  Both exact in bf16.
template <int FMT>
__device__ __forceinline__ uint32_t scale_bf16_bits(uint32_t b) {
  if (FMT == MOE_FP4_MX) return b ? (b << 7) : 0x0040u;
  const uint32_t e = (b >> 3) & 15u, m = b & 7u;
  if (e) return ((e + 120u) << 7) | (m << 4);
  const __nv_bfloat16 v = __float2bfloat16_rn((float)m * 0.001953125f);
  return (uint32_t)(*reinterpret_cast<const uint16_t*>(&v));
}

// Eight E2M1 codes (w: element i in bits 4i .. 4i+3) -> the bits of eight bf16 values
// 2^-126 times the codes' values (o[0] holds elements 0 and 1, ...).  A code's magnitude
// bits e1 e0 m placed at bf16 bits 8..6, its sign at bit 15, read as a bf16 number:
// exponent field e, so for e > 0 the value is 2^(e-127) (1 + m/2) and for e = 0 the
// subnormal m 2^-127, while E2M1 is 2^(e-1) (1 + m/2) and m / 2: both 2^-126 times it.
// One shift of the word places codes i and i + 4 in the two halves of a bf16 pair; byte
// permutes then pair the elements in order.
__device__ __forceinline__ void e2m1x8_to_bf16_bits(uint32_t w, uint32_t (&o)[4]) {
  constexpr uint32_t MAG = 0x01C001C0u, SGN = 0x80008000u;
  const uint32_t p0 = ((w << 6) & MAG) | ((w << 12) & SGN);   // elements 0, 4
  const uint32_t p1 = ((w << 2) & MAG) | ((w << 8) & SGN);    // 1, 5
  const uint32_t p2 = ((w >> 2) & MAG) | ((w << 4) & SGN);    // 2, 6
  const uint32_t p3 = ((w >> 6) & MAG) | (w & SGN);           // 3, 7
  o[0] = __byte_perm(p0, p1, 0x5410);
  o[1] = __byte_perm(p2, p3, 0x5410);
  o[2] = __byte_perm(p0, p1, 0x7632);
  o[3] = __byte_perm(p2, p3, 0x7632);
}

// Expands chunks [c0, c1) of one row of a block: codes at src (32 bytes), the row's scale
// bytes packed little-endian in sc (MX: 2, chunks 0-3 and 4-7; NV: 4, chunk pairs).
template <int FMT>
__device__ __forceinline__ void convert_chunks(const uint8_t* src, uint32_t sc, uint8_t* dst_block, int r, int c0,
                                               int c1) {
  const uint4 q0 = *reinterpret_cast<const uint4*>(src);
  const uint4 q1 = *reinterpret_cast<const uint4*>(src + 16);
  const uint32_t w[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    if (c < c0 || c >= c1) continue;
    const uint32_t sb = FMT == MOE_FP4_MX ? scale_bf16_bits<FMT>((sc >> (8 * (c >> 2))) & 0xffu)
                                          : scale_bf16_bits<FMT>((sc >> (8 * (c >> 1))) & 0xffu);
    const uint32_t s2u = sb | (sb << 16);
    const __nv_bfloat162 s2 = *reinterpret_cast<const __nv_bfloat162*>(&s2u);
    constexpr uint32_t kTwo126 = 0x7E807E80u;   // bf16 pair 2^126, 2^126
    const __nv_bfloat162 t2 = *reinterpret_cast<const __nv_bfloat162*>(&kTwo126);
    uint32_t o[4];
    e2m1x8_to_bf16_bits(w[c], o);
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      __nv_bfloat162 v = *reinterpret_cast<const __nv_bfloat162*>(&o[b]);
      v = __hmul2(__hmul2(v, t2), s2);          // exact: the code's value, then at most 6 significant bits
      o[b] = *reinterpret_cast<uint32_t*>(&v);
    }
    *reinterpret_cast<uint4*>(dst_block + r * 128 + ((c ^ (r & 7)) << 4)) = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

// One-dimensional bulk copy global -> this CTA's shared memory, completing on an mbarrier.
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "l"(src), "r"(bytes), "r"(bar)
               : "memory");
}

template <int MODE, int FMT, typename OutT>
__global__ void __launch_bounds__(Wm4Cfg<MODE>::threads, 1)
grouped_gemm_wm4_kernel(const __grid_constant__ CUtensorMap tmC, const __grid_constant__ CUtensorMap tmX,
                        const uint8_t* __restrict__ scales_t, const float* __restrict__ tensor_scale,
                        const int32_t* __restrict__ offsets, int E, int K, int d, int F, long long rows_max,
                        const float* __restrict__ gate_of_row, OutT* __restrict__ out, int* err) {
  using C = Wm4Cfg<MODE>;
  constexpr int kBlockElems = FMT == MOE_FP4_MX ? 32 : 16;
  constexpr int kSpr = BK / kBlockElems;                    // scale bytes per row and k-block
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int* tile_start = reinterpret_cast<int*>(smem + C::tiles);
  int* sh32 = reinterpret_cast<int*>(smem + C::sh32);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::misc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::misc + 4);
  const uint32_t rank = cluster_ctarank();
  const int cid = (int)(blockIdx.x >> 1), ncl = (int)(gridDim.x >> 1);

  const int m_tiles = wm_m_tiles<MODE>(F, d);
  build_tile_starts(offsets, E, C::NT, m_tiles, rows_max, tile_start, sh32, err);
  const int total = tile_start[E];
  if (cid >= total) return;   // both CTAs of the pair see the same cid: uniform, nothing allocated

  const uint32_t bar_packed = sb + C::bars;
  const uint32_t bar_full = bar_packed + 8 * C::stages;
  const uint32_t bar_empty = bar_full + 8 * C::stages;
  const uint32_t bar_tfull = bar_empty + 8 * C::stages;
  const uint32_t bar_tempty = bar_tfull + 16;
  const uint32_t bar_fin = bar_tempty + 16;
  auto a_off = [&](int s, int a) { return s * C::stage_pitch + a * kWBlock; };
  auto b_off = [&](int s) { return s * C::stage_pitch + C::a_blocks * kWBlock; };
  auto p_off = [&](int s, int a) { return s * C::stage_pitch + C::a_blocks * kWBlock + C::b_bytes + a * C::packed_block; };
  auto s_off = [&](int s, int a) {
    return s * C::stage_pitch + C::a_blocks * (kWBlock + C::packed_block) + C::b_bytes + a * C::scale_block;
  };
  const long long rows_total = MODE == 0 ? (long long)E * 2 * F : (long long)E * d;
  const long long rows_pad = rows_total + kFp4PadRows;     // the prepared scales' row count

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::stages; ++s) {
      mbar_init(bar_packed + 8 * s, 1);
      mbar_init(bar_full + 8 * s, 2 * C::cvt_warps / C::cvt_groups);   // one arrive per warp of a group, both CTAs
      mbar_init(bar_empty + 8 * s, 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(bar_tfull + 8 * a, 1);
      mbar_init(bar_tempty + 8 * a, 2 * 32 * C::epi_warps);
    }
    mbar_init(bar_fin, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(kWTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int KB = K / BK;                                     // K is a multiple of 64

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer (both CTAs)
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int last_phase[C::stages];
#pragma unroll
      for (int s = 0; s < C::stages; ++s) last_phase[s] = -1;
      bool ok = true;
      for (int tile = cid; ok && tile < total; tile += ncl) {
        const TileCoord tc = tile_coord(tile_start, offsets, E, C::NT, tile);
        const int n = wm_n<MODE>(tc.rows);
        const int w_row = MODE == 0 ? tc.e * 2 * F + tc.n_tile * 256 + (int)rank * kWRows
                                    : tc.e * d + tc.n_tile * 256 + (int)rank * kWRows;
        const int x_row = tc.row0 + (int)rank * (n / 2);
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait(bar_empty + 8 * stage, phase ^ 1u, abort_flag, err)) { ok = false; break; }
          const uint32_t pk = bar_packed + 8 * stage;
          mbar_expect_tx(pk, (uint32_t)(C::a_blocks * (C::packed_block + kWRows * kSpr) + (n / 2) * BK * 2));
#pragma unroll
          for (int a = 0; a < C::a_blocks; ++a) {
            const int row = w_row + (a ? F : 0);
            tma_load_2d(sb + (uint32_t)p_off(stage, a), &tmC, pk, kb * (BK / 2), row);
            bulk_load(sb + (uint32_t)s_off(stage, a), scales_t + ((long long)kb * rows_pad + row) * kSpr,
                      (uint32_t)(kWRows * kSpr), pk);
          }
          for (int xb = 0; xb < n / 2; xb += kWXBox)      // n / 2 is a multiple of 16
            tma_load_2d(sb + (uint32_t)(b_off(stage) + xb * BK * 2), &tmX, pk, kb * BK, x_row + xb);
          last_phase[stage] = (int)phase;
          if (++stage == C::stages) { stage = 0; phase ^= 1u; }
        }
      }
      if (!ok) {
        for (int s = 0; s < C::stages; ++s)
          if (last_phase[s] >= 0) mbar_wait_drain(bar_packed + 8 * s, (uint32_t)last_phase[s], err);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (even CTA)
    if (lane == 0 && rank == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      bool ok = true;
      for (int tile = cid; ok && tile < total; tile += ncl, ++it) {
        const int acc = it & 1;
        const uint32_t acc_phase = (uint32_t)(it >> 1) & 1u;
        const TileCoord tc = tile_coord(tile_start, offsets, E, C::NT, tile);
        const uint32_t idesc = make_idesc(2 * kWRows, wm_n<MODE>(tc.rows));
        if (!mbar_wait(bar_tempty + 8 * acc, acc_phase ^ 1u, abort_flag, err)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * 256);
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait(bar_full + 8 * stage, phase, abort_flag, err)) { ok = false; break; }
          tc_fence_after();
          const uint64_t bdesc = sw128_desc(sb + (uint32_t)b_off(stage));
          const uint64_t adesc0 = sw128_desc(sb + (uint32_t)a_off(stage, 0));
          const uint64_t adesc1 = sw128_desc(sb + (uint32_t)a_off(stage, MODE == 0 ? 1 : 0));
#pragma unroll
          for (int kk = 0; kk < BK / UMMA_K; ++kk) {
            const uint32_t accumulate = (kb | kk) != 0 ? 1u : 0u;
            umma_bf16_pair(d_tmem, adesc0 + 2 * kk, bdesc + 2 * kk, idesc, accumulate);
            if (MODE == 0) umma_bf16_pair(d_tmem + 128, adesc1 + 2 * kk, bdesc + 2 * kk, idesc, accumulate);
          }
          umma_commit_pair_both(bar_empty + 8 * stage);
          if (++stage == C::stages) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        umma_commit_pair_both(bar_tfull + 8 * acc);
      }
      umma_commit_pair(bar_fin);
      mbar_wait_drain(bar_fin, 0, err);
    }
  } else if (warp < 2 + C::epi_warps) {
    // ------------------------------------------------------------ epilogue (both CTAs)
    const int q = warp & 3;
    uint8_t* stage = smem + C::stage + (warp - 2) * kStageWarpBytes;
    int it = 0;
    for (int tile = cid; tile < total; tile += ncl, ++it) {
      const TileCoord tc = tile_coord(tile_start, offsets, E, C::NT, tile);
      const int acc = it & 1;
      const uint32_t acc_phase = (uint32_t)(it >> 1) & 1u;
      // the first gates, fetched while the tile's MMAs still run
      const float g0 = MODE == 1 ? wm_gate(gate_of_row, tc, 0, lane) : 1.f;
      const float g1 = MODE == 1 ? wm_gate(gate_of_row, tc, 1, lane) : 1.f;
      const bool got = mbar_wait(bar_tfull + 8 * acc, acc_phase, abort_flag, err);
      if (!__all_sync(0xffffffffu, got)) break;
      __syncwarp();
      tc_fence_after();
      const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * 256);
      const float ws = tensor_scale ? __ldg(tensor_scale + tc.e) : 1.f;
      wm_epilogue_tile<MODE, OutT>(taddr, stage, lane, tc, (int)rank, q, d, F, ws, gate_of_row, out, g0, g1);
      tc_fence_before();
      mbar_arrive_remote(map_to_rank(bar_tempty + 8 * acc, 0));
    }
  } else {
    // ------------------------------------------------------------ converters (both CTAs)
    // kCvtGroups groups of warps take the stages in turn (group g the stages g, g + G, ...),
    // so G stages are decoded at once; a thread owns kWRows / group-size weight rows of its
    // stages (every block and chunk of them).
    constexpr int G = C::cvt_groups, GT = C::cvt_warps * 32 / G;   // groups, threads per group
    const int ct = threadIdx.x - 64 - 32 * C::epi_warps;     // 0 .. 32 cvt_warps - 1
    const int grp = ct / GT, r0 = ct % GT;                   // its group, its first row
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    int seq = 0;
    for (int tile = cid; ok && tile < total; tile += ncl) {
      for (int kb = 0; kb < KB; ++kb, ++seq) {
        if (seq % G == grp) {
          const bool got = mbar_wait(bar_packed + 8 * stage, phase, abort_flag, err);
          if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
#pragma unroll
          for (int r = r0; r < kWRows; r += GT)
#pragma unroll
            for (int a = 0; a < C::a_blocks; ++a) {
              const uint8_t* sc_p = smem + s_off(stage, a) + r * kSpr;
              const uint32_t sc = FMT == MOE_FP4_MX ? (uint32_t)*reinterpret_cast<const uint16_t*>(sc_p)
                                                    : *reinterpret_cast<const uint32_t*>(sc_p);
              convert_chunks<FMT>(smem + p_off(stage, a) + r * (BK / 2), sc, smem + a_off(stage, a), r, 0, 8);
            }
          fence_proxy_async_smem();                         // the MMAs read these through the async proxy
          __syncwarp();                                     // the warp's rows are written and fenced
          if (lane == 0) mbar_arrive_cluster(map_to_rank(bar_full + 8 * stage, 0));
        }
        if (++stage == C::stages) { stage = 0; phase ^= 1u; }
      }
    }
  }

  __syncthreads();
  cluster_sync();                                           // no remote arrive after a CTA exits
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(kWTmemCols) : "memory");
  }
}

template <int MODE, int FMT, typename OutT>
moe_status launch_wm4(const CUtensorMap& mc, const CUtensorMap& mx, const uint8_t* scales_t, const float* tscale,
                      const int32_t* offsets, int E, int K, int d, int F, long long rows_max, const float* gate_of_row,
                      void* out, cudaStream_t s) {
  using C = Wm4Cfg<MODE>;
  static std::atomic<int> configured[kMaxDevices];
  const moe_status st = ensure_smem_limit(configured, grouped_gemm_wm4_kernel<MODE, FMT, OutT>, C::smem);
  if (st != MOE_OK) return st;
  const long long max_tiles = ((rows_max + C::NT - 1) / C::NT + E) * (long long)wm_m_tiles<MODE>(F, d);
  int pairs = num_sms() / 2;
  if (max_tiles < pairs) pairs = (int)max_tiles;
  if (pairs < 1) pairs = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * pairs, 1, 1);
  cfg.blockDim = dim3(C::threads, 1, 1);
  cfg.dynamicSmemBytes = C::smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cuda_status(cudaLaunchKernelEx(&cfg, grouped_gemm_wm4_kernel<MODE, FMT, OutT>, mc, mx, scales_t, tscale,
                                        offsets, E, K, d, F, rows_max, gate_of_row, static_cast<OutT*>(out),
                                        err_ptr()));
}

// The k-block-major scale layout: out[kb][row][j] = in[row][kb * (64/block) + j] for
// rows < rows_total, zero for the padding rows.  One byte per thread, grid-stride.
__global__ void __launch_bounds__(256)
fp4_scales_kernel(const uint8_t* __restrict__ in, long long rows, int K, int spr, uint8_t* __restrict__ out) {
  const long long rows_pad = rows + kFp4PadRows;
  const long long per_kb = rows_pad * spr;
  const long long n = (long long)(K / BK) * per_kb;
  const long long ld = K / (BK / spr);                       // scale bytes per row of the input
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
    const long long kb = i / per_kb, rem = i - kb * per_kb;
    const long long row = rem / spr;
    const int j = (int)(rem - row * spr);
    out[i] = row < rows ? __ldg(in + row * ld + kb * spr + j) : (uint8_t)0;
  }
}

template <int MODE, typename OutT, bool GATHER = false>
moe_status launch_wm(const CUtensorMap& mw, const CUtensorMap& mx, const int32_t* offsets, int E, int K, int d,
                     int F, long long rows_max, const float* gate_of_row, void* out, cudaStream_t s,
                     const int32_t* token_of_row = nullptr, int n_tokens = 0) {
  using C = WmCfg<MODE>;
  static std::atomic<int> configured[kMaxDevices];
  const moe_status st = ensure_smem_limit(configured, grouped_gemm_wm_kernel<MODE, OutT, GATHER>, C::smem);
  if (st != MOE_OK) return st;
  const long long max_tiles = ((rows_max + C::NT - 1) / C::NT + E) * (long long)wm_m_tiles<MODE>(F, d);
  int pairs = num_sms() / 2;
  if (max_tiles < pairs) pairs = (int)max_tiles;
  if (pairs < 1) pairs = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * pairs, 1, 1);
  cfg.blockDim = dim3(C::threads, 1, 1);
  cfg.dynamicSmemBytes = C::smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cuda_status(cudaLaunchKernelEx(&cfg, grouped_gemm_wm_kernel<MODE, OutT, GATHER>, mw, mx, offsets, E, K, d,
                                        F, rows_max, gate_of_row, static_cast<OutT*>(out), err_ptr(), token_of_row,
                                        n_tokens));
}

}  // namespace

size_t fp4_scales_bytes(long long rows, int K, int fmt) {
  const int spr = BK / (fmt == MOE_FP4_MX ? 32 : 16);
  return (size_t)(K / BK) * (size_t)(rows + kFp4PadRows) * spr;
}

moe_status launch_prepare_fp4_scales(const uint8_t* scales, long long rows, int K, int fmt, uint8_t* out,
                                     cudaStream_t s) {
  const int spr = BK / (fmt == MOE_FP4_MX ? 32 : 16);
  const long long n = (long long)(K / BK) * (rows + kFp4PadRows) * spr;
  long long blocks = (n + 255) / 256;
  const long long cap = (long long)num_sms() * 16;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  fp4_scales_kernel<<<(unsigned)blocks, 256, 0, s>>>(scales, rows, K, spr, out);
  return check_launch();
}


// Gate/up, weight-major: H [rows_max, F] bf16 from x_perm [rows_max, d] and W_gu [E][2F][d].
moe_status launch_gate_up_wm(const void* x_rows, const int32_t* offsets, int E, int d, int F, long long rows_max,
                             const void* W_gu, void* h, cudaStream_t s) {
  if (rows_max == 0) return MOE_OK;
  if (d < BK || F < 8) return MOE_ERR_UNSUPPORTED;
  CUtensorMap mw, mx;
  if (!make_map(&mw, W_gu, (unsigned long long)E * 2 * F, d, kWRows)) return MOE_ERR_UNSUPPORTED;
  if (!make_map(&mx, x_rows, (unsigned long long)rows_max, d, kWXBox)) return MOE_ERR_UNSUPPORTED;
  return launch_wm<0, __nv_bfloat16>(mw, mx, offsets, E, d, d, F, rows_max, nullptr, h, s);
}

// Gate/up, weight-major, gathered: H [rows_max, F] bf16 from the token rows x[token_of_row[r]]
// (x [T, d] bf16) and W_gu [E][2F][d]; no permuted copy of x.
moe_status launch_gate_up_wm_gather(const void* x, const int32_t* token_of_row, int T, const int32_t* offsets, int E,
                                    int d, int F, long long rows_max, const void* W_gu, void* h, cudaStream_t s) {
  if (rows_max == 0 || T == 0) return MOE_OK;
  if (d < BK || F < 8) return MOE_ERR_UNSUPPORTED;
  CUtensorMap mw, mx;
  if (!make_map(&mw, W_gu, (unsigned long long)E * 2 * F, d, kWRows)) return MOE_ERR_UNSUPPORTED;
  if (!make_map(&mx, x, (unsigned long long)T, d, 1)) return MOE_ERR_UNSUPPORTED;   // one-row box: row gathers
  return launch_wm<0, __nv_bfloat16, true>(mw, mx, offsets, E, d, d, F, rows_max, nullptr, h, s, token_of_row, T);
}

// Down, weight-major: gated rows [rows_max, d] (bf16 or fp32) from H [rows_max, F] and W_dn [E][d][F].
moe_status launch_down_wm(const void* h, const int32_t* offsets, int E, int d, int F, long long rows_max,
                          const void* W_dn, const float* gate_of_row, int y_dtype, void* y_rows, cudaStream_t s) {
  if (rows_max == 0) return MOE_OK;
  if (F < BK || d < 8) return MOE_ERR_UNSUPPORTED;
  CUtensorMap mw, mx;
  if (!make_map(&mw, W_dn, (unsigned long long)E * d, F, kWRows)) return MOE_ERR_UNSUPPORTED;
  if (!make_map(&mx, h, (unsigned long long)rows_max, F, kWXBox)) return MOE_ERR_UNSUPPORTED;
  if (y_dtype == MOE_F32) return launch_wm<1, float>(mw, mx, offsets, E, F, d, F, rows_max, gate_of_row, y_rows, s);
  return launch_wm<1, __nv_bfloat16>(mw, mx, offsets, E, F, d, F, rows_max, gate_of_row, y_rows, s);
}

// Gate/up and down with 4-bit weights, weight-major.  Codes [rows, K/2] as
// moe_quantize_fp4_host writes them (rows = E 2F or E d), scales in the layout of
// launch_prepare_fp4_scales; tensor_scale [E] fp32 per expert (NVFP4) or NULL (MXFP4).  K
// (d for gate/up, F for down) must be a multiple of 64.
moe_status launch_gate_up_fp4(const void* x_rows, const int32_t* offsets, int E, int d, int F, long long rows_max,
                              const uint8_t* codes, const uint8_t* scales_t, int fmt, const float* tensor_scale,
                              void* h, cudaStream_t s) {
  if (rows_max == 0) return MOE_OK;
  CUtensorMap mc, mx;
  if (!make_map_u8(&mc, codes, (unsigned long long)E * 2 * F, d / 2, BK / 2, kWRows)) return MOE_ERR_UNSUPPORTED;
  if (!make_map(&mx, x_rows, (unsigned long long)rows_max, d, kWXBox)) return MOE_ERR_UNSUPPORTED;
  if (fmt == MOE_FP4_MX)
    return launch_wm4<0, MOE_FP4_MX, __nv_bfloat16>(mc, mx, scales_t, nullptr, offsets, E, d, d, F, rows_max,
                                                     nullptr, h, s);
  return launch_wm4<0, MOE_FP4_NV, __nv_bfloat16>(mc, mx, scales_t, tensor_scale, offsets, E, d, d, F, rows_max,
                                                   nullptr, h, s);
}

moe_status launch_down_fp4(const void* h, const int32_t* offsets, int E, int d, int F, long long rows_max,
                           const uint8_t* codes, const uint8_t* scales_t, int fmt, const float* tensor_scale,
                           const float* gate_of_row, int y_dtype, void* y_rows, cudaStream_t s) {
  if (rows_max == 0) return MOE_OK;
  CUtensorMap mc, mx;
  if (!make_map_u8(&mc, codes, (unsigned long long)E * d, F / 2, BK / 2, kWRows)) return MOE_ERR_UNSUPPORTED;
  if (!make_map(&mx, h, (unsigned long long)rows_max, F, kWXBox)) return MOE_ERR_UNSUPPORTED;
  const float* ts = fmt == MOE_FP4_NV ? tensor_scale : nullptr;
#define MOE_WM4(FMT, T) \
  return launch_wm4<1, FMT, T>(mc, mx, scales_t, ts, offsets, E, F, d, F, rows_max, gate_of_row, y_rows, s)
  if (fmt == MOE_FP4_MX) {
    if (y_dtype == MOE_F32) MOE_WM4(MOE_FP4_MX, float);
    MOE_WM4(MOE_FP4_MX, __nv_bfloat16);
  }
  if (y_dtype == MOE_F32) MOE_WM4(MOE_FP4_NV, float);
  MOE_WM4(MOE_FP4_NV, __nv_bfloat16);
#undef MOE_WM4
}

}  // namespace moe
