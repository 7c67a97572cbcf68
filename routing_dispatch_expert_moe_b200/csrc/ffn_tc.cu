// Grouped SwiGLU expert GEMMs on the 5th-generation tensor cores (sm_100a).
//
// Expert FFN: "Hugging Face 图解 Mixture of Experts（MoE）原理、训练与推理权衡", section
// "什么是混合专家模型" (each expert is an FFN) and section "更多关于高效训练的内容"
// (experts receive uneven numbers of tokens; handle them without padding or drops).
// SwiGLU form: H = silu(X Wg^T) * (X Wu^T), Y = gate * (H Wd^T), no biases.
//
// Two persistent kernel templates (single CTA, and CTA pairs below), one per-mode
// producer and epilogue:
//   MODE 0 (gate_up): A = X [rows, d], B = W_gu[e] ([2F, d], gate rows then up rows).
//       A 256-wide B tile holds 128 gate rows and the matching 128 up rows, so one
//       128x256 accumulator carries g (columns 0..127) and u (128..255) for the same
//       128 features; the epilogue writes H = silu(g) * u as bf16.
//   MODE 1 (down): A = H [rows, F], B = W_dn[e] ([d, F]); the epilogue scales each row
//       by gate_of_row and writes bf16 or fp32 rows.
//   MODE 3 (down + combine): as MODE 1, but the gated row is added into the fp32 output
//       row of its token (y[token_of_row[r]] += ...) with 16-byte vector atomics, so the
//       gated rows never reach memory and no separate combine pass runs.  The fp32 sum
//       order over a token's experts is whatever order the tiles finish in.
//   MODE 4 (gate_up, gathered): as MODE 0, but the A rows are gathered straight from the
//       token matrix, A row r = x[token_of_row[r]], so no permuted copy of x is written
//       or read.  The producer warp copies them with 16-byte cp.async into the same
//       128-byte-swizzled layout TMA writes; B still arrives by TMA.
//
// Per CTA (1 per SM, 192 threads):
//   warp 0   TMA producer: 128x64 A tile + 256x64 B tile per stage (128-byte swizzle),
//            4-stage ring of mbarriers (full: TMA bytes landed, empty: MMAs done).
//   warp 1   allocates 512 TMEM columns; one thread issues tcgen05.mma
//            (kind::f16, bf16 x bf16 -> fp32, M=128, N=256, K=16) and tcgen05.commit.
//   warps 2-5 epilogue: tcgen05.ld 32x32b (thread = accumulator row), fused SwiGLU or
//            gate scaling, bf16 rounding, masked 16-byte stores.  Two 256-column TMEM
//            accumulators let the epilogue of tile i overlap the mainloop of tile i+1.
// Tiles come from the device-side schedule built from the offsets array; a tile never
// writes a row outside its expert's range or a column outside the output width.
// Every barrier wait is bounded (MOE_DEVERR_PIPE_TIMEOUT, then an orderly exit: MMAs
// drained, outstanding TMA loads awaited, TMEM freed).
// The CTA-pair kernel (further below) runs 256x256 tiles over two SMs with cta_group::2
// MMAs; it is used when groups average at least 256 rows.  No load uses cluster
// multicast.
#include <cuda.h>
#include <stdlib.h>
#include <string.h>

#include "common.cuh"
#include "tc_prims.cuh"
#include "tile_sched.cuh"

namespace moe {
namespace {

constexpr int BM = 128, BN = 256, STAGES = 4;
constexpr int kThreadsTC = 192;
constexpr int A_STAGE = BM * BK * 2;   // 16 KB
constexpr int B_STAGE = BN * BK * 2;   // 32 KB
constexpr int kMaxE = 1024;
constexpr uint32_t kTmemCols = 512;

struct L {
  static constexpr int a = 0;
  static constexpr int b = STAGES * A_STAGE;
  static constexpr int bars = b + STAGES * B_STAGE;
  static constexpr int nbars = 2 * STAGES + 4 + 1;          // full, empty, tfull[2], tempty[2], fin
  static constexpr int misc = bars + nbars * 8;              // tmem slot, abort flag
  static constexpr int tiles = misc + 16;                    // int tile_start[kMaxE + 1]
  static constexpr int sh32 = tiles + (kMaxE + 1) * 4;      // int[32]
  static constexpr int stage = (sh32 + 32 * 4 + 15) / 16 * 16;   // 4 epilogue warps x 32 x 144 B
  static constexpr int end = stage + 4 * 32 * (32 * 4 + 16);
};
constexpr size_t kSmemBytes = L::end + 1024;                 // + alignment slack

// Output column tiles per row tile: 128 H features per gate/up tile (128 gate + 128 up
// accumulator columns), 256 outputs per down tile.
template <int MODE>
__host__ __device__ __forceinline__ int n_tiles_of(int F, int N_out) {
  if (MODE == 0 || MODE == 4) return (F + 127) / 128;
  return (N_out + BN - 1) / BN;
}

// L2 policy that keeps lines resident ahead of streaming data (the fp32 output rows the
// fused combine adds into are touched by every expert of their token).
__device__ __forceinline__ uint64_t l2_evict_last_policy() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}
// 16-byte vector atomic add (no return value) with an L2 cache policy.
__device__ __forceinline__ void red_add_v4(float* p, const float4& v, uint64_t pol) {
  asm volatile("red.global.add.L2::cache_hint.v4.f32 [%0], {%1, %2, %3, %4}, %5;" ::"l"(p), "f"(v.x), "f"(v.y),
               "f"(v.z), "f"(v.w), "l"(pol)
               : "memory");
}

// MODE 3: the same turn-around, then each 16-byte piece is added into the output row of
// its token (tok: this lane's row's token, -1 = skip).  Every atomic instruction of the
// warp covers 4 rows x 128 contiguous bytes.
__device__ __forceinline__ void stage_red32(uint8_t* stage, const float (&v)[32], int lane, float* y, int tok,
                                            long long ld, int col, int ncols, uint64_t pol) {
  float4* dst = reinterpret_cast<float4*>(stage + lane * kStagePitchF32);
#pragma unroll
  for (int q = 0; q < 8; ++q) dst[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
  __syncwarp();
  const int rs = lane >> 3, cv = lane & 7;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int r = i * 4 + rs;
    const int t = __shfl_sync(0xffffffffu, tok, r);
    const float4 x = *reinterpret_cast<const float4*>(stage + r * kStagePitchF32 + cv * 16);
    if (t >= 0 && col + cv * 4 + 4 <= ncols) red_add_v4(y + (long long)t * ld + col + cv * 4, x, pol);
  }
  __syncwarp();
}

// OutT: element type of the output rows (MODE 0 always writes bf16 H; MODE 1 writes
// bf16 or fp32 gated rows; MODE 3 adds into fp32 token rows).
// One tile's epilogue for one warp: its 32 accumulator rows (TMEM lanes at taddr) become
// output rows wrow0 .. wrow0 + wrows - 1.  The whole warp must call it (tcgen05.ld is
// .sync.aligned); rows past wrows are read but not stored.
//   MODE 0: columns [0,128) gate, [128,256) up -> H = silu(g) * u for features n_tile*128 + ...
//   MODE 1: 256 columns -> gate_of_row[row] * acc for outputs n_tile*256 + ...
// MODE 1 / 3 process the 32-column chunks [c_begin, c_end) of the 256 (a warp may own half).
template <int MODE, typename OutT>
__device__ __forceinline__ void epilogue_tile(uint32_t taddr, uint8_t* stage, int lane, long long wrow0, int wrows,
                                              int n_tile, int F, int N_out, const float* __restrict__ gate_of_row,
                                              OutT* __restrict__ out, const int32_t* __restrict__ token_of_row,
                                              int n_tokens, int* err, float gs, int c_begin = 0,
                                              int c_end = BN / 32) {
  if constexpr (MODE == 3) {
    const int n0 = n_tile * BN;
    const uint64_t pol = l2_evict_last_policy();
    int tok = -1;
    if (lane < wrows) {
      tok = __ldg(token_of_row + wrow0 + lane);
      if ((unsigned)tok >= (unsigned)n_tokens) {
        record_error(err, MOE_DEVERR_ROW);
        tok = -1;
      }
    }
#pragma unroll 1
    for (int c = c_begin; c < c_end; ++c) {
      uint32_t v32[32];
      tmem_ld32(taddr + c * 32, v32);
      tmem_wait_ld();
      tmem_regs_ready(v32);
      float y[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) y[i] = __uint_as_float(v32[i]) * gs;
      stage_red32(stage, y, lane, reinterpret_cast<float*>(out), tok, N_out, n0 + c * 32, N_out, pol);
    }
  } else if constexpr (MODE == 0 || MODE == 4) {
    const int f0 = n_tile * 128;
#pragma unroll 1
    for (int c = 0; c < 4; ++c) {
      uint32_t g[32], u[32];
      tmem_ld32(taddr + c * 32, g);
      tmem_ld32(taddr + 128 + c * 32, u);
      tmem_wait_ld();
      tmem_regs_ready(g);
      tmem_regs_ready(u);
      float h[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const float gi = __uint_as_float(g[i]);
        // fast exp / divide: H is rounded to bf16 next, far coarser than their error; the
        // exact forms made this epilogue the bound of the gate/up GEMM
        h[i] = __fdividef(gi, 1.f + __expf(-gi)) * __uint_as_float(u[i]);
      }
      stage_store32<OutT>(stage, h, lane, out, wrow0, wrows, F, f0 + c * 32, F);
    }
  } else {
    static_assert(MODE == 1, "grouped GEMM modes: 0 gate/up, 1 down, 3 down + combine, 4 gathered gate/up");
    const int n0 = n_tile * BN;
    // two 32-column chunks per TMEM wait: with K = F of a few k-blocks this epilogue is as
    // long as the tile's mainloop, and each wait is a full TMEM round trip
#pragma unroll 1
    for (int c = c_begin; c < c_end; c += 2) {
      const bool two = c + 1 < c_end;                      // warp-uniform
      uint32_t va[32], vb[32];
      tmem_ld32(taddr + c * 32, va);
      if (two) tmem_ld32(taddr + (c + 1) * 32, vb);
      tmem_wait_ld();
      tmem_regs_ready(va);
      tmem_regs_ready(vb);
      float y[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) y[i] = __uint_as_float(va[i]) * gs;
      stage_store32<OutT>(stage, y, lane, out, wrow0, wrows, N_out, n0 + c * 32, N_out);
      if (two) {
#pragma unroll
        for (int i = 0; i < 32; ++i) y[i] = __uint_as_float(vb[i]) * gs;
        stage_store32<OutT>(stage, y, lane, out, wrow0, wrows, N_out, n0 + (c + 1) * 32, N_out);
      }
    }
  }
}

// Producer warp of the gathered gate/up GEMM (MODE 4).  Per stage, lane 0 arms the full
// barrier with the B bytes and issues B's TMA loads; every lane copies its share of the
// 128 A rows (lane = 16-byte chunk lane & 7 of rows lane >> 3, +4, +8, ...), each row
// x[token_of_row[r]][k-block], with cp.async into the 128-byte-swizzled layout: chunk c
// of row r lands at r * 128 + ((c ^ (r & 7)) * 16).  Rows past the tile and columns past
// K are zero-filled.  Each lane then queues a hardware arrival on the stage's full
// barrier that fires when its copies have landed (count 1 + 32), so the warp moves on
// to the next stage at once; the MMA thread fences the stage for the async proxy after
// its wait.
// (Measured: slower than the permute copy plus the box-loaded GEMM, because every A tile
// is re-read once per n-tile as 128-byte rows; it saves the permuted buffer.  TMA row
// gathers, four rows per instruction and 32 per stage here, were slower still: 1.26
// against 0.76 ms on the 8192-token, 64-expert layer.)
__device__ __forceinline__ void gather_producer(const CUtensorMap* tmB, uint32_t sb, uint32_t bar_full,
                                                uint32_t bar_empty, const int* tile_start,
                                                const int32_t* __restrict__ offsets, int E, int K, int F,
                                                const int32_t* __restrict__ token_of_row, int n_tokens,
                                                const __nv_bfloat16* __restrict__ x, volatile int* abort_flag,
                                                int* err) {
  const int lane = threadIdx.x & 31;
  const int cv = lane & 7, rsub = lane >> 3;
  const int KB = (K + BK - 1) / BK;
  const int total = tile_start[E];
  int stage = 0;
  uint32_t phase = 0;
  int last_phase[STAGES];
#pragma unroll
  for (int s = 0; s < STAGES; ++s) last_phase[s] = -1;
  bool ok = true;
  for (int tile = blockIdx.x; ok && tile < total; tile += gridDim.x) {
    const TileCoord tc = tile_coord(tile_start, offsets, E, BM, tile);
    int tok[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const int r = i * 4 + rsub;
      int t = -1;
      if (r < tc.rows) {
        t = __ldg(token_of_row + tc.row0 + r);
        if ((unsigned)t >= (unsigned)n_tokens) {
          record_error(err, MOE_DEVERR_ROW);
          t = -1;
        }
      }
      tok[i] = t;
    }
    const int g_row = tc.e * 2 * F + tc.n_tile * 128;
    for (int kb = 0; kb < KB; ++kb) {
      const bool got = mbar_wait(bar_empty + 8 * stage, phase ^ 1u, abort_flag, err);
      if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
      const uint32_t full = bar_full + 8 * stage;
      const uint32_t a_dst = sb + L::a + stage * A_STAGE;
      if (lane == 0) {
        const uint32_t b_dst = sb + L::b + stage * B_STAGE;
        mbar_expect_tx(full, B_STAGE);
        tma_load_2d(b_dst, tmB, full, kb * BK, g_row);
        tma_load_2d(b_dst + B_STAGE / 2, tmB, full, kb * BK, g_row + F);
        last_phase[stage] = (int)phase;
      }
      const int kcol = kb * BK + cv * 8;
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const int r = i * 4 + rsub;
        const bool v = tok[i] >= 0 && kcol < K;
        const __nv_bfloat16* src = x + (v ? (long long)tok[i] * K + kcol : 0LL);
        cp_async16(a_dst + r * 128 + ((cv ^ (r & 7)) << 4), src, v ? 16u : 0u);
      }
      cp_async_arrive_noinc(full);
      if (++stage == STAGES) { stage = 0; phase ^= 1u; }
    }
  }
  cp_async_wait_all();                      // no copy may land after the CTA has exited
  if (!ok && lane == 0) {
    // let every issued B copy land before the CTA can exit
    for (int s = 0; s < STAGES; ++s)
      if (last_phase[s] >= 0) mbar_wait_drain(bar_full + 8 * s, (uint32_t)last_phase[s], err);
  }
}

template <int MODE, typename OutT>
__global__ void __launch_bounds__(kThreadsTC, 1)
grouped_gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                       const int32_t* __restrict__ offsets, int E, int K, int N_out, int F,
                       long long rows_max, const float* __restrict__ gate_of_row,
                       OutT* __restrict__ out, const int32_t* __restrict__ token_of_row, int n_tokens,
                       const __nv_bfloat16* __restrict__ a_gather, int* err) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int* tile_start = reinterpret_cast<int*>(smem + L::tiles);
  int* sh32 = reinterpret_cast<int*>(smem + L::sh32);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::misc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::misc + 4);

  const int n_tiles = n_tiles_of<MODE>(F, N_out);
  build_tile_starts(offsets, E, BM, n_tiles, rows_max, tile_start, sh32, err);
  const int total = tile_start[E];
  if ((int)blockIdx.x >= total) return;   // uniform: nothing allocated yet

  const uint32_t bar_full = sb + L::bars;
  const uint32_t bar_empty = bar_full + 8 * STAGES;
  const uint32_t bar_tfull = bar_empty + 8 * STAGES;
  const uint32_t bar_tempty = bar_tfull + 16;
  const uint32_t bar_fin = bar_tempty + 16;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      // gathered A: the B expect_tx arrival plus one cp.async arrival per producer lane
      mbar_init(bar_full + 8 * s, MODE == 4 ? 1 + 32 : 1);
      mbar_init(bar_empty + 8 * s, 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(bar_tfull + 8 * a, 1);
      mbar_init(bar_tempty + 8 * a, 128);
    }
    mbar_init(bar_fin, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int KB = (K + BK - 1) / BK;

  if (MODE == 4 && warp == 0) {
    gather_producer(&tmB, sb, bar_full, bar_empty, tile_start, offsets, E, K, F, token_of_row, n_tokens, a_gather,
                    abort_flag, err);
  } else if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int last_phase[STAGES];
#pragma unroll
      for (int s = 0; s < STAGES; ++s) last_phase[s] = -1;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < total; tile += gridDim.x) {
        const TileCoord tc = tile_coord(tile_start, offsets, E, BM, tile);
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait(bar_empty + 8 * stage, phase ^ 1u, abort_flag, err)) { ok = false; break; }
          const uint32_t full = bar_full + 8 * stage;
          mbar_expect_tx(full, A_STAGE + B_STAGE);
          const uint32_t a_dst = sb + L::a + stage * A_STAGE;
          const uint32_t b_dst = sb + L::b + stage * B_STAGE;
          tma_load_2d(a_dst, &tmA, full, kb * BK, tc.row0);
          if (MODE == 0) {
            const int g_row = tc.e * 2 * F + tc.n_tile * 128;
            tma_load_2d(b_dst, &tmB, full, kb * BK, g_row);
            tma_load_2d(b_dst + B_STAGE / 2, &tmB, full, kb * BK, g_row + F);
          } else {
            tma_load_2d(b_dst, &tmB, full, kb * BK, tc.e * N_out + tc.n_tile * BN);
          }
          last_phase[stage] = (int)phase;
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      if (!ok) {
        // let every issued copy land before the CTA can exit
        for (int s = 0; s < STAGES; ++s)
          if (last_phase[s] >= 0) mbar_wait_drain(bar_full + 8 * s, (uint32_t)last_phase[s], err);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < total; tile += gridDim.x, ++it) {
        const int acc = it & 1;
        const uint32_t acc_phase = (uint32_t)(it >> 1) & 1u;
        if (!mbar_wait(bar_tempty + 8 * acc, acc_phase ^ 1u, abort_flag, err)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait(bar_full + 8 * stage, phase, abort_flag, err)) { ok = false; break; }
          tc_fence_after();
          if (MODE == 4) fence_proxy_async_smem();   // A rows were written by cp.async (generic proxy)
          const uint64_t adesc = sw128_desc(sb + L::a + stage * A_STAGE);
          const uint64_t bdesc = sw128_desc(sb + L::b + stage * B_STAGE);
#pragma unroll
          for (int kk = 0; kk < BK / UMMA_K; ++kk)   // +32 bytes along K per step (>> 4 = 2)
            umma_bf16(d_tmem, adesc + 2 * kk, bdesc + 2 * kk, make_idesc(BM, BN),
                      (kb | kk) != 0 ? 1u : 0u);
          umma_commit(bar_empty + 8 * stage);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        umma_commit(bar_tfull + 8 * acc);
      }
      // all issued MMAs complete before TMEM can be released
      umma_commit(bar_fin);
      mbar_wait_drain(bar_fin, 0, err);
    }
  } else {
    // ------------------------------------------------------------ epilogue (warps 2..5)
    const int q = warp & 3;                 // TMEM lane quarter this warp may access
    const int r_in = q * 32 + lane;         // accumulator row == tile row
    uint8_t* stage = smem + L::stage + (warp - 2) * kStageWarpBytes;
    int it = 0;
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x, ++it) {
      const TileCoord tc = tile_coord(tile_start, offsets, E, BM, tile);
      const int acc = it & 1;
      const uint32_t acc_phase = (uint32_t)(it >> 1) & 1u;
      const long long wrow0 = (long long)tc.row0 + q * 32;          // first row of this warp
      const int wrows = min(32, max(0, tc.rows - q * 32));          // valid rows of this warp
      // the row's gate, fetched while the tile's MMAs still run
      const float gs = ((MODE == 1 || MODE == 3) && lane < wrows && gate_of_row) ? __ldg(gate_of_row + wrow0 + lane)
                                                                                  : 1.f;
      const bool got = mbar_wait(bar_tfull + 8 * acc, acc_phase, abort_flag, err);
      // tcgen05.ld is .sync.aligned: the whole warp goes on, or the whole warp stops
      if (!__all_sync(0xffffffffu, got)) break;
      __syncwarp();
      tc_fence_after();
      const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * BN);
      (void)r_in;
      // a warp past the group's last row has nothing to read or store (warp-uniform)
      if (wrows > 0)
        epilogue_tile<MODE, OutT>(taddr, stage, lane, wrow0, wrows, tc.n_tile, F, N_out, gate_of_row, out,
                                  token_of_row, n_tokens, err, gs);
      tc_fence_before();
      mbar_arrive(bar_tempty + 8 * acc);
    }
  }

  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(kTmemCols) : "memory");
  }
}

// =====================================================================================
// CTA-pair version: a cluster of 2 CTAs computes a 256 x 256 tile.  Each CTA stages its
// own 128 rows of A and half (128 rows) of B per k-block -- 32 KB instead of 48 KB, so a
// 6-stage ring fits -- and the even CTA issues cta_group::2 MMAs that read both CTAs'
// stages and accumulate each CTA's 128 rows in that CTA's TMEM.
//   full[s]   (even CTA only) : even CTA's expect_tx + both CTAs' TMA bytes
//   empty[s]  (both CTAs)     : MMA completion, multicast commit
//   tfull[a]  (both CTAs)     : accumulator ready, multicast commit
//   tempty[a] (even CTA only) : 256 epilogue threads of both CTAs
// Cluster barriers after set-up and before teardown; every wait bounded.
// =====================================================================================
constexpr int B2_STAGE = BM * BK * 2;                        // 128 B-rows per CTA: 16 KB

// Configuration of the CTA-pair kernel.  WIDE (down GEMMs with a short K, chosen at
// launch): eight epilogue warps, two per TMEM lane quarter, each taking half of the 256
// output columns, and five stages to make room for their staging.  With K <= 512 a tile
// has at most 8 k-blocks and its 256-column fp32 epilogue, not the operand stream, sets
// the pace; at longer K the sixth stage is worth more (measured).
template <bool WIDE>
struct PairCfg {
  static constexpr int stages = WIDE ? 5 : 6;
  static constexpr int epi_warps = WIDE ? 8 : 4;
  static constexpr int threads = 64 + 32 * epi_warps;
  static constexpr int a = 0;
  static constexpr int b = stages * A_STAGE;
  static constexpr int bars = b + stages * B2_STAGE;
  static constexpr int nbars = 2 * stages + 4 + 1;
  static constexpr int misc = bars + nbars * 8;
  static constexpr int tiles = misc + 16;
  static constexpr int sh32 = tiles + (kMaxE + 1) * 4;
  static constexpr int stage = (sh32 + 32 * 4 + 15) / 16 * 16;
  static constexpr int end = stage + epi_warps * kStageWarpBytes;
  static constexpr size_t smem = end + 1024;
  static_assert(smem <= 232448, "shared memory per CTA");
};

template <int MODE, typename OutT, bool WIDE>
__global__ void __launch_bounds__(PairCfg<WIDE>::threads, 1)
grouped_gemm_tc2_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                        const int32_t* __restrict__ offsets, int E, int K, int N_out, int F,
                        long long rows_max, const float* __restrict__ gate_of_row,
                        OutT* __restrict__ out, const int32_t* __restrict__ token_of_row, int n_tokens,
                       int* err) {
  using C = PairCfg<WIDE>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int* tile_start = reinterpret_cast<int*>(smem + C::tiles);
  int* sh32 = reinterpret_cast<int*>(smem + C::sh32);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::misc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::misc + 4);
  const uint32_t rank = cluster_ctarank();                   // 0 = even CTA (MMA issuer)
  const int cid = (int)(blockIdx.x >> 1), ncl = (int)(gridDim.x >> 1);
  constexpr int PM = 2 * BM;                                 // rows per pair tile

  const int n_tiles = n_tiles_of<MODE>(F, N_out);
  build_tile_starts(offsets, E, PM, n_tiles, rows_max, tile_start, sh32, err);
  const int total = tile_start[E];
  if (cid >= total) return;   // both CTAs of the pair see the same cid: uniform, nothing allocated

  const uint32_t bar_full = sb + C::bars;
  const uint32_t bar_empty = bar_full + 8 * C::stages;
  const uint32_t bar_tfull = bar_empty + 8 * C::stages;
  const uint32_t bar_tempty = bar_tfull + 16;
  const uint32_t bar_fin = bar_tempty + 16;

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
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();                                           // peer barriers initialised
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int KB = (K + BK - 1) / BK;

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
        const TileCoord tc = tile_coord(tile_start, offsets, E, PM, tile);
        const int a_row = tc.row0 + (int)rank * BM;
        int b_row;
        if (MODE == 0) b_row = tc.e * 2 * F + (rank ? F : 0) + tc.n_tile * 128;   // even: gate, odd: up
        else b_row = tc.e * N_out + tc.n_tile * BN + (int)rank * BM;
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait(bar_empty + 8 * stage, phase ^ 1u, abort_flag, err)) { ok = false; break; }
          if (rank == 0) mbar_expect_tx(bar_full + 8 * stage, 2 * (A_STAGE + B2_STAGE));
          const uint32_t full_c = map_to_rank(bar_full + 8 * stage, 0);
          tma_load_2d_pair(sb + C::a + stage * A_STAGE, &tmA, full_c, kb * BK, a_row);
          tma_load_2d_pair(sb + C::b + stage * B2_STAGE, &tmB, full_c, kb * BK, b_row);
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
        if (!mbar_wait(bar_tempty + 8 * acc, acc_phase ^ 1u, abort_flag, err)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait(bar_full + 8 * stage, phase, abort_flag, err)) { ok = false; break; }
          tc_fence_after();
          const uint64_t adesc = sw128_desc(sb + C::a + stage * A_STAGE);
          const uint64_t bdesc = sw128_desc(sb + C::b + stage * B2_STAGE);
#pragma unroll
          for (int kk = 0; kk < BK / UMMA_K; ++kk)
            umma_bf16_pair(d_tmem, adesc + 2 * kk, bdesc + 2 * kk, make_idesc(2 * BM, BN), (kb | kk) != 0 ? 1u : 0u);
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
    const int q = warp & 3;                                  // TMEM lane quarter this warp may access
    const int ew = warp - 2;
    const int c_begin = WIDE ? (ew >> 2) * 4 : 0;            // its column chunks
    const int c_end = WIDE ? c_begin + 4 : BN / 32;
    uint8_t* stage = smem + C::stage + ew * kStageWarpBytes;
    int it = 0;
    for (int tile = cid; tile < total; tile += ncl, ++it) {
      const TileCoord tc = tile_coord(tile_start, offsets, E, PM, tile);
      const int acc = it & 1;
      const uint32_t acc_phase = (uint32_t)(it >> 1) & 1u;
      const int cta_rows = min(BM, max(0, tc.rows - (int)rank * BM));
      const long long wrow0 = (long long)tc.row0 + (int)rank * BM + q * 32;
      const int wrows = min(32, max(0, cta_rows - q * 32));
      // the row's gate, fetched while the tile's MMAs still run
      const float gs = ((MODE == 1 || MODE == 3) && lane < wrows && gate_of_row) ? __ldg(gate_of_row + wrow0 + lane)
                                                                                  : 1.f;
      const bool got = mbar_wait(bar_tfull + 8 * acc, acc_phase, abort_flag, err);
      if (!__all_sync(0xffffffffu, got)) break;
      __syncwarp();
      tc_fence_after();
      const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * BN);
      // a warp past the group's last row has nothing to read or store (warp-uniform): with
      // many small groups most of a 256-row tile is padding
      if (wrows > 0)
        epilogue_tile<MODE, OutT>(taddr, stage, lane, wrow0, wrows, tc.n_tile, F, N_out, gate_of_row, out,
                                  token_of_row, n_tokens, err, gs, c_begin, c_end);
      tc_fence_before();
      mbar_arrive_remote(map_to_rank(bar_tempty + 8 * acc, 0));
    }
  }

  __syncthreads();
  cluster_sync();                                           // no remote arrive after a CTA exits
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(kTmemCols) : "memory");
  }
}

template <int MODE, typename OutT>
moe_status launch_tc(const CUtensorMap& ma, const CUtensorMap& mb, const int32_t* offsets, int E, int K, int N_out,
                     int F, long long rows_max, const float* gate_of_row, void* out, cudaStream_t s,
                     const int32_t* token_of_row = nullptr, int n_tokens = 0,
                     const __nv_bfloat16* a_gather = nullptr) {
  static std::atomic<int> configured[kMaxDevices];
  const moe_status st = ensure_smem_limit(configured, grouped_gemm_tc_kernel<MODE, OutT>, kSmemBytes);
  if (st != MOE_OK) return st;
  const int n_tiles = n_tiles_of<MODE>(F, N_out);
  const long long max_tiles = ((rows_max + BM - 1) / BM + E) * (long long)n_tiles;
  int grid = num_sms();
  if (max_tiles < grid) grid = (int)max_tiles;
  if (grid < 1) grid = 1;
  grouped_gemm_tc_kernel<MODE, OutT><<<grid, kThreadsTC, kSmemBytes, s>>>(
      ma, mb, offsets, E, K, N_out, F, rows_max, gate_of_row, static_cast<OutT*>(out), token_of_row, n_tokens,
      a_gather, err_ptr());
  return check_launch();
}

}  // namespace

// Returns MOE_ERR_UNSUPPORTED when a tensor map cannot be encoded (caller falls back).
// CTA pairs pay off when groups average at least one full 256-row pair tile; smaller
// groups keep the single-CTA kernel (less padding in ragged groups).
// Down GEMMs with K = F up to this use the eight-epilogue-warp pair configuration.
constexpr int kWideMaxK = 512;
constexpr long long kPairRowsMin = 1024;

// Token-major tiles: CTA pairs (256 rows per tile) when the groups average at least 1024
// rows, single CTAs (128 rows) otherwise: with smaller groups most tiles are part-empty,
// and a 128-row tile wastes half the tensor work of a 256-row one (measured on the stress
// layer's down GEMM, 585 rows per expert at most and 146 on average: 1.15 ms single
// against 1.29 ms in pairs).  MOE_B200_TOKEN_TILES=pairs|single forces one.
static bool use_pairs(long long rows_max, int groups) {
  const char* v = getenv("MOE_B200_TOKEN_TILES");
  if (v && strcmp(v, "pairs") == 0) return groups > 0;
  if (v && strcmp(v, "single") == 0) return false;
  return groups > 0 && rows_max / groups >= kPairRowsMin;
}

template <int MODE, typename OutT, bool WIDE = false>
moe_status launch_tc2(const CUtensorMap& ma, const CUtensorMap& mb, const int32_t* offsets, int E, int K, int N_out,
                      int F, long long rows_max, const float* gate_of_row, void* out, cudaStream_t s,
                      const int32_t* token_of_row = nullptr, int n_tokens = 0) {
  static std::atomic<int> configured[kMaxDevices];
  const moe_status st =
      ensure_smem_limit(configured, grouped_gemm_tc2_kernel<MODE, OutT, WIDE>, PairCfg<WIDE>::smem);
  if (st != MOE_OK) return st;
  const int n_tiles = n_tiles_of<MODE>(F, N_out);
  const long long max_tiles = ((rows_max + 2 * BM - 1) / (2 * BM) + E) * (long long)n_tiles;
  int pairs = num_sms() / 2;
  if (max_tiles < pairs) pairs = (int)max_tiles;
  if (pairs < 1) pairs = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * pairs, 1, 1);
  cfg.blockDim = dim3(PairCfg<WIDE>::threads, 1, 1);
  cfg.dynamicSmemBytes = PairCfg<WIDE>::smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cuda_status(cudaLaunchKernelEx(&cfg, grouped_gemm_tc2_kernel<MODE, OutT, WIDE>, ma, mb, offsets, E, K, N_out, F,
                                        rows_max, gate_of_row, static_cast<OutT*>(out), token_of_row, n_tokens,
                                        err_ptr()));
}

// Token-major tiles (this file) pay off when the groups are large: a 256-row tile is then
// full.  When the groups average under kWeightMajorBelow rows -- many experts, or a cap
// that keeps few rows each -- skew leaves most experts with a few dozen rows, and the
// weight-major tiles (ffn_wm.cu), whose token side is the group rounded up to 32, waste
// far less tensor work.  That holds for gate/up (K = d: long mainloops).  The down GEMM
// (K = F, a few k-blocks per tile) measured faster token-major at every group size tried
// (stress workload: 1.4 against 2.0 ms), so it takes weight-major tiles only when forced.
// MOE_B200_EXPERT_TILES=tokens|weights overrides the choice for both (for measuring one
// against the other).
constexpr long long kWeightMajorBelow = 1024;

bool prefer_weight_major(long long rows_max, int E, bool down) {
  const char* v = getenv("MOE_B200_EXPERT_TILES");      // read per call: a host-side string lookup
  if (v && strcmp(v, "tokens") == 0) return false;
  if (v && strcmp(v, "weights") == 0) return true;
  return !down && E > 0 && rows_max / E < kWeightMajorBelow;
}

moe_status launch_gate_up_tc(const void* x_rows, const int32_t* offsets, int E, int d, int F, long long rows_max,
                             const void* W_gu, void* h, cudaStream_t s) {
  if (rows_max == 0) return MOE_OK;
  if (d < BK || F < 8) return MOE_ERR_UNSUPPORTED;
  if (prefer_weight_major(rows_max, E, false)) {
    const moe_status st = launch_gate_up_wm(x_rows, offsets, E, d, F, rows_max, W_gu, h, s);
    if (st != MOE_ERR_UNSUPPORTED) return st;
  }
  CUtensorMap ma, mb;
  if (!make_map(&ma, x_rows, (unsigned long long)rows_max, d, BM)) return MOE_ERR_UNSUPPORTED;
  if (!make_map(&mb, W_gu, (unsigned long long)E * 2 * F, d, 128)) return MOE_ERR_UNSUPPORTED;
  if (use_pairs(rows_max, E))
    return launch_tc2<0, __nv_bfloat16>(ma, mb, offsets, E, d, F, F, rows_max, nullptr, h, s);
  return launch_tc<0, __nv_bfloat16>(ma, mb, offsets, E, d, F, F, rows_max, nullptr, h, s);
}

moe_status launch_down_tc(const void* h, const int32_t* offsets, int E, int d, int F, long long rows_max,
                          const void* W_dn, const float* gate_of_row, int y_dtype, void* y_rows, cudaStream_t s) {
  if (rows_max == 0) return MOE_OK;
  if (F < BK || d < 8) return MOE_ERR_UNSUPPORTED;
  if (prefer_weight_major(rows_max, E, true)) {
    const moe_status st = launch_down_wm(h, offsets, E, d, F, rows_max, W_dn, gate_of_row, y_dtype, y_rows, s);
    if (st != MOE_ERR_UNSUPPORTED) return st;
  }
  const bool pair = use_pairs(rows_max, E);
  CUtensorMap ma, mb;
  if (!make_map(&ma, h, (unsigned long long)rows_max, F, BM)) return MOE_ERR_UNSUPPORTED;
  if (!make_map(&mb, W_dn, (unsigned long long)E * d, F, pair ? BM : BN)) return MOE_ERR_UNSUPPORTED;
  if (pair) {
    if (F <= kWideMaxK) {
      if (y_dtype == MOE_F32)
        return launch_tc2<1, float, true>(ma, mb, offsets, E, F, d, F, rows_max, gate_of_row, y_rows, s);
      return launch_tc2<1, __nv_bfloat16, true>(ma, mb, offsets, E, F, d, F, rows_max, gate_of_row, y_rows, s);
    }
    if (y_dtype == MOE_F32)
      return launch_tc2<1, float>(ma, mb, offsets, E, F, d, F, rows_max, gate_of_row, y_rows, s);
    return launch_tc2<1, __nv_bfloat16>(ma, mb, offsets, E, F, d, F, rows_max, gate_of_row, y_rows, s);
  }
  if (y_dtype == MOE_F32)
    return launch_tc<1, float>(ma, mb, offsets, E, F, d, F, rows_max, gate_of_row, y_rows, s);
  return launch_tc<1, __nv_bfloat16>(ma, mb, offsets, E, F, d, F, rows_max, gate_of_row, y_rows, s);
}

// Down GEMM with the combine fused into its epilogue: y[token_of_row[r]] += gate_of_row[r] *
// (H[r] W_dn[e]^T), y fp32 [T, d] already initialised by the caller.
moe_status launch_down_combine_tc(const void* h, const int32_t* offsets, int E, int d, int F, long long rows_max,
                                  const void* W_dn, const float* gate_of_row, const int32_t* token_of_row, int T,
                                  float* y, cudaStream_t s) {
  if (rows_max == 0 || T == 0) return MOE_OK;
  if (F < BK || d < 8) return MOE_ERR_UNSUPPORTED;
  const bool pair = use_pairs(rows_max, E);
  CUtensorMap ma, mb;
  if (!make_map(&ma, h, (unsigned long long)rows_max, F, BM)) return MOE_ERR_UNSUPPORTED;
  if (!make_map(&mb, W_dn, (unsigned long long)E * d, F, pair ? BM : BN)) return MOE_ERR_UNSUPPORTED;
  if (pair && F <= kWideMaxK)
    return launch_tc2<3, float, true>(ma, mb, offsets, E, F, d, F, rows_max, gate_of_row, y, s, token_of_row, T);
  if (pair) return launch_tc2<3, float>(ma, mb, offsets, E, F, d, F, rows_max, gate_of_row, y, s, token_of_row, T);
  return launch_tc<3, float>(ma, mb, offsets, E, F, d, F, rows_max, gate_of_row, y, s, token_of_row, T);
}

// Gate/up GEMM with the dispatch fused into its producer: A row r = x[token_of_row[r]]
// (x [T, d] bf16), no permuted copy of x.  Single-CTA tiles (the gather producer fills
// one CTA's stages).
moe_status launch_gate_up_gather_tc(const void* x, const int32_t* token_of_row, int T, const int32_t* offsets, int E,
                                    int d, int F, long long rows_max, const void* W_gu, void* h, cudaStream_t s) {
  if (rows_max == 0 || T == 0) return MOE_OK;
  if (d < BK || F < 8) return MOE_ERR_UNSUPPORTED;
  if (prefer_weight_major(rows_max, E, false)) {
    const moe_status st = launch_gate_up_wm_gather(x, token_of_row, T, offsets, E, d, F, rows_max, W_gu, h, s);
    if (st != MOE_ERR_UNSUPPORTED) return st;
  }
  CUtensorMap mb;
  if (!make_map(&mb, W_gu, (unsigned long long)E * 2 * F, d, 128)) return MOE_ERR_UNSUPPORTED;
  return launch_tc<4, __nv_bfloat16>(mb, mb, offsets, E, d, F, F, rows_max, nullptr, h, s, token_of_row, T,
                                     static_cast<const __nv_bfloat16*>(x));
}

}  // namespace moe
