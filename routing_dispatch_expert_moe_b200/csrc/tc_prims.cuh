// tcgen05 / TMA / mbarrier primitives shared by the tensor-core kernels (sm_100a):
// shared-memory descriptors for the 128-byte-swizzled K-major operands TMA writes, the
// instruction descriptor of kind::f16 MMAs, bounded mbarrier waits, single-CTA and
// CTA-pair (cta_group::2) MMA issue and commit, TMEM loads, the epilogue's shared-memory
// turn-around for coalesced stores, and the host-side tensor-map encoder.
// No load anywhere uses cluster multicast.
#pragma once

#include <cuda.h>

#include "common.cuh"

namespace moe {
namespace {

constexpr int BK = 64, UMMA_K = 16;                            // k-block (one 128-byte row), MMA K
constexpr unsigned long long kWaitLimitNs = 2000000000ull;   // 2 s per barrier wait

// instruction descriptor: D fp32, A bf16, B bf16, both K-major, N = n, M = m
constexpr uint32_t make_idesc(int m, int n) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(m >> 4) << 24);
}
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait.  Returns false when the limit passes (records the error, raises the
// CTA's abort flag) or when another role has already aborted.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag, int* err) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 63u) == 0u) {
      if (*abort_flag) return false;
      if (global_timer_ns() - t0 > kWaitLimitNs) {
        record_error(err, MOE_DEVERR_PIPE_TIMEOUT);
        *abort_flag = 1;
        return false;
      }
    }
  }
}
// Bounded wait that ignores the abort flag (used to drain in-flight work on exit).
__device__ __forceinline__ void mbar_wait_drain(uint32_t bar, uint32_t parity, int* err) {
  const uint64_t t0 = global_timer_ns();
  for (uint32_t i = 0;; ++i) {
    if (mbar_try_wait(bar, parity)) return;
    if ((i & 63u) == 63u && global_timer_ns() - t0 > kWaitLimitNs) {
      record_error(err, MOE_DEVERR_PIPE_TIMEOUT);
      return;
    }
  }
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, uint32_t bar, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
      : "memory");
}

// Orders generic-proxy shared-memory writes this thread has made or observed (stores, or
// other threads' cp.async copies acquired through an mbarrier) before later async-proxy
// accesses (the tensor cores read operands through the async proxy).
__device__ __forceinline__ void fence_proxy_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void umma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}

// ---- CTA-pair (cta_group::2) forms: an M=256 MMA issued by the pair's even CTA over
// both CTAs' shared memory, accumulating into both CTAs' TMEM ----

__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// The same shared-memory object in CTA `rank` of the cluster (shared::cluster address).
__device__ __forceinline__ uint32_t map_to_rank(uint32_t saddr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
  return r;
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release;\n\tbarrier.cluster.wait.acquire;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
// Arrive on a barrier that may live in the peer CTA, releasing at CTA scope only.  The
// accumulator-free signal of an epilogue needs no ordering of the thread's global stores
// (only its TMEM reads, which tcgen05.wait::ld and tcgen05.fence::before_thread_sync
// order); a cluster-scope release would make every epilogue thread wait until all of its
// earlier global stores are visible cluster-wide, once per tile.
__device__ __forceinline__ void mbar_arrive_remote(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
// TMA load into this CTA's shared memory whose completion is counted on an mbarrier that
// may live in the peer CTA (the pair's even CTA); no multicast.
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap* map, uint32_t bar_cluster, int x,
                                                 int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], "
      "[%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar_cluster)
      : "memory");
}
// 16-byte cp.async global -> shared; src_bytes = 0 writes zeros without reading.
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
// Arrive on the mbarrier once all of this thread's earlier cp.async copies have landed
// (the barrier's expected count includes this arrival: .noinc).
__device__ __forceinline__ void cp_async_arrive_noinc(uint32_t bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }
// TMA row gather (tile::gather4) of a CTA pair: rows y0..y3 of a 2D tensor map whose box
// is 64 columns x 1 row, columns x .. x+63, land as four consecutive 128-byte rows at dst
// in this CTA's shared memory, swizzled as a tiled load of the same map would place them
// (dst 512-byte aligned); completion is counted on the pair's even-CTA barrier.
// Coordinates must lie inside the tensor.  No multicast.
__device__ __forceinline__ void tma_gather4_pair(uint32_t dst, const CUtensorMap* map, uint32_t bar_cluster, int x,
                                                 int y0, int y1, int y2, int y3) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.tile::gather4.mbarrier::complete_tx::bytes "
      "[%0], [%1, {%2, %3, %4, %5, %6}], [%7];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y0), "r"(y1), "r"(y2), "r"(y3), "r"(bar_cluster)
      : "memory");
}
__device__ __forceinline__ void umma_bf16_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                               uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Completion of the pair's MMAs arrives on the barrier at this offset in both CTAs.
__device__ __forceinline__ void umma_commit_pair_both(uint32_t bar) {
  const uint16_t both = 0x3;
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;"
               ::"r"(bar), "h"(both)
               : "memory");
}
__device__ __forceinline__ void umma_commit_pair(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}

// K-major operand in the canonical 128-byte-swizzle layout written by TMA:
// rows of 128 bytes (64 bf16), 8-row atoms of 1024 bytes stacked densely.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
  uint64_t d = (uint64_t)((saddr >> 4) & 0x3FFFu);   // start address >> 4
  d |= (uint64_t)1 << 16;                            // leading byte offset (unused when swizzled)
  d |= (uint64_t)(1024 >> 4) << 32;                  // stride byte offset: one 8-row atom
  d |= (uint64_t)1 << 46;                            // descriptor version for sm_100
  d |= (uint64_t)2 << 61;                            // 128-byte swizzle
  return d;
}

#define MOE_R32(r) \
  "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), \
  "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), \
  "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), \
  "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
#define MOE_RW32(r) \
  "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]), \
  "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15]), \
  "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]), "+r"(r[22]), "+r"(r[23]), \
  "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]), "+r"(r[29]), "+r"(r[30]), "+r"(r[31])

// 32 consecutive fp32 accumulator columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : MOE_R32(r)
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
// Ties the loaded registers to the preceding wait so no use is scheduled above it.
__device__ __forceinline__ void tmem_regs_ready(uint32_t (&r)[32]) { asm volatile("" : MOE_RW32(r)); }

// Epilogue staging: each epilogue warp turns its 32 rows x 32 columns (one value per
// lane-row from tcgen05.ld) around in shared memory, so that every global store
// instruction writes whole 128-byte lines of 4 (fp32) or 8 (bf16) rows instead of 32
// half-filled sectors.  Row pitch padded by 16 bytes: conflict-free 16-byte accesses.
constexpr int kStagePitchF32 = 32 * 4 + 16;
constexpr int kStagePitchB16 = 32 * 2 + 16;
constexpr int kStageWarpBytes = 32 * kStagePitchF32;

template <typename OutT>
__device__ __forceinline__ void stage_store32(uint8_t* stage, const float (&v)[32], int lane, OutT* out,
                                              long long row0, int rows_valid, long long ld, int col, int ncols) {
  if constexpr (sizeof(OutT) == 4) {
    float4* dst = reinterpret_cast<float4*>(stage + lane * kStagePitchF32);
#pragma unroll
    for (int q = 0; q < 8; ++q) dst[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
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
    uint4* dst = reinterpret_cast<uint4*>(stage + lane * kStagePitchB16);
#pragma unroll
    for (int q = 0; q < 4; ++q)
      dst[q] = make_uint4(pack_bf16x2(v[8 * q], v[8 * q + 1]), pack_bf16x2(v[8 * q + 2], v[8 * q + 3]),
                          pack_bf16x2(v[8 * q + 4], v[8 * q + 5]), pack_bf16x2(v[8 * q + 6], v[8 * q + 7]));
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

}  // namespace

namespace {
// ---------------------------------------------------------------- host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn lookup_encode_fn() {
  void* p = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
      q == cudaDriverEntryPointSuccess)
    return reinterpret_cast<EncodeTiledFn>(p);
  return nullptr;
}

// Looked up once (a function-local static: initialised once even with several host threads).
EncodeTiledFn encode_fn() {
  static const EncodeTiledFn fn = lookup_encode_fn();
  return fn;
}

// 2D bf16 tensor [rows, cols] row-major; box = box_rows x 64 columns, 128-byte swizzle.
bool make_map(CUtensorMap* m, const void* ptr, unsigned long long rows, unsigned long long cols, unsigned box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
  cuuint32_t box[2] = {(cuuint32_t)BK, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2D byte tensor [rows, cols] row-major (no swizzle); box = box_cols bytes x box_rows.
bool make_map_u8(CUtensorMap* m, const void* ptr, unsigned long long rows, unsigned long long cols, unsigned box_cols,
                 unsigned box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)cols};
  cuuint32_t box[2] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(ptr), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace
}  // namespace moe
