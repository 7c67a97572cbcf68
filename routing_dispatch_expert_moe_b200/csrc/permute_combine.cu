// Dispatch (permute) and combine.
//
// Sources: "Hugging Face 图解 Mixture of Experts（MoE）原理、训练与推理权衡", section
// "什么是稀疏性？", eq. y = sum_i G(x)_i E_i(x); handbook news post (hub.geekagi.cn),
// "MoE 到底省了什么" (the router sends each token to a few experts and merges their
// outputs) and item 3 (tokens dispatched and results gathered back every layer);
// handbook article (zicq.com), "MoE 的核心机制" (dispatch and aggregation are the real
// bottleneck).
//
// Both kernels are pure data movement, bound by HBM bandwidth, one warp per token.
//   permute: x[t] is read once and written to each of its kept rows, by bulk copies
//            through shared memory (or, for rows too long for the buffers, 16-byte vectors
//            from registers, a warp instruction covering 512 contiguous bytes).
//   combine: all k rows of a token are loaded before any is added (k independent loads in
//            flight per lane), summed in fp32 in slot order, then the shared-expert row,
//            then rounded to nearest even.
#include "common.cuh"
#include "row8.cuh"
#include "tc_prims.cuh"

namespace moe {
namespace {

// Permute by bulk copies.  A warp takes the tokens t0, t0 + nw, ...: lane 0 brings token
// t's row into a shared-memory buffer with one bulk copy (global -> shared, completing on
// the buffer's mbarrier), then lanes 0..k-1 each write it to one kept row of x_perm with
// one bulk copy back (shared -> global).  Three buffers per warp: the load of the token
// two ahead is issued once the stores of the token before have read their buffer (their
// writes may still be in flight), so a warp keeps two loads and the latest stores in
// flight without the SM issuing any per-vector loads or stores.  Row bytes a multiple of
// 16.  Every wait is bounded; on a timeout the warp stops and drains what it issued.
// Four warps with three buffers each, two loads issued ahead (4 x 3 with one ahead and
// 6 x 2 measured within 2% of it; this one was ahead of the per-vector copy on both the
// 7168- and the 2048-wide rows).
constexpr int kPermWarps = 4, kPermBufs = 3, kPermDepth = 2;   // depth: loads issued ahead
constexpr int kPermHead = (8 * kPermBufs * kPermWarps + 4 + 127) / 128 * 128;  // mbarriers + abort flag
static_assert(kPermDepth >= 1 && kPermDepth < kPermBufs, "a buffer is reloaded only after its stores have read it");

__device__ __forceinline__ void bulk_load_row(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "l"(src), "r"(bytes), "r"(bar)
               : "memory");
}
__device__ __forceinline__ void bulk_store_row(void* dst, uint32_t src, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst), "r"(src), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

__global__ void __launch_bounds__(32 * kPermWarps)
permute_bulk_kernel(const uint8_t* __restrict__ x, int T, int row_bytes, int row_pitch, int k,
                    const int32_t* __restrict__ row_of, long long rows_max, uint8_t* __restrict__ x_perm, int* err) {
  extern __shared__ __align__(128) uint8_t psm[];
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const uint32_t bar0 = smem_u32(psm) + (uint32_t)(8 * kPermBufs * w);
  const uint32_t buf0 = smem_u32(psm) + (uint32_t)kPermHead + (uint32_t)(row_pitch * kPermBufs * w);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(psm + 8 * kPermBufs * kPermWarps);
  if (threadIdx.x == 0) *abort_flag = 0;
  if (lane == 0) {
    for (int b = 0; b < kPermBufs; ++b) mbar_init(bar0 + 8 * b, 1);
    fence_mbar_init();
  }
  __syncthreads();
  const long long nw = (long long)gridDim.x * kPermWarps;
  const long long t0 = (long long)blockIdx.x * kPermWarps + w;
  const long long n_iter = t0 < T ? (T - t0 + nw - 1) / nw : 0;
  int issued = 0;                                         // loads issued (iterations 0 .. issued - 1)
  auto issue_load = [&](long long i) {
    if (i < n_iter) {
      if (lane == 0) {
        const uint32_t b = (uint32_t)(i % kPermBufs);
        mbar_expect_tx(bar0 + 8 * b, (uint32_t)row_bytes);
        bulk_load_row(buf0 + b * (uint32_t)row_pitch, x + (t0 + i * nw) * row_bytes, (uint32_t)row_bytes, bar0 + 8 * b);
      }
      issued = (int)i + 1;
    }
  };
  for (int j = 0; j < kPermDepth; ++j) issue_load(j);
  long long i = 0;
  for (; i < n_iter; ++i) {
    const long long t = t0 + i * nw;
    const uint32_t b = (uint32_t)(i % kPermBufs);
    int r = -1;
    if (lane < k) {
      r = __ldg(row_of + t * k + lane);
      if (r >= rows_max) { record_error(err, MOE_DEVERR_ROW); r = -1; }
    }
    const bool got = mbar_wait(bar0 + 8 * b, (uint32_t)((i / kPermBufs) & 1), abort_flag, err);
    if (!__all_sync(0xffffffffu, got)) break;
    if (r >= 0) bulk_store_row(x_perm + (long long)r * row_bytes, buf0 + b * (uint32_t)row_pitch, (uint32_t)row_bytes);
    bulk_commit();                                        // every lane: an empty group where it stored nothing
    bulk_wait_read<kPermBufs - kPermDepth>();             // the stores of token i + depth - bufs have read their buffer
    __syncwarp();
    issue_load(i + kPermDepth);                           // into that buffer
  }
  bulk_wait_all();                                        // the stores are done before the CTA exits
  if (lane == 0)                                          // after a timeout: let every issued load land
    for (long long j = i; j < issued; ++j)
      mbar_wait_drain(bar0 + 8 * (uint32_t)(j % kPermBufs), (uint32_t)((j / kPermBufs) & 1), err);
}

template <int UNROLL>
__global__ void __launch_bounds__(256)
permute_kernel(const uint4* __restrict__ x, int T, int nvec, int k, const int32_t* __restrict__ row_of,
               long long rows_max, uint4* __restrict__ x_perm, int* err) {
  const unsigned lane = threadIdx.x & 31;
  const int warps = blockDim.x >> 5;
  const long long nw = (long long)gridDim.x * warps;
  for (long long t = (long long)blockIdx.x * warps + (threadIdx.x >> 5); t < T; t += nw) {
    int my_row = -1;
    if (lane < (unsigned)k) {
      my_row = __ldg(row_of + t * k + lane);
      if (my_row >= rows_max) { record_error(err, MOE_DEVERR_ROW); my_row = -1; }
      if (my_row < -1) my_row = -1;
    }
    const uint4* src = x + t * nvec;
    // warp-uniform trip count: every lane reaches each shuffle below, also when a row has
    // fewer than 32 vectors (lanes past the row's end only skip their loads and stores)
    for (int base = 0; base < nvec; base += 32 * UNROLL) {
      uint4 buf[UNROLL];
#pragma unroll
      for (int u = 0; u < UNROLL; ++u) {
        const int v = base + (int)lane + 32 * u;
        if (v < nvec) buf[u] = ld_stream(src + v);
      }
      for (int j = 0; j < k; ++j) {
        const int r = __shfl_sync(0xffffffffu, my_row, j);
        if (r < 0) continue;
        uint4* dst = x_perm + (long long)r * nvec;
#pragma unroll
        for (int u = 0; u < UNROLL; ++u) {
          const int v = base + (int)lane + 32 * u;
          if (v < nvec) dst[v] = buf[u];
        }
      }
    }
  }
}

// KMAX: compile-time bound on k (multiple of 8).  The token's kept slots are first
// compacted, in slot order, into a per-warp list in shared memory (a ballot gives each
// kept slot its position), so dropped slots cost nothing, every batch of loads is full,
// and the list costs no registers (two blocks fit on an SM).  Each lane then loads R kept
// rows for VPI 8-element vectors (16 independent 16-byte loads in flight for bf16 rows)
// and adds them in slot order: the same fp32 sum as visiting every slot.
template <typename InT, typename OutT, int KMAX>
__global__ void __launch_bounds__(256, 2)
combine_kernel(const void* __restrict__ y_rows, const int32_t* __restrict__ row_of,
               const float* __restrict__ topk_gate, const void* __restrict__ shared_y, int T, int d, int k,
               long long rows_max, void* __restrict__ y, int* err) {
  // kept rows per batch x vectors per lane: 16 loads in flight either way; k <= 8 keeps
  // one batch for a token that keeps all its slots, larger k (where capacity drops most
  // slots) four rows so that a token keeping four still fills the batch
  constexpr int R = KMAX <= 8 ? 8 : 4;
  constexpr int VPI = (sizeof(InT) == 2 ? 16 : 8) / R;
  __shared__ int s_row[8][32];
  __shared__ float s_gate[8][32];
  const unsigned lane = threadIdx.x & 31;
  const int wib = threadIdx.x >> 5;
  const int warps = blockDim.x >> 5;
  const long long nw = (long long)gridDim.x * warps;
  const bool scale = topk_gate != nullptr;
  const int n8 = d >> 3;
  int* krow = s_row[wib];
  float* kgate = s_gate[wib];
  for (long long t = (long long)blockIdx.x * warps + wib; t < T; t += nw) {
    int my_row = -1;
    float my_gate = 1.f;
    if (lane < (unsigned)k) {
      my_row = __ldg(row_of + t * k + lane);
      if (my_row >= rows_max) { record_error(err, MOE_DEVERR_ROW); my_row = -1; }
      if (my_row < -1) my_row = -1;
      if (scale) my_gate = __ldg(topk_gate + t * k + lane);
    }
    // kept slots in slot order -> positions 0 .. nk-1
    const unsigned kept = __ballot_sync(0xffffffffu, my_row >= 0);
    const int nk = __popc(kept);
    __syncwarp();                                       // the previous token's list is read
    if (my_row >= 0) {
      const int pos = __popc(kept & ((1u << lane) - 1u));
      krow[pos] = my_row;
      kgate[pos] = my_gate;
    }
    __syncwarp();
    for (int v0 = lane; v0 < n8; v0 += 32 * VPI) {
      float acc[VPI][8];
#pragma unroll
      for (int u = 0; u < VPI; ++u)
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[u][i] = 0.f;
#pragma unroll 1
      for (int j0 = 0; j0 < KMAX; j0 += R) {
        if (j0 >= nk) break;
        Row8<InT> buf[VPI][R];
#pragma unroll
        for (int jj = 0; jj < R; ++jj)
#pragma unroll
          for (int u = 0; u < VPI; ++u)
            if (j0 + jj < nk && v0 + 32 * u < n8)
              buf[u][jj].load(y_rows, (long long)krow[j0 + jj] * d + (v0 + 32 * u) * 8);
#pragma unroll
        for (int jj = 0; jj < R; ++jj)
#pragma unroll
          for (int u = 0; u < VPI; ++u)
            if (j0 + jj < nk && v0 + 32 * u < n8) buf[u][jj].add(acc[u], kgate[j0 + jj], scale);
      }
#pragma unroll
      for (int u = 0; u < VPI; ++u) {
        const int v = v0 + 32 * u;
        if (v >= n8) continue;
        if (shared_y) {
          Row8<InT> sv;
          sv.load(shared_y, t * d + v * 8);
          sv.add(acc[u], 1.f, false);
        }
        store8<OutT>(y, t * d + v * 8, acc[u]);
      }
    }
  }
}

unsigned grid_for_warps(long long warps_needed) {
  long long blocks = (warps_needed + 7) / 8;
  const long long cap = (long long)num_sms() * 8;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  return (unsigned)blocks;
}

template <typename InT, typename OutT, int KMAX>
moe_status run_combine(const void* y_rows, const int32_t* row_of, const float* topk_gate, const void* shared_y,
                       int T, int d, int k, long long rows_max, void* y, cudaStream_t s) {
  combine_kernel<InT, OutT, KMAX><<<grid_for_warps(T), 256, 0, s>>>(y_rows, row_of, topk_gate, shared_y, T, d, k,
                                                                   rows_max, y, err_ptr());
  return check_launch();
}

template <typename InT, typename OutT>
moe_status combine_k(const void* y_rows, const int32_t* row_of, const float* topk_gate, const void* shared_y,
                     int T, int d, int k, long long rows_max, void* y, cudaStream_t s) {
  if (k <= 8) return run_combine<InT, OutT, 8>(y_rows, row_of, topk_gate, shared_y, T, d, k, rows_max, y, s);
  if (k <= 16) return run_combine<InT, OutT, 16>(y_rows, row_of, topk_gate, shared_y, T, d, k, rows_max, y, s);
  return run_combine<InT, OutT, 32>(y_rows, row_of, topk_gate, shared_y, T, d, k, rows_max, y, s);
}

// Final rounding of the combine: out[i] = bf16_rne(in[i]); with clear, in[i] = 0 after
// it is read (so an accumulation buffer is ready for the next sum without a separate
// fill).  Eight values per thread and step (two 16-byte loads, one 16-byte store),
// grid-stride; a scalar tail for n % 8.
__global__ void __launch_bounds__(256)
round_bf16_kernel(float* __restrict__ in, long long n, __nv_bfloat16* __restrict__ out, int clear) {
  const long long n8 = n / 8;
  const long long stride = (long long)gridDim.x * blockDim.x;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n8; i += stride) {
    float4* p = reinterpret_cast<float4*>(in) + 2 * i;
    const float4 a = p[0];
    const float4 b = p[1];
    const float f[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
    reinterpret_cast<uint4*>(out)[i] = pack8(f);
    if (clear) p[0] = p[1] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
  for (long long i = 8 * n8 + (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride) {
    out[i] = __float2bfloat16_rn(in[i]);
    if (clear) in[i] = 0.f;
  }
}

}  // namespace

moe_status launch_permute(const void* x, int dtype, int T, int d, int k, const int32_t* row_of,
                          long long rows_max, void* x_perm, cudaStream_t s) {
  if (T == 0) return MOE_OK;
  const int esz = dtype == MOE_F32 ? 4 : 2;
  const int row_bytes = d * esz;                         // a multiple of 16 (d % 8 == 0)
  const int row_pitch = (row_bytes + 127) / 128 * 128;
  const size_t smem = kPermHead + (size_t)kPermWarps * kPermBufs * row_pitch;
  if (smem <= 232448) {
    static std::atomic<int> configured[kMaxDevices];   // the limit once, at the largest size a launch may ask
    const moe_status st = ensure_smem_limit(configured, permute_bulk_kernel, 232448);
    if (st != MOE_OK) return st;
    const int per_sm = (int)(232448 / (smem + 1024));
    const long long ctas = (T + kPermWarps - 1) / kPermWarps;
    const long long cap = (long long)num_sms() * (per_sm < 1 ? 1 : per_sm);
    permute_bulk_kernel<<<(unsigned)(ctas < cap ? ctas : cap), 32 * kPermWarps, smem, s>>>(
        static_cast<const uint8_t*>(x), T, row_bytes, row_pitch, k, row_of, rows_max,
        static_cast<uint8_t*>(x_perm), err_ptr());
    return check_launch();
  }
  const int nvec = row_bytes / 16;                       // rows too long for the buffers
  permute_kernel<4><<<grid_for_warps(T), 256, 0, s>>>(static_cast<const uint4*>(x), T, nvec, k, row_of,
                                                      rows_max, static_cast<uint4*>(x_perm), err_ptr());
  return check_launch();
}

moe_status launch_combine(const void* y_rows, int rows_dtype, const int32_t* row_of, const float* topk_gate,
                          const void* shared_y, int T, int d, int k, long long rows_max, int y_dtype,
                          void* y, cudaStream_t s) {
  if (T == 0) return MOE_OK;
  const bool in32 = rows_dtype == MOE_F32, out32 = y_dtype == MOE_F32;
  if (in32 && out32) return combine_k<float, float>(y_rows, row_of, topk_gate, shared_y, T, d, k, rows_max, y, s);
  if (in32) return combine_k<float, __nv_bfloat16>(y_rows, row_of, topk_gate, shared_y, T, d, k, rows_max, y, s);
  if (out32) return combine_k<__nv_bfloat16, float>(y_rows, row_of, topk_gate, shared_y, T, d, k, rows_max, y, s);
  return combine_k<__nv_bfloat16, __nv_bfloat16>(y_rows, row_of, topk_gate, shared_y, T, d, k, rows_max, y, s);
}

moe_status launch_round_bf16(float* in, long long n, void* out, int clear, cudaStream_t s) {
  if (n == 0) return MOE_OK;
  long long blocks = (n / 8 + 255) / 256;
  const long long cap = 8LL * num_sms();
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  round_bf16_kernel<<<(unsigned)blocks, 256, 0, s>>>(in, n, static_cast<__nv_bfloat16*>(out), clear);
  return check_launch();
}

}  // namespace moe
