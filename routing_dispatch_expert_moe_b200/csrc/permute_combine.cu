// Dispatch (permute) and combine.
//
// Sources: "Hugging Face 图解 Mixture of Experts（MoE）原理、训练与推理权衡", section
// "什么是稀疏性？", eq. y = sum_i G(x)_i E_i(x); handbook news post (hub.geekagi.cn),
// "MoE 到底省了什么" (the router sends each token to a few experts and merges their
// outputs) and item 3 (tokens dispatched and results gathered back every layer);
// handbook article (zicq.com), "MoE 的核心机制" (dispatch and aggregation are the real
// bottleneck).
//
// Both kernels are pure data movement, bound by HBM bandwidth: one warp per token,
// each lane moves 16-byte vectors so a warp instruction covers 512 contiguous bytes of
// the hidden dimension.
//   permute: x[t] is read once and written to each of its kept rows (k stores per load).
//   combine: all k rows of a token are loaded before any is added (k independent loads in
//            flight per lane), summed in fp32 in slot order, then the shared-expert row,
//            then rounded to nearest even.
#include "common.cuh"

namespace moe {
namespace {

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
    for (int v0 = lane; v0 < nvec; v0 += 32 * UNROLL) {
      uint4 buf[UNROLL];
#pragma unroll
      for (int u = 0; u < UNROLL; ++u) {
        const int v = v0 + 32 * u;
        if (v < nvec) buf[u] = ld_stream(src + v);
      }
      for (int j = 0; j < k; ++j) {
        const int r = __shfl_sync(0xffffffffu, my_row, j);
        if (r < 0) continue;
        uint4* dst = x_perm + (long long)r * nvec;
#pragma unroll
        for (int u = 0; u < UNROLL; ++u) {
          const int v = v0 + 32 * u;
          if (v < nvec) dst[v] = buf[u];
        }
      }
    }
  }
}

template <typename T>
struct Vec;
template <>
struct Vec<__nv_bfloat16> {
  static constexpr int N = 8;
  __device__ static void unpack(const uint4& v, float* f) { unpack8(v, f); }
  __device__ static uint4 pack(const float* f) { return pack8(f); }
};
template <>
struct Vec<float> {
  static constexpr int N = 4;
  __device__ static void unpack(const uint4& v, float* f) {
    f[0] = __uint_as_float(v.x); f[1] = __uint_as_float(v.y);
    f[2] = __uint_as_float(v.z); f[3] = __uint_as_float(v.w);
  }
  __device__ static uint4 pack(const float* f) {
    return make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]),
                      __float_as_uint(f[3]));
  }
};

// KMAX: compile-time bound on k (all k rows of a token are held in registers).
template <typename DT, int KMAX>
__global__ void __launch_bounds__(256)
combine_kernel(const uint4* __restrict__ y_rows, const int32_t* __restrict__ row_of,
               const float* __restrict__ topk_gate, const uint4* __restrict__ shared_y, int T,
               int nvec, int k, long long rows_max, uint4* __restrict__ y, int* err) {
  constexpr int N = Vec<DT>::N;
  const unsigned lane = threadIdx.x & 31;
  const int warps = blockDim.x >> 5;
  const long long nw = (long long)gridDim.x * warps;
  for (long long t = (long long)blockIdx.x * warps + (threadIdx.x >> 5); t < T; t += nw) {
    int my_row = -1;
    float my_gate = 1.f;
    if (lane < (unsigned)k) {
      my_row = __ldg(row_of + t * k + lane);
      if (my_row >= rows_max) { record_error(err, MOE_DEVERR_ROW); my_row = -1; }
      if (my_row < -1) my_row = -1;
      if (topk_gate) my_gate = __ldg(topk_gate + t * k + lane);
    }
    int rows[KMAX];
    float gates[KMAX];
#pragma unroll
    for (int j = 0; j < KMAX; ++j) {
      rows[j] = __shfl_sync(0xffffffffu, my_row, j);
      gates[j] = __shfl_sync(0xffffffffu, my_gate, j);
    }
    for (int v = lane; v < nvec; v += 32) {
      uint4 buf[KMAX];
#pragma unroll
      for (int j = 0; j < KMAX; ++j)
        if (j < k && rows[j] >= 0) buf[j] = ld_stream(y_rows + (long long)rows[j] * nvec + v);
      uint4 sv;
      if (shared_y) sv = ld_stream(shared_y + t * nvec + v);
      float acc[N];
#pragma unroll
      for (int i = 0; i < N; ++i) acc[i] = 0.f;
#pragma unroll
      for (int j = 0; j < KMAX; ++j) {
        if (j < k && rows[j] >= 0) {
          float f[N];
          Vec<DT>::unpack(buf[j], f);
          if (topk_gate) {
#pragma unroll
            for (int i = 0; i < N; ++i) acc[i] = fmaf(gates[j], f[i], acc[i]);
          } else {
#pragma unroll
            for (int i = 0; i < N; ++i) acc[i] += f[i];
          }
        }
      }
      if (shared_y) {
        float f[N];
        Vec<DT>::unpack(sv, f);
#pragma unroll
        for (int i = 0; i < N; ++i) acc[i] += f[i];
      }
      y[t * nvec + v] = Vec<DT>::pack(acc);
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

template <typename DT, int KMAX>
moe_status run_combine(const void* y_rows, const int32_t* row_of, const float* topk_gate,
                       const void* shared_y, int T, int nvec, int k, long long rows_max, void* y,
                       cudaStream_t s) {
  combine_kernel<DT, KMAX><<<grid_for_warps(T), 256, 0, s>>>(
      static_cast<const uint4*>(y_rows), row_of, topk_gate, static_cast<const uint4*>(shared_y), T, nvec, k,
      rows_max, static_cast<uint4*>(y), err_ptr());
  return check_launch();
}

template <typename DT>
moe_status combine_k(const void* y_rows, const int32_t* row_of, const float* topk_gate,
                     const void* shared_y, int T, int nvec, int k, long long rows_max, void* y,
                     cudaStream_t s) {
  if (k <= 1) return run_combine<DT, 1>(y_rows, row_of, topk_gate, shared_y, T, nvec, k, rows_max, y, s);
  if (k <= 2) return run_combine<DT, 2>(y_rows, row_of, topk_gate, shared_y, T, nvec, k, rows_max, y, s);
  if (k <= 4) return run_combine<DT, 4>(y_rows, row_of, topk_gate, shared_y, T, nvec, k, rows_max, y, s);
  if (k <= 8) return run_combine<DT, 8>(y_rows, row_of, topk_gate, shared_y, T, nvec, k, rows_max, y, s);
  if (k <= 16) return run_combine<DT, 16>(y_rows, row_of, topk_gate, shared_y, T, nvec, k, rows_max, y, s);
  return run_combine<DT, 32>(y_rows, row_of, topk_gate, shared_y, T, nvec, k, rows_max, y, s);
}

}  // namespace

moe_status launch_permute(const void* x, int dtype, int T, int d, int k, const int32_t* row_of,
                          long long rows_max, void* x_perm, cudaStream_t s) {
  if (T == 0) return MOE_OK;
  const int esz = dtype == MOE_F32 ? 4 : 2;
  const int nvec = d * esz / 16;
  permute_kernel<4><<<grid_for_warps(T), 256, 0, s>>>(static_cast<const uint4*>(x), T, nvec, k, row_of,
                                                      rows_max, static_cast<uint4*>(x_perm), err_ptr());
  return check_launch();
}

moe_status launch_combine(const void* y_rows, const int32_t* row_of, const float* topk_gate,
                          const void* shared_y, int dtype, int T, int d, int k, long long rows_max,
                          void* y, cudaStream_t s) {
  if (T == 0) return MOE_OK;
  const int esz = dtype == MOE_F32 ? 4 : 2;
  const int nvec = d * esz / 16;
  if (dtype == MOE_F32) return combine_k<float>(y_rows, row_of, topk_gate, shared_y, T, nvec, k, rows_max, y, s);
  return combine_k<__nv_bfloat16>(y_rows, row_of, topk_gate, shared_y, T, nvec, k, rows_max, y, s);
}

}  // namespace moe
