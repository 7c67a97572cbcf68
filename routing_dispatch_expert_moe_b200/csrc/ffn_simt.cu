// Grouped SwiGLU expert FFN on the fp32 SIMT pipe.
//
// Used for fp32 activations (the tensor-core kinds take no fp32 operands) and as an
// independent second implementation of the bf16 path.  Same contract as the tcgen05
// kernels: expert e owns rows [offsets[e], offsets[e+1]); W_gu[e] holds W_gate in rows
// 0..F-1 and W_up in rows F..2F-1; W_dn[e] is [d, F].
//   gate_up: H[r, f] = silu(sum_c X[r,c] Wg[f,c]) * (sum_c X[r,c] Wu[f,c])
//   down:    Y[r, n] = gate_of_row[r] * sum_f H[r,f] Wd[n,f]
//   down + combine: y[token_of_row[r], n] += gate_of_row[r] * sum_f H[r,f] Wd[n,f]  (fp32 atomics)
//   gate_up, gathered: as gate_up with X[r] = x[token_of_row[r]] (no permuted copy of x)
// Expert FFN: "Mixture of Experts Explained" (zh), section "什么是混合专家模型" (each
// expert is an FFN); SwiGLU form silu(x Wg^T) * (x Wu^T) Wd^T without biases.
//
// Tiles of 64 rows x 64 output columns, K staged 16 at a time through shared memory,
// 4 x 4 register micro-tiles (gate and up both, for gate_up), persistent grid walking
// the device-side tile schedule.
#include "common.cuh"
#include "tile_sched.cuh"

namespace moe {
namespace {

constexpr int kBM = 64, kBN = 64, kBK = 16, kThreads = 256;
constexpr int kMaxE = 1024;

template <typename DT>
__device__ __forceinline__ float ld_elem(const DT* p);
template <>
__device__ __forceinline__ float ld_elem<float>(const float* p) { return __ldg(p); }
template <>
__device__ __forceinline__ float ld_elem<__nv_bfloat16>(const __nv_bfloat16* p) {
  return __bfloat162float(__ldg(p));
}

template <typename DT>
__device__ __forceinline__ void st_elem(DT* p, float v);
template <>
__device__ __forceinline__ void st_elem<float>(float* p, float v) { *p = v; }
template <>
__device__ __forceinline__ void st_elem<__nv_bfloat16>(__nv_bfloat16* p, float v) { *p = __float2bfloat16_rn(v); }

// MODE 0: gate_up (A = x_rows [*, d], B = W_gu [E][2F][d], out = H [*, F])
// MODE 1: down    (A = H [*, F], B = W_dn [E][d][F], out = Y [*, d], scaled by gate_of_row)
// MODE 2: down + combine (as MODE 1, out = y [T, d] fp32, rows added into their token's row)
// MODE 3: gate_up with A = x [T, d] read through token_of_row
// OT: output element type (MODE 0 writes H in the activation dtype; MODE 1 writes the
// gated rows in the caller's choice of bf16 or fp32).
template <typename DT, int MODE, typename OT>
__global__ void __launch_bounds__(kThreads)
grouped_simt_kernel(const DT* __restrict__ A, const DT* __restrict__ B, const int32_t* __restrict__ offsets,
                    int E, int K, int N, int F, long long rows_max, const float* __restrict__ gate_of_row,
                    OT* __restrict__ out, const int32_t* __restrict__ token_of_row, int n_tokens, int* err) {
  __shared__ int tile_start[kMaxE + 1];
  __shared__ int sh32[32];
  __shared__ __align__(16) float As[kBK][kBM + 4];
  __shared__ __align__(16) float Bs[kBK][kBN + 4];
  constexpr bool GU = MODE == 0 || MODE == 3;               // gate/up (else down)
  __shared__ __align__(16) float Us[GU ? kBK : 1][kBN + 4];
  __shared__ int toks[MODE == 3 ? kBM : 1];

  const int n_tiles = (N + kBN - 1) / kBN;
  build_tile_starts(offsets, E, kBM, n_tiles, rows_max, tile_start, sh32, err);
  const int total = tile_start[E];
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const long long b_rows = GU ? 2LL * F : (long long)N;   // B rows per expert

  for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
    const TileCoord tc = tile_coord(tile_start, offsets, E, kBM, tile);
    const int n0 = tc.n_tile * kBN;
    const DT* Be = B + (long long)tc.e * b_rows * K;
    if (MODE == 3) {
      __syncthreads();                                     // the previous tile is done with toks
      for (int i = threadIdx.x; i < kBM; i += kThreads) {
        int t = -1;
        if (i < tc.rows) {
          t = __ldg(token_of_row + tc.row0 + i);
          if ((unsigned)t >= (unsigned)n_tokens) {
            record_error(err, MOE_DEVERR_ROW);
            t = -1;
          }
        }
        toks[i] = t;
      }
      __syncthreads();
    }
    float acc[4][4], accu[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[i][j] = accu[i][j] = 0.f;

    for (int k0 = 0; k0 < K; k0 += kBK) {
      __syncthreads();
      // A tile: 64 rows x 16 k, stored k-major
      for (int i = threadIdx.x; i < kBM * kBK; i += kThreads) {
        const int r = i / kBK, kk = i % kBK;
        float v = 0.f;
        const long long arow = MODE == 3 ? (long long)toks[r] : (long long)(tc.row0 + r);
        if (r < tc.rows && arow >= 0 && k0 + kk < K) v = ld_elem(A + arow * K + k0 + kk);
        As[kk][r] = v;
      }
      for (int i = threadIdx.x; i < kBN * kBK; i += kThreads) {
        const int n = i / kBK, kk = i % kBK;
        float g = 0.f, u = 0.f;
        if (n0 + n < N && k0 + kk < K) {
          g = ld_elem(Be + (long long)(n0 + n) * K + k0 + kk);
          if (GU) u = ld_elem(Be + (long long)(F + n0 + n) * K + k0 + kk);
        }
        Bs[kk][n] = g;
        if (GU) Us[kk][n] = u;
      }
      __syncthreads();
#pragma unroll
      for (int kk = 0; kk < kBK; ++kk) {
        const float4 a = *reinterpret_cast<const float4*>(&As[kk][ty * 4]);
        const float4 b = *reinterpret_cast<const float4*>(&Bs[kk][tx * 4]);
        const float av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
        if (GU) {
          const float4 u = *reinterpret_cast<const float4*>(&Us[kk][tx * 4]);
          const float uv[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
          for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) accu[i][j] = fmaf(av[i], uv[j], accu[i][j]);
        }
      }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int r = ty * 4 + i;
      if (r >= tc.rows) continue;
      const long long row = tc.row0 + r;
      const float gsc = (!GU && gate_of_row) ? __ldg(gate_of_row + row) : 1.f;
      int tok = 0;
      if (MODE == 2) {
        tok = __ldg(token_of_row + row);
        if ((unsigned)tok >= (unsigned)n_tokens) {
          record_error(err, MOE_DEVERR_ROW);
          continue;
        }
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int n = n0 + tx * 4 + j;
        if (n >= N) continue;
        float v;
        if (GU) {
          const float g = acc[i][j];
          v = g / (1.f + expf(-g)) * accu[i][j];
        } else {
          v = acc[i][j] * gsc;
        }
        if (MODE == 2) atomicAdd(reinterpret_cast<float*>(out) + (long long)tok * N + n, v);
        else st_elem<OT>(out + row * N + n, v);
      }
    }
  }
}

template <typename DT, int MODE, typename OT>
moe_status run_simt(const void* A, const void* B, const int32_t* offsets, int E, int K, int N, int F,
                    long long rows_max, const float* gate_of_row, void* out, cudaStream_t s,
                    const int32_t* token_of_row = nullptr, int n_tokens = 0) {
  const int grid = 2 * num_sms();
  grouped_simt_kernel<DT, MODE, OT><<<grid, kThreads, 0, s>>>(
      static_cast<const DT*>(A), static_cast<const DT*>(B), offsets, E, K, N, F, rows_max, gate_of_row,
      static_cast<OT*>(out), token_of_row, n_tokens, err_ptr());
  return check_launch();
}

}  // namespace

moe_status launch_gate_up_simt(const void* x_rows, int dtype, const int32_t* offsets, int E, int d,
                               int F, long long rows_max, const void* W_gu, void* h, cudaStream_t s) {
  if (rows_max == 0) return MOE_OK;
  if (dtype == MOE_F32)
    return run_simt<float, 0, float>(x_rows, W_gu, offsets, E, d, F, F, rows_max, nullptr, h, s);
  return run_simt<__nv_bfloat16, 0, __nv_bfloat16>(x_rows, W_gu, offsets, E, d, F, F, rows_max, nullptr, h, s);
}

moe_status launch_down_simt(const void* h, int dtype, const int32_t* offsets, int E, int d, int F,
                            long long rows_max, const void* W_dn, const float* gate_of_row,
                            int y_dtype, void* y_rows, cudaStream_t s) {
  if (rows_max == 0) return MOE_OK;
  const bool f32out = y_dtype == MOE_F32;
  if (dtype == MOE_F32)
    return f32out ? run_simt<float, 1, float>(h, W_dn, offsets, E, F, d, F, rows_max, gate_of_row, y_rows, s)
                  : run_simt<float, 1, __nv_bfloat16>(h, W_dn, offsets, E, F, d, F, rows_max, gate_of_row, y_rows, s);
  return f32out ? run_simt<__nv_bfloat16, 1, float>(h, W_dn, offsets, E, F, d, F, rows_max, gate_of_row, y_rows, s)
                : run_simt<__nv_bfloat16, 1, __nv_bfloat16>(h, W_dn, offsets, E, F, d, F, rows_max, gate_of_row,
                                                            y_rows, s);
}

moe_status launch_down_combine_simt(const void* h, int dtype, const int32_t* offsets, int E, int d, int F,
                                    long long rows_max, const void* W_dn, const float* gate_of_row,
                                    const int32_t* token_of_row, int T, float* y, cudaStream_t s) {
  if (rows_max == 0 || T == 0) return MOE_OK;
  if (dtype == MOE_F32)
    return run_simt<float, 2, float>(h, W_dn, offsets, E, F, d, F, rows_max, gate_of_row, y, s, token_of_row, T);
  return run_simt<__nv_bfloat16, 2, float>(h, W_dn, offsets, E, F, d, F, rows_max, gate_of_row, y, s, token_of_row,
                                          T);
}

moe_status launch_gate_up_gather_simt(const void* x, int dtype, const int32_t* token_of_row, int T,
                                      const int32_t* offsets, int E, int d, int F, long long rows_max,
                                      const void* W_gu, void* h, cudaStream_t s) {
  if (rows_max == 0 || T == 0) return MOE_OK;
  if (dtype == MOE_F32)
    return run_simt<float, 3, float>(x, W_gu, offsets, E, d, F, F, rows_max, nullptr, h, s, token_of_row, T);
  return run_simt<__nv_bfloat16, 3, __nv_bfloat16>(x, W_gu, offsets, E, d, F, F, rows_max, nullptr, h, s,
                                                  token_of_row, T);
}

}  // namespace moe
