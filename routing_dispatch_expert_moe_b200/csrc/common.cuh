// Internal helpers shared by the MoE-layer kernels (sm_100a).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include <atomic>

#include "moe.h"

namespace moe {

constexpr int kWarp = 32;

// ---- device error word (address of the library's __device__ int, per device) ----
int* err_ptr();                       // host: current device's error word address (or null)
cudaError_t& last_cuda_error_ref();   // host: last CUDA error seen by a call

__device__ __forceinline__ void record_error(int* err, int code) {
  if (err) atomicCAS(err, 0, code);
}

// ---- bf16 helpers ----
__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xffff0000u); }

// Round-to-nearest-even float -> bf16 pair packed as (lo | hi << 16).
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&p);
}

// 8 values from one 16-byte vector of bf16.
__device__ __forceinline__ void unpack8(const uint4& v, float* f) {
  f[0] = bf16_lo(v.x); f[1] = bf16_hi(v.x);
  f[2] = bf16_lo(v.y); f[3] = bf16_hi(v.y);
  f[4] = bf16_lo(v.z); f[5] = bf16_hi(v.z);
  f[6] = bf16_lo(v.w); f[7] = bf16_hi(v.w);
}

__device__ __forceinline__ uint4 pack8(const float* f) {
  uint4 v;
  v.x = pack_bf16x2(f[0], f[1]);
  v.y = pack_bf16x2(f[2], f[3]);
  v.z = pack_bf16x2(f[4], f[5]);
  v.w = pack_bf16x2(f[6], f[7]);
  return v;
}

// Streaming (evict-first) 16-byte global accesses.
__device__ __forceinline__ uint4 ld_stream(const uint4* p) {
  uint4 v;
  asm volatile("ld.global.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
  return v;
}

__device__ __forceinline__ unsigned lane_id() {
  unsigned r;
  asm volatile("mov.u32 %0, %%laneid;" : "=r"(r));
  return r;
}

__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Host-side per-device tables (kernel attributes raised once, symbol addresses looked up
// once) are indexed by the CUDA device ordinal; ordinals from kMaxDevices up are not
// supported.  Entries are atomics: several host threads may race to fill one, and since
// every writer stores the same value the race is benign.
constexpr int kMaxDevices = 64;

// The current device's ordinal, or -1 when it cannot be read or has no table slot.
inline int device_slot() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return -1;
  return dev;
}

// Raises a kernel's dynamic shared-memory limit once per device (never inside a launch
// sequence that may be captured into a CUDA graph after the first call on that device).
template <typename Kernel>
inline moe_status ensure_smem_limit(std::atomic<int> (&done)[kMaxDevices], Kernel kern, size_t bytes) {
  const int dev = device_slot();
  if (dev < 0) return MOE_ERR_UNSUPPORTED;
  if (done[dev].load(std::memory_order_acquire)) return MOE_OK;
  const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e != cudaSuccess) {
    last_cuda_error_ref() = e;
    return MOE_ERR_CUDA;
  }
  done[dev].store(1, std::memory_order_release);
  return MOE_OK;
}

inline int num_sms() {
  static std::atomic<int> cached[kMaxDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) dev = 0;
  if (dev < 0 || dev >= kMaxDevices) {
    int n = 0;
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n > 0 ? n : 148;
  }
  int n = cached[dev].load(std::memory_order_relaxed);
  if (!n) {
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
    cached[dev].store(n, std::memory_order_relaxed);
  }
  return n;
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline moe_status check_launch() {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    last_cuda_error_ref() = e;
    return MOE_ERR_CUDA;
  }
  return MOE_OK;
}

inline moe_status cuda_status(cudaError_t e) {
  if (e != cudaSuccess) {
    last_cuda_error_ref() = e;
    return MOE_ERR_CUDA;
  }
  return MOE_OK;
}

// ---- launchers implemented in the kernel files (arguments already validated) ----
moe_status launch_route(const void* x, int x_dtype, const float* Wg, const void* Wg_split, const float* logit_offset,
                        const float* select_bias, int T, int d, int E, int k, int score, int renormalize,
                        float scale, float* logits, int32_t* topk_idx, float* topk_gate, void* ws, cudaStream_t s);
size_t route_workspace_bytes(int T, int d, int E, bool prepared);
moe_status launch_router_logits(const void* x, int x_dtype, const float* Wg, const void* Wg_split,
                                const float* logit_offset, int T, int d, int E, float* logits, void* ws,
                                cudaStream_t s);
size_t router_logits_workspace_bytes(int T, int d, int E, bool prepared);

// Tensor-core router (router_tc.cu): experts in n_tiles tiles of NE (a multiple of 32,
// at most kRouterMaxNE) per GEMM tile.
constexpr int kRouterMaxNE = 256;
struct RouterGeom {
  int NE, n_tiles;
};
RouterGeom router_geom(int E);
bool router_side_by_side(int NE);
size_t router_weight_bytes(int d, int E);          // prepared (split) weight; 0 = no tensor-core router
bool tc_router_applies(int x_dtype, int T, int d, int E);
moe_status launch_prepare_router_weight(const float* Wg, int d, int E, void* W3, cudaStream_t s);
moe_status launch_router_tc(const void* x, int T, int d, int E, const void* W3, const float* logit_offset,
                            float* logits, int fuse_k, const float* sel_bias, int score, int renorm, float scale,
                            int32_t* topk_idx, float* topk_gate, cudaStream_t s);
moe_status launch_route_fixed(const float* logits, int T, int E, int k, int score, int renormalize, float scale,
                              int rule, const int32_t* token_id, uint32_t seed, int32_t* topk_idx,
                              float* topk_gate, cudaStream_t s);
moe_status launch_route_noisy(const float* logits, const float* logits_noise, const float* noise, int T, int E,
                              int k, float scale, float* H, int32_t* topk_idx, float* topk_gate, cudaStream_t s);

moe_status launch_histogram_scan(const int32_t* topk_idx, const float* topk_gate, int T, int k,
                                 int E, int capacity, int32_t* counts, int32_t* kept,
                                 int32_t* offsets, int32_t* row_of, int32_t* token_of_row,
                                 float* gate_of_row, long long rows_max, void* ws, cudaStream_t s);
size_t histogram_scan_workspace_bytes(int T, int k, int E);
size_t histogram_scan_noalloc_limit();
moe_status launch_histogram_scan_caps(const int32_t* topk_idx, const float* topk_gate, int T, int k, int E,
                                      const int32_t* caps, int32_t* counts, int32_t* kept, int32_t* offsets,
                                      int32_t* row_of, int32_t* token_of_row, float* gate_of_row, long long rows_max,
                                      void* ws, cudaStream_t s);
moe_status ep_plan_host(const int32_t* counts, int G, int g, int E, int capacity, int32_t* caps, int64_t* send_rows,
                        int64_t* recv_rows, int32_t* local_offsets, int64_t* regroup);
moe_status ep_dst_base_host(const int32_t* counts, int G, int g, int E, int capacity, int32_t* dst_base);
moe_status launch_ep_dispatch(const void* x, int dtype, int T, int d, int k, const int32_t* topk_idx,
                              const int32_t* row_of, const int32_t* offsets, const int32_t* dst_base, int E, int G,
                              const void* const* peer_rows, const long long* peer_cap, long long rows_max,
                              cudaStream_t s);
moe_status launch_ep_combine(const void* const* peer_rows, int rows_dtype, const long long* peer_cap, int G,
                             const int32_t* topk_idx, const int32_t* row_of, const float* topk_gate,
                             const int32_t* offsets, const int32_t* dst_base, int E, int T, int d, int k,
                             long long rows_max, int y_dtype, void* y, cudaStream_t s);
moe_status launch_ep_regroup(const void* src, long long src_rows, int row_bytes, const long long* table, int n,
                             int inverse, void* dst, long long dst_rows, cudaStream_t s);
moe_status launch_scan_wait_check(const int32_t* topk_idx, const float* topk_gate, int T, int k, int E,
                                  int capacity, int32_t* counts, int32_t* kept, int32_t* offsets, int32_t* row_of,
                                  int32_t* token_of_row, float* gate_of_row, long long rows_max, void* ws,
                                  unsigned long long wait_ns, cudaStream_t s);
moe_status launch_histogram_scan_noalloc(const int32_t* topk_idx, const float* topk_gate, int T, int k, int E,
                                         int capacity, int32_t* counts, int32_t* kept, int32_t* offsets,
                                         int32_t* row_of, int32_t* token_of_row, float* gate_of_row,
                                         long long rows_max, cudaStream_t s);

moe_status launch_permute(const void* x, int dtype, int T, int d, int k, const int32_t* row_of,
                          long long rows_max, void* x_perm, cudaStream_t s);
moe_status launch_combine(const void* y_rows, int rows_dtype, const int32_t* row_of, const float* topk_gate,
                          const void* shared_y, int T, int d, int k, long long rows_max, int y_dtype,
                          void* y, cudaStream_t s);

int fp4_block(int fmt);
moe_status quantize_fp4_host(const float* W, long long rows, long long K, int fmt, uint8_t* codes, uint8_t* scales,
                             float* tensor_scale, int threads);
moe_status dequantize_fp4_host(const uint8_t* codes, const uint8_t* scales, const float* tensor_scale, long long rows,
                               long long K, int fmt, float* W, int threads);

moe_status launch_round_bf16(float* in, long long n, void* out, int clear, cudaStream_t s);

moe_status launch_router_stats(const float* logits, const int32_t* counts, const int32_t* kept,
                               int T, int E, int k, int score, float* load, float* stats5,
                               void* ws, cudaStream_t s);
size_t router_stats_workspace_bytes(int T, int E);

moe_status launch_gate_up_simt(const void* x_rows, int dtype, const int32_t* offsets, int E, int d,
                               int F, long long rows_max, const void* W_gu, void* h,
                               cudaStream_t s);
moe_status launch_down_simt(const void* h, int dtype, const int32_t* offsets, int E, int d, int F,
                            long long rows_max, const void* W_dn, const float* gate_of_row,
                            int y_dtype, void* y_rows, cudaStream_t s);
moe_status launch_down_combine_simt(const void* h, int dtype, const int32_t* offsets, int E, int d, int F,
                                    long long rows_max, const void* W_dn, const float* gate_of_row,
                                    const int32_t* token_of_row, int T, float* y, cudaStream_t s);
moe_status launch_down_combine_tc(const void* h, const int32_t* offsets, int E, int d, int F, long long rows_max,
                                  const void* W_dn, const float* gate_of_row, const int32_t* token_of_row, int T,
                                  float* y, cudaStream_t s);
moe_status launch_gate_up_gather_simt(const void* x, int dtype, const int32_t* token_of_row, int T,
                                      const int32_t* offsets, int E, int d, int F, long long rows_max,
                                      const void* W_gu, void* h, cudaStream_t s);
moe_status launch_gate_up_gather_tc(const void* x, const int32_t* token_of_row, int T, const int32_t* offsets, int E,
                                    int d, int F, long long rows_max, const void* W_gu, void* h, cudaStream_t s);
// Weight-major grouped GEMMs (ffn_wm.cu): tiles of 256 weight rows x the expert's tokens.
moe_status launch_gate_up_wm(const void* x_rows, const int32_t* offsets, int E, int d, int F, long long rows_max,
                             const void* W_gu, void* h, cudaStream_t s);
moe_status launch_gate_up_wm_gather(const void* x, const int32_t* token_of_row, int T, const int32_t* offsets, int E,
                                    int d, int F, long long rows_max, const void* W_gu, void* h, cudaStream_t s);
moe_status launch_down_wm(const void* h, const int32_t* offsets, int E, int d, int F, long long rows_max,
                          const void* W_dn, const float* gate_of_row, int y_dtype, void* y_rows, cudaStream_t s);
moe_status launch_gate_up_fp4(const void* x_rows, const int32_t* offsets, int E, int d, int F, long long rows_max,
                              const uint8_t* codes, const uint8_t* scales, int fmt, const float* tensor_scale,
                              void* h, cudaStream_t s);
moe_status launch_down_fp4(const void* h, const int32_t* offsets, int E, int d, int F, long long rows_max,
                           const uint8_t* codes, const uint8_t* scales, int fmt, const float* tensor_scale,
                           const float* gate_of_row, int y_dtype, void* y_rows, cudaStream_t s);
size_t fp4_scales_bytes(long long rows, int K, int fmt);
moe_status launch_prepare_fp4_scales(const uint8_t* scales, long long rows, int K, int fmt, uint8_t* out,
                                     cudaStream_t s);
// Whether a grouped GEMM over E experts and rows_max rows takes the weight-major tiles.
bool prefer_weight_major(long long rows_max, int E, bool down);

moe_status launch_gate_up_tc(const void* x_rows, const int32_t* offsets, int E, int d, int F,
                             long long rows_max, const void* W_gu, void* h, cudaStream_t s);
moe_status launch_down_tc(const void* h, const int32_t* offsets, int E, int d, int F,
                          long long rows_max, const void* W_dn, const float* gate_of_row,
                          int y_dtype, void* y_rows, cudaStream_t s);

}  // namespace moe
