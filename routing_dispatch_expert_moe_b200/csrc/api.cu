// extern "C" entry points of libmoe_b200.so: argument validation, workspace queries,
// the device error word, and dispatch to the kernel launchers.  See include/moe.h for
// the contract of every call.
#include <math.h>
#include <string.h>

#include "common.cuh"

// The one piece of library state: a per-device error word written by kernels.
__device__ int g_moe_device_error = 0;

namespace moe {

static thread_local cudaError_t g_last_cuda = cudaSuccess;
cudaError_t& last_cuda_error_ref() { return g_last_cuda; }

int* err_ptr() {
  static std::atomic<int*> cached[kMaxDevices];
  const int dev = device_slot();
  if (dev < 0) return nullptr;
  int* p = cached[dev].load(std::memory_order_acquire);
  if (!p) {
    void* a = nullptr;
    if (cudaGetSymbolAddress(&a, g_moe_device_error) == cudaSuccess) {
      p = static_cast<int*>(a);
      cached[dev].store(p, std::memory_order_release);
    }
  }
  return p;
}

}  // namespace moe

using namespace moe;

namespace {

constexpr int kMaxE = 1024;
constexpr int kMaxK = 32;
constexpr long long kMaxT = 1LL << 24;

inline cudaStream_t S(void* s) { return static_cast<cudaStream_t>(s); }

// cuMemGetAddressRange through the runtime's driver entry point (the allocation that holds
// a pointer: CUDA IPC hands out whole allocations).
typedef int (*RangeFn)(void** base, size_t* bytes, void* ptr);
static RangeFn range_fn() {
  void* p = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint("cuMemGetAddressRange", &p, cudaEnableDefault, &q) == cudaSuccess &&
      q == cudaDriverEntryPointSuccess)
    return reinterpret_cast<RangeFn>(p);
  return nullptr;
}

bool dtype_ok(int32_t dt) { return dt == MOE_BF16 || dt == MOE_F32; }

moe_status check_dims(int32_t T, int32_t E, int32_t k) {
  if (T < 0 || E < 1 || k < 1 || k > E) return MOE_ERR_INVALID_ARG;
  if (E > kMaxE || k > kMaxK || (long long)T >= kMaxT) return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

moe_status check_d(int32_t d) {
  if (d < 1) return MOE_ERR_INVALID_ARG;
  if (d % 8 != 0) return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

}  // namespace

extern "C" {

int32_t moe_version(void) { return 10000; }

const char* moe_status_str(int32_t s) {
  switch (s) {
    case MOE_OK: return "MOE_OK";
    case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG";
    case MOE_ERR_UNSUPPORTED: return "MOE_ERR_UNSUPPORTED";
    case MOE_ERR_WORKSPACE: return "MOE_ERR_WORKSPACE";
    case MOE_ERR_CUDA: return "MOE_ERR_CUDA";
    case MOE_ERR_DEVICE: return "MOE_ERR_DEVICE";
    default: return "MOE_ERR_UNKNOWN";
  }
}

const char* moe_last_cuda_error(void) { return cudaGetErrorString(g_last_cuda); }

int32_t moe_capacity(int32_t T, int32_t E, int32_t k, double capacity_factor, int32_t per_assignment) {
  if (T < 0 || E < 1 || k < 1) return -2;
  if (!(capacity_factor > 0.0)) return -1;
  const double tokens = per_assignment ? (double)T * (double)k : (double)T;
  const double c = ceil(capacity_factor * tokens / (double)E);
  if (c > 2147483647.0) return 2147483647;
  return (int32_t)c;
}

int64_t moe_rows_max(int32_t T, int32_t E, int32_t k, int32_t capacity) {
  if (T < 0 || E < 1 || k < 1) return -1;
  const int64_t A = (int64_t)T * k;
  if (capacity < 0) return A;
  const int64_t c = (int64_t)E * capacity;
  return c < A ? c : A;
}

int32_t moe_gate_up_weight_major(int64_t rows_max, int32_t E) {
  if (rows_max < 0 || E < 1) return -1;
  return prefer_weight_major(rows_max, E, false) ? 1 : 0;
}

size_t moe_route_workspace_bytes(int32_t T, int32_t d, int32_t E) {
  if (T < 0 || d < 1 || E < 1) return 0;
  return route_workspace_bytes(T, d, E, false);
}

size_t moe_router_weight_bytes(int32_t d, int32_t E) {
  if (d < 1 || E < 1 || E > kMaxE || d % 8 != 0) return 0;
  return router_weight_bytes(d, E);
}

moe_status moe_prepare_router_weight(const float* Wg, int32_t d, int32_t E, void* Wg_split, size_t bytes,
                                     void* stream) {
  if (d < 1 || E < 1) return MOE_ERR_INVALID_ARG;
  if (E > kMaxE || d % 8 != 0) return MOE_ERR_UNSUPPORTED;
  const size_t need = router_weight_bytes(d, E);
  if (need == 0) return MOE_ERR_UNSUPPORTED;
  if (!Wg || !Wg_split) return MOE_ERR_INVALID_ARG;
  if (bytes < need) return MOE_ERR_WORKSPACE;
  if (!aligned16(Wg_split)) return MOE_ERR_UNSUPPORTED;
  return launch_prepare_router_weight(Wg, d, E, Wg_split, S(stream));
}

moe_status moe_route(const void* x, int32_t x_dtype, const float* Wg, const void* Wg_split, const float* logit_offset,
                     const float* select_bias, int32_t T, int32_t d, int32_t E, int32_t k, int32_t score,
                     int32_t renormalize, float scale, float* logits, int32_t* topk_idx, float* topk_gate,
                     void* workspace, size_t workspace_bytes, void* stream) {
  moe_status st = check_dims(T, E, k);
  if (st != MOE_OK) return st;
  if ((st = check_d(d)) != MOE_OK) return st;
  if (!dtype_ok(x_dtype) || score < MOE_SCORE_SOFTMAX || score > MOE_SCORE_SQRT_SOFTPLUS ||
      (renormalize != 0 && renormalize != 1) || !isfinite(scale))
    return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  if (!x || !Wg || !logits || !topk_idx || !topk_gate) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(Wg_split)) return MOE_ERR_UNSUPPORTED;
  const size_t need = route_workspace_bytes(T, d, E, Wg_split != nullptr);
  if (need > 0 && (!workspace || workspace_bytes < need)) return MOE_ERR_WORKSPACE;
  return launch_route(x, x_dtype, Wg, Wg_split, logit_offset, select_bias, T, d, E, k, score, renormalize, scale,
                      logits, topk_idx, topk_gate, workspace, S(stream));
}

size_t moe_router_logits_workspace_bytes(int32_t T, int32_t d, int32_t E) {
  if (T < 0 || d < 1 || E < 1) return 0;
  return router_logits_workspace_bytes(T, d, E, false);
}

moe_status moe_router_logits(const void* x, int32_t x_dtype, const float* Wg, const void* Wg_split,
                             const float* logit_offset, int32_t T, int32_t d, int32_t E, float* logits,
                             void* workspace, size_t workspace_bytes, void* stream) {
  moe_status st = check_dims(T, E, 1);
  if (st != MOE_OK) return st;
  if ((st = check_d(d)) != MOE_OK) return st;
  if (!dtype_ok(x_dtype)) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  if (!x || !Wg || !logits) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(Wg_split)) return MOE_ERR_UNSUPPORTED;
  const size_t need = router_logits_workspace_bytes(T, d, E, Wg_split != nullptr);
  if (need > 0 && (!workspace || workspace_bytes < need)) return MOE_ERR_WORKSPACE;
  return launch_router_logits(x, x_dtype, Wg, Wg_split, logit_offset, T, d, E, logits, workspace, S(stream));
}

moe_status moe_route_fixed(const float* logits, int32_t T, int32_t E, int32_t k, int32_t score, int32_t renormalize,
                           float scale, int32_t rule, const int32_t* token_id, uint32_t seed, int32_t* topk_idx,
                           float* topk_gate, void* stream) {
  moe_status st = check_dims(T, E, k);
  if (st != MOE_OK) return st;
  if (score < MOE_SCORE_SOFTMAX || score > MOE_SCORE_SQRT_SOFTPLUS || (renormalize != 0 && renormalize != 1) ||
      !isfinite(scale) || (rule != MOE_SELECT_UNIFORM && rule != MOE_SELECT_HASH))
    return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  if (!logits || !topk_idx || !topk_gate || (rule == MOE_SELECT_HASH && !token_id)) return MOE_ERR_INVALID_ARG;
  return launch_route_fixed(logits, T, E, k, score, renormalize, scale, rule, token_id, seed, topk_idx, topk_gate,
                            S(stream));
}

moe_status moe_route_noisy(const float* logits, const float* logits_noise, const float* noise, int32_t T, int32_t E,
                           int32_t k, float scale, float* H, int32_t* topk_idx, float* topk_gate, void* stream) {
  moe_status st = check_dims(T, E, k);
  if (st != MOE_OK) return st;
  if (!isfinite(scale)) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  if (!logits || !logits_noise || !noise || !H || !topk_idx || !topk_gate) return MOE_ERR_INVALID_ARG;
  return launch_route_noisy(logits, logits_noise, noise, T, E, k, scale, H, topk_idx, topk_gate, S(stream));
}

int32_t moe_fp4_block_size(int32_t fmt) { return fp4_block(fmt); }

moe_status moe_quantize_fp4_host(const float* W, int64_t rows, int64_t K, int32_t fmt, uint8_t* codes,
                                 uint8_t* scales, float* tensor_scale, int32_t threads) {
  const int B = fp4_block(fmt);
  if (B < 0 || rows < 0 || K < 0 || threads < 0) return MOE_ERR_INVALID_ARG;
  if (K % B != 0) return MOE_ERR_UNSUPPORTED;
  if (fmt == MOE_FP4_NV && !tensor_scale) return MOE_ERR_INVALID_ARG;
  if (rows == 0 || K == 0) {
    if (fmt == MOE_FP4_NV) *tensor_scale = 1.0f;
    return MOE_OK;
  }
  if (!W || !codes || !scales) return MOE_ERR_INVALID_ARG;
  return quantize_fp4_host(W, rows, K, fmt, codes, scales, tensor_scale, threads);
}

moe_status moe_dequantize_fp4_host(const uint8_t* codes, const uint8_t* scales, const float* tensor_scale,
                                   int64_t rows, int64_t K, int32_t fmt, float* W, int32_t threads) {
  const int B = fp4_block(fmt);
  if (B < 0 || rows < 0 || K < 0 || threads < 0) return MOE_ERR_INVALID_ARG;
  if (K % B != 0) return MOE_ERR_UNSUPPORTED;
  if (rows == 0 || K == 0) return MOE_OK;
  if (!codes || !scales || !W || (fmt == MOE_FP4_NV && !tensor_scale)) return MOE_ERR_INVALID_ARG;
  return dequantize_fp4_host(codes, scales, tensor_scale, rows, K, fmt, W, threads);
}

size_t moe_histogram_scan_workspace_bytes(int32_t T, int32_t k, int32_t E) {
  if (T < 0 || k < 1 || E < 1) return 0;
  return histogram_scan_workspace_bytes(T, k, E);
}

moe_status moe_histogram_scan(const int32_t* topk_idx, const float* topk_gate, int32_t T, int32_t k, int32_t E,
                              int32_t capacity, int32_t* counts, int32_t* kept, int32_t* offsets, int32_t* row_of,
                              int32_t* token_of_row, float* gate_of_row, void* workspace, size_t workspace_bytes,
                              void* stream) {
  moe_status st = check_dims(T, E, k);
  if (st != MOE_OK) return st;
  if (capacity < -1) return MOE_ERR_INVALID_ARG;
  if (!counts || !kept || !offsets) return MOE_ERR_INVALID_ARG;
  if (T > 0 && (!topk_idx || !topk_gate || !row_of || !token_of_row || !gate_of_row)) return MOE_ERR_INVALID_ARG;
  const size_t need = histogram_scan_workspace_bytes(T, k, E);
  if (need > 0 && (!workspace || workspace_bytes < need)) return MOE_ERR_WORKSPACE;
  const long long rows_max = moe_rows_max(T, E, k, capacity);
  return launch_histogram_scan(topk_idx, topk_gate, T, k, E, capacity, counts, kept, offsets, row_of, token_of_row,
                               gate_of_row, rows_max, workspace, S(stream));
}

moe_status moe_histogram_scan_noalloc(const int32_t* topk_idx, const float* topk_gate, int32_t T, int32_t k,
                                      int32_t E, int32_t capacity, int32_t* counts, int32_t* kept, int32_t* offsets,
                                      int32_t* row_of, int32_t* token_of_row, float* gate_of_row, void* stream) {
  moe_status st = check_dims(T, E, k);
  if (st != MOE_OK) return st;
  if (capacity < -1) return MOE_ERR_INVALID_ARG;
  // sizes beyond the fixed scratch are refused before the pointers are even looked at
  if (histogram_scan_workspace_bytes(T, k, E) > histogram_scan_noalloc_limit()) return MOE_ERR_WORKSPACE;
  if (!counts || !kept || !offsets) return MOE_ERR_INVALID_ARG;
  if (T > 0 && (!topk_idx || !topk_gate || !row_of || !token_of_row || !gate_of_row)) return MOE_ERR_INVALID_ARG;
  const long long rows_max = moe_rows_max(T, E, k, capacity);
  return launch_histogram_scan_noalloc(topk_idx, topk_gate, T, k, E, capacity, counts, kept, offsets, row_of,
                                       token_of_row, gate_of_row, rows_max, S(stream));
}

moe_status moe_histogram_scan_caps(const int32_t* topk_idx, const float* topk_gate, int32_t T, int32_t k, int32_t E,
                                   const int32_t* caps, int32_t* counts, int32_t* kept, int32_t* offsets,
                                   int32_t* row_of, int32_t* token_of_row, float* gate_of_row, void* workspace,
                                   size_t workspace_bytes, void* stream) {
  moe_status st = check_dims(T, E, k);
  if (st != MOE_OK) return st;
  if (!caps || !counts || !kept || !offsets) return MOE_ERR_INVALID_ARG;
  if (T > 0 && (!topk_idx || !topk_gate || !row_of || !token_of_row || !gate_of_row)) return MOE_ERR_INVALID_ARG;
  const size_t need = histogram_scan_workspace_bytes(T, k, E);
  if (need > 0 && (!workspace || workspace_bytes < need)) return MOE_ERR_WORKSPACE;
  return launch_histogram_scan_caps(topk_idx, topk_gate, T, k, E, caps, counts, kept, offsets, row_of, token_of_row,
                                    gate_of_row, (long long)T * k, workspace, S(stream));
}

moe_status moe_ep_plan_host(const int32_t* counts, int32_t G, int32_t g, int32_t E, int32_t capacity, int32_t* caps,
                            int64_t* send_rows, int64_t* recv_rows, int32_t* local_offsets, int64_t* regroup) {
  if (G < 1 || g < 0 || g >= G || E < 1 || capacity < -1) return MOE_ERR_INVALID_ARG;
  if (E % G != 0 || E > kMaxE) return MOE_ERR_UNSUPPORTED;
  if (!counts || !caps || !send_rows || !recv_rows || !local_offsets || !regroup) return MOE_ERR_INVALID_ARG;
  for (long long i = 0; i < (long long)G * E; ++i)
    if (counts[i] < 0) return MOE_ERR_INVALID_ARG;
  return ep_plan_host(counts, G, g, E, capacity, caps, send_rows, recv_rows, local_offsets, regroup);
}

moe_status moe_ep_regroup(const void* src, int64_t src_rows, int32_t row_bytes, const int64_t* table, int32_t n,
                          int32_t inverse, void* dst, int64_t dst_rows, void* stream) {
  if (src_rows < 0 || dst_rows < 0 || n < 0 || row_bytes < 1 || (inverse != 0 && inverse != 1))
    return MOE_ERR_INVALID_ARG;
  if (row_bytes % 16 != 0) return MOE_ERR_UNSUPPORTED;
  if (n == 0) return MOE_OK;
  if (!table || (src_rows > 0 && !src) || (dst_rows > 0 && !dst)) return MOE_ERR_INVALID_ARG;
  if (!aligned16(src) || !aligned16(dst)) return MOE_ERR_UNSUPPORTED;
  return launch_ep_regroup(src, src_rows, row_bytes, reinterpret_cast<const long long*>(table), n, inverse, dst,
                           dst_rows, S(stream));
}

moe_status moe_ep_dst_base_host(const int32_t* counts, int32_t G, int32_t g, int32_t E, int32_t capacity,
                                int32_t* dst_base) {
  if (G < 1 || g < 0 || g >= G || E < 1 || capacity < -1) return MOE_ERR_INVALID_ARG;
  if (E % G != 0 || E > kMaxE) return MOE_ERR_UNSUPPORTED;
  if (!counts || !dst_base) return MOE_ERR_INVALID_ARG;
  for (long long i = 0; i < (long long)G * E; ++i)
    if (counts[i] < 0) return MOE_ERR_INVALID_ARG;
  return ep_dst_base_host(counts, G, g, E, capacity, dst_base);
}

moe_status moe_ep_dispatch(const void* x, int32_t dtype, int32_t T, int32_t d, int32_t k, const int32_t* topk_idx,
                           const int32_t* row_of, const int32_t* offsets, const int32_t* dst_base, int32_t E,
                           int32_t G, int64_t rows_max, const void* const* peer_rows, const int64_t* peer_rows_cap,
                           void* stream) {
  moe_status st = check_dims(T, E, k);
  if (st != MOE_OK) return st;
  if (dtype != MOE_BF16 && dtype != MOE_F32) return MOE_ERR_INVALID_ARG;
  if (G < 1 || E % G != 0 || d < 1 || rows_max < 0) return MOE_ERR_INVALID_ARG;
  if (((long long)d * (dtype == MOE_F32 ? 4 : 2)) % 16 != 0) return MOE_ERR_UNSUPPORTED;
  if (T == 0) return MOE_OK;
  if (!x || !topk_idx || !row_of || !offsets || !dst_base || !peer_rows || !peer_rows_cap) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x)) return MOE_ERR_UNSUPPORTED;
  return launch_ep_dispatch(x, dtype, T, d, k, topk_idx, row_of, offsets, dst_base, E, G, peer_rows,
                            reinterpret_cast<const long long*>(peer_rows_cap), rows_max, S(stream));
}

moe_status moe_ep_combine(const void* const* peer_rows, int32_t rows_dtype, const int64_t* peer_rows_cap, int32_t G,
                          const int32_t* topk_idx, const int32_t* row_of, const float* topk_gate,
                          const int32_t* offsets, const int32_t* dst_base, int32_t E, int32_t T, int32_t d, int32_t k,
                          int64_t rows_max, int32_t y_dtype, void* y, void* stream) {
  moe_status st = check_dims(T, E, k);
  if (st != MOE_OK) return st;
  if ((rows_dtype != MOE_BF16 && rows_dtype != MOE_F32) || (y_dtype != MOE_BF16 && y_dtype != MOE_F32))
    return MOE_ERR_INVALID_ARG;
  if (G < 1 || E % G != 0 || d < 1 || rows_max < 0) return MOE_ERR_INVALID_ARG;
  if (d % 8 != 0) return MOE_ERR_UNSUPPORTED;
  if (T == 0) return MOE_OK;
  if (!peer_rows || !peer_rows_cap || !topk_idx || !row_of || !topk_gate || !offsets || !dst_base || !y)
    return MOE_ERR_INVALID_ARG;
  if (!aligned16(y)) return MOE_ERR_UNSUPPORTED;
  return launch_ep_combine(peer_rows, rows_dtype, reinterpret_cast<const long long*>(peer_rows_cap), G, topk_idx,
                           row_of, topk_gate, offsets, dst_base, E, T, d, k, rows_max, y_dtype, y, S(stream));
}

int32_t moe_ipc_handle_bytes(void) { return (int32_t)sizeof(cudaIpcMemHandle_t); }

moe_status moe_ipc_get_handle(const void* ptr, void* handle, int64_t* offset) {
  if (!ptr || !handle || !offset) return MOE_ERR_INVALID_ARG;
  void* base = nullptr;
  size_t bytes = 0;
  static const RangeFn range = range_fn();
  if (!range) return MOE_ERR_UNSUPPORTED;
  if (range(&base, &bytes, const_cast<void*>(ptr)) != 0) return MOE_ERR_INVALID_ARG;
  cudaIpcMemHandle_t h;
  const moe_status st = cuda_status(cudaIpcGetMemHandle(&h, base));
  if (st != MOE_OK) return st;
  memcpy(handle, &h, sizeof(h));
  *offset = (int64_t)(static_cast<const char*>(ptr) - static_cast<const char*>(base));
  return MOE_OK;
}

moe_status moe_ipc_open_handle(const void* handle, int64_t offset, void** ptr, void** base) {
  if (!handle || !ptr || !base || offset < 0) return MOE_ERR_INVALID_ARG;
  cudaIpcMemHandle_t h;
  memcpy(&h, handle, sizeof(h));
  void* b = nullptr;
  const moe_status st = cuda_status(cudaIpcOpenMemHandle(&b, h, cudaIpcMemLazyEnablePeerAccess));
  if (st != MOE_OK) return st;
  *base = b;
  *ptr = static_cast<char*>(b) + offset;
  return MOE_OK;
}

moe_status moe_ipc_close(void* base) {
  if (!base) return MOE_ERR_INVALID_ARG;
  return cuda_status(cudaIpcCloseMemHandle(base));
}

moe_status moe_scan_wait_check(const int32_t* topk_idx, const float* topk_gate, int32_t T, int32_t k, int32_t E,
                               int32_t capacity, int32_t* counts, int32_t* kept, int32_t* offsets, int32_t* row_of,
                               int32_t* token_of_row, float* gate_of_row, uint64_t wait_ns, void* workspace,
                               size_t workspace_bytes, void* stream) {
  moe_status st = check_dims(T, E, k);
  if (st != MOE_OK) return st;
  if (capacity < -1 || wait_ns < 1000ull || wait_ns > 1000000000ull) return MOE_ERR_INVALID_ARG;
  if (T <= 256) return MOE_ERR_INVALID_ARG;              // needs a chunk after the withheld first one
  if (!counts || !kept || !offsets || !topk_idx || !topk_gate || !row_of || !token_of_row || !gate_of_row)
    return MOE_ERR_INVALID_ARG;
  const size_t need = histogram_scan_workspace_bytes(T, k, E);
  if (!workspace || workspace_bytes < need) return MOE_ERR_WORKSPACE;
  const long long rows_max = moe_rows_max(T, E, k, capacity);
  return launch_scan_wait_check(topk_idx, topk_gate, T, k, E, capacity, counts, kept, offsets, row_of, token_of_row,
                                gate_of_row, rows_max, workspace, (unsigned long long)wait_ns, S(stream));
}

moe_status moe_permute(const void* x, int32_t dtype, int32_t T, int32_t d, int32_t k, const int32_t* row_of,
                       int64_t rows_max, void* x_perm, void* stream) {
  if (T < 0 || k < 1 || rows_max < 0) return MOE_ERR_INVALID_ARG;
  if (k > kMaxK || (long long)T >= kMaxT) return MOE_ERR_UNSUPPORTED;
  moe_status st = check_d(d);
  if (st != MOE_OK) return st;
  if (!dtype_ok(dtype)) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  if (!x || !row_of || (rows_max > 0 && !x_perm)) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(x_perm)) return MOE_ERR_UNSUPPORTED;
  return launch_permute(x, dtype, T, d, k, row_of, rows_max, x_perm, S(stream));
}

static moe_status check_ffn(const void* a, int32_t dtype, const int32_t* offsets, int32_t E, int32_t d, int32_t F,
                            int64_t rows_max, const void* W, const void* out) {
  if (E < 1 || d < 1 || F < 1 || rows_max < 0) return MOE_ERR_INVALID_ARG;
  if (E > kMaxE) return MOE_ERR_UNSUPPORTED;
  if (d % 8 != 0 || F % 8 != 0) return MOE_ERR_UNSUPPORTED;
  if (rows_max >= (1LL << 31)) return MOE_ERR_UNSUPPORTED;
  if (!dtype_ok(dtype)) return MOE_ERR_INVALID_ARG;
  if (!offsets || !W) return MOE_ERR_INVALID_ARG;
  if (rows_max > 0 && (!a || !out)) return MOE_ERR_INVALID_ARG;
  if (!aligned16(a) || !aligned16(W) || !aligned16(out)) return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

moe_status moe_expert_gate_up(const void* x_rows, int32_t dtype, const int32_t* offsets, int32_t E, int32_t d,
                              int32_t F, int64_t rows_max, const void* W_gu, void* h, void* stream) {
  moe_status st = check_ffn(x_rows, dtype, offsets, E, d, F, rows_max, W_gu, h);
  if (st != MOE_OK || rows_max == 0) return st;
  if (dtype == MOE_BF16) {
    st = launch_gate_up_tc(x_rows, offsets, E, d, F, rows_max, W_gu, h, S(stream));
    if (st != MOE_ERR_UNSUPPORTED) return st;
  }
  return launch_gate_up_simt(x_rows, dtype, offsets, E, d, F, rows_max, W_gu, h, S(stream));
}

moe_status moe_expert_gate_up_gather(const void* x, int32_t dtype, int32_t T, const int32_t* token_of_row,
                                     const int32_t* offsets, int32_t E, int32_t d, int32_t F, int64_t rows_max,
                                     const void* W_gu, void* h, void* stream) {
  if (T < 0) return MOE_ERR_INVALID_ARG;
  if ((long long)T >= kMaxT) return MOE_ERR_UNSUPPORTED;
  moe_status st = check_ffn(x, dtype, offsets, E, d, F, rows_max, W_gu, h);
  if (st != MOE_OK || rows_max == 0 || T == 0) return st;
  if (!token_of_row) return MOE_ERR_INVALID_ARG;
  if (dtype == MOE_BF16) {
    st = launch_gate_up_gather_tc(x, token_of_row, T, offsets, E, d, F, rows_max, W_gu, h, S(stream));
    if (st != MOE_ERR_UNSUPPORTED) return st;
  }
  return launch_gate_up_gather_simt(x, dtype, token_of_row, T, offsets, E, d, F, rows_max, W_gu, h, S(stream));
}

moe_status moe_expert_down(const void* h, int32_t dtype, const int32_t* offsets, int32_t E, int32_t d, int32_t F,
                           int64_t rows_max, const void* W_dn, const float* gate_of_row, int32_t y_dtype,
                           void* y_rows, void* stream) {
  moe_status st = check_ffn(h, dtype, offsets, E, d, F, rows_max, W_dn, y_rows);
  if (st != MOE_OK) return st;
  if (!dtype_ok(y_dtype)) return MOE_ERR_INVALID_ARG;
  if (rows_max == 0) return MOE_OK;
  if (dtype == MOE_BF16) {
    st = launch_down_tc(h, offsets, E, d, F, rows_max, W_dn, gate_of_row, y_dtype, y_rows, S(stream));
    if (st != MOE_ERR_UNSUPPORTED) return st;
  }
  return launch_down_simt(h, dtype, offsets, E, d, F, rows_max, W_dn, gate_of_row, y_dtype, y_rows, S(stream));
}

moe_status moe_grouped_ffn(const void* x_rows, int32_t dtype, const int32_t* offsets, int32_t E, int32_t d, int32_t F,
                           int64_t rows_max, const void* W_gu, const void* W_dn, const float* gate_of_row, void* h,
                           int32_t y_dtype, void* y_rows, void* stream) {
  if (!dtype_ok(y_dtype)) return MOE_ERR_INVALID_ARG;
  moe_status st = moe_expert_gate_up(x_rows, dtype, offsets, E, d, F, rows_max, W_gu, h, stream);
  if (st != MOE_OK) return st;
  return moe_expert_down(h, dtype, offsets, E, d, F, rows_max, W_dn, gate_of_row, y_dtype, y_rows, stream);
}

size_t moe_fp4_scales_bytes(int64_t rows, int32_t K, int32_t fmt) {
  if (rows < 0 || K < 0 || K % 64 != 0 || fp4_block(fmt) < 0) return 0;
  return fp4_scales_bytes(rows, K, fmt);
}

moe_status moe_prepare_fp4_scales(const uint8_t* scales, int64_t rows, int32_t K, int32_t fmt, uint8_t* out,
                                  size_t bytes, void* stream) {
  if (rows < 0 || K < 0 || fp4_block(fmt) < 0) return MOE_ERR_INVALID_ARG;
  if (K % 64 != 0) return MOE_ERR_UNSUPPORTED;
  if (!out || (rows > 0 && K > 0 && !scales)) return MOE_ERR_INVALID_ARG;
  if (bytes < fp4_scales_bytes(rows, K, fmt)) return MOE_ERR_WORKSPACE;
  if (!aligned16(out)) return MOE_ERR_UNSUPPORTED;
  if (K == 0) return MOE_OK;
  return launch_prepare_fp4_scales(scales, rows, K, fmt, out, S(stream));
}

static moe_status check_fp4(const void* a, const int32_t* offsets, int32_t E, int32_t d, int32_t F, int64_t rows_max,
                            const uint8_t* codes, const uint8_t* scales, int32_t fmt, const float* tensor_scale,
                            const void* out) {
  if (E < 1 || d < 1 || F < 1 || rows_max < 0 || fp4_block(fmt) < 0) return MOE_ERR_INVALID_ARG;
  if (E > kMaxE || d % 64 != 0 || F % 64 != 0 || rows_max >= (1LL << 31)) return MOE_ERR_UNSUPPORTED;
  if (!offsets || !codes || !scales || (fmt == MOE_FP4_NV && !tensor_scale)) return MOE_ERR_INVALID_ARG;
  if (rows_max > 0 && (!a || !out)) return MOE_ERR_INVALID_ARG;
  if (!aligned16(a) || !aligned16(codes) || !aligned16(scales) || !aligned16(out)) return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

moe_status moe_expert_gate_up_fp4(const void* x_rows, const int32_t* offsets, int32_t E, int32_t d, int32_t F,
                                  int64_t rows_max, const uint8_t* codes, const uint8_t* scales, int32_t fmt,
                                  const float* tensor_scale, void* h, void* stream) {
  moe_status st = check_fp4(x_rows, offsets, E, d, F, rows_max, codes, scales, fmt, tensor_scale, h);
  if (st != MOE_OK || rows_max == 0) return st;
  return launch_gate_up_fp4(x_rows, offsets, E, d, F, rows_max, codes, scales, fmt, tensor_scale, h, S(stream));
}

moe_status moe_expert_down_fp4(const void* h, const int32_t* offsets, int32_t E, int32_t d, int32_t F,
                               int64_t rows_max, const uint8_t* codes, const uint8_t* scales, int32_t fmt,
                               const float* tensor_scale, const float* gate_of_row, int32_t y_dtype, void* y_rows,
                               void* stream) {
  moe_status st = check_fp4(h, offsets, E, d, F, rows_max, codes, scales, fmt, tensor_scale, y_rows);
  if (st != MOE_OK) return st;
  if (!dtype_ok(y_dtype)) return MOE_ERR_INVALID_ARG;
  if (rows_max == 0) return MOE_OK;
  return launch_down_fp4(h, offsets, E, d, F, rows_max, codes, scales, fmt, tensor_scale, gate_of_row, y_dtype,
                         y_rows, S(stream));
}

moe_status moe_expert_down_combine(const void* h, int32_t dtype, const int32_t* offsets, int32_t E, int32_t d,
                                   int32_t F, int64_t rows_max, const void* W_dn, const float* gate_of_row,
                                   const int32_t* token_of_row, int32_t T, int32_t accumulate, float* y,
                                   void* stream) {
  if (T < 0 || (accumulate != 0 && accumulate != 1)) return MOE_ERR_INVALID_ARG;
  if ((long long)T >= kMaxT) return MOE_ERR_UNSUPPORTED;
  moe_status st = check_ffn(h, dtype, offsets, E, d, F, rows_max, W_dn, y);
  if (st != MOE_OK) return st;
  if (T == 0) return MOE_OK;
  if (!y || (rows_max > 0 && !token_of_row)) return MOE_ERR_INVALID_ARG;
  if (!accumulate) {
    st = cuda_status(cudaMemsetAsync(y, 0, (size_t)T * (size_t)d * sizeof(float), S(stream)));
    if (st != MOE_OK) return st;
  }
  if (rows_max == 0) return MOE_OK;
  if (dtype == MOE_BF16) {
    st = launch_down_combine_tc(h, offsets, E, d, F, rows_max, W_dn, gate_of_row, token_of_row, T, y, S(stream));
    if (st != MOE_ERR_UNSUPPORTED) return st;
  }
  return launch_down_combine_simt(h, dtype, offsets, E, d, F, rows_max, W_dn, gate_of_row, token_of_row, T, y,
                                  S(stream));
}

moe_status moe_combine(const void* y_rows, int32_t rows_dtype, const int32_t* row_of, const float* topk_gate,
                       const void* shared_y, int32_t T, int32_t d, int32_t k, int64_t rows_max, int32_t y_dtype,
                       void* y, void* stream) {
  if (T < 0 || k < 1 || rows_max < 0) return MOE_ERR_INVALID_ARG;
  if (k > kMaxK || (long long)T >= kMaxT) return MOE_ERR_UNSUPPORTED;
  moe_status st = check_d(d);
  if (st != MOE_OK) return st;
  if (!dtype_ok(rows_dtype) || !dtype_ok(y_dtype)) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  if (!row_of || !y || (rows_max > 0 && !y_rows)) return MOE_ERR_INVALID_ARG;
  if (!aligned16(y_rows) || !aligned16(shared_y) || !aligned16(y)) return MOE_ERR_UNSUPPORTED;
  return launch_combine(y_rows, rows_dtype, row_of, topk_gate, shared_y, T, d, k, rows_max, y_dtype, y, S(stream));
}

size_t moe_router_stats_workspace_bytes(int32_t T, int32_t E) {
  if (T < 0 || E < 1) return 0;
  return router_stats_workspace_bytes(T, E);
}

moe_status moe_router_stats(const float* logits, const int32_t* counts, const int32_t* kept, int32_t T, int32_t E,
                            int32_t k, int32_t score, float* load, float* stats5, void* workspace,
                            size_t workspace_bytes, void* stream) {
  moe_status st = check_dims(T, E, k);
  if (st != MOE_OK) return st;
  if (score < MOE_SCORE_SOFTMAX || score > MOE_SCORE_SQRT_SOFTPLUS) return MOE_ERR_INVALID_ARG;
  if (!counts || !kept || !load || !stats5 || (T > 0 && !logits)) return MOE_ERR_INVALID_ARG;
  const size_t need = router_stats_workspace_bytes(T, E);
  if (T > 0 && (!workspace || workspace_bytes < need)) return MOE_ERR_WORKSPACE;
  return launch_router_stats(logits, counts, kept, T, E, k, score, load, stats5, workspace, S(stream));
}

size_t moe_workspace_bytes(int32_t T, int32_t d, int32_t E, int32_t k) {
  size_t a = moe_route_workspace_bytes(T, d, E);
  size_t b = moe_histogram_scan_workspace_bytes(T, k, E);
  size_t c = moe_router_stats_workspace_bytes(T, E);
  size_t m = a > b ? a : b;
  return m > c ? m : c;
}

moe_status moe_round_output(float* y32, int64_t n, void* y, int32_t clear, void* stream) {
  if (n < 0 || (clear != 0 && clear != 1)) return MOE_ERR_INVALID_ARG;
  if (n == 0) return MOE_OK;
  if (!y32 || !y) return MOE_ERR_INVALID_ARG;
  if (!aligned16(y32) || !aligned16(y)) return MOE_ERR_UNSUPPORTED;
  return launch_round_bf16(y32, n, y, clear, S(stream));
}

moe_status moe_zero(void* p, size_t bytes, void* stream) {
  if (bytes == 0) return MOE_OK;
  if (!p) return MOE_ERR_INVALID_ARG;
  if (!aligned16(p)) return MOE_ERR_UNSUPPORTED;
  return cuda_status(cudaMemsetAsync(p, 0, bytes, S(stream)));
}

moe_status moe_get_device_error(int32_t* code, void* stream) {
  if (!code) return MOE_ERR_INVALID_ARG;
  *code = 0;
  int host = 0;
  cudaError_t e = cudaMemcpyFromSymbolAsync(&host, g_moe_device_error, sizeof(int), 0, cudaMemcpyDeviceToHost, S(stream));
  if (e == cudaSuccess) e = cudaStreamSynchronize(S(stream));
  if (e != cudaSuccess) { g_last_cuda = e; return MOE_ERR_CUDA; }
  if (host != 0) {
    const int zero = 0;
    e = cudaMemcpyToSymbolAsync(g_moe_device_error, &zero, sizeof(int), 0, cudaMemcpyHostToDevice, S(stream));
    if (e == cudaSuccess) e = cudaStreamSynchronize(S(stream));
    if (e != cudaSuccess) { g_last_cuda = e; return MOE_ERR_CUDA; }
  }
  *code = host;
  return host ? MOE_ERR_DEVICE : MOE_OK;
}

}  // extern "C"
