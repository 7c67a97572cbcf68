// Histogram, capacity clamp, token-order ranks, offsets and row maps.
//
// Sources: "Hugging Face 图解 Mixture of Experts（MoE）原理、训练与推理权衡", section
// "MoE 与 Transformer" (expert capacity: an expert takes at most `capacity` tokens;
// an overflowing token leaves through the residual or is dropped) and section
// "Switch Transformer" (Expert Capacity = tokens per batch / experts x capacity
// factor); section "更多关于高效训练的内容" (uneven groups, no padding).  Handbook
// article (zicq.com), "Router 与负载均衡为何决定训练成败": tokens beyond the capacity
// limit are dropped.
//
// rank(t, j) = #{t' < t : expert idx[t, j] is in the top-k of t'}  (token order).
//
// Kernel 1 (rank_kernel), one CTA per chunk of 256 tokens, chunk id taken from an
// atomic ticket so that chunk c-1 has always started before chunk c:
//   * each warp owns 32 consecutive tokens; for every (token, slot) it sets bit `lane`
//     of a per-warp, per-expert 32-bit mask in shared memory (atomicOr);
//   * popcount of a mask = that warp's count for the expert; popcount of the mask
//     below the lane = rank inside the warp; an exclusive prefix over the 8 warps gives
//     the rank inside the chunk -- all in token order, no sort;
//   * the chunk's per-expert count is published to global memory as one 32-bit word
//     (2 flag bits | 30 value bits) and every expert runs its own decoupled look-back
//     over earlier chunks (bounded spin; a wait that gives up records
//     MOE_DEVERR_SCAN_TIMEOUT and continues);
//   * the last chunk holds the inclusive totals: it writes counts, kept = min(count,
//     capacity) and offsets = exclusive scan of kept.
// Kernel 2 (scatter_kernel): row_of = offsets[e] + rank if rank < capacity else -1,
//   token_of_row, gate_of_row.
#include "common.cuh"

namespace moe {
namespace {

constexpr int kChunk = 256;          // tokens per chunk (8 warps x 32)
constexpr int kRankThreads = 256;
constexpr uint32_t kFlagAgg = 1u << 30;
constexpr uint32_t kFlagInc = 2u << 30;
constexpr uint32_t kValMask = (1u << 30) - 1;
constexpr unsigned long long kSpinLimitNs = 1000000000ull;  // 1 s

struct ScanWs {
  uint32_t* ticket;   // [1] (padded to 256 B)
  uint32_t* status;   // [C][E]
  int32_t* rank;      // [T*k]
  size_t clear_bytes; // ticket + status
};

size_t align256(size_t b) { return (b + 255) & ~size_t(255); }

ScanWs carve(void* ws, int T, int k, int E) {
  const int C = (T + kChunk - 1) / kChunk;
  char* p = static_cast<char*>(ws);
  ScanWs w;
  w.ticket = reinterpret_cast<uint32_t*>(p);
  w.status = reinterpret_cast<uint32_t*>(p + 256);
  w.clear_bytes = 256 + (size_t)C * E * 4;
  w.rank = reinterpret_cast<int32_t*>(p + align256(w.clear_bytes));
  return w;
}

__device__ __forceinline__ uint32_t ld_volatile(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.volatile.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_volatile(uint32_t* p, uint32_t v) {
  asm volatile("st.volatile.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__global__ void __launch_bounds__(kRankThreads)
rank_kernel(const int32_t* __restrict__ topk_idx, int T, int k, int E, int capacity,
            const int32_t* __restrict__ caps, int nchunks,
            uint32_t* __restrict__ ticket, uint32_t* __restrict__ status, int32_t* __restrict__ rank,
            int32_t* __restrict__ counts, int32_t* __restrict__ kept, int32_t* __restrict__ offsets,
            unsigned long long spin_limit_ns, int* err) {
  extern __shared__ __align__(16) uint32_t sm[];
  uint32_t* masks = sm;                                            // [8][E]
  uint32_t* wpre = masks + 8 * E;                                  // [8][E] warp-exclusive prefix
  int32_t* sidx = reinterpret_cast<int32_t*>(wpre + 8 * E);        // [256*k]
  int32_t* base = sidx + kChunk * k;                               // [E]
  uint32_t* tots = reinterpret_cast<uint32_t*>(base + E);         // [E]
  __shared__ int s_chunk;
  __shared__ int s_warp[32];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) s_chunk = (int)atomicAdd(ticket, 1u);
  for (int i = tid; i < 8 * E; i += kRankThreads) masks[i] = 0u;
  __syncthreads();
  const int chunk = s_chunk;
  if (chunk >= nchunks) return;   // never with the launch below; defensive
  const int t0 = chunk * kChunk;
  const int ntok = min(kChunk, T - t0);
  const long long a0 = (long long)t0 * k;
  for (int i = tid; i < ntok * k; i += kRankThreads) sidx[i] = __ldg(topk_idx + a0 + i);
  __syncthreads();

  const int tl = warp * 32 + lane;
  if (tl < ntok) {
    for (int j = 0; j < k; ++j) {
      const int e = sidx[tl * k + j];
      if ((unsigned)e >= (unsigned)E) { record_error(err, MOE_DEVERR_EXPERT_ID); continue; }
      const uint32_t bit = 1u << lane;
      const uint32_t old = atomicOr(&masks[warp * E + e], bit);
      if (old & bit) record_error(err, MOE_DEVERR_DUP_EXPERT);
    }
  }
  __syncthreads();

  const bool last = (chunk == nchunks - 1);
  for (int e = tid; e < E; e += kRankThreads) {
    uint32_t run = 0;
#pragma unroll
    for (int w = 0; w < 8; ++w) {
      wpre[w * E + e] = run;
      run += __popc(masks[w * E + e]);
    }
    const uint32_t tot = run;
    uint32_t excl = 0;
    uint32_t* my = status + (size_t)chunk * E + e;
    if (chunk == 0) {
      st_volatile(my, kFlagInc | tot);
    } else {
      st_volatile(my, kFlagAgg | tot);
      int p = chunk - 1;
      unsigned long long t_start = 0;
      unsigned spins = 0;
      while (p >= 0) {
        const uint32_t v = ld_volatile(status + (size_t)p * E + e);
        const uint32_t f = v & ~kValMask;
        if (f == 0u) {
          if (spins == 0) t_start = global_timer_ns();
          if ((++spins & 63u) == 0u && global_timer_ns() - t_start > spin_limit_ns) {
            record_error(err, MOE_DEVERR_SCAN_TIMEOUT);
            break;
          }
          __nanosleep(64);
          continue;
        }
        excl += v & kValMask;
        if (f == kFlagInc) break;
        --p;
      }
      st_volatile(my, kFlagInc | ((excl + tot) & kValMask));
    }
    base[e] = (int32_t)excl;
    tots[e] = excl + tot;   // inclusive total (used by the last chunk)
  }
  __syncthreads();
  if (tl < ntok) {
    const uint32_t lt = (1u << lane) - 1u;
    for (int j = 0; j < k; ++j) {
      const int e = sidx[tl * k + j];
      int r = -1;
      if ((unsigned)e < (unsigned)E) {
        r = base[e] + (int)wpre[warp * E + e] + __popc(masks[warp * E + e] & lt);
      }
      sidx[tl * k + j] = r;
    }
  }
  __syncthreads();
  for (int i = tid; i < ntok * k; i += kRankThreads) rank[a0 + i] = sidx[i];

  if (last) {
    // counts / kept / offsets from the inclusive totals
    int carry = 0;
    for (int e0 = 0; e0 < E; e0 += kRankThreads) {
      const int e = e0 + tid;
      int kv = 0;
      if (e < E) {
        const int c = (int)tots[e];
        const int cap_e = caps ? max(0, __ldg(caps + e)) : capacity;
        kv = cap_e < 0 ? c : min(c, cap_e);
        counts[e] = c;
        kept[e] = kv;
      }
      // block exclusive scan of kv
      int v = kv;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += n;
      }
      if (lane == 31) s_warp[warp] = v;
      __syncthreads();
      if (warp == 0) {
        int w = lane < (kRankThreads / 32) ? s_warp[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int n = __shfl_up_sync(0xffffffffu, w, o);
          if (lane >= o) w += n;
        }
        s_warp[lane] = w;   // inclusive over warps
      }
      __syncthreads();
      const int warp_excl = warp > 0 ? s_warp[warp - 1] : 0;
      if (e < E) offsets[e] = carry + warp_excl + v - kv;
      carry += s_warp[kRankThreads / 32 - 1];
      __syncthreads();
    }
    if (tid == 0) offsets[E] = carry;
  }
}

__global__ void __launch_bounds__(256)
scatter_kernel(const int32_t* __restrict__ topk_idx, const float* __restrict__ topk_gate,
               const int32_t* __restrict__ rank, const int32_t* __restrict__ offsets, int T, int k,
               int E, int capacity, const int32_t* __restrict__ caps, long long rows_max,
               int32_t* __restrict__ row_of,
               int32_t* __restrict__ token_of_row, float* __restrict__ gate_of_row, int* err) {
  const long long A = (long long)T * k;
  for (long long a = (long long)blockIdx.x * blockDim.x + threadIdx.x; a < A;
       a += (long long)gridDim.x * blockDim.x) {
    const int e = __ldg(topk_idx + a);
    int row = -1;
    if ((unsigned)e < (unsigned)E) {
      const int r = __ldg(rank + a);
      const int cap_e = caps ? max(0, __ldg(caps + e)) : capacity;
      if (r >= 0 && (cap_e < 0 || r < cap_e)) {
        const long long rr = (long long)__ldg(offsets + e) + r;
        if (rr < rows_max) row = (int)rr;
        else record_error(err, MOE_DEVERR_ROW);
      }
    }
    row_of[a] = row;
    if (row >= 0) {
      token_of_row[row] = (int32_t)(a / k);
      gate_of_row[row] = __ldg(topk_gate + a);
    }
  }
}

size_t rank_smem_bytes(int k, int E) {
  return (size_t)8 * E * 4 * 2 + (size_t)kChunk * k * 4 + (size_t)E * 4 * 2;
}

}  // namespace

// ---------------------------------------------------------------------------------
// Scratch for callers that cannot allocate (moe_histogram_scan_noalloc): a fixed 4 MiB
// array in device memory, held by every GPU that loads the library until exit.  The
// name is only a host-side handle: host code must look up its device address.
// ---------------------------------------------------------------------------------
constexpr size_t kNoAllocScratchBytes = size_t(4) << 20;
static __device__ __align__(256) unsigned char g_scan_scratch[kNoAllocScratchBytes];

// Device address of g_scan_scratch on the current device, looked up once per device
// (the first call on a device makes the lookup, so it must come before any stream
// capture on that device).
static moe_status noalloc_scratch(void** out) {
  static std::atomic<void*> cached[kMaxDevices];
  const int dev = device_slot();
  if (dev < 0) return MOE_ERR_UNSUPPORTED;
  void* p = cached[dev].load(std::memory_order_acquire);
  if (!p) {
    const cudaError_t e = cudaGetSymbolAddress(&p, g_scan_scratch);
    if (e != cudaSuccess) return cuda_status(e);
    cached[dev].store(p, std::memory_order_release);
  }
  *out = p;
  return MOE_OK;
}

size_t histogram_scan_noalloc_limit() { return kNoAllocScratchBytes; }

moe_status launch_histogram_scan_noalloc(const int32_t* topk_idx, const float* topk_gate, int T, int k, int E,
                                         int capacity, int32_t* counts, int32_t* kept, int32_t* offsets,
                                         int32_t* row_of, int32_t* token_of_row, float* gate_of_row,
                                         long long rows_max, cudaStream_t s) {
  if (histogram_scan_workspace_bytes(T, k, E) > kNoAllocScratchBytes) return MOE_ERR_WORKSPACE;
  void* ws = nullptr;
  if (T > 0) {
    moe_status st = noalloc_scratch(&ws);
    if (st != MOE_OK) return st;
  }
  // the launcher clears the ticket and look-back words before the kernels run
  return launch_histogram_scan(topk_idx, topk_gate, T, k, E, capacity, counts, kept, offsets, row_of, token_of_row,
                               gate_of_row, rows_max, ws, s);
}

size_t histogram_scan_workspace_bytes(int T, int k, int E) {
  if (T <= 0) return 0;
  const int C = (T + kChunk - 1) / kChunk;
  return align256(256 + (size_t)C * E * 4) + align256((size_t)T * k * 4);
}

// The kernels of moe_histogram_scan.  first_ticket > 0 and spin_limit_ns: the diagnostic
// form of moe_scan_wait_check (chunks 0 .. first_ticket - 1 never run, so the look-back of
// every later chunk waits for words nobody publishes, until spin_limit_ns).
static moe_status run_histogram_scan(const int32_t* topk_idx, const float* topk_gate, int T, int k, int E,
                                     int capacity, const int32_t* caps, int32_t* counts, int32_t* kept,
                                     int32_t* offsets, int32_t* row_of, int32_t* token_of_row, float* gate_of_row,
                                     long long rows_max, void* ws, cudaStream_t s, unsigned first_ticket,
                                     unsigned long long spin_limit_ns);

moe_status launch_histogram_scan(const int32_t* topk_idx, const float* topk_gate, int T, int k,
                                 int E, int capacity, int32_t* counts, int32_t* kept,
                                 int32_t* offsets, int32_t* row_of, int32_t* token_of_row,
                                 float* gate_of_row, long long rows_max, void* ws, cudaStream_t s) {
  return run_histogram_scan(topk_idx, topk_gate, T, k, E, capacity, nullptr, counts, kept, offsets, row_of,
                            token_of_row, gate_of_row, rows_max, ws, s, 0u, kSpinLimitNs);
}

// The same with a per-expert capacity (device [E]): expert e keeps its first caps[e]
// assignments in token order.
moe_status launch_histogram_scan_caps(const int32_t* topk_idx, const float* topk_gate, int T, int k, int E,
                                      const int32_t* caps, int32_t* counts, int32_t* kept, int32_t* offsets,
                                      int32_t* row_of, int32_t* token_of_row, float* gate_of_row, long long rows_max,
                                      void* ws, cudaStream_t s) {
  return run_histogram_scan(topk_idx, topk_gate, T, k, E, -1, caps, counts, kept, offsets, row_of, token_of_row,
                            gate_of_row, rows_max, ws, s, 0u, kSpinLimitNs);
}

moe_status launch_scan_wait_check(const int32_t* topk_idx, const float* topk_gate, int T, int k, int E,
                                  int capacity, int32_t* counts, int32_t* kept, int32_t* offsets, int32_t* row_of,
                                  int32_t* token_of_row, float* gate_of_row, long long rows_max, void* ws,
                                  unsigned long long wait_ns, cudaStream_t s) {
  return run_histogram_scan(topk_idx, topk_gate, T, k, E, capacity, nullptr, counts, kept, offsets, row_of,
                            token_of_row, gate_of_row, rows_max, ws, s, 1u, wait_ns);
}

static moe_status run_histogram_scan(const int32_t* topk_idx, const float* topk_gate, int T, int k, int E,
                                     int capacity, const int32_t* caps, int32_t* counts, int32_t* kept,
                                     int32_t* offsets, int32_t* row_of, int32_t* token_of_row, float* gate_of_row,
                                     long long rows_max, void* ws, cudaStream_t s, unsigned first_ticket,
                                     unsigned long long spin_limit_ns) {
  if (T == 0) {
    moe_status st = cuda_status(cudaMemsetAsync(counts, 0, (size_t)E * 4, s));
    if (st == MOE_OK) st = cuda_status(cudaMemsetAsync(kept, 0, (size_t)E * 4, s));
    if (st == MOE_OK) st = cuda_status(cudaMemsetAsync(offsets, 0, (size_t)(E + 1) * 4, s));
    return st;
  }
  ScanWs w = carve(ws, T, k, E);
  moe_status st = cuda_status(cudaMemsetAsync(ws, 0, w.clear_bytes, s));
  if (st != MOE_OK) return st;
  if (first_ticket) {   // the ticket counter starts past the withheld chunks (a small value: one byte)
    st = cuda_status(cudaMemsetAsync(w.ticket, (int)first_ticket, 1, s));
    if (st != MOE_OK) return st;
  }
  const int nchunks = (T + kChunk - 1) / kChunk;
  const size_t smem = rank_smem_bytes(k, E);
  // raise the limit once per device to the largest size any supported (k, E) needs, so
  // that no attribute call happens inside a launch sequence captured into a CUDA graph
  static std::atomic<int> configured[kMaxDevices];
  st = ensure_smem_limit(configured, rank_kernel, rank_smem_bytes(32, 1024));
  if (st != MOE_OK) return st;
  int* err = err_ptr();
  rank_kernel<<<nchunks, kRankThreads, smem, s>>>(topk_idx, T, k, E, capacity, caps, nchunks, w.ticket, w.status,
                                                 w.rank, counts, kept, offsets, spin_limit_ns, err);
  st = check_launch();
  if (st != MOE_OK) return st;
  const long long A = (long long)T * k;
  long long blocks = (A + 255) / 256;
  const long long cap = (long long)num_sms() * 8;
  if (blocks > cap) blocks = cap;
  scatter_kernel<<<(unsigned)blocks, 256, 0, s>>>(topk_idx, topk_gate, w.rank, offsets, T, k, E, capacity, caps,
                                                  rows_max, row_of, token_of_row, gate_of_row, err);
  return check_launch();
}

}  // namespace moe
