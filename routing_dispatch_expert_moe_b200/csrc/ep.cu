// Expert-parallel forward: the dispatch plan of one rank (host) and the regrouping of
// exchanged rows (device).
//
// Sources: "Hugging Face 图解 Mixture of Experts（MoE）原理、训练与推理权衡", section
// "让 MoE 起飞" / expert parallelism (experts live on different workers; each token is
// sent to the workers holding its experts and the results are sent back) and section
// "Switch Transformer" (capacity per expert); handbook news post (hub.geekagi.cn),
// "真正难在三个环节" item 3 (the per-layer dispatch and combine all-to-all is where the
// time of a distributed MoE layer goes).
//
// G ranks; each holds its own tokens and E / G experts, split contiguously: rank h owns
// experts [h E/G, (h+1) E/G).  The global token order is rank 0's tokens, then rank 1's,
// and so on, so capacity drops stay in token order across the ranks: with every rank's
// per-expert counts c[s][e] (all-gathered), rank s keeps the first
//   kept[s][e] = clamp(capacity - sum_{s' < s} c[s'][e], 0, c[s][e])
// of its assignments to expert e (all of them without a capacity).  A rank sends its kept
// rows of expert e to e's owner; its permuted buffer is already grouped by destination
// (experts are contiguous per rank), so one all-to-all with these row counts moves them.
// The owner receives them source by source, each source's rows grouped by expert, and
// regroups them expert by expert (sources in rank order inside an expert), the layout
// its grouped GEMMs read.  The results go back through the inverse regrouping and the
// reverse all-to-all.
#include <vector>

#include "common.cuh"
#include "row8.cuh"

namespace moe {
namespace {

// Row copies of the regrouping: table entry i = (src_off, dst_off, rows) in rows.
// Forward: dst[dst_off + r] = src[src_off + r]; inverse: dst[src_off + r] = src[dst_off + r].
// One block per entry (grid-stride over entries), 16-byte vectors along the row.
__global__ void __launch_bounds__(256)
regroup_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst, int vec_per_row,
               const long long* __restrict__ table, int n, int inverse, long long src_rows, long long dst_rows,
               int* err) {
  for (int i = blockIdx.x; i < n; i += gridDim.x) {
    long long from = __ldg(table + 3 * i), to = __ldg(table + 3 * i + 1);
    const long long rows = __ldg(table + 3 * i + 2);
    if (inverse) {
      const long long t = from;
      from = to;
      to = t;
    }
    if (rows < 0 || from < 0 || to < 0 || from + rows > src_rows || to + rows > dst_rows) {
      if (threadIdx.x == 0) record_error(err, MOE_DEVERR_ROW);
      continue;
    }
    const long long nv = rows * vec_per_row;
    const uint4* s = src + from * vec_per_row;
    uint4* d = dst + to * vec_per_row;
    for (long long v = threadIdx.x; v < nv; v += blockDim.x) d[v] = s[v];
  }
}

// The owner's position of this rank's kept assignment (row r of its expert-major rows, of
// expert e): dst_base[e] + (r - offsets[e]); -1 for a dropped slot, and -1 with the error
// word set for a row that is not expert e's, an expert out of range or a position past
// the owner's buffer.
__device__ __forceinline__ long long ep_dst_of(int r, int e, const int32_t* __restrict__ offsets,
                                               const int32_t* __restrict__ dst_base, int E, int El, int G,
                                               const long long* __restrict__ peer_cap, long long rows_max, int* h_out,
                                               int* err) {
  *h_out = 0;
  if (r < 0) return -1;
  if ((unsigned)e >= (unsigned)E || (long long)r >= rows_max) {
    record_error(err, MOE_DEVERR_ROW);
    return -1;
  }
  const int o0 = __ldg(offsets + e), o1 = __ldg(offsets + e + 1);
  const int h = e / El;
  if (r < o0 || r >= o1 || h >= G) {
    record_error(err, MOE_DEVERR_ROW);
    return -1;
  }
  const long long dst = (long long)__ldg(dst_base + e) + (r - o0);
  if (dst < 0 || dst >= __ldg(peer_cap + h)) {
    record_error(err, MOE_DEVERR_ROW);
    return -1;
  }
  *h_out = h;
  return dst;
}

// Owner h's buffer (a peer's memory through NVLink, or this GPU's own).
template <typename P>
__device__ __forceinline__ P* peer_base(const void* const* __restrict__ peer_rows, int h) {
  return reinterpret_cast<P*>(__ldg(reinterpret_cast<const unsigned long long*>(peer_rows) + h));
}

// Dispatch fused with the exchange: a warp per token reads x[t] once and stores it into
// each kept slot's owner buffer at its final expert-major position.  The permute, the
// all-to-all and the regrouping in one pass; 16-byte vectors, UNROLL per lane in flight.
template <int UNROLL>
__global__ void __launch_bounds__(256)
ep_dispatch_kernel(const uint4* __restrict__ x, int T, int nvec, int k, const int32_t* __restrict__ topk_idx,
                   const int32_t* __restrict__ row_of, const int32_t* __restrict__ offsets,
                   const int32_t* __restrict__ dst_base, int E, int El, const void* const* __restrict__ peer_rows,
                   const long long* __restrict__ peer_cap, int G, long long rows_max, int* err) {
  const unsigned lane = threadIdx.x & 31;
  const int warps = blockDim.x >> 5;
  const long long nw = (long long)gridDim.x * warps;
  for (long long t = (long long)blockIdx.x * warps + (threadIdx.x >> 5); t < T; t += nw) {
    long long my_dst = -1;
    int my_h = 0;
    if (lane < (unsigned)k) {
      const int r = __ldg(row_of + t * k + lane);
      const int e = __ldg(topk_idx + t * k + lane);
      my_dst = ep_dst_of(r, e, offsets, dst_base, E, El, G, peer_cap, rows_max, &my_h, err);
    }
    const uint4* src = x + t * nvec;
    // warp-uniform trip count: every lane reaches each shuffle below
    for (int base = 0; base < nvec; base += 32 * UNROLL) {
      uint4 buf[UNROLL];
#pragma unroll
      for (int u = 0; u < UNROLL; ++u) {
        const int v = base + (int)lane + 32 * u;
        if (v < nvec) buf[u] = ld_stream(src + v);
      }
      for (int j = 0; j < k; ++j) {
        const long long dst = __shfl_sync(0xffffffffu, my_dst, j);
        const int h = __shfl_sync(0xffffffffu, my_h, j);
        if (dst < 0) continue;
        uint4* owner = peer_base<uint4>(peer_rows, h);
        if (!owner) continue;
        uint4* row = owner + dst * nvec;
#pragma unroll
        for (int u = 0; u < UNROLL; ++u) {
          const int v = base + (int)lane + 32 * u;
          if (v < nvec) row[v] = buf[u];
        }
      }
    }
  }
}

// Combine fused with the exchange back: a warp per token gathers its kept slots' rows from
// their owners' buffers (peer loads), multiplies each by its gate and adds them in slot
// order in fp32 (as moe_combine does with gates), then rounds to the output type.  The
// kept slots' row pointers are compacted per warp in shared memory (a ballot gives
// positions).
template <typename InT, typename OutT, int KMAX>
__global__ void __launch_bounds__(256, 2)
ep_combine_kernel(const void* const* __restrict__ peer_rows, const long long* __restrict__ peer_cap, int G,
                  const int32_t* __restrict__ topk_idx, const int32_t* __restrict__ row_of,
                  const float* __restrict__ topk_gate, const int32_t* __restrict__ offsets,
                  const int32_t* __restrict__ dst_base, int E, int El, int T, int d, int k, long long rows_max,
                  void* __restrict__ y, int* err) {
  constexpr int R = KMAX <= 8 ? 8 : 4;                 // kept rows per batch of loads
  constexpr int VPI = (sizeof(InT) == 2 ? 16 : 8) / R;  // 8-element vectors per lane per batch
  __shared__ const InT* s_ptr[8][32];
  __shared__ float s_gate[8][32];
  const unsigned lane = threadIdx.x & 31;
  const int wib = threadIdx.x >> 5;
  const int warps = blockDim.x >> 5;
  const long long nw = (long long)gridDim.x * warps;
  const int n8 = d >> 3;
  const InT** kptr = s_ptr[wib];
  float* kgate = s_gate[wib];
  for (long long t = (long long)blockIdx.x * warps + wib; t < T; t += nw) {
    const InT* my_ptr = nullptr;
    float my_gate = 0.f;
    if (lane < (unsigned)k) {
      const int r = __ldg(row_of + t * k + lane);
      const int e = __ldg(topk_idx + t * k + lane);
      int h = 0;
      const long long dst = ep_dst_of(r, e, offsets, dst_base, E, El, G, peer_cap, rows_max, &h, err);
      const InT* owner = dst >= 0 ? peer_base<const InT>(peer_rows, h) : nullptr;
      if (owner) {
        my_ptr = owner + dst * d;
        my_gate = __ldg(topk_gate + t * k + lane);
      }
    }
    const unsigned kept = __ballot_sync(0xffffffffu, my_ptr != nullptr);
    const int nk = __popc(kept);
    __syncwarp();                                       // the previous token's list is read
    if (my_ptr) {
      const int pos = __popc(kept & ((1u << lane) - 1u));
      kptr[pos] = my_ptr;
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
            if (j0 + jj < nk && v0 + 32 * u < n8) buf[u][jj].load(kptr[j0 + jj], (long long)(v0 + 32 * u) * 8);
#pragma unroll
        for (int jj = 0; jj < R; ++jj)
#pragma unroll
          for (int u = 0; u < VPI; ++u)
            if (j0 + jj < nk && v0 + 32 * u < n8) buf[u][jj].add(acc[u], kgate[j0 + jj], true);
      }
#pragma unroll
      for (int u = 0; u < VPI; ++u) {
        const int v = v0 + 32 * u;
        if (v < n8) store8<OutT>(y, t * d + v * 8, acc[u]);
      }
    }
  }
}

}  // namespace

// kept[s][e]: rank s's assignments to expert e that survive the capacity, the global token
// order being rank 0's tokens, then rank 1's, ...
static std::vector<int64_t> kept_matrix(const int32_t* counts, int G, int E, int capacity) {
  std::vector<int64_t> kept((size_t)G * E);
  for (int e = 0; e < E; ++e) {
    int64_t base = 0;
    for (int s = 0; s < G; ++s) {
      const int64_t c = counts[(size_t)s * E + e];
      int64_t k = c;
      if (capacity >= 0) {
        k = (int64_t)capacity - base;
        if (k < 0) k = 0;
        if (k > c) k = c;
      }
      kept[(size_t)s * E + e] = k;
      base += c;
    }
  }
  return kept;
}

moe_status ep_plan_host(const int32_t* counts, int G, int g, int E, int capacity, int32_t* caps, int64_t* send_rows,
                        int64_t* recv_rows, int32_t* local_offsets, int64_t* regroup) {
  const int El = E / G;
  const std::vector<int64_t> kept = kept_matrix(counts, G, E, capacity);
  for (int e = 0; e < E; ++e) caps[e] = (int32_t)kept[(size_t)g * E + e];
  for (int h = 0; h < G; ++h) {
    int64_t snd = 0, rcv = 0;
    for (int j = 0; j < El; ++j) {
      snd += kept[(size_t)g * E + h * El + j];        // my rows for h's experts
      rcv += kept[(size_t)h * E + g * El + j];        // h's rows for my experts
    }
    send_rows[h] = snd;
    recv_rows[h] = rcv;
  }
  // my experts' rows, expert by expert
  local_offsets[0] = 0;
  for (int j = 0; j < El; ++j) {
    int64_t tot = 0;
    for (int s = 0; s < G; ++s) tot += kept[(size_t)s * E + g * El + j];
    local_offsets[j + 1] = (int32_t)(local_offsets[j] + tot);
  }
  // regroup table: source s's rows of local expert j
  int64_t recv_base = 0;
  for (int s = 0; s < G; ++s) {
    int64_t in_src = 0;
    for (int j = 0; j < El; ++j) {
      int64_t before = 0;                              // earlier sources' rows of expert j
      for (int s2 = 0; s2 < s; ++s2) before += kept[(size_t)s2 * E + g * El + j];
      const int64_t rows = kept[(size_t)s * E + g * El + j];
      int64_t* t = regroup + 3 * ((size_t)s * El + j);
      t[0] = recv_base + in_src;
      t[1] = local_offsets[j] + before;
      t[2] = rows;
      in_src += rows;
    }
    recv_base += recv_rows[s];
  }
  return MOE_OK;
}

// For rank g's rows of expert e (kept, in token order), their first position in the owner's
// expert-major buffer: the owner's offset of e among its experts plus the rows of e that
// earlier ranks keep.
moe_status ep_dst_base_host(const int32_t* counts, int G, int g, int E, int capacity, int32_t* dst_base) {
  const int El = E / G;
  const std::vector<int64_t> kept = kept_matrix(counts, G, E, capacity);
  for (int h = 0; h < G; ++h) {
    int64_t loc = 0;                                   // owner h's rows before its expert j
    for (int j = 0; j < El; ++j) {
      const int e = h * El + j;
      int64_t before = 0;
      for (int s = 0; s < g; ++s) before += kept[(size_t)s * E + e];
      dst_base[e] = (int32_t)(loc + before);
      for (int s = 0; s < G; ++s) loc += kept[(size_t)s * E + e];
    }
  }
  return MOE_OK;
}

moe_status launch_ep_regroup(const void* src, long long src_rows, int row_bytes, const long long* table, int n,
                             int inverse, void* dst, long long dst_rows, cudaStream_t s) {
  if (n == 0) return MOE_OK;
  int blocks = n;
  const int cap = num_sms() * 8;
  if (blocks > cap) blocks = cap;
  regroup_kernel<<<blocks, 256, 0, s>>>(static_cast<const uint4*>(src), static_cast<uint4*>(dst), row_bytes / 16,
                                        table, n, inverse, src_rows, dst_rows, err_ptr());
  return check_launch();
}


moe_status launch_ep_dispatch(const void* x, int dtype, int T, int d, int k, const int32_t* topk_idx,
                              const int32_t* row_of, const int32_t* offsets, const int32_t* dst_base, int E, int G,
                              const void* const* peer_rows, const long long* peer_cap, long long rows_max,
                              cudaStream_t s) {
  if (T == 0) return MOE_OK;
  const int esz = dtype == MOE_F32 ? 4 : 2;
  const int nvec = d * esz / 16;
  long long blocks = ((long long)T + 7) / 8;
  const long long cap = (long long)num_sms() * 8;
  if (blocks > cap) blocks = cap;
  ep_dispatch_kernel<4><<<(unsigned)blocks, 256, 0, s>>>(static_cast<const uint4*>(x), T, nvec, k, topk_idx, row_of,
                                                          offsets, dst_base, E, E / G, peer_rows, peer_cap, G,
                                                          rows_max, err_ptr());
  return check_launch();
}

template <typename InT, typename OutT>
static moe_status ep_combine_k(const void* const* peer_rows, const long long* peer_cap, int G, const int32_t* topk_idx,
                               const int32_t* row_of, const float* topk_gate, const int32_t* offsets,
                               const int32_t* dst_base, int E, int T, int d, int k, long long rows_max, void* y,
                               cudaStream_t s) {
  long long blocks = ((long long)T + 7) / 8;
  const long long cap = (long long)num_sms() * 8;
  if (blocks > cap) blocks = cap;
#define MOE_EPC(KM)                                                                                                 \
  ep_combine_kernel<InT, OutT, KM><<<(unsigned)blocks, 256, 0, s>>>(peer_rows, peer_cap, G, topk_idx, row_of,    \
                                                                     topk_gate, offsets, dst_base, E, E / G, T, d, \
                                                                     k, rows_max, y, err_ptr())
  if (k <= 8) MOE_EPC(8);
  else if (k <= 16) MOE_EPC(16);
  else MOE_EPC(32);
#undef MOE_EPC
  return check_launch();
}

moe_status launch_ep_combine(const void* const* peer_rows, int rows_dtype, const long long* peer_cap, int G,
                             const int32_t* topk_idx, const int32_t* row_of, const float* topk_gate,
                             const int32_t* offsets, const int32_t* dst_base, int E, int T, int d, int k,
                             long long rows_max, int y_dtype, void* y, cudaStream_t s) {
  if (T == 0) return MOE_OK;
  const bool in32 = rows_dtype == MOE_F32, out32 = y_dtype == MOE_F32;
  if (in32 && out32)
    return ep_combine_k<float, float>(peer_rows, peer_cap, G, topk_idx, row_of, topk_gate, offsets, dst_base, E, T, d,
                                      k, rows_max, y, s);
  if (in32)
    return ep_combine_k<float, __nv_bfloat16>(peer_rows, peer_cap, G, topk_idx, row_of, topk_gate, offsets, dst_base,
                                              E, T, d, k, rows_max, y, s);
  if (out32)
    return ep_combine_k<__nv_bfloat16, float>(peer_rows, peer_cap, G, topk_idx, row_of, topk_gate, offsets, dst_base,
                                              E, T, d, k, rows_max, y, s);
  return ep_combine_k<__nv_bfloat16, __nv_bfloat16>(peer_rows, peer_cap, G, topk_idx, row_of, topk_gate, offsets,
                                                    dst_base, E, T, d, k, rows_max, y, s);
}

}  // namespace moe
