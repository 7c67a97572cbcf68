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

}  // namespace

moe_status ep_plan_host(const int32_t* counts, int G, int g, int E, int capacity, int32_t* caps, int64_t* send_rows,
                        int64_t* recv_rows, int32_t* local_offsets, int64_t* regroup) {
  const int El = E / G;
  // kept[s][e] in token order across the ranks
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

}  // namespace moe
