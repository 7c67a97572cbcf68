// Router statistics: per-expert load, aux load-balancing loss, router z-loss, drops,
// max/mean load, coefficient of variation.
//
// Sources: "Hugging Face 图解 Mixture of Experts（MoE）原理、训练与推理权衡", the
// auxiliary loss that pushes all experts toward equal importance (token load
// balancing; simplified in section "Switch Transformer") and the router z-loss that
// penalises large logits entering the gate (section "使用路由器 Z-loss 稳定训练").  The
// pages print neither formula; the forms used are
//   aux = E * sum_e f_e * P_e,  f_e = counts[e] / (T k),  P_e = mean_t p[t, e]
//         (p = softmax(l) for softmax scoring, s / sum_e s otherwise),
//   z   = mean_t (logsumexp_e l[t, e])^2.
// Handbook article (zicq.com) "Router 与负载均衡为何决定训练成败": monitor the max
// per-expert load ratio and the drop rate.
//
// Deterministic: stage 1 reduces each CTA's tokens into per-CTA partials in a fixed
// order (fp64); stage 2 sums the partials in a fixed lane-strided order followed by a
// fixed butterfly, so the result does not depend on scheduling.
#include "common.cuh"
#include "tc_prims.cuh"

namespace moe {
namespace {

constexpr int kStatsThreads = 512;
constexpr int kStatsPer = (1024 + kStatsThreads - 1) / kStatsThreads;   // experts per thread (E <= 1024)

// Score of one logit (fp32 transcendentals; every sum that uses them is fp64).
__device__ __forceinline__ float score_f(float l, float m, int score) {
  if (score == MOE_SCORE_SOFTMAX) return expf(l - m);
  if (score == MOE_SCORE_SIGMOID) return 1.f / (1.f + expf(-l));
  return sqrtf(fmaxf(l, 0.f) + log1pf(expf(-fabsf(l))));
}

constexpr int kSub = kStatsThreads / 32;   // tokens per sub-chunk: one per warp

// Stage 1: each CTA owns tokens [t_begin, t_end), taken kSub at a time.
//   (a) warp w takes token c0 + w: copies its logits into shared memory (independent
//       coalesced loads) while taking m = max_e l, then se = sum_e exp(l - m) and
//       ss = sum_e s_e (fp64 sums, fixed lane-strided order and butterfly), overwriting
//       each logit by its score s_e; z2 += (m + log se)^2;
//   (b) a thread per expert: P_e += s_e(t) / ss(t) over the sub-chunk's tokens, in order,
//       from shared memory.
// Every score is computed once.  Writes the CTA's P partials [E] and z2 partial.
__global__ void __launch_bounds__(kStatsThreads, 2)
stats_partial_kernel(const float* __restrict__ logits, int T, int E, int score, int tokens_per_cta,
                     double* __restrict__ partP, double* __restrict__ partZ, int* err) {
  extern __shared__ float s_sc[];            // [kSub][E]
  __shared__ double s_inv[kSub];
  __shared__ double redz[kStatsThreads / 32];
  __shared__ uint64_t s_bar[kSub];           // one row copy in flight per warp
  // rows of a whole number of 16-byte pieces arrive by one bulk copy each: the sub-chunk's
  // kSub rows are all in flight at once instead of a few loads per lane at a time
  const bool bulk = (E & 3) == 0 && (reinterpret_cast<uintptr_t>(logits) & 15u) == 0;
  const unsigned lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int nwarps = kStatsThreads / 32;
  const long long t_begin = (long long)blockIdx.x * tokens_per_cta;
  const long long t_end = min((long long)T, t_begin + tokens_per_cta);
  double z2 = 0.0;
  // this thread's experts: e = threadIdx.x + i * kStatsThreads, i < kStatsPer
  double P[kStatsPer];
#pragma unroll
  for (int q = 0; q < kStatsPer; ++q) P[q] = 0.0;
  if (threadIdx.x < kSub) mbar_init(smem_u32(&s_bar[threadIdx.x]), 1);
  fence_mbar_init();
  __syncthreads();
  uint32_t phase = 0;
  for (long long c0 = t_begin; c0 < t_end; c0 += kSub, phase ^= 1u) {
    const int n = (int)min((long long)kSub, t_end - c0);
    if (warp < n) {
      const float* row = logits + (c0 + warp) * E;
      float* srow = s_sc + warp * E;
      float mf = -INFINITY;
      if (bulk) {
        const uint32_t bar = smem_u32(&s_bar[warp]);
        if (lane == 0) {
          fence_proxy_async_smem();          // the previous sub-chunk's reads and writes of the row
          mbar_expect_tx(bar, (uint32_t)E * 4u);
          asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                       ::"r"(smem_u32(srow)), "l"(row), "r"((uint32_t)E * 4u), "r"(bar)
                       : "memory");
        }
        mbar_wait_drain(bar, phase, err);    // bounded
#pragma unroll 4
        for (int e = lane; e < E; e += 32) mf = fmaxf(mf, srow[e]);
      } else {
#pragma unroll 4
        for (int e = lane; e < E; e += 32) {
          const float l = __ldg(row + e);
          srow[e] = l;
          mf = fmaxf(mf, l);
        }
      }
#pragma unroll
      for (int o = 16; o; o >>= 1) mf = fmaxf(mf, __shfl_xor_sync(0xffffffffu, mf, o));
      double se = 0.0, ss = 0.0;
      // unrolled so the transcendentals of several elements are in flight; the fp64 sums
      // still add in element order
#pragma unroll 4
      for (int e = lane; e < E; e += 32) {
        const float l = srow[e];
        const float ex = expf(l - mf);
        const float sv = score == MOE_SCORE_SOFTMAX ? ex : score_f(l, mf, score);
        se += (double)ex;
        ss += (double)sv;
        srow[e] = sv;
      }
#pragma unroll
      for (int o = 16; o; o >>= 1) {
        se += __shfl_xor_sync(0xffffffffu, se, o);
        ss += __shfl_xor_sync(0xffffffffu, ss, o);
      }
      if (lane == 0) {
        s_inv[warp] = 1.0 / ss;
        const double lse = (double)mf + log(se);
        z2 += lse * lse;
      }
    }
    __syncthreads();
#pragma unroll
    for (int q = 0; q < kStatsPer; ++q) {
      const int e = (int)threadIdx.x + q * kStatsThreads;
      if (e < E) {
        double acc = P[q];
        for (int i = 0; i < n; ++i) acc += (double)s_sc[i * E + e] * s_inv[i];
        P[q] = acc;
      }
    }
    __syncthreads();
  }
#pragma unroll
  for (int q = 0; q < kStatsPer; ++q) {
    const int e = (int)threadIdx.x + q * kStatsThreads;
    if (e < E) partP[(long long)blockIdx.x * E + e] = P[q];
  }
  if (lane == 0) redz[warp] = z2;
  __syncthreads();
  if (threadIdx.x == 0) {
    double acc = 0.0;
    for (int w = 0; w < nwarps; ++w) acc += redz[w];
    partZ[blockIdx.x] = acc;
  }
}

// Stage 2a: P_e summed over the partial rows, 32 experts per CTA.  Lane = expert (whole
// 256-byte lines per warp load), warp w takes rows w, w + 8, w + 16, ... (8 loads in
// flight), then the 8 warp sums are added in warp order: a fixed order.
__global__ void __launch_bounds__(256)
stats_reduce_kernel(const double* __restrict__ partP, int nparts, int E, double* __restrict__ Pout) {
  __shared__ double wsum[8][32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int e = blockIdx.x * 32 + lane;
  double p = 0.0;
  if (e < E) {
    int b = warp;
    for (; b + 8 * 7 < nparts; b += 8 * 8) {
      double v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) v[u] = __ldg(partP + (long long)(b + 8 * u) * E + e);
#pragma unroll
      for (int u = 0; u < 8; ++u) p += v[u];
    }
    for (; b < nparts; b += 8) p += __ldg(partP + (long long)b * E + e);
  }
  wsum[warp][lane] = p;
  __syncthreads();
  if (warp == 0 && e < E) {
    double t = 0.0;
#pragma unroll
    for (int w = 0; w < 8; ++w) t += wsum[w][lane];
    Pout[e] = t;
  }
}

// Stage 2b: one CTA of 1024 threads: the z partials, then the four per-expert sums (aux,
// kept, variance, max) reduced together in one pass.
__global__ void __launch_bounds__(1024)
stats_final_kernel(const double* __restrict__ Psum, const double* __restrict__ partZ, int nparts,
                   const int32_t* __restrict__ counts, const int32_t* __restrict__ kept, int T, int E,
                   int k, float* __restrict__ load, float* __restrict__ stats5) {
  __shared__ double Ps[1024];
  __shared__ double red[4][32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  double z = 0.0;
  if (warp == nw - 1) {                       // the z partials, on the last warp
    int b = lane;
    for (; b + 32 * 7 < nparts; b += 32 * 8) {
      double v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) v[u] = __ldg(partZ + b + 32 * u);
#pragma unroll
      for (int u = 0; u < 8; ++u) z += v[u];
    }
    for (; b < nparts; b += 32) z += __ldg(partZ + b);
#pragma unroll
    for (int o = 16; o; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
  }
  for (int e = threadIdx.x; e < E; e += blockDim.x) Ps[e] = Psum[e];
  __syncthreads();
  const double TK = (double)T * k;
  const double mean = TK / E;
  double s[4] = {0.0, 0.0, 0.0, 0.0};          // aux, kept, variance, max count
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    const double c = (double)counts[e];
    const double f = c / TK;
    load[e] = (float)f;
    s[0] += f * (Ps[e] / (double)T);
    s[1] += (double)kept[e];
    s[2] += (c - mean) * (c - mean);
    s[3] = fmax(s[3], c);
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) {
#pragma unroll
    for (int q = 0; q < 3; ++q) s[q] += __shfl_xor_sync(0xffffffffu, s[q], o);
    s[3] = fmax(s[3], __shfl_xor_sync(0xffffffffu, s[3], o));
  }
  if (lane == 0) {
#pragma unroll
    for (int q = 0; q < 4; ++q) red[q][warp] = s[q];
  }
  __syncthreads();
  if (warp == 0) {
    double t[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) t[q] = lane < nw ? red[q][lane] : 0.0;
#pragma unroll
    for (int o = 16; o; o >>= 1) {
#pragma unroll
      for (int q = 0; q < 3; ++q) t[q] += __shfl_xor_sync(0xffffffffu, t[q], o);
      t[3] = fmax(t[3], __shfl_xor_sync(0xffffffffu, t[3], o));
    }
    if (lane == 0) {
      stats5[0] = (float)(E * t[0]);
      stats5[2] = (float)(TK - t[1]);
      stats5[3] = (float)(t[3] / mean);
      stats5[4] = (float)(sqrt(t[2] / E) / mean);
    }
  }
  if (warp == nw - 1 && lane == 0) stats5[1] = (float)(z / (double)T);
}


int stats_parts(int T) {
  const int want = 2 * num_sms();
  int parts = (T + 31) / 32;           // at least 32 tokens per CTA
  return parts < want ? (parts < 1 ? 1 : parts) : want;
}

}  // namespace

size_t router_stats_workspace_bytes(int T, int E) {
  const int parts = stats_parts(T > 0 ? T : 1);
  return ((size_t)parts * E + parts + E) * sizeof(double);   // partials [parts][E], z partials, P [E]
}

moe_status launch_router_stats(const float* logits, const int32_t* counts, const int32_t* kept,
                               int T, int E, int k, int score, float* load, float* stats5,
                               void* ws, cudaStream_t s) {
  if (T == 0) {
    moe_status st = cuda_status(cudaMemsetAsync(load, 0, (size_t)E * 4, s));
    if (st == MOE_OK) st = cuda_status(cudaMemsetAsync(stats5, 0, 5 * 4, s));
    return st;
  }
  const int parts = stats_parts(T);
  double* pP = static_cast<double*>(ws);
  double* pZ = pP + (size_t)parts * E;
  double* pSum = pZ + parts;
  const int tpc = (T + parts - 1) / parts;
  static std::atomic<int> configured[kMaxDevices];
  const size_t smem = (size_t)kSub * E * sizeof(float);    // up to 64 KB (E = 1024)
  moe_status st0 = ensure_smem_limit(configured, stats_partial_kernel, (size_t)kSub * 1024 * sizeof(float));
  if (st0 != MOE_OK) return st0;
  stats_partial_kernel<<<parts, kStatsThreads, smem, s>>>(logits, T, E, score, tpc, pP, pZ, err_ptr());
  moe_status st = check_launch();
  if (st != MOE_OK) return st;
  stats_reduce_kernel<<<(E + 31) / 32, 256, 0, s>>>(pP, parts, E, pSum);
  st = check_launch();
  if (st != MOE_OK) return st;
  stats_final_kernel<<<1, 1024, 0, s>>>(pSum, pZ, parts, counts, kept, T, E, k, load, stats5);
  return check_launch();
}

}  // namespace moe
