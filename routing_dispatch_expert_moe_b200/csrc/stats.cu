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

namespace moe {
namespace {

constexpr int kStatsThreads = 256;

__device__ __forceinline__ float warp_max_f(float v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ double warp_sum_dd(double v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

template <int EPL>
__global__ void __launch_bounds__(kStatsThreads)
stats_partial_kernel(const float* __restrict__ logits, int T, int E, int score, int tokens_per_cta,
                     double* __restrict__ partP, double* __restrict__ partZ) {
  __shared__ double red[32 * EPL];            // running sum over warps, warp order
  __shared__ double redz[kStatsThreads / 32];
  const unsigned lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int nwarps = kStatsThreads / 32;
  const long long t_begin = (long long)blockIdx.x * tokens_per_cta;
  const long long t_end = min((long long)T, t_begin + tokens_per_cta);

  double P[EPL];
#pragma unroll
  for (int i = 0; i < EPL; ++i) P[i] = 0.0;
  double z2 = 0.0;
  for (long long t = t_begin + warp; t < t_end; t += nwarps) {
    float l[EPL];
    float mf = -INFINITY;
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
      const int e = lane + 32 * i;
      l[i] = e < E ? __ldg(logits + t * E + e) : -INFINITY;
      mf = fmaxf(mf, l[i]);
    }
    const double m = (double)warp_max_f(mf);
    double se = 0.0, ss = 0.0;
    double sc[EPL];
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
      const bool ok = lane + 32 * i < (unsigned)E;
      const double ex = ok ? exp((double)l[i] - m) : 0.0;
      se += ex;
      double s = 0.0;
      if (ok) {
        if (score == MOE_SCORE_SOFTMAX) s = ex;
        else if (score == MOE_SCORE_SIGMOID) s = 1.0 / (1.0 + exp(-(double)l[i]));
        else s = sqrt(fmax((double)l[i], 0.0) + log1p(exp(-fabs((double)l[i]))));
      }
      sc[i] = s;
      ss += s;
    }
    se = warp_sum_dd(se);
    ss = warp_sum_dd(ss);
    const double inv = 1.0 / ss;
#pragma unroll
    for (int i = 0; i < EPL; ++i) P[i] += sc[i] * inv;
    const double lse = m + log(se);
    z2 += lse * lse;
  }
  for (int w = 0; w < nwarps; ++w) {
    if (warp == w) {
#pragma unroll
      for (int i = 0; i < EPL; ++i) red[lane + 32 * i] = (w == 0 ? 0.0 : red[lane + 32 * i]) + P[i];
    }
    __syncthreads();
  }
  if (lane == 0) redz[warp] = z2;
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += kStatsThreads) partP[(long long)blockIdx.x * E + e] = red[e];
  if (threadIdx.x == 0) {
    double acc = 0.0;
    for (int w = 0; w < nwarps; ++w) acc += redz[w];
    partZ[blockIdx.x] = acc;
  }
}

// Stage 2: one CTA of 1024 threads.  P_e: the threads form G = 1024 / E groups of E;
// thread (g, e) sums partial rows g, g + G, g + 2G, ... of expert e (consecutive threads
// read consecutive experts of one row: whole lines per warp load, 8 loads in flight),
// then the G group sums are added in group order.  The four per-expert sums (aux, kept,
// variance, max) are reduced together in one pass.
__global__ void __launch_bounds__(1024)
stats_final_kernel(const double* __restrict__ partP, const double* __restrict__ partZ, int nparts,
                   const int32_t* __restrict__ counts, const int32_t* __restrict__ kept, int T, int E,
                   int k, float* __restrict__ load, float* __restrict__ stats5) {
  __shared__ double Ps[1024];
  __shared__ double grp[1024];
  __shared__ double red[4][32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  const int G = max(1, (int)blockDim.x / E);                 // E <= 1024
  if ((int)threadIdx.x < G * E) {
    const int e = (int)threadIdx.x % E, g = (int)threadIdx.x / E;
    double p = 0.0;
    int b = g;
    for (; b + 7 * G < nparts; b += 8 * G) {
      double v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) v[u] = __ldg(partP + (long long)(b + u * G) * E + e);
#pragma unroll
      for (int u = 0; u < 8; ++u) p += v[u];
    }
    for (; b < nparts; b += G) p += __ldg(partP + (long long)b * E + e);
    grp[threadIdx.x] = p;
  }
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
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    double p = 0.0;
    for (int g = 0; g < G; ++g) p += grp[g * E + e];
    Ps[e] = p;
  }
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

template <int EPL>
moe_status run_partial(const float* logits, int T, int E, int score, int parts, double* pP, double* pZ,
                       cudaStream_t s) {
  const int tpc = (T + parts - 1) / parts;
  stats_partial_kernel<EPL><<<parts, kStatsThreads, 0, s>>>(logits, T, E, score, tpc, pP, pZ);
  return check_launch();
}

}  // namespace

size_t router_stats_workspace_bytes(int T, int E) {
  const int parts = stats_parts(T > 0 ? T : 1);
  return ((size_t)parts * E + parts) * sizeof(double);
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
  const int epl = (E + 31) / 32;
  moe_status st;
  if (epl <= 1) st = run_partial<1>(logits, T, E, score, parts, pP, pZ, s);
  else if (epl <= 2) st = run_partial<2>(logits, T, E, score, parts, pP, pZ, s);
  else if (epl <= 4) st = run_partial<4>(logits, T, E, score, parts, pP, pZ, s);
  else if (epl <= 8) st = run_partial<8>(logits, T, E, score, parts, pP, pZ, s);
  else if (epl <= 16) st = run_partial<16>(logits, T, E, score, parts, pP, pZ, s);
  else st = run_partial<32>(logits, T, E, score, parts, pP, pZ, s);
  if (st != MOE_OK) return st;
  stats_final_kernel<<<1, 1024, 0, s>>>(pP, pZ, parts, counts, kept, T, E, k, load, stats5);
  return check_launch();
}

}  // namespace moe
