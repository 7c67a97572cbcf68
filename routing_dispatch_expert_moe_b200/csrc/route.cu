// Router: fp32 logits, scoring, selection-only bias, top-k, gates.
//
// Sources: "Hugging Face 图解 Mixture of Experts（MoE）原理、训练与推理权衡" (Chinese
// rendering of "Mixture of Experts Explained"), section "什么是稀疏性？":
//   G_sigma(x) = Softmax(x . W_g);  KeepTopK(v, k);  G(x) = Softmax(KeepTopK(H(x), k));
// section "Switch Transformer": the router is computed in full precision because of
// its exponential.  Handbook news post (hub.geekagi.cn), "真正难在三个环节" item 1
// (routing in FP32) and item 2 (loss-free balancing bias); the quoted tweet lists
// softmax, sigmoid and sqrt(softplus) routers.  Handbook digest (agihunt.info):
// routing scale factor near sqrt(k).
//
// Two kernels:
//   logits_kernel  tiled SIMT GEMM  l = x . Wg (+ offset), fp32 FMA; W_g and x staged
//                  through shared memory, 8 experts x TM tokens per thread, optional
//                  split over d (partials summed in a fixed order by the next kernel).
//   topk_kernel    one warp per token: lanes own experts lane, lane+32, ...; k rounds of
//                  a shuffle arg-max on (key desc, index asc); gates in fp32.
#include "common.cuh"

#include <float.h>

namespace moe {
namespace {

constexpr int kLogitThreads = 256;
constexpr int kKC = 32;  // d-chunk staged per iteration

template <typename XT>
struct XLoad;
template <>
struct XLoad<__nv_bfloat16> {
  static constexpr int kPerVec = 8;
  __device__ static void load(const void* base, long long elem, bool ok, float* f) {
    if (ok) {
      uint4 v = __ldg(reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(base) + elem));
      unpack8(v, f);
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) f[i] = 0.f;
    }
  }
};
template <>
struct XLoad<float> {
  static constexpr int kPerVec = 4;
  __device__ static void load(const void* base, long long elem, bool ok, float* f) {
    if (ok) {
      float4 v = __ldg(reinterpret_cast<const float4*>(static_cast<const float*>(base) + elem));
      f[0] = v.x; f[1] = v.y; f[2] = v.z; f[3] = v.w;
    } else {
      f[0] = f[1] = f[2] = f[3] = 0.f;
    }
  }
};

// Tile: BT tokens x BE experts; thread micro-tile TM tokens x 8 experts.
template <typename XT, int BE, int TM>
__global__ void __launch_bounds__(kLogitThreads)
logits_kernel(const void* __restrict__ x, const float* __restrict__ Wg,
              const float* __restrict__ logit_offset, int T, int d, int E,
              int chunks_per_split, float* __restrict__ out, long long split_stride) {
  constexpr int TN = 8;
  constexpr int EG = BE / TN;                 // expert groups
  constexpr int TG = kLogitThreads / EG;      // token groups
  constexpr int BT = TG * TM;                 // tokens per CTA
  constexpr int PV = XLoad<XT>::kPerVec;      // x values per 16-byte vector
  constexpr int XV = BT * kKC / PV;           // x vectors per chunk
  constexpr int XV_PER_T = (XV + kLogitThreads - 1) / kLogitThreads;
  constexpr int WV = kKC * BE;                // W scalars per chunk
  constexpr int WV_PER_T = (WV + kLogitThreads - 1) / kLogitThreads;

  extern __shared__ __align__(16) float smem[];
  float* xs = smem;                 // [kKC][BT]
  float* wsm = smem + kKC * BT;     // [kKC][BE]

  const int tid = threadIdx.x;
  const int eg = tid % EG, tg = tid / EG;
  const int t0 = blockIdx.x * BT;
  const int e0 = blockIdx.y * BE;
  const int nchunks = (d + kKC - 1) / kKC;
  const int c_begin = blockIdx.z * chunks_per_split;
  const int c_end = min(nchunks, c_begin + chunks_per_split);

  float acc[TM][TN];
#pragma unroll
  for (int i = 0; i < TM; ++i)
#pragma unroll
    for (int j = 0; j < TN; ++j) acc[i][j] = 0.f;

  float xr[XV_PER_T][PV];
  float wr[WV_PER_T];

  auto gload = [&](int c) {
    const int kk0 = c * kKC;
#pragma unroll
    for (int r = 0; r < XV_PER_T; ++r) {
      const int v = tid + r * kLogitThreads;
      const int q = v / BT, t = v % BT;          // q-major: a warp covers 32 tokens
      const int col = kk0 + q * PV;
      const bool ok = (v < XV) && (t0 + t < T) && (col < d);
      XLoad<XT>::load(x, (long long)(t0 + t) * d + col, ok, xr[r]);
    }
#pragma unroll
    for (int r = 0; r < WV_PER_T; ++r) {
      const int v = tid + r * kLogitThreads;
      const int kk = v / BE, e = v % BE;
      const bool ok = (v < WV) && (kk0 + kk < d) && (e0 + e < E);
      wr[r] = ok ? __ldg(Wg + (long long)(kk0 + kk) * E + e0 + e) : 0.f;
    }
  };
  auto sstore = [&]() {
#pragma unroll
    for (int r = 0; r < XV_PER_T; ++r) {
      const int v = tid + r * kLogitThreads;
      if (v < XV) {
        const int q = v / BT, t = v % BT;
#pragma unroll
        for (int i = 0; i < PV; ++i) xs[(q * PV + i) * BT + t] = xr[r][i];
      }
    }
#pragma unroll
    for (int r = 0; r < WV_PER_T; ++r) {
      const int v = tid + r * kLogitThreads;
      if (v < WV) wsm[v] = wr[r];   // [kk][e] layout == v
    }
  };

  if (c_begin < c_end) gload(c_begin);
  for (int c = c_begin; c < c_end; ++c) {
    __syncthreads();
    sstore();
    __syncthreads();
    if (c + 1 < c_end) gload(c + 1);
#pragma unroll 8
    for (int kk = 0; kk < kKC; ++kk) {
      float xv[TM], wv[TN];
      if constexpr (TM == 4) {
        float4 a = *reinterpret_cast<const float4*>(&xs[kk * BT + tg * TM]);
        xv[0] = a.x; xv[1] = a.y; xv[2] = a.z; xv[3] = a.w;
      } else {
        float2 a = *reinterpret_cast<const float2*>(&xs[kk * BT + tg * TM]);
        xv[0] = a.x; xv[1] = a.y;
      }
      // experts {eg*4 .. +3} and {BE/2 + eg*4 .. +3}: a phase of 8 lanes reads 128
      // contiguous bytes per vector, free of bank conflicts
      float4 b0 = *reinterpret_cast<const float4*>(&wsm[kk * BE + eg * 4]);
      float4 b1 = *reinterpret_cast<const float4*>(&wsm[kk * BE + BE / 2 + eg * 4]);
      wv[0] = b0.x; wv[1] = b0.y; wv[2] = b0.z; wv[3] = b0.w;
      wv[4] = b1.x; wv[5] = b1.y; wv[6] = b1.z; wv[7] = b1.w;
#pragma unroll
      for (int i = 0; i < TM; ++i)
#pragma unroll
        for (int j = 0; j < TN; ++j) acc[i][j] = fmaf(xv[i], wv[j], acc[i][j]);
    }
  }

  float* dst = out + blockIdx.z * split_stride;
  const bool add_off = (logit_offset != nullptr) && (gridDim.z == 1);
#pragma unroll
  for (int i = 0; i < TM; ++i) {
    const int t = t0 + tg * TM + i;
    if (t >= T) continue;
#pragma unroll
    for (int j = 0; j < TN; ++j) {
      const int e = e0 + (j < 4 ? eg * 4 + j : BE / 2 + eg * 4 + (j - 4));
      if (e < E) dst[(long long)t * E + e] = acc[i][j] + (add_off ? __ldg(logit_offset + e) : 0.f);
    }
  }
}

// ---------------------------------------------------------------------------------
// top-k + gates: one warp per token.
// ---------------------------------------------------------------------------------
struct Cand {
  float kf;     // key when no selection bias (the logit)
  double kd;    // key with a selection bias (score + bias, fp64)
  int idx;
  float logit;
};

template <bool BIAS>
__device__ __forceinline__ bool better(const Cand& a, const Cand& b) {
  if (BIAS) {
    if (a.kd != b.kd) return a.kd > b.kd;
  } else {
    if (a.kf != b.kf) return a.kf > b.kf;
  }
  return a.idx < b.idx;
}

__device__ __forceinline__ double score_d(double l, int score) {
  if (score == MOE_SCORE_SIGMOID) return 1.0 / (1.0 + exp(-l));
  // MOE_SCORE_SQRT_SOFTPLUS
  return sqrt(fmax(l, 0.0) + log1p(exp(-fabs(l))));
}

__device__ __forceinline__ float score_f(float l, int score) {
  if (score == MOE_SCORE_SIGMOID) return 1.f / (1.f + expf(-l));
  return sqrtf(fmaxf(l, 0.f) + log1pf(expf(-fabsf(l))));
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ double warp_sum_d(double v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

template <int EPL, bool BIAS>
__global__ void __launch_bounds__(256)
topk_kernel(const float* __restrict__ partial, int nsplit, long long split_stride,
            const float* __restrict__ logit_offset, const float* __restrict__ select_bias,
            int T, int E, int k, int score, int renorm, float scale,
            float* __restrict__ logits, int write_logits,
            int32_t* __restrict__ topk_idx, float* __restrict__ topk_gate) {
  const unsigned lane = threadIdx.x & 31;
  const int warps = blockDim.x >> 5;
  const long long gw = (long long)blockIdx.x * warps + (threadIdx.x >> 5);
  const long long nw = (long long)gridDim.x * warps;

  for (long long t = gw; t < T; t += nw) {
    float l[EPL];
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
      const int e = lane + 32 * i;
      float v = -INFINITY;
      if (e < E) {
        float s = 0.f;
        for (int p = 0; p < nsplit; ++p) s += partial[p * split_stride + t * E + e];
        if (nsplit > 1 && logit_offset) s += __ldg(logit_offset + e);
        v = s;
        if (write_logits) logits[t * E + e] = v;
      }
      l[i] = v;
    }

    // selection keys
    float kf[EPL];
    double kd[EPL];
    if (BIAS) {
      double m = 0.0, z = 1.0;
      if (score == MOE_SCORE_SOFTMAX) {
        float mf = -INFINITY;
#pragma unroll
        for (int i = 0; i < EPL; ++i) mf = fmaxf(mf, l[i]);
        m = (double)warp_max(mf);
        double zs = 0.0;
#pragma unroll
        for (int i = 0; i < EPL; ++i)
          if (lane + 32 * i < (unsigned)E) zs += exp((double)l[i] - m);
        z = warp_sum_d(zs);
      }
#pragma unroll
      for (int i = 0; i < EPL; ++i) {
        const int e = lane + 32 * i;
        if (e < E) {
          const double sc = (score == MOE_SCORE_SOFTMAX) ? exp((double)l[i] - m) / z
                                                         : score_d((double)l[i], score);
          double key = sc + (double)__ldg(select_bias + e);
          kd[i] = (key != key) ? -INFINITY : key;
        } else {
          kd[i] = -INFINITY;
        }
        kf[i] = 0.f;
      }
    } else {
#pragma unroll
      for (int i = 0; i < EPL; ++i) {
        kf[i] = (l[i] != l[i]) ? -INFINITY : l[i];
        kd[i] = 0.0;
      }
    }

    // local best among untaken (ties: lower index == lower i on this lane)
    uint32_t taken = 0;
    auto local_best = [&]() {
      Cand b;
      b.kf = -INFINITY; b.kd = -INFINITY; b.idx = 0x7fffffff; b.logit = 0.f;
#pragma unroll
      for (int i = 0; i < EPL; ++i) {
        const int e = lane + 32 * i;
        if (e < E && !((taken >> i) & 1u)) {
          Cand c;
          c.kf = kf[i]; c.kd = kd[i]; c.idx = e; c.logit = l[i];
          if (better<BIAS>(c, b)) b = c;
        }
      }
      return b;
    };
    int sel_idx = 0;
    float sel_logit = 0.f;
    if constexpr (!BIAS) {
      // One 64-bit key per candidate: order-preserving bits of the logit above the
      // bit-inverted expert index, so an unsigned max picks the larger logit and, on
      // equal logits, the lower index.  0 marks an empty or already-taken slot (no finite
      // or infinite float maps to 0).
      uint64_t key[EPL];
#pragma unroll
      for (int i = 0; i < EPL; ++i) {
        const int e = lane + 32 * i;
        const uint32_t u = __float_as_uint(kf[i] + 0.0f);     // -0 and +0 compare equal as floats
        const uint32_t ord = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
        key[i] = e < E ? ((uint64_t)ord << 32) | (uint32_t)(~(uint32_t)e) : 0ull;
      }
      uint64_t best = 0;
#pragma unroll
      for (int i = 0; i < EPL; ++i) best = key[i] > best ? key[i] : best;
      for (int j = 0; j < k; ++j) {
        uint64_t w = best;
#pragma unroll
        for (int o = 16; o; o >>= 1) {
          const uint64_t c = __shfl_xor_sync(0xffffffffu, w, o);
          w = c > w ? c : w;
        }
        const int e = (int)(~(uint32_t)w);
        if (lane == (unsigned)j) {
          const uint32_t ord = (uint32_t)(w >> 32);
          sel_idx = e;
          sel_logit = __uint_as_float((ord & 0x80000000u) ? (ord & 0x7fffffffu) : ~ord);
        }
        if ((unsigned)(e & 31) == lane) {          // the owner drops it and refreshes its best
          best = 0;
#pragma unroll
          for (int i = 0; i < EPL; ++i) {
            if (i == (e >> 5)) key[i] = 0ull;
            best = key[i] > best ? key[i] : best;
          }
        }
      }
    }
    Cand mine = local_best();
    for (int j = 0; BIAS && j < k; ++j) {
      Cand w = mine;
#pragma unroll
      for (int o = 16; o; o >>= 1) {
        Cand c;
        if constexpr (BIAS) {
          c.kd = __shfl_xor_sync(0xffffffffu, w.kd, o);
          c.kf = 0.f;
        } else {
          c.kf = __shfl_xor_sync(0xffffffffu, w.kf, o);
          c.kd = 0.0;
        }
        c.idx = __shfl_xor_sync(0xffffffffu, w.idx, o);
        c.logit = __shfl_xor_sync(0xffffffffu, w.logit, o);
        if (better<BIAS>(c, w)) w = c;
      }
      if (lane == (unsigned)j) { sel_idx = w.idx; sel_logit = w.logit; }
      if (w.idx >= 0 && w.idx < E && (unsigned)(w.idx & 31) == lane) {
        taken |= 1u << (w.idx >> 5);
        mine = local_best();
      }
    }

    // gates (fp32 results).  The softmax over the kept logits takes the difference to the
    // maximum and its exponential in fp64: an fp32 difference of two logits far apart is
    // itself rounded, by up to half an ulp of the difference, which moves a small gate by
    // that much relatively; in fp64 the gate is within half an fp32 ulp.
    const bool act = lane < (unsigned)k;
    float g;
    if (score == MOE_SCORE_SOFTMAX) {
      if (renorm) {
        const float m = warp_max(act ? sel_logit : -INFINITY);
        const double ex = act ? exp((double)sel_logit - (double)m) : 0.0;
        g = (float)(ex / warp_sum_d(ex));
      } else {
        float mf = -INFINITY;
#pragma unroll
        for (int i = 0; i < EPL; ++i) mf = fmaxf(mf, l[i]);
        const float M = warp_max(mf);
        float zs = 0.f;
#pragma unroll
        for (int i = 0; i < EPL; ++i)
          if (lane + 32 * i < (unsigned)E) zs += expf(l[i] - M);
        const float Z = warp_sum(zs);
        g = expf(sel_logit - M) / Z;
      }
    } else {
      const float s = act ? score_f(sel_logit, score) : 0.f;
      g = renorm ? s / warp_sum(s) : s;
    }
    g *= scale;
    if (act) {
      topk_idx[t * k + lane] = sel_idx;
      topk_gate[t * k + lane] = g;
    }
  }
}

// ---------------------------------------------------------------------------------
// Tensor-core router operand: W_g [d, E] fp32 split into three bf16 terms
//   hi = bf16(w), mid = bf16(w - hi), lo = bf16(w - hi - mid)
// (each subtraction is exact in fp32; hi + mid + lo carries w to about 24 bits, and x is
// bf16, so every product x * term is exact in fp32).  Layout W3 [n_tiles * 256, d] bf16,
// K-major: n-tile j holds experts 64j..64j+63 as rows [0,64) hi, [64,128) mid,
// [128,192) lo, [192,256) padding (never written, never loaded; rows of experts past E
// are not written either: they only feed accumulator columns that are never stored).
// One 32 x 32 shared-memory transpose per block.
// ---------------------------------------------------------------------------------
__global__ void __launch_bounds__(256)
split_router_weight_kernel(const float* __restrict__ Wg, int d, int E, __nv_bfloat16* __restrict__ W3,
                           int32_t* __restrict__ offs2, int T) {
  __shared__ float tile[32][33];
  const int c0 = blockIdx.x * 32, e0 = blockIdx.y * 32;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;   // 32 x 8
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int c = c0 + ty + 8 * i, e = e0 + tx;
    tile[ty + 8 * i][tx] = (c < d && e < E) ? __ldg(Wg + (long long)c * E + e) : 0.f;
  }
  __syncthreads();
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int e = e0 + ty + 8 * i, c = c0 + tx;
    if (e >= E || c >= d) continue;
    const float w = tile[tx][ty + 8 * i];
    const __nv_bfloat16 hi = __float2bfloat16_rn(w);
    const float r1 = w - __bfloat162float(hi);
    const __nv_bfloat16 mid = __float2bfloat16_rn(r1);
    const __nv_bfloat16 lo = __float2bfloat16_rn(r1 - __bfloat162float(mid));
    const long long base = (long long)(e >> 6) * 256 + (e & 63);
    W3[(base + 0) * d + c] = hi;
    W3[(base + 64) * d + c] = mid;
    W3[(base + 128) * d + c] = lo;
  }
  if (blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0) {
    offs2[0] = 0;
    offs2[1] = T;
  }
}

struct LogitsPlan {
  int BE, TM, BT, nsplit, chunks_per_split;
  size_t smem;
};

LogitsPlan plan_logits(int T, int d, int E) {
  LogitsPlan p;
  p.BE = E > 32 ? 64 : (E > 16 ? 32 : (E > 8 ? 16 : 8));
  p.TM = p.BE >= 32 ? 4 : 2;
  const int EG = p.BE / 8, TG = kLogitThreads / EG;
  p.BT = TG * p.TM;
  p.smem = (size_t)(kKC * p.BT + kKC * p.BE) * sizeof(float);
  const int nchunks = (d + kKC - 1) / kKC;
  const long long ctas = (long long)((T + p.BT - 1) / p.BT) * ((E + p.BE - 1) / p.BE);
  int s = 1;
  const long long target = 2LL * num_sms();
  while (ctas * s < target && nchunks / (2 * s) >= 4) s *= 2;
  p.nsplit = s;
  p.chunks_per_split = (nchunks + s - 1) / s;
  return p;
}

template <typename XT, int BE, int TM>
moe_status run_logits(const void* x, const float* Wg, const float* off, int T, int d, int E,
                      const LogitsPlan& p, float* out, long long split_stride, cudaStream_t s) {
  auto kern = logits_kernel<XT, BE, TM>;
  // the shared-memory size is fixed per instantiation: raise the limit once per device,
  // never inside a launch sequence that may be captured into a CUDA graph
  static int configured[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  dev &= 63;
  if (p.smem > 48 * 1024 && !configured[dev]) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)p.smem);
    if (e != cudaSuccess) return cuda_status(e);
    configured[dev] = 1;
  }
  dim3 grid((T + p.BT - 1) / p.BT, (E + BE - 1) / BE, p.nsplit);
  kern<<<grid, kLogitThreads, p.smem, s>>>(x, Wg, off, T, d, E, p.chunks_per_split, out, split_stride);
  return check_launch();
}

template <typename XT>
moe_status dispatch_logits(const void* x, const float* Wg, const float* off, int T, int d, int E,
                           const LogitsPlan& p, float* out, long long split_stride, cudaStream_t s) {
  switch (p.BE) {
    case 64: return run_logits<XT, 64, 4>(x, Wg, off, T, d, E, p, out, split_stride, s);
    case 32: return run_logits<XT, 32, 4>(x, Wg, off, T, d, E, p, out, split_stride, s);
    case 16: return run_logits<XT, 16, 2>(x, Wg, off, T, d, E, p, out, split_stride, s);
    default: return run_logits<XT, 8, 2>(x, Wg, off, T, d, E, p, out, split_stride, s);
  }
}

template <int EPL>
moe_status run_topk(bool bias, const float* partial, int nsplit, long long split_stride,
                    const float* off, const float* sel_bias, int T, int E, int k, int score,
                    int renorm, float scale, float* logits, int write_logits, int32_t* idx,
                    float* gate, cudaStream_t s) {
  const int threads = 256;
  const long long warps_needed = T;
  long long blocks = (warps_needed + 7) / 8;
  const long long cap = (long long)num_sms() * 8;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  if (bias)
    topk_kernel<EPL, true><<<(unsigned)blocks, threads, 0, s>>>(partial, nsplit, split_stride, off, sel_bias, T, E, k,
                                                       score, renorm, scale, logits, write_logits, idx, gate);
  else
    topk_kernel<EPL, false><<<(unsigned)blocks, threads, 0, s>>>(partial, nsplit, split_stride, off, sel_bias, T, E, k,
                                                        score, renorm, scale, logits, write_logits, idx, gate);
  return check_launch();
}

// ---------------------------------------------------------------------------------
// Routing variants (the learned router's logits are still computed; only the
// selection changes, and the gates follow the learned path's rule):
//   forced-uniform selection: handbook news post, "真正难在三个环节" item 2 (a control
//     run with routing forced uniform was about 1.5x faster: the speed headroom);
//   hash selection: handbook digest, "已确认" (DeepSeek-V4 picks the experts of its
//     first three MoE layers by a fixed hash of the token id);
//   noisy top-k: "Mixture of Experts Explained", section "什么是稀疏性？", eq.
//     H(x)_i = (x.W_g)_i + StandardNormal() * Softplus((x.W_noise)_i).
// ---------------------------------------------------------------------------------

// MurmurHash3's 32-bit finalizer (Appleby): a bijection on 32-bit words.
__device__ __forceinline__ uint32_t fmix32(uint32_t h) {
  h ^= h >> 16;
  h *= 0x85ebca6bu;
  h ^= h >> 13;
  h *= 0xc2b2ae35u;
  h ^= h >> 16;
  return h;
}

// One warp per token; lane j < k owns slot j.
//   uniform: slot j of token t takes expert (t k + j) mod E;
//   hash:    Floyd's sampling of k distinct experts out of E, draw j from the word
//            fmix32(fmix32(id ^ seed) + j): with n = E - k + j, r = word mod (n + 1);
//            slot j takes r unless an earlier slot holds it (one ballot), else n.
// Gates as in topk_kernel, over the chosen experts' logits.
__global__ void __launch_bounds__(256)
fixed_select_kernel(const float* __restrict__ logits, int T, int E, int k, int score, int renorm,
                    float scale, int rule, const int32_t* __restrict__ token_id, uint32_t seed,
                    int32_t* __restrict__ topk_idx, float* __restrict__ topk_gate) {
  const unsigned lane = threadIdx.x & 31;
  const int warps = blockDim.x >> 5;
  const long long gw = (long long)blockIdx.x * warps + (threadIdx.x >> 5);
  const long long nw = (long long)gridDim.x * warps;
  const bool act = lane < (unsigned)k;
  for (long long t = gw; t < T; t += nw) {
    int mine = 0;
    if (rule == MOE_SELECT_UNIFORM) {
      mine = (int)((t * k + lane) % E);
    } else {
      const uint32_t base = fmix32((uint32_t)__ldg(token_id + t) ^ seed);
      for (int j = 0; j < k; ++j) {                 // same trip count on every lane
        const int n = E - k + j;
        const int r = (int)(fmix32(base + (uint32_t)j) % (uint32_t)(n + 1));
        const bool dup = __any_sync(0xffffffffu, lane < (unsigned)j && mine == r);
        if (lane == (unsigned)j) mine = dup ? n : r;
      }
    }
    const float* row = logits + t * E;
    const float l = act ? __ldg(row + mine) : 0.f;
    float g;
    if (score == MOE_SCORE_SOFTMAX) {
      if (renorm) {                                 // fp64 difference and exponential, as topk_kernel
        const float m = warp_max(act ? l : -INFINITY);
        const double ex = act ? exp((double)l - (double)m) : 0.0;
        g = (float)(ex / warp_sum_d(ex));
      } else {
        float mf = -INFINITY;
        for (int e = lane; e < E; e += 32) mf = fmaxf(mf, __ldg(row + e));
        const float M = warp_max(mf);
        float zs = 0.f;
        for (int e = lane; e < E; e += 32) zs += expf(__ldg(row + e) - M);
        g = expf(l - M) / warp_sum(zs);
      }
    } else {
      const float sc = act ? score_f(l, score) : 0.f;
      g = renorm ? sc / warp_sum(sc) : sc;
    }
    if (act) {
      topk_idx[t * k + lane] = mine;
      topk_gate[t * k + lane] = g * scale;
    }
  }
}

// H = l + n * softplus(l_noise) in fp32 (softplus written max(z, 0) + log1p(exp(-|z|))),
// one rounding for the product and sum.  Grid-stride over the T x E elements.
__global__ void __launch_bounds__(256)
noisy_logits_kernel(const float* __restrict__ logits, const float* __restrict__ logits_noise,
                    const float* __restrict__ noise, long long n, float* __restrict__ H) {
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (long long)gridDim.x * blockDim.x) {
    const float z = __ldg(logits_noise + i);
    const float sp = fmaxf(z, 0.f) + log1pf(expf(-fabsf(z)));
    H[i] = fmaf(__ldg(noise + i), sp, __ldg(logits + i));
  }
}

}  // namespace

// The tensor-core router takes bf16 x with d >= 64 and E a multiple of 4 (16-byte logit
// rows); anything else runs the fp32 SIMT router.
static bool tc_router_ok(int x_dtype, int d, int E) { return x_dtype == MOE_BF16 && d >= 64 && E % 4 == 0; }
static size_t tc_router_w3_bytes(int d, int E) { return (size_t)((E + 63) / 64) * 256 * d * 2; }

// Split W_g into three bf16 terms, then one tcgen05 GEMM writes logits (+ offset), or,
// with splits > 1, the partial logits of each K run to planes [splits, T, E] (no offset).
// Workspace: 256 bytes (the one-group offsets {0, T}) + the split weight (+ the planes,
// placed by the caller).  The split weight's rows for experts past E and its pad rows are
// left unwritten: they only reach accumulator columns that are never stored.
static moe_status tc_logits(const void* x, const float* Wg, const float* logit_offset, int T, int d, int E,
                            float* out, void* ws, cudaStream_t s, int splits) {
  int32_t* offs2 = static_cast<int32_t*>(ws);
  __nv_bfloat16* W3 = reinterpret_cast<__nv_bfloat16*>(static_cast<char*>(ws) + 256);
  dim3 g((d + 31) / 32, (E + 31) / 32);
  split_router_weight_kernel<<<g, 256, 0, s>>>(Wg, d, E, W3, offs2, T);
  moe_status st = check_launch();
  if (st != MOE_OK) return st;
  return launch_router_logits_tc(x, offs2, T, d, E, W3, splits > 1 ? nullptr : logit_offset, out, s, splits);
}

// The K-split planes of the tensor-core router sit after the split weight.
static size_t tc_router_planes_bytes(int T, int d, int E) {
  const int S = router_k_splits(T, d, E);
  return S > 1 ? (size_t)S * T * E * sizeof(float) : 0;
}

// Workspace one call with exactly T tokens uses: the split weight and, when the router
// splits K, its partial logits (tensor cores) or its split-K partials (SIMT).
static size_t route_workspace_at(int T, int d, int E) {
  if (T <= 0 || E <= 0 || d <= 0) return 0;
  LogitsPlan p = plan_logits(T, d, E);
  const size_t simt = p.nsplit > 1 ? (size_t)p.nsplit * T * E * sizeof(float) : 0;
  const size_t tc = (E % 4 == 0 && d >= 64) ? 256 + tc_router_w3_bytes(d, E) + tc_router_planes_bytes(T, d, E) : 0;
  return simt > tc ? simt : tc;
}

// The query covers every batch of at most T tokens, so one workspace serves a layer whose
// batches vary: a smaller batch may split K more ways and use more.  Both split choices
// depend on the batch only through its number of row tiles (128, 256 or 512 rows for the
// SIMT router, 256-row pairs for the tensor cores, which also start at 256 rows), which is
// constant on each run (128 (q - 1), 128 q]; the bytes grow with the tokens inside a run,
// so the top of each run (and T itself) bounds it.
size_t route_workspace_bytes(int T, int d, int E) {
  if (T <= 0 || E <= 0 || d <= 0) return 0;
  size_t most = route_workspace_at(T, d, E);
  for (int t = 128; t < T; t += 128) {
    const size_t w = route_workspace_at(t, d, E);
    if (w > most) most = w;
  }
  return most;
}

moe_status launch_route(const void* x, int x_dtype, const float* Wg, const float* logit_offset,
                        const float* select_bias, int T, int d, int E, int k, int score,
                        int renormalize, float scale, float* logits, int32_t* topk_idx,
                        float* topk_gate, void* ws, cudaStream_t s) {
  if (T == 0) return MOE_OK;
  LogitsPlan p = plan_logits(T, d, E);
  float* partial = logits;
  const long long split_stride = (long long)T * E;
  moe_status st = MOE_ERR_UNSUPPORTED;
  if (tc_router_ok(x_dtype, d, E)) {
    // K splits when the GEMM has too few tiles; the top-k adds the planes in order
    const int S = router_k_splits(T, d, E);
    float* planes = reinterpret_cast<float*>(static_cast<char*>(ws) + 256 + tc_router_w3_bytes(d, E));
    st = tc_logits(x, Wg, logit_offset, T, d, E, S > 1 ? planes : logits, ws, s, S);
    if (st != MOE_OK && st != MOE_ERR_UNSUPPORTED) return st;
    if (st == MOE_OK) {
      p.nsplit = S;
      partial = S > 1 ? planes : logits;
    }
  }
  if (st == MOE_ERR_UNSUPPORTED) {
    partial = p.nsplit > 1 ? static_cast<float*>(ws) : logits;
    st = x_dtype == MOE_F32
             ? dispatch_logits<float>(x, Wg, logit_offset, T, d, E, p, partial, split_stride, s)
             : dispatch_logits<__nv_bfloat16>(x, Wg, logit_offset, T, d, E, p, partial, split_stride, s);
  }
  if (st != MOE_OK) return st;
  const int write = p.nsplit > 1 ? 1 : 0;
  const int epl = (E + 31) / 32;
  const bool bias = select_bias != nullptr;
#define MOE_TOPK(N) return run_topk<N>(bias, partial, p.nsplit, split_stride, logit_offset, select_bias, T, E, k, \
                                       score, renormalize, scale, logits, write, topk_idx, topk_gate, s)
  if (epl <= 1) MOE_TOPK(1);
  if (epl <= 2) MOE_TOPK(2);
  if (epl <= 4) MOE_TOPK(4);
  if (epl <= 8) MOE_TOPK(8);
  if (epl <= 16) MOE_TOPK(16);
  MOE_TOPK(32);
#undef MOE_TOPK
}

size_t router_logits_workspace_bytes(int T, int d, int E) {
  if (T <= 0 || E <= 0 || d <= 0) return 0;
  return (E % 4 == 0 && d >= 64) ? 256 + tc_router_w3_bytes(d, E) : 0;
}

// The router alone: the tensor-core GEMM where it applies, else the SIMT GEMM in one
// pass over d (no split, so it writes the logits with their offset itself).
moe_status launch_router_logits(const void* x, int x_dtype, const float* Wg, const float* logit_offset, int T,
                                int d, int E, float* logits, void* ws, cudaStream_t s) {
  if (T == 0) return MOE_OK;
  if (tc_router_ok(x_dtype, d, E)) {
    const moe_status st = tc_logits(x, Wg, logit_offset, T, d, E, logits, ws, s, 1);
    if (st != MOE_ERR_UNSUPPORTED) return st;
  }
  LogitsPlan p = plan_logits(T, d, E);
  p.nsplit = 1;
  p.chunks_per_split = (d + kKC - 1) / kKC;
  const long long stride = (long long)T * E;
  return x_dtype == MOE_F32 ? dispatch_logits<float>(x, Wg, logit_offset, T, d, E, p, logits, stride, s)
                            : dispatch_logits<__nv_bfloat16>(x, Wg, logit_offset, T, d, E, p, logits, stride, s);
}

moe_status launch_route_fixed(const float* logits, int T, int E, int k, int score, int renormalize, float scale,
                              int rule, const int32_t* token_id, uint32_t seed, int32_t* topk_idx,
                              float* topk_gate, cudaStream_t s) {
  if (T == 0) return MOE_OK;
  long long blocks = ((long long)T + 7) / 8;                 // 8 warps (tokens) per block
  const long long cap = (long long)num_sms() * 8;
  if (blocks > cap) blocks = cap;
  fixed_select_kernel<<<(unsigned)blocks, 256, 0, s>>>(logits, T, E, k, score, renormalize, scale, rule, token_id,
                                                       seed, topk_idx, topk_gate);
  return check_launch();
}

moe_status launch_route_noisy(const float* logits, const float* logits_noise, const float* noise, int T, int E,
                              int k, float scale, float* H, int32_t* topk_idx, float* topk_gate, cudaStream_t s) {
  if (T == 0) return MOE_OK;
  const long long n = (long long)T * E;
  long long blocks = (n + 255) / 256;
  const long long cap = (long long)num_sms() * 16;
  if (blocks > cap) blocks = cap;
  noisy_logits_kernel<<<(unsigned)blocks, 256, 0, s>>>(logits, logits_noise, noise, n, H);
  moe_status st = check_launch();
  if (st != MOE_OK) return st;
  // KeepTopK on H, then the softmax over the kept H (the learned softmax router's path
  // with H in place of the logits; no offset, no selection bias)
  const int epl = (E + 31) / 32;
#define MOE_TOPK(N) return run_topk<N>(false, H, 1, n, nullptr, nullptr, T, E, k, MOE_SCORE_SOFTMAX, 1, scale, \
                                       H, 0, topk_idx, topk_gate, s)
  if (epl <= 1) MOE_TOPK(1);
  if (epl <= 2) MOE_TOPK(2);
  if (epl <= 4) MOE_TOPK(4);
  if (epl <= 8) MOE_TOPK(8);
  if (epl <= 16) MOE_TOPK(16);
  MOE_TOPK(32);
#undef MOE_TOPK
}

}  // namespace moe
