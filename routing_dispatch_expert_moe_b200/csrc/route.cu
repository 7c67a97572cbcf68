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
// The tensor-core router with the top-k in its epilogue (router_tc.cu) serves bf16 x
// with at least 256 tokens; this file holds the rest:
//   logits_kernel  tiled SIMT GEMM  l = x . Wg (+ offset), fp32 FMA; W_g and x staged
//                  through shared memory, 8 experts x TM tokens per thread, optional
//                  split over d (partials summed in a fixed order by the next kernel);
//                  for fp32 x, small batches, d < 64 or E not a multiple of 4.
//   topk_kernel    one warp per token: lanes own experts lane, lane+32, ...; k rounds of
//                  a shuffle arg-max on (key desc, index asc); gates in fp32.  After the
//                  SIMT router, after the tensor-core router for softmax scores with a
//                  selection bias, and for noisy top-k.
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
  static std::atomic<int> configured[kMaxDevices];
  if (p.smem > 48 * 1024) {
    const moe_status st = ensure_smem_limit(configured, kern, p.smem);
    if (st != MOE_OK) return st;
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

// SIMT router workspace of a call with exactly T tokens: its split-K partials.
static size_t simt_workspace_at(int T, int d, int E) {
  if (T <= 0 || E <= 0 || d <= 0) return 0;
  LogitsPlan p = plan_logits(T, d, E);
  return p.nsplit > 1 ? (size_t)p.nsplit * T * E * sizeof(float) : 0;
}

// The query covers every batch of at most T tokens and either x dtype, so one workspace
// serves a layer whose batches vary.  The SIMT router (fp32 x, batches under 256 tokens,
// shapes the tensor cores do not take) may split K more ways for a smaller batch: the
// split choice depends on the batch only through its number of row tiles (128, 256 or
// 512 rows), constant on each run (128 (q - 1), 128 q], and the bytes grow with the
// tokens inside a run, so the top of each run (and T itself) bounds it.  The tensor-core
// router needs room for the split weight when it is not given a prepared one.
size_t route_workspace_bytes(int T, int d, int E, bool prepared) {
  if (T <= 0 || E <= 0 || d <= 0) return 0;
  size_t most = simt_workspace_at(T, d, E);
  for (int t = 128; t < T; t += 128) {
    const size_t w = simt_workspace_at(t, d, E);
    if (w > most) most = w;
  }
  if (!prepared && tc_router_applies(MOE_BF16, T, d, E)) {
    const size_t w = router_weight_bytes(d, E);
    if (w > most) most = w;
  }
  return most;
}

template <int EPL>
static moe_status topk_dispatch(bool bias, const float* partial, int nsplit, long long split_stride, const float* off,
                                const float* sel_bias, int T, int E, int k, int score, int renorm, float scale,
                                float* logits, int write_logits, int32_t* idx, float* gate, cudaStream_t s) {
  return run_topk<EPL>(bias, partial, nsplit, split_stride, off, sel_bias, T, E, k, score, renorm, scale, logits,
                       write_logits, idx, gate, s);
}

static moe_status run_topk_any(bool bias, const float* partial, int nsplit, long long split_stride, const float* off,
                               const float* sel_bias, int T, int E, int k, int score, int renorm, float scale,
                               float* logits, int write_logits, int32_t* idx, float* gate, cudaStream_t s) {
  const int epl = (E + 31) / 32;
#define MOE_TOPK(N) return topk_dispatch<N>(bias, partial, nsplit, split_stride, off, sel_bias, T, E, k, score, renorm, \
                                            scale, logits, write_logits, idx, gate, s)
  if (epl <= 1) MOE_TOPK(1);
  if (epl <= 2) MOE_TOPK(2);
  if (epl <= 4) MOE_TOPK(4);
  if (epl <= 8) MOE_TOPK(8);
  if (epl <= 16) MOE_TOPK(16);
  MOE_TOPK(32);
#undef MOE_TOPK
}

// The prepared weight to use: the caller's, or one split into the workspace now.
static moe_status router_weight(const float* Wg, const void* Wg_split, int d, int E, void* ws, const void** W3,
                                cudaStream_t s) {
  if (Wg_split) {
    *W3 = Wg_split;
    return MOE_OK;
  }
  *W3 = ws;
  return launch_prepare_router_weight(Wg, d, E, ws, s);
}

moe_status launch_route(const void* x, int x_dtype, const float* Wg, const void* Wg_split, const float* logit_offset,
                        const float* select_bias, int T, int d, int E, int k, int score, int renormalize,
                        float scale, float* logits, int32_t* topk_idx, float* topk_gate, void* ws, cudaStream_t s) {
  if (T == 0) return MOE_OK;
  const bool bias = select_bias != nullptr;
  if (tc_router_applies(x_dtype, T, d, E)) {
    const void* W3 = nullptr;
    moe_status st = router_weight(Wg, Wg_split, d, E, ws, &W3, s);
    if (st != MOE_OK) return st;
    // top-k and gates in the GEMM's epilogue, except for softmax scores with a selection
    // bias, whose keys need the whole row's normaliser before any comparison
    const bool fuse = !(score == MOE_SCORE_SOFTMAX && bias);
    st = launch_router_tc(x, T, d, E, W3, logit_offset, logits, fuse ? k : 0, select_bias, score, renormalize, scale,
                          topk_idx, topk_gate, s);
    if (st != MOE_ERR_UNSUPPORTED) {
      if (st != MOE_OK || fuse) return st;
      return run_topk_any(bias, logits, 1, (long long)T * E, logit_offset, select_bias, T, E, k, score, renormalize,
                          scale, logits, 0, topk_idx, topk_gate, s);
    }
  }
  LogitsPlan p = plan_logits(T, d, E);
  float* partial = p.nsplit > 1 ? static_cast<float*>(ws) : logits;
  const long long split_stride = (long long)T * E;
  moe_status st = x_dtype == MOE_F32
                      ? dispatch_logits<float>(x, Wg, logit_offset, T, d, E, p, partial, split_stride, s)
                      : dispatch_logits<__nv_bfloat16>(x, Wg, logit_offset, T, d, E, p, partial, split_stride, s);
  if (st != MOE_OK) return st;
  return run_topk_any(bias, partial, p.nsplit, split_stride, logit_offset, select_bias, T, E, k, score, renormalize,
                      scale, logits, p.nsplit > 1 ? 1 : 0, topk_idx, topk_gate, s);
}

size_t router_logits_workspace_bytes(int T, int d, int E, bool prepared) {
  if (T <= 0 || E <= 0 || d <= 0 || prepared) return 0;
  // any batch of at least 256 tokens takes the tensor-core path
  return (T >= 256 && tc_router_applies(MOE_BF16, T, d, E)) ? router_weight_bytes(d, E) : 0;
}

// The router alone: the tensor-core GEMM where it applies, else the SIMT GEMM in one
// pass over d (no split, so it writes the logits with their offset itself).
moe_status launch_router_logits(const void* x, int x_dtype, const float* Wg, const void* Wg_split,
                                const float* logit_offset, int T, int d, int E, float* logits, void* ws,
                                cudaStream_t s) {
  if (T == 0) return MOE_OK;
  if (tc_router_applies(x_dtype, T, d, E)) {
    const void* W3 = nullptr;
    moe_status st = router_weight(Wg, Wg_split, d, E, ws, &W3, s);
    if (st != MOE_OK) return st;
    st = launch_router_tc(x, T, d, E, W3, logit_offset, logits, 0, nullptr, 0, 0, 1.f, nullptr, nullptr, s);
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
  return run_topk_any(false, H, 1, n, nullptr, nullptr, T, E, k, MOE_SCORE_SOFTMAX, 1, scale, H, 0, topk_idx,
                      topk_gate, s);
}

}  // namespace moe
