// Router on the 5th-generation tensor cores: fp32-faithful logits from a bf16 x and an
// fp32 W_g, with the top-k selection and the gates computed in the GEMM's epilogue.
//
// Sources: "Hugging Face 图解 Mixture of Experts（MoE）原理、训练与推理权衡", section
// "什么是稀疏性？" (G_sigma(x) = Softmax(x . W_g), KeepTopK, G(x) = Softmax(KeepTopK(H, k)))
// and section "Switch Transformer" (the router stays in full precision); handbook news
// post (hub.geekagi.cn), "真正难在三个环节" item 1 (FP32 routing) and item 2 (loss-free
// selection bias); handbook digest (agihunt.info), "已确认" (sqrt(softplus) scores, a
// routing scale near sqrt(k)).
//
// Exact operand split.  x is bf16; W_g is fp32.  W_g = hi + mid + lo with
//   hi = bf16(w), mid = bf16(w - hi), lo = bf16(w - hi - mid)
// (each subtraction is exact in fp32 and the three terms carry w's 24 significant bits),
// so every product x * term is exact in fp32 and the MMAs add exact products with fp32
// accumulation: the logits are fp32 sums of the exact x * W_g products.  The split is
// done once when the weights are loaded (moe_prepare_router_weight), not per forward.
//
// Prepared weight layout: experts are cut into n_tiles tiles of NE experts (NE a multiple
// of 32, at most 256; n_tiles = ceil(E / 256)); tile j owns experts j*NE .. j*NE+NE-1 and
// the rows [3 j NE, 3 j NE + NE) = hi, then NE rows of mid, then NE rows of lo of the
// K-major bf16 matrix W3 [3 n_tiles NE, d].  Rows of experts past E are zero.
//
// GEMM: CTA pairs (cta_group::2), 256 tokens x NE experts per tile.  Per 64-wide k-block
// each CTA stages 128 rows of x and NE/2 rows of each of the three terms (TMA, 128-byte
// swizzle); the even CTA issues, per 16-wide k step, three M=256 x N=NE MMAs (hi, mid,
// lo) into ONE fp32 TMEM accumulator.  Two accumulators (2 x 256 columns) let the
// epilogue of one tile overlap the mainloop of the next.
//
// Epilogue (thread = token row, the TMEM lane): logit = acc + offset, written to the
// logits matrix through a shared-memory turn-around (whole 128-byte lines per store).
// With the top-k fused (KMAX > 0), each thread also keeps its token's best KMAX
// candidates in registers as it streams its row's experts; one CTA pair walks all
// expert tiles of its 256 tokens in order, so after the last tile the selection is
// complete: it writes topk_idx and the gates.  Selection keys: the logit itself (no
// selection bias), or score(l) + bias evaluated in fp64; ties go to the lower expert
// index (experts arrive in increasing index order and only a strictly larger key moves
// ahead).  Gates: softmax over the kept logits from fp64 differences to their maximum;
// or the sigmoid / sqrt(softplus) scores renormalised over the kept ones (fp32); times
// the scale.  Without renormalisation the softmax gate is the full softmax probability
// (running max and fp64 normaliser over all experts).
//
// Every barrier wait is bounded (MOE_DEVERR_PIPE_TIMEOUT, then an orderly exit).  No
// load uses cluster multicast.
#include "common.cuh"
#include "tc_prims.cuh"

#include <float.h>
#include <type_traits>
#include <stdlib.h>
#include <string.h>

namespace moe {
namespace {

constexpr int kRThreads = 192;          // warp 0 TMA, warp 1 MMA, warps 2-5 epilogue
constexpr int RBM = 128;                // token rows per CTA (a pair covers 256)
constexpr int kRAStage = RBM * BK * 2;  // 16 KB of x per stage
constexpr int kRMaxStages = 8;
constexpr uint32_t kRTmemCols = 512;    // two accumulators of up to 256 columns
constexpr int kRSmemLimit = 232448;     // 227 KB opt-in maximum per CTA

struct RLayout {
  int stage_bytes, stages, bars, misc, staging, end;
};

__host__ __device__ inline RLayout router_layout(int NE, int stages) {
  RLayout l;
  l.stage_bytes = kRAStage + 3 * (NE / 2) * BK * 2;   // x rows + three term blocks
  l.stages = stages;
  l.bars = stages * l.stage_bytes;
  l.misc = l.bars + (2 * kRMaxStages + 5) * 8;
  l.staging = (l.misc + 16 + 127) / 128 * 128;
  l.end = l.staging + 4 * kStageWarpBytes;
  return l;
}

// The CTA pair's i-th work unit: (row tile, expert tile).  Fused top-k: one pair takes
// whole row tiles and walks their expert tiles in order.  Logits only: units are spread
// expert-tile fastest over the pairs (the consecutive pairs share each slice of x).
__device__ __forceinline__ bool unit_of(bool fused, int i, int cid, int ncl, int n_rt, int n_tiles, int* rt, int* j) {
  if (fused) {
    *rt = cid + (i / n_tiles) * ncl;
    *j = i - (i / n_tiles) * n_tiles;
    return *rt < n_rt;
  }
  const long long u = (long long)cid + (long long)i * ncl;
  if (u >= (long long)n_rt * n_tiles) return false;
  *rt = (int)(u / n_tiles);
  *j = (int)(u - (long long)(*rt) * n_tiles);
  return true;
}

__device__ __forceinline__ double score_d(double l, int score) {
  if (score == MOE_SCORE_SIGMOID) return 1.0 / (1.0 + exp(-l));
  return sqrt(fmax(l, 0.0) + log1p(exp(-fabs(l))));   // MOE_SCORE_SQRT_SOFTPLUS
}
__device__ __forceinline__ float score_f(float l, int score) {
  if (score == MOE_SCORE_SIGMOID) return 1.f / (1.f + expf(-l));
  return sqrtf(fmaxf(l, 0.f) + log1pf(expf(-fabsf(l))));
}

// Order-preserving 32 / 64-bit images of float / double (larger image = larger value,
// -0 and +0 equal); 0 is below the image of every value, -inf included, and marks an
// empty candidate slot.
__device__ __forceinline__ uint32_t ord32(float v) {
  const uint32_t u = __float_as_uint(v + 0.0f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float unord32(uint32_t o) {
  return __uint_as_float((o & 0x80000000u) ? (o & 0x7fffffffu) : ~o);
}
__device__ __forceinline__ uint64_t ord64(double v) {
  const uint64_t u = (uint64_t)__double_as_longlong(v + 0.0);
  return (u >> 63) ? ~u : (u | (1ull << 63));
}

// A thread's running top-KMAX, sorted by key descending.  No bias: key = ord32(logit)
// (NaN as -inf), the logit recoverable from the key; candidates arrive in increasing
// expert order and only a strictly larger key moves ahead of an entry, so among equal
// logits the lower index stays ahead.  Bias: key = ord64(score + bias), the logit kept
// beside it.  Key 0 is below every candidate's key and marks an empty slot.
template <int KMAX, bool BIAS>
struct TopK {
  using Key = typename std::conditional<BIAS, uint64_t, uint32_t>::type;
  Key key[KMAX];
  int idx[KMAX];
  float lg[BIAS ? KMAX : 1];
  float M;      // running maximum logit (non-renormalised softmax gates)
  double Z;     // running sum of exp(l - M) in fp64

  __device__ __forceinline__ void reset() {
#pragma unroll
    for (int i = 0; i < KMAX; ++i) {
      key[i] = 0;
      idx[i] = 0;
      if (BIAS) lg[i] = 0.f;
    }
    M = -INFINITY;
    Z = 0.0;
  }
  // Insertion into the sorted list, all positions at once: compare the candidate with
  // every entry (independent compares), then each entry at or after the insertion point
  // takes its predecessor's value, the one at the insertion point the candidate.  Same
  // result as bubbling the candidate down, without a chain of k dependent steps (the
  // epilogue runs one warp per SM sub-partition, so dependent latency is not hidden).
  __device__ __forceinline__ void insert(Key kc, int e, float l) {
    if (!(kc > key[KMAX - 1])) return;
    bool up[KMAX];
#pragma unroll
    for (int i = 0; i < KMAX; ++i) up[i] = kc > key[i];
#pragma unroll
    for (int i = KMAX - 1; i >= 1; --i) {                  // descending: entry i - 1 is still old
      key[i] = up[i] ? (up[i - 1] ? key[i - 1] : kc) : key[i];
      idx[i] = up[i] ? (up[i - 1] ? idx[i - 1] : e) : idx[i];
      if (BIAS) lg[i] = up[i] ? (up[i - 1] ? lg[i - 1] : l) : lg[i];
    }
    key[0] = up[0] ? kc : key[0];
    idx[0] = up[0] ? e : idx[0];
    if (BIAS) lg[0] = up[0] ? l : lg[0];
  }
  __device__ __forceinline__ int index_of(int i) const { return idx[i]; }
  __device__ __forceinline__ float logit_of(int i) const {
    if constexpr (BIAS) return lg[i];
    else return unord32(key[i]);
  }
};

// The no-bias selection key: the logit's ordered image, NaN ranking as -inf.
__device__ __forceinline__ uint32_t plain_key(float l) { return ord32((l == l) ? l : -INFINITY); }

template <int KMAX, bool BIAS>
__device__ __forceinline__ void topk_norm(TopK<KMAX, BIAS>& st, float l) {
  if (l == l && l != -INFINITY) {                  // running normaliser of the full softmax
    if (l > st.M) {
      st.Z = st.Z * exp((double)st.M - (double)l) + 1.0;
      st.M = l;
    } else {
      st.Z += exp((double)l - (double)st.M);
    }
  }
}

template <int KMAX, bool BIAS>
__device__ __forceinline__ void topk_consider(TopK<KMAX, BIAS>& st, float l, int e, int score, bool full_softmax,
                                              const float* __restrict__ sel_bias) {
  if (full_softmax) topk_norm<KMAX, BIAS>(st, l);
  if (BIAS) {
    double kd = -INFINITY;
    if (l == l) {
      kd = score_d((double)l, score) + (double)__ldg(sel_bias + e);
      if (kd != kd) kd = -INFINITY;
    }
    st.insert(ord64(kd), e, l);
  } else {
    st.insert(plain_key(l), e, l);
  }
}

// Gates of the selected experts for one token, written by the thread that owns it.  The
// kept logits go to the thread's scratch row (KMAX floats of shared memory) and the gates
// are computed in rolled loops over it: each pair may run this once, from a cold
// instruction cache, so one copy of the fp64 exp code instead of 2 KMAX inlined ones.
// Same operations in the same order as a direct evaluation.
template <int KMAX, bool BIAS>
__device__ __forceinline__ void topk_write(const TopK<KMAX, BIAS>& st, long long t, int k, int score, int renorm,
                                           float scale, float* scratch, int32_t* __restrict__ topk_idx,
                                           float* __restrict__ topk_gate) {
#pragma unroll
  for (int j = 0; j < KMAX; ++j) {
    if (j < k) {
      topk_idx[t * k + j] = st.index_of(j);
      scratch[j] = st.logit_of(j);
    }
  }
  float* g_out = topk_gate + t * k;
  if (score == MOE_SCORE_SOFTMAX) {
    if (renorm) {
      // softmax over the kept logits; the first entry holds the largest logit (no bias)
      const double m = (double)scratch[0];
      double z = 0.0;
#pragma unroll 1
      for (int j = 0; j < k; ++j) z += exp((double)scratch[j] - m);
#pragma unroll 1
      for (int j = 0; j < k; ++j) g_out[j] = (float)(exp((double)scratch[j] - m) / z) * scale;
    } else {
#pragma unroll 1
      for (int j = 0; j < k; ++j) g_out[j] = (float)(exp((double)scratch[j] - (double)st.M) / st.Z) * scale;
    }
  } else {
    float s = 0.f;
#pragma unroll 1
    for (int j = 0; j < k; ++j) s += score_f(scratch[j], score);
#pragma unroll 1
    for (int j = 0; j < k; ++j) {
      const float g = score_f(scratch[j], score);
      g_out[j] = (renorm ? g / s : g) * scale;
    }
  }
}

// SIDE: the three terms side by side in one MMA of N = 3 NE (NE <= 64), summed in the
// epilogue, instead of three MMAs of N = NE into one accumulator: at small NE, four wide
// MMAs per k-block instead of twelve narrow ones.  The prepared weight is the same (a
// tile's hi, mid, lo rows are contiguous); each CTA loads its 3 NE / 2 rows in one box.
template <int KMAX, bool BIAS, bool SIDE>
__global__ void __launch_bounds__(kRThreads, 1)
router_tc_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW, int T, int d,
                 int E, int NE, int n_tiles, int stages, const float* __restrict__ logit_offset,
                 float* __restrict__ logits, const float* __restrict__ sel_bias, int k, int score, int renorm,
                 float scale, int32_t* __restrict__ topk_idx, float* __restrict__ topk_gate, int* err) {
  constexpr bool kFused = KMAX > 0;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  const RLayout Ly = router_layout(NE, stages);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Ly.misc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Ly.misc + 4);
  const uint32_t rank = cluster_ctarank();
  const int cid = (int)(blockIdx.x >> 1), ncl = (int)(gridDim.x >> 1);
  const int n_rt = (T + 2 * RBM - 1) / (2 * RBM);
  const int KB = (d + BK - 1) / BK;
  const int half = NE / 2;                       // term rows per CTA
  const uint32_t term_bytes = (uint32_t)half * BK * 2;

  const uint32_t bar_full = sb + Ly.bars;
  const uint32_t bar_empty = bar_full + 8 * kRMaxStages;
  const uint32_t bar_tfull = bar_empty + 8 * kRMaxStages;
  const uint32_t bar_tempty = bar_tfull + 16;
  const uint32_t bar_fin = bar_tempty + 16;
  auto a_stage = [&](int s) { return sb + (uint32_t)(s * Ly.stage_bytes); };
  auto b_stage = [&](int s, int t) { return sb + (uint32_t)(s * Ly.stage_bytes + kRAStage) + (uint32_t)t * term_bytes; };

  if (threadIdx.x == 0) {
    for (int s = 0; s < stages; ++s) {
      mbar_init(bar_full + 8 * s, 1);
      mbar_init(bar_empty + 8 * s, 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(bar_tfull + 8 * a, 1);
      mbar_init(bar_tempty + 8 * a, 2 * 128);
    }
    mbar_init(bar_fin, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(kRTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer (both CTAs)
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued = 0, last_par = 0;                 // per stage: a load issued, its phase parity
      bool ok = true;
      int rt, j;
      for (int i = 0; ok && unit_of(kFused, i, cid, ncl, n_rt, n_tiles, &rt, &j); ++i) {
        const int a_row = rt * 2 * RBM + (int)rank * RBM;
        const int b_row = j * 3 * NE + (int)rank * half;
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait(bar_empty + 8 * stage, phase ^ 1u, abort_flag, err)) { ok = false; break; }
          if (rank == 0) mbar_expect_tx(bar_full + 8 * stage, 2u * (uint32_t)(kRAStage + 3 * term_bytes));
          const uint32_t full_c = map_to_rank(bar_full + 8 * stage, 0);
          tma_load_2d_pair(a_stage(stage), &tmX, full_c, kb * BK, a_row);
          if (SIDE) {
            tma_load_2d_pair(b_stage(stage, 0), &tmW, full_c, kb * BK, j * 3 * NE + (int)rank * (3 * half));
          } else {
#pragma unroll
            for (int t = 0; t < 3; ++t) tma_load_2d_pair(b_stage(stage, t), &tmW, full_c, kb * BK, b_row + t * NE);
          }
          issued |= 1u << stage;
          last_par = (last_par & ~(1u << stage)) | (phase << stage);
          if (++stage == stages) { stage = 0; phase ^= 1u; }
        }
      }
      if (!ok && rank == 0) {
        for (int s = 0; s < stages; ++s)
          if ((issued >> s) & 1u) mbar_wait_drain(bar_full + 8 * s, (last_par >> s) & 1u, err);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (even CTA)
    if (lane == 0 && rank == 0) {
      const uint32_t idesc = make_idesc(2 * RBM, SIDE ? 3 * NE : NE);
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      int rt, j;
      for (int it = 0; ok && unit_of(kFused, it, cid, ncl, n_rt, n_tiles, &rt, &j); ++it) {
        const int acc = it & 1;
        const uint32_t acc_phase = (uint32_t)(it >> 1) & 1u;
        if (!mbar_wait(bar_tempty + 8 * acc, acc_phase ^ 1u, abort_flag, err)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * 256);
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait(bar_full + 8 * stage, phase, abort_flag, err)) { ok = false; break; }
          tc_fence_after();
          const uint64_t adesc = sw128_desc(a_stage(stage));
          uint64_t bdesc[3];
#pragma unroll
          for (int t = 0; t < 3; ++t) bdesc[t] = sw128_desc(b_stage(stage, t));
#pragma unroll
          for (int kk = 0; kk < BK / UMMA_K; ++kk) {
            if (SIDE) {                   // columns [0, NE) hi, [NE, 2 NE) mid, [2 NE, 3 NE) lo
              umma_bf16_pair(d_tmem, adesc + 2 * kk, bdesc[0] + 2 * kk, idesc, (kb | kk) != 0 ? 1u : 0u);
            } else {
#pragma unroll
              for (int t = 0; t < 3; ++t)   // +32 bytes along K per step (>> 4 = 2)
                umma_bf16_pair(d_tmem, adesc + 2 * kk, bdesc[t] + 2 * kk, idesc, (kb | kk | t) != 0 ? 1u : 0u);
            }
          }
          umma_commit_pair_both(bar_empty + 8 * stage);
          if (++stage == stages) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        umma_commit_pair_both(bar_tfull + 8 * acc);
      }
      umma_commit_pair(bar_fin);
      mbar_wait_drain(bar_fin, 0, err);
    }
  } else {
    // ------------------------------------------------------------ epilogue (both CTAs)
    const int q = warp & 3;                                  // TMEM lane quarter of this warp
    uint8_t* stage = smem + Ly.staging + (warp - 2) * kStageWarpBytes;
    const bool full_softmax = kFused && score == MOE_SCORE_SOFTMAX && !renorm;
    TopK<(kFused ? KMAX : 1), BIAS> st;
    st.reset();
    int rt, j;
    for (int it = 0; unit_of(kFused, it, cid, ncl, n_rt, n_tiles, &rt, &j); ++it) {
      const int acc = it & 1;
      const uint32_t acc_phase = (uint32_t)(it >> 1) & 1u;
      const bool got = mbar_wait(bar_tfull + 8 * acc, acc_phase, abort_flag, err);
      if (!__all_sync(0xffffffffu, got)) break;
      __syncwarp();
      tc_fence_after();
      const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * 256);
      const long long row0 = (long long)rt * 2 * RBM + (int)rank * RBM + q * 32;   // this warp's first row
      const int wrows = (int)min(32LL, max(0LL, (long long)T - row0));
      const int e0 = j * NE;
#pragma unroll 1
      for (int c = 0; c < NE / 32; ++c) {
        uint32_t v[32];
        float lv[32];
        tmem_ld32(taddr + c * 32, v);
        if (SIDE) {
          // (hi + mid) + lo, one 32-column block at a time (fewer live registers)
          tmem_wait_ld();
          tmem_regs_ready(v);
#pragma unroll
          for (int i = 0; i < 32; ++i) lv[i] = __uint_as_float(v[i]);
#pragma unroll
          for (int t = 1; t < 3; ++t) {
            tmem_ld32(taddr + t * NE + c * 32, v);
            tmem_wait_ld();
            tmem_regs_ready(v);
#pragma unroll
            for (int i = 0; i < 32; ++i) lv[i] += __uint_as_float(v[i]);
          }
        } else {
          tmem_wait_ld();
          tmem_regs_ready(v);
#pragma unroll
          for (int i = 0; i < 32; ++i) lv[i] = __uint_as_float(v[i]);
        }
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const int e = e0 + c * 32 + i;
          const float off = (logit_offset && e < E) ? __ldg(logit_offset + e) : 0.f;
          lv[i] += off;
        }
        stage_store32<float>(stage, lv, lane, logits, row0, wrows, E, e0 + c * 32, E);
        if constexpr (kFused) {
          // the token's 32 logits are still in its staging row: a rolled loop over them
          // keeps the selection code small (a pair may run this epilogue only once, from
          // a cold instruction cache)
          const float4* mine = reinterpret_cast<const float4*>(stage + lane * kStagePitchF32);
          const int ec = e0 + c * 32;
          if constexpr (!BIAS) {
            // Two passes.  First every candidate is tested against the thread's current
            // k-th key (and feeds the full-softmax normaliser); then the warp inserts only
            // the candidates that passed, lowest position first, as many rounds as the
            // busiest lane needs.  The k-th key only grows, so a candidate that fails the
            // test now would be rejected later too: the same selection as inserting every
            // candidate in turn, without running the insertion wherever any one lane of
            // the warp needs it.
            // Every entry of the list has a lower index than this chunk's candidates, so a
            // candidate's key exceeds the k-th key exactly when its logit (NaN as -inf)
            // exceeds the k-th logit, or the list still has a free slot (key 0).
            uint32_t pass = 0;
            const uint32_t klast = st.key[KMAX - 1];
            const bool open = klast == 0u;
            const float thr = unord32(klast);
#pragma unroll 2
            for (int qd = 0; qd < 8; ++qd) {
              const float4 f = mine[qd];
              const float fv[4] = {f.x, f.y, f.z, f.w};
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                const int e = ec + 4 * qd + i;
                if (e < E) {
                  if (full_softmax) topk_norm<KMAX, BIAS>(st, fv[i]);
                  if (open || (fv[i] == fv[i] && fv[i] > thr)) pass |= 1u << (4 * qd + i);
                }
              }
            }
            const float* row = reinterpret_cast<const float*>(mine);
#pragma unroll 1
            while (__any_sync(0xffffffffu, pass != 0)) {
              if (pass) {
                const int p = __ffs(pass) - 1;
                pass &= pass - 1;
                const float l = row[p];
                st.insert(plain_key(l), ec + p, l);
              }
            }
          } else {
#pragma unroll 1
            for (int qd = 0; qd < 8; ++qd) {
              const float4 f = mine[qd];
              const float fv[4] = {f.x, f.y, f.z, f.w};
              const int eb = ec + 4 * qd;
#pragma unroll
              for (int i = 0; i < 4; ++i)
                if (eb + i < E) topk_consider<KMAX, BIAS>(st, fv[i], eb + i, score, full_softmax, sel_bias);
            }
          }
        }
      }
      tc_fence_before();
      mbar_arrive_remote(map_to_rank(bar_tempty + 8 * acc, 0));
      if constexpr (kFused) {
        if (j == n_tiles - 1) {
          if (lane < wrows)
            topk_write<KMAX, BIAS>(st, row0 + lane, k, score, renorm, scale,
                                   reinterpret_cast<float*>(stage + lane * kStagePitchF32), topk_idx, topk_gate);
          st.reset();
        }
      }
    }
  }

  __syncthreads();
  cluster_sync();                                           // no remote arrive after a CTA exits
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(kRTmemCols) : "memory");
  }
}

// Prepared weight: W3[(3 j + t) NE + r][c] = term t of W_g[c][j NE + r] (zero past E).
// One 32 x 32 shared-memory transpose per block.
__global__ void __launch_bounds__(256)
prepare_router_weight_kernel(const float* __restrict__ Wg, int d, int E, int NE, int E_pad,
                             __nv_bfloat16* __restrict__ W3) {
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
    if (e >= E_pad || c >= d) continue;
    const float w = tile[tx][ty + 8 * i];
    const __nv_bfloat16 hi = __float2bfloat16_rn(w);
    const float r1 = w - __bfloat162float(hi);
    const __nv_bfloat16 mid = __float2bfloat16_rn(r1);
    const __nv_bfloat16 lo = __float2bfloat16_rn(r1 - __bfloat162float(mid));
    const int jt = e / NE, r = e - jt * NE;
    const long long base = (long long)jt * 3 * NE + r;
    W3[base * d + c] = hi;
    W3[(base + NE) * d + c] = mid;
    W3[(base + 2 * NE) * d + c] = lo;
  }
}

template <int KMAX, bool BIAS, bool SIDE>
moe_status launch_router_kernel(const CUtensorMap& mx, const CUtensorMap& mw, int T, int d, int E, int NE,
                                int n_tiles, const float* off, float* logits, const float* sel_bias, int k,
                                int score, int renorm, float scale, int32_t* idx, float* gate, cudaStream_t s) {
  static std::atomic<int> configured[kMaxDevices];
  moe_status st = ensure_smem_limit(configured, router_tc_kernel<KMAX, BIAS, SIDE>, (size_t)kRSmemLimit);
  if (st != MOE_OK) return st;
  // as many stages as fit next to the epilogue staging
  int stages = kRMaxStages;
  while (stages > 2 && router_layout(NE, stages).end + 1024 > kRSmemLimit) --stages;
  const size_t smem = (size_t)router_layout(NE, stages).end + 1024;
  const int n_rt = (T + 2 * RBM - 1) / (2 * RBM);
  const long long units = KMAX > 0 ? n_rt : (long long)n_rt * n_tiles;
  int pairs = num_sms() / 2;
  if (units < pairs) pairs = (int)units;
  if (pairs < 1) pairs = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * pairs, 1, 1);
  cfg.blockDim = dim3(kRThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cuda_status(cudaLaunchKernelEx(&cfg, router_tc_kernel<KMAX, BIAS, SIDE>, mx, mw, T, d, E, NE, n_tiles, stages, off,
                                        logits, sel_bias, k, score, renorm, scale, idx, gate, err_ptr()));
}

}  // namespace

// The side-by-side layout applies while the three terms fit one MMA (3 NE <= 256 columns,
// 3 NE / 2 rows per CTA in one TMA box); MOE_B200_ROUTER_TERMS=stacked|side forces one
// (for measuring one against the other).
bool router_side_by_side(int NE) {
  const char* v = getenv("MOE_B200_ROUTER_TERMS");
  if (v && strcmp(v, "stacked") == 0) return false;
  if (v && strcmp(v, "side") == 0) return NE <= 64;
  return NE <= 64;
}

RouterGeom router_geom(int E) {
  RouterGeom g;
  g.n_tiles = (E + kRouterMaxNE - 1) / kRouterMaxNE;
  if (g.n_tiles < 1) g.n_tiles = 1;
  const int per = (E + g.n_tiles - 1) / g.n_tiles;
  g.NE = (per + 31) / 32 * 32;
  return g;
}

size_t router_weight_bytes(int d, int E) {
  if (d < BK || E < 1 || E % 4 != 0) return 0;
  const RouterGeom g = router_geom(E);
  return (size_t)g.n_tiles * 3 * g.NE * (size_t)d * 2;
}

bool tc_router_applies(int x_dtype, int T, int d, int E) {
  return x_dtype == MOE_BF16 && T >= 2 * RBM && d >= BK && d % 8 == 0 && E % 4 == 0;
}

moe_status launch_prepare_router_weight(const float* Wg, int d, int E, void* W3, cudaStream_t s) {
  const RouterGeom g = router_geom(E);
  const int E_pad = g.n_tiles * g.NE;
  dim3 grid((d + 31) / 32, (E_pad + 31) / 32);
  prepare_router_weight_kernel<<<grid, 256, 0, s>>>(Wg, d, E, g.NE, E_pad, static_cast<__nv_bfloat16*>(W3));
  return check_launch();
}

// Logits (+ offset) and, when fuse_k > 0, the top-k and gates of every token.  The caller
// has checked tc_router_applies and holds the prepared weight W3.  Returns
// MOE_ERR_UNSUPPORTED when a tensor map cannot be encoded.
moe_status launch_router_tc(const void* x, int T, int d, int E, const void* W3, const float* logit_offset,
                            float* logits, int fuse_k, const float* sel_bias, int score, int renorm, float scale,
                            int32_t* topk_idx, float* topk_gate, cudaStream_t s) {
  if (T == 0) return MOE_OK;
  const RouterGeom g = router_geom(E);
  CUtensorMap mx, mw;
  if (!make_map(&mx, x, (unsigned long long)T, d, RBM)) return MOE_ERR_UNSUPPORTED;
  const unsigned box = router_side_by_side(g.NE) ? 3 * g.NE / 2 : g.NE / 2;
  if (!make_map(&mw, W3, (unsigned long long)g.n_tiles * 3 * g.NE, d, box)) return MOE_ERR_UNSUPPORTED;
  const bool bias = sel_bias != nullptr;
  // NE <= 64: the three terms side by side (one MMA of N = 3 NE per k step)
  const bool side = router_side_by_side(g.NE);
#define MOE_RT(KM, B)                                                                                            \
  return side ? launch_router_kernel<KM, B, true>(mx, mw, T, d, E, g.NE, g.n_tiles, logit_offset, logits,       \
                                                  sel_bias, fuse_k, score, renorm, scale, topk_idx, topk_gate, s) \
              : launch_router_kernel<KM, B, false>(mx, mw, T, d, E, g.NE, g.n_tiles, logit_offset, logits,      \
                                                   sel_bias, fuse_k, score, renorm, scale, topk_idx, topk_gate, s)
  if (fuse_k <= 0) MOE_RT(0, false);
  if (fuse_k <= 8) {
    if (bias) MOE_RT(8, true);
    MOE_RT(8, false);
  }
  if (fuse_k <= 16) {
    if (bias) MOE_RT(16, true);
    MOE_RT(16, false);
  }
  if (bias) MOE_RT(32, true);
  MOE_RT(32, false);
#undef MOE_RT
}

}  // namespace moe
