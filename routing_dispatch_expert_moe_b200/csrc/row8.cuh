// Eight consecutive elements of a row as one or two 16-byte vectors, in the row's storage
// type (bf16 or fp32), with the fp32 accumulate and the store used by the combines.
#pragma once

#include "common.cuh"

namespace moe {

// Eight consecutive elements of a row, in the row's storage type.
template <typename T>
struct Row8;
template <>
struct Row8<__nv_bfloat16> {
  uint4 a;
  __device__ __forceinline__ void load(const void* base, long long e) {
    a = ld_stream(reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(base) + e));
  }
  __device__ __forceinline__ void add(float* acc, float g, bool scale) const {
    float f[8];
    unpack8(a, f);
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = scale ? fmaf(g, f[i], acc[i]) : acc[i] + f[i];
  }
};
template <>
struct Row8<float> {
  uint4 a, b;
  __device__ __forceinline__ void load(const void* base, long long e) {
    const uint4* p = reinterpret_cast<const uint4*>(static_cast<const float*>(base) + e);
    a = ld_stream(p);
    b = ld_stream(p + 1);
  }
  __device__ __forceinline__ void add(float* acc, float g, bool scale) const {
    const float f[8] = {__uint_as_float(a.x), __uint_as_float(a.y), __uint_as_float(a.z), __uint_as_float(a.w),
                        __uint_as_float(b.x), __uint_as_float(b.y), __uint_as_float(b.z), __uint_as_float(b.w)};
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = scale ? fmaf(g, f[i], acc[i]) : acc[i] + f[i];
  }
};

template <typename T>
__device__ __forceinline__ void store8(void* base, long long e, const float* f);
template <>
__device__ __forceinline__ void store8<__nv_bfloat16>(void* base, long long e, const float* f) {
  *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(base) + e) = pack8(f);
}
template <>
__device__ __forceinline__ void store8<float>(void* base, long long e, const float* f) {
  float4* p = reinterpret_cast<float4*>(static_cast<float*>(base) + e);
  p[0] = make_float4(f[0], f[1], f[2], f[3]);
  p[1] = make_float4(f[4], f[5], f[6], f[7]);
}

}  // namespace moe
