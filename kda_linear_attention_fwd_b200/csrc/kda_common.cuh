// Shared device helpers for the KDA kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#define KDA_DEVICE __device__ __forceinline__

namespace kda {

// Element-type traits: loads widen to fp32, stores round to nearest even.
template <typename T> struct Elem;
template <> struct Elem<float> {
    static KDA_DEVICE float load(const float *p) { return *p; }
    static KDA_DEVICE void store(float *p, float x) { *p = x; }
};
template <> struct Elem<__nv_bfloat16> {
    static KDA_DEVICE float load(const __nv_bfloat16 *p) { return __bfloat162float(*p); }
    static KDA_DEVICE void store(__nv_bfloat16 *p, float x) { *p = __float2bfloat16_rn(x); }
};

template <typename T> KDA_DEVICE float ld(const T *p) { return Elem<T>::load(p); }
template <typename T> KDA_DEVICE void st(T *p, float x) { Elem<T>::store(p, x); }

// Streamed (evict-first) global accesses for data touched exactly once.
KDA_DEVICE float4 ld_stream(const float4 *p) { return __ldcs(p); }
KDA_DEVICE void st_stream(float4 *p, float4 v) { __stcs(p, v); }

KDA_DEVICE float warp_sum(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

}  // namespace kda
