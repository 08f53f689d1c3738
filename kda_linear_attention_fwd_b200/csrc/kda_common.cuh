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

// Bits of the flags word of the extended entry points (bit 0 is the
// qk_l2norm switch of the plain ones).
constexpr int FLAG_L2NORM = 1;       // q, k divided by their L2 norms (+1e-6 under the root)
constexpr int FLAG_BETA_LOGITS = 2;  // beta given as logits: sigmoid applied on load
constexpr int FLAG_GATE_LOGITS = 4;  // gate given as logits: sigmoid applied on load
constexpr int FLAG_CLAMP_G = 8;      // log-decay clamped from below at ln(0.0067)
constexpr int FLAG_ALL = 15;

// ln(0.0067): the smallest single-step retention of the forget gate
constexpr float kLogDecayFloor = -5.005647752585217f;

KDA_DEVICE float sigmoid_f(float x) { return 1.f / (1.f + __expf(-x)); }
KDA_DEVICE float beta_in(float x, int flags) { return (flags & FLAG_BETA_LOGITS) ? sigmoid_f(x) : x; }
KDA_DEVICE float gate_in(float x, int flags) { return (flags & FLAG_GATE_LOGITS) ? sigmoid_f(x) : x; }
KDA_DEVICE float g_in(float x, int flags) { return (flags & FLAG_CLAMP_G) ? fmaxf(x, kLogDecayFloor) : x; }

KDA_DEVICE float warp_sum(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

}  // namespace kda
