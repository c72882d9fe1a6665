// common.cuh -- small device helpers shared by the CKDA kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "ckda.h"

namespace ckda {

constexpr float kL2Eps = 1e-6f;  // x / sqrt(sum x^2 + eps), per head
constexpr int kMaxHalfDim = 64;  // dk <= 128

// Rotary frequencies omega_i = theta^(-2i/rot_dims), computed on the host and passed by value
// (so that concurrent calls with different bases never share state), each as a 0.64 fixed-point
// count of turns per position: turns[i] = round(2^64 frac(omega_i / 2 pi)).
struct RopeParams {
    unsigned long long turns[kMaxHalfDim];   // i < rot_dims / 2 (0 beyond)
    int enabled;     // rope_theta > 0
    int convention;  // 0 half-split, 1 interleaved (both over the first rot_dims channels)
    int rot_dims;    // channels rotated: dk, or dk / 2 (the rest carried through)
};

// sin and cos of the position angle p * omega for a frequency given as fixed-point turns per
// position (RopeParams::turns).  p * turns mod 2^64 is the fractional turn count of p * omega,
// exact in integer arithmetic at any position (an fp32 product p * omega would carry ~4e-3 rad
// of error at 64k tokens); its top 32 bits, read as a signed fraction of a turn, give the angle
// reduced to [-pi, pi) to within 2^-32 of a turn.  On that argument the fast hardware sin/cos is
// accurate to a few 1e-7 (absolute), far below the bf16 resolution of the rotated activations.
__device__ __forceinline__ void rope_sincos(long long p, unsigned long long turns, float* s,
                                            float* c) {
    const unsigned long long t = (unsigned long long)p * turns;
    const float r = (float)(int)(unsigned)(t >> 32) * 1.4629180792671596e-09f;   // 2 pi / 2^32
    __sincosf(r, s, c);
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

// Sum over aligned groups of G lanes (G a power of two <= 32).
template <int G>
__device__ __forceinline__ float group_sum(float x) {
#pragma unroll
    for (int o = G / 2; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

// ---- element loads / stores -------------------------------------------------------------
// Load N consecutive elements (16 bytes total) as floats.
template <typename T, int N>
struct Vec16;

template <>
struct Vec16<float, 4> {
    __device__ __forceinline__ static void load(const float* p, float* x) {
        float4 v = *reinterpret_cast<const float4*>(p);
        x[0] = v.x; x[1] = v.y; x[2] = v.z; x[3] = v.w;
    }
    __device__ __forceinline__ static void store(float* p, const float* x) {
        *reinterpret_cast<float4*>(p) = make_float4(x[0], x[1], x[2], x[3]);
    }
};

template <>
struct Vec16<__nv_bfloat16, 8> {
    __device__ __forceinline__ static void load(const __nv_bfloat16* p, float* x) {
        uint4 v = *reinterpret_cast<const uint4*>(p);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            x[2 * i] = __uint_as_float(w[i] << 16);
            x[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
        }
    }
    __device__ __forceinline__ static void store(__nv_bfloat16* p, const float* x) {
        uint32_t w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            __nv_bfloat162 h = __floats2bfloat162_rn(x[2 * i], x[2 * i + 1]);
            w[i] = *reinterpret_cast<uint32_t*>(&h);
        }
        *reinterpret_cast<uint4*>(p) = make_uint4(w[0], w[1], w[2], w[3]);
    }
};

template <typename T>
struct ElemsPer16 { static constexpr int value = 16 / (int)sizeof(T); };

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }
template <typename T>
__device__ __forceinline__ T from_f32(float x);
template <>
__device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

// Gates from logits ("Complex KDA" paper summary, Methodology, CKDA Definition):
// alpha = 2 sigma(a) - 1 (= tanh(a / 2), formed as (1 - e) / (1 + e) with e = exp(-|a|), which
// loses no precision near |alpha| = 1) and beta = 2 sigma(b).
__device__ __forceinline__ float gate_alpha(float a) {
    const float e = __expf(-fabsf(a));
    return copysignf(__fdividef(1.f - e, 1.f + e), a);
}
__device__ __forceinline__ float gate_beta(float b) { return __fdividef(2.f, 1.f + __expf(-b)); }

}  // namespace ckda
