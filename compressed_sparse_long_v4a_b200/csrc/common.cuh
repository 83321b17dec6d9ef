// common.cuh -- device helpers shared by the libv4a kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "v4a.h"

namespace v4a {

constexpr int kNumSMs = 148;  // B200: two dies of 74 SMs

// ---------------------------------------------------------------------
// element loads: 8 consecutive elements (16 bytes of bf16, 32 of fp32)
// ---------------------------------------------------------------------

__device__ __forceinline__ float bf16_bits_to_float(uint32_t h16) { return __uint_as_float(h16 << 16); }

__device__ __forceinline__ void unpack_bf16x8(const uint4& v, float f[8]) {
    f[0] = __uint_as_float(v.x << 16);
    f[1] = __uint_as_float(v.x & 0xffff0000u);
    f[2] = __uint_as_float(v.y << 16);
    f[3] = __uint_as_float(v.y & 0xffff0000u);
    f[4] = __uint_as_float(v.z << 16);
    f[5] = __uint_as_float(v.z & 0xffff0000u);
    f[6] = __uint_as_float(v.w << 16);
    f[7] = __uint_as_float(v.w & 0xffff0000u);
}

template <typename T>
struct Vec8;

template <>
struct Vec8<float> {
    static __device__ __forceinline__ void load(const float* p, float f[8]) {
        float4 a = *reinterpret_cast<const float4*>(p);
        float4 b = *reinterpret_cast<const float4*>(p + 4);
        f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
        f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
    }
    static __device__ __forceinline__ void load_nc(const float* p, float f[8]) {
        float4 a = __ldg(reinterpret_cast<const float4*>(p));
        float4 b = __ldg(reinterpret_cast<const float4*>(p + 4));
        f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
        f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
    }
    static __device__ __forceinline__ void store(float* p, const float f[8]) {
        *reinterpret_cast<float4*>(p) = make_float4(f[0], f[1], f[2], f[3]);
        *reinterpret_cast<float4*>(p + 4) = make_float4(f[4], f[5], f[6], f[7]);
    }
};

template <>
struct Vec8<__nv_bfloat16> {
    static __device__ __forceinline__ void load(const __nv_bfloat16* p, float f[8]) {
        uint4 v = *reinterpret_cast<const uint4*>(p);
        unpack_bf16x8(v, f);
    }
    static __device__ __forceinline__ void load_nc(const __nv_bfloat16* p, float f[8]) {
        uint4 v = __ldg(reinterpret_cast<const uint4*>(p));
        unpack_bf16x8(v, f);
    }
    static __device__ __forceinline__ void store(__nv_bfloat16* p, const float f[8]) {
        __nv_bfloat162 h[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
        *reinterpret_cast<uint4*>(p) = *reinterpret_cast<uint4*>(h);
    }
};

// 8 e4m3 codes (8 bytes) -> 8 floats (exact: every e4m3 value is a float)
__device__ __forceinline__ void unpack_e4m3x8(const uint2& v, float f[8]) {
    const uint32_t w[2] = {v.x, v.y};
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        __half2_raw lo = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(w[i] & 0xffffu), __NV_E4M3);
        __half2_raw hi = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(w[i] >> 16), __NV_E4M3);
        float2 a = __half22float2(*reinterpret_cast<__half2*>(&lo));
        float2 b = __half22float2(*reinterpret_cast<__half2*>(&hi));
        f[4 * i + 0] = a.x;
        f[4 * i + 1] = a.y;
        f[4 * i + 2] = b.x;
        f[4 * i + 3] = b.y;
    }
}

// two floats -> two e4m3 codes (round to nearest even, saturate to +-448)
__device__ __forceinline__ uint16_t pack_e4m3x2(float a, float b) {
    return (uint16_t)__nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3);
}

// ---------------------------------------------------------------------
// MXFP4 (OCP Microscaling v1.0): e2m1 codes, blocks of 32 sharing 2^X, X
// stored as the E8M0 byte X + 127
// ---------------------------------------------------------------------

// X = max(floor(log2(amax)) - 2, -127) for a block with largest magnitude amax (-127 if amax is 0
// or below the normal range); read off the binary32 exponent field, so exact
__device__ __forceinline__ int mx_block_exp(float amax) {
    const int ef = (int)((__float_as_uint(amax) >> 23) & 0xff);  // amax >= 0
    const int x = ef - 127 - 2;
    return (ef == 0 || x < -127) ? -127 : x;
}
// 2^k for k in [-126, 127] as a binary32 bit pattern (exact)
__device__ __forceinline__ float pow2i(int k) { return __uint_as_float((uint32_t)(k + 127) << 23); }
// 2^(e - 127) for an E8M0 byte e (e = 0 is the subnormal 2^-127; 255, NaN in the format, is not
// produced by the quantiser and gives +inf here)
__device__ __forceinline__ float e8m0_value(uint32_t e) { return e ? __uint_as_float(e << 23) : 0x1p-127f; }
// nearest e2m1 code of x (ties to the even code, |x| > 6 clamps to 6, the sign kept even when the
// magnitude rounds to 0): the magnitude code counts the rounding thresholds that |x| passes, the
// strict ones being ties that go down to an even code
__device__ __forceinline__ uint32_t e2m1_code(float x) {
    const float a = fabsf(x);
    const uint32_t m = (uint32_t)(a > 0.25f) + (uint32_t)(a >= 0.75f) + (uint32_t)(a > 1.25f) +
                       (uint32_t)(a >= 1.75f) + (uint32_t)(a > 2.5f) + (uint32_t)(a >= 3.5f) + (uint32_t)(a > 5.0f);
    return m | ((__float_as_uint(x) >> 28) & 0x8u);
}
// value of an e2m1 code
__device__ __forceinline__ float e2m1_value(uint32_t c) {
    const uint32_t e = (c >> 1) & 3u, f = c & 1u;
    const float mag = e ? __uint_as_float(((e + 126u) << 23) | (f << 22)) : 0.5f * (float)f;
    return (c & 8u) ? -mag : mag;
}
// Quantise 8 consecutive elements of a 32-element block held by 4 consecutive lanes (lanes 4k ..
// 4k+3 of the warp, in element order; all 32 lanes take part): returns the 8 codes packed in a
// 32-bit word (element 2i in the low nibble of byte i) and the block's X in *x_out.
__device__ __forceinline__ uint32_t mx_quantize8(const float v[8], int* x_out) {
    float a = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) a = fmaxf(a, fabsf(v[i]));
    a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 1));
    a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 2));
    const int x = mx_block_exp(a);
    // v * 2^-X: exact (a power of two) except for results below the normal range, which are far
    // below the smallest e2m1 step and round to 0 either way.  2^-X for X = -127 is 2^127.
    const float inv = pow2i(-x);
    uint32_t w = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) w |= e2m1_code(v[i] * inv) << (4 * i);
    *x_out = x;
    return w;
}

// ---------------------------------------------------------------------
// order-preserving float -> uint32 (larger float -> larger key); -0 == +0
// ---------------------------------------------------------------------
__device__ __forceinline__ uint32_t float_to_ordered(float f) {
    f += 0.0f;  // -0 -> +0
    uint32_t u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float ordered_to_float(uint32_t k) {
    uint32_t u = (k & 0x80000000u) ? (k & 0x7fffffffu) : ~k;
    return __uint_as_float(u);
}

// ---------------------------------------------------------------------
// warp reductions
// ---------------------------------------------------------------------
template <int WIDTH>
__device__ __forceinline__ float group_max(float v) {
#pragma unroll
    for (int o = WIDTH / 2; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

template <int WIDTH>
__device__ __forceinline__ float group_sum(float v) {
#pragma unroll
    for (int o = WIDTH / 2; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__host__ __device__ __forceinline__ long long n_visible(long long t, int m) { return (t + 1) / m; }

// Programmatic dependent launch.  Every kernel of the library is launched with launch_pdl(), so it may
// be scheduled while the kernel before it on the stream is still finishing; griddep_wait() then
// blocks until that kernel has completed and its memory is visible (a no-op when there is no such
// dependency), so every thread calls it before its first global memory access (reads and writes);
// griddep_launch_dependents() lets the next kernel's blocks be scheduled once every block of this
// grid has called it, so they can set up (shared memory, barriers, tensor memory) meanwhile.
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// Output RoPE at minus the query position ("1M Context != Lossless Long Memory", section 8): the
// pair k of the last R dims of a d-dim row turns by -t * base^(-2k/R).  sin/cos of that angle,
// reduced and evaluated in double (t reaches 1M, the angle hundreds of thousands of radians).
__device__ __forceinline__ void rope_sincos(long long t, int k, int rope_dims, float base, float* s, float* c) {
    const double ang = -(double)t * pow((double)base, -2.0 * (double)k / (double)rope_dims);
    const double r = remainder(ang, 6.283185307179586476925286766559);
    double sd, cd;
    sincos(r, &sd, &cd);
    *s = (float)sd;
    *c = (float)cd;
}
// the rotated value of output dim `dim` (in the RoPE part) from its value v and its pair partner p
__device__ __forceinline__ float rope_apply(int dim, float v, float p, float s, float c) {
    return (dim & 1) ? fmaf(p, s, v * c) : fmaf(v, c, -p * s);
}

}  // namespace v4a
