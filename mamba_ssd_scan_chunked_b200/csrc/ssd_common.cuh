// Device-side helpers shared by the libssd kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace ssd {

// Bits of the device error word (see ssd_get_device_error).
constexpr unsigned kErrChainTimeout = 1u;   // an inter-chunk state hand-off wait gave up
constexpr unsigned kErrChainAborted = 2u;   // a wait was cut short because another one gave up
constexpr unsigned kErrAsyncTimeout = 4u;   // a TMA/MMA completion did not arrive in time

typedef __nv_bfloat16 bf16;

__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(bf16 v) { return __bfloat162float(v); }

template <typename T> __device__ __forceinline__ T from_f32(float v);
template <> __device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ bf16 from_f32<bf16>(float v) { return __float2bfloat16_rn(v); }

// softplus(z) = log(1 + e^z).  Above z = 20 the correction log1p(e^-z) is below
// 2.1e-9 and the result is z to fp32 precision; below, log1pf(expf(z)) is
// accurate and underflows to exactly 0 for very negative z.
__device__ __forceinline__ float softplus_f32(float z) {
    return z > 20.f ? z : log1pf(expf(z));
}

// 16-byte vector of VEC elements of T, converted to/from fp32.
template <typename T> struct Vec16;
template <> struct Vec16<float> {
    static constexpr int N = 4;
    __device__ __forceinline__ static void unpack(uint4 v, float* out) {
        out[0] = __uint_as_float(v.x); out[1] = __uint_as_float(v.y);
        out[2] = __uint_as_float(v.z); out[3] = __uint_as_float(v.w);
    }
    __device__ __forceinline__ static uint4 pack(const float* in) {
        return make_uint4(__float_as_uint(in[0]), __float_as_uint(in[1]), __float_as_uint(in[2]),
                          __float_as_uint(in[3]));
    }
    __device__ __forceinline__ static void load(const float* p, float* out) {
        float4 v = *reinterpret_cast<const float4*>(p);
        out[0] = v.x; out[1] = v.y; out[2] = v.z; out[3] = v.w;
    }
    __device__ __forceinline__ static void load_stream(const float* p, float* out) {
        float4 v = __ldcs(reinterpret_cast<const float4*>(p));
        out[0] = v.x; out[1] = v.y; out[2] = v.z; out[3] = v.w;
    }
    __device__ __forceinline__ static void store(float* p, const float* in) {
        *reinterpret_cast<float4*>(p) = make_float4(in[0], in[1], in[2], in[3]);
    }
    __device__ __forceinline__ static void store_stream(float* p, const float* in) {
        __stcs(reinterpret_cast<float4*>(p), make_float4(in[0], in[1], in[2], in[3]));
    }
};
template <> struct Vec16<bf16> {
    static constexpr int N = 8;
    __device__ __forceinline__ static void unpack(uint4 v, float* out) {
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            out[2 * i] = __uint_as_float(w[i] << 16);
            out[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
        }
    }
    __device__ __forceinline__ static uint4 pack(const float* in) {
        uint32_t w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            __nv_bfloat162 t = __floats2bfloat162_rn(in[2 * i], in[2 * i + 1]);
            w[i] = *reinterpret_cast<uint32_t*>(&t);
        }
        return make_uint4(w[0], w[1], w[2], w[3]);
    }
    __device__ __forceinline__ static void load(const bf16* p, float* out) {
        unpack(*reinterpret_cast<const uint4*>(p), out);
    }
    __device__ __forceinline__ static void load_stream(const bf16* p, float* out) {
        unpack(__ldcs(reinterpret_cast<const uint4*>(p)), out);
    }
    __device__ __forceinline__ static void store(bf16* p, const float* in) {
        *reinterpret_cast<uint4*>(p) = pack(in);
    }
    __device__ __forceinline__ static void store_stream(bf16* p, const float* in) {
        __stcs(reinterpret_cast<uint4*>(p), pack(in));
    }
};

}  // namespace ssd
