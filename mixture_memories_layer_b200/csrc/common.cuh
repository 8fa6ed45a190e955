// Device helpers shared by the MoM kernels: element loads/stores for the two
// activation types, warp reductions, and the workspace error record.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "mom.h"

namespace mom {

typedef __nv_bfloat16 bf16;

// ---------------------------------------------------------------- errors --
// The first MOM_WS_HEADER_BYTES of a workspace: {code, info, ...}.  The first
// violation wins; later ones are dropped.
__device__ __forceinline__ void record_error(void* ws, int code, long long info) {
    if (ws == nullptr) return;
    int32_t* rec = reinterpret_cast<int32_t*>(ws);
    if (atomicCAS(rec, 0, code) == 0) rec[1] = (int32_t)info;
}

// ----------------------------------------------------------- conversions --
__device__ __forceinline__ float to_f(float v) { return v; }
__device__ __forceinline__ float to_f(bf16 v) { return __bfloat162float(v); }
template <typename T> __device__ __forceinline__ T from_f(float v);
template <> __device__ __forceinline__ float from_f<float>(float v) { return v; }
template <> __device__ __forceinline__ bf16 from_f<bf16>(float v) { return __float2bfloat16_rn(v); }

// Load N consecutive elements (N in {1,2,4,8}) into floats.  The address must
// be aligned to N * sizeof(T) bytes.
template <int N> __device__ __forceinline__ void load_vec(const float* p, float* out) {
    if constexpr (N == 8) {
        float4 a = *reinterpret_cast<const float4*>(p);
        float4 b = *reinterpret_cast<const float4*>(p + 4);
        out[0] = a.x; out[1] = a.y; out[2] = a.z; out[3] = a.w;
        out[4] = b.x; out[5] = b.y; out[6] = b.z; out[7] = b.w;
    } else if constexpr (N == 4) {
        float4 a = *reinterpret_cast<const float4*>(p);
        out[0] = a.x; out[1] = a.y; out[2] = a.z; out[3] = a.w;
    } else if constexpr (N == 2) {
        float2 a = *reinterpret_cast<const float2*>(p);
        out[0] = a.x; out[1] = a.y;
    } else {
        out[0] = *p;
    }
}
template <int N> __device__ __forceinline__ void load_vec(const bf16* p, float* out) {
    if constexpr (N == 8) {
        uint4 u = *reinterpret_cast<const uint4*>(p);
        const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            float2 f = __bfloat1622float2(h[i]);
            out[2 * i] = f.x; out[2 * i + 1] = f.y;
        }
    } else if constexpr (N == 4) {
        uint2 u = *reinterpret_cast<const uint2*>(p);
        const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            float2 f = __bfloat1622float2(h[i]);
            out[2 * i] = f.x; out[2 * i + 1] = f.y;
        }
    } else if constexpr (N == 2) {
        float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(p));
        out[0] = f.x; out[1] = f.y;
    } else {
        out[0] = __bfloat162float(*p);
    }
}

template <int N> __device__ __forceinline__ void store_vec(float* p, const float* v) {
    if constexpr (N == 8) {
        *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
        *reinterpret_cast<float4*>(p + 4) = make_float4(v[4], v[5], v[6], v[7]);
    } else if constexpr (N == 4) {
        *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
    } else if constexpr (N == 2) {
        *reinterpret_cast<float2*>(p) = make_float2(v[0], v[1]);
    } else {
        *p = v[0];
    }
}
template <int N> __device__ __forceinline__ void store_vec(bf16* p, const float* v) {
    if constexpr (N == 8) {
        uint4 u;
        __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
        for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
        *reinterpret_cast<uint4*>(p) = u;
    } else if constexpr (N == 4) {
        uint2 u;
        __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&u);
        h[0] = __floats2bfloat162_rn(v[0], v[1]);
        h[1] = __floats2bfloat162_rn(v[2], v[3]);
        *reinterpret_cast<uint2*>(p) = u;
    } else if constexpr (N == 2) {
        *reinterpret_cast<__nv_bfloat162*>(p) = __floats2bfloat162_rn(v[0], v[1]);
    } else {
        *p = __float2bfloat16_rn(v[0]);
    }
}

// ------------------------------------------------------------ reductions --
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Butterfly-reduces N independent values across the warp (all lanes get all sums).
template <int N> __device__ __forceinline__ void warp_sum_n(float* v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
#pragma unroll
        for (int i = 0; i < N; ++i) v[i] += __shfl_xor_sync(0xffffffffu, v[i], o);
    }
}

__device__ __forceinline__ float sigmoidf_(float z) { return 1.0f / (1.0f + expf(-z)); }
__device__ __forceinline__ float softplusf_(float z) { return z > 20.0f ? z : log1pf(expf(z)); }

__host__ __device__ __forceinline__ int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }

}  // namespace mom
