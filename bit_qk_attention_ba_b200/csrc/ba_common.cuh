// ba_common.cuh -- small device/host helpers shared by the libba kernels.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "../../include/ba.h"

namespace ba {

// Status bits a kernel may record in the device status word.
enum : unsigned {
    kStatusTimeoutProducer = 1u << 0,  // load warp gave up on a barrier
    kStatusTimeoutMma      = 1u << 1,  // MMA warp gave up on a barrier
    kStatusTimeoutSoftmax  = 1u << 2,  // softmax warps gave up on a barrier
    kStatusTimeoutEpilogue = 1u << 3,
    kStatusBadLaunch       = 1u << 4,  // kernel found a launch shape it cannot serve
    kStatusTimeoutCopy     = 1u << 5,  // a kernel gave up waiting for its bulk copies
};

__host__ __device__ inline int words_for(int d) { return (d + 31) / 32; }
__host__ __device__ inline int64_t round_up64(int64_t x, int64_t m) { return (x + m - 1) / m * m; }
__host__ __device__ inline int ceil_div(int a, int b) { return (a + b - 1) / b; }

template <typename T> __device__ __forceinline__ float to_f32(T x);
template <> __device__ __forceinline__ float to_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }

// Host: pointer alignment test.
inline bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Address of this device's status word (set up once per device in ba_api.cu).
unsigned* device_status_ptr();

}  // namespace ba
