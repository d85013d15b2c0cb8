// ba_pack.cu -- KD1 pre-pass: sign bits and per-token mean-|x| scale.
//
// BA notes, Key design 1 (Scaled Binary Representations): each query/key token
// becomes a +-1 vector plus one scale that keeps its magnitude.  This pass is
// HBM-bound (read d values, write d/8 bytes + 4 bytes per token), so it is
// written for coalescing: each lane loads one 16-byte vector, a token is a
// run of consecutive lanes, and a warp load covers whole tokens back to back.
#include "ba_prepass.cuh"

namespace ba {

// E elements per 16-byte vector (8 for bf16, 4 for fp32).  G = d / E lanes per
// token; a warp handles floor(32 / G) tokens per step.  Requires d % E == 0,
// G <= 32 and a 16-byte aligned base.
template <typename T>
__global__ void __launch_bounds__(256)
pack_vec_kernel(const T* __restrict__ x, int64_t tokens, int d,
                uint32_t* __restrict__ bits, float* __restrict__ mu)
{
    constexpr int E = 16 / sizeof(T);
    const int G = d / E;                 // lanes per token
    const int per_warp = 32 / G;         // tokens per warp step
    const int lane = threadIdx.x & 31;
    const int slot = lane / G;           // which token of this step
    const int chunk = lane - slot * G;   // which 16-byte vector of the token
    const bool active_lane = slot < per_warp;
    const int W = words_for(d);
    const int first_ch = chunk * E;      // first channel this lane holds
    const int word = first_ch >> 5;      // word the lane's bits land in
    const int shift = first_ch & 31;
    const int head = slot * G;           // first lane of this token
    const int word_head = head + ((word * 32) / E);  // first lane of this word
    const int lanes_in_word = min(32 / E, G - (word * 32) / E);

    const int64_t warp_global = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const int64_t warp_stride = (int64_t)gridDim.x * (blockDim.x >> 5);

    for (int64_t base = warp_global * per_warp; base < tokens; base += warp_stride * per_warp) {
        const int64_t t = base + slot;
        const bool live = active_lane && t < tokens;
        uint32_t my_bits = 0;
        float s = 0.f;
        if (live) {
            const uint4 raw = *reinterpret_cast<const uint4*>(x + t * d + first_ch);
            const T* v = reinterpret_cast<const T*>(&raw);
#pragma unroll
            for (int e = 0; e < E; ++e) {
                const float f = to_f32<T>(v[e]);
                my_bits |= (f >= 0.f ? 1u : 0u) << e;
                s += fabsf(f);
            }
        }
        // OR the lane bit-fields of one word together at the word's first lane.
        uint32_t wv = my_bits << shift;
        uint32_t acc = wv;
        for (int k = 1; k < 32 / E; ++k) {
            const uint32_t other = __shfl_sync(0xffffffffu, wv, min(lane + k, 31));
            if (lane == word_head && k < lanes_in_word) acc |= other;
        }
        // Sum |x| over the token's lanes at its first lane (fixed order).
        float tot = s;
        for (int k = 1; k < G; ++k) {   // G is warp-uniform
            const float other = __shfl_sync(0xffffffffu, s, min(lane + k, 31));
            if (lane == head) tot += other;
        }
        if (live && lane == word_head) bits[t * W + word] = acc;
        if (live && lane == head) mu[t] = __fdiv_rn(tot, (float)d);
    }
}

// One thread per token for the common head sizes: the token's NV 16-byte
// vectors are loaded at once (NV loads in flight per thread, no shuffles),
// its sign bits and |x| sum built in registers in channel order.
template <typename T, int NV>
__global__ void __launch_bounds__(256)
pack_row_kernel(const T* __restrict__ x, int64_t tokens, int d, uint32_t* __restrict__ bits,
                float* __restrict__ mu)
{
    constexpr int W = (NV * (16 / (int)sizeof(T)) + 31) / 32;
    const int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (t >= tokens) return;
    pack_token<T, NV>(x + t * d, d, bits + t * W, mu + t);
}

// General fallback: one warp per token, channel c on lane c % 32.
template <typename T>
__global__ void __launch_bounds__(256)
pack_any_kernel(const T* __restrict__ x, int64_t tokens, int d,
                uint32_t* __restrict__ bits, float* __restrict__ mu)
{
    const int lane = threadIdx.x & 31;
    const int W = words_for(d);
    const int64_t warp_global = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const int64_t warp_stride = (int64_t)gridDim.x * (blockDim.x >> 5);
    for (int64_t t = warp_global; t < tokens; t += warp_stride) {
        float s = 0.f;
        for (int w = 0; w < W; ++w) {
            const int c = w * 32 + lane;
            float f = -1.f;
            bool pos = false;
            if (c < d) {
                f = to_f32<T>(x[t * d + c]);
                pos = f >= 0.f;
                s += fabsf(f);
            }
            const uint32_t word = __ballot_sync(0xffffffffu, pos);
            if (lane == 0) bits[t * W + w] = word;
        }
        for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
        if (lane == 0) mu[t] = __fdiv_rn(s, (float)d);
    }
}

template <typename T>
static cudaError_t launch_pack_t(const void* x, int64_t tokens, int d, uint32_t* bits, float* mu,
                                 cudaStream_t st, int sm_count)
{
    constexpr int E = 16 / sizeof(T);
    const T* xp = static_cast<const T*>(x);
    const int threads = 256;
    if (d % E == 0 && aligned(x, 16)) {
        const unsigned blocks = (unsigned)((tokens + threads - 1) / threads);
        switch (d / E) {
#define BA_PACK_ROW(NV) case NV: pack_row_kernel<T, NV><<<blocks, threads, 0, st>>>(xp, tokens, d, bits, mu); return cudaGetLastError();
            BA_PACK_ROW(2) BA_PACK_ROW(4) BA_PACK_ROW(8) BA_PACK_ROW(9) BA_PACK_ROW(12) BA_PACK_ROW(16)
#undef BA_PACK_ROW
            default: break;
        }
    }
    if (d % E == 0 && d / E <= 32 && aligned(x, 16)) {
        const int per_warp = 32 / (d / E);
        const int64_t warps = (tokens + per_warp - 1) / per_warp;
        int64_t blocks = (warps + 7) / 8;
        blocks = blocks < (int64_t)sm_count * 16 ? blocks : (int64_t)sm_count * 16;
        pack_vec_kernel<T><<<(unsigned)blocks, threads, 0, st>>>(xp, tokens, d, bits, mu);
    } else {
        int64_t blocks = (tokens + 7) / 8;
        blocks = blocks < (int64_t)sm_count * 16 ? blocks : (int64_t)sm_count * 16;
        pack_any_kernel<T><<<(unsigned)blocks, threads, 0, st>>>(xp, tokens, d, bits, mu);
    }
    return cudaGetLastError();
}

cudaError_t launch_pack(const void* x, ba_dtype dt, int64_t tokens, int d, uint32_t* bits,
                        float* mu, cudaStream_t st, int sm_count)
{
    if (dt == BA_BF16) return launch_pack_t<__nv_bfloat16>(x, tokens, d, bits, mu, st, sm_count);
    return launch_pack_t<float>(x, tokens, d, bits, mu, st, sm_count);
}

}  // namespace ba
