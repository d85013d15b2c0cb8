// ba_quantv.cu -- KD3 pre-pass: channel-wise symmetric int8 quantisation of V.
//
// BA notes, Key design 3 (Hybrid Quantization): V is quantised channel-wise to
// 8 bits so the PV product can run on the integer tensor path.  Reading: per
// (batch, head, channel) over the N tokens, scale = absmax / 127 (IEEE fp32
// division), code = round-half-even(v / scale) (IEEE fp32 division), clamped
// to +-127.
//
// Three launches, no scratch memory: (1) column absmax folded into the sv
// output with atomicMax on the (non-negative) float bit patterns, (2)
// quantise a tile of keys and write it transposed into the channel-major
// [B, H, d, ldv] code layout, (3) turn the stored absmax into the scale.
#include "ba_common.cuh"

namespace ba {

template <typename T, int E>
__global__ void __launch_bounds__(256)
vabsmax_kernel(const T* __restrict__ v, int N, int d, int rows_per_cta, unsigned* __restrict__ amax)
{
    __shared__ unsigned red[128];
    const int CV = d / E;                 // vectors per token row
    const int RY = 256 / CV;              // rows handled in parallel
    const int cv = threadIdx.x % CV;
    const int ry = threadIdx.x / CV;
    const int64_t bh = blockIdx.y;
    const int r0 = blockIdx.x * rows_per_cta;
    const int r1 = min(N, r0 + rows_per_cta);
    for (int c = threadIdx.x; c < d; c += blockDim.x) red[c] = 0u;
    __syncthreads();
    float m[E];
#pragma unroll
    for (int e = 0; e < E; ++e) m[e] = 0.f;
    if (ry < RY) {
        for (int r = r0 + ry; r < r1; r += RY) {
            const T* p = v + ((bh * N + r) * d + cv * E);
            if constexpr (E == 1) {
                m[0] = fmaxf(m[0], fabsf(to_f32<T>(p[0])));
            } else {
                const uint4 raw = *reinterpret_cast<const uint4*>(p);
                const T* x = reinterpret_cast<const T*>(&raw);
#pragma unroll
                for (int e = 0; e < E; ++e) m[e] = fmaxf(m[e], fabsf(to_f32<T>(x[e])));
            }
        }
#pragma unroll
        for (int e = 0; e < E; ++e) atomicMax(&red[cv * E + e], __float_as_uint(m[e]));
    }
    __syncthreads();
    for (int c = threadIdx.x; c < d; c += blockDim.x)
        if (red[c]) atomicMax(&amax[bh * d + c], red[c]);
}

// Tile of 64 keys of one (b, h): quantise and store channel-major.
template <typename T>
__global__ void __launch_bounds__(256)
vquant_kernel(const T* __restrict__ v, int N, int d, int64_t ldv,
              const unsigned* __restrict__ amax, int8_t* __restrict__ vq)
{
    constexpr int KT = 64;
    __shared__ float scale[128];
    __shared__ __align__(16) int8_t qt[128][KT];
    const int64_t bh = blockIdx.y;
    const int j0 = blockIdx.x * KT;
    for (int c = threadIdx.x; c < d; c += blockDim.x)
        scale[c] = __fdiv_rn(__uint_as_float(amax[bh * d + c]), 127.0f);
    __syncthreads();
    for (int idx = threadIdx.x; idx < KT * d; idx += blockDim.x) {
        const int j = idx / d, c = idx - j * d;
        const int key = j0 + j;
        int q = 0;
        if (key < N) {
            const float s = scale[c];
            if (s != 0.f) {
                const float r = __fdiv_rn(to_f32<T>(v[(bh * N + key) * d + c]), s);
                q = __float2int_rn(r);
                q = max(-127, min(127, q));
            }
        }
        qt[c][j] = (int8_t)q;
    }
    __syncthreads();
    const int groups = KT / 16;
    for (int idx = threadIdx.x; idx < d * groups; idx += blockDim.x) {
        const int c = idx / groups, g = idx - c * groups;
        const int64_t col = (int64_t)j0 + g * 16;
        if (col < ldv)
            *reinterpret_cast<uint4*>(vq + (bh * d + c) * ldv + col) =
                *reinterpret_cast<const uint4*>(&qt[c][g * 16]);
    }
}

__global__ void vscale_kernel(float* sv, int64_t n)
{
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i < n) sv[i] = __fdiv_rn(sv[i], 127.0f);   // sv holds absmax bits == the float itself
}

template <typename T>
static cudaError_t launch_quant_v_t(const void* v, int B, int H, int N, int d, int8_t* vq, float* sv,
                                    cudaStream_t st)
{
    const T* vp = static_cast<const T*>(v);
    const int64_t BH = (int64_t)B * H;
    const int64_t ldv = round_up64(N, 16);
    cudaError_t e = cudaMemsetAsync(sv, 0, sizeof(float) * BH * d, st);
    if (e != cudaSuccess) return e;
    constexpr int E = 16 / sizeof(T);
    const int rows = 512;
    dim3 g1(ceil_div(N, rows), (unsigned)BH);
    unsigned* amax = reinterpret_cast<unsigned*>(sv);
    if (d % E == 0 && aligned(v, 16))
        vabsmax_kernel<T, E><<<g1, 256, 0, st>>>(vp, N, d, rows, amax);
    else
        vabsmax_kernel<T, 1><<<g1, 256, 0, st>>>(vp, N, d, rows, amax);
    dim3 g2(ceil_div((int)ldv, 64), (unsigned)BH);
    vquant_kernel<T><<<g2, 256, 0, st>>>(vp, N, d, ldv, amax, vq);
    const int64_t n = BH * d;
    vscale_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(sv, n);
    return cudaGetLastError();
}

cudaError_t launch_quant_v(const void* v, ba_dtype dt, int B, int H, int N, int d, int8_t* vq,
                           float* sv, cudaStream_t st)
{
    if (dt == BA_BF16) return launch_quant_v_t<__nv_bfloat16>(v, B, H, N, d, vq, sv, st);
    return launch_quant_v_t<float>(v, B, H, N, d, vq, sv, st);
}

}  // namespace ba
