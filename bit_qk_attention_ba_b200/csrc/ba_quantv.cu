// ba_quantv.cu -- KD3 pre-pass: channel-wise symmetric int8 quantisation of V.
//
// BA notes, Key design 3 (Hybrid Quantization): V is quantised channel-wise to
// 8 bits so the PV product can run on the integer tensor path.  Reading: per
// (batch, head, channel) over the N tokens, scale = absmax / 127 (IEEE fp32
// division), code = round-half-even(v / scale) (IEEE fp32 division), clamped
// to +-127.
//
// When the codes of one (batch, head) fit in shared memory (the ViT / DiT
// shapes), one launch does everything with one HBM read of V: one CTA per
// (b, h) takes the channel absmax in a first sweep over the rows, writes the
// scales, and quantises in a second sweep (served from L2) into channel-major
// code rows.  Otherwise three launches, no scratch memory: (1)
// column absmax folded into the sv output with atomicMax on the
// (non-negative) float bit patterns, (2) quantise a tile of keys and write it
// transposed into the channel-major [B, H, d, ldv] code layout, (3) turn the
// stored absmax into the scale.  In both, codes are transposed through
// shared memory rows whose stride is an odd number of 4-byte words, so the
// byte writes of a warp (consecutive channels) land in distinct banks.
#include "ba_prepass.cuh"

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
    constexpr int QS = KT + 4;          // code row stride: 17 words
    __shared__ float scale[128], rscale[128];
    __shared__ __align__(16) uint8_t qt[128 * QS];
    const int64_t bh = blockIdx.y;
    const int j0 = blockIdx.x * KT;
    for (int c = threadIdx.x; c < d; c += blockDim.x) {
        const float sc = __fdiv_rn(__uint_as_float(amax[bh * d + c]), 127.0f);
        scale[c] = sc;
        rscale[c] = __frcp_rn(sc);
    }
    __syncthreads();
    // (key j, channel c) with c fastest, stepped without a division per element.
    const int nt = blockDim.x, dj = nt / d, dc = nt - dj * d;
    int j = threadIdx.x / d, c = threadIdx.x - j * d;
    for (; j < KT; j += dj, c += dc) {
        if (c >= d) { c -= d; ++j; if (j >= KT) break; }
        const int key = j0 + j;
        qt[c * QS + j] = (uint8_t)((key < N) ? vcode(to_f32<T>(v[(bh * N + key) * d + c]), scale[c], rscale[c]) : 0u);
    }
    __syncthreads();
    for (int idx = threadIdx.x; idx < d * (KT / 16); idx += blockDim.x) {
        const int c = idx >> 2, g = idx & 3;
        const int64_t col = (int64_t)j0 + g * 16;
        if (col < ldv) store_codes16(vq + (bh * d + c) * ldv + col, qt + c * QS + g * 16);
    }
}

// One CTA per (b, h): absmax, scales and codes with V read from HBM once.
template <typename T>
__global__ void __launch_bounds__(256, 4)
vquant_small_kernel(const T* __restrict__ v, int N, int d, int64_t ldv, int8_t* __restrict__ vq,
                    float* __restrict__ sv)
{
    extern __shared__ __align__(16) uint8_t qt[];
    __shared__ VBlockShared sh;
    const int64_t bh = blockIdx.x;
    vblock_quant<T>(v + bh * N * d, N, d, ldv, vq + bh * d * ldv, sv + bh * d, qt, sh);
}

__global__ void vscale_kernel(float* sv, int64_t n)
{
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i < n) sv[i] = __fdiv_rn(sv[i], 127.0f);   // sv holds absmax bits == the float itself
}

// The tiled path's first half: zero sv, then fold every tile's channel
// absmax into it as the bits of the (non-negative) floats.
template <typename T>
static cudaError_t launch_v_absmax_t(const void* v, int B, int H, int N, int d, float* sv, cudaStream_t st)
{
    const T* vp = static_cast<const T*>(v);
    const int64_t BH = (int64_t)B * H;
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
    return cudaGetLastError();
}

// The tiled path's last step: sv (absmax bits) -> scale = absmax / 127.
cudaError_t launch_v_scale(float* sv, int64_t n, cudaStream_t st)
{
    vscale_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(sv, n);
    return cudaGetLastError();
}

cudaError_t launch_v_absmax(const void* v, ba_dtype dt, int B, int H, int N, int d, float* sv, cudaStream_t st)
{
    if (dt == BA_BF16) return launch_v_absmax_t<__nv_bfloat16>(v, B, H, N, d, sv, st);
    return launch_v_absmax_t<float>(v, B, H, N, d, sv, st);
}

template <typename T>
static cudaError_t launch_quant_v_t(const void* v, int B, int H, int N, int d, int8_t* vq, float* sv,
                                    cudaStream_t st)
{
    const T* vp = static_cast<const T*>(v);
    const int64_t BH = (int64_t)B * H;
    const int64_t ldv = round_up64(N, 16);
    // Single pass when one (b, h) block of V and its codes fit in shared memory.
    const int64_t small_smem = vblock_smem_bytes(N, d);
    if ((d * sizeof(T)) % 16 == 0 && aligned(v, 16) && small_smem <= kVBlockMaxSmem) {
        auto k = vquant_small_kernel<T>;
        cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)small_smem);
        if (e != cudaSuccess) return e;
        k<<<(unsigned)BH, 256, (size_t)small_smem, st>>>(vp, N, d, ldv, vq, sv);
        return cudaGetLastError();
    }
    cudaError_t e = launch_v_absmax_t<T>(v, B, H, N, d, sv, st);
    if (e != cudaSuccess) return e;
    dim3 g2(ceil_div((int)ldv, 64), (unsigned)BH);
    vquant_kernel<T><<<g2, 256, 0, st>>>(vp, N, d, ldv, reinterpret_cast<const unsigned*>(sv), vq);
    e = cudaGetLastError();
    return e == cudaSuccess ? launch_v_scale(sv, BH * d, st) : e;
}

cudaError_t launch_quant_v(const void* v, ba_dtype dt, int B, int H, int N, int d, int8_t* vq,
                           float* sv, cudaStream_t st)
{
    if (dt == BA_BF16) return launch_quant_v_t<__nv_bfloat16>(v, B, H, N, d, vq, sv, st);
    return launch_quant_v_t<float>(v, B, H, N, d, vq, sv, st);
}

}  // namespace ba
