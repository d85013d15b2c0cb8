// ba_quantv.cu -- KD3 pre-pass: channel-wise symmetric int8 quantisation of V.
//
// BA notes, Key design 3 (Hybrid Quantization): V is quantised channel-wise to
// 8 bits so the PV product can run on the integer tensor path.  Reading: per
// (batch, head, channel) over the N tokens, scale = absmax / 127 (IEEE fp32
// division), code = round-half-even(v / scale) (IEEE fp32 division), clamped
// to +-127.
//
// When all N keys of one (batch, head) fit in shared memory (the ViT / DiT
// shapes), one launch does everything with one read of V: one CTA per (b, h)
// stages the [N, d] block, takes the channel absmax, writes the scales and
// the codes channel-major.  Otherwise three launches, no scratch memory: (1)
// column absmax folded into the sv output with atomicMax on the
// (non-negative) float bit patterns, (2) quantise a tile of keys and write it
// transposed into the channel-major [B, H, d, ldv] code layout, (3) turn the
// stored absmax into the scale.  In both, codes are transposed through
// shared memory rows whose stride is an odd number of 4-byte words, so the
// byte writes of a warp (consecutive channels) land in distinct banks.
#include "ba_common.cuh"
#include "ba_sm100.cuh"

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

// code = clamp(round_half_even(fl32(x / s)), -127, 127); 0 for an all-zero channel.
// rs = fl32(1 / s).  Here |x| <= 127 s, so t = fl32(x * rs) is within 3e-5 of
// x / s and fl32(x / s) within 8e-6 of it: when t is more than 1e-4 away from
// a rounding boundary (k + 1/2), both round to the same integer, and the code
// is rint(t); otherwise the IEEE quotient is formed and rounded.  Either way
// the result equals rounding fl32(x / s).
__device__ __forceinline__ uint32_t vcode(float x, float s, float rs)
{
    if (s == 0.f) return 0u;
    const float t = x * rs;
    const float k = (t + 12582912.f) - 12582912.f;     // round-half-even of t (|t| < 2^22)
    int q;
    if (0.5f - fabsf(t - k) > 1e-4f) q = (int)k;
    else q = __float2int_rn(__fdiv_rn(x, s));
    q = max(-127, min(127, q));
    return (uint32_t)(q & 0xFF);
}

// 16 codes of channel row `row` (4-byte aligned, in shared memory) -> 16 bytes of vq.
__device__ __forceinline__ void store_codes16(int8_t* dst, const uint8_t* row)
{
    const uint32_t* q4 = reinterpret_cast<const uint32_t*>(row);
    *reinterpret_cast<uint4*>(dst) = make_uint4(q4[0], q4[1], q4[2], q4[3]);
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

// All N keys of one (b, h) in shared memory (tile [N][d] of V, then the codes
// [d][ldv + 4]): absmax, scale and codes from a single read of V.
template <typename T>
__global__ void __launch_bounds__(512)
vquant_small_kernel(const T* __restrict__ v, int N, int d, int64_t ldv, int8_t* __restrict__ vq,
                    float* __restrict__ sv, unsigned* __restrict__ status)
{
    extern __shared__ __align__(16) uint8_t sm_raw[];
    __shared__ unsigned amax[128];
    __shared__ float scale[128], rscale[128];
    T* tile = reinterpret_cast<T*>(sm_raw);
    const int64_t tile_bytes = (int64_t)N * d * sizeof(T);
    const int qs = (int)ldv + 4;        // odd number of 4-byte words (ldv % 16 == 0)
    uint8_t* qt = sm_raw + tile_bytes;
    __shared__ __align__(8) uint64_t bar;
    const int64_t bh = blockIdx.x;
    const int tid = threadIdx.x, nt = blockDim.x;
    // The whole block comes in with bulk copies (at most 64 KB each) on one
    // mbarrier; the wait is bounded and a timeout only leaves the codes of this
    // block unwritten after flagging the device status word.
    if (tid == 0) {
        sm100::mbar_init(&bar, 1);
        sm100::fence_mbar_init();
    }
    for (int c = tid; c < d; c += nt) amax[c] = 0u;
    __syncthreads();
    if (tid == 0) {
        sm100::mbar_arrive_expect_tx(&bar, (uint32_t)tile_bytes);
        const uint8_t* src = reinterpret_cast<const uint8_t*>(v + bh * N * d);
        for (int64_t off = 0; off < tile_bytes; off += 65536) {
            const uint32_t n = (uint32_t)min((int64_t)65536, tile_bytes - off);
            sm100::bulk_load(sm_raw + off, src + off, n, &bar);
        }
    }
    const bool landed = sm100::mbar_wait(&bar, 0, nullptr);
    if (!__syncthreads_and(landed)) {
        if (tid == 0) atomicOr(status, kStatusTimeoutProducer);
        return;
    }
    // Each thread owns four consecutive channels (d % 4 == 0 here) and walks
    // the rows: one 8- or 16-byte shared-memory read per row, the scales in
    // registers.
    const int G4 = d / 4;
    const int dr = nt / G4;
    const bool active = tid < dr * G4;
    const int c4 = tid % G4, r0 = tid / G4;
    auto load4 = [&](int r, float (&x)[4]) {
        if constexpr (sizeof(T) == 2) {
            const uint2 raw = *reinterpret_cast<const uint2*>(tile + r * d + 4 * c4);
            const T* h = reinterpret_cast<const T*>(&raw);
#pragma unroll
            for (int e = 0; e < 4; ++e) x[e] = to_f32<T>(h[e]);
        } else {
            const float4 raw = *reinterpret_cast<const float4*>(tile + r * d + 4 * c4);
            x[0] = raw.x; x[1] = raw.y; x[2] = raw.z; x[3] = raw.w;
        }
    };
    if (active) {
        float m[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
        for (int r = r0; r < N; r += dr) {
            float x[4];
            load4(r, x);
#pragma unroll
            for (int e = 0; e < 4; ++e) m[e] = fmaxf(m[e], fabsf(x[e]));
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) atomicMax(&amax[4 * c4 + e], __float_as_uint(m[e]));
    }
    __syncthreads();
    for (int c = tid; c < d; c += nt) {
        const float s = __fdiv_rn(__uint_as_float(amax[c]), 127.0f);
        scale[c] = s;
        rscale[c] = __frcp_rn(s);
        sv[bh * d + c] = s;
    }
    __syncthreads();
    if (active) {
        float sc[4], rs[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            sc[e] = scale[4 * c4 + e];
            rs[e] = rscale[4 * c4 + e];
        }
        uint8_t* qrow = qt + (4 * c4) * qs;
        const int rows = (int)ldv;
#pragma unroll 2
        for (int r = r0; r < rows; r += dr) {
            float x[4] = {0.f, 0.f, 0.f, 0.f};
            if (r < N) load4(r, x);
#pragma unroll
            for (int e = 0; e < 4; ++e)
                qrow[e * qs + r] = (uint8_t)((r < N) ? vcode(x[e], sc[e], rs[e]) : 0u);
        }
    }
    __syncthreads();
    const int g16 = (int)(ldv / 16);
    for (int idx = tid; idx < d * g16; idx += nt) {
        const int c = idx / g16, g = idx - c * g16;
        store_codes16(vq + (bh * d + c) * ldv + 16 * g, qt + c * qs + 16 * g);
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
    // Single pass when one (b, h) block of V and its codes fit in shared memory.
    const int64_t small_smem = (int64_t)N * d * sizeof(T) + (int64_t)d * (ldv + 4);
    if ((d * sizeof(T)) % 16 == 0 && aligned(v, 16) && small_smem <= 200 * 1024) {
        auto k = vquant_small_kernel<T>;
        cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)small_smem);
        if (e != cudaSuccess) return e;
        unsigned* status = device_status_ptr();
        if (!status) return cudaErrorInvalidDevice;
        k<<<(unsigned)BH, 512, (size_t)small_smem, st>>>(vp, N, d, ldv, vq, sv, status);
        return cudaGetLastError();
    }
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
