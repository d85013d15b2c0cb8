// ba_attn_simt.cu -- the BinaryAttention forward on CUDA cores only.
//
// QK variant "popc": every score is d - 2 popcount(XOR) over 32-bit words
// (BA notes, Key design 1), scaled and biased (Key design 2).  The keys are
// walked twice in tiles of 32 staged in shared memory (Overall framework):
// the first sweep finds the exact row maximum, the second quantises
// P~ = exp(S - m) to u8 with scale 1/255 and multiplies it with the int8 V
// codes by dp4a (u8 x s8 -> s32), Key design 3.  One thread owns one query
// row.  This is the plain, any-shape path and
// the CUDA-core point of the QK variant comparison; the tensor-core kernel is
// in ba_attn_tc.cu.
#include <math.h>

#include "ba_common.cuh"

namespace ba {

__device__ __forceinline__ int dp4a_u8s8(uint32_t a_u8x4, uint32_t b_s8x4, int c)
{
    int d;
    asm("dp4a.u32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a_u8x4), "r"(b_s8x4), "r"(c));
    return d;
}

__device__ __forceinline__ float bias_at(int kind, const float* __restrict__ bias, int64_t ld,
                                         int h, int N, int gh, int gw, int i, int j)
{
    if (kind == BA_BIAS_DENSE) return __ldg(bias + ((int64_t)h * N + i) * ld + j);
    if (kind == BA_BIAS_RELPOS2D) {
        const int ri = i / gw, ci = i - ri * gw, rj = j / gw, cj = j - rj * gw;
        const int64_t per_head = (int64_t)(2 * gh - 1) * (2 * gw - 1);
        return __ldg(bias + h * per_head + (int64_t)(ri - rj + gh - 1) * (2 * gw - 1) + (ci - cj + gw - 1));
    }
    if (kind == BA_BIAS_RELPOS2D_CLS) {   // token 0 is the class token; three class entries follow the grid
        const int64_t grid = (int64_t)(2 * gh - 1) * (2 * gw - 1);
        const float* t = bias + h * (grid + 3);
        if (i == 0) return __ldg(t + grid + (j == 0 ? 2 : 0));
        if (j == 0) return __ldg(t + grid + 1);
        const int pi = i - 1, pj = j - 1;
        const int ri = pi / gw, ci = pi - ri * gw, rj = pj / gw, cj = pj - rj * gw;
        return __ldg(t + (int64_t)(ri - rj + gh - 1) * (2 * gw - 1) + (ci - cj + gw - 1));
    }
    return 0.f;
}

template <typename OutT> __device__ __forceinline__ void store_out(OutT* p, float v);
template <> __device__ __forceinline__ void store_out<float>(float* p, float v) { *p = v; }
template <> __device__ __forceinline__ void store_out<__nv_bfloat16>(__nv_bfloat16* p, float v) { *p = __float2bfloat16_rn(v); }

// W words per token (d <= 32 W); the accumulator holds 32 W channels.
template <int W, typename OutT>
__global__ void __launch_bounds__(128)
attn_simt_kernel(const uint32_t* __restrict__ bq, const float* __restrict__ muq,
                 const uint32_t* __restrict__ bk, const float* __restrict__ muk,
                 const int8_t* __restrict__ vq, const float* __restrict__ sv,
                 int bias_kind, const float* __restrict__ bias, int64_t bias_ld, int gh, int gw,
                 int H, int N, int d, int64_t ldv, OutT* __restrict__ out)
{
    constexpr int KT = 32;           // keys per tile
    constexpr int DV = 32 * W;       // channels held per row
    __shared__ uint32_t s_k[KT][W];
    __shared__ float s_muk[KT];
    __shared__ __align__(16) uint32_t s_v[DV][KT / 4];   // int8 codes, 4 keys per word

    const int64_t bh = blockIdx.y;
    const int h = (int)(bh % H);
    const int i = blockIdx.x * 128 + threadIdx.x;
    const bool row_ok = i < N;

    uint32_t q[W];
#pragma unroll
    for (int w = 0; w < W; ++w) q[w] = row_ok ? bq[(bh * N + i) * W + w] : 0u;
    const float cq = row_ok ? muq[bh * N + i] / sqrtf((float)d) : 0.f;

    // Pass A: the exact row maximum.  Pass B: P~ = exp(S - m) against it, so
    // the u8 codes need no later rescaling and the PV sum stays in int32.
    float m = -INFINITY, l = 0.f;
    int acc[DV];
#pragma unroll
    for (int c = 0; c < DV; ++c) acc[c] = 0;

    for (int pass = 0; pass < 2; ++pass) {
        for (int j0 = 0; j0 < N; j0 += KT) {
            __syncthreads();
            for (int idx = threadIdx.x; idx < KT * W; idx += blockDim.x) {
                const int r = idx / W, w = idx - r * W;
                s_k[r][w] = (j0 + r < N) ? bk[(bh * N + j0 + r) * W + w] : 0u;
            }
            if (threadIdx.x < KT) s_muk[threadIdx.x] = (j0 + threadIdx.x < N) ? muk[bh * N + j0 + threadIdx.x] : 0.f;
            if (pass == 1) {
                for (int idx = threadIdx.x; idx < DV * 2; idx += blockDim.x) {   // two 16-byte halves per channel
                    const int c = idx >> 1, half = idx & 1;
                    const int64_t col = (int64_t)j0 + half * 16;
                    uint4 val = make_uint4(0u, 0u, 0u, 0u);
                    if (c < d && col < ldv) val = *reinterpret_cast<const uint4*>(vq + (bh * d + c) * ldv + col);
                    *reinterpret_cast<uint4*>(&s_v[c][half * 4]) = val;
                }
            }
            __syncthreads();

            float s[KT];
#pragma unroll
            for (int jj = 0; jj < KT; ++jj) {
                const int j = j0 + jj;
                float val = -INFINITY;
                if (j < N) {
                    int ham = 0;
#pragma unroll
                    for (int w = 0; w < W; ++w) ham += __popc(q[w] ^ s_k[jj][w]);
                    const float z = (float)(d - 2 * ham);
                    const float b = row_ok ? bias_at(bias_kind, bias, bias_ld, h, N, gh, gw, i, j) : 0.f;
                    val = fmaf(cq * s_muk[jj], z, b);
                }
                s[jj] = val;
                if (pass == 0) m = fmaxf(m, val);
            }
            if (pass == 0) continue;

            uint32_t pw[KT / 4];
#pragma unroll
            for (int w = 0; w < KT / 4; ++w) pw[w] = 0u;
#pragma unroll
            for (int jj = 0; jj < KT; ++jj) {
                const float p = expf(s[jj] - m);
                l += p;
                const uint32_t pq = (uint32_t)__float2int_rn(255.f * p);
                pw[jj >> 2] |= pq << (8 * (jj & 3));
            }
#pragma unroll
            for (int c = 0; c < DV; ++c) {
#pragma unroll
                for (int w = 0; w < KT / 4; ++w) acc[c] = dp4a_u8s8(pw[w], s_v[c][w], acc[c]);
            }
        }
    }

    if (row_ok) {
        const float inv = 1.f / (255.f * l);
        OutT* dst = out + (bh * N + i) * d;
#pragma unroll
        for (int c = 0; c < DV; ++c)
            if (c < d) store_out<OutT>(dst + c, sv[bh * d + c] * (float)acc[c] * inv);
    }
}

template <typename OutT>
static cudaError_t launch_simt_t(const uint32_t* bq, const float* muq, const uint32_t* bk, const float* muk,
                                 const int8_t* vq, const float* sv, int bias_kind, const float* bias,
                                 int64_t bias_ld, int gh, int gw, int B, int H, int N, int d,
                                 OutT* out, cudaStream_t st)
{
    dim3 grid(ceil_div(N, 128), (unsigned)((int64_t)B * H));
    const int64_t ldv = round_up64(N, 16);
#define BA_SIMT_CASE(WW) \
    attn_simt_kernel<WW, OutT><<<grid, 128, 0, st>>>(bq, muq, bk, muk, vq, sv, bias_kind, bias, bias_ld, \
                                                     gh, gw, H, N, d, ldv, out)
    switch (words_for(d)) {
        case 1: BA_SIMT_CASE(1); break;
        case 2: BA_SIMT_CASE(2); break;
        case 3: BA_SIMT_CASE(3); break;
        default: BA_SIMT_CASE(4); break;
    }
#undef BA_SIMT_CASE
    return cudaGetLastError();
}

cudaError_t launch_attn_simt(const uint32_t* bq, const float* muq, const uint32_t* bk, const float* muk,
                             const int8_t* vq, const float* sv, int bias_kind, const float* bias,
                             int64_t bias_ld, int gh, int gw, int B, int H, int N, int d,
                             void* out, ba_dtype out_dt, cudaStream_t st)
{
    if (out_dt == BA_BF16)
        return launch_simt_t<__nv_bfloat16>(bq, muq, bk, muk, vq, sv, bias_kind, bias, bias_ld, gh, gw,
                                            B, H, N, d, static_cast<__nv_bfloat16*>(out), st);
    return launch_simt_t<float>(bq, muq, bk, muk, vq, sv, bias_kind, bias, bias_ld, gh, gw,
                                B, H, N, d, static_cast<float*>(out), st);
}

}  // namespace ba
