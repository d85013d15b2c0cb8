// ba_prepass.cu -- the fused pre-pass: pack Q, pack K and quantise V in one
// launch.
//
// Method source: the paper-notes page "BinaryAttention: One-Bit QK-Attention
// for Vision and Diffusion Transformers" (CVPR 2026), Key design 1 (sign bits
// and the per-token scale of Q and K) and Key design 3 (channel-wise int8 V).
// These are the two HBM-bound steps in front of the attention kernel.  One CTA
// takes one (b, h): its warps pack the head's N query and N key tokens with
// coalesced loads staged through shared memory, then the CTA quantises the
// head's V (channel absmax, then codes transposed through shared memory,
// reusing the same shared memory).  The routines are the ones the separate
// passes run (ba_prepass.cuh), so the results are bit-identical to
// ba_pack_qk + ba_pack_qk + ba_quant_v.
#include <algorithm>

#include "ba_prepass.cuh"

namespace ba {

cudaError_t launch_pack(const void* x, ba_dtype dt, int64_t tokens, int d, uint32_t* bits,
                        float* mu, cudaStream_t st, int sm_count);
cudaError_t launch_quant_v(const void* v, ba_dtype dt, int B, int H, int N, int d, int8_t* vq,
                           float* sv, cudaStream_t st);
bool prepass_tma_serves(int d, int esize);
int prepass_tma_launches(int N);
cudaError_t launch_prepass_tma(const void* q, const void* k, const void* v, ba_dtype dt, int B, int H, int N, int d,
                               uint32_t* bq, float* muq, uint32_t* bk, float* muk, int8_t* vq, float* sv,
                               cudaStream_t st);

namespace {

// 384 threads at <= 56 registers: three CTAs per SM, so the one-CTA-per-head
// grids of the vision shapes (B H <= 444) are resident in a single wave.
constexpr int kThreads = 384;

template <typename T, int NV>
__global__ void __launch_bounds__(kThreads, 3)
prepass_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v, int N, int d,
               int64_t ldv, uint32_t* __restrict__ bq, float* __restrict__ muq, uint32_t* __restrict__ bk,
               float* __restrict__ muk, int8_t* __restrict__ vq, float* __restrict__ sv)
{
    constexpr int W = (NV * (16 / (int)sizeof(T)) + 31) / 32;
    extern __shared__ __align__(16) uint8_t smem[];
    __shared__ VBlockShared sh;
    const int64_t bh = blockIdx.x;
    const int64_t base = bh * N;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nwarps = blockDim.x >> 5;
    uint4* wbuf = reinterpret_cast<uint4*>(smem) + warp * pack_buffer_slots<NV>();
    pack_tokens_warp<T, NV>(q + base * d, N, d, bq + base * W, muq + base, wbuf, warp, nwarps, lane);
    pack_tokens_warp<T, NV>(k + base * d, N, d, bk + base * W, muk + base, wbuf, warp, nwarps, lane);
    __syncthreads();                    // the code tile below reuses the token buffers
    vblock_quant<T>(v + base * d, N, d, ldv, vq + bh * d * ldv, sv + bh * d, smem, sh);
}

// 16-byte vectors per token when the fused kernel serves head size d, else 0.
int fused_vectors(int N, int d, int esize)
{
    if ((d * esize) % 16 != 0) return 0;
    const int nv = d * esize / 16;
    if (nv != 2 && nv != 4 && nv != 8 && nv != 9 && nv != 12 && nv != 16) return 0;
    return vblock_smem_bytes(N, d) <= kVBlockMaxSmem ? nv : 0;
}

template <typename T, int NV>
cudaError_t launch_fused(const void* q, const void* k, const void* v, int BH, int N, int d, uint32_t* bq,
                         float* muq, uint32_t* bk, float* muk, int8_t* vq, float* sv, cudaStream_t st)
{
    auto kern = prepass_kernel<T, NV>;
    const int64_t tokens_smem = (int64_t)(kThreads / 32) * pack_buffer_slots<NV>() * 16;
    const int64_t smem = std::max(vblock_smem_bytes(N, d), tokens_smem);
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<(unsigned)BH, kThreads, (size_t)smem, st>>>(static_cast<const T*>(q), static_cast<const T*>(k),
                                                        static_cast<const T*>(v), N, d, round_up64(N, 16), bq,
                                                        muq, bk, muk, vq, sv);
    return cudaGetLastError();
}

template <typename T>
cudaError_t launch_fused_t(int nv, const void* q, const void* k, const void* v, int BH, int N, int d,
                           uint32_t* bq, float* muq, uint32_t* bk, float* muk, int8_t* vq, float* sv,
                           cudaStream_t st)
{
    switch (nv) {
#define BA_PREPASS_CASE(NV) \
        case NV: return launch_fused<T, NV>(q, k, v, BH, N, d, bq, muq, bk, muk, vq, sv, st);
        BA_PREPASS_CASE(2) BA_PREPASS_CASE(4) BA_PREPASS_CASE(8) BA_PREPASS_CASE(9) BA_PREPASS_CASE(12)
        BA_PREPASS_CASE(16)
#undef BA_PREPASS_CASE
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

// Kernel launches launch_prepass makes for 16-byte aligned inputs.
int prepass_launch_count(int N, int d, ba_dtype dt)
{
    const int es = dt == BA_BF16 ? 2 : 4;
    const bool v_one_block = (d * es) % 16 == 0 && vblock_smem_bytes(N, d) <= kVBlockMaxSmem;
    if (prepass_tma_serves(d, es)) return prepass_tma_launches(N);
    if (fused_vectors(N, d, es)) return 1;
    return 2 + (v_one_block ? 1 : 3);
}

cudaError_t launch_prepass(const void* q, const void* k, const void* v, ba_dtype dt, int B, int H, int N,
                           int d, uint32_t* bq, float* muq, uint32_t* bk, float* muk, int8_t* vq, float* sv,
                           cudaStream_t st, int sm_count)
{
    const int es = dt == BA_BF16 ? 2 : 4;
    const int nv = fused_vectors(N, d, es);
    const int BH = B * H;
    const bool al16 = aligned(q, 16) && aligned(k, 16) && aligned(v, 16);
    if (al16 && prepass_tma_serves(d, es)) {
        // 128-byte tokens: the TMA-fed kernel (ba_prepass_tma.cu).
        const cudaError_t e = launch_prepass_tma(q, k, v, dt, B, H, N, d, bq, muq, bk, muk, vq, sv, st);
        if (e != cudaErrorNotSupported) return e;
    }
    if (nv && al16) {
        if (dt == BA_BF16)
            return launch_fused_t<__nv_bfloat16>(nv, q, k, v, BH, N, d, bq, muq, bk, muk, vq, sv, st);
        return launch_fused_t<float>(nv, q, k, v, BH, N, d, bq, muq, bk, muk, vq, sv, st);
    }
    const int64_t tokens = (int64_t)BH * N;
    cudaError_t e = launch_pack(q, dt, tokens, d, bq, muq, st, sm_count);
    if (e == cudaSuccess) e = launch_pack(k, dt, tokens, d, bk, muk, st, sm_count);
    if (e == cudaSuccess) e = launch_quant_v(v, dt, B, H, N, d, vq, sv, st);
    return e;
}

}  // namespace ba
