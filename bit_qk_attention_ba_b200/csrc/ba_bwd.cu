// ba_bwd.cu -- the training-side backward pass with straight-through
// estimators, on CUDA cores.
//
// BA notes (paper-notes page "BinaryAttention: One-Bit QK-Attention for
// Vision and Diffusion Transformers", CVPR 2026), Key design 4: quantisation-
// aware training applies sign to Q and K in the forward pass and passes the
// gradient through it with a straight-through estimator (STE).  Readings (the
// page says no more): every quantiser (sign, the u8 rounding of P~, the int8
// rounding of V) passes its gradient straight through, the sign's optionally
// clipped to |x| <= clip; the scale mu = mean |x|, the bias and the softmax
// are differentiated exactly; the row maximum is a constant.  With
// P = P~ / l, P^ = round(255 P~) / (255 l) (what the forward's product used)
// and V^ = sv vq:
//   dV_j   = sum_i P^_ij dO_i
//   dS_ij  = P_ij (dO_i . V^_j - D_i),   D_i = dO_i . O_i  (O: forward output)
//   dz_ij  = dS_ij mu_q,i mu_k,j / sqrt(d)
//   dq_ic  = [|q_ic| <= clip] sum_j dz_ij t_jc + sign(q_ic) / d sum_j dS_ij mu_k,j z_ij / sqrt(d)
//   dk_jc  = [|k_jc| <= clip] sum_i dz_ij s_ic + sign(k_jc) / d sum_i dS_ij mu_q,i z_ij / sqrt(d)
//   dbias += dS (summed over the batch and over every (i, j) reading an entry)
//
// Four launches, each one thread per query row or per key (dq for d <= 32,
// 64 or 128: two threads per row, each with half the channels), the other side
// streamed through shared memory in tiles of 32 tokens:
//   bwd_stats_kernel : exact row maximum m, l = sum_j exp(S - m), D_i
//   bwd_dq2_kernel / bwd_dq_kernel : dq
//   bwd_dk_kernel    : dk (and dbias, added with atomics: the lanes of a warp
//                      hold consecutive keys, so the additions coalesce)
//   bwd_dv_kernel    : dv
// Scores are formed as in the forward's CUDA-core kernel:
// S = (mu_q / sqrt(d)) mu_k z + b in fp32, z = d - 2 popcount(xor).
#include <math.h>

#include "ba_common.cuh"

namespace ba {
namespace bwd {
namespace {

constexpr int TILE = 32;       // tokens of the streamed side per shared-memory tile
constexpr int ROWS = 128;      // threads (rows or keys) per CTA

__device__ __forceinline__ float bias_of(int kind, const float* __restrict__ bias, int64_t ld, int h, int N,
                                         int gh, int gw, int i, int j)
{
    if (kind == BA_BIAS_DENSE) return __ldg(bias + ((int64_t)h * N + i) * ld + j);
    if (kind == BA_BIAS_NONE) return 0.f;
    const int64_t grid = (int64_t)(2 * gh - 1) * (2 * gw - 1);
    if (kind == BA_BIAS_RELPOS2D) {
        const int ri = i / gw, ci = i - ri * gw, rj = j / gw, cj = j - rj * gw;
        return __ldg(bias + h * grid + (int64_t)(ri - rj + gh - 1) * (2 * gw - 1) + (ci - cj + gw - 1));
    }
    const float* t = bias + h * (grid + 3);
    if (i == 0) return __ldg(t + grid + (j == 0 ? 2 : 0));
    if (j == 0) return __ldg(t + grid + 1);
    const int pi = i - 1, pj = j - 1;
    const int ri = pi / gw, ci = pi - ri * gw, rj = pj / gw, cj = pj - rj * gw;
    return __ldg(t + (int64_t)(ri - rj + gh - 1) * (2 * gw - 1) + (ci - cj + gw - 1));
}

// Where the gradient of b_ij goes: dense [H, N, ld], or the table entry.
__device__ __forceinline__ float* dbias_at(int kind, float* dbias, int64_t ld, int h, int N, int gh, int gw, int i,
                                           int j)
{
    if (kind == BA_BIAS_DENSE) return dbias + ((int64_t)h * N + i) * ld + j;
    const int64_t grid = (int64_t)(2 * gh - 1) * (2 * gw - 1);
    if (kind == BA_BIAS_RELPOS2D) {
        const int ri = i / gw, ci = i - ri * gw, rj = j / gw, cj = j - rj * gw;
        return dbias + h * grid + (int64_t)(ri - rj + gh - 1) * (2 * gw - 1) + (ci - cj + gw - 1);
    }
    float* t = dbias + h * (grid + 3);
    if (i == 0) return t + grid + (j == 0 ? 2 : 0);
    if (j == 0) return t + grid + 1;
    const int pi = i - 1, pj = j - 1;
    const int ri = pi / gw, ci = pi - ri * gw, rj = pj / gw, cj = pj - rj * gw;
    return t + (int64_t)(ri - rj + gh - 1) * (2 * gw - 1) + (ci - cj + gw - 1);
}

struct Args {
    const uint32_t* bq; const float* muq; const uint32_t* bk; const float* muk;
    const int8_t* vq; const float* sv;
    int bias_kind; const float* bias; int64_t bias_ld; int gh, gw;
    int H, N, d; int64_t ldv;
    float rsd;                  // 1 / sqrt(d)
    const float* out; const float* dout;
    float* m; float* l; float* D;   // [BH, N] row statistics
};

template <typename T> __device__ __forceinline__ float ld_val(const T* p);
template <> __device__ __forceinline__ float ld_val<float>(const float* p) { return __ldg(p); }
template <> __device__ __forceinline__ float ld_val<__nv_bfloat16>(const __nv_bfloat16* p) { return __bfloat162float(*p); }

// z of the row's bits against a staged token's bits.
template <int W>
__device__ __forceinline__ int zdot(const uint32_t (&a)[W], const uint32_t* b, int d)
{
    int ham = 0;
#pragma unroll
    for (int w = 0; w < W; ++w) ham += __popc(a[w] ^ b[w]);
    return d - 2 * ham;
}

// Row statistics: exact maximum, unquantised sum, D = dO . O.
template <int W>
__global__ void __launch_bounds__(ROWS) bwd_stats_kernel(const Args a)
{
    __shared__ uint32_t s_k[TILE][W];
    __shared__ float s_mu[TILE];
    const int64_t bh = blockIdx.y;
    const int h = (int)(bh % a.H), N = a.N;
    const int i = blockIdx.x * ROWS + threadIdx.x;
    const bool ok = i < N;
    const int ie = ok ? i : N - 1;
    uint32_t q[W];
#pragma unroll
    for (int w = 0; w < W; ++w) q[w] = __ldg(a.bq + (bh * N + ie) * W + w);
    const float cq = __ldg(a.muq + bh * N + ie) * a.rsd;
    float m = -INFINITY, l = 0.f;
    for (int pass = 0; pass < 2; ++pass) {
        for (int j0 = 0; j0 < N; j0 += TILE) {
            __syncthreads();
            for (int e = threadIdx.x; e < TILE * W; e += ROWS) {
                const int r = e / W, w = e - r * W;
                s_k[r][w] = (j0 + r < N) ? __ldg(a.bk + (bh * N + j0 + r) * W + w) : 0u;
            }
            if (threadIdx.x < TILE) s_mu[threadIdx.x] = (j0 + threadIdx.x < N) ? __ldg(a.muk + bh * N + j0 + threadIdx.x) : 0.f;
            __syncthreads();
            const int nk = min(TILE, N - j0);
            for (int jj = 0; jj < nk; ++jj) {
                const float S = fmaf(cq * s_mu[jj], (float)zdot<W>(q, s_k[jj], a.d),
                                     bias_of(a.bias_kind, a.bias, a.bias_ld, h, N, a.gh, a.gw, ie, j0 + jj));
                if (pass == 0) m = fmaxf(m, S);
                else l += expf(S - m);
            }
        }
    }
    if (ok) {
        float Dv = 0.f;
        const float* o = a.out + (bh * N + i) * a.d;
        const float* g = a.dout + (bh * N + i) * a.d;
        for (int c = 0; c < a.d; ++c) Dv = fmaf(__ldg(g + c), __ldg(o + c), Dv);
        a.m[bh * N + i] = m;
        a.l[bh * N + i] = l;
        a.D[bh * N + i] = Dv;
    }
}

// Stage TILE keys of head bh: bits, key scales and dequantised values (float,
// [TILE][32 W], zero past d and past N).
template <int W>
__device__ __forceinline__ void stage_keys(const Args& a, int64_t bh, int j0, uint32_t (*s_k)[W], float* s_mu,
                                           float (*s_v)[32 * W])
{
    const int N = a.N;
    for (int e = threadIdx.x; e < TILE * W; e += blockDim.x) {
        const int r = e / W, w = e - r * W;
        s_k[r][w] = (j0 + r < N) ? __ldg(a.bk + (bh * N + j0 + r) * W + w) : 0u;
    }
    for (int r = threadIdx.x; r < TILE; r += blockDim.x) s_mu[r] = (j0 + r < N) ? __ldg(a.muk + bh * N + j0 + r) : 0.f;
    if (s_v != nullptr)
        for (int e = threadIdx.x; e < TILE * 32 * W; e += blockDim.x) {
            const int c = e / TILE, r = e - c * TILE;      // consecutive threads: consecutive keys of a channel
            float val = 0.f;
            if (c < a.d && j0 + r < N) val = __ldg(a.sv + bh * a.d + c) * (float)a.vq[(bh * a.d + c) * a.ldv + j0 + r];
            s_v[r][c] = val;
        }
}

// dq: one thread per query row.  A dense bias tile (the CTA's rows x TILE
// keys) is staged through shared memory with coalesced loads.
template <int W, typename InT>
__global__ void __launch_bounds__(ROWS) bwd_dq_kernel(const Args a, const InT* __restrict__ q_raw, float clip,
                                                      float* __restrict__ dq)
{
    constexpr int DC = 32 * W;
    __shared__ uint32_t s_k[TILE][W];
    __shared__ float s_mu[TILE];
    __shared__ __align__(16) float s_v[TILE][DC];
    __shared__ float s_b[ROWS][TILE + 1];
    const int64_t bh = blockIdx.y;
    const int h = (int)(bh % a.H), N = a.N, d = a.d;
    const int i = blockIdx.x * ROWS + threadIdx.x;
    const bool ok = i < N;
    const int ie = ok ? i : N - 1;
    uint32_t q[W];
#pragma unroll
    for (int w = 0; w < W; ++w) q[w] = __ldg(a.bq + (bh * N + ie) * W + w);
    const float muq = __ldg(a.muq + bh * N + ie);
    const float cq = muq * a.rsd;
    const float m = a.m[bh * N + ie], inv_l = 1.f / a.l[bh * N + ie], Dv = a.D[bh * N + ie];
    float g[DC], ds[DC];
#pragma unroll
    for (int c = 0; c < DC; ++c) {
        g[c] = (c < d) ? __ldg(a.dout + (bh * N + ie) * d + c) : 0.f;
        ds[c] = 0.f;
    }
    float dmu = 0.f;
    const int row0 = blockIdx.x * ROWS;
    for (int j0 = 0; j0 < N; j0 += TILE) {
        __syncthreads();
        stage_keys<W>(a, bh, j0, s_k, s_mu, s_v);
        if (a.bias_kind == BA_BIAS_DENSE) {
            // warp w loads rows w, w + 4, ...: each row's TILE keys are one 128-byte line
            const int lane = threadIdx.x & 31;
            for (int r = threadIdx.x >> 5; r < ROWS; r += ROWS / 32) {
                const int ii = min(row0 + r, N - 1);
                s_b[r][lane] = (j0 + lane < N) ? __ldg(a.bias + ((int64_t)h * N + ii) * a.bias_ld + j0 + lane) : 0.f;
            }
        }
        __syncthreads();
        const int nk = min(TILE, N - j0);
        for (int jj = 0; jj < nk; ++jj) {
            const int j = j0 + jj;
            const int z = zdot<W>(q, s_k[jj], d);
            const float bij = (a.bias_kind == BA_BIAS_DENSE) ? s_b[threadIdx.x][jj]
                            : bias_of(a.bias_kind, a.bias, a.bias_ld, h, N, a.gh, a.gw, ie, j);
            const float S = fmaf(cq * s_mu[jj], (float)z, bij);
            const float P = expf(S - m) * inv_l;
            float dp = 0.f;
#pragma unroll
            for (int c = 0; c < DC; c += 4) {
                const float4 v4 = *reinterpret_cast<const float4*>(&s_v[jj][c]);
                dp = fmaf(g[c], v4.x, dp);
                dp = fmaf(g[c + 1], v4.y, dp);
                dp = fmaf(g[c + 2], v4.z, dp);
                dp = fmaf(g[c + 3], v4.w, dp);
            }
            const float dS = P * (dp - Dv);
            dmu = fmaf(dS * s_mu[jj], (float)z, dmu);
            const float dz = dS * cq * s_mu[jj];
#pragma unroll
            for (int w = 0; w < W; ++w) {
                const uint32_t bits = s_k[jj][w];
#pragma unroll
                for (int b = 0; b < 32; ++b) ds[32 * w + b] += ((bits >> b) & 1u) ? dz : -dz;
            }
        }
    }
    if (ok) {
        const float dmuq = dmu * a.rsd / (float)d;     // d mu / d q_c = sign(q_c) / d
        const InT* xr = q_raw + (bh * N + i) * d;
        float* dst = dq + (bh * N + i) * d;
#pragma unroll
        for (int c = 0; c < DC; ++c) {
            if (c < d) {
                const float x = ld_val<InT>(xr + c);
                const float sgn = ((q[c >> 5] >> (c & 31)) & 1u) ? 1.f : -1.f;
                dst[c] = (fabsf(x) <= clip ? ds[c] : 0.f) + dmuq * sgn;
            }
        }
    }
}

// dq with a row's channels split over two adjacent threads (half h takes
// channels h DC / 2 .. (h + 1) DC / 2 - 1): half the accumulators per thread,
// so twice the warps per SM; the two halves of dO . V^ meet by one shuffle.
// For W = 1, 2, 4 (each half a whole number of sign words, or half a word).
// The arithmetic of every (row, key, channel) is that of bwd_dq_kernel.
template <int W, typename InT>
__global__ void __launch_bounds__(ROWS) bwd_dq2_kernel(const Args a, const InT* __restrict__ q_raw, float clip,
                                                       float* __restrict__ dq)
{
    constexpr int DC = 32 * W, HC = DC / 2, RPC = ROWS / 2;
    constexpr int VS = DC + 4;                 // s_v row stride; the second half starts 4 floats later
    static_assert(W == 1 || W == 2 || W == 4, "halves of whole sign words");
    __shared__ uint32_t s_k[TILE][W];
    __shared__ float s_mu[TILE];
    __shared__ __align__(16) float s_v[TILE][VS];
    __shared__ float s_b[RPC][TILE + 1];
    const int64_t bh = blockIdx.y;
    const int h = (int)(bh % a.H), N = a.N, d = a.d;
    const int half = threadIdx.x & 1, lr = threadIdx.x >> 1;
    const int c0 = half * HC;                  // first channel of this thread
    const int vo = half * (HC + 4);            // where those channels sit in a row of s_v
    const int i = blockIdx.x * RPC + lr;
    const bool ok = i < N;
    const int ie = ok ? i : N - 1;
    uint32_t q[W];
#pragma unroll
    for (int w = 0; w < W; ++w) q[w] = __ldg(a.bq + (bh * N + ie) * W + w);
    const float muq = __ldg(a.muq + bh * N + ie);
    const float cq = muq * a.rsd;
    const float m = a.m[bh * N + ie], inv_l = 1.f / a.l[bh * N + ie], Dv = a.D[bh * N + ie];
    float g[HC], ds[HC];
#pragma unroll
    for (int cc = 0; cc < HC; ++cc) {
        g[cc] = (c0 + cc < d) ? __ldg(a.dout + (bh * N + ie) * d + c0 + cc) : 0.f;
        ds[cc] = 0.f;
    }
    float dmu = 0.f;
    const int row0 = blockIdx.x * RPC;
    for (int j0 = 0; j0 < N; j0 += TILE) {
        __syncthreads();
        for (int e = threadIdx.x; e < TILE * W; e += ROWS) {
            const int r = e / W, w = e - r * W;
            s_k[r][w] = (j0 + r < N) ? __ldg(a.bk + (bh * N + j0 + r) * W + w) : 0u;
        }
        for (int r = threadIdx.x; r < TILE; r += ROWS) s_mu[r] = (j0 + r < N) ? __ldg(a.muk + bh * N + j0 + r) : 0.f;
        for (int e = threadIdx.x; e < TILE * DC; e += ROWS) {
            const int c = e / TILE, r = e - c * TILE;      // consecutive threads: consecutive keys of a channel
            float val = 0.f;
            if (c < d && j0 + r < N) val = __ldg(a.sv + bh * d + c) * (float)a.vq[(bh * d + c) * a.ldv + j0 + r];
            s_v[r][c + (c >= HC ? 4 : 0)] = val;
        }
        if (a.bias_kind == BA_BIAS_DENSE) {
            const int lane = threadIdx.x & 31;
            for (int r = threadIdx.x >> 5; r < RPC; r += ROWS / 32) {
                const int ii = min(row0 + r, N - 1);
                s_b[r][lane] = (j0 + lane < N) ? __ldg(a.bias + ((int64_t)h * N + ii) * a.bias_ld + j0 + lane) : 0.f;
            }
        }
        __syncthreads();
        const int nk = min(TILE, N - j0);
        for (int jj = 0; jj < nk; ++jj) {
            const int j = j0 + jj;
            const int z = zdot<W>(q, s_k[jj], d);
            const float bij = (a.bias_kind == BA_BIAS_DENSE) ? s_b[lr][jj]
                            : bias_of(a.bias_kind, a.bias, a.bias_ld, h, N, a.gh, a.gw, ie, j);
            const float S = fmaf(cq * s_mu[jj], (float)z, bij);
            const float P = expf(S - m) * inv_l;
            float dp = 0.f;
#pragma unroll
            for (int cc = 0; cc < HC; cc += 4) {
                const float4 v4 = *reinterpret_cast<const float4*>(&s_v[jj][vo + cc]);
                dp = fmaf(g[cc], v4.x, dp);
                dp = fmaf(g[cc + 1], v4.y, dp);
                dp = fmaf(g[cc + 2], v4.z, dp);
                dp = fmaf(g[cc + 3], v4.w, dp);
            }
            dp += __shfl_xor_sync(0xffffffffu, dp, 1);
            const float dS = P * (dp - Dv);
            dmu = fmaf(dS * s_mu[jj], (float)z, dmu);
            const float dz = dS * cq * s_mu[jj];
#pragma unroll
            for (int w = 0; w < (W == 1 ? 1 : W / 2); ++w) {
                const uint32_t bits = (W == 1) ? (s_k[jj][0] >> (16 * half)) : s_k[jj][half * (W / 2) + w];
#pragma unroll
                for (int b = 0; b < (W == 1 ? 16 : 32); ++b) ds[32 * w + b] += ((bits >> b) & 1u) ? dz : -dz;
            }
        }
    }
    if (ok) {
        const float dmuq = dmu * a.rsd / (float)d;     // d mu / d q_c = sign(q_c) / d
        const InT* xr = q_raw + (bh * N + i) * d;
        float* dst = dq + (bh * N + i) * d;
#pragma unroll
        for (int cc = 0; cc < HC; ++cc) {
            const int c = c0 + cc;
            if (c < d) {
                const float x = ld_val<InT>(xr + c);
                const float sgn = ((q[c >> 5] >> (c & 31)) & 1u) ? 1.f : -1.f;
                dst[c] = (fabsf(x) <= clip ? ds[cc] : 0.f) + dmuq * sgn;
            }
        }
    }
}

// Stage TILE query rows of head bh: bits, scales, row statistics, dO rows.
template <int W>
__device__ __forceinline__ void stage_rows(const Args& a, int64_t bh, int i0, uint32_t (*s_q)[W], float* s_mu,
                                           float* s_m, float* s_il, float* s_D, float (*s_g)[32 * W])
{
    const int N = a.N;
    for (int e = threadIdx.x; e < TILE * W; e += blockDim.x) {
        const int r = e / W, w = e - r * W;
        s_q[r][w] = (i0 + r < N) ? __ldg(a.bq + (bh * N + i0 + r) * W + w) : 0u;
    }
    for (int r = threadIdx.x; r < TILE; r += blockDim.x) {
        const bool ok = i0 + r < N;
        s_mu[r] = ok ? __ldg(a.muq + bh * N + i0 + r) : 0.f;
        s_m[r] = ok ? a.m[bh * N + i0 + r] : 0.f;
        s_il[r] = ok ? 1.f / a.l[bh * N + i0 + r] : 0.f;
        if (s_D) s_D[r] = ok ? a.D[bh * N + i0 + r] : 0.f;
    }
    for (int e = threadIdx.x; e < TILE * 32 * W; e += blockDim.x) {
        const int r = e / (32 * W), c = e - r * (32 * W);
        s_g[r][c] = (c < a.d && i0 + r < N) ? __ldg(a.dout + (bh * N + i0 + r) * a.d + c) : 0.f;
    }
}

// dk: one thread per key; dbias (optional) receives dS by atomics.
template <int W, typename InT>
__global__ void __launch_bounds__(ROWS) bwd_dk_kernel(const Args a, const InT* __restrict__ k_raw, float clip,
                                                      float* __restrict__ dk, float* __restrict__ dbias)
{
    constexpr int DC = 32 * W;
    __shared__ uint32_t s_q[TILE][W];
    __shared__ float s_mu[TILE], s_m[TILE], s_il[TILE], s_D[TILE];
    __shared__ __align__(16) float s_g[TILE][DC];
    const int64_t bh = blockIdx.y;
    const int h = (int)(bh % a.H), N = a.N, d = a.d;
    const int j = blockIdx.x * ROWS + threadIdx.x;
    const bool ok = j < N;
    const int je = ok ? j : N - 1;
    uint32_t kb[W];
#pragma unroll
    for (int w = 0; w < W; ++w) kb[w] = __ldg(a.bk + (bh * N + je) * W + w);
    const float muk = __ldg(a.muk + bh * N + je);
    float vh[DC], dt[DC];
#pragma unroll
    for (int c = 0; c < DC; ++c) {
        vh[c] = (c < d) ? __ldg(a.sv + bh * d + c) * (float)a.vq[(bh * d + c) * a.ldv + je] : 0.f;
        dt[c] = 0.f;
    }
    float dmu = 0.f;
    for (int i0 = 0; i0 < N; i0 += TILE) {
        __syncthreads();
        stage_rows<W>(a, bh, i0, s_q, s_mu, s_m, s_il, s_D, s_g);
        __syncthreads();
        const int nr = min(TILE, N - i0);
        for (int ii = 0; ii < nr; ++ii) {
            const int i = i0 + ii;
            const int z = zdot<W>(s_q[ii], kb, d);
            const float cq = s_mu[ii] * a.rsd;
            const float S = fmaf(cq * muk, (float)z, bias_of(a.bias_kind, a.bias, a.bias_ld, h, N, a.gh, a.gw, i, je));
            const float P = expf(S - s_m[ii]) * s_il[ii];
            float dp = 0.f;
#pragma unroll
            for (int c = 0; c < DC; c += 4) {
                const float4 g4 = *reinterpret_cast<const float4*>(&s_g[ii][c]);
                dp = fmaf(g4.x, vh[c], dp);
                dp = fmaf(g4.y, vh[c + 1], dp);
                dp = fmaf(g4.z, vh[c + 2], dp);
                dp = fmaf(g4.w, vh[c + 3], dp);
            }
            const float dS = P * (dp - s_D[ii]);
            dmu = fmaf(dS * s_mu[ii], (float)z, dmu);
            const float dz = dS * cq * muk;
#pragma unroll
            for (int w = 0; w < W; ++w) {
                const uint32_t bits = s_q[ii][w];
#pragma unroll
                for (int b = 0; b < 32; ++b) dt[32 * w + b] += ((bits >> b) & 1u) ? dz : -dz;
            }
            if (dbias != nullptr && ok) atomicAdd(dbias_at(a.bias_kind, dbias, a.bias_ld, h, N, a.gh, a.gw, i, j), dS);
        }
    }
    if (ok) {
        const float dmuk = dmu * a.rsd / (float)d;
        const InT* xr = k_raw + (bh * N + j) * d;
        float* dst = dk + (bh * N + j) * d;
#pragma unroll
        for (int c = 0; c < DC; ++c) {
            if (c < d) {
                const float x = ld_val<InT>(xr + c);
                const float sgn = ((kb[c >> 5] >> (c & 31)) & 1u) ? 1.f : -1.f;
                dst[c] = (fabsf(x) <= clip ? dt[c] : 0.f) + dmuk * sgn;
            }
        }
    }
}

// dv: one thread per key, dv_j = sum_i round(255 P~_ij) / (255 l_i) dO_i.
template <int W>
__global__ void __launch_bounds__(ROWS) bwd_dv_kernel(const Args a, float* __restrict__ dv)
{
    constexpr int DC = 32 * W;
    __shared__ uint32_t s_q[TILE][W];
    __shared__ float s_mu[TILE], s_m[TILE], s_il[TILE];
    __shared__ __align__(16) float s_g[TILE][DC];
    const int64_t bh = blockIdx.y;
    const int h = (int)(bh % a.H), N = a.N, d = a.d;
    const int j = blockIdx.x * ROWS + threadIdx.x;
    const bool ok = j < N;
    const int je = ok ? j : N - 1;
    uint32_t kb[W];
#pragma unroll
    for (int w = 0; w < W; ++w) kb[w] = __ldg(a.bk + (bh * N + je) * W + w);
    const float muk = __ldg(a.muk + bh * N + je);
    float acc[DC];
#pragma unroll
    for (int c = 0; c < DC; ++c) acc[c] = 0.f;
    for (int i0 = 0; i0 < N; i0 += TILE) {
        __syncthreads();
        stage_rows<W>(a, bh, i0, s_q, s_mu, s_m, s_il, nullptr, s_g);
        __syncthreads();
        const int nr = min(TILE, N - i0);
        for (int ii = 0; ii < nr; ++ii) {
            const int i = i0 + ii;
            const int z = zdot<W>(s_q[ii], kb, d);
            const float S = fmaf(s_mu[ii] * a.rsd * muk, (float)z,
                                 bias_of(a.bias_kind, a.bias, a.bias_ld, h, N, a.gh, a.gw, i, je));
            const float Ph = (float)__float2int_rn(255.f * expf(S - s_m[ii])) * (s_il[ii] * (1.f / 255.f));
#pragma unroll
            for (int c = 0; c < DC; c += 4) {
                const float4 g4 = *reinterpret_cast<const float4*>(&s_g[ii][c]);
                acc[c] = fmaf(Ph, g4.x, acc[c]);
                acc[c + 1] = fmaf(Ph, g4.y, acc[c + 1]);
                acc[c + 2] = fmaf(Ph, g4.z, acc[c + 2]);
                acc[c + 3] = fmaf(Ph, g4.w, acc[c + 3]);
            }
        }
    }
    if (ok) {
        float* dst = dv + (bh * N + j) * d;
#pragma unroll
        for (int c = 0; c < DC; ++c)
            if (c < d) dst[c] = acc[c];
    }
}

template <int W, typename InT>
cudaError_t launch_w(const Args& a, int BH, const InT* q, const InT* k, float clip, float* dq, float* dk, float* dv,
                     float* dbias, cudaStream_t st)
{
    dim3 grid(ceil_div(a.N, ROWS), BH);
    bwd_stats_kernel<W><<<grid, ROWS, 0, st>>>(a);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    if constexpr (W == 3) {
        bwd_dq_kernel<W, InT><<<grid, ROWS, 0, st>>>(a, q, clip, dq);
    } else {
        dim3 grid2(ceil_div(a.N, ROWS / 2), BH);
        bwd_dq2_kernel<W, InT><<<grid2, ROWS, 0, st>>>(a, q, clip, dq);
    }
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    bwd_dk_kernel<W, InT><<<grid, ROWS, 0, st>>>(a, k, clip, dk, dbias);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    bwd_dv_kernel<W><<<grid, ROWS, 0, st>>>(a, dv);
    return cudaGetLastError();
}

template <typename InT>
cudaError_t launch_t(const Args& a, int BH, const InT* q, const InT* k, float clip, float* dq, float* dk, float* dv,
                     float* dbias, cudaStream_t st)
{
    switch (words_for(a.d)) {
        case 1: return launch_w<1, InT>(a, BH, q, k, clip, dq, dk, dv, dbias, st);
        case 2: return launch_w<2, InT>(a, BH, q, k, clip, dq, dk, dv, dbias, st);
        case 3: return launch_w<3, InT>(a, BH, q, k, clip, dq, dk, dv, dbias, st);
        default: return launch_w<4, InT>(a, BH, q, k, clip, dq, dk, dv, dbias, st);
    }
}

}  // namespace
}  // namespace bwd

int64_t attn_bwd_workspace_bytes(int B, int H, int N) { return 3 * round_up64((int64_t)B * H * N * 4, 256); }

int64_t attn_bwd_dbias_elems(int bias_kind, int H, int N, int64_t ld, int gh, int gw)
{
    if (bias_kind == BA_BIAS_DENSE) return (int64_t)H * N * ld;
    if (bias_kind == BA_BIAS_RELPOS2D) return (int64_t)H * (2 * gh - 1) * (2 * gw - 1);
    if (bias_kind == BA_BIAS_RELPOS2D_CLS) return (int64_t)H * ((2 * gh - 1) * (2 * gw - 1) + 3);
    return 0;
}

cudaError_t launch_attn_bwd(const void* q, const void* k, ba_dtype dt, const uint32_t* bq, const float* muq,
                            const uint32_t* bk, const float* muk, const int8_t* vq, const float* sv, int bias_kind,
                            const float* bias, int64_t bias_ld, int gh, int gw, int B, int H, int N, int d,
                            const float* out, const float* dout, float clip, void* workspace, float* dq, float* dk,
                            float* dv, float* dbias, cudaStream_t st)
{
    bwd::Args a;
    a.bq = bq; a.muq = muq; a.bk = bk; a.muk = muk; a.vq = vq; a.sv = sv;
    a.bias_kind = bias_kind; a.bias = bias; a.bias_ld = bias_ld; a.gh = gh; a.gw = gw;
    a.H = H; a.N = N; a.d = d; a.ldv = round_up64(N, 16);
    a.rsd = (float)(1.0 / sqrt((double)d));
    a.out = out; a.dout = dout;
    const int64_t stat = round_up64((int64_t)B * H * N * 4, 256);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    a.m = reinterpret_cast<float*>(ws);
    a.l = reinterpret_cast<float*>(ws + stat);
    a.D = reinterpret_cast<float*>(ws + 2 * stat);
    if (dbias != nullptr && bias_kind != BA_BIAS_NONE) {
        const cudaError_t e = cudaMemsetAsync(dbias, 0, attn_bwd_dbias_elems(bias_kind, H, N, bias_ld, gh, gw) * 4, st);
        if (e != cudaSuccess) return e;
    } else {
        dbias = nullptr;
    }
    if (dt == BA_BF16)
        return bwd::launch_t<__nv_bfloat16>(a, B * H, static_cast<const __nv_bfloat16*>(q),
                                            static_cast<const __nv_bfloat16*>(k), clip, dq, dk, dv, dbias, st);
    return bwd::launch_t<float>(a, B * H, static_cast<const float*>(q), static_cast<const float*>(k), clip, dq, dk,
                                dv, dbias, st);
}

}  // namespace ba
