// ba_decode.cu -- the BinaryAttention forward in decode shape: Nq (<= 16)
// query tokens of each (batch, head) attend to an Nk-token cache of packed
// key sign bits, key scales and int8 value codes.
//
// Method source: the paper-notes page "BinaryAttention: One-Bit QK-Attention
// for Vision and Diffusion Transformers" (CVPR 2026).  Key designs 1-3 define
// the arithmetic (z = d - 2 popc(q XOR k); S = z mu_q mu_k / sqrt(d) + b;
// u8 P~ codes against the exact row maximum, int8 V, int32 PV); the page's
// "Related work and inspiration" section names a compressed KV cache for LLM
// inference as the place the binary scores carry over to, which is this
// shape: a 1-bit key cache (d / 8 bytes per key) and an int8 value cache.
//
// With few query rows the work is streaming the cache from HBM, so the keys
// are split over CTAs (split s of a head takes keys [s C, s C + C)), and the
// exact-maximum reading survives the split: one launch takes each split's row
// maxima, the next reduces them to the exact maximum m_i, quantises
// P~ = exp(S - m_i) to u8 codes against it and forms each split's int32 PV
// sums and P~ row sums; since every split quantises against the same m_i,
// adding the splits' integer sums is exact.  The last split CTA of each head
// to finish (an atomic ticket) adds the splits and applies the epilogue
// O = sv acc / (255 l).  The second launch bulk-copies its split's V code
// rows into shared memory first, so they stream in while the codes are formed.
#include <math.h>

#include <algorithm>

#include "ba_common.cuh"
#include "ba_sm100.cuh"

namespace ba {
namespace dec {

constexpr int MAXQ = 16;          // query rows per head this path serves
constexpr int THREADS = 256;
constexpr int MAX_CHUNK = 1024;   // keys per split
constexpr int V_TILE = 64 * 1024; // at most this many V code bytes of a split in shared memory
constexpr uint64_t kCopyWaitNs = 2000000000ull;
constexpr float LOG2E = 1.4426950408889634f;

struct Params {
    const uint32_t* bq;
    const float* muq;
    const uint32_t* bk;
    const float* muk;
    const int8_t* vq;
    const float* sv;
    const float* bias;   // dense [H, Nq, bias_ld] or null
    int64_t bias_ld;
    int H, Nq, Nk, d, S, C;
    int SA, CA;          // splits of the maximum sweep (wider: its per-key work is small)
    int bk_vec;          // key bits 4 W-byte aligned: one vector load per key (W = 2 or 4)
    int64_t ldv;
    float* pmax;         // [BH][SA][Nq] row maxima of the maximum sweep's splits
    float* psum;         // [BH][S][Nq] split sums of P~
    int* pacc;           // [BH][S][Nq][d] int32 PV sums of each split
    unsigned* ticket;    // [BH] split CTAs of the head done (zeroed by the maximum sweep)
    void* out;
    int out_bf16;
    unsigned* status;
};

// Row stride of a split's V codes in shared memory: C + 16 bytes, an odd
// number of 16-byte chunks (C % 16 == 0), so 16-byte reads of consecutive
// channels hit distinct bank groups.
__host__ __device__ inline int v_stride(int C) { return C + 16; }

// Dynamic shared memory of decode_pv_kernel: the split's V codes [d][C + 16],
// the u8 P codes [Nq][C] and the int32 PV sums [Nq][d].
__host__ __device__ inline int pv_smem_bytes(int d, int Nq, int C) { return d * v_stride(C) + Nq * C + Nq * d * 4; }

__device__ __forceinline__ int dp4a_u8s8(uint32_t a_u8x4, uint32_t b_s8x4, int c)
{
    int r;
    asm("dp4a.u32.s32 %0, %1, %2, %3;" : "=r"(r) : "r"(a_u8x4), "r"(b_s8x4), "r"(c));
    return r;
}

// atomicAdd(ticket, 1) with release and acquire semantics at GPU scope.
__device__ __forceinline__ unsigned ticket_acq_rel(unsigned* ticket)
{
    unsigned old;
    asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], 1;" : "=r"(old) : "l"(ticket) : "memory");
    return old;
}

__device__ __forceinline__ float ex2(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// The query side of head bh in shared memory: sign words and mu_q / sqrt(d).
template <int W>
__device__ __forceinline__ void load_queries(const Params& p, int64_t bh, uint32_t (&qs)[MAXQ][W], float (&cq)[MAXQ])
{
    const float rsd = 1.f / sqrtf((float)p.d);
    for (int e = threadIdx.x; e < p.Nq * W; e += blockDim.x) {
        const int i = e / W, w = e - i * W;
        qs[i][w] = __ldg(p.bq + (bh * p.Nq + i) * W + w);
    }
    for (int i = threadIdx.x; i < p.Nq; i += blockDim.x) cq[i] = __ldg(p.muq + bh * p.Nq + i) * rsd;
}

// The W sign words of key j: one 8- or 16-byte load when the rows are aligned for it.
template <int W>
__device__ __forceinline__ void load_key(const Params& p, int64_t bh, int j, uint32_t (&kb)[W])
{
    const uint32_t* src = p.bk + (bh * p.Nk + j) * W;
    if constexpr (W == 2) {
        if (p.bk_vec) {
            const uint2 t = __ldg(reinterpret_cast<const uint2*>(src));
            kb[0] = t.x;
            kb[1] = t.y;
            return;
        }
    } else if constexpr (W == 4) {
        if (p.bk_vec) {
            const uint4 t = __ldg(reinterpret_cast<const uint4*>(src));
            kb[0] = t.x; kb[1] = t.y; kb[2] = t.z; kb[3] = t.w;
            return;
        }
    }
#pragma unroll
    for (int w = 0; w < W; ++w) kb[w] = __ldg(src + w);
}

// S_ij for key j of head bh (same expression in both sweeps, so the second
// sweep reproduces the first's values bit for bit).
template <int W>
__device__ __forceinline__ float score(const Params& p, int h, const uint32_t (&kb)[W], float mk,
                                       const uint32_t (&qs)[MAXQ][W], const float (&cq)[MAXQ], int i, int j)
{
    int ham = 0;
#pragma unroll
    for (int w = 0; w < W; ++w) ham += __popc(qs[i][w] ^ kb[w]);
    const float b = p.bias ? __ldg(p.bias + ((int64_t)h * p.Nq + i) * p.bias_ld + j) : 0.f;
    return fmaf((float)(p.d - 2 * ham) * mk, cq[i], b);
}

// Block-wide reduction of NQ per-thread values (max or sum), lane order
// fixed; result in red[i] for every thread after the call.
template <bool IS_MAX, int NQ>
__device__ __forceinline__ void block_reduce(float (&v)[NQ], int nq, float (&red)[THREADS / 32][MAXQ],
                                             float (&out)[MAXQ])
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int i = 0; i < NQ; ++i) {
        if (i >= nq) break;
        float x = v[i];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const float y = __shfl_xor_sync(0xffffffffu, x, o);
            x = IS_MAX ? fmaxf(x, y) : x + y;
        }
        if (lane == 0) red[warp][i] = x;
    }
    __syncthreads();
    if (threadIdx.x < nq) {
        float x = red[0][threadIdx.x];
        for (int w = 1; w < THREADS / 32; ++w) x = IS_MAX ? fmaxf(x, red[w][threadIdx.x]) : x + red[w][threadIdx.x];
        out[threadIdx.x] = x;
    }
    __syncthreads();
}

// Sweep 1: the row maxima of split blockIdx.x of head blockIdx.y.
// NQ: the compile-time bound on the query rows (1, or MAXQ for 2 .. MAXQ).
template <int W, int NQ>
__global__ void __launch_bounds__(THREADS, 4)
decode_max_kernel(const Params p)
{
    __shared__ uint32_t qs[MAXQ][W];
    __shared__ float cq[MAXQ];
    __shared__ float red[THREADS / 32][MAXQ];
    __shared__ float res[MAXQ];
    const int s = blockIdx.x;
    const int64_t bh = blockIdx.y;
    const int h = (int)(bh % p.H);
    if (s == 0 && threadIdx.x == 0) p.ticket[bh] = 0u;   // for the P.V launch after this one
    load_queries<W>(p, bh, qs, cq);
    __syncthreads();
    float mx[NQ];
#pragma unroll
    for (int i = 0; i < NQ; ++i) mx[i] = -INFINITY;
    const int j1 = min(p.Nk, (s + 1) * p.CA);
    // KB keys per thread in flight: their loads first, then the scores.
    constexpr int KB = NQ == 1 ? 8 : 4;
    for (int j = s * p.CA + threadIdx.x; j < j1; j += KB * blockDim.x) {
        uint32_t kb[KB][W];
        float mk[KB];
#pragma unroll
        for (int u = 0; u < KB; ++u) {
            const int ju = j + u * blockDim.x;
            if (ju < j1) {
                load_key<W>(p, bh, ju, kb[u]);
                mk[u] = __ldg(p.muk + bh * p.Nk + ju);
            }
        }
#pragma unroll
        for (int u = 0; u < KB; ++u) {
            const int ju = j + u * blockDim.x;
            if (ju >= j1) break;
#pragma unroll
            for (int i = 0; i < NQ; ++i) {
                if (i >= p.Nq) break;
                mx[i] = fmaxf(mx[i], score<W>(p, h, kb[u], mk[u], qs, cq, i, ju));
            }
        }
    }
    block_reduce<true, NQ>(mx, p.Nq, red, res);
    if (threadIdx.x < p.Nq) p.pmax[(bh * p.SA + s) * p.Nq + threadIdx.x] = res[threadIdx.x];
}

// Sweep 2: exact m_i from the split maxima, u8 codes of this split's keys,
// the split's P~ sums and int32 PV sums.  The split's V code rows are
// bulk-copied into shared memory first, so they stream in while the codes
// are formed.
template <int W, int NQ>
__global__ void __launch_bounds__(THREADS, 3)
decode_pv_kernel(const Params p)
{
    extern __shared__ __align__(16) uint8_t dsm[];
    __shared__ __align__(8) uint64_t vbar;
    __shared__ uint32_t qs[MAXQ][W];
    __shared__ float cq[MAXQ];
    __shared__ float negm[MAXQ];
    __shared__ float red[THREADS / 32][MAXQ];
    __shared__ float res[MAXQ];
    const int s = blockIdx.x;
    const int64_t bh = blockIdx.y;
    const int h = (int)(bh % p.H);
    const int d = p.d;
    const int j0 = s * p.C;
    const int len = min(p.Nk - j0, p.C);
    const int len16 = (len + 15) & ~15;       // <= ldv - j0: the copies stay inside the code rows
    const int vst = v_stride(p.C);
    uint8_t* vt = dsm;                        // [d][vst] V codes of keys j0 .. j0 + len16
    uint8_t* pq = dsm + (size_t)d * vst;      // [Nq][C] u8 P codes
    int* sacc = reinterpret_cast<int*>(pq + (size_t)p.Nq * p.C);   // [Nq][d] PV sums
    if (threadIdx.x == 0) {
        sm100::mbar_init(&vbar, 1);
        sm100::fence_mbar_init();
        sm100::mbar_arrive_expect_tx(&vbar, (uint32_t)(d * len16));
    }
    __syncthreads();
    if (threadIdx.x < d)
        sm100::bulk_load(vt + (size_t)threadIdx.x * vst, p.vq + (bh * d + threadIdx.x) * p.ldv + j0,
                         (uint32_t)len16, &vbar);
    // KB keys per thread in flight: their loads first, then the codes.  The
    // first batch is loaded before the query side, so both round trips overlap.
    constexpr int KB = 4;
    uint32_t kb[KB][W];
    float mk[KB];
    auto load_batch = [&](int jb) {
#pragma unroll
        for (int u = 0; u < KB; ++u) {
            const int jj = jb + u * blockDim.x;
#pragma unroll
            for (int w = 0; w < W; ++w) kb[u][w] = 0u;
            mk[u] = 0.f;
            if (jj < len) {
                load_key<W>(p, bh, j0 + jj, kb[u]);
                mk[u] = __ldg(p.muk + bh * p.Nk + j0 + jj);
            }
        }
    };
    load_batch(threadIdx.x);
    load_queries<W>(p, bh, qs, cq);
    if (threadIdx.x < p.Nq) {
        float m = -INFINITY;
        for (int t = 0; t < p.SA; ++t) m = fmaxf(m, p.pmax[(bh * p.SA + t) * p.Nq + threadIdx.x]);
        negm[threadIdx.x] = -m * LOG2E;
    }
    for (int e = threadIdx.x; e < p.Nq * d; e += blockDim.x) sacc[e] = 0;
    __syncthreads();
    float l[NQ];
#pragma unroll
    for (int i = 0; i < NQ; ++i) l[i] = 0.f;
    for (int jb = threadIdx.x; jb < len16; jb += KB * blockDim.x) {
        if (jb != (int)threadIdx.x) load_batch(jb);
#pragma unroll
        for (int u = 0; u < KB; ++u) {
            const int jj = jb + u * blockDim.x;
            if (jj >= len16) break;
            const bool live = jj < len;
#pragma unroll
            for (int i = 0; i < NQ; ++i) {
                if (i >= p.Nq) break;
                uint32_t code = 0u;
                if (live) {
                    const float pr = ex2(fmaf(score<W>(p, h, kb[u], mk[u], qs, cq, i, j0 + jj), LOG2E, negm[i]));
                    l[i] += pr;
                    code = (uint32_t)__float2int_rn(255.f * pr);
                }
                pq[i * p.C + jj] = (uint8_t)code;
            }
        }
    }
    block_reduce<false, NQ>(l, p.Nq, red, res);   // also orders the code writes before the reads below
    if (threadIdx.x < p.Nq) p.psum[(bh * p.S + s) * p.Nq + threadIdx.x] = res[threadIdx.x];
    // Every thread waits for the copies (none may land after the CTA ends).
    const bool have_v = sm100::mbar_wait(&vbar, 0, nullptr, kCopyWaitNs);
    if (!have_v && threadIdx.x == 0) atomicOr(p.status, kStatusTimeoutCopy);

    // PV: thread (g, c) takes channel c and key slice g of the split (G =
    // THREADS / d slices of whole 16-key groups), for every row; 16 keys per
    // step: one 16-byte read of the channel's codes, one 16-byte read of each
    // row's P codes (the same address across the warp), four dp4a each.  The
    // slices' sums meet in shared memory (integer adds: order-free).
    const int G = THREADS / d;
    const bool pv_thread = have_v && threadIdx.x < G * d;
    const int c = threadIdx.x % d, g = threadIdx.x / d;
    const int groups = len16 / 16;
    const int k_lo = pv_thread ? 16 * (groups * g / G) : 0;
    const int k_hi = pv_thread ? 16 * (groups * (g + 1) / G) : 0;
    int acc[NQ];
#pragma unroll
    for (int i = 0; i < NQ; ++i) acc[i] = 0;
    const uint8_t* vrow = vt + (size_t)c * vst;
#pragma unroll 2
    for (int k = k_lo; k < k_hi; k += 16) {
        const uint4 vv = *reinterpret_cast<const uint4*>(vrow + k);
#pragma unroll
        for (int i = 0; i < NQ; ++i) {
            if (i >= p.Nq) break;
            const uint4 a = *reinterpret_cast<const uint4*>(pq + i * p.C + k);
            int t = acc[i];
            t = dp4a_u8s8(a.x, vv.x, t);
            t = dp4a_u8s8(a.y, vv.y, t);
            t = dp4a_u8s8(a.z, vv.z, t);
            acc[i] = dp4a_u8s8(a.w, vv.w, t);
        }
    }
    if (pv_thread) {
#pragma unroll
        for (int i = 0; i < NQ; ++i) {
            if (i >= p.Nq) break;
            atomicAdd(&sacc[i * d + c], acc[i]);
        }
    }
    __syncthreads();
    int* dst = p.pacc + ((bh * p.S + s) * p.Nq) * d;
    for (int e = threadIdx.x; e < p.Nq * d; e += blockDim.x) dst[e] = sacc[e];

    // The head's last split CTA to finish adds the splits (int64 code sums,
    // P~ sums in split order) and applies the epilogue O = sv acc / (255 l).
    // The CTA's stores are ordered before thread 0's ticket by the barrier,
    // and the ticket is a release (publishing them, cumulatively) and an
    // acquire (the last CTA then sees every split's stores): one round trip.
    __shared__ unsigned s_last;
    __syncthreads();
    if (threadIdx.x == 0) s_last = ticket_acq_rel(&p.ticket[bh]) == (unsigned)(p.S - 1);
    __syncthreads();
    if (!s_last) return;
    for (int e = threadIdx.x; e < p.Nq * d; e += blockDim.x) {
        const int i = e / d, c2 = e - i * d;
        long long tot = 0;
        float lt = 0.f;
#pragma unroll 8
        for (int t = 0; t < p.S; ++t) {
            tot += __ldcg(p.pacc + ((bh * p.S + t) * p.Nq + i) * d + c2);
            lt += __ldcg(p.psum + (bh * p.S + t) * p.Nq + i);
        }
        const float o = __ldg(p.sv + bh * d + c2) * (float)tot / (255.f * lt);
        const int64_t oi = (bh * p.Nq + i) * d + c2;
        if (p.out_bf16) static_cast<__nv_bfloat16*>(p.out)[oi] = __float2bfloat16_rn(o);
        else static_cast<float*>(p.out)[oi] = o;
    }
}

// Splits per head: enough CTAs for about four per SM, at most MAX_CHUNK keys
// (and at most V_TILE bytes of V codes) and at least 256 keys per split
// (chunk lengths a multiple of 16).
struct Split {
    int S, C;     // PV sweep: splits and keys per split
    int SA, CA;   // maximum sweep: four PV splits per split
};

inline int max_chunk(int d) { return std::min(MAX_CHUNK, V_TILE / d / 16 * 16); }

inline Split choose_split(int64_t BH, int Nk, int d, int sm_count)
{
    const int64_t want = (4 * (int64_t)sm_count + BH - 1) / BH;
    int S = (int)std::max<int64_t>(1, std::min<int64_t>(want, (Nk + 255) / 256));
    const int cmax = max_chunk(d);
    S = std::max(S, (Nk + cmax - 1) / cmax);
    int C = (Nk + S - 1) / S;
    C = (C + 15) / 16 * 16;
    S = (Nk + C - 1) / C;
    const int CA = 4 * C;
    return {S, C, (Nk + CA - 1) / CA, CA};
}

inline int64_t workspace_bytes(int64_t BH, int Nk, int d, int sm_count)
{
    const Split sp = choose_split(BH, Nk, d, sm_count);
    const int64_t rows = BH * sp.S * MAXQ;
    return rows * 4 * 2 + rows * d * 4 + BH * 4;
}

template <int W, int NQ>
cudaError_t launch_wq(Params p, int64_t BH, cudaStream_t st)
{
    decode_max_kernel<W, NQ><<<dim3(p.SA, (unsigned)BH), THREADS, 0, st>>>(p);
    const int smem = pv_smem_bytes(p.d, p.Nq, p.C);
    auto pv = decode_pv_kernel<W, NQ>;
    cudaError_t e = cudaFuncSetAttribute(pv, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    pv<<<dim3(p.S, (unsigned)BH), THREADS, smem, st>>>(p);
    return cudaGetLastError();
}

template <int W>
cudaError_t launch_w(Params p, int64_t BH, cudaStream_t st)
{
    return p.Nq == 1 ? launch_wq<W, 1>(p, BH, st) : launch_wq<W, MAXQ>(p, BH, st);
}

}  // namespace dec

int64_t attn_decode_workspace_bytes(int B, int H, int Nk, int d, int sm_count)
{
    return dec::workspace_bytes((int64_t)B * H, Nk, d, sm_count);
}

cudaError_t launch_attn_decode(const uint32_t* bq, const float* muq, int Nq, const uint32_t* bk, const float* muk,
                               const int8_t* vq, const float* sv, int Nk, const float* bias, int64_t bias_ld,
                               int B, int H, int d, void* workspace, void* out, ba_dtype out_dt,
                               cudaStream_t st, int sm_count)
{
    const int64_t BH = (int64_t)B * H;
    const dec::Split sp = dec::choose_split(BH, Nk, d, sm_count);
    const int64_t rows = BH * sp.S * dec::MAXQ;
    dec::Params p;
    p.bq = bq; p.muq = muq; p.bk = bk; p.muk = muk; p.vq = vq; p.sv = sv;
    p.bias = bias; p.bias_ld = bias_ld;
    p.H = H; p.Nq = Nq; p.Nk = Nk; p.d = d; p.S = sp.S; p.C = sp.C; p.SA = sp.SA; p.CA = sp.CA;
    const int W = words_for(d);
    p.bk_vec = (W == 2 || W == 4) && aligned(bk, 4u * W);
    p.ldv = round_up64(Nk, 16);
    p.pmax = static_cast<float*>(workspace);
    p.psum = p.pmax + rows;
    p.pacc = reinterpret_cast<int*>(p.psum + rows);
    p.ticket = reinterpret_cast<unsigned*>(p.pacc + rows * d);
    p.out = out;
    p.out_bf16 = out_dt == BA_BF16;
    p.status = device_status_ptr();
    if (!p.status) return cudaErrorNotSupported;
    switch (words_for(d)) {
        case 1: return dec::launch_w<1>(p, BH, st);
        case 2: return dec::launch_w<2>(p, BH, st);
        case 3: return dec::launch_w<3>(p, BH, st);
        default: return dec::launch_w<4>(p, BH, st);
    }
}

}  // namespace ba
