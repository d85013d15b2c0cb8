// ba_attn_b1.cu -- the BinaryAttention forward with the Q.K product on the
// warp-level single-bit tensor-core MMA (mma.sync m16n8k128, .b1 operands,
// XOR + popcount accumulation) and P.V on the warp-level u8 x s8 MMA
// (mma.sync m16n8k32).
//
// Method source: the paper-notes page "BinaryAttention: One-Bit QK-Attention
// for Vision and Diffusion Transformers" (CVPR 2026).  The Hamming distance of
// two sign vectors is popc(q XOR k), so the MMA gives z = d - 2 popc directly
// (Key design 1); S = z mu_q mu_k / sqrt(d) + b (Key design 2); the keys are
// swept twice, first for the exact row maximum m, then to quantise
// P~ = exp(S - m) to u8 codes with scale 1/255 and multiply them with the
// int8 V codes (Key design 3, Overall framework).
//
// Layout.  A CTA is four warps; each warp owns 16 query rows, whose sign bits
// sit in registers as the A fragment of the .b1 MMA.  Key tiles of 64 keys
// (sign bits, key scales and, in the second sweep, the V codes) are staged in
// shared memory by cp.async in a ring of three and read with ldmatrix.  Inside
// each pair of QK n-tiles the keys are permuted so that the accumulator
// fragment holds, per thread, four consecutive keys of a row: exactly the four
// bytes the u8 A fragment of the PV MMA wants, so P never leaves registers and
// V is read in its natural key order.
#include <math.h>

#include "ba_common.cuh"
#include "ba_sm100.cuh"

namespace ba {
namespace b1 {

constexpr int WARPS = 4;
constexpr int BM = 16 * WARPS;   // query rows per CTA
constexpr int KT = 64;           // keys per staged tile
constexpr int STAGES = 3;
constexpr int VROW = KT + 16;    // V tile row stride in bytes: 8 rows hit 8 distinct bank quads
constexpr float LOG2E = 1.4426950408889634f;

__device__ __forceinline__ void cp_async4(uint32_t dst, const void* src, bool valid)
{
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(dst), "l"(src), "r"(valid ? 4 : 0)
                 : "memory");
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(valid ? 16 : 0)
                 : "memory");
}

__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }

template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], uint32_t addr)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}

// D (16 x 8, s32) = sum over 128 bit positions of popc(A XOR B); C = 0.
__device__ __forceinline__ void mma_b1(int (&c)[4], uint32_t a0, uint32_t a1, uint32_t b)
{
    asm("mma.sync.aligned.m16n8k128.row.col.s32.b1.b1.s32.xor.popc "
        "{%0, %1, %2, %3}, {%4, %5}, {%6}, {%7, %7, %7, %7};"
        : "=r"(c[0]), "=r"(c[1]), "=r"(c[2]), "=r"(c[3])
        : "r"(a0), "r"(a1), "r"(b), "r"(0));
}

// C (16 x 8, s32) += A (16 x 32 u8) . B (32 x 8 s8).
__device__ __forceinline__ void mma_u8s8(int (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1)
{
    asm("mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 "
        "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ float ex2(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Shared-memory slot of key k (0..63) of a tile.  With k = 16h + 4a + 2e + b,
// the key becomes column 2a + b of QK n-tile 2h + e; a thread with
// threadID_in_group a then holds keys 16h + 4a .. 16h + 4a + 3 of its rows in
// the accumulators of n-tiles 2h and 2h + 1.
__device__ __forceinline__ int key_slot(int k)
{
    return (k & ~15) | (((k >> 1) & 1) << 3) | (((k >> 2) & 3) << 1) | (k & 1);
}

struct Params {
    const uint32_t* bq;
    const float* muq;
    const uint32_t* bk;
    const float* muk;
    const int8_t* vq;
    const float* sv;
    const float* bias;
    int64_t bias_ld;
    int gh, gw;
    int H, N, d;
    int64_t ldv;
    void* out;
    int out_pairs;   // d is even and out is aligned for two-element stores
};

template <int NCP, int W, typename OutT, int BIAS>
__global__ void __launch_bounds__(32 * WARPS)
attn_b1_kernel(const Params p)
{
    constexpr int DVP = 16 * NCP;    // V channels staged (d rounded up to 16)
    constexpr int NCH = 2 * NCP;     // 8-channel n-tiles of the PV product
    __shared__ __align__(128) uint32_t s_k[STAGES][KT * 4];      // 16-byte slot per key
    __shared__ __align__(16) float s_mk[STAGES][KT];
    constexpr bool RP = BIAS == BA_BIAS_RELPOS2D || BIAS == BA_BIAS_RELPOS2D_CLS;
    constexpr int CLS = BIAS == BA_BIAS_RELPOS2D_CLS ? 1 : 0;   // token 0 is a class token
    __shared__ __align__(16) int s_ko[STAGES][RP ? KT : 1];
    __shared__ __align__(128) uint8_t s_v[STAGES][DVP * VROW];

    const int N = p.N, d = p.d;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, t = lane & 3;
    const int64_t bh = blockIdx.y;
    const int head = (int)(bh % p.H);
    const int r0 = blockIdx.x * BM + warp * 16 + g, r1 = r0 + 8;
    const bool ok0 = r0 < N, ok1 = r1 < N;

    // Words W..3 of every key slot stay zero (cp.async fills words 0..W-1).
    if constexpr (W < 4) {
        constexpr int PADW = 4 - W;
        for (int idx = tid; idx < STAGES * KT * PADW; idx += 32 * WARPS) {
            const int slot = idx / PADW, w = W + idx % PADW;
            s_k[slot / KT][(slot % KT) * 4 + w] = 0u;
        }
    }

    // A fragment of the .b1 MMA: word t of rows g and g + 8 of this warp.
    const uint32_t qa0 = (ok0 && t < W) ? __ldg(p.bq + (bh * N + r0) * W + t) : 0u;
    const uint32_t qa1 = (ok1 && t < W) ? __ldg(p.bq + (bh * N + r1) * W + t) : 0u;
    const float rsd = 1.f / sqrtf((float)d);
    const float cq0 = ok0 ? __ldg(p.muq + bh * N + r0) * rsd : 0.f;
    const float cq1 = ok1 ? __ldg(p.muq + bh * N + r1) * rsd : 0.f;

    const float* brow0 = nullptr;
    const float* brow1 = nullptr;
    const float* tab = nullptr;
    int rb0 = 0, rb1 = 0;
    // Class-token rows and the three class entries (query class -> patch key,
    // patch query -> class key, class -> class); row r1 = r0 + 8 is never 0.
    const bool cls0 = CLS && r0 == 0;
    float c2t = 0.f, t2c = 0.f, c2c = 0.f;
    if (BIAS == BA_BIAS_DENSE) {
        brow0 = p.bias + ((int64_t)head * N + (ok0 ? r0 : 0)) * p.bias_ld;
        brow1 = p.bias + ((int64_t)head * N + (ok1 ? r1 : 0)) * p.bias_ld;
    } else if (RP) {
        // Patch rows gather table[rb - ko] (ko: the key's patch offset); the
        // class row gathers from the table centre so every index stays in
        // range, and its values are replaced below.
        const int w2 = 2 * p.gw - 1;
        const int64_t G = (int64_t)(2 * p.gh - 1) * w2;
        tab = p.bias + (int64_t)head * (G + 3 * CLS);
        const int a0 = ok0 && !cls0 ? r0 - CLS : 0, a1 = ok1 ? r1 - CLS : 0;
        rb0 = (a0 / p.gw + p.gh - 1) * w2 + (a0 % p.gw + p.gw - 1);
        rb1 = (a1 / p.gw + p.gh - 1) * w2 + (a1 % p.gw + p.gw - 1);
        if (CLS) {
            c2t = __ldg(tab + G);
            t2c = __ldg(tab + G + 1);
            c2c = __ldg(tab + G + 2);
        }
    }

    const int T = ceil_div(N, KT);
    const int steps = 2 * T;

    auto load = [&](int step, int st) {
        const bool pass_b = step >= T;
        const int j0 = (pass_b ? step - T : step) * KT;
        if (tid < KT) {
            const int j = j0 + tid;
            const bool v = j < N;
            const uint32_t* src = p.bk + (bh * N + (v ? j : 0)) * W;
            const uint32_t dst = sm100::smem_addr(&s_k[st][key_slot(tid) * 4]);
#pragma unroll
            for (int w = 0; w < W; ++w) cp_async4(dst + 4 * w, src + w, v);
        } else {
            const int k = tid - KT, j = j0 + k;
            const bool v = j < N;
            cp_async4(sm100::smem_addr(&s_mk[st][k]), p.muk + bh * N + (v ? j : 0), v);
            if (RP) {   // the key's patch offset; -1 marks the class key
                const int pj = j - CLS;
                s_ko[st][k] = !v ? 0 : (pj < 0 ? -1 : (pj / p.gw) * (2 * p.gw - 1) + pj % p.gw);
            }
        }
        if (pass_b) {
            const uint32_t vb = sm100::smem_addr(&s_v[st][0]);
            for (int idx = tid; idx < DVP * 4; idx += 32 * WARPS) {
                const int c = idx >> 2, q = idx & 3;
                const int64_t col = (int64_t)j0 + 16 * q;
                const bool v = c < d && col < p.ldv;
                cp_async16(vb + c * VROW + 16 * q, p.vq + (bh * d + (v ? c : 0)) * p.ldv + (v ? col : 0), v);
            }
        }
    };

    // Scores of this thread's 32 (row, key) pairs of a tile: rows r0 / r1,
    // keys 16 hh + 4 t + e.  z holds the popcounts of the eight n-tiles.
    auto scores = [&](const int (&z)[8][4], int st, int j0, float (&s0)[16], float (&s1)[16]) {
#pragma unroll
        for (int hh = 0; hh < 4; ++hh) {
            const int kb = 16 * hh + 4 * t;
            const float4 mk = *reinterpret_cast<const float4*>(&s_mk[st][kb]);
            const float mkv[4] = {mk.x, mk.y, mk.z, mk.w};
            float b0[4] = {0.f, 0.f, 0.f, 0.f}, b1v[4] = {0.f, 0.f, 0.f, 0.f};
            if (BIAS == BA_BIAS_DENSE) {
                if (j0 + kb < N) {   // ld % 4 == 0 and ld >= N: the whole vector is in the row
                    const float4 x0 = __ldg(reinterpret_cast<const float4*>(brow0 + j0 + kb));
                    const float4 x1 = __ldg(reinterpret_cast<const float4*>(brow1 + j0 + kb));
                    b0[0] = x0.x; b0[1] = x0.y; b0[2] = x0.z; b0[3] = x0.w;
                    b1v[0] = x1.x; b1v[1] = x1.y; b1v[2] = x1.z; b1v[3] = x1.w;
                }
            } else if (RP) {
                const int4 ko = *reinterpret_cast<const int4*>(&s_ko[st][kb]);
                const int kov[4] = {ko.x, ko.y, ko.z, ko.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    b0[e] = __ldg(tab + rb0 - kov[e]);
                    b1v[e] = __ldg(tab + rb1 - kov[e]);
                    if (CLS) {
                        const bool key_cls = kov[e] < 0;
                        b0[e] = key_cls ? (cls0 ? c2c : t2c) : (cls0 ? c2t : b0[e]);
                        b1v[e] = key_cls ? t2c : b1v[e];
                    }
                }
            }
            const int hm0[4] = {z[2 * hh][0], z[2 * hh][1], z[2 * hh + 1][0], z[2 * hh + 1][1]};
            const int hm1[4] = {z[2 * hh][2], z[2 * hh][3], z[2 * hh + 1][2], z[2 * hh + 1][3]};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float z0 = (float)(d - 2 * hm0[e]), z1 = (float)(d - 2 * hm1[e]);
                float a = fmaf(z0 * mkv[e], cq0, b0[e]);
                float b = fmaf(z1 * mkv[e], cq1, b1v[e]);
                if (j0 + kb + e >= N) a = b = -INFINITY;
                s0[4 * hh + e] = a;
                s1[4 * hh + e] = b;
            }
        }
    };

    float m0 = -INFINITY, m1 = -INFINITY, neg0 = 0.f, neg1 = 0.f, l0 = 0.f, l1 = 0.f;
    int acc[NCH][4];
#pragma unroll
    for (int n = 0; n < NCH; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0;

    // ldmatrix row addresses of this lane: K slots lane / lane + 32; V rows
    // (channel 8 (m >> 1) + r, key offset 16 (m & 1)) of matrix m = lane / 8.
    const int vm = lane >> 3, vr = lane & 7;
    const uint32_t v_lane = (uint32_t)((8 * (vm >> 1) + vr) * VROW + 16 * (vm & 1));

#pragma unroll 1
    for (int s = 0; s < STAGES - 1; ++s) {
        if (s < steps) load(s, s);
        cp_async_commit();
    }

    int st = 0, st_load = STAGES - 1;
#pragma unroll 1
    for (int s = 0; s < steps; ++s) {
        cp_async_wait<STAGES - 2>();
        __syncthreads();
        if (s + STAGES - 1 < steps) load(s + STAGES - 1, st_load);
        cp_async_commit();

        const bool pass_b = s >= T;
        const int j0 = (pass_b ? s - T : s) * KT;
        if (s == T) {   // first step of the second sweep: the exact row maxima
            m0 = fmaxf(m0, __shfl_xor_sync(0xffffffffu, m0, 1));
            m0 = fmaxf(m0, __shfl_xor_sync(0xffffffffu, m0, 2));
            m1 = fmaxf(m1, __shfl_xor_sync(0xffffffffu, m1, 1));
            m1 = fmaxf(m1, __shfl_xor_sync(0xffffffffu, m1, 2));
            neg0 = -m0 * LOG2E;
            neg1 = -m1 * LOG2E;
        }

        int z[8][4];
        {
            const uint32_t ka = sm100::smem_addr(&s_k[st][0]) + 16 * lane;
            uint32_t kb0[4], kb1[4];
            ldsm_x4(kb0, ka);
            ldsm_x4(kb1, ka + 512);
#pragma unroll
            for (int n = 0; n < 4; ++n) {
                mma_b1(z[n], qa0, qa1, kb0[n]);
                mma_b1(z[n + 4], qa0, qa1, kb1[n]);
            }
        }
        float s0[16], s1[16];
        scores(z, st, j0, s0, s1);

        if (!pass_b) {
#pragma unroll
            for (int e = 0; e < 16; ++e) {
                m0 = fmaxf(m0, s0[e]);
                m1 = fmaxf(m1, s1[e]);
            }
        } else {
            // P~ codes: byte e of pk[row][hh] is round-half-even(255 P~) of key 16 hh + 4 t + e.
            uint32_t pk0[4], pk1[4];
#pragma unroll
            for (int hh = 0; hh < 4; ++hh) {
                uint32_t c0[4], c1[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float pa = ex2(fmaf(s0[4 * hh + e], LOG2E, neg0));
                    const float pb = ex2(fmaf(s1[4 * hh + e], LOG2E, neg1));
                    l0 += pa;
                    l1 += pb;
                    c0[e] = __float_as_uint(fmaf(pa, 255.f, 12582912.f));
                    c1[e] = __float_as_uint(fmaf(pb, 255.f, 12582912.f));
                }
                pk0[hh] = __byte_perm(__byte_perm(c0[0], c0[1], 0x0040), __byte_perm(c0[2], c0[3], 0x0040), 0x5410);
                pk1[hh] = __byte_perm(__byte_perm(c1[0], c1[1], 0x0040), __byte_perm(c1[2], c1[3], 0x0040), 0x5410);
            }
            const uint32_t vbase = sm100::smem_addr(&s_v[st][0]) + v_lane;
#pragma unroll
            for (int kc = 0; kc < 2; ++kc) {
                const uint32_t a[4] = {pk0[2 * kc], pk1[2 * kc], pk0[2 * kc + 1], pk1[2 * kc + 1]};
#pragma unroll
                for (int cp = 0; cp < NCP; ++cp) {
                    uint32_t vb[4];
                    ldsm_x4(vb, vbase + cp * 16 * VROW + kc * 32);
                    mma_u8s8(acc[2 * cp], a, vb[0], vb[1]);
                    mma_u8s8(acc[2 * cp + 1], a, vb[2], vb[3]);
                }
            }
        }
        if (++st == STAGES) st = 0;
        if (++st_load == STAGES) st_load = 0;
    }
    cp_async_wait<0>();

    l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
    l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
    const float inv0 = 1.f / (255.f * l0), inv1 = 1.f / (255.f * l1);

    // Accumulator fragment: channels 8 n + 2 t, 8 n + 2 t + 1 of rows r0 / r1.
    OutT* out = static_cast<OutT*>(p.out);
    const float* svp = p.sv + bh * d;
    const bool pairs = p.out_pairs != 0;
#pragma unroll
    for (int n = 0; n < NCH; ++n) {
        const int c = 8 * n + 2 * t;
        if (c >= d) continue;
        const bool two = c + 1 < d;
        const float sa = __ldg(svp + c), sb = two ? __ldg(svp + c + 1) : 0.f;
        const float o00 = (float)acc[n][0] * sa * inv0, o01 = (float)acc[n][1] * sb * inv0;
        const float o10 = (float)acc[n][2] * sa * inv1, o11 = (float)acc[n][3] * sb * inv1;
#pragma unroll
        for (int rr = 0; rr < 2; ++rr) {
            if (!(rr ? ok1 : ok0)) continue;
            OutT* dst = out + (bh * N + (rr ? r1 : r0)) * d + c;
            const float x0 = rr ? o10 : o00, x1 = rr ? o11 : o01;
            if (pairs) {
                if constexpr (sizeof(OutT) == 2) {
                    *reinterpret_cast<__nv_bfloat162*>(dst) = __floats2bfloat162_rn(x0, x1);
                } else {
                    *reinterpret_cast<float2*>(dst) = make_float2(x0, x1);
                }
            } else {
                if constexpr (sizeof(OutT) == 2) {
                    dst[0] = __float2bfloat16_rn(x0);
                    if (two) dst[1] = __float2bfloat16_rn(x1);
                } else {
                    dst[0] = x0;
                    if (two) dst[1] = x1;
                }
            }
        }
    }
}

template <int NCP, int W, typename OutT>
static void launch_bias(const Params& p, int bias_kind, dim3 grid, cudaStream_t st)
{
    if (bias_kind == BA_BIAS_DENSE)
        attn_b1_kernel<NCP, W, OutT, BA_BIAS_DENSE><<<grid, 32 * WARPS, 0, st>>>(p);
    else if (bias_kind == BA_BIAS_RELPOS2D)
        attn_b1_kernel<NCP, W, OutT, BA_BIAS_RELPOS2D><<<grid, 32 * WARPS, 0, st>>>(p);
    else if (bias_kind == BA_BIAS_RELPOS2D_CLS)
        attn_b1_kernel<NCP, W, OutT, BA_BIAS_RELPOS2D_CLS><<<grid, 32 * WARPS, 0, st>>>(p);
    else
        attn_b1_kernel<NCP, W, OutT, BA_BIAS_NONE><<<grid, 32 * WARPS, 0, st>>>(p);
}

// d <= 128: W = ceil(d / 32) sign words, NCP = ceil(d / 16) channel pairs of n-tiles.
template <typename OutT>
static void launch_shape(const Params& p, int bias_kind, dim3 grid, cudaStream_t st)
{
    switch ((p.d + 15) / 16) {
        case 1: launch_bias<1, 1, OutT>(p, bias_kind, grid, st); break;
        case 2: launch_bias<2, 1, OutT>(p, bias_kind, grid, st); break;
        case 3: launch_bias<3, 2, OutT>(p, bias_kind, grid, st); break;
        case 4: launch_bias<4, 2, OutT>(p, bias_kind, grid, st); break;
        case 5: launch_bias<5, 3, OutT>(p, bias_kind, grid, st); break;
        case 6: launch_bias<6, 3, OutT>(p, bias_kind, grid, st); break;
        case 7: launch_bias<7, 4, OutT>(p, bias_kind, grid, st); break;
        default: launch_bias<8, 4, OutT>(p, bias_kind, grid, st); break;
    }
}

}  // namespace b1

cudaError_t launch_attn_b1(const uint32_t* bq, const float* muq, const uint32_t* bk, const float* muk,
                           const int8_t* vq, const float* sv, int bias_kind, const float* bias,
                           int64_t bias_ld, int gh, int gw, int B, int H, int N, int d,
                           void* out, ba_dtype out_dt, cudaStream_t st)
{
    const uintptr_t esz = out_dt == BA_BF16 ? 2 : 4;
    const int pairs = (d % 2 == 0) && aligned(out, 2 * esz);
    const b1::Params p{bq, muq, bk, muk, vq, sv, bias, bias_ld, gh, gw, H, N, d, round_up64(N, 16), out, pairs};
    const dim3 grid(ceil_div(N, b1::BM), (unsigned)((int64_t)B * H));
    if (out_dt == BA_BF16)
        b1::launch_shape<__nv_bfloat16>(p, bias_kind, grid, st);
    else
        b1::launch_shape<float>(p, bias_kind, grid, st);
    return cudaGetLastError();
}

}  // namespace ba
