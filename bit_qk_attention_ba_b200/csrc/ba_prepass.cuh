// ba_prepass.cuh -- device routines of the two pre-passes, shared by their
// separate kernels (ba_pack.cu, ba_quantv.cu) and by the fused pre-pass
// (ba_prepass.cu), so every path produces the same bits, scales and codes.
//
// Method source: the paper-notes page "BinaryAttention: One-Bit QK-Attention
// for Vision and Diffusion Transformers" (CVPR 2026).  Key design 1: a token
// becomes its sign vector (bit = x >= 0) and one scale, the mean |x|.  Key
// design 3: V is quantised channel-wise to int8 with a symmetric absmax scale.
#pragma once

#include "ba_common.cuh"
#include "ba_sm100.cuh"

namespace ba {

// One token held as NV 16-byte vectors (E = 16 / sizeof(T) channels each, so
// d = NV E): the sign bits are built in registers in channel order; the |x|
// sum is pairwise in one fixed order (within a vector, then over the
// vectors), which keeps the dependency chains short; mu = sum / d.  Every
// packing path of the common head sizes ends here, so all of them give the
// same bits and the same mu.
template <typename T, int NV>
__device__ __forceinline__ void pack_vectors(const uint4 (&raw)[NV], int d, uint32_t* __restrict__ bits,
                                             float* __restrict__ mu)
{
    constexpr int E = 16 / sizeof(T);
    constexpr int W = (NV * E + 31) / 32;
    uint32_t w[W];
#pragma unroll
    for (int i = 0; i < W; ++i) w[i] = 0u;
    float vs[NV];
#pragma unroll
    for (int k = 0; k < NV; ++k) {
        const T* v = reinterpret_cast<const T*>(&raw[k]);
        if constexpr (sizeof(T) == 2) {
            // The eight sign bits at once: an ordered x >= 0 on each bf16 pair
            // (all ones per true half; -0 counts as >= 0, NaN does not), the
            // halves' upper bytes gathered in channel order, each byte's low
            // bit moved to bit i of a nibble by one multiply.
            const uint32_t* h = &raw[k].x;
            const __nv_bfloat162 zero = __float2bfloat162_rn(0.f);
            uint32_t m[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) m[q] = __hge2_mask(*reinterpret_cast<const __nv_bfloat162*>(&h[q]), zero);
            const uint32_t lo = __byte_perm(m[0], m[1], 0x7531), hi = __byte_perm(m[2], m[3], 0x7531);
            const uint32_t b8 = (((lo & 0x01010101u) * 0x01020408u) >> 24) |
                                ((((hi & 0x01010101u) * 0x01020408u) >> 24) << 4);
            w[(k * E) >> 5] |= b8 << ((k * E) & 31);
        }
        float a[E];
#pragma unroll
        for (int e = 0; e < E; ++e) {
            const int c = k * E + e;
            const float f = to_f32<T>(v[e]);
            if constexpr (sizeof(T) != 2) w[c >> 5] |= (f >= 0.f ? 1u : 0u) << (c & 31);
            a[e] = fabsf(f);
        }
#pragma unroll
        for (int st = 1; st < E; st *= 2)
#pragma unroll
            for (int e = 0; e + st < E; e += 2 * st) a[e] += a[e + st];
        vs[k] = a[0];
    }
#pragma unroll
    for (int st = 1; st < NV; st *= 2)
#pragma unroll
        for (int k = 0; k + st < NV; k += 2 * st) vs[k] += vs[k + st];
#pragma unroll
    for (int i = 0; i < W; ++i) bits[i] = w[i];
    *mu = __fdiv_rn(vs[0], (float)d);
}

// One token read straight from global memory (its NV vectors in flight at once).
template <typename T, int NV>
__device__ __forceinline__ void pack_token(const T* __restrict__ x, int d, uint32_t* __restrict__ bits,
                                           float* __restrict__ mu)
{
    const uint4* src = reinterpret_cast<const uint4*>(x);
    uint4 raw[NV];
#pragma unroll
    for (int k = 0; k < NV; ++k) raw[k] = __ldg(src + k);
    pack_vectors<T, NV>(raw, d, bits, mu);
}

// Tokens a warp packs per round in pack_tokens_warp, and the 16-byte slots of
// its shared-memory buffer (one padding slot per token).
template <int NV> __host__ __device__ constexpr int pack_round_tokens() { return NV <= 9 ? 32 : 16; }
template <int NV> __host__ __device__ constexpr int pack_buffer_slots() { return pack_round_tokens<NV>() * (NV + 1); }

// The N tokens of one head packed by the warps of a CTA with coalesced loads:
// per round a warp reads the TPR tokens' TPR NV vectors as consecutive 16-byte
// loads (each warp load covers 512 contiguous bytes), parks them in its
// buffer `wbuf` (token-major, stride NV + 1 slots: conflict-free per
// quarter-warp), and lane l then packs token l from there.
template <typename T, int NV>
__device__ __forceinline__ void pack_tokens_warp(const T* __restrict__ x, int N, int d, uint32_t* __restrict__ bits,
                                                 float* __restrict__ mu, uint4* wbuf, int warp, int nwarps, int lane)
{
    constexpr int TPR = pack_round_tokens<NV>();
    constexpr int NVP = NV + 1;
    constexpr int PER_LANE = TPR * NV / 32;
    constexpr int W = (NV * (16 / (int)sizeof(T)) + 31) / 32;
    const uint4* src = reinterpret_cast<const uint4*>(x);
    for (int t0 = warp * TPR; t0 < N; t0 += nwarps * TPR) {
        const int nvec = min(TPR, N - t0) * NV;
        uint4 r[PER_LANE];
#pragma unroll
        for (int k = 0; k < PER_LANE; ++k) {
            const int vi = k * 32 + lane;
            r[k] = vi < nvec ? __ldg(src + (int64_t)t0 * NV + vi) : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int k = 0; k < PER_LANE; ++k) {
            const int vi = k * 32 + lane;
            wbuf[vi + vi / NV] = r[k];          // token vi / NV, slot vi % NV
        }
        __syncwarp();
        if (lane < TPR && t0 + lane < N) {
            uint4 raw[NV];
#pragma unroll
            for (int v = 0; v < NV; ++v) raw[v] = wbuf[lane * NVP + v];
            pack_vectors<T, NV>(raw, d, bits + (int64_t)(t0 + lane) * W, mu + t0 + lane);
        }
        __syncwarp();
    }
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

// vcode of four values of one channel (x0..x3, consecutive keys), packed
// little-endian into one word.  t = x * rs on fp32 pairs; t + 1.5 * 2^23 holds
// round-half-even(t) in its low byte (|t| <= 127 (1 + 2^-22) here, so no
// clamp is needed); any value within 1e-4 of a rounding boundary sends the
// four through vcode, the IEEE-quotient path.
__device__ __forceinline__ uint32_t vcode4(float x0, float x1, float x2, float x3, float s, float rs)
{
    if (s == 0.f) return 0u;
    const uint64_t RS = sm100::f2_pack(rs, rs);
    const uint64_t M = sm100::f2_pack(12582912.f, 12582912.f), NM = sm100::f2_pack(-12582912.f, -12582912.f);
    const uint64_t t01 = sm100::f2_mul(sm100::f2_pack(x0, x1), RS);
    const uint64_t t23 = sm100::f2_mul(sm100::f2_pack(x2, x3), RS);
    const uint64_t m01 = sm100::f2_add(t01, M), m23 = sm100::f2_add(t23, M);
    float e0, e1, e2, e3;
    sm100::f2_unpack(sm100::f2_add(t01, sm100::f2_add(m01, NM) ^ 0x8000000080000000ull), e0, e1);   // t - k
    sm100::f2_unpack(sm100::f2_add(t23, sm100::f2_add(m23, NM) ^ 0x8000000080000000ull), e2, e3);
    const float far = fmaxf(fmaxf(fabsf(e0), fabsf(e1)), fmaxf(fabsf(e2), fabsf(e3)));
    if (!(far < 0.4999f)) {
        return vcode(x0, s, rs) | (vcode(x1, s, rs) << 8) | (vcode(x2, s, rs) << 16) | (vcode(x3, s, rs) << 24);
    }
    float a, b, c, d;
    sm100::f2_unpack(m01, a, b);
    sm100::f2_unpack(m23, c, d);
    return __byte_perm(__byte_perm(__float_as_uint(a), __float_as_uint(b), 0x0040),
                       __byte_perm(__float_as_uint(c), __float_as_uint(d), 0x0040), 0x5410);
}

// 16 codes of channel row `row` (4-byte aligned, in shared memory) -> 16 bytes of vq.
__device__ __forceinline__ void store_codes16(int8_t* dst, const uint8_t* row)
{
    const uint32_t* q4 = reinterpret_cast<const uint32_t*>(row);
    *reinterpret_cast<uint4*>(dst) = make_uint4(q4[0], q4[1], q4[2], q4[3]);
}

// Shared state of the one-CTA-per-(b, h) V quantisation: the channel absmax,
// the scales, and (in dynamic shared memory) the channel-major code rows.
struct VBlockShared {
    unsigned amax[128];
    float scale[128], rscale[128];
};

// Largest code tile (bytes of dynamic shared memory) the one-CTA-per-(b, h)
// V quantisation takes; longer sequences use the tiled kernels.
constexpr int64_t kVBlockMaxSmem = 100 * 1024;

// Row stride of the code rows in shared memory: ldv + 4 bytes, an odd number
// of 4-byte words (ldv % 16 == 0), so byte writes of neighbouring channels
// land in different banks.
__host__ __device__ inline int64_t vblock_smem_bytes(int N, int d)
{
    return (int64_t)d * (round_up64(N, 16) + 4);
}

// Channel e of a 16-byte vector of T, as fp32.
template <typename T>
__device__ __forceinline__ float vec_elem(const uint4& raw, int e)
{
    if constexpr (sizeof(T) == 2) {
        const uint32_t w = (&raw.x)[e >> 1];
        return __uint_as_float((e & 1) ? (w & 0xFFFF0000u) : (w << 16));
    } else {
        return __uint_as_float((&raw.x)[e]);
    }
}

// V of one (b, h) quantised by one CTA: requires d * sizeof(T) % 16 == 0 and
// a 16-byte aligned block.  Thread i takes 16-byte vector i % G of a row
// (G = d * sizeof(T) / 16, E channels).  Sweep 1 walks rows i / G, i / G + R,
// ... (R = threads / G), takes the channel absmax in registers (bf16 pairs
// for bf16 input) and folds it into shared memory; sweep 2 reads groups of
// four consecutive rows again (from L2), quantises them and writes each
// channel's four codes as one word of the channel-major code rows in shared
// memory; the rows go out as 16-byte stores.  V is read from HBM once and
// nothing of it is staged.
template <typename T>
__device__ __forceinline__ void vblock_quant(const T* __restrict__ v_bh, int N, int d, int64_t ldv,
                                             int8_t* __restrict__ vq_bh, float* __restrict__ sv_bh,
                                             uint8_t* qt, VBlockShared& sh)
{
    constexpr int E = 16 / sizeof(T);
    const int tid = threadIdx.x, nt = blockDim.x;
    const int G = d / E;
    const int R = nt / G;
    const bool active = tid < R * G;
    const int cv = tid % G, r0 = tid / G;
    const int qs = (int)ldv + 4;
    const uint4* src = reinterpret_cast<const uint4*>(v_bh) + cv;
    for (int c = tid; c < d; c += nt) sh.amax[c] = 0u;
    __syncthreads();
    if (active) {
        float m[E];
        if constexpr (sizeof(T) == 2) {
            __nv_bfloat162 m2[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) m2[j] = __float2bfloat162_rn(0.f);
#pragma unroll 8
            for (int r = r0; r < N; r += R) {
                const uint4 raw = __ldg(src + (int64_t)r * G);
                const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
                for (int j = 0; j < 4; ++j) m2[j] = __hmax2(m2[j], __habs2(h[j]));
            }
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                m[2 * j] = __low2float(m2[j]);
                m[2 * j + 1] = __high2float(m2[j]);
            }
        } else {
#pragma unroll
            for (int e = 0; e < E; ++e) m[e] = 0.f;
#pragma unroll 8
            for (int r = r0; r < N; r += R) {
                const uint4 raw = __ldg(src + (int64_t)r * G);
#pragma unroll
                for (int e = 0; e < E; ++e) m[e] = fmaxf(m[e], fabsf(vec_elem<T>(raw, e)));
            }
        }
#pragma unroll
        for (int e = 0; e < E; ++e) atomicMax(&sh.amax[E * cv + e], __float_as_uint(m[e]));
    }
    __syncthreads();
    for (int c = tid; c < d; c += nt) {
        const float s = __fdiv_rn(__uint_as_float(sh.amax[c]), 127.0f);
        sh.scale[c] = s;
        sh.rscale[c] = __frcp_rn(s);
        sv_bh[c] = s;
    }
    __syncthreads();
    if (active) {
        float sc[E], rs[E];
#pragma unroll
        for (int e = 0; e < E; ++e) {
            sc[e] = sh.scale[E * cv + e];
            rs[e] = sh.rscale[E * cv + e];
        }
        uint8_t* qrow = qt + (E * cv) * qs;
        const int rows = (int)ldv;           // a multiple of 16: row groups never straddle it
#pragma unroll 1
        for (int r = 4 * r0; r < rows; r += 4 * R) {
            uint4 raw[4];
#pragma unroll
            for (int i = 0; i < 4; ++i)
                raw[i] = (r + i < N) ? __ldg(src + (int64_t)(r + i) * G) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
            for (int e = 0; e < E; ++e) {
                const uint32_t w = vcode4(vec_elem<T>(raw[0], e), vec_elem<T>(raw[1], e), vec_elem<T>(raw[2], e),
                                          vec_elem<T>(raw[3], e), sc[e], rs[e]);
                *reinterpret_cast<uint32_t*>(qrow + e * qs + r) = w;
            }
        }
    }
    __syncthreads();
    const int g16 = (int)(ldv / 16);
    for (int idx = tid; idx < d * g16; idx += nt) {
        const int c = idx / g16, g = idx - c * g16;
        store_codes16(vq_bh + c * ldv + 16 * g, qt + c * qs + 16 * g);
    }
}

}  // namespace ba
