// ba_attn_tc_common.cuh -- pieces shared by the two tensor-core attention
// kernels (ba_attn_tc.cu: 128-key steps, one row block per CTA;
// ba_attn_tc_pair.cu: 64-key steps, persistent CTAs whose work tiles are the
// same rows of two batch elements, for a dense bias shared over the batch).
//
// Method source: the paper-notes page "BinaryAttention: One-Bit QK-Attention
// for Vision and Diffusion Transformers" (CVPR 2026), Key designs 1-3.
#pragma once

#include <cudaTypedefs.h>

#include <mutex>

#include "ba_common.cuh"
#include "ba_sm100.cuh"

namespace ba {
namespace tc {

using namespace sm100;

constexpr int BM = 128;                 // query rows per row group (= TMEM lanes)
constexpr int TILE_KEYS = 64;           // keys one softmax thread handles per step
constexpr uint32_t TMEM_COLS = 512;
// Both kernels run 10 warps (8 softmax, 1 loader, 1 MMA); warps are given
// registers in groups of four, so 12 x 32 threads share the file: 168 each.
constexpr int MAX_REGS = 168;
constexpr float LOG2E = 1.4426950408889634f;
constexpr int QK_I8 = 0, QK_F8 = 1;
// Bias variants of the kernels: the three of the ABI, plus a rel-pos fast
// path for grid widths that are multiples of 128 (a row block then lies in one
// grid row and a key tile in one grid row, so its bias is one window of a
// table row).
constexpr int BIAS_RP_FAST = 3;
// The rel-pos bias over a token set whose token 0 is a class token (the ABI's
// BA_BIAS_RELPOS2D_CLS): the general gather plus the three class entries.
constexpr int BIAS_RP_CLS = 4;
__host__ __device__ constexpr bool is_relpos(int b)
{
    return b == BA_BIAS_RELPOS2D || b == BIAS_RP_FAST || b == BIAS_RP_CLS;
}
// Bias variants whose staged key tiles carry the per-key table offsets.
__host__ __device__ constexpr bool has_koff(int b) { return b == BA_BIAS_RELPOS2D || b == BIAS_RP_CLS; }
constexpr size_t kSmemLimit = 227u * 1024u;

__host__ __device__ inline uint32_t align_up(uint32_t x, uint32_t a) { return (x + a - 1) / a * a; }

// One staged key tile of `keys` keys: keys x dpad bytes of +-1 operand
// (K-major core matrices), the key scales, and for the general rel-pos biases
// the key offsets rj (2 gw - 1) + cj (-1 for a class key).
__host__ __device__ inline uint32_t tile_bytes(int keys, int dpad, int bias_kind)
{
    return (uint32_t)(keys * dpad + keys * 4 + (has_koff(bias_kind) ? keys * 4 : 0));
}

inline int dv_of(int d) { return (d + 15) / 16 * 16; }

// 16 sign bits -> 16 bytes of +-1 operands (+1 where the bit is set); byte
// lanes whose bit in `valid` is 0 are forced to 0 (padding channels).
template <int QK>
__device__ __forceinline__ uint4 expand16(uint32_t bits, uint32_t valid)
{
    uint32_t o[4];
#pragma unroll
    for (int n = 0; n < 4; ++n) {
        const uint32_t nib = (bits >> (4 * n)) & 0xFu;
        const uint32_t spread = (nib * 0x00204081u) & 0x01010101u;
        uint32_t v = (QK == QK_I8) ? ((spread * 0xFEu) ^ 0xFFFFFFFFu)     // 0x01 / 0xFF
                                   : ((spread * 0x80u) ^ 0xB8B8B8B8u);    // e4m3 +1.0 / -1.0
        const uint32_t vn = (valid >> (4 * n)) & 0xFu;
        if (vn != 0xFu) v &= ((vn * 0x00204081u) & 0x01010101u) * 0xFFu;
        o[n] = v;
    }
    return make_uint4(o[0], o[1], o[2], o[3]);
}

__device__ __forceinline__ float ex2(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Byte offset of (row r, 16-byte chunk kc) in a K-major, non-swizzled operand
// whose rows hold `chunks` 16-byte chunks: 8 x 16-byte core matrices, chunk
// neighbours 128 bytes apart, 8-row groups chunks * 128 bytes apart.
__device__ __forceinline__ uint32_t core_off(int r, int kc, int chunks)
{
    return (uint32_t)((r >> 3) * chunks * 128 + kc * 128 + (r & 7) * 16);
}

// Warp-uniform bounded wait: every lane polls, all agree on the outcome.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                          uint64_t limit_ns = 2000000000ull)
{
    const bool ok = mbar_wait(bar, parity, abort_flag, limit_ns);
    return __all_sync(0xffffffffu, ok);
}

__device__ __forceinline__ void fail(volatile int* abort_flag, unsigned* status, unsigned bit)
{
    *abort_flag = 1;
    atomicOr(status, bit);
}

// Advance a running step index i in a ring of n slots, kept as slot = i % n
// and parity = (i / n) & 1 (no division per step).
__device__ __forceinline__ void ring_next(int& slot, uint32_t& parity, int n)
{
    if (++slot == n) {
        slot = 0;
        parity ^= 1u;
    }
}

template <typename OutT> __device__ __forceinline__ void store1(OutT* p, float v);
template <> __device__ __forceinline__ void store1<float>(float* p, float v) { *p = v; }
template <> __device__ __forceinline__ void store1<__nv_bfloat16>(__nv_bfloat16* p, float v) { *p = __float2bfloat16_rn(v); }

// Epilogue for 16 output channels of one row: o_c = sv_c * acc_c * inv for
// the first n (<= 16) of them, stored as two (bf16) or four (fp32) 16-byte
// vectors when all 16 are valid and dst is 16-byte aligned, else one by one.
template <typename OutT>
__device__ __forceinline__ void store_out16(OutT* dst, const uint32_t (&acc)[16], const float* svp, float inv, int n)
{
    float o[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) o[e] = (e < n) ? __int2float_rn((int)acc[e]) * __ldg(svp + e) * inv : 0.f;
    if (n == 16 && (reinterpret_cast<uintptr_t>(dst) & 15u) == 0) {
        if constexpr (sizeof(OutT) == 2) {
            uint32_t w[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const __nv_bfloat162 h2 = __floats2bfloat162_rn(o[2 * e], o[2 * e + 1]);
                w[e] = *reinterpret_cast<const uint32_t*>(&h2);
            }
            uint4* d4 = reinterpret_cast<uint4*>(dst);
            d4[0] = make_uint4(w[0], w[1], w[2], w[3]);
            d4[1] = make_uint4(w[4], w[5], w[6], w[7]);
        } else {
            float4* d4 = reinterpret_cast<float4*>(dst);
#pragma unroll
            for (int e = 0; e < 4; ++e) d4[e] = make_float4(o[4 * e], o[4 * e + 1], o[4 * e + 2], o[4 * e + 3]);
        }
    } else {
#pragma unroll
        for (int e = 0; e < 16; ++e)
            if (e < n) store1<OutT>(dst + e, o[e]);
    }
}

// KEYS (64 or 32) keys of one row: S = z * mu_k * cq + b (Key design 2) on
// packed pairs, then either the row maximum (pass A) or P~ = exp(S - m), the
// row sum and the u8 codes round(255 P~) (pass B).  MASK drops keys >= N.
// Two independent max / sum accumulators keep the dependency chains short.
// For BIAS_RP_CLS, cls3 points at the head's three class entries (class
// query -> patch key, patch query -> class key, class -> class), a key offset
// of -1 marks the class key, and cls_row marks the class query's row.
template <int QK, int BIAS, bool PASS_B, bool MASK, int KEYS = TILE_KEYS, bool EXP16 = false>
__device__ __forceinline__ void softmax_tile(const uint32_t (&zr)[KEYS], const float* mks, const uint8_t* bsm_row,
                                             int bsm_sw, const float* rp_copy, const int* koff,
                                             const float* tab_h, int rel_base, int nvalid,
                                             uint64_t cq2, uint64_t neg2, float (&mx)[2], uint64_t (&l2)[2],
                                             uint32_t (&pw)[KEYS / 4], const float* cls3 = nullptr,
                                             bool cls_row = false)
{
    float c2t = 0.f, key_cls = 0.f;
    if (BIAS == BIAS_RP_CLS) {
        c2t = __ldg(cls3);
        key_cls = __ldg(cls3 + (cls_row ? 2 : 1));
    }
    const uint64_t L2E = f2_pack(LOG2E, LOG2E);
    const uint64_t C255 = f2_pack(255.f, 255.f);
    const uint64_t MAGIC = f2_pack(12582912.f, 12582912.f);
    // The key scales and bias values come from shared memory; they are
    // fetched PF groups of four keys ahead so their latency overlaps math.
    constexpr int PF = 3;
    auto fetch = [&](int k4, float4& mk, float4& bb) {
        mk = *reinterpret_cast<const float4*>(mks + 4 * k4);
        bb = make_float4(0.f, 0.f, 0.f, 0.f);
        if (BIAS == BA_BIAS_DENSE) {
            bb = *reinterpret_cast<const float4*>(bsm_row + (k4 >> 3) * 16384 + (((k4 & 7) ^ bsm_sw) << 4));
        } else if (BIAS == BIAS_RP_FAST) {
            bb = *reinterpret_cast<const float4*>(rp_copy + 4 * k4);
        } else if (BIAS == BA_BIAS_RELPOS2D || BIAS == BIAS_RP_CLS) {
            const int4 ko = *reinterpret_cast<const int4*>(koff + 4 * k4);
            bb = make_float4(__ldg(tab_h + rel_base - ko.x), __ldg(tab_h + rel_base - ko.y),
                             __ldg(tab_h + rel_base - ko.z), __ldg(tab_h + rel_base - ko.w));
            if (BIAS == BIAS_RP_CLS) {
                bb.x = ko.x < 0 ? key_cls : (cls_row ? c2t : bb.x);
                bb.y = ko.y < 0 ? key_cls : (cls_row ? c2t : bb.y);
                bb.z = ko.z < 0 ? key_cls : (cls_row ? c2t : bb.z);
                bb.w = ko.w < 0 ? key_cls : (cls_row ? c2t : bb.w);
            }
        }
    };
    float4 mkq[PF], bbq[PF];
#pragma unroll
    for (int k = 0; k < PF; ++k) fetch(k, mkq[k], bbq[k]);
#pragma unroll
    for (int k4 = 0; k4 < KEYS / 4; ++k4) {
        const float4 mk = mkq[k4 % PF];
        const float4 bb = bbq[k4 % PF];
        if (k4 + PF < KEYS / 4) fetch(k4 + PF, mkq[k4 % PF], bbq[k4 % PF]);
        uint64_t z01, z23;
        if (QK == QK_F8) {
            z01 = f2_pack(__uint_as_float(zr[4 * k4]), __uint_as_float(zr[4 * k4 + 1]));
            z23 = f2_pack(__uint_as_float(zr[4 * k4 + 2]), __uint_as_float(zr[4 * k4 + 3]));
        } else {   // s32 -> f32 exactly: |z| < 2^22, so 1.5 * 2^23 + z is exact
            const uint64_t NM = f2_pack(-12582912.f, -12582912.f);
            z01 = f2_add(f2_pack(__uint_as_float(zr[4 * k4] + 0x4B400000u),
                                 __uint_as_float(zr[4 * k4 + 1] + 0x4B400000u)), NM);
            z23 = f2_add(f2_pack(__uint_as_float(zr[4 * k4 + 2] + 0x4B400000u),
                                 __uint_as_float(zr[4 * k4 + 3] + 0x4B400000u)), NM);
        }
        uint64_t s01 = f2_fma(f2_mul(z01, f2_pack(mk.x, mk.y)), cq2, f2_pack(bb.x, bb.y));
        uint64_t s23 = f2_fma(f2_mul(z23, f2_pack(mk.z, mk.w)), cq2, f2_pack(bb.z, bb.w));
        if (MASK) {
            float a, b, c, e;
            f2_unpack(s01, a, b);
            f2_unpack(s23, c, e);
            const int j = 4 * k4;
            a = (j < nvalid) ? a : -INFINITY;
            b = (j + 1 < nvalid) ? b : -INFINITY;
            c = (j + 2 < nvalid) ? c : -INFINITY;
            e = (j + 3 < nvalid) ? e : -INFINITY;
            s01 = f2_pack(a, b);
            s23 = f2_pack(c, e);
        }
        if (!PASS_B) {
            float a, b, c, e;
            f2_unpack(s01, a, b);
            f2_unpack(s23, c, e);
            mx[k4 & 1] = fmax3(mx[k4 & 1], a, b);
            mx[k4 & 1] = fmax3(mx[k4 & 1], c, e);
        } else if (EXP16) {
            // P~ on the f16x2 path: one MUFU operation gives two exponentials;
            // the codes come from an f16 fma (255 P~ + 1024 has ulp 1, so its
            // low byte is round-half-even(255 P~)); the row sum stays fp32.
            float a, b, c, e;
            f2_unpack(f2_fma(s01, L2E, neg2), a, b);
            f2_unpack(f2_fma(s23, L2E, neg2), c, e);
            const uint32_t h01 = ex2_f16x2(f16x2_from(a, b));
            const uint32_t h23 = ex2_f16x2(f16x2_from(c, e));
            constexpr uint32_t H255 = 0x5BF85BF8u, H1024 = 0x64006400u;
            pw[k4] = __byte_perm(fma_f16x2(h01, H255, H1024), fma_f16x2(h23, H255, H1024), 0x6420);
            l2[k4 & 1] = f2_add(l2[k4 & 1], f2_add(f2_from_f16x2(h01), f2_from_f16x2(h23)));
        } else {
            float a, b, c, e;
            f2_unpack(f2_fma(s01, L2E, neg2), a, b);
            f2_unpack(f2_fma(s23, L2E, neg2), c, e);
            const uint64_t p01 = f2_pack(ex2(a), ex2(b));
            const uint64_t p23 = f2_pack(ex2(c), ex2(e));
            l2[k4 & 1] = f2_add(l2[k4 & 1], f2_add(p01, p23));
            float q0, q1, q2, q3;                      // low byte = round-half-even(255 P~)
            f2_unpack(f2_fma(p01, C255, MAGIC), q0, q1);
            f2_unpack(f2_fma(p23, C255, MAGIC), q2, q3);
            pw[k4] = __byte_perm(__byte_perm(__float_as_uint(q0), __float_as_uint(q1), 0x0040),
                                 __byte_perm(__float_as_uint(q2), __float_as_uint(q3), 0x0040), 0x5410);
        }
    }
}

inline PFN_cuTensorMapEncodeTiled_v12000 encode_fn()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
    });
    return fn;
}

}  // namespace tc
}  // namespace ba
