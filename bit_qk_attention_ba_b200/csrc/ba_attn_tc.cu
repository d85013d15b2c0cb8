// ba_attn_tc.cu -- the BinaryAttention forward on the sm_100a tensor cores.
//
// BA notes (paper-notes page "BinaryAttention: One-Bit QK-Attention for
// Vision and Diffusion Transformers", CVPR 2026):
//   Key design 1: s_i . t_j from sign bits, per-token scales mu
//   Key design 2: S_ij = mu_q,i mu_k,j s_i.t_j / sqrt(d) + b_ij
//   Key design 3: P~ = exp(S - m) as u8 with scale 1/255, channel-wise int8
//                 V, integer PV product
//   Overall framework: a tiled attention in the FlashAttention2 style.
//
// The A100 design on the page (mma.sync .b1 for QK, mma.sync u8.s8 for PV,
// one pass with a running maximum) is prior art.  This kernel is built for
// Blackwell:
//   * a CTA owns two groups of 128 query rows, one softmax thread per query
//     row (row = TMEM lane), so row reductions need no shuffles.  With a
//     dense bias the groups are the same rows of two batch elements, so one
//     bias tile serves both; otherwise they are two row blocks of one head,
//     so one key/value tile serves both;
//   * the keys are swept twice: pass A finds the exact row maximum m_i, pass
//     B quantises P~ = exp(S - m_i) against it.  The u8 codes are then the
//     ones an exact-maximum reference produces, and the int32 PV accumulator
//     never needs rescaling;
//   * a staging pre-pass turns the key sign bits into +-1 tensor-core
//     operands once per call (kind::i8 bytes, or e4m3 +-1 for kind::f8f6f4),
//     laid out tile by tile in the shared-memory order the QK product reads,
//     each 64-key tile followed by its key scales; for a 2-D relative-position
//     bias it also writes every table row reversed, in four copies shifted
//     by one entry, so any bias window a tile needs is one aligned copy;
//   * one loader thread moves everything with bulk copies and TMA (key tiles,
//     bias windows or dense bias boxes, V tiles) into a 2..4-stage ring: the
//     loader issues no loads or stores of its own;
//   * QK runs on tcgen05.mma into double-buffered S tiles in TMEM, so the
//     next tile's QK overlaps this tile's softmax; both kinds are exact;
//   * PV runs on tcgen05.mma kind::i8 with u8 P read straight from TMEM (the
//     softmax writes it over the S tile it came from) and s8 V tiles,
//     accumulating in TMEM across all key tiles;
//   * the softmax pulls each 64-key S tile out of TMEM with one load and does
//     its arithmetic on packed fp32 pairs (fma/mul/add .f32x2) with a 3-input
//     max; a bias window is read as reversed copies, four keys per 16-byte
//     load.
// Warps 0-7 run the softmax (two groups of four), warp 8 loads, warp 9
// issues the MMAs and owns TMEM.
//
// Every wait on an mbarrier is bounded; on a timeout the kernel records a bit
// in the device status word, tells the other roles to stop, lets issued copies
// and tensor-core work drain, frees TMEM and returns.
#include <cudaTypedefs.h>

#include <mutex>

#include "ba_common.cuh"
#include "ba_sm100.cuh"

namespace ba {
namespace {

using namespace sm100;

constexpr int BM = 128;                 // query rows per group (= TMEM lanes)
constexpr int NG = 2;                   // row groups per CTA
constexpr int BN = 64;                  // keys per tile
constexpr int MAX_STAGES = 4;
constexpr int NUM_SOFTMAX_WARPS = 4 * NG;                   // 8
constexpr int LOAD_WARP = NUM_SOFTMAX_WARPS;                // 8
constexpr int MMA_WARP = LOAD_WARP + 1;                     // 9
constexpr int NUM_THREADS = 32 * (MMA_WARP + 1);            // 320
// Warps are given registers in groups of four: 10 warps leave 168 per thread.
constexpr int MAX_REGS = 168;
constexpr uint32_t TMEM_COLS = 512;
constexpr float LOG2E = 1.4426950408889634f;
constexpr int QK_I8 = 0, QK_F8 = 1;
// Bias variants of the kernel: the three of the ABI, plus a rel-pos fast path
// for grid widths that are multiples of 128 (a row group then lies in one grid
// row and a key tile in one grid row, so its bias is one window of a table row).
constexpr int BIAS_RP_FAST = 3;
__host__ __device__ constexpr bool is_relpos(int b) { return b == BA_BIAS_RELPOS2D || b == BIAS_RP_FAST; }
constexpr int RP_WIN = 192;             // entries per shifted copy of a window (191 used)
constexpr int RP_STRIDE = 200;          // floats between copies in shared memory (8 words mod 32)
constexpr uint32_t RP_COPY_BYTES = RP_WIN * 4;

// Barrier slots.
enum {
    B_QREADY = 0,
    B_FULL = 1,                      // [stage] key tiles, bias (and V in pass B) landed
    B_EMPTY = B_FULL + MAX_STAGES,   // [stage] stage may be overwritten
    B_SFULL = B_EMPTY + MAX_STAGES,  // [NG][2] S tile in TMEM ready
    B_SDONE = B_SFULL + 2 * NG,      // [NG][2] softmax done with the S buffer (pass B: u8 P written into it)
    B_OREADY = B_SDONE + 2 * NG,     // every PV finished
    B_FINAL = B_OREADY + 1,
    NUM_BARS
};

// One staged key tile: BN keys x dpad bytes of +-1 operand (K-major core
// matrices), the BN key scales, and for the general rel-pos bias the BN key
// offsets rj (2 gw - 1) + cj.
__host__ __device__ inline uint32_t tile_bytes(int dpad, int bias_kind)
{
    return (uint32_t)(BN * dpad + BN * 4 + (bias_kind == BA_BIAS_RELPOS2D ? BN * 4 : 0));
}

struct Layout {
    uint32_t stages, kvg, tile; // pipeline depth; key/value sets per stage (1 or 2); staged tile bytes
    uint32_t v, v_bytes;        // [stage][kvg] V tiles (SW64 K-major, dv rows x 64 bytes)
    uint32_t b;                 // [stage][2] dense bias boxes, 16 KB each (SW128)
    uint32_t q, q_bytes;        // [NG] Q operands
    uint32_t k, k_bytes;        // [stage] kvg staged key tiles
    uint32_t rp;                // [stage][NG][4][RP_STRIDE] rel-pos windows
    uint32_t bars, misc, total;
};

__host__ __device__ inline uint32_t align_up(uint32_t x, uint32_t a) { return (x + a - 1) / a * a; }

__host__ __device__ inline Layout make_layout(int dpad, int dv, int bias_kind, int stages)
{
    Layout L;
    L.stages = stages;
    L.kvg = (bias_kind == BA_BIAS_DENSE) ? 2u : 1u;
    L.tile = tile_bytes(dpad, bias_kind == BIAS_RP_FAST ? BA_BIAS_NONE : bias_kind);
    uint32_t off = 0;
    L.v_bytes = align_up((uint32_t)dv * BN, 1024);
    L.v = off; off += stages * L.kvg * L.v_bytes;
    L.b = off; off += (bias_kind == BA_BIAS_DENSE) ? stages * 2 * 16384u : 0u;
    L.q_bytes = align_up((uint32_t)BM * dpad, 1024);
    L.q = off; off += NG * L.q_bytes;
    L.k_bytes = align_up(L.kvg * L.tile, 128);
    L.k = off; off += stages * L.k_bytes;
    L.rp = off; off += (bias_kind == BIAS_RP_FAST) ? stages * NG * 4 * RP_STRIDE * 4u : 0u;
    L.bars = off; off += NUM_BARS * 8;
    L.misc = off; off += 16;            // TMEM base address, abort flag
    L.total = off;
    return L;
}

struct Params {
    const uint32_t* bq;
    const float* muq;
    const uint8_t* kst;      // staged key tiles [B*H][n_tiles][tile]
    const float* rps;        // staged rel-pos rows [H][2 gh - 1][4][2 gw] (fast path)
    const float* sv;
    const float* table;      // 2-D relative-position table (general rel-pos path)
    void* out;
    int B, H, N, d, W, dpad, dv, n_tiles, stages;
    int gh, gw;
    float q_scale;           // 1 / sqrt(d)
    unsigned* status;
};

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
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag)
{
    const bool ok = mbar_wait(bar, parity, abort_flag);
    return __all_sync(0xffffffffu, ok);
}

__device__ __forceinline__ void fail(volatile int* abort_flag, unsigned* status, unsigned bit)
{
    *abort_flag = 1;
    atomicOr(status, bit);
}

template <typename OutT> __device__ __forceinline__ void store1(OutT* p, float v);
template <> __device__ __forceinline__ void store1<float>(float* p, float v) { *p = v; }
template <> __device__ __forceinline__ void store1<__nv_bfloat16>(__nv_bfloat16* p, float v) { *p = __float2bfloat16_rn(v); }

// Which (batch*head, first query row) a row group of this CTA covers, and
// whether that group exists.  Dense bias: groups are batch elements 2z and
// 2z+1 of head y, rows 128x.  Otherwise: rows 256x and 256x+128 of head y.
template <bool PAIR>
__device__ __forceinline__ void group_coords(const Params& p, int g, int& bh, int& q0, bool& exists)
{
    if (PAIR) {
        int b = 2 * blockIdx.z + g;
        exists = b < p.B;
        if (!exists) b = p.B - 1;
        bh = b * p.H + blockIdx.y;
        q0 = blockIdx.x * BM;
    } else {
        bh = blockIdx.y;
        q0 = blockIdx.x * (BM * NG) + g * BM;
        exists = q0 < p.N;
    }
}

// One 64-key tile of one row: S = z * mu_k * cq + b (Key design 2) on packed
// pairs, then either the row maximum (pass A) or P~ = exp(S - m), the row sum
// and the u8 codes round(255 P~) (pass B).  MASK drops keys >= N.  Two
// independent max / sum accumulators keep the dependency chains short.
template <int QK, int BIAS, bool PASS_B, bool MASK>
__device__ __forceinline__ void softmax_tile(const uint32_t (&zr)[64], const float* mks, const uint8_t* bsm_row,
                                             int bsm_sw, const float* rp_copy, const int* koff,
                                             const float* tab_h, int rel_base, int nvalid,
                                             uint64_t cq2, uint64_t neg2, float (&mx)[2], uint64_t (&l2)[2],
                                             uint32_t (&pw)[16])
{
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
        } else if (BIAS == BA_BIAS_RELPOS2D) {
            const int4 ko = *reinterpret_cast<const int4*>(koff + 4 * k4);
            bb = make_float4(__ldg(tab_h + rel_base - ko.x), __ldg(tab_h + rel_base - ko.y),
                             __ldg(tab_h + rel_base - ko.z), __ldg(tab_h + rel_base - ko.w));
        }
    };
    float4 mkq[PF], bbq[PF];
#pragma unroll
    for (int k = 0; k < PF; ++k) fetch(k, mkq[k], bbq[k]);
#pragma unroll
    for (int k4 = 0; k4 < BN / 4; ++k4) {
        const float4 mk = mkq[k4 % PF];
        const float4 bb = bbq[k4 % PF];
        if (k4 + PF < BN / 4) fetch(k4 + PF, mkq[k4 % PF], bbq[k4 % PF]);
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

template <int QK, typename OutT, int BIAS>
__global__ void __maxnreg__(MAX_REGS)
attn_tc_kernel(const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_b,
               const Params p)
{
    constexpr bool PAIR = (BIAS == BA_BIAS_DENSE);
    constexpr int KVG = PAIR ? 2 : 1;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const Layout L = make_layout(p.dpad, p.dv, BIAS, p.stages);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.bars);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L.misc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L.misc + 4);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int N = p.N, W = p.W, T = p.n_tiles, U = 2 * T;   // steps: pass A then pass B
    const int S = p.stages;
    const int chunks = p.dpad / 16;
    const int h = PAIR ? (int)blockIdx.y : (int)(blockIdx.y % p.H);
    const float* tab_h = (BIAS == BA_BIAS_RELPOS2D)
                             ? p.table + (size_t)h * (2 * p.gh - 1) * (2 * p.gw - 1) : nullptr;

    if (threadIdx.x == 0) {
        mbar_init(&bars[B_QREADY], NUM_SOFTMAX_WARPS);
        for (int s = 0; s < S; ++s) {
            mbar_init(&bars[B_FULL + s], 1);
            mbar_init(&bars[B_EMPTY + s], NUM_SOFTMAX_WARPS + 1);
        }
        for (int b = 0; b < 2 * NG; ++b) {
            mbar_init(&bars[B_SFULL + b], 1);
            mbar_init(&bars[B_SDONE + b], 4);
        }
        mbar_init(&bars[B_OREADY], 1);
        mbar_init(&bars[B_FINAL], 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == MMA_WARP) {
        tmem_alloc(tmem_slot, TMEM_COLS);
        tmem_relinquish();
    }
    if (warp == LOAD_WARP && lane == 0) {
        prefetch_tmap(&tm_v);
        if (BIAS == BA_BIAS_DENSE) prefetch_tmap(&tm_b);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == LOAD_WARP) {
        // ---------------------------------------------------------------- loader
        // One thread fills stage u % S for step u: the staged key tile(s), the
        // bias of the tile (two windows of reversed table rows, one per group,
        // each in four shifted copies; or two dense-bias boxes), and in pass B
        // the V tile(s).  All copies complete on the stage's FULL barrier.
        if (lane == 0) {
            int kvbh0, kvbh1, q0g[NG];
            {
                bool ex;
                group_coords<PAIR>(p, 0, kvbh0, q0g[0], ex);
                group_coords<PAIR>(p, 1, kvbh1, q0g[1], ex);
                if (!PAIR) kvbh1 = kvbh0;
            }
            const size_t row_len = 2 * (size_t)p.gw;
            const float* rps_h = (BIAS == BIAS_RP_FAST) ? p.rps + (size_t)h * (2 * p.gh - 1) * 4 * row_len : nullptr;
            int rp_ri[NG], rp_ci[NG];
#pragma unroll
            for (int g = 0; g < NG; ++g) {
                const int q0 = (q0g[g] < N) ? q0g[g] : N - BM;     // an empty group still reads inside the table
                rp_ri[g] = (BIAS == BIAS_RP_FAST) ? q0 / p.gw : 0;
                rp_ci[g] = (BIAS == BIAS_RP_FAST) ? q0 - rp_ri[g] * p.gw : 0;
            }
            const uint32_t step_bytes = KVG * L.tile + (BIAS == BIAS_RP_FAST ? NG * 4 * RP_COPY_BYTES : 0u) +
                                        (BIAS == BA_BIAS_DENSE ? 2 * 16384u : 0u);
            const uint32_t v_bytes = (uint32_t)(KVG * p.dv * BN);
            int issued = 0;
            for (int u = 0; u < U; ++u) {
                const int s = u % S;
                const bool pass_b = u >= T;
                const int t = pass_b ? u - T : u;
                const int j0 = t * BN;
                if (u >= S && !mbar_wait(&bars[B_EMPTY + s], (u / S - 1) & 1, abort_flag)) {
                    fail(abort_flag, p.status, kStatusTimeoutProducer);
                    break;
                }
                uint64_t* full = &bars[B_FULL + s];
                mbar_arrive_expect_tx(full, step_bytes + (pass_b ? v_bytes : 0u));
                uint8_t* kdst = smem + L.k + s * L.k_bytes;
                bulk_load(kdst, p.kst + ((size_t)kvbh0 * T + t) * L.tile, L.tile, full);
                if (KVG > 1) bulk_load(kdst + L.tile, p.kst + ((size_t)kvbh1 * T + t) * L.tile, L.tile, full);
                if (BIAS == BIAS_RP_FAST) {
                    // Window of group g: entries xs .. xs + 191 of the reversed
                    // row for ri - rj, xs = gw - 128 - (ci0 - cj0), in each copy.
                    const int rj = j0 / p.gw, cj0 = j0 - rj * p.gw;
#pragma unroll
                    for (int g = 0; g < NG; ++g) {
                        const int rho = rp_ri[g] - rj + p.gh - 1;
                        const int xs = p.gw - BM - (rp_ci[g] - cj0);
                        const float* src = rps_h + (size_t)rho * 4 * row_len + xs;
                        float* dst = reinterpret_cast<float*>(smem + L.rp) + (size_t)(s * NG + g) * 4 * RP_STRIDE;
#pragma unroll
                        for (int m = 0; m < 4; ++m)
                            bulk_load(dst + m * RP_STRIDE, src + m * row_len, RP_COPY_BYTES, full);
                    }
                }
                if (BIAS == BA_BIAS_DENSE)
                    for (int bx = 0; bx < 2; ++bx)
                        tma_load_3d(smem + L.b + (s * 2 + bx) * 16384, &tm_b, full, j0 + 32 * bx,
                                    (int)blockIdx.x * BM, h);
                if (pass_b) {
                    tma_load_3d(smem + L.v + (s * KVG) * L.v_bytes, &tm_v, full, j0, 0, kvbh0);
                    if (KVG > 1) tma_load_3d(smem + L.v + (s * KVG + 1) * L.v_bytes, &tm_v, full, j0, 0, kvbh1);
                }
                issued = u + 1;
            }
            // On an abort, let copies already issued land before the CTA exits.
            if (*abort_flag)
                for (int u = (issued > S ? issued - S : 0); u < issued; ++u)
                    mbar_wait(&bars[B_FULL + u % S], (u / S) & 1, nullptr, 100000000ull);
        }
        __syncwarp();
    } else if (warp == MMA_WARP) {
        // ---------------------------------------------------------------- MMA issue
        if (lane == 0) {
            const uint32_t idesc_qk = (QK == QK_I8) ? instr_desc(kCS32, kFmtS8, kFmtS8, BM, BN)
                                                    : instr_desc(kCF32, kFmtE4M3, kFmtE4M3, BM, BN);
            const uint32_t idesc_pv = instr_desc(kCS32, kFmtU8, kFmtS8, BM, p.dv);
            const uint32_t sbo_qk = (uint32_t)chunks * 128u;
            bool ok = mbar_wait(&bars[B_QREADY], 0, abort_flag);
            // Descriptors are built once; moving along a buffer only adds to the
            // start-address field (bytes / 16), which never carries out.
            const uint64_t dq0 = smem_desc(smem_addr(smem + L.q), 128, sbo_qk, kLayoutNone);
            const uint64_t dk0 = smem_desc(smem_addr(smem + L.k), 128, sbo_qk, kLayoutNone);
            const uint64_t dv0 = smem_desc(smem_addr(smem + L.v), 16, 512, kLayoutSw64);
            const uint32_t q_step = L.q_bytes >> 4, v_step = L.v_bytes >> 4;
            const int kq = p.dpad / 32;
            auto issue_qk = [&](int u) -> bool {
                const int s = u % S, buf = u & 1;
                if (!mbar_wait(&bars[B_FULL + s], (u / S) & 1, abort_flag)) return false;
                for (int g = 0; g < NG; ++g)
                    if (u >= 2 && !mbar_wait(&bars[B_SDONE + 2 * g + buf], ((u >> 1) - 1) & 1, abort_flag))
                        return false;
                tc_fence_after();
                for (int g = 0; g < NG; ++g) {
                    const uint64_t dq = dq0 + g * q_step;
                    const uint64_t dk = dk0 + ((s * L.k_bytes + (PAIR ? g : 0) * L.tile) >> 4);
                    const uint32_t d_tmem = tmem + (2 * g + buf) * BN;
                    for (int kk = 0; kk < kq; ++kk)
                        mma_ss<QK>(d_tmem, dq + kk * 16, dk + kk * 16, idesc_qk, kk > 0 ? 1u : 0u);
                    mma_commit(&bars[B_SFULL + 2 * g + buf]);
                }
                return true;
            };
            if (ok) ok = issue_qk(0);
            for (int u = 0; ok && u < U; ++u) {
                if (u + 1 < U && !(ok = issue_qk(u + 1))) break;
                if (u >= T) {
                    // PV: u8 P (in the S buffer's first BN/4 TMEM columns) x s8 V.
                    const int t = u - T, buf = u & 1, s = u % S;
                    for (int g = 0; g < NG && ok; ++g)
                        ok = mbar_wait(&bars[B_SDONE + 2 * g + buf], (u >> 1) & 1, abort_flag);
                    if (!ok) break;
                    tc_fence_after();
                    for (int g = 0; g < NG; ++g) {
                        const uint64_t dv = dv0 + (s * KVG + (PAIR ? g : 0)) * v_step;
                        const uint32_t a_tmem = tmem + (2 * g + buf) * BN;
                        for (int kk = 0; kk < BN / 32; ++kk)
                            mma_ts_i8(tmem + 256 + 128 * g, a_tmem + kk * 8, dv + kk * 2, idesc_pv,
                                      (t > 0 || kk > 0) ? 1u : 0u);
                    }
                }
                mma_commit(&bars[B_EMPTY + u % S]);
            }
            if (ok) mma_commit(&bars[B_OREADY]);
            if (!ok) fail(abort_flag, p.status, kStatusTimeoutMma);
            // Let every issued MMA finish before TMEM is released.
            mma_commit(&bars[B_FINAL]);
            if (!mbar_wait(&bars[B_FINAL], 0, nullptr, 4000000000ull)) atomicOr(p.status, kStatusTimeoutMma);
        }
        __syncwarp();
    } else {
        // ---------------------------------------------------------------- softmax + epilogue
        const int g = warp >> 2;                      // row group
        const int quarter = warp & 3;                 // TMEM lanes this warp may access
        const int r = quarter * 32 + lane;            // row within the group
        int bh, q0;
        bool group_exists;
        group_coords<PAIR>(p, g, bh, q0, group_exists);
        const int i = q0 + r;
        const bool row_ok = group_exists && i < N;
        const int ie = (i < N) ? i : N - 1;
        const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
        const int kvx = PAIR ? g : 0;

        // Q operand of this row, padding channels zeroed.
        {
            uint8_t* qop = smem + L.q + g * L.q_bytes;
            const uint32_t* src = p.bq + ((size_t)bh * N + ie) * W;
            for (int w = 0; w < W; ++w) {
                const uint32_t bits = row_ok ? __ldg(src + w) : 0u;
                const int nvalid = min(32, p.d - 32 * w);
                const uint32_t vm = nvalid >= 32 ? 0xFFFFFFFFu : ((1u << nvalid) - 1u);
                *reinterpret_cast<uint4*>(qop + core_off(r, 2 * w, chunks)) = expand16<QK>(bits & 0xFFFFu, vm & 0xFFFFu);
                *reinterpret_cast<uint4*>(qop + core_off(r, 2 * w + 1, chunks)) = expand16<QK>(bits >> 16, vm >> 16);
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[B_QREADY]);
        }
        const float cq = row_ok ? __ldg(p.muq + (size_t)bh * N + i) * p.q_scale : 0.f;
        const uint64_t cq2 = f2_pack(cq, cq);
        int rel_base = 0, rp_off = 0;
        if (is_relpos(BIAS)) {
            if (BIAS == BIAS_RP_FAST) {
                const int sidx = (BM - 1) - r;             // 127 - (ci - ci0)
                const int m = sidx & 3;
                rp_off = (g * 4 + m) * RP_STRIDE + (sidx - m);
            } else {
                const int ri = ie / p.gw, ci = ie - ri * p.gw;
                rel_base = (ri + p.gh - 1) * (2 * p.gw - 1) + ci + p.gw - 1;
            }
        }

        float mrow = -INFINITY;
        uint64_t l2[2] = {f2_pack(0.f, 0.f), f2_pack(0.f, 0.f)};
        uint64_t neg2 = 0;
        bool ok = true;
        for (int u = 0; u < U; ++u) {
            const int s = u % S, buf = u & 1;
            const bool pass_b = u >= T;
            const int t = pass_b ? u - T : u;
            const int j0 = t * BN;
            ok = warp_wait(&bars[B_SFULL + 2 * g + buf], (u >> 1) & 1, abort_flag) &&
                 warp_wait(&bars[B_FULL + s], (u / S) & 1, abort_flag);
            if (!ok) break;
            tc_fence_after();
            const bool ragged = j0 + BN > N;
            const uint8_t* tile_s = smem + L.k + s * L.k_bytes + kvx * L.tile;
            const float* muk_s = reinterpret_cast<const float*>(tile_s + BN * p.dpad);
            const int* koff_s = reinterpret_cast<const int*>(tile_s + BN * p.dpad + BN * 4);
            const uint8_t* bsm_row = smem + L.b + s * 2 * 16384 + r * 128;
            const float* rpc = (BIAS == BIAS_RP_FAST)
                ? reinterpret_cast<const float*>(smem + L.rp) + (size_t)s * NG * 4 * RP_STRIDE + rp_off : nullptr;
            const int nvalid = N - j0;
            uint32_t zr[64];
            tmem_ld64(tmem + (2 * g + buf) * BN + lane_base, zr);
            tmem_wait_ld();
            uint32_t pw[16];
            float mx[2] = {-INFINITY, -INFINITY};
            if (!pass_b) {
                if (ragged)
                    softmax_tile<QK, BIAS, false, true>(zr, muk_s, bsm_row, r & 7, rpc, koff_s, tab_h, rel_base,
                                                        nvalid, cq2, neg2, mx, l2, pw);
                else
                    softmax_tile<QK, BIAS, false, false>(zr, muk_s, bsm_row, r & 7, rpc, koff_s, tab_h, rel_base,
                                                         nvalid, cq2, neg2, mx, l2, pw);
                mrow = fmax3(mrow, mx[0], mx[1]);
            } else {
                if (ragged)
                    softmax_tile<QK, BIAS, true, true>(zr, muk_s, bsm_row, r & 7, rpc, koff_s, tab_h, rel_base,
                                                       nvalid, cq2, neg2, mx, l2, pw);
                else
                    softmax_tile<QK, BIAS, true, false>(zr, muk_s, bsm_row, r & 7, rpc, koff_s, tab_h, rel_base,
                                                        nvalid, cq2, neg2, mx, l2, pw);
                // The u8 codes go back into this row's lane of the S buffer: the
                // PV product reads them from TMEM.
                tmem_st16(tmem + (2 * g + buf) * BN + lane_base, pw);
                tmem_wait_st();
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&bars[B_SDONE + 2 * g + buf]);
                mbar_arrive(&bars[B_EMPTY + s]);
            }
            if (u == T - 1) neg2 = f2_pack(-mrow * LOG2E, -mrow * LOG2E);
        }

        // Epilogue: O = sv * acc / (255 l).
        if (ok) ok = warp_wait(&bars[B_OREADY], 0, abort_flag);
        if (!ok) {
            if (lane == 0) fail(abort_flag, p.status, kStatusTimeoutSoftmax);
        } else {
            tc_fence_after();
            float la, lb, lc, ld;
            f2_unpack(l2[0], la, lb);
            f2_unpack(l2[1], lc, ld);
            const float inv = 1.f / (255.f * ((la + lb) + (lc + ld)));
            OutT* dst = static_cast<OutT*>(p.out) + ((size_t)bh * N + ie) * p.d;
            const float* svp = p.sv + (size_t)bh * p.d;
            for (int c = 0; c < p.dv; c += 16) {
                uint32_t acc[16];
                tmem_ld16(tmem + 256 + 128 * g + c + lane_base, acc);
                tmem_wait_ld();
                if (row_ok) {
#pragma unroll
                    for (int e = 0; e < 16; ++e)
                        if (c + e < p.d) store1<OutT>(dst + c + e, __int2float_rn((int)acc[e]) * __ldg(svp + c + e) * inv);
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == MMA_WARP) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

// ------------------------------------------------------------------ host side

PFN_cuTensorMapEncodeTiled_v12000 encode_fn()
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

int dv_of(int d) { return (d + 15) / 16 * 16; }

constexpr size_t kSmemLimit = 227u * 1024u;

size_t smem_bytes(int d, int bias_kind, int stages)
{
    const Layout L = make_layout(32 * words_for(d), dv_of(d), bias_kind, stages);
    return (size_t)L.total + 1024;   // slack for the manual 1 KB alignment
}

// Deepest pipeline (2..4 stages) that fits; 0 if even 2 do not.
int pick_stages(int d, int bias_kind)
{
    for (int s = MAX_STAGES; s >= 2; --s)
        if (smem_bytes(d, bias_kind, s) <= kSmemLimit) return s;
    return 0;
}

template <int QK, typename OutT, int BIAS>
cudaError_t launch_t(const CUtensorMap& tv, const CUtensorMap& tb, const Params& p, size_t smem, cudaStream_t st)
{
    auto kern = attn_tc_kernel<QK, OutT, BIAS>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid = (BIAS == BA_BIAS_DENSE)
                    ? dim3(ceil_div(p.N, BM), p.H, ceil_div(p.B, 2))
                    : dim3(ceil_div(p.N, BM * NG), p.B * p.H, 1);
    kern<<<grid, NUM_THREADS, smem, st>>>(tv, tb, p);
    return cudaGetLastError();
}

template <int QK, typename OutT>
cudaError_t launch_bias(int kind, const CUtensorMap& tv, const CUtensorMap& tb, const Params& p, size_t smem,
                        cudaStream_t st)
{
    if (kind == BA_BIAS_DENSE) return launch_t<QK, OutT, BA_BIAS_DENSE>(tv, tb, p, smem, st);
    if (kind == BIAS_RP_FAST) return launch_t<QK, OutT, BIAS_RP_FAST>(tv, tb, p, smem, st);
    if (kind == BA_BIAS_RELPOS2D) return launch_t<QK, OutT, BA_BIAS_RELPOS2D>(tv, tb, p, smem, st);
    return launch_t<QK, OutT, BA_BIAS_NONE>(tv, tb, p, smem, st);
}

// The kernel variant for an ABI bias kind.
int kernel_bias(int bias_kind, int gw)
{
    return (bias_kind == BA_BIAS_RELPOS2D && gw % BM == 0) ? BIAS_RP_FAST : bias_kind;
}

// Workspace layout: staged key tiles, then (fast rel-pos path) staged table rows.
struct Workspace {
    int64_t kst_bytes, rps_off, rps_bytes, total;
};

Workspace workspace_layout(int B, int H, int N, int d, int bias_kind, int gh, int gw)
{
    const int vb = kernel_bias(bias_kind, gw);
    Workspace w;
    const int64_t tile = tile_bytes(32 * words_for(d), vb == BIAS_RP_FAST ? BA_BIAS_NONE : vb);
    w.kst_bytes = (int64_t)B * H * ceil_div(N, BN) * tile;
    w.rps_off = round_up64(w.kst_bytes, 256);
    w.rps_bytes = (vb == BIAS_RP_FAST) ? (int64_t)H * (2 * gh - 1) * 4 * (2 * (int64_t)gw) * 4 : 0;
    w.total = w.rps_off + w.rps_bytes;
    return w;
}

// Staging of the key side, one CTA per (64-key tile, batch*head): +-1 operand
// bytes in core-matrix order, the key scales (0 past N), and for the general
// rel-pos bias the key offsets rj (2 gw - 1) + cj.  Keys past N get operand
// rows of their (zero) sign bits; the kernel masks them out of the softmax.
template <int QK>
__global__ void __launch_bounds__(128)
stage_k_kernel(const uint32_t* __restrict__ bk, const float* __restrict__ muk, int N, int W, int T,
               int koff_gw, uint32_t tile, uint8_t* __restrict__ kst)
{
    const int t = blockIdx.x;
    const size_t bh = blockIdx.y;
    uint8_t* dst = kst + (bh * T + t) * tile;
    const int dpad = 32 * W, chunks = 2 * W;
    for (int e = threadIdx.x; e < BN * W; e += blockDim.x) {
        const int r = e / W, w = e - r * W;
        const int j = t * BN + r;
        const uint32_t bits = (j < N) ? __ldg(bk + (bh * N + j) * W + w) : 0u;
        *reinterpret_cast<uint4*>(dst + core_off(r, 2 * w, chunks)) = expand16<QK>(bits & 0xFFFFu, 0xFFFFu);
        *reinterpret_cast<uint4*>(dst + core_off(r, 2 * w + 1, chunks)) = expand16<QK>(bits >> 16, 0xFFFFu);
    }
    float* mu = reinterpret_cast<float*>(dst + BN * dpad);
    int* ko = reinterpret_cast<int*>(dst + BN * dpad + BN * 4);
    for (int r = threadIdx.x; r < BN; r += blockDim.x) {
        const int j = t * BN + r;
        mu[r] = (j < N) ? __ldg(muk + bh * N + j) : 0.f;
        if (koff_gw > 0) {
            const int jj = (j < N) ? j : N - 1;
            const int rj = jj / koff_gw;
            ko[r] = rj * (2 * koff_gw - 1) + (jj - rj * koff_gw);
        }
    }
}

// Staging of the rel-pos table for the fast path: for head h and row rho of
// the table, copy m holds the reversed row shifted by m,
// rps[h][rho][m][x] = table[h][rho][2 gw - 2 - (x + m)] (0 past the row's end).
__global__ void __launch_bounds__(256)
stage_rp_kernel(const float* __restrict__ table, int gh, int gw, int64_t total, float* __restrict__ rps)
{
    const int64_t row_len = 2 * (int64_t)gw;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t x = i % row_len;
        const int64_t rest = i / row_len;              // (h (2 gh - 1) + rho) * 4 + m
        const int m = (int)(rest & 3);
        const int64_t row = rest >> 2;                 // h (2 gh - 1) + rho
        const int64_t src = x + m;
        rps[i] = (src <= 2 * (int64_t)gw - 2) ? __ldg(table + row * (2 * gw - 1) + (2 * gw - 2 - src)) : 0.f;
    }
}

}  // namespace

bool attn_tc_supports(int bias_kind, int gh, int gw, int N, int d)
{
    (void)gh; (void)N;
    if (d < 1 || d > 128) return false;
    return pick_stages(d, kernel_bias(bias_kind, gw)) >= 2;
}

int64_t attn_tc_workspace_bytes(int B, int H, int N, int d, int bias_kind, int gh, int gw)
{
    if (!attn_tc_supports(bias_kind, gh, gw, N, d)) return 0;
    return workspace_layout(B, H, N, d, bias_kind, gh, gw).total;
}

cudaError_t launch_attn_tc(const uint32_t* bq, const float* muq, const uint32_t* bk, const float* muk,
                           const int8_t* vq, const float* sv, int bias_kind, const float* bias,
                           int64_t bias_ld, int gh, int gw, int B, int H, int N, int d,
                           void* workspace, int64_t workspace_bytes,
                           void* out, ba_dtype out_dt, int variant, unsigned* status, cudaStream_t st)
{
    if (!attn_tc_supports(bias_kind, gh, gw, N, d)) return cudaErrorNotSupported;
    const Workspace ws = workspace_layout(B, H, N, d, bias_kind, gh, gw);
    if (workspace == nullptr || workspace_bytes < ws.total) return cudaErrorInvalidValue;
    auto encode = encode_fn();
    if (!encode) return cudaErrorNotSupported;
    const int BH = B * H;
    const int dv = dv_of(d);
    const int64_t ldv = round_up64(N, 16);
    const int vb = kernel_bias(bias_kind, gw);
    const bool f8 = variant != BA_QK_TC_I8;

    CUtensorMap tv, tb;
    memset(&tv, 0, sizeof(tv));
    memset(&tb, 0, sizeof(tb));
    {
        cuuint64_t dims[3] = {(cuuint64_t)ldv, (cuuint64_t)d, (cuuint64_t)BH};
        cuuint64_t strides[2] = {(cuuint64_t)ldv, (cuuint64_t)ldv * d};
        cuuint32_t box[3] = {(cuuint32_t)BN, (cuuint32_t)dv, 1};
        cuuint32_t es[3] = {1, 1, 1};
        if (encode(&tv, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<int8_t*>(vq), dims, strides, box, es,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    if (bias_kind == BA_BIAS_DENSE) {
        cuuint64_t dims[3] = {(cuuint64_t)bias_ld, (cuuint64_t)N, (cuuint64_t)H};
        cuuint64_t strides[2] = {(cuuint64_t)bias_ld * 4, (cuuint64_t)bias_ld * 4 * N};
        cuuint32_t box[3] = {32, (cuuint32_t)BM, 1};
        cuuint32_t es[3] = {1, 1, 1};
        if (encode(&tb, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<float*>(bias), dims, strides, box, es,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }

    Params p;
    p.bq = bq; p.muq = muq; p.sv = sv;
    p.kst = static_cast<const uint8_t*>(workspace);
    p.rps = (vb == BIAS_RP_FAST) ? reinterpret_cast<const float*>(static_cast<uint8_t*>(workspace) + ws.rps_off)
                                 : nullptr;
    p.table = bias_kind == BA_BIAS_RELPOS2D ? bias : nullptr;
    p.out = out;
    p.B = B; p.H = H; p.N = N; p.d = d; p.W = words_for(d); p.dpad = 32 * p.W; p.dv = dv;
    p.n_tiles = ceil_div(N, BN);
    p.stages = pick_stages(d, vb);
    p.gh = gh; p.gw = gw;
    p.q_scale = (float)(1.0 / sqrt((double)d));
    p.status = status;

    // Staging pre-passes (same stream, so the attention kernel sees them).
    {
        const uint32_t tile = tile_bytes(p.dpad, vb == BIAS_RP_FAST ? BA_BIAS_NONE : vb);
        uint8_t* kst = static_cast<uint8_t*>(workspace);
        const int koff_gw = (vb == BA_BIAS_RELPOS2D) ? gw : 0;
        dim3 grid(p.n_tiles, BH);
        if (f8) stage_k_kernel<QK_F8><<<grid, 128, 0, st>>>(bk, muk, N, p.W, p.n_tiles, koff_gw, tile, kst);
        else stage_k_kernel<QK_I8><<<grid, 128, 0, st>>>(bk, muk, N, p.W, p.n_tiles, koff_gw, tile, kst);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
        if (vb == BIAS_RP_FAST) {
            const int64_t total = ws.rps_bytes / 4;
            const int blocks = (int)((total + 255) / 256 < 148 * 8 ? (total + 255) / 256 : 148 * 8);
            stage_rp_kernel<<<blocks, 256, 0, st>>>(bias, gh, gw, total,
                                                     reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + ws.rps_off));
            e = cudaGetLastError();
            if (e != cudaSuccess) return e;
        }
    }

    // One CTA per SM: each takes all 512 TMEM columns.
    size_t smem = smem_bytes(d, vb, p.stages);
    if (smem < 120u * 1024u) smem = 120u * 1024u;

    if (out_dt == BA_BF16)
        return f8 ? launch_bias<QK_F8, __nv_bfloat16>(vb, tv, tb, p, smem, st)
                  : launch_bias<QK_I8, __nv_bfloat16>(vb, tv, tb, p, smem, st);
    return f8 ? launch_bias<QK_F8, float>(vb, tv, tb, p, smem, st)
              : launch_bias<QK_I8, float>(vb, tv, tb, p, smem, st);
}

}  // namespace ba
