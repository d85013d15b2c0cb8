// ba_attn_tc.cu -- the BinaryAttention forward on the sm_100a tensor cores.
//
// BA notes (paper-notes page "BinaryAttention: One-Bit QK-Attention for
// Vision and Diffusion Transformers", CVPR 2026):
//   Key design 1: s_i . t_j from sign bits, per-token scales mu
//   Key design 2: S_ij = mu_q,i mu_k,j s_i.t_j / sqrt(d) + b_ij
//   Key design 3: P~ as u8 with scale 1/255, int8 V per channel, integer PV
//   Overall framework: FlashAttention2-style tiling with an online softmax.
//
// The A100 design on the page (mma.sync .b1 for QK, mma.sync u8.s8 for PV) is
// prior art; this kernel is built for Blackwell instead:
//   * one CTA per 128-query tile (M = 128 = TMEM lanes, one softmax thread per
//     query row, so row max / row sum need no shuffles);
//   * QK on tcgen05.mma with the sign bits expanded to +-1 operands in shared
//     memory (kind::i8 -> s32, or kind::f8f6f4 with e4m3 +-1 -> f32; both
//     exact), accumulating S in TMEM, double-buffered so QK of the next key
//     tile overlaps the softmax of this one;
//   * PV on tcgen05.mma kind::i8 with u8 P and s8 V (K-major int8 V tiles
//     brought in by TMA with 128-byte swizzle), the s32 accumulator living in
//     TMEM across all key tiles;
//   * the online softmax keeps m and l in registers; when a warp's running
//     maxima move, that warp rescales its accumulator rows in TMEM with a
//     fixed-point multiply (exact to half a unit);
//   * a dense bias tile is staged by TMA (128-byte swizzle, conflict-free
//     reads); a 2-D relative-position bias is gathered from the per-head table
//     through a per-key offset the load warp precomputes.
// Warp roles: warp 0 loads (TMA + sign-bit expansion), warp 1 issues MMAs and
// owns TMEM, warps 2..5 run the softmax and the epilogue.
//
// Every wait on an mbarrier is bounded; on a timeout the kernel records a bit
// in the device status word, tells the other roles to stop, lets in-flight
// tensor-core work drain, frees TMEM and returns.
#include <cudaTypedefs.h>

#include <mutex>

#include "ba_common.cuh"
#include "ba_sm100.cuh"

namespace ba {
namespace {

using namespace sm100;

constexpr int BM = 128;          // query rows per CTA (= TMEM lanes)
constexpr int BN = 128;          // keys per tile
constexpr int STAGES = 2;        // key/value/bias buffers
constexpr int NUM_THREADS = 192;
constexpr uint32_t TMEM_COLS = 512;
constexpr float LOG2E = 1.4426950408889634f;
constexpr int QK_I8 = 0, QK_F8 = 1;

// Barrier slots.
enum {
    B_Q = 0,
    B_SFULL = 1,     // 2: S tile in TMEM buffer b ready
    B_SEMPTY = 3,    // 2: softmax has read S buffer b
    B_PFULL = 5,     // P tile written (and accumulator rescaled)
    B_PVDONE = 6,    // PV of the tile finished
    B_KFULL = 7,     // STAGES: K operand, mu_k, key offsets ready
    B_VFULL = 9,     // STAGES: V (and dense bias) TMA landed
    B_KVEMPTY = 11,  // STAGES: stage may be overwritten
    B_FINAL = 13,
    NUM_BARS = 14
};

struct Layout {
    uint32_t v[STAGES], b[STAGES], q, k[STAGES], p, muk[STAGES], koff[STAGES], bars, misc, total;
};

__host__ __device__ inline uint32_t align_up(uint32_t x, uint32_t a) { return (x + a - 1) / a * a; }

__host__ __device__ inline Layout make_layout(int dpad, int dv, bool dense_bias)
{
    Layout L;
    uint32_t off = 0;
    for (int s = 0; s < STAGES; ++s) { (s ? L.v[1] : L.v[0]) = off; off = align_up(off + dv * 128u, 1024); }
    for (int s = 0; s < STAGES; ++s) { (s ? L.b[1] : L.b[0]) = off; off = align_up(off + (dense_bias ? 4u * 16384u : 0u), 1024); }
    L.q = off; off = align_up(off + BM * (uint32_t)dpad, 1024);
    for (int s = 0; s < STAGES; ++s) { (s ? L.k[1] : L.k[0]) = off; off = align_up(off + BN * (uint32_t)dpad, 1024); }
    L.p = off; off = align_up(off + BM * BN, 1024);
    for (int s = 0; s < STAGES; ++s) { (s ? L.muk[1] : L.muk[0]) = off; off += BN * 4; }
    for (int s = 0; s < STAGES; ++s) { (s ? L.koff[1] : L.koff[0]) = off; off += BN * 4; }
    L.bars = off; off += NUM_BARS * 8;
    L.misc = off; off += 16;        // TMEM base address, abort flag
    L.total = off;
    return L;
}

struct Params {
    const uint32_t* bq;
    const float* muq;
    const uint32_t* bk;
    const float* muk;
    const float* sv;
    const float* table;      // 2-D relative-position table (global)
    void* out;
    int H, N, d, W, dpad, dv, n_tiles;
    int gh, gw;
    float q_scale;           // 1 / sqrt(d)
    unsigned* status;
};

// 16 sign bits -> 16 bytes of +-1 operands (+1 where the bit is set), with
// byte lanes whose bit in `valid` is 0 forced to 0 (padding channels).
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

// Byte offset of (row r, 16-byte chunk kc) in a K-major, non-swizzled
// operand whose rows hold `chunks` 16-byte chunks: 8x16-byte core matrices,
// chunk-adjacent core matrices 128 bytes apart, 8-row groups chunks*128 apart.
__device__ __forceinline__ uint32_t core_off(int r, int kc, int chunks)
{
    return (uint32_t)((r >> 3) * chunks * 128 + kc * 128 + (r & 7) * 16);
}

// Warp-uniform bounded wait: every lane polls; all agree on the outcome.
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

template <int QK, typename OutT, int BIAS>
__global__ void __launch_bounds__(NUM_THREADS, 1)
attn_tc_kernel(const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_b,
               const Params p)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const Layout L = make_layout(p.dpad, p.dv, BIAS == BA_BIAS_DENSE);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.bars);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L.misc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L.misc + 4);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int bh = blockIdx.y;
    const int h = bh % p.H;
    const int q0 = blockIdx.x * BM;
    const int N = p.N, W = p.W, T = p.n_tiles;
    const int chunks = p.dpad / 16;

    if (threadIdx.x == 0) {
        mbar_init(&bars[B_Q], 4);
        for (int b = 0; b < 2; ++b) {
            mbar_init(&bars[B_SFULL + b], 1);
            mbar_init(&bars[B_SEMPTY + b], 4);
        }
        mbar_init(&bars[B_PFULL], 4);
        mbar_init(&bars[B_PVDONE], 1);
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&bars[B_KFULL + s], 1);
            mbar_init(&bars[B_VFULL + s], 1);
            mbar_init(&bars[B_KVEMPTY + s], 1);
        }
        mbar_init(&bars[B_FINAL], 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, TMEM_COLS);
        tmem_relinquish();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tmap(&tm_v);
        if (BIAS == BA_BIAS_DENSE) prefetch_tmap(&tm_b);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------------------ loads
        for (int t = 0; t < T; ++t) {
            const int s = t % STAGES, use = t / STAGES;
            if (t >= STAGES && !warp_wait(&bars[B_KVEMPTY + s], (use - 1) & 1, abort_flag)) {
                if (lane == 0) fail(abort_flag, p.status, kStatusTimeoutProducer);
                break;
            }
            const int j0 = t * BN;
            if (lane == 0) {
                const uint32_t bytes = (uint32_t)p.dv * 128u + (BIAS == BA_BIAS_DENSE ? 4u * 16384u : 0u);
                mbar_arrive_expect_tx(&bars[B_VFULL + s], bytes);
                tma_load_3d(smem + (s ? L.v[1] : L.v[0]), &tm_v, &bars[B_VFULL + s], j0, 0, bh);
                if (BIAS == BA_BIAS_DENSE)
                    for (int b = 0; b < 4; ++b)
                        tma_load_3d(smem + (s ? L.b[1] : L.b[0]) + b * 16384, &tm_b, &bars[B_VFULL + s], j0 + 32 * b, q0, h);
            }
            uint8_t* kop = smem + (s ? L.k[1] : L.k[0]);
            float* muk_s = reinterpret_cast<float*>(smem + (s ? L.muk[1] : L.muk[0]));
            int* koff_s = reinterpret_cast<int*>(smem + (s ? L.koff[1] : L.koff[0]));
            for (int r = lane; r < BN; r += 32) {
                const int j = j0 + r;
                const bool valid = j < N;
                const uint32_t* src = p.bk + ((size_t)bh * N + j) * W;
                for (int w = 0; w < W; ++w) {
                    const uint32_t bits = valid ? __ldg(src + w) : 0u;
                    *reinterpret_cast<uint4*>(kop + core_off(r, 2 * w, chunks)) = expand16<QK>(bits & 0xFFFFu, 0xFFFFu);
                    *reinterpret_cast<uint4*>(kop + core_off(r, 2 * w + 1, chunks)) = expand16<QK>(bits >> 16, 0xFFFFu);
                }
                muk_s[r] = valid ? __ldg(p.muk + (size_t)bh * N + j) : 0.f;
                if (BIAS == BA_BIAS_RELPOS2D) {
                    const int jj = valid ? j : N - 1;
                    const int rj = jj / p.gw, cj = jj - rj * p.gw;
                    koff_s[r] = rj * (2 * p.gw - 1) + cj;
                }
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[B_KFULL + s]);
        }
        // On an abort, let TMA copies already issued land before the CTA exits.
        if (*abort_flag && lane == 0) {
            for (int t = (T > STAGES ? T - STAGES : 0); t < T; ++t)
                mbar_wait(&bars[B_VFULL + t % STAGES], (t / STAGES) & 1, nullptr, 100000000ull);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issue
        if (lane == 0) {
            const uint32_t idesc_qk = (QK == QK_I8) ? instr_desc(kCS32, kFmtS8, kFmtS8, BM, BN)
                                                    : instr_desc(kCF32, kFmtE4M3, kFmtE4M3, BM, BN);
            const uint32_t idesc_pv = instr_desc(kCS32, kFmtU8, kFmtS8, BM, p.dv);
            const uint32_t sbo_qk = (uint32_t)chunks * 128u;
            const uint32_t q_base = smem_addr(smem + L.q);
            const uint32_t p_base = smem_addr(smem + L.p);
            const uint32_t tm_o = tmem + 256;
            bool ok = mbar_wait(&bars[B_Q], 0, abort_flag) && mbar_wait(&bars[B_KFULL], 0, abort_flag);
            auto issue_qk = [&](int buf, int stage) {
                const uint32_t k_base = smem_addr(smem + (stage ? L.k[1] : L.k[0]));
                for (int kk = 0; kk < p.dpad / 32; ++kk) {
                    const uint64_t a = smem_desc(q_base + kk * 256, 128, sbo_qk, kLayoutNone);
                    const uint64_t b = smem_desc(k_base + kk * 256, 128, sbo_qk, kLayoutNone);
                    mma_ss<QK>(tmem + buf * 128, a, b, idesc_qk, kk > 0 ? 1u : 0u);
                }
                mma_commit(&bars[B_SFULL + buf]);
            };
            if (ok) {
                tc_fence_after();
                issue_qk(0, 0);
            }
            for (int t = 0; ok && t < T; ++t) {
                const int s = t % STAGES;
                if (t + 1 < T) {
                    const int s1 = (t + 1) % STAGES, buf = (t + 1) & 1;
                    ok = mbar_wait(&bars[B_KFULL + s1], ((t + 1) / STAGES) & 1, abort_flag);
                    if (ok && t + 1 >= 2) ok = mbar_wait(&bars[B_SEMPTY + buf], (((t + 1) >> 1) - 1) & 1, abort_flag);
                    if (!ok) break;
                    tc_fence_after();
                    issue_qk(buf, s1);
                }
                ok = mbar_wait(&bars[B_PFULL], t & 1, abort_flag) &&
                     mbar_wait(&bars[B_VFULL + s], (t / STAGES) & 1, abort_flag);
                if (!ok) break;
                tc_fence_after();
                const uint32_t v_base = smem_addr(smem + (s ? L.v[1] : L.v[0]));
                for (int kk = 0; kk < BN / 32; ++kk) {
                    const uint64_t a = smem_desc(p_base + kk * 256, 128, 1024, kLayoutNone);
                    const uint64_t b = smem_desc(v_base + kk * 32, 16, 1024, kLayoutSw128);
                    mma_ss<QK_I8>(tm_o, a, b, idesc_pv, (t > 0 || kk > 0) ? 1u : 0u);
                }
                mma_commit(&bars[B_PVDONE]);
                mma_commit(&bars[B_KVEMPTY + s]);
            }
            if (!ok) fail(abort_flag, p.status, kStatusTimeoutMma);
            // Let every issued MMA finish before TMEM is released.
            mma_commit(&bars[B_FINAL]);
            if (!mbar_wait(&bars[B_FINAL], 0, abort_flag, 4000000000ull)) atomicOr(p.status, kStatusTimeoutMma);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ softmax + epilogue
        const int quarter = warp & 3;                 // TMEM lanes this warp may access
        const int r = quarter * 32 + lane;            // row within the tile
        const int i = q0 + r;
        const bool row_ok = i < N;
        const int ie = row_ok ? i : N - 1;
        const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;

        // Q operand: this thread's row, padding channels zeroed.
        {
            uint8_t* qop = smem + L.q;
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
            if (lane == 0) mbar_arrive(&bars[B_Q]);
        }
        const float cq = row_ok ? __ldg(p.muq + (size_t)bh * N + i) * p.q_scale : 0.f;
        int rel_base = 0;
        const float* tab = p.table;
        if (BIAS == BA_BIAS_RELPOS2D) {
            const int ri = ie / p.gw, ci = ie - ri * p.gw;
            rel_base = (ri + p.gh - 1) * (2 * p.gw - 1) + ci + p.gw - 1;
            tab += (size_t)h * (2 * p.gh - 1) * (2 * p.gw - 1);
        }

        float m = -INFINITY, l = 0.f;
        bool ok = true;
        for (int t = 0; t < T; ++t) {
            const int s = t % STAGES, buf = t & 1;
            const int j0 = t * BN;
            ok = warp_wait(&bars[B_SFULL + buf], (t >> 1) & 1, abort_flag) &&
                 warp_wait(&bars[B_KFULL + s], (t / STAGES) & 1, abort_flag);
            if (ok && BIAS == BA_BIAS_DENSE) ok = warp_wait(&bars[B_VFULL + s], (t / STAGES) & 1, abort_flag);
            if (!ok) break;
            tc_fence_after();

            float sc[BN];
            {
                uint32_t z[32];
#pragma unroll
                for (int c = 0; c < BN / 32; ++c) {
                    tmem_ld32(tmem + buf * 128 + c * 32 + lane_base, z);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; ++e)
                        sc[c * 32 + e] = (QK == QK_I8) ? __int2float_rn((int)z[e]) : __uint_as_float(z[e]);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[B_SEMPTY + buf]);

            // S = mu_q mu_k z / sqrt(d) + b  (Key design 2), and the tile max
            const float* muk_s = reinterpret_cast<const float*>(smem + (s ? L.muk[1] : L.muk[0]));
            const int* koff_s = reinterpret_cast<const int*>(smem + (s ? L.koff[1] : L.koff[0]));
            const uint8_t* bsm = smem + (s ? L.b[1] : L.b[0]) + r * 128;
            float mx = -INFINITY;
#pragma unroll
            for (int c4 = 0; c4 < BN / 4; ++c4) {
                const float4 mk = *reinterpret_cast<const float4*>(muk_s + 4 * c4);
                float bb[4] = {0.f, 0.f, 0.f, 0.f};
                if (BIAS == BA_BIAS_DENSE) {
                    const int box = c4 >> 3, k = c4 & 7;
                    const float4 v = *reinterpret_cast<const float4*>(bsm + box * 16384 + ((k ^ (r & 7)) << 4));
                    bb[0] = v.x; bb[1] = v.y; bb[2] = v.z; bb[3] = v.w;
                } else if (BIAS == BA_BIAS_RELPOS2D) {
                    const int4 ko = *reinterpret_cast<const int4*>(koff_s + 4 * c4);
                    bb[0] = __ldg(tab + rel_base - ko.x);
                    bb[1] = __ldg(tab + rel_base - ko.y);
                    bb[2] = __ldg(tab + rel_base - ko.z);
                    bb[3] = __ldg(tab + rel_base - ko.w);
                }
                const float mkv[4] = {mk.x, mk.y, mk.z, mk.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int c = 4 * c4 + e;
                    const float x = fmaf(sc[c] * mkv[e], cq, bb[e]);
                    sc[c] = x;
                    mx = fmaxf(mx, x);
                }
            }
            if (j0 + BN > N) {               // ragged last tile: keys >= N do not exist
                mx = -INFINITY;
#pragma unroll
                for (int c = 0; c < BN; ++c) {
                    if (j0 + c >= N) sc[c] = -INFINITY;
                    mx = fmaxf(mx, sc[c]);
                }
            }
            const float m_new = fmaxf(m, mx);
            const float alpha = ex2((m - m_new) * LOG2E);      // 0 on the first tile
            const float neg = -m_new * LOG2E;
            l *= alpha;

            // P buffer and accumulator are free once PV of the previous tile is done.
            if (t > 0 && !warp_wait(&bars[B_PVDONE], (t - 1) & 1, abort_flag)) { ok = false; break; }
            if (t > 0 && __any_sync(0xffffffffu, alpha < 1.f)) {
                tc_fence_after();
                const long long aq = (long long)__float2uint_rn(alpha * 2147483648.0f);
                for (int c = 0; c < p.dv; c += 16) {
                    uint32_t acc[16];
                    tmem_ld16(tmem + 256 + c + lane_base, acc);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 16; ++e)
                        acc[e] = (uint32_t)(int)(((long long)(int)acc[e] * aq + (1ll << 30)) >> 31);
                    tmem_st16(tmem + 256 + c + lane_base, acc);
                }
                tmem_wait_st();
            }

            // P~ = exp(S - m), l += P~, pq = round(255 P~) as u8 (Key design 3)
            uint8_t* prow = smem + L.p + (r >> 3) * 1024 + (r & 7) * 16;
#pragma unroll
            for (int kc = 0; kc < BN / 16; ++kc) {
                uint32_t wv[4];
#pragma unroll
                for (int g = 0; g < 4; ++g) {
                    uint32_t b4[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float pr = ex2(fmaf(sc[kc * 16 + g * 4 + e], LOG2E, neg));
                        l += pr;
                        b4[e] = __float_as_uint(fmaf(pr, 255.f, 12582912.f));   // low byte = rint(255 P~)
                    }
                    wv[g] = __byte_perm(__byte_perm(b4[0], b4[1], 0x0040), __byte_perm(b4[2], b4[3], 0x0040), 0x5410);
                }
                *reinterpret_cast<uint4*>(prow + kc * 128) = make_uint4(wv[0], wv[1], wv[2], wv[3]);
            }
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[B_PFULL]);
            m = m_new;
        }

        // Epilogue: O = sv * acc / (255 l).
        if (ok) ok = warp_wait(&bars[B_PVDONE], (T - 1) & 1, abort_flag);
        if (!ok) {
            if (lane == 0) fail(abort_flag, p.status, kStatusTimeoutSoftmax);
        } else {
            tc_fence_after();
            const float inv = 1.f / (255.f * l);
            OutT* dst = static_cast<OutT*>(p.out) + ((size_t)bh * N + ie) * p.d;
            const float* svp = p.sv + (size_t)bh * p.d;
            for (int c = 0; c < p.dv; c += 16) {
                uint32_t acc[16];
                tmem_ld16(tmem + 256 + c + lane_base, acc);
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
    if (warp == 1) {
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

size_t smem_bytes(int d, int bias_kind)
{
    const Layout L = make_layout(32 * words_for(d), dv_of(d), bias_kind == BA_BIAS_DENSE);
    return (size_t)L.total + 1024;   // slack for the manual 1 KB alignment
}

template <int QK, typename OutT, int BIAS>
cudaError_t launch_t(const CUtensorMap& tv, const CUtensorMap& tb, const Params& p, int BH, size_t smem,
                     cudaStream_t st)
{
    auto kern = attn_tc_kernel<QK, OutT, BIAS>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid(ceil_div(p.N, BM), BH);
    kern<<<grid, NUM_THREADS, smem, st>>>(tv, tb, p);
    return cudaGetLastError();
}

template <int QK, typename OutT>
cudaError_t launch_bias(int kind, const CUtensorMap& tv, const CUtensorMap& tb, const Params& p, int BH,
                        size_t smem, cudaStream_t st)
{
    if (kind == BA_BIAS_DENSE) return launch_t<QK, OutT, BA_BIAS_DENSE>(tv, tb, p, BH, smem, st);
    if (kind == BA_BIAS_RELPOS2D) return launch_t<QK, OutT, BA_BIAS_RELPOS2D>(tv, tb, p, BH, smem, st);
    return launch_t<QK, OutT, BA_BIAS_NONE>(tv, tb, p, BH, smem, st);
}

}  // namespace

bool attn_tc_supports(int bias_kind, int gh, int gw, int N, int d)
{
    (void)gh; (void)gw; (void)N;
    if (d < 1 || d > 128) return false;
    // The whole pipeline must fit one CTA's shared memory, with room to keep a
    // second CTA off the SM (it would only wait for tensor memory).
    return smem_bytes(d, bias_kind) <= 227u * 1024u;
}

cudaError_t launch_attn_tc(const uint32_t* bq, const float* muq, const uint32_t* bk, const float* muk,
                           const int8_t* vq, const float* sv, int bias_kind, const float* bias,
                           int64_t bias_ld, int gh, int gw, int B, int H, int N, int d,
                           void* out, ba_dtype out_dt, int variant, unsigned* status, cudaStream_t st)
{
    if (!attn_tc_supports(bias_kind, gh, gw, N, d)) return cudaErrorNotSupported;
    auto encode = encode_fn();
    if (!encode) return cudaErrorNotSupported;
    const int BH = B * H;
    const int dv = dv_of(d);
    const int64_t ldv = round_up64(N, 16);

    CUtensorMap tv, tb;
    memset(&tv, 0, sizeof(tv));
    memset(&tb, 0, sizeof(tb));
    {
        cuuint64_t dims[3] = {(cuuint64_t)ldv, (cuuint64_t)d, (cuuint64_t)BH};
        cuuint64_t strides[2] = {(cuuint64_t)ldv, (cuuint64_t)ldv * d};
        cuuint32_t box[3] = {(cuuint32_t)BN, (cuuint32_t)dv, 1};
        cuuint32_t es[3] = {1, 1, 1};
        if (encode(&tv, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<int8_t*>(vq), dims, strides, box, es,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
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
    p.bq = bq; p.muq = muq; p.bk = bk; p.muk = muk; p.sv = sv;
    p.table = bias_kind == BA_BIAS_RELPOS2D ? bias : nullptr;
    p.out = out;
    p.H = H; p.N = N; p.d = d; p.W = words_for(d); p.dpad = 32 * p.W; p.dv = dv;
    p.n_tiles = ceil_div(N, BN);
    p.gh = gh; p.gw = gw;
    p.q_scale = (float)(1.0 / sqrt((double)d));
    p.status = status;

    // Ask for enough shared memory that only one CTA fits on an SM: each CTA
    // takes all 512 TMEM columns.
    size_t smem = smem_bytes(d, bias_kind);
    if (smem < 120u * 1024u) smem = 120u * 1024u;

    const bool f8 = variant == BA_QK_TC_F8;
    if (out_dt == BA_BF16)
        return f8 ? launch_bias<QK_F8, __nv_bfloat16>(bias_kind, tv, tb, p, BH, smem, st)
                  : launch_bias<QK_I8, __nv_bfloat16>(bias_kind, tv, tb, p, BH, smem, st);
    return f8 ? launch_bias<QK_F8, float>(bias_kind, tv, tb, p, BH, smem, st)
              : launch_bias<QK_I8, float>(bias_kind, tv, tb, p, BH, smem, st);
}

}  // namespace ba
