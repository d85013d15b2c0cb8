// ba_attn_tc_pair.cu -- the tensor-core attention for a dense bias shared
// over the batch: a work tile is the same 128 query rows of two batch
// elements (two row groups), so one staged bias tile serves both.  The kernel
// is persistent (one CTA per SM walks tiles blockIdx.x, + gridDim.x, ...): the
// loader and the MMA thread start the next tile while the softmax warps are
// still in the previous tile's epilogue, and no CTA launch, TMEM allocation or
// pipeline fill is paid per tile.
//
// BA notes (paper-notes page "BinaryAttention: One-Bit QK-Attention for
// Vision and Diffusion Transformers", CVPR 2026): Key designs 1-3 and the
// tiled Overall framework, as in ba_attn_tc.cu.  Differences from that kernel:
//   * two row groups per CTA, one softmax thread per row, 64-key steps: the
//     QK product of a group is N = 64, its S tile double-buffered in TMEM
//     (2 groups x 2 buffers x 64 columns, outputs at columns 256 and 384);
//   * per stage the loader brings two staged 64-key tiles (one per batch
//     element), two dense-bias boxes of 32 keys x 128 rows (TMA, 128-byte
//     swizzle) shared by both groups, and in pass B two V tiles.
// Warps 0-7 run the softmax (two groups of four), warp 8 loads, warp 9
// issues the MMAs and owns TMEM.  Every mbarrier wait is bounded; on a timeout
// the kernel records a status bit, lets issued work drain, frees TMEM and
// returns.
#include "ba_attn_tc_common.cuh"
#include "ba_tc_warp.cuh"

namespace ba {
namespace tc {
namespace {

constexpr int NG = 2;                   // row groups per CTA (batch elements 2z, 2z + 1)
constexpr int BN = 64;                  // keys per step
constexpr int KVG = 2;                  // key/value sets per stage
constexpr int MAX_STAGES = 4;
constexpr int NUM_SOFTMAX_WARPS = 4 * NG;                   // 8
constexpr int LOAD_WARP = NUM_SOFTMAX_WARPS;                // 8
constexpr int MMA_WARP = LOAD_WARP + 1;                     // 9
constexpr int NUM_THREADS = 32 * (MMA_WARP + 1);            // 320

// Barrier slots.
enum {
    B_QREADY = 0,
    B_FULL = 1,                      // [stage] key tiles, bias (and V in pass B) landed
    B_EMPTY = B_FULL + MAX_STAGES,   // [stage] stage may be overwritten
    B_SFULL = B_EMPTY + MAX_STAGES,  // [NG][2] S tile in TMEM ready
    B_SDONE = B_SFULL + 2 * NG,      // [NG][2] softmax done with the S buffer (pass B: u8 P written into it)
    B_OREADY = B_SDONE + 2 * NG,     // every PV of the tile finished (one phase per tile)
    B_OFREE = B_OREADY + 1,          // the softmax warps read the tile's output accumulators
    B_FINAL = B_OFREE + 1,
    NUM_BARS
};

struct Layout {
    uint32_t stages, tile;      // pipeline depth; staged 64-key tile bytes
    uint32_t v, v_bytes;        // [stage][KVG] V tiles (SW64 K-major, dv rows x 64 bytes)
    uint32_t b;                 // [stage][2] dense bias boxes, 16 KB each (SW128)
    uint32_t q, q_bytes;        // [NG] Q operands
    uint32_t k, k_bytes;        // [stage] KVG staged key tiles
    uint32_t bars, misc, total;
};

__host__ __device__ inline Layout make_layout(int dpad, int dv, int stages)
{
    Layout L;
    L.stages = stages;
    L.tile = tile_bytes(BN, dpad, BA_BIAS_DENSE);
    uint32_t off = 0;
    L.v_bytes = align_up((uint32_t)dv * BN, 1024);
    L.v = off; off += stages * KVG * L.v_bytes;
    L.b = off; off += stages * 2 * 16384u;
    L.q_bytes = align_up((uint32_t)BM * dpad, 1024);
    L.q = off; off += NG * L.q_bytes;
    L.k_bytes = align_up(KVG * L.tile, 128);
    L.k = off; off += stages * L.k_bytes;
    L.bars = off; off += NUM_BARS * 8;
    L.misc = off; off += 16;            // TMEM base address, abort flag
    L.total = off;
    return L;
}

struct Params {
    const uint32_t* bq;
    const float* muq;
    const uint8_t* kst;      // staged key tiles [B*H][n_tiles][tile]
    const float* sv;
    void* out;
    int B, H, N, d, W, dpad, dv, n_tiles, stages;
    int tiles_x, tiles;      // row blocks per head; work tiles (row block, head, batch pair)
    float q_scale;           // 1 / sqrt(d)
    unsigned* status;
};

// Work tile k = (row block x, head y, batch pair z), x fastest.
struct TileCoord {
    int x, y, z;
};
__device__ __forceinline__ TileCoord tile_coord(const Params& p, int k)
{
    TileCoord c;
    c.x = k % p.tiles_x;
    const int rest = k / p.tiles_x;
    c.y = rest % p.H;
    c.z = rest / p.H;
    return c;
}

// Which (batch*head, first query row) group g of a tile covers and whether it
// exists: batch elements 2z and 2z + 1 of head y, rows 128 x.
__device__ __forceinline__ void group_coords(const Params& p, const TileCoord& tc, int g, int& bh, int& q0,
                                             bool& exists)
{
    int b = 2 * tc.z + g;
    exists = b < p.B;
    if (!exists) b = p.B - 1;
    bh = b * p.H + tc.y;
    q0 = tc.x * BM;
}

template <int QK, typename OutT>
__global__ void __maxnreg__(MAX_REGS)
attn_pair_kernel(const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_b,
                 const Params p)
{
    constexpr int BIAS = BA_BIAS_DENSE;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const Layout L = make_layout(p.dpad, p.dv, p.stages);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.bars);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L.misc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L.misc + 4);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int N = p.N, W = p.W, T = p.n_tiles, U = 2 * T;   // steps: pass A then pass B
    const int S = p.stages;
    const int chunks = p.dpad / 16;

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
        mbar_init(&bars[B_OFREE], NUM_SOFTMAX_WARPS);
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
        prefetch_tmap(&tm_b);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == LOAD_WARP) {
        // ---------------------------------------------------------------- loader
        // One thread fills stage u % S for step u: the two staged key tiles,
        // two dense-bias boxes (keys j0 .. j0 + 63 of the CTA's 128 rows), and
        // in pass B the two V tiles.  All copies complete on the stage's FULL
        // barrier.
        if (lane == 0) {
            const uint32_t step_bytes = KVG * L.tile + 2 * 16384u;
            const uint32_t v_bytes = (uint32_t)(KVG * p.dv * BN);
            int64_t issued = 0, gstep = 0;         // steps issued, all tiles
            int r_s = 0;                           // stage of the running step = gstep % S
            uint32_t r_p = 0;                      // (gstep / S) & 1
            bool ok = true;
            for (int k = blockIdx.x; ok && k < p.tiles; k += gridDim.x) {
                const TileCoord tc = tile_coord(p, k);
                int kvbh0, kvbh1, q0g;
                bool ex;
                group_coords(p, tc, 0, kvbh0, q0g, ex);
                group_coords(p, tc, 1, kvbh1, q0g, ex);
                for (int u = 0; u < U; ++u, ++gstep, ring_next(r_s, r_p, S)) {
                    const int s = r_s;
                    const bool pass_b = u >= T;
                    const int t = pass_b ? u - T : u;
                    const int j0 = t * BN;
                    if (gstep >= S && !mbar_wait(&bars[B_EMPTY + s], r_p ^ 1u, abort_flag)) {
                        fail(abort_flag, p.status, kStatusTimeoutProducer);
                        ok = false;
                        break;
                    }
                    uint64_t* full = &bars[B_FULL + s];
                    mbar_arrive_expect_tx(full, step_bytes + (pass_b ? v_bytes : 0u));
                    uint8_t* kdst = smem + L.k + s * L.k_bytes;
                    bulk_load(kdst, p.kst + ((size_t)kvbh0 * T + t) * L.tile, L.tile, full);
                    bulk_load(kdst + L.tile, p.kst + ((size_t)kvbh1 * T + t) * L.tile, L.tile, full);
                    for (int bx = 0; bx < 2; ++bx)
                        tma_load_3d(smem + L.b + (s * 2 + bx) * 16384, &tm_b, full, j0 + 32 * bx, q0g, tc.y);
                    if (pass_b) {
                        tma_load_3d(smem + L.v + (s * KVG) * L.v_bytes, &tm_v, full, j0, 0, kvbh0);
                        tma_load_3d(smem + L.v + (s * KVG + 1) * L.v_bytes, &tm_v, full, j0, 0, kvbh1);
                    }
                    issued = gstep + 1;
                }
            }
            // On an abort, let copies already issued land before the CTA exits.
            if (*abort_flag)
                for (int64_t w = (issued > S ? issued - S : 0); w < issued; ++w)
                    mbar_wait(&bars[B_FULL + (int)(w % S)], (uint32_t)((w / S) & 1), nullptr, 100000000ull);
        }
        __syncwarp();
    } else if (warp == MMA_WARP) {
        // ---------------------------------------------------------------- MMA issue
        // The whole warp runs this loop with uniform control flow and ring
        // state; one elected lane issues each tensor-core instruction.
        const uint32_t idesc_qk = (QK == QK_I8) ? instr_desc(kCS32, kFmtS8, kFmtS8, BM, BN)
                                                : instr_desc(kCF32, kFmtE4M3, kFmtE4M3, BM, BN);
        const uint32_t idesc_pv = instr_desc(kCS32, kFmtU8, kFmtS8, BM, p.dv);
        const uint32_t sbo_qk = (uint32_t)chunks * 128u;
        // Descriptors are built once; moving along a buffer only adds to the
        // start-address field (bytes / 16), which never carries out.
        const uint64_t dq0 = smem_desc(smem_addr(smem + L.q), 128, sbo_qk, kLayoutNone);
        const uint64_t dk0 = smem_desc(smem_addr(smem + L.k), 128, sbo_qk, kLayoutNone);
        const uint64_t dv0 = smem_desc(smem_addr(smem + L.v), 16, 512, kLayoutSw64);
        const uint32_t q_step = L.q_bytes >> 4, v_step = L.v_bytes >> 4;
        const int kq = p.dpad / 32;
        // Steps run on across tiles: the S buffer of global step w is w & 1, in
        // its use (w >> 1); ring slots and parities are running counters.
        int q_s = 0;                               // stage of the next QK
        uint32_t q_sp = 0;
        auto issue_qk = [&](int64_t w) -> bool {
            const int s = q_s, buf = (int)(w & 1);
            if (!warp_wait(&bars[B_FULL + s], q_sp, abort_flag)) return false;
            for (int g = 0; g < NG; ++g)
                if (w >= 2 && !warp_wait(&bars[B_SDONE + 2 * g + buf], (uint32_t)(((w >> 1) - 1) & 1), abort_flag))
                    return false;
            tc_fence_after();
            for (int g = 0; g < NG; ++g) {
                const uint64_t dq = dq0 + g * q_step;
                const uint64_t dk = dk0 + ((s * L.k_bytes + g * L.tile) >> 4);
                const uint32_t d_tmem = tmem + (2 * g + buf) * BN;
                for (int kk = 0; kk < kq; ++kk)
                    mma_ss_warp<QK>(d_tmem, dq + kk * 16, dk + kk * 16, idesc_qk, kk > 0 ? 1u : 0u);
                mma_commit_warp(&bars[B_SFULL + 2 * g + buf]);
            }
            ring_next(q_s, q_sp, S);
            return true;
        };
        bool ok = true;
        int p_s = 0;                               // stage of the running step
        uint32_t p_sp = 0;
        int64_t gbase = 0;                         // global index of the tile's first step
        int kt = 0;                                // tiles done by this CTA
        for (int k = blockIdx.x; ok && k < p.tiles; k += gridDim.x, ++kt, gbase += U) {
            // Q of this tile written by the softmax warps.
            if (!(ok = warp_wait(&bars[B_QREADY], (uint32_t)(kt & 1), abort_flag))) break;
            if (!(ok = issue_qk(gbase))) break;
            for (int u = 0; ok && u < U; ++u, ring_next(p_s, p_sp, S)) {
                const int64_t w = gbase + u;
                if (u + 1 < U && !(ok = issue_qk(w + 1))) break;
                if (u >= T) {
                    // PV: u8 P (in the S buffer's first BN/4 TMEM columns) x s8 V.
                    const int t = u - T, buf = (int)(w & 1), s = p_s;
                    // The first PV of a tile overwrites the output accumulators:
                    // the softmax warps must have read the previous tile's.
                    if (t == 0 && kt > 0 &&
                        !(ok = warp_wait(&bars[B_OFREE], (uint32_t)((kt - 1) & 1), abort_flag)))
                        break;
                    for (int g = 0; g < NG && ok; ++g)
                        ok = warp_wait(&bars[B_SDONE + 2 * g + buf], (uint32_t)((w >> 1) & 1), abort_flag);
                    if (!ok) break;
                    tc_fence_after();
                    for (int g = 0; g < NG; ++g) {
                        const uint64_t dv = dv0 + (s * KVG + g) * v_step;
                        const uint32_t a_tmem = tmem + (2 * g + buf) * BN;
#pragma unroll
                        for (int kk = 0; kk < BN / 32; ++kk)
                            mma_ts_i8_warp(tmem + 256 + 128 * g, a_tmem + kk * 8, dv + kk * 2, idesc_pv,
                                           (t > 0 || kk > 0) ? 1u : 0u);
                    }
                }
                mma_commit_warp(&bars[B_EMPTY + p_s]);
            }
            if (ok) mma_commit_warp(&bars[B_OREADY]);
        }
        if (!ok && lane == 0) fail(abort_flag, p.status, kStatusTimeoutMma);
        __syncwarp();
        // Let every issued MMA finish before TMEM is released.
        mma_commit_warp(&bars[B_FINAL]);
        if (!warp_wait(&bars[B_FINAL], 0, nullptr, 4000000000ull) && lane == 0) atomicOr(p.status, kStatusTimeoutMma);
        __syncwarp();
    } else {
        // ---------------------------------------------------------------- softmax + epilogue
        const int g = warp >> 2;                      // row group
        const int quarter = warp & 3;                 // TMEM lanes this warp may access
        const int r = quarter * 32 + lane;            // row within the group
        const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
        const int kvx = g;
        uint8_t* qop = smem + L.q + g * L.q_bytes;
        // Q operand of this row for tile k, padding channels zeroed.  This
        // group's QK products of the previous tile have all completed (its last
        // S tile was waited for), so the operand may be overwritten.
        auto write_q = [&](int k) {
            int bh, q0;
            bool ex;
            group_coords(p, tile_coord(p, k), g, bh, q0, ex);
            const int i = q0 + r;
            const bool rok = ex && i < N;
            const uint32_t* src = p.bq + ((size_t)bh * N + ((i < N) ? i : N - 1)) * W;
            for (int w = 0; w < W; ++w) {
                const uint32_t bits = rok ? __ldg(src + w) : 0u;
                const int nvalid = min(32, p.d - 32 * w);
                const uint32_t vm = nvalid >= 32 ? 0xFFFFFFFFu : ((1u << nvalid) - 1u);
                *reinterpret_cast<uint4*>(qop + core_off(r, 2 * w, chunks)) = expand16<QK>(bits & 0xFFFFu, vm & 0xFFFFu);
                *reinterpret_cast<uint4*>(qop + core_off(r, 2 * w + 1, chunks)) = expand16<QK>(bits >> 16, vm >> 16);
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[B_QREADY]);
        };
        bool ok = true;
        int r_s = 0;                                  // stage of the running step
        uint32_t r_sp = 0;
        int64_t gbase = 0;                            // global index of the tile's first step
        int kt = 0;
        if ((int)blockIdx.x < p.tiles) write_q(blockIdx.x);
        for (int k = blockIdx.x; ok && k < p.tiles; k += gridDim.x, ++kt, gbase += U) {
            int bh, q0;
            bool group_exists;
            group_coords(p, tile_coord(p, k), g, bh, q0, group_exists);
            const int i = q0 + r;
            const bool row_ok = group_exists && i < N;
            const int ie = (i < N) ? i : N - 1;
            const float cq = row_ok ? __ldg(p.muq + (size_t)bh * N + i) * p.q_scale : 0.f;
            const uint64_t cq2 = f2_pack(cq, cq);
            float mrow = -INFINITY;
            uint64_t l2[2] = {f2_pack(0.f, 0.f), f2_pack(0.f, 0.f)};
            uint64_t neg2 = 0;
            for (int u = 0; u < U; ++u, ring_next(r_s, r_sp, S)) {
                const int64_t w = gbase + u;
                const int s = r_s, buf = (int)(w & 1);
                const bool pass_b = u >= T;
                const int t = pass_b ? u - T : u;
                const int j0 = t * BN;
                ok = warp_wait(&bars[B_SFULL + 2 * g + buf], (uint32_t)((w >> 1) & 1), abort_flag) &&
                     warp_wait(&bars[B_FULL + s], r_sp, abort_flag);
                if (!ok) break;
                tc_fence_after();
                const bool ragged = j0 + BN > N;
                const uint8_t* tile_s = smem + L.k + s * L.k_bytes + kvx * L.tile;
                const float* muk_s = reinterpret_cast<const float*>(tile_s + BN * p.dpad);
                const uint8_t* bsm_row = smem + L.b + s * 2 * 16384 + r * 128;
                const int nvalid = N - j0;
                uint32_t zr[64];
                tmem_ld64(tmem + (2 * g + buf) * BN + lane_base, zr);
                tmem_wait_ld();
                uint32_t pw[16];
                float mx[2] = {-INFINITY, -INFINITY};
                if (!pass_b) {
                    if (ragged)
                        softmax_tile<QK, BIAS, false, true>(zr, muk_s, bsm_row, r & 7, nullptr, nullptr, nullptr, 0,
                                                            nvalid, cq2, neg2, mx, l2, pw);
                    else
                        softmax_tile<QK, BIAS, false, false>(zr, muk_s, bsm_row, r & 7, nullptr, nullptr, nullptr, 0,
                                                             nvalid, cq2, neg2, mx, l2, pw);
                    mrow = fmax3(mrow, mx[0], mx[1]);
                } else {
                    if (ragged)
                        softmax_tile<QK, BIAS, true, true>(zr, muk_s, bsm_row, r & 7, nullptr, nullptr, nullptr, 0,
                                                           nvalid, cq2, neg2, mx, l2, pw);
                    else
                        softmax_tile<QK, BIAS, true, false>(zr, muk_s, bsm_row, r & 7, nullptr, nullptr, nullptr, 0,
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
            if (!ok) break;
            // The next tile's Q goes in now, so its QK products overlap this epilogue.
            if (k + (int)gridDim.x < p.tiles) write_q(k + gridDim.x);

            // Epilogue: O = sv * acc / (255 l).
            if (!(ok = warp_wait(&bars[B_OREADY], (uint32_t)(kt & 1), abort_flag))) break;
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
                if (row_ok) store_out16<OutT>(dst + c, acc, svp + c, inv, min(16, p.d - c));
            }
            // The output accumulators may take the next tile's PV products.
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[B_OFREE]);
        }
        if (!ok && lane == 0) fail(abort_flag, p.status, kStatusTimeoutSoftmax);
    }

    tc_fence_before();
    __syncthreads();
    if (warp == MMA_WARP) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}


// ------------------------------------------------------------------ host side

size_t smem_bytes(int d, int stages)
{
    const Layout L = make_layout(32 * words_for(d), dv_of(d), stages);
    return (size_t)L.total + 1024;   // slack for the manual 1 KB alignment
}

// Deepest pipeline (2..4 stages) that fits; 0 if even 2 do not.
int pick_stages(int d)
{
    for (int s = MAX_STAGES; s >= 2; --s)
        if (smem_bytes(d, s) <= kSmemLimit) return s;
    return 0;
}

template <int QK, typename OutT>
cudaError_t launch_t(const CUtensorMap& tv, const CUtensorMap& tb, const Params& p, size_t smem, cudaStream_t st)
{
    auto kern = attn_pair_kernel<QK, OutT>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    // Persistent: one CTA per SM (each takes all TMEM columns), at most one per tile.
    const int grid = p.tiles < sms ? p.tiles : sms;
    kern<<<grid, NUM_THREADS, smem, st>>>(tv, tb, p);
    return cudaGetLastError();
}

}  // namespace
}  // namespace tc

using namespace tc;

bool pair_supports(int d) { return d >= 1 && d <= 128 && pick_stages(d) >= 2; }

// Dense bias [H, N, bias_ld] fp32; key tiles already staged (64 keys per tile).
cudaError_t launch_attn_pair(const uint32_t* bq, const float* muq, const uint8_t* kst, const int8_t* vq,
                             const float* sv, const float* bias, int64_t bias_ld, int B, int H, int N, int d,
                             void* out, ba_dtype out_dt, bool f8, unsigned* status, cudaStream_t st)
{
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
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    {
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
    p.bq = bq; p.muq = muq; p.kst = kst; p.sv = sv; p.out = out;
    p.B = B; p.H = H; p.N = N; p.d = d; p.W = words_for(d); p.dpad = 32 * p.W; p.dv = dv;
    p.n_tiles = ceil_div(N, BN);
    p.tiles_x = ceil_div(N, BM);
    p.tiles = p.tiles_x * H * ceil_div(B, 2);
    p.stages = pick_stages(d);
    p.q_scale = (float)(1.0 / sqrt((double)d));
    p.status = status;
    if (p.stages < 2) return cudaErrorNotSupported;
    // One CTA per SM: each takes all 512 TMEM columns.
    size_t smem = smem_bytes(d, p.stages);
    if (smem < 120u * 1024u) smem = 120u * 1024u;
    if (out_dt == BA_BF16)
        return f8 ? launch_t<QK_F8, __nv_bfloat16>(tv, tb, p, smem, st) : launch_t<QK_I8, __nv_bfloat16>(tv, tb, p, smem, st);
    return f8 ? launch_t<QK_F8, float>(tv, tb, p, smem, st) : launch_t<QK_I8, float>(tv, tb, p, smem, st);
}

}  // namespace ba
