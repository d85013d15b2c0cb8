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
//   * a CTA owns 128 query rows (row = TMEM lane) and walks the keys in
//     steps of 128: one QK product of N = 128 per step, the widest tile whose
//     S fits three times in TMEM next to the output accumulator.  Four softmax
//     threads share a row, each taking 32 keys of a step (16 softmax warps, so
//     four per SM sub-partition hide each other's TMEM-load and arithmetic
//     latency); they combine their row maxima once (end of pass A) and their
//     row sums once (epilogue);
//   * the keys are swept twice: pass A finds the exact row maximum m_i, pass
//     B quantises P~ = exp(S - m_i) against it.  The u8 codes are then the
//     ones an exact-maximum reference produces, and the int32 PV accumulator
//     never needs rescaling;
//   * a staging pre-pass turns the key sign bits into +-1 tensor-core
//     operands once per call (kind::i8 bytes, or e4m3 +-1 for kind::f8f6f4),
//     laid out step by step in the shared-memory order the QK product reads,
//     each 128-key tile followed by its key scales; for a 2-D relative-
//     position bias it also writes every table row reversed, in four copies
//     shifted by one entry, so any bias window a step needs is four aligned
//     copies;
//   * one loader thread moves everything with bulk copies and TMA (key tiles,
//     bias windows or dense bias boxes, V tiles) into a 2..4-stage ring: the
//     loader issues no loads or stores of its own;
//   * QK runs on tcgen05.mma into three S buffers in TMEM, issued up to two
//     steps ahead of the softmax; both kinds are exact;
//   * PV runs on tcgen05.mma kind::i8 with u8 P read straight from TMEM (each
//     softmax thread writes its codes over the S columns it has already read)
//     and s8 V tiles, accumulating in TMEM across all key tiles;
//   * the softmax pulls its 32 keys of an S tile out of TMEM with one load
//     and does its arithmetic on packed fp32 pairs (fma/mul/add .f32x2) with
//     a 3-input max; a bias window is read as reversed copies, four keys per
//     16-byte load;
//   * ring slots and mbarrier parities are counters advanced once per step
//     (no division by the runtime stage count).
// Warps 0-15 run the softmax (warp w: TMEM lanes 32 (w % 4) .., keys
// 32 (w / 4) .. of each step), warp 16 loads, warp 17 issues the MMAs and owns
// TMEM.
//
// Every wait on an mbarrier is bounded; on a timeout the kernel records a bit
// in the device status word, tells the other roles to stop, lets issued copies
// and tensor-core work drain, frees TMEM and returns.
#include "ba_attn_tc_common.cuh"
#include "ba_tc_warp.cuh"

namespace ba {

cudaError_t launch_attn_pair(const uint32_t* bq, const float* muq, const uint8_t* kst, const int8_t* vq,
                             const float* sv, const float* bias, int64_t bias_ld, int B, int H, int N, int d,
                             void* out, ba_dtype out_dt, bool f8, unsigned* status, cudaStream_t st);
bool pair_supports(int d);

namespace tc {
namespace {

constexpr int BN = 128;                 // keys per step (N of the QK product)
constexpr int KQ = 4;                   // softmax threads per row (key quarters of a step)
constexpr int KT = BN / KQ;             // keys per softmax thread per step (32)
constexpr int NSB = 3;                  // S buffers in TMEM
constexpr uint32_t O_COL = NSB * BN;    // TMEM column of the output accumulator
constexpr int MAX_STAGES = 4;
constexpr int NUM_SOFTMAX_WARPS = 4 * KQ;                   // 16
constexpr int LOAD_WARP = NUM_SOFTMAX_WARPS;                // 16
constexpr int MMA_WARP = LOAD_WARP + 1;                     // 17
constexpr int NUM_THREADS = 32 * (MMA_WARP + 1);            // 576
// 576 threads share the 64K-entry register file: at most 113 registers each
// (the launch bound below lets the compiler know).
constexpr int RP_WIN = 256;             // entries per shifted copy of a window (255 used)
constexpr int RP_STRIDE = 264;          // floats between copies in shared memory (8 words mod 32)
constexpr uint32_t RP_COPY_BYTES = RP_WIN * 4;

// Barrier slots.
enum {
    B_QREADY = 0,
    B_FULL = 1,                      // [stage] key tiles, bias (and V in pass B) landed
    B_EMPTY = B_FULL + MAX_STAGES,   // [stage] stage may be overwritten
    B_SFULL = B_EMPTY + MAX_STAGES,  // [NSB] S tile in TMEM ready
    B_SDONE = B_SFULL + NSB,         // [NSB] softmax done with the S buffer (pass B: u8 P written into it)
    B_XMAX = B_SDONE + NSB,          // both halves posted their partial row maxima
    B_XSUM = B_XMAX + 1,             // both halves posted their partial row sums
    B_OREADY = B_XSUM + 1,           // every PV finished
    B_FINAL = B_OREADY + 1,
    NUM_BARS
};

struct Layout {
    uint32_t stages, tile;      // pipeline depth; staged tile bytes
    uint32_t v, v_bytes;        // [stage][2] V boxes of 64 keys (SW64 K-major, dv rows x 64 bytes)
    uint32_t b;                 // [stage][4] dense bias boxes of 32 keys, 16 KB each (SW128)
    uint32_t q, q_bytes;        // Q operand
    uint32_t k, k_bytes;        // [stage] staged key tile
    uint32_t rp;                // [stage][4][RP_STRIDE] rel-pos window copies
    uint32_t xmax, xsum;        // [KQ][BM] partial row maxima / sums
    uint32_t bars, misc, total;
};

__host__ __device__ inline Layout make_layout(int dpad, int dv, int bias_kind, int stages)
{
    Layout L;
    L.stages = stages;
    L.tile = tile_bytes(BN, dpad, bias_kind == BIAS_RP_FAST ? BA_BIAS_NONE : bias_kind);
    uint32_t off = 0;
    L.v_bytes = align_up((uint32_t)dv * 64, 1024);
    L.v = off; off += stages * 2 * L.v_bytes;
    L.b = off; off += (bias_kind == BA_BIAS_DENSE) ? stages * 4 * 16384u : 0u;
    L.q_bytes = align_up((uint32_t)BM * dpad, 1024);
    L.q = off; off += L.q_bytes;
    L.k_bytes = align_up(L.tile, 128);
    L.k = off; off += stages * L.k_bytes;
    L.rp = off; off += (bias_kind == BIAS_RP_FAST) ? stages * 4 * RP_STRIDE * 4u : 0u;
    L.xmax = off; off += KQ * BM * 4;
    L.xsum = off; off += KQ * BM * 4;
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
    uint64_t wait_ns;        // give-up time of every barrier wait (2 s in production)
    int starve_step;         // testing only: the loader stops before this step (-1: never)
};

template <int QK, typename OutT, int BIAS>
__global__ void __launch_bounds__(NUM_THREADS, 1)
attn_tc_kernel(const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_b,
               const Params p)
{
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
    const int bh = blockIdx.y;                             // batch * head
    const int h = bh % p.H;
    const int q0 = blockIdx.x * BM;                        // first query row of the CTA
    // General rel-pos: the head's table (with a class token, the grid entries
    // are followed by the three class entries, cls3).
    const size_t rp_grid = (size_t)(2 * p.gh - 1) * (2 * p.gw - 1);
    const float* tab_h = (BIAS == BA_BIAS_RELPOS2D) ? p.table + h * rp_grid
                       : (BIAS == BIAS_RP_CLS)      ? p.table + h * (rp_grid + 3) : nullptr;
    const float* cls3 = (BIAS == BIAS_RP_CLS) ? tab_h + rp_grid : nullptr;

    if (threadIdx.x == 0) {
        mbar_init(&bars[B_QREADY], NUM_SOFTMAX_WARPS);
        for (int s = 0; s < S; ++s) {
            mbar_init(&bars[B_FULL + s], 1);
            mbar_init(&bars[B_EMPTY + s], NUM_SOFTMAX_WARPS + 1);
        }
        for (int b = 0; b < NSB; ++b) {
            mbar_init(&bars[B_SFULL + b], 1);
            mbar_init(&bars[B_SDONE + b], NUM_SOFTMAX_WARPS);
        }
        mbar_init(&bars[B_XMAX], NUM_SOFTMAX_WARPS);
        mbar_init(&bars[B_XSUM], NUM_SOFTMAX_WARPS);
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
        // The warp fills stage u % S for step u (uniform loop, one elected
        // lane issuing the copies in order, key tile first): the staged key
        // tile, the bias of the step (the window of a reversed table row in
        // four shifted copies, or four dense-bias boxes), and in pass B two V
        // boxes.  All copies complete on the stage's FULL barrier.
        {
            const size_t row_len = 2 * (size_t)p.gw;
            const float* rps_h = (BIAS == BIAS_RP_FAST) ? p.rps + (size_t)h * (2 * p.gh - 1) * 4 * row_len : nullptr;
            const int ri = (BIAS == BIAS_RP_FAST) ? q0 / p.gw : 0;
            const int ci0 = (BIAS == BIAS_RP_FAST) ? q0 - ri * p.gw : 0;
            const uint32_t step_bytes = L.tile + (BIAS == BIAS_RP_FAST ? 4 * RP_COPY_BYTES : 0u) +
                                        (BIAS == BA_BIAS_DENSE ? 4 * 16384u : 0u);
            const uint32_t v_bytes = (uint32_t)(2 * p.dv * 64);
            int issued = 0;
            int r_s = 0;                           // stage of step u = u % S
            uint32_t r_p = 0;                      // (u / S) & 1
            for (int u = 0; u < U; ++u, ring_next(r_s, r_p, S)) {
                const int s = r_s;
                const bool pass_b = u >= T;
                const int t = pass_b ? u - T : u;
                const int j0 = t * BN;
                // Testing only: issue nothing from this step on, so the roles
                // that wait for it give up (no copy is left in flight: the MMA
                // warp has waited for every earlier stage before it reaches
                // this one).
                if (u == p.starve_step) break;
                if (u >= S && !warp_wait(&bars[B_EMPTY + s], r_p ^ 1u, abort_flag, p.wait_ns)) {
                    if (lane == 0) fail(abort_flag, p.status, kStatusTimeoutProducer);
                    break;
                }
                uint64_t* full = &bars[B_FULL + s];
                if (elect_one()) {
                    mbar_arrive_expect_tx(full, step_bytes + (pass_b ? v_bytes : 0u));
                    bulk_load(smem + L.k + s * L.k_bytes, p.kst + ((size_t)bh * T + t) * L.tile, L.tile, full);
                    if (BIAS == BIAS_RP_FAST) {
                        // Entries xs .. xs + 255 of the reversed row for ri - rj,
                        // xs = gw - 128 - (ci0 - cj0), from each shifted copy.
                        const int rj = j0 / p.gw, cj0 = j0 - rj * p.gw;
                        const int rho = ri - rj + p.gh - 1;
                        const int xs = p.gw - BM - (ci0 - cj0);
                        const float* srcw = rps_h + (size_t)rho * 4 * row_len + xs;
                        float* dst = reinterpret_cast<float*>(smem + L.rp) + (size_t)s * 4 * RP_STRIDE;
#pragma unroll
                        for (int m = 0; m < 4; ++m)
                            bulk_load(dst + m * RP_STRIDE, srcw + m * row_len, RP_COPY_BYTES, full);
                    }
                    if (BIAS == BA_BIAS_DENSE)
                        for (int bx = 0; bx < 4; ++bx)
                            tma_load_3d(smem + L.b + (s * 4 + bx) * 16384, &tm_b, full, j0 + 32 * bx, q0, h);
                    if (pass_b)
                        for (int vb = 0; vb < 2; ++vb)
                            tma_load_3d(smem + L.v + (s * 2 + vb) * L.v_bytes, &tm_v, full, j0 + 64 * vb, 0, bh);
                }
                __syncwarp();
                issued = u + 1;
            }
            // On an abort, let copies already issued land before the CTA exits.
            if (__any_sync(0xffffffffu, *abort_flag != 0))
                for (int u = (issued > S ? issued - S : 0); u < issued; ++u)
                    warp_wait(&bars[B_FULL + u % S], (u / S) & 1, nullptr, 100000000ull);
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
        bool ok = warp_wait(&bars[B_QREADY], 0, abort_flag, p.wait_ns);
        // Descriptors are built once; moving along a buffer only adds to the
        // start-address field (bytes / 16), which never carries out.
        const uint64_t dq0 = smem_desc(smem_addr(smem + L.q), 128, sbo_qk, kLayoutNone);
        const uint64_t dk0 = smem_desc(smem_addr(smem + L.k), 128, sbo_qk, kLayoutNone);
        const uint64_t dv0 = smem_desc(smem_addr(smem + L.v), 16, 512, kLayoutSw64);
        const uint32_t k_step = L.k_bytes >> 4, v_step = L.v_bytes >> 4;
        const int kq = p.dpad / 32;
        // QK of step u into S buffer u % NSB, once the softmax is done with
        // the step that used it last (its PV, issued earlier, reads P before
        // this product overwrites it: one thread's tcgen05 ops run in order).
        // Stage and S buffer of the next QK (issued for steps in order):
        // slot = step % ring size, parity = (step / ring size) & 1.
        int q_s = 0, q_b = 0;
        uint32_t q_sp = 0, q_bp = 0;
        auto issue_qk = [&](int u) -> bool {
            const int s = q_s, b = q_b;
            if (!warp_wait(&bars[B_FULL + s], q_sp, abort_flag, p.wait_ns)) return false;
            if (u >= NSB && !warp_wait(&bars[B_SDONE + b], q_bp ^ 1u, abort_flag, p.wait_ns)) return false;
            tc_fence_after();
            const uint64_t dk = dk0 + s * k_step;
            const uint32_t d_tmem = tmem + b * BN;
            for (int kk = 0; kk < kq; ++kk)
                mma_ss_warp<QK>(d_tmem, dq0 + kk * 16, dk + kk * 16, idesc_qk, kk > 0 ? 1u : 0u);
            mma_commit_warp(&bars[B_SFULL + b]);
            ring_next(q_s, q_sp, S);
            ring_next(q_b, q_bp, NSB);
            return true;
        };
        // QK runs LA steps ahead: two when four stages hold the key tiles of
        // the steps in flight, else one.
        const int LA = (S >= 4) ? 2 : 1;
        for (int u = 0; ok && u < LA && u < U; ++u) ok = issue_qk(u);
        int p_s = 0, p_b = 0;                      // stage and S buffer of step u
        uint32_t p_sp = 0, p_bp = 0;
        for (int u = 0; ok && u < U; ++u, ring_next(p_s, p_sp, S), ring_next(p_b, p_bp, NSB)) {
            if (u + LA < U && !(ok = issue_qk(u + LA))) break;
            if (u >= T) {
                // PV: u8 P x s8 V, K = 32 keys per product.  The P codes of
                // keys 32 kq .. 32 kq + 31 sit in columns 32 kq .. 32 kq + 7 of
                // the S buffer.
                const int t = u - T, b = p_b, s = p_s;
                if (!(ok = warp_wait(&bars[B_SDONE + b], p_bp, abort_flag, p.wait_ns))) break;
                tc_fence_after();
                const uint32_t a_tmem = tmem + b * BN;
#pragma unroll
                for (int kk = 0; kk < BN / 32; ++kk)
                    mma_ts_i8_warp(tmem + O_COL, a_tmem + kk * KT,
                                   dv0 + (s * 2 + (kk >> 1)) * v_step + (kk & 1) * 2,
                                   idesc_pv, (t > 0 || kk > 0) ? 1u : 0u);
            }
            mma_commit_warp(&bars[B_EMPTY + p_s]);
        }
        if (ok) mma_commit_warp(&bars[B_OREADY]);
        if (!ok && lane == 0) fail(abort_flag, p.status, kStatusTimeoutMma);
        __syncwarp();
        // Let every issued MMA finish before TMEM is released.
        mma_commit_warp(&bars[B_FINAL]);
        if (!warp_wait(&bars[B_FINAL], 0, nullptr, 4000000000ull) && lane == 0) atomicOr(p.status, kStatusTimeoutMma);
        __syncwarp();
    } else {
        // ---------------------------------------------------------------- softmax + epilogue
        const int quarter = warp & 3;                 // TMEM lanes this warp may access
        const int kq = warp >> 2;                     // which 32 keys of each step
        const int r = quarter * 32 + lane;            // row within the CTA
        const int i = q0 + r;
        const bool row_ok = i < N;
        const int ie = row_ok ? i : N - 1;
        const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;

        // Q operand of this row, padding channels zeroed (the row's threads split the words).
        {
            uint8_t* qop = smem + L.q;
            const uint32_t* src = p.bq + ((size_t)bh * N + ie) * W;
            for (int w = kq; w < W; w += KQ) {
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
        bool cls_row = false;
        if (is_relpos(BIAS)) {
            if (BIAS == BIAS_RP_FAST) {
                // Row r reads window entries 127 - r + k; copy m = (127 - r) % 4
                // starts that run on a 16-byte boundary.
                const int sidx = (BM - 1) - r;
                const int m = sidx & 3;
                rp_off = m * RP_STRIDE + (sidx - m) + kq * KT;
            } else {
                // Patch index of the row; the class row (token 0 with a class
                // token) gathers from the table centre, always in range, and
                // takes the class entries instead.
                cls_row = BIAS == BIAS_RP_CLS && ie == 0;
                const int pe = (BIAS == BIAS_RP_CLS) ? (cls_row ? 0 : ie - 1) : ie;
                const int ri = pe / p.gw, ci = pe - ri * p.gw;
                rel_base = (ri + p.gh - 1) * (2 * p.gw - 1) + ci + p.gw - 1;
            }
        }

        float mrow = -INFINITY;
        uint64_t l2[2] = {f2_pack(0.f, 0.f), f2_pack(0.f, 0.f)};
        uint64_t neg2 = 0;
        bool ok = true;
        int r_s = 0, r_b = 0;                         // stage and S buffer of step u
        uint32_t r_sp = 0, r_bp = 0;
        for (int u = 0; u < U; ++u, ring_next(r_s, r_sp, S), ring_next(r_b, r_bp, NSB)) {
            const int s = r_s, b = r_b;
            const bool pass_b = u >= T;
            const int t = pass_b ? u - T : u;
            const int jh = t * BN + kq * KT;          // first key of this thread's quarter
            ok = warp_wait(&bars[B_SFULL + b], r_bp, abort_flag, p.wait_ns) &&
                 warp_wait(&bars[B_FULL + s], r_sp, abort_flag, p.wait_ns);
            if (!ok) break;
            tc_fence_after();
            const bool ragged = jh + KT > N;
            const uint8_t* tile_s = smem + L.k + s * L.k_bytes;
            const float* muk_s = reinterpret_cast<const float*>(tile_s + BN * p.dpad) + kq * KT;
            const int* koff_s = reinterpret_cast<const int*>(tile_s + BN * p.dpad + BN * 4) + kq * KT;
            const uint8_t* bsm_row = smem + L.b + (s * 4 + kq) * 16384 + r * 128;
            const float* rpc = (BIAS == BIAS_RP_FAST)
                ? reinterpret_cast<const float*>(smem + L.rp) + (size_t)s * 4 * RP_STRIDE + rp_off : nullptr;
            const int nvalid = N - jh;
            const uint32_t s_col = tmem + b * BN;
            uint32_t zr[KT];
            tmem_ld32(s_col + kq * KT + lane_base, zr);
            tmem_wait_ld();
            uint32_t pw[KT / 4];
            float mx[2] = {-INFINITY, -INFINITY};
            if (!pass_b) {
                if (ragged)
                    softmax_tile<QK, BIAS, false, true, KT>(zr, muk_s, bsm_row, r & 7, rpc, koff_s, tab_h, rel_base,
                                                        nvalid, cq2, neg2, mx, l2, pw, cls3, cls_row);
                else
                    softmax_tile<QK, BIAS, false, false, KT>(zr, muk_s, bsm_row, r & 7, rpc, koff_s, tab_h, rel_base,
                                                         nvalid, cq2, neg2, mx, l2, pw, cls3, cls_row);
                mrow = fmax3(mrow, mx[0], mx[1]);
            } else {
                if (ragged)
                    softmax_tile<QK, BIAS, true, true, KT>(zr, muk_s, bsm_row, r & 7, rpc, koff_s, tab_h, rel_base,
                                                       nvalid, cq2, neg2, mx, l2, pw, cls3, cls_row);
                else
                    softmax_tile<QK, BIAS, true, false, KT>(zr, muk_s, bsm_row, r & 7, rpc, koff_s, tab_h, rel_base,
                                                        nvalid, cq2, neg2, mx, l2, pw, cls3, cls_row);
                // The u8 codes of these 32 keys go back into this row's lane of
                // the S buffer, over the first 8 columns of this thread's own
                // quarter (already read; the other quarters' S columns are
                // never written here): the PV product reads them from TMEM.
                tmem_st8(s_col + kq * KT + lane_base, pw);
                tmem_wait_st();
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&bars[B_SDONE + b]);
                mbar_arrive(&bars[B_EMPTY + s]);
            }
            if (u == T - 1) {
                // Row maximum = the largest of the quarters' maxima.
                float* xm = reinterpret_cast<float*>(smem + L.xmax);
                xm[kq * BM + r] = mrow;
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars[B_XMAX]);
                if (!warp_wait(&bars[B_XMAX], 0, abort_flag, p.wait_ns)) { ok = false; break; }
                mrow = fmaxf(fmax3(xm[r], xm[BM + r], xm[2 * BM + r]), xm[3 * BM + r]);
                neg2 = f2_pack(-mrow * LOG2E, -mrow * LOG2E);
            }
        }

        // Epilogue: O = sv * acc / (255 l), l = the quarters' sums in a fixed order.
        if (ok) ok = warp_wait(&bars[B_OREADY], 0, abort_flag, p.wait_ns);
        if (ok) {
            float la, lb, lc, ld;
            f2_unpack(l2[0], la, lb);
            f2_unpack(l2[1], lc, ld);
            float* xs = reinterpret_cast<float*>(smem + L.xsum);
            xs[kq * BM + r] = (la + lb) + (lc + ld);
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[B_XSUM]);
            ok = warp_wait(&bars[B_XSUM], 0, abort_flag, p.wait_ns);
        }
        if (!ok) {
            if (lane == 0) fail(abort_flag, p.status, kStatusTimeoutSoftmax);
        } else {
            tc_fence_after();
            const float* xs = reinterpret_cast<const float*>(smem + L.xsum);
            const float inv = 1.f / (255.f * ((xs[r] + xs[BM + r]) + (xs[2 * BM + r] + xs[3 * BM + r])));
            OutT* dst = static_cast<OutT*>(p.out) + ((size_t)bh * N + ie) * p.d;
            const float* svp = p.sv + (size_t)bh * p.d;
            for (int c = kq * 16; c < p.dv; c += 16 * KQ) {
                uint32_t acc[16];
                tmem_ld16(tmem + O_COL + c + lane_base, acc);
                tmem_wait_ld();
                if (row_ok) store_out16<OutT>(dst + c, acc, svp + c, inv, min(16, p.d - c));
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
    dim3 grid(ceil_div(p.N, BM), p.B * p.H, 1);
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
    if (kind == BIAS_RP_CLS) return launch_t<QK, OutT, BIAS_RP_CLS>(tv, tb, p, smem, st);
    return launch_t<QK, OutT, BA_BIAS_NONE>(tv, tb, p, smem, st);
}

// The kernel variant for an ABI bias kind.
int kernel_bias(int bias_kind, int gw)
{
    if (bias_kind == BA_BIAS_RELPOS2D_CLS) return BIAS_RP_CLS;
    return (bias_kind == BA_BIAS_RELPOS2D && gw % BM == 0) ? BIAS_RP_FAST : bias_kind;
}

// A dense bias shared over the batch goes to the paired kernel (two batch
// elements per CTA share each bias tile) when there are two to pair.
bool use_pair(int bias_kind, int B) { return bias_kind == BA_BIAS_DENSE && B >= 2; }

// Workspace layout: staged key tiles (64 keys each for the paired kernel, 128
// for this one), then (fast rel-pos path) staged table rows.
struct Workspace {
    int keys;
    int64_t tile, kst_bytes, rps_off, rps_bytes, total;
};

Workspace workspace_layout(int B, int H, int N, int d, int bias_kind, int gh, int gw)
{
    const int vb = kernel_bias(bias_kind, gw);
    Workspace w;
    w.keys = use_pair(bias_kind, B) ? 64 : BN;
    w.tile = tile_bytes(w.keys, 32 * words_for(d), vb == BIAS_RP_FAST ? BA_BIAS_NONE : vb);
    w.kst_bytes = (int64_t)B * H * ceil_div(N, w.keys) * w.tile;
    w.rps_off = round_up64(w.kst_bytes, 256);
    w.rps_bytes = (vb == BIAS_RP_FAST) ? (int64_t)H * (2 * gh - 1) * 4 * (2 * (int64_t)gw) * 4 : 0;
    w.total = w.rps_off + w.rps_bytes;
    return w;
}

// Staging of the key side, one CTA per (KEYS-key tile, batch*head): +-1 operand
// bytes in core-matrix order, the key scales (0 past N), and for the general
// rel-pos bias the key offsets rj (2 gw - 1) + cj of each key's patch (with
// koff_cls = 1, token 0 is a class token: offset -1, and token j >= 1 is
// patch j - 1).  Keys past N get operand rows of their (zero) sign bits; the
// kernel masks them out of the softmax.
template <int QK, int KEYS>
__global__ void __launch_bounds__(128)
stage_k_kernel(const uint32_t* __restrict__ bk, const float* __restrict__ muk, int N, int W, int T,
               int koff_gw, int koff_cls, uint32_t tile, uint8_t* __restrict__ kst)
{
    const int t = blockIdx.x;
    const size_t bh = blockIdx.y;
    uint8_t* dst = kst + (bh * T + t) * tile;
    const int dpad = 32 * W, chunks = 2 * W;
    for (int e = threadIdx.x; e < KEYS * W; e += blockDim.x) {
        const int r = e / W, w = e - r * W;
        const int j = t * KEYS + r;
        const uint32_t bits = (j < N) ? __ldg(bk + (bh * N + j) * W + w) : 0u;
        *reinterpret_cast<uint4*>(dst + core_off(r, 2 * w, chunks)) = expand16<QK>(bits & 0xFFFFu, 0xFFFFu);
        *reinterpret_cast<uint4*>(dst + core_off(r, 2 * w + 1, chunks)) = expand16<QK>(bits >> 16, 0xFFFFu);
    }
    float* mu = reinterpret_cast<float*>(dst + KEYS * dpad);
    int* ko = reinterpret_cast<int*>(dst + KEYS * dpad + KEYS * 4);
    for (int r = threadIdx.x; r < KEYS; r += blockDim.x) {
        const int j = t * KEYS + r;
        mu[r] = (j < N) ? __ldg(muk + bh * N + j) : 0.f;
        if (koff_gw > 0) {
            const int jj = ((j < N) ? j : N - 1) - koff_cls;
            const int rj = jj / koff_gw;
            ko[r] = jj < 0 ? -1 : rj * (2 * koff_gw - 1) + (jj - rj * koff_gw);
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
}  // namespace tc

using namespace tc;

bool attn_tc_supports(int bias_kind, int gh, int gw, int N, int d)
{
    (void)gh; (void)N;
    if (d < 1 || d > 128) return false;
    return pick_stages(d, kernel_bias(bias_kind, gw)) >= 2 && pair_supports(d);
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
                           void* out, ba_dtype out_dt, int variant, unsigned* status, cudaStream_t st,
                           int starve_step, uint64_t wait_ns)
{
    if (!attn_tc_supports(bias_kind, gh, gw, N, d)) return cudaErrorNotSupported;
    // the starved-loader test mode exists for the 128-key kernel only
    if (starve_step >= 0 && use_pair(bias_kind, B)) return cudaErrorNotSupported;
    const Workspace ws = workspace_layout(B, H, N, d, bias_kind, gh, gw);
    if (workspace == nullptr || workspace_bytes < ws.total) return cudaErrorInvalidValue;
    auto encode = encode_fn();
    if (!encode) return cudaErrorNotSupported;
    const int BH = B * H;
    const int dv = dv_of(d);
    const int64_t ldv = round_up64(N, 16);
    const int vb = kernel_bias(bias_kind, gw);
    // BA_QK_AUTO takes the faster kind per kernel, as measured on B200:
    // kind::f8f6f4 (fp32 scores straight from TMEM, no integer conversion in
    // the softmax) for the 128-key kernel, kind::i8 for the paired one.
    const bool f8 = variant == BA_QK_TC_F8 || (variant == BA_QK_AUTO && !use_pair(bias_kind, B));

    CUtensorMap tv, tb;
    memset(&tv, 0, sizeof(tv));
    memset(&tb, 0, sizeof(tb));
    {
        cuuint64_t dims[3] = {(cuuint64_t)ldv, (cuuint64_t)d, (cuuint64_t)BH};
        cuuint64_t strides[2] = {(cuuint64_t)ldv, (cuuint64_t)ldv * d};
        cuuint32_t box[3] = {64, (cuuint32_t)dv, 1};
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
    p.table = (bias_kind == BA_BIAS_RELPOS2D || bias_kind == BA_BIAS_RELPOS2D_CLS) ? bias : nullptr;
    p.out = out;
    p.B = B; p.H = H; p.N = N; p.d = d; p.W = words_for(d); p.dpad = 32 * p.W; p.dv = dv;
    p.n_tiles = ceil_div(N, BN);
    p.stages = pick_stages(d, vb);
    p.gh = gh; p.gw = gw;
    p.q_scale = (float)(1.0 / sqrt((double)d));
    p.status = status;
    p.wait_ns = wait_ns;
    p.starve_step = starve_step;

    // Staging pre-passes (same stream, so the attention kernel sees them).
    {
        const uint32_t tile = (uint32_t)ws.tile;
        uint8_t* kst = static_cast<uint8_t*>(workspace);
        const int koff_gw = has_koff(vb) ? gw : 0;
        const int koff_cls = vb == BIAS_RP_CLS ? 1 : 0;
        const int tiles = ceil_div(N, ws.keys);
        dim3 grid(tiles, BH);
        if (ws.keys == 64) {
            if (f8) stage_k_kernel<QK_F8, 64><<<grid, 128, 0, st>>>(bk, muk, N, p.W, tiles, koff_gw, koff_cls, tile, kst);
            else stage_k_kernel<QK_I8, 64><<<grid, 128, 0, st>>>(bk, muk, N, p.W, tiles, koff_gw, koff_cls, tile, kst);
        } else {
            if (f8) stage_k_kernel<QK_F8, BN><<<grid, 128, 0, st>>>(bk, muk, N, p.W, tiles, koff_gw, koff_cls, tile, kst);
            else stage_k_kernel<QK_I8, BN><<<grid, 128, 0, st>>>(bk, muk, N, p.W, tiles, koff_gw, koff_cls, tile, kst);
        }
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

    if (use_pair(bias_kind, B))
        return launch_attn_pair(bq, muq, static_cast<const uint8_t*>(workspace), vq, sv, bias, bias_ld, B, H, N, d,
                                out, out_dt, f8, status, st);

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
