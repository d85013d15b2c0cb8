// ba_prepass_tma.cu -- the pre-pass for 128-, 144- and 256-byte tokens (bf16
// d = 64, 72 and 128, fp32 d = 32, 36 and 64), fed by tensor-memory-accelerator
// copies.
//
// Method source: the paper-notes page "BinaryAttention: One-Bit QK-Attention
// for Vision and Diffusion Transformers" (CVPR 2026), Key design 1 (sign bits
// and the per-token mean-|x| scale of Q and K) and Key design 3 (channel-wise
// symmetric int8 V).  Both are HBM-bound streaming steps: what decides their
// speed is how many bytes are in flight while the arithmetic runs, so the
// work is cut into small units and several CTAs share an SM.
//
// Rows reach shared memory as 128-row boxes of one 3-D tensor map per tensor
// ([BH][N][token bytes]; 128-byte rows with the 128-byte swizzle, the 16-byte
// chunk j of row r at position j ^ (r & 7); 144-byte rows as they are, nine
// chunks a row; either way every access pattern below is free of bank
// conflicts; rows past the end of the head are zero-filled).  A CTA has
// three box slots.  Work units, V first so the longest ones start in the first wave:
//
//   V, whole head (N <= 768): the head's boxes stream through the slots twice:
//   sweep 1 takes the channel absmax, sweep 2 (the same boxes again, now from
//   L2) writes the codes with the scales of sweep 1.
//   V, codes of 384 rows (longer heads): the channel absmax comes from an
//   earlier launch (vabsmax_kernel, as the bits of the non-negative floats in
//   sv); only the codes are written here.
//   Q or K, 384 tokens: all three boxes issued at the start; a thread per token,
//   packed by pack_vectors (the routine of every packing path of these
//   sizes), so the bits and mu equal those of the other paths, bit for bit.
//
// Codes: a warp takes the channels of one chunk, lane l the four keys
// 4l .. 4l + 3 of a box, visited in a lane-dependent rotation (no bank
// conflicts); each channel's four codes (vcode4, the rounding of every path)
// are put back in key order by one byte permutation and go out as one word,
// 128 contiguous bytes per warp store.
#include <algorithm>
#include <cudaTypedefs.h>

#include "ba_prepass.cuh"
#include "ba_attn_tc_common.cuh"

namespace ba {
namespace {

using namespace sm100;

constexpr int kThreads = 256;
constexpr int kBoxRows = 128;                 // rows per tensor copy (one box)
constexpr int kSlots = 3;                     // box slots of a CTA (copies in flight)
constexpr int kUnitRows = kSlots * kBoxRows;  // rows of a Q, K or V-codes unit
constexpr int kVWholeMaxLd = 1024;            // V of a head in one unit up to this code-row length
constexpr uint64_t kCopyWaitNs = 2000000000ull;

enum : int { kVNone = 0, kVWhole = 1, kVCodes = 2 };

struct PrepassMaps {
    CUtensorMap q, k, v;                      // [BH][N][NV 16 bytes], box (NV 16 bytes, 128 rows, 1)
};

// Tokens of NV 16-byte chunks: 8 (128-byte rows, copied with the 128-byte
// swizzle: chunk j of row r at position j ^ (r & 7)), 9 (144-byte rows,
// copied as they are: an odd number of chunks per row already spreads
// consecutive rows over the bank groups) or 16 (each token two 128-byte rows
// 2r and 2r + 1 of a 4-D copy, swizzled as the 128-byte rows are).
template <int NV> __host__ __device__ constexpr int box_bytes() { return kBoxRows * NV * 16; }
template <int NV> __host__ __device__ constexpr int buf_align() { return NV == 9 ? 128 : 1024; }

template <int NV>
__device__ __forceinline__ uint4 ld_chunk(const uint8_t* box, int r, int j)
{
    if constexpr (NV == 8) {
        return *reinterpret_cast<const uint4*>(box + r * 128 + ((j ^ (r & 7)) << 4));
    } else if constexpr (NV == 16) {
        const int row = 2 * r + (j >> 3);
        return *reinterpret_cast<const uint4*>(box + row * 128 + (((j & 7) ^ (row & 7)) << 4));
    } else {
        return *reinterpret_cast<const uint4*>(box + (r * NV + j) * 16);
    }
}

// A 4-D tensor copy (the 256-byte tokens' map: 128-byte half, half, row, head).
__device__ __forceinline__ void tma_load_4d(void* dst, const CUtensorMap* map, uint64_t* bar, int x, int y, int z,
                                            int w)
{
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5, %6}], [%2];"
        ::"r"(smem_addr(dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_addr(bar)),
          "r"(x), "r"(y), "r"(z), "r"(w)
        : "memory");
}

// The codes of rows 4 lane .. 4 lane + 3 of one box for the E channels of
// chunk cw, written to vq rows (channel) at key offset key0 + 4 lane.
template <typename T, int NV>
__device__ __forceinline__ void codes_of_box(const uint8_t* box, int cw, int lane, const float (&sc)[16 / sizeof(T)],
                                             const float (&rs)[16 / sizeof(T)], int8_t* vq_c0, int64_t ldv,
                                             int key0)
{
    constexpr int E = 16 / sizeof(T);
    const int base = 4 * lane;
    if (key0 + base >= ldv) return;           // ldv % 16 == 0: a group is all in or all out
    const int rot = (lane >> 1) & 3;
    const uint32_t sel = rot == 0 ? 0x3210u : rot == 1 ? 0x2103u : rot == 2 ? 0x1032u : 0x0321u;
    uint4 raw[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) raw[i] = ld_chunk<NV>(box, base + ((i + rot) & 3), cw);
#pragma unroll
    for (int e = 0; e < E; ++e) {
        const uint32_t word = vcode4(vec_elem<T>(raw[0], e), vec_elem<T>(raw[1], e), vec_elem<T>(raw[2], e),
                                     vec_elem<T>(raw[3], e), sc[e], rs[e]);
        *reinterpret_cast<uint32_t*>(vq_c0 + (size_t)e * ldv + key0 + base) = __byte_perm(word, 0u, sel);
    }
}

// Channel absmax of chunk cv over the rows rr, rr + R, ... (< nrows) of one
// box into m (bf16 pairs for bf16 input, as in vblock_quant, so the maxima
// are the same).
template <typename T, int NV>
__device__ __forceinline__ void absmax_of_box(const uint8_t* box, int cv, int rr, int R, int nrows,
                                              uint32_t (&m)[4])
{
    const int n = min(nrows, kBoxRows);
    for (int r = rr; r < n; r += R) {
        const uint4 raw = ld_chunk<NV>(box, r, cv);
        if constexpr (sizeof(T) == 2) {
            const uint32_t* h = &raw.x;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const __nv_bfloat162 a = __habs2(*reinterpret_cast<const __nv_bfloat162*>(&h[q]));
                __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162*>(&m[q]);
                b = __hmax2(b, a);
                m[q] = *reinterpret_cast<const uint32_t*>(&b);
            }
        } else {
#pragma unroll
            for (int q = 0; q < 4; ++q)
                m[q] = __float_as_uint(fmaxf(__uint_as_float(m[q]), fabsf(vec_elem<T>(raw, q))));
        }
    }
}

template <typename T, int NV>
__global__ void __launch_bounds__(kThreads, 4)
prepass_tma_kernel(const __grid_constant__ PrepassMaps maps, int N, int d, int64_t ldv, int nq, int vmode,
                   uint32_t* __restrict__ bq, float* __restrict__ muq, uint32_t* __restrict__ bk,
                   float* __restrict__ muk, int8_t* __restrict__ vq, float* __restrict__ sv,
                   unsigned* __restrict__ status)
{
    constexpr int E = 16 / sizeof(T);         // channels per 16-byte chunk; NV chunks per token
    constexpr int BB = box_bytes<NV>();
    constexpr int RG = kThreads / NV;         // row groups of the absmax sweep (thread = (chunk, row group))
    extern __shared__ uint8_t smem_raw[];
    __shared__ __align__(8) uint64_t full[kSlots];
    __shared__ unsigned amax[NV * E];
    __shared__ float s_scale[NV * E], s_rscale[NV * E];
    __shared__ int s_fail;
    uint8_t* buf = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + buf_align<NV>() - 1) &
                                              ~uintptr_t(buf_align<NV>() - 1));
    const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
    const int nbv = (int)((ldv + kBoxRows - 1) / kBoxRows);     // boxes of a head's V rows
    const int v_units = vmode == kVWhole ? 1 : vmode == kVCodes ? (int)((ldv + kUnitRows - 1) / kUnitRows) : 0;
    const int64_t BH = gridDim.x / (v_units + 2 * nq);
    int64_t bh;
    int kind, chunk;                          // kind 0: Q, 1: K, 2: V
    if ((int64_t)blockIdx.x < BH * v_units) {
        bh = blockIdx.x / v_units;
        kind = 2;
        chunk = blockIdx.x - (int)bh * v_units;
    } else {
        const int64_t u = blockIdx.x - BH * v_units;
        bh = u / (2 * nq);
        const int k = (int)(u - bh * 2 * nq);
        kind = k < nq ? 0 : 1;
        chunk = k < nq ? k : k - nq;
    }
    const CUtensorMap* map = kind == 0 ? &maps.q : kind == 1 ? &maps.k : &maps.v;
    const bool streamed = kind == 2 && vmode == kVWhole;
    const int row0 = streamed ? 0 : chunk * kUnitRows;
    // Rows the unit covers: tokens for Q / K, code columns for V.
    const int rows = streamed ? (int)ldv : min(kUnitRows, (kind == 2 ? (int)ldv : N) - row0);
    const int boxes = streamed ? 2 * nbv : (rows + kBoxRows - 1) / kBoxRows;   // copies, in order
    if (tid == 0) {
        prefetch_tmap(map);
        for (int i = 0; i < kSlots; ++i) mbar_init(&full[i], 1);
        fence_mbar_init();
        s_fail = 0;
    }
    for (int c = tid; c < NV * E; c += kThreads) amax[c] = 0u;
    __syncthreads();
    // Copy i lands in slot i % kSlots (phase (i / kSlots) & 1): box i of the unit, or
    // for a streamed V box i % nbv of the head.
    auto issue = [&](int i) {
        const int b = streamed ? i % nbv : i;
        mbar_arrive_expect_tx(&full[i % kSlots], (uint32_t)BB);
        if constexpr (NV == 16)
            tma_load_4d(buf + (i % kSlots) * BB, map, &full[i % kSlots], 0, 0, row0 + b * kBoxRows, (int)bh);
        else
            tma_load_3d(buf + (i % kSlots) * BB, map, &full[i % kSlots], 0, row0 + b * kBoxRows, (int)bh);
    };
    if (tid == 0)
        for (int i = 0; i < min(boxes, kSlots); ++i) issue(i);
    auto wait_copy = [&](int i) {
        if (mbar_wait(&full[i % kSlots], (uint32_t)((i / kSlots) & 1), nullptr, kCopyWaitNs)) return true;
        s_fail = 1;
        atomicOr(status, kStatusTimeoutCopy);
        return false;
    };

    if (kind < 2) {
        // ---------------------------------------------------- Q or K: a thread per token
        for (int t = tid; t < rows; t += kThreads) {
            if (!wait_copy(t / kBoxRows)) break;
            const uint8_t* box = buf + (t / kBoxRows) * BB;
            const int r = t % kBoxRows;
            uint4 raw[NV];
#pragma unroll
            for (int j = 0; j < NV; ++j) raw[j] = ld_chunk<NV>(box, r, j);
            const int64_t g = (int64_t)bh * N + row0 + t;
            pack_vectors<T, NV>(raw, d, (kind == 0 ? bq : bk) + g * words_for(d), (kind == 0 ? muq : muk) + g);
        }
        for (int i = 0; i < boxes; ++i) wait_copy(i);      // nothing may land after the CTA ends
    } else if (!streamed) {
        // ---------------------------------------------------- V codes, absmax given (bits of sv)
        // Work items (box i, chunk cw) go round the warps.
        for (int it = w; it < boxes * NV; it += kThreads / 32) {
            const int i = it / NV, cw = it - i * NV;
            float sc[E], rs[E];
#pragma unroll
            for (int e = 0; e < E; ++e) {
                sc[e] = __fdiv_rn(__uint_as_float(reinterpret_cast<const unsigned*>(sv)[bh * d + E * cw + e]), 127.0f);
                rs[e] = __frcp_rn(sc[e]);
            }
            if (wait_copy(i))
                codes_of_box<T, NV>(buf + i * BB, cw, lane, sc, rs, vq + ((size_t)bh * d + (size_t)E * cw) * ldv, ldv,
                                    row0 + i * kBoxRows);
        }
        for (int i = 0; i < boxes; ++i) wait_copy(i);
    } else {
        // ---------------------------------------------------- V of the whole head, two sweeps
        uint32_t m[4] = {0u, 0u, 0u, 0u};
        const int cv = tid % NV, rr = tid / NV;
        int issued = min(boxes, kSlots);
        for (int i = 0; i < boxes; ++i) {
            const bool have = i < issued && wait_copy(i);
            const uint8_t* box = buf + (i % kSlots) * BB;
            if (i < nbv) {
                if (have && rr < RG) absmax_of_box<T, NV>(box, cv, rr, RG, N - i * kBoxRows, m);
                if (i == nbv - 1) {
                    float mf[E];
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        if constexpr (sizeof(T) == 2) {
                            mf[2 * q] = __uint_as_float(m[q] << 16);
                            mf[2 * q + 1] = __uint_as_float(m[q] & 0xFFFF0000u);
                        } else {
                            mf[q] = __uint_as_float(m[q]);
                        }
                    }
                    if constexpr (NV == 8 || NV == 16) {
                        // Fold the lanes that share the chunk (l, l ^ NV, ...), then the warps.
#pragma unroll
                        for (int e = 0; e < E; ++e) {
                            unsigned u = __float_as_uint(mf[e]);
#pragma unroll
                            for (int o = NV; o < 32; o *= 2) u = max(u, __shfl_xor_sync(0xffffffffu, u, o));
                            if (lane < NV) atomicMax(&amax[E * cv + e], u);
                        }
                    } else if (rr < RG) {
#pragma unroll
                        for (int e = 0; e < E; ++e) atomicMax(&amax[E * cv + e], __float_as_uint(mf[e]));
                    }
                    __syncthreads();
                    if (tid < d) {
                        const float s = __fdiv_rn(__uint_as_float(amax[tid]), 127.0f);
                        s_scale[tid] = s;
                        s_rscale[tid] = __frcp_rn(s);
                        sv[bh * d + tid] = s;
                    }
                    __syncthreads();
                }
            } else if (have) {
                for (int cw = w; cw < NV; cw += kThreads / 32) {
                    float sc[E], rs[E];
#pragma unroll
                    for (int e = 0; e < E; ++e) {
                        sc[e] = s_scale[E * cw + e];
                        rs[e] = s_rscale[E * cw + e];
                    }
                    codes_of_box<T, NV>(box, cw, lane, sc, rs, vq + ((size_t)bh * d + (size_t)E * cw) * ldv, ldv,
                                        (i - nbv) * kBoxRows);
                }
            }
            __syncthreads();                                // slot i % kSlots is free again
            if (!s_fail && i + kSlots < boxes) {
                if (tid == 0) issue(i + kSlots);
                issued = i + kSlots + 1;
            }
        }
    }
}

template <typename T, int NV>
cudaError_t launch_tma_t(const void* q, const void* k, const void* v, ba_dtype dt, int BH, int N, int d, int vmode,
                         uint32_t* bq, float* muq, uint32_t* bk, float* muk, int8_t* vq, float* sv,
                         cudaStream_t st)
{
    auto encode = tc::encode_fn();
    unsigned* status = device_status_ptr();
    if (!encode || !status) return cudaErrorNotSupported;
    const int64_t ldv = round_up64(N, 16);
    const int nq = ceil_div(N, kUnitRows);
    PrepassMaps maps;
    // [BH][N][token]; 256-byte tokens as [BH][N][2][128 bytes] (4-D), so each
    // half is a 128-byte row the swizzle applies to.
    const int rank = NV == 16 ? 4 : 3;
    const cuuint64_t inner = NV == 16 ? (cuuint64_t)d / 2 : (cuuint64_t)d;
    const cuuint64_t dims3[3] = {inner, (cuuint64_t)N, (cuuint64_t)BH};
    const cuuint64_t dims4[4] = {inner, 2u, (cuuint64_t)N, (cuuint64_t)BH};
    const cuuint64_t strides3[2] = {(cuuint64_t)NV * 16u, (cuuint64_t)N * NV * 16u};
    const cuuint64_t strides4[3] = {128u, (cuuint64_t)NV * 16u, (cuuint64_t)N * NV * 16u};
    const cuuint32_t box3[3] = {(cuuint32_t)inner, (cuuint32_t)kBoxRows, 1u};
    const cuuint32_t box4[4] = {(cuuint32_t)inner, 2u, (cuuint32_t)kBoxRows, 1u};
    const cuuint32_t es[4] = {1u, 1u, 1u, 1u};
    const cuuint64_t* dims = NV == 16 ? dims4 : dims3;
    const cuuint64_t* strides = NV == 16 ? strides4 : strides3;
    const cuuint32_t* box = NV == 16 ? box4 : box3;
    const CUtensorMapDataType ty = dt == BA_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
    const void* src[3] = {q, k, v};
    CUtensorMap* dst[3] = {&maps.q, &maps.k, &maps.v};
    for (int i = 0; i < 3; ++i)
        if (encode(dst[i], ty, rank, const_cast<void*>(src[i]), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   NV == 9 ? CU_TENSOR_MAP_SWIZZLE_NONE : CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    const int smem = kSlots * box_bytes<NV>() + buf_align<NV>();   // the box slots + alignment slack
    auto kern = prepass_tma_kernel<T, NV>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    const int v_units = vmode == kVWhole ? 1 : vmode == kVCodes ? (int)((ldv + kUnitRows - 1) / kUnitRows) : 0;
    const int64_t units = (int64_t)BH * (v_units + 2 * nq);
    kern<<<(unsigned)units, kThreads, (size_t)smem, st>>>(maps, N, d, ldv, nq, vmode, bq, muq, bk, muk, vq, sv,
                                                         status);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_v_absmax(const void* v, ba_dtype dt, int B, int H, int N, int d, float* sv, cudaStream_t st);
cudaError_t launch_v_scale(float* sv, int64_t n, cudaStream_t st);

// Shapes the TMA pre-pass serves: 128-, 144- and 256-byte tokens.  V of a head in
// the same launch up to 1024 code columns; longer heads take the channel
// absmax in a launch before it and turn it into scales in one after it.
bool prepass_tma_serves(int d, int esize) { return d * esize == 128 || d * esize == 144 || d * esize == 256; }
int prepass_tma_launches(int N) { return round_up64(N, 16) <= kVWholeMaxLd ? 1 : 3; }

// q, k, v 16-byte aligned.  cudaErrorNotSupported: nothing was launched.
cudaError_t launch_prepass_tma(const void* q, const void* k, const void* v, ba_dtype dt, int B, int H, int N, int d,
                               uint32_t* bq, float* muq, uint32_t* bk, float* muk, int8_t* vq, float* sv,
                               cudaStream_t st)
{
    const int es = dt == BA_BF16 ? 2 : 4;
    if (!prepass_tma_serves(d, es)) return cudaErrorNotSupported;
    const int BH = B * H;
    const bool whole = prepass_tma_launches(N) == 1;
    cudaError_t e = cudaSuccess;
    if (!whole) {
        if (!tc::encode_fn() || !device_status_ptr()) return cudaErrorNotSupported;
        e = launch_v_absmax(v, dt, B, H, N, d, sv, st);
        if (e != cudaSuccess) return e;
    }
    const int vmode = whole ? kVWhole : kVCodes;
    if (d * es == 128)
        e = dt == BA_BF16 ? launch_tma_t<__nv_bfloat16, 8>(q, k, v, dt, BH, N, d, vmode, bq, muq, bk, muk, vq, sv, st)
                          : launch_tma_t<float, 8>(q, k, v, dt, BH, N, d, vmode, bq, muq, bk, muk, vq, sv, st);
    else if (d * es == 256)
        e = dt == BA_BF16 ? launch_tma_t<__nv_bfloat16, 16>(q, k, v, dt, BH, N, d, vmode, bq, muq, bk, muk, vq, sv, st)
                          : launch_tma_t<float, 16>(q, k, v, dt, BH, N, d, vmode, bq, muq, bk, muk, vq, sv, st);
    else
        e = dt == BA_BF16 ? launch_tma_t<__nv_bfloat16, 9>(q, k, v, dt, BH, N, d, vmode, bq, muq, bk, muk, vq, sv, st)
                          : launch_tma_t<float, 9>(q, k, v, dt, BH, N, d, vmode, bq, muq, bk, muk, vq, sv, st);
    if (e == cudaSuccess && !whole) e = launch_v_scale(sv, (int64_t)BH * d, st);
    return e;
}

}  // namespace ba
