// ba_scores.cu -- KD1 debug path: the integer binary score matrix.
//
// BA notes, Key design 1: s_i . t_j computed with XNOR + popcount; with sign
// bits packed LSB first and zero padding, s.t = d - 2 popcount(bq XOR bk).
// Output-bound (4 bytes per score); tiles of 64 x 64 scores per CTA with both
// operand tiles staged in shared memory.
#include "ba_common.cuh"

namespace ba {

template <int W>
__global__ void __launch_bounds__(256)
scores_kernel(const uint32_t* __restrict__ bq, const uint32_t* __restrict__ bk, int N, int d,
              int32_t* __restrict__ z)
{
    constexpr int T = 64;
    __shared__ uint32_t sq[T][W];
    __shared__ uint32_t sk[T][W + 1];
    const int64_t bh = blockIdx.z;
    const int i0 = blockIdx.y * T, j0 = blockIdx.x * T;
    for (int idx = threadIdx.x; idx < T * W; idx += blockDim.x) {
        const int r = idx / W, w = idx - r * W;
        sq[r][w] = (i0 + r < N) ? bq[(bh * N + i0 + r) * W + w] : 0u;
        sk[r][w] = (j0 + r < N) ? bk[(bh * N + j0 + r) * W + w] : 0u;
    }
    __syncthreads();
    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
#pragma unroll
    for (int a = 0; a < 4; ++a) {
        const int i = ty * 4 + a;
        uint32_t q[W];
#pragma unroll
        for (int w = 0; w < W; ++w) q[w] = sq[i][w];
#pragma unroll
        for (int b = 0; b < 4; ++b) {
            const int j = tx + 16 * b;
            int ham = 0;
#pragma unroll
            for (int w = 0; w < W; ++w) ham += __popc(q[w] ^ sk[j][w]);
            if (i0 + i < N && j0 + j < N)
                z[(bh * N + i0 + i) * (int64_t)N + j0 + j] = d - 2 * ham;
        }
    }
}

cudaError_t launch_scores(const uint32_t* bq, const uint32_t* bk, int B, int H, int N, int d,
                          int32_t* z, cudaStream_t st)
{
    dim3 grid(ceil_div(N, 64), ceil_div(N, 64), (unsigned)((int64_t)B * H));
    switch (words_for(d)) {
        case 1: scores_kernel<1><<<grid, 256, 0, st>>>(bq, bk, N, d, z); break;
        case 2: scores_kernel<2><<<grid, 256, 0, st>>>(bq, bk, N, d, z); break;
        case 3: scores_kernel<3><<<grid, 256, 0, st>>>(bq, bk, N, d, z); break;
        default: scores_kernel<4><<<grid, 256, 0, st>>>(bq, bk, N, d, z); break;
    }
    return cudaGetLastError();
}

}  // namespace ba
