// Cell summaries, "FreeSolo" summary §3.3 eq. (5):
//   kbar_c = (1/s) sum_{j in cell c} k_j,   a_c = max_{j in cell c} ||k_j||_2.
//
// One warp per cell; the cell is s = 32 rows of d = 64 keys, read once with 16-byte
// loads (a row is 8 lanes of bf16 or 16 lanes of f32), all loads of a warp issued
// before any use.  HBM-bound: 4 KiB (bf16) read and 260 B written per cell.
#include "fs_common.cuh"

namespace fs {

template <typename T>
__global__ void __launch_bounds__(256) summaries_kernel(const T *__restrict__ K,
                                                        float *__restrict__ kbar,
                                                        float *__restrict__ amax,
                                                        long long ncell, int C, int Nk) {
    constexpr int VEC = Vec<T>::N;        // elements per 16-byte load
    constexpr int LPR = kD / VEC;         // lanes per key row
    constexpr int RPP = 32 / LPR;         // rows per warp pass
    constexpr int PASSES = kS / RPP;
    const long long cell = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (cell >= ncell) return;
    const int lane = threadIdx.x & 31;
    const long long bh = cell / C;
    const int c = (int)(cell - bh * C);
    const T *base = K + ((size_t)bh * Nk + (size_t)c * kS) * kD;
    const int col = (lane % LPR) * VEC;
    const int row0 = lane / LPR;

    float x[PASSES][VEC];
#pragma unroll
    for (int p = 0; p < PASSES; p++) Vec<T>::load(base + (size_t)(row0 + p * RPP) * kD + col, x[p]);

    float sum[VEC];
#pragma unroll
    for (int e = 0; e < VEC; e++) sum[e] = 0.f;
    float maxsq = 0.f;
#pragma unroll
    for (int p = 0; p < PASSES; p++) {
        float sq = 0.f;
#pragma unroll
        for (int e = 0; e < VEC; e++) {
            sum[e] += x[p][e];
            sq = fmaf(x[p][e], x[p][e], sq);
        }
#pragma unroll
        for (int o = LPR / 2; o > 0; o >>= 1) sq += __shfl_xor_sync(kFull, sq, o);
        maxsq = fmaxf(maxsq, sq);
    }
#pragma unroll
    for (int o = LPR; o < 32; o <<= 1) {
#pragma unroll
        for (int e = 0; e < VEC; e++) sum[e] += __shfl_xor_sync(kFull, sum[e], o);
        maxsq = fmaxf(maxsq, __shfl_xor_sync(kFull, maxsq, o));
    }
    if (lane < LPR) {
        float *dst = kbar + (size_t)cell * kD + col;
#pragma unroll
        for (int e = 0; e < VEC; e += 4)
            *reinterpret_cast<float4 *>(dst + e) =
                make_float4(sum[e] * (1.f / kS), sum[e + 1] * (1.f / kS),
                            sum[e + 2] * (1.f / kS), sum[e + 3] * (1.f / kS));
    }
    if (lane == 0) amax[cell] = sqrtf(maxsq);
}

cudaError_t launch_summaries(const Dev &P, fs_dtype dt, const void *K, float *kbar,
                             float *amax, cudaStream_t st) {
    const long long ncell = (long long)P.B * P.H * P.C;
    if (ncell == 0) return cudaSuccess;
    const int warps = 8;
    const long long blocks = (ncell + warps - 1) / warps;
    LaunchScope scope(kSummaries, st);
    if (dt == FS_BF16)
        summaries_kernel<__nv_bfloat16><<<(unsigned)blocks, warps * 32, 0, st>>>(
            (const __nv_bfloat16 *)K, kbar, amax, ncell, P.C, P.Nk);
    else
        summaries_kernel<float><<<(unsigned)blocks, warps * 32, 0, st>>>(
            (const float *)K, kbar, amax, ncell, P.C, P.Nk);
    return cudaGetLastError();
}

}  // namespace fs
