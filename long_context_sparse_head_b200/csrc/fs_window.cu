// Local RoPE branch and the range combination (CUDA-core version),
// "FreeSolo" summary §3.2 eqs. (3)-(4) and §3.1 eq. (2):
//   o_i^sr = softmax_{j in [i-w, i]}((R(i)q_i).(R(j)k_j) / sqrt(d)) V,
//   O_i    = o_i^sr + alpha_h o_i^lr        (alpha_h o_i^lr precomputed by the readout).
//
// One CTA per 64 consecutive query rows of a (batch, head).  RoPE is applied while
// staging Q and each 64-key chunk in shared memory, with angles measured from the tile's
// first query position: by eq. (3) only j - i matters, and offsets of at most w + 64
// keep the fp32 angles exact to ~1e-5 rad at any sequence length.
#include "fs_common.cuh"

namespace fs {

namespace {
constexpr int TPB = 256;
constexpr int BQ = 64;      // query rows per CTA
constexpr int BK = 64;      // keys per chunk

struct WindowSmem {
    float qs[BQ][kD];
    float kt[BK][kD + 1];
    float vt[BK][kD];
};

// Stage `rows` rows starting at src (row stride kD), rotating pair m of row t by angle
// (off0 + t) * theta_m; rows past `rows` are zero-filled.
template <typename T, int LD>
__device__ __forceinline__ void stage_rotated(float (*dst)[LD], const T *src, int rows, int off0,
                                              const float *theta) {
    for (int t = threadIdx.x; t < 64 * (kD / 2); t += TPB) {
        const int row = t / (kD / 2), m = t % (kD / 2);
        float x0 = 0.f, x1 = 0.f;
        if (row < rows) {
            x0 = to_f<T>(src[(size_t)row * kD + 2 * m]);
            x1 = to_f<T>(src[(size_t)row * kD + 2 * m + 1]);
        }
        float sn, cs;
        sincosf((float)(off0 + row) * theta[m], &sn, &cs);
        dst[row][2 * m] = x0 * cs - x1 * sn;
        dst[row][2 * m + 1] = x0 * sn + x1 * cs;
    }
}
}  // namespace

template <typename T>
__global__ void __launch_bounds__(TPB) window_kernel(Dev P, const T *__restrict__ Q,
                                                     const T *__restrict__ K,
                                                     const T *__restrict__ V,
                                                     const float *__restrict__ olr,
                                                     T *__restrict__ O) {
    extern __shared__ __align__(16) uint8_t smraw[];
    WindowSmem &sm = *reinterpret_cast<WindowSmem *>(smraw);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int bh = blockIdx.y;
    const int r0 = blockIdx.x * BQ;
    const int nrows = min(BQ, P.Nq - r0);
    const int pb = P.q0 + r0;                          // position of the tile's first query
    const int j_lo = max(0, pb - P.w);
    const int j_hi = pb + nrows - 1;                   // last key any row needs
    const size_t kvbase = (size_t)bh * P.Nk * kD;

    stage_rotated<T, kD>(sm.qs, Q + ((size_t)bh * P.Nq + r0) * kD, nrows, 0, P.theta);

    constexpr int RPW = BQ / (TPB / 32);               // rows per warp = 8
    float mrow[RPW], lrow[RPW], acc0[RPW], acc1[RPW];
#pragma unroll
    for (int k = 0; k < RPW; k++) { mrow[k] = -INFINITY; lrow[k] = 0.f; acc0[k] = acc1[k] = 0.f; }

    for (int jc = j_lo; jc <= j_hi; jc += BK) {
        const int nk = min(BK, j_hi - jc + 1);
        __syncthreads();
        stage_rotated<T, kD + 1>(sm.kt, K + kvbase + (size_t)jc * kD, nk, jc - pb, P.theta);
        for (int t = tid; t < BK * kD; t += TPB) {
            const int row = t / kD, m = t % kD;
            sm.vt[row][m] = row < nk ? to_f<T>(V[kvbase + (size_t)(jc + row) * kD + m]) : 0.f;
        }
        __syncthreads();
#pragma unroll 1
        for (int k = 0; k < RPW; k++) {
            const int rr = warp * RPW + k;
            if (rr >= nrows) break;
            const int i = pb + rr;
            const int j0 = jc + lane, j1 = jc + lane + 32;
            const bool v0 = (j0 - jc) < nk && j0 >= i - P.w && j0 <= i;
            const bool v1 = (j1 - jc) < nk && j1 >= i - P.w && j1 <= i;
            if (!__any_sync(kFull, v0 || v1)) continue;
            float l0 = 0.f, l1 = 0.f;
#pragma unroll 16
            for (int m = 0; m < kD; m++) {
                const float q = sm.qs[rr][m];
                l0 = fmaf(q, sm.kt[lane][m], l0);
                l1 = fmaf(q, sm.kt[lane + 32][m], l1);
            }
            l0 = v0 ? l0 * P.scale : -INFINITY;
            l1 = v1 ? l1 * P.scale : -INFINITY;
            const float mnew = fmaxf(mrow[k], warp_max(fmaxf(l0, l1)));
            const float corr = expf(mrow[k] - mnew);
            const float p0 = v0 ? expf(l0 - mnew) : 0.f;
            const float p1 = v1 ? expf(l1 - mnew) : 0.f;
            lrow[k] = lrow[k] * corr + warp_sum(p0 + p1);
            float a0 = acc0[k] * corr, a1 = acc1[k] * corr;
#pragma unroll 8
            for (int j = 0; j < 32; j++) {
                const float pj = __shfl_sync(kFull, p0, j);
                const float2 v = *reinterpret_cast<const float2 *>(&sm.vt[j][2 * lane]);
                a0 = fmaf(pj, v.x, a0);
                a1 = fmaf(pj, v.y, a1);
            }
#pragma unroll 8
            for (int j = 0; j < 32; j++) {
                const float pj = __shfl_sync(kFull, p1, j);
                const float2 v = *reinterpret_cast<const float2 *>(&sm.vt[32 + j][2 * lane]);
                a0 = fmaf(pj, v.x, a0);
                a1 = fmaf(pj, v.y, a1);
            }
            acc0[k] = a0; acc1[k] = a1; mrow[k] = mnew;
        }
    }

#pragma unroll
    for (int k = 0; k < RPW; k++) {
        const int rr = warp * RPW + k;
        if (rr >= nrows) break;
        const size_t row = (size_t)bh * P.Nq + r0 + rr;
        float o0 = acc0[k] / lrow[k], o1 = acc1[k] / lrow[k];
        if (olr) {
            const float2 x = *reinterpret_cast<const float2 *>(&olr[row * kD + 2 * lane]);
            o0 += x.x;
            o1 += x.y;
        }
        O[row * kD + 2 * lane] = from_f<T>(o0);
        O[row * kD + 2 * lane + 1] = from_f<T>(o1);
    }
}

cudaError_t launch_window(const Dev &P, fs_dtype dt, const void *Q, const void *K,
                          const void *V, const float *olr, void *O, cudaStream_t st) {
    if (P.Nq == 0) return cudaSuccess;
    const dim3 grid((P.Nq + BQ - 1) / BQ, P.B * P.H);
    const size_t smem = sizeof(WindowSmem);
    LaunchScope scope(kWindow, st);
    if (dt == FS_BF16) {
        auto k = window_kernel<__nv_bfloat16>;
        cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        k<<<grid, TPB, smem, st>>>(P, (const __nv_bfloat16 *)Q, (const __nv_bfloat16 *)K,
                                   (const __nv_bfloat16 *)V, olr, (__nv_bfloat16 *)O);
    } else {
        auto k = window_kernel<float>;
        cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        k<<<grid, TPB, smem, st>>>(P, (const float *)Q, (const float *)K, (const float *)V, olr,
                                   (float *)O);
    }
    return cudaGetLastError();
}

}  // namespace fs
