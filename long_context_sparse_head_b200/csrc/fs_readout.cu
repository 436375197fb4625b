// Long-range token readout, "FreeSolo" summary §3.3 eq. (9) (CUDA-core version):
//   u_i = softmax_{j in cells of S_i}(q_i.k_j / sqrt(d)) V,   o_i^lr = RMSNorm(u_i),
// with unrotated (NoPE) q and k.  Writes alpha_h * o_i^lr (fp32) for the window kernel's
// epilogue to add (eq. (2)).
//
// One CTA per (batch*head, position group).  The union of the group's selected cells is
// walked in ascending order; each cell's 32 keys and values are staged once in shared
// memory and read by every row that selected it.  A warp owns four rows and keeps an
// online softmax (running max, sum, two output dims per lane) for each.
#include "fs_common.cuh"

namespace fs {

namespace {
constexpr int TPB = 256;
constexpr int ROWS = kS;

struct ReadoutSmem {
    float qs[ROWS][kD];
    float kt[kS][kD + 1];
    float vt[kS][kD];
    int sel[ROWS][kMaxK];
    // followed by the union bitmap: ceil(C / 32) words
};
}  // namespace

template <typename T>
__global__ void __launch_bounds__(TPB) readout_kernel(Dev P, const T *__restrict__ Q,
                                                      const T *__restrict__ K,
                                                      const T *__restrict__ V,
                                                      const int32_t *__restrict__ idx,
                                                      float *__restrict__ olr, int G_lo) {
    extern __shared__ __align__(16) uint8_t smraw[];
    ReadoutSmem &sm = *reinterpret_cast<ReadoutSmem *>(smraw);
    unsigned *bitmap = reinterpret_cast<unsigned *>(smraw + sizeof(ReadoutSmem));
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int bh = blockIdx.y, G = G_lo + blockIdx.x, h = bh % P.H;
    const int i_lo = max(G * kS, P.q0), i_hi = min((G + 1) * kS, P.Nk);
    const int nrows = i_hi - i_lo, r_lo = i_lo - P.q0;
    if (nrows <= 0) return;
    const int Kc = P.K;
    const int nwords = (P.C + 31) / 32;

    for (int t = tid; t < nwords; t += TPB) bitmap[t] = 0u;
    for (int t = tid; t < ROWS * kD; t += TPB) {
        const int rr = t / kD, m = t % kD;
        sm.qs[rr][m] = rr < nrows ? to_f<T>(Q[((size_t)bh * P.Nq + r_lo + rr) * kD + m]) : 0.f;
    }
    __syncthreads();
    for (int t = tid; t < ROWS * Kc; t += TPB) {
        const int rr = t / Kc, e = t % Kc;
        int c = -1;
        if (rr < nrows) c = idx[((size_t)bh * P.Nq + r_lo + rr) * Kc + e];
        if (c >= P.C) c = -1;                       // ignore out-of-range caller cells
        sm.sel[rr][e] = c;
        if (c >= 0) atomicOr(&bitmap[c >> 5], 1u << (c & 31));
    }
    __syncthreads();

    constexpr int RPW = ROWS / (TPB / 32);          // rows per warp = 4
    float mrow[RPW], lrow[RPW], acc0[RPW], acc1[RPW];
    int cur[RPW];
#pragma unroll
    for (int k = 0; k < RPW; k++) { mrow[k] = -INFINITY; lrow[k] = 0.f; acc0[k] = acc1[k] = 0.f; cur[k] = 0; }

    const size_t kvbase = (size_t)bh * P.Nk * kD;
    constexpr int VEC = Vec<T>::N;
    for (int wi = 0; wi < nwords; wi++) {
        unsigned bits = bitmap[wi];
        while (bits) {
            const int c = wi * 32 + __ffs(bits) - 1;
            bits &= bits - 1;
            __syncthreads();                        // previous cell's readers are done
            for (int t = tid; t < kS * kD / VEC; t += TPB) {
                const int row = (t * VEC) / kD, m0 = (t * VEC) % kD;
                float xk[VEC], xv[VEC];
                Vec<T>::load(K + kvbase + ((size_t)c * kS + row) * kD + m0, xk);
                Vec<T>::load(V + kvbase + ((size_t)c * kS + row) * kD + m0, xv);
#pragma unroll
                for (int e = 0; e < VEC; e++) { sm.kt[row][m0 + e] = xk[e]; sm.vt[row][m0 + e] = xv[e]; }
            }
            __syncthreads();
#pragma unroll
            for (int k = 0; k < RPW; k++) {
                const int rr = warp + k * (TPB / 32);
                if (rr >= nrows || cur[k] >= Kc || sm.sel[rr][cur[k]] != c) continue;
                cur[k]++;
                float lg = 0.f;
#pragma unroll 16
                for (int m = 0; m < kD; m++) lg = fmaf(sm.qs[rr][m], sm.kt[lane][m], lg);
                lg *= P.scale;
                const float mnew = fmaxf(mrow[k], warp_max(lg));
                const float corr = expf(mrow[k] - mnew);
                const float p = expf(lg - mnew);
                lrow[k] = lrow[k] * corr + warp_sum(p);
                float a0 = acc0[k] * corr, a1 = acc1[k] * corr;
#pragma unroll 8
                for (int j = 0; j < kS; j++) {
                    const float pj = __shfl_sync(kFull, p, j);
                    const float2 v = *reinterpret_cast<const float2 *>(&sm.vt[j][2 * lane]);
                    a0 = fmaf(pj, v.x, a0);
                    a1 = fmaf(pj, v.y, a1);
                }
                acc0[k] = a0; acc1[k] = a1; mrow[k] = mnew;
            }
        }
    }

    const float alpha = P.alpha[h];
#pragma unroll
    for (int k = 0; k < RPW; k++) {
        const int rr = warp + k * (TPB / 32);
        if (rr >= nrows) continue;
        float o0 = 0.f, o1 = 0.f;
        if (lrow[k] > 0.f) {
            const float u0 = acc0[k] / lrow[k], u1 = acc1[k] / lrow[k];
            const float ms = warp_sum(u0 * u0 + u1 * u1) * (1.f / kD);
            const float inv = 1.f / sqrtf(ms + P.rms_eps);
            o0 = alpha * u0 * inv;
            o1 = alpha * u1 * inv;
        }
        *reinterpret_cast<float2 *>(&olr[((size_t)bh * P.Nq + r_lo + rr) * kD + 2 * lane]) =
            make_float2(o0, o1);
    }
}

cudaError_t launch_readout(const Dev &P, fs_dtype dt, const void *Q, const void *K,
                           const void *V, const int32_t *idx, float *olr, cudaStream_t st) {
    if (P.Nq == 0) return cudaSuccess;
    const int G_lo = P.q0 / kS, G_hi = (P.Nk - 1) / kS;
    const dim3 grid(G_hi - G_lo + 1, P.B * P.H);
    const size_t smem = sizeof(ReadoutSmem) + sizeof(unsigned) * (size_t)((P.C + 31) / 32);
    LaunchScope scope(kReadout, st);
    if (dt == FS_BF16) {
        auto k = readout_kernel<__nv_bfloat16>;
        cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        k<<<grid, TPB, smem, st>>>(P, (const __nv_bfloat16 *)Q, (const __nv_bfloat16 *)K,
                                   (const __nv_bfloat16 *)V, idx, olr, G_lo);
    } else {
        auto k = readout_kernel<float>;
        cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        k<<<grid, TPB, smem, st>>>(P, (const float *)Q, (const float *)K, (const float *)V, idx,
                                   olr, G_lo);
    }
    return cudaGetLastError();
}

// Per-row variant, for selections that differ across the rows of a group (the FS-B
// search picks cells anywhere in the prefix, so a group's union is large and each staged
// cell serves few rows).  One warp per query row, lane m holding dimensions (2m, 2m+1): a
// cell's 32 logits come from per-lane partial products and a transposed butterfly sum
// (lane t: token t), then an online softmax over the row's cells; no shared memory.
namespace {
constexpr int kRowsPerBlock = 4;

template <typename T>
__global__ void __launch_bounds__(kRowsPerBlock * 32) readout_rows_kernel(Dev P, const T *__restrict__ Q,
                                                                         const T *__restrict__ K,
                                                                         const T *__restrict__ V,
                                                                         const int32_t *__restrict__ idx,
                                                                         float *__restrict__ olr) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int bh = blockIdx.y, h = bh % P.H;
    const int r = blockIdx.x * kRowsPerBlock + warp;
    if (r >= P.Nq) return;                                   // warp-uniform
    const size_t row = (size_t)bh * P.Nq + r;
    const size_t kb = (size_t)bh * P.Nk;
    const float2 q = ld_pair<T>(Q + row * kD + 2 * lane);
    float m = -INFINITY, l = 0.f, u0 = 0.f, u1 = 0.f;
    for (int e = 0; e < P.K; e++) {
        const int c = idx[row * P.K + e];
        if ((unsigned)c >= (unsigned)P.C) continue;           // -1 padding, out-of-range cells
        const T *kc = K + (kb + (size_t)c * kS) * kD + 2 * lane;
        const T *vc = V + (kb + (size_t)c * kS) * kD + 2 * lane;
        float v[32];
#pragma unroll
        for (int t = 0; t < 32; t++) {
            const float2 k2 = ld_pair<T>(kc + t * kD);
            v[t] = fmaf(q.x, k2.x, q.y * k2.y);
        }
        const float x = transpose_sum32(v, lane) * P.scale;  // lane t: token t's logit
        const float mn = fmaxf(m, warp_max(x));
        const float corr = __expf(m - mn);                    // 0 while m is -inf
        const float p = __expf(x - mn);
        l = l * corr + warp_sum(p);
        u0 *= corr;
        u1 *= corr;
#pragma unroll
        for (int t = 0; t < 32; t++) {
            const float pt = __shfl_sync(kFull, p, t);
            const float2 v2 = ld_pair<T>(vc + t * kD);
            u0 = fmaf(pt, v2.x, u0);
            u1 = fmaf(pt, v2.y, u1);
        }
        m = mn;
    }
    float o0 = 0.f, o1 = 0.f;
    if (l > 0.f) {
        const float y0 = u0 / l, y1 = u1 / l;
        const float inv = rsqrtf(warp_sum(y0 * y0 + y1 * y1) * (1.f / kD) + P.rms_eps);
        o0 = P.alpha[h] * y0 * inv;
        o1 = P.alpha[h] * y1 * inv;
    }
    *reinterpret_cast<float2 *>(&olr[row * kD + 2 * lane]) = make_float2(o0, o1);
}
}  // namespace

cudaError_t launch_readout_rows(const Dev &P, fs_dtype dt, const void *Q, const void *K,
                                const void *V, const int32_t *idx, float *olr, cudaStream_t st) {
    if (P.Nq == 0) return cudaSuccess;
    const dim3 grid((P.Nq + kRowsPerBlock - 1) / kRowsPerBlock, P.B * P.H);
    LaunchScope scope(kReadoutRows, st);
    if (dt == FS_BF16)
        readout_rows_kernel<__nv_bfloat16><<<grid, kRowsPerBlock * 32, 0, st>>>(
            P, (const __nv_bfloat16 *)Q, (const __nv_bfloat16 *)K, (const __nv_bfloat16 *)V, idx, olr);
    else
        readout_rows_kernel<float><<<grid, kRowsPerBlock * 32, 0, st>>>(P, (const float *)Q, (const float *)K,
                                                                        (const float *)V, idx, olr);
    return cudaGetLastError();
}

}  // namespace fs
