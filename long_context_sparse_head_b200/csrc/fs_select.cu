// Long-range cell selection, "FreeSolo" summary §3.3 eqs. (7)-(8) (CUDA-core version).
//
// One CTA per (batch*head, position group G): the rows whose positions lie in
// [G*s, (G+1)*s) share the candidate prefix C_i = cells [0, n) (w is a multiple of s),
// hence share A_i.  The CTA
//   1. builds A (eq. (8)) from the TopP exit table: c in A iff c >= n - W or n < exit(c),
//   2. scores the rows against A in chunks of 64 cells (eq. (7), fp32 dot products with
//      the fp32 mean keys; the erf prior when lambda is given),
//   3. keeps each row's K best (larger score, ties to the lower cell) by rank counting
//      over the running top list plus the chunk, and
//   4. writes the kept cells in ascending order, -1 padded.
#include "fs_common.cuh"

namespace fs {

namespace {
constexpr int CH = 64;       // cells scored per chunk
constexpr int TPB = 256;     // threads per CTA (8 warps)
constexpr int ROWS = kS;     // rows per position group

struct SelectSmem {
    float qs[ROWS][kD];
    float kb[CH][kD + 1];
    float sc[ROWS][CH];
    float top_s[ROWS][kMaxK];
    int top_c[ROWS][kMaxK];
    int chunk_cells[CH];
    int alist[kMaxAdmit];
    int warp_cnt[TPB / 32];
    int nA;
};
}  // namespace

template <typename T>
__global__ void __launch_bounds__(TPB) select_kernel(Dev P, const T *__restrict__ Q,
                                                     const float *__restrict__ kbar,
                                                     const float *__restrict__ amax,
                                                     const int *__restrict__ exitn,
                                                     int32_t *__restrict__ idx, int G_lo) {
    extern __shared__ __align__(16) uint8_t smraw[];
    SelectSmem &sm = *reinterpret_cast<SelectSmem *>(smraw);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int bh = blockIdx.y, G = G_lo + blockIdx.x, h = bh % P.H;
    const int i_lo = max(G * kS, P.q0), i_hi = min((G + 1) * kS, P.Nk);
    const int nrows = i_hi - i_lo, r_lo = i_lo - P.q0;
    const int Kc = P.K;
    const int n = cand_count(i_lo, P.w, P.C);
    int32_t *out = idx + ((size_t)bh * P.Nq + r_lo) * Kc;
    if (nrows <= 0) return;
    if (n == 0 || Kc == 0) {
        for (int t = tid; t < nrows * Kc; t += TPB) out[t] = -1;
        return;
    }
    const float *a = amax + (size_t)bh * P.C;

    // 1. admitted cells, ascending (block-wide ordered compaction)
    int nA = n;
    if (P.prune) {
        const int *ex = exitn + (size_t)bh * P.C;
        if (tid == 0) sm.nA = 0;
        __syncthreads();
        for (int base = 0; base < n; base += TPB) {
            const int c = base + tid;
            const bool mem = c < n && (c >= n - P.W || n < ex[c]);
            const unsigned m = __ballot_sync(kFull, mem);
            if (lane == 0) sm.warp_cnt[warp] = __popc(m);
            __syncthreads();
            int off = sm.nA;
            for (int k = 0; k < warp; k++) off += sm.warp_cnt[k];
            const int pos = off + __popc(m & ((1u << lane) - 1u));
            if (mem && pos < kMaxAdmit) sm.alist[pos] = c;   // bound holds unless a_c is NaN
            __syncthreads();
            if (tid == 0) {
                int tot = 0;
                for (int k = 0; k < TPB / 32; k++) tot += sm.warp_cnt[k];
                sm.nA += tot;
            }
            __syncthreads();
        }
        nA = min(sm.nA, kMaxAdmit);
    }

    // query rows of the group, widened to fp32 (unrotated: NoPE, eq. (7))
    for (int t = tid; t < ROWS * kD; t += TPB) {
        const int rr = t / kD, m = t % kD;
        sm.qs[rr][m] = rr < nrows ? to_f<T>(Q[((size_t)bh * P.Nq + r_lo + rr) * kD + m]) : 0.f;
    }

    // 2-3. score chunk by chunk, merge into each row's running top-K
    int ntop = 0;
    for (int t0 = 0; t0 < nA; t0 += CH) {
        const int nch = min(CH, nA - t0);
        __syncthreads();
        if (tid < CH) sm.chunk_cells[tid] = tid < nch ? (P.prune ? sm.alist[t0 + tid] : t0 + tid) : 0;
        __syncthreads();
        for (int t = tid; t < nch * kD; t += TPB) {
            const int cc = t / kD, m = t % kD;
            sm.kb[cc][m] = kbar[((size_t)bh * P.C + sm.chunk_cells[cc]) * kD + m];
        }
        __syncthreads();
        {
            const int cc = tid % CH;
            if (cc < nch) {
                const int c = sm.chunk_cells[cc];
                const float prior_a = P.has_prior ? P.lambda[h] * a[c] : 0.f;
                const float pc = (c + 0.5f) * kS;
                for (int rr = tid / CH; rr < nrows; rr += TPB / CH) {
                    float acc = 0.f;
#pragma unroll 16
                    for (int m = 0; m < kD; m++) acc = fmaf(sm.qs[rr][m], sm.kb[cc][m], acc);
                    float r = acc * P.scale;
                    if (P.has_prior)
                        r += prior_a * erff(((float)(i_lo + rr) - pc) * P.inv2sigma[h]);
                    sm.sc[rr][cc] = r;
                }
            }
        }
        __syncthreads();
        for (int rr = warp; rr < nrows; rr += TPB / 32) {
            const int m = ntop + nch;                // <= kMaxK + CH = 128
            float es[4];
            int ec[4], rank[4];
#pragma unroll
            for (int j = 0; j < 4; j++) {
                const int e = lane + 32 * j;
                es[j] = -INFINITY; ec[j] = 0x7fffffff; rank[j] = 0;
                if (e < m) {
                    if (e < ntop) { es[j] = sm.top_s[rr][e]; ec[j] = sm.top_c[rr][e]; }
                    else { es[j] = sm.sc[rr][e - ntop]; ec[j] = sm.chunk_cells[e - ntop]; }
                }
            }
            for (int e2 = 0; e2 < m; e2++) {
                float s2; int c2;
                if (e2 < ntop) { s2 = sm.top_s[rr][e2]; c2 = sm.top_c[rr][e2]; }
                else { s2 = sm.sc[rr][e2 - ntop]; c2 = sm.chunk_cells[e2 - ntop]; }
#pragma unroll
                for (int j = 0; j < 4; j++) rank[j] += (s2 > es[j]) || (s2 == es[j] && c2 < ec[j]);
            }
            __syncwarp();
#pragma unroll
            for (int j = 0; j < 4; j++) {
                const int e = lane + 32 * j;
                if (e < m && rank[j] < Kc) { sm.top_s[rr][rank[j]] = es[j]; sm.top_c[rr][rank[j]] = ec[j]; }
            }
            __syncwarp();
        }
        ntop = min(Kc, ntop + nch);
    }
    __syncthreads();

    // 4. ascending cell order, -1 padding
    for (int rr = warp; rr < nrows; rr += TPB / 32) {
        for (int e = lane; e < Kc; e += 32) {
            if (e < ntop) {
                const int c = sm.top_c[rr][e];
                int slot = 0;
                for (int e2 = 0; e2 < ntop; e2++) slot += sm.top_c[rr][e2] < c;
                out[(size_t)rr * Kc + slot] = c;
            } else {
                out[(size_t)rr * Kc + e] = -1;
            }
        }
    }
}

cudaError_t launch_select(const Dev &P, fs_dtype dt, const void *Q, const float *kbar,
                          const float *amax, const int *exitn, int32_t *idx, cudaStream_t st) {
    if (P.Nq == 0) return cudaSuccess;
    const int G_lo = P.q0 / kS, G_hi = (P.Nk - 1) / kS;
    const dim3 grid(G_hi - G_lo + 1, P.B * P.H);
    const size_t smem = sizeof(SelectSmem);
    LaunchScope scope(kSelect, st);
    if (dt == FS_BF16) {
        auto k = select_kernel<__nv_bfloat16>;
        cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        k<<<grid, TPB, smem, st>>>(P, (const __nv_bfloat16 *)Q, kbar, amax, exitn, idx, G_lo);
    } else {
        auto k = select_kernel<float>;
        cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        k<<<grid, TPB, smem, st>>>(P, (const float *)Q, kbar, amax, exitn, idx, G_lo);
    }
    return cudaGetLastError();
}

}  // namespace fs
