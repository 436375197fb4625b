// Token-level rerank of the long-range selection, "FreeSolo" summary §3.4 eq. (12):
//   rt_ic = log sum_{j in I_c} exp(q_i . k_j / sqrt(d)) + lambda_h a_c erf((i - p_c) / (2 sigma_h))
// over the raw (NoPE) keys of cell c's tokens.  Reading: a shortlist of A_i, its
// `shortlist` best cells by eq. (7) (all of A_i for shortlist <= 0), is rescored by eq. (12)
// and the K best form S_i (ties: lower cell index), as in eq. (7)'s top-K.
//
// One CTA per (batch, head, 32 consecutive query positions aligned to 32): those rows share
// the prefix |C_i| (w is a multiple of s = 32), hence A_i.  The CTA builds A once from the
// TopP exit table, then
//   - eq. (7) scores of every (row, admitted cell), one thread per pair;
//   - eq. (12): each warp takes admitted cells in turn, stages the cell's 32 keys in
//     shared memory, and lane r (the group's row r, query in registers) computes the 32
//     token logits, their max and sum of exponentials: no reductions across lanes, and
//     each key is read once per group instead of once per row;
//   - per row: the shortlist by eq. (7), then the top-K by eq. (12), by rank counting.
// CUDA cores; |A_i| <= 128 cells.
#include "fs_common.cuh"

namespace fs {
namespace {

constexpr int kGroup = 32, kAmax = 128, kThreads = 256, kWarps = kThreads / 32;

struct RerankArgs {
    int Nq, Nk, q0, w, C, K, W, P, H, prune, shortlist;
    float scale;
    float lambda[FS_MAX_HEADS];
    float inv2sigma[FS_MAX_HEADS];
};

struct RerankSmem {
    float q[kGroup][kD];                 // the group's queries
    float r7[kGroup][kAmax];             // eq. (7) scores
    float r12[kGroup][kAmax];            // eq. (12) scores
    float kt[kWarps][kS][kD];            // one cell's keys per warp
    uint32_t insl[kGroup][kAmax / 32];   // shortlist membership per row
    uint32_t sel[kGroup][kAmax / 32];    // selected per row
    int acell[kAmax];                    // A (ascending)
    int wcnt[kWarps];
    int nA;
};

template <typename T>
__global__ void __launch_bounds__(kThreads) rerank_kernel(const RerankArgs A, const T *__restrict__ Q,
                                                          const T *__restrict__ K, const float *__restrict__ kbar,
                                                          const float *__restrict__ amax, const int *__restrict__ exitn,
                                                          int32_t *__restrict__ idx) {
    extern __shared__ __align__(16) uint8_t smraw[];
    RerankSmem &sm = *reinterpret_cast<RerankSmem *>(smraw);
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    const int bh = blockIdx.y, h = bh % A.H;
    // positions [g0, g0 + 32) of this group; rows r with q0 + r inside, in [0, Nq)
    const int g0 = (A.q0 / kGroup + blockIdx.x) * kGroup;
    const int n = cand_count(g0, A.w, A.C);      // the group's prefix |C_i|
    const float *kb = kbar + (size_t)bh * A.C * kD;
    const float *am = amax + (size_t)bh * A.C;
    const int *ex = exitn + (size_t)bh * A.C;

    // ---- A: admitted cells of prefix n (eq. (8)), ascending, by block-wide compaction
    int total = 0;
    for (int c0 = 0; c0 < n; c0 += kThreads) {
        const int c = c0 + t;
        const bool adm = c < n && (!A.prune || c >= n - A.W || n < ex[c]);
        const unsigned m = __ballot_sync(kFull, adm);
        if (lane == 0) sm.wcnt[warp] = __popc(m);
        __syncthreads();
        int pos = total + __popc(m & ((1u << lane) - 1u)), tot = 0;
        for (int k = 0; k < kWarps; k++) {
            if (k < warp) pos += sm.wcnt[k];
            tot += sm.wcnt[k];
        }
        if (adm && pos < kAmax) sm.acell[pos] = c;
        total += tot;
        __syncthreads();
    }
    const int nA = min(total, kAmax);            // the host guarantees total <= kAmax
    // ---- the group's queries
    for (int e = t; e < kGroup * kD; e += kThreads) {
        const int row = e / kD, pos = g0 + row;
        const int qr = pos - A.q0;
        sm.q[row][e % kD] = (qr >= 0 && qr < A.Nq) ? to_f<T>(Q[((size_t)bh * A.Nq + qr) * kD + e % kD]) : 0.f;
    }
    __syncthreads();
    // ---- eq. (7): one thread per (row, cell)
    for (int e = t; e < kGroup * nA; e += kThreads) {
        const int row = e / nA, a = e % nA, c = sm.acell[a];
        const float4 *k4 = reinterpret_cast<const float4 *>(kb + (size_t)c * kD);
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int d4 = 0; d4 < kD / 4; d4++) {
            const float4 v = __ldg(k4 + d4);
            acc[d4 & 3] = fmaf(sm.q[row][4 * d4], v.x, fmaf(sm.q[row][4 * d4 + 1], v.y,
                          fmaf(sm.q[row][4 * d4 + 2], v.z, fmaf(sm.q[row][4 * d4 + 3], v.w, acc[d4 & 3]))));
        }
        float r = ((acc[0] + acc[1]) + (acc[2] + acc[3])) * A.scale;
        if (A.lambda[h] != 0.f)
            r += A.lambda[h] * am[c] * erff(((float)(g0 + row - c * kS) - 0.5f * kS) * A.inv2sigma[h]);
        sm.r7[row][a] = r;
    }
    // ---- eq. (12): warp per cell, lane = row, log-sum-exp over the cell's tokens
    float q[kD];
#pragma unroll
    for (int e = 0; e < kD; e++) q[e] = sm.q[lane][e];
    const T *Kbh = K + (size_t)bh * A.Nk * kD;
    for (int a = warp; a < nA; a += kWarps) {
        const int c = sm.acell[a];
        const T *src = Kbh + (size_t)c * kS * kD;
        // the cell's 32 x 64 keys, 16-byte loads (coalesced), widened to float
        for (int e = lane * Vec<T>::N; e < kS * kD; e += 32 * Vec<T>::N) {
            float x[Vec<T>::N];
            Vec<T>::load(src + e, x);
#pragma unroll
            for (int u = 0; u < Vec<T>::N; u++) sm.kt[warp][(e + u) / kD][(e + u) % kD] = x[u];
        }
        __syncwarp();
        // the 32 token logits (independent), then one max and one sum of exponentials
        float lg[kS];
#pragma unroll
        for (int j = 0; j < kS; j++) {
            float acc[4] = {0.f, 0.f, 0.f, 0.f};
            const float4 *kj = reinterpret_cast<const float4 *>(sm.kt[warp][j]);   // broadcast
#pragma unroll
            for (int e4 = 0; e4 < kD / 4; e4++) {
                const float4 k4 = kj[e4];
                acc[0] = fmaf(q[4 * e4], k4.x, acc[0]);
                acc[1] = fmaf(q[4 * e4 + 1], k4.y, acc[1]);
                acc[2] = fmaf(q[4 * e4 + 2], k4.z, acc[2]);
                acc[3] = fmaf(q[4 * e4 + 3], k4.w, acc[3]);
            }
            lg[j] = ((acc[0] + acc[1]) + (acc[2] + acc[3])) * A.scale;
        }
        float m = lg[0];
#pragma unroll
        for (int j = 1; j < kS; j++) m = fmaxf(m, lg[j]);
        float se[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int j = 0; j < kS; j++) se[j & 3] += exp2f((lg[j] - m) * 1.4426950408889634f);
        const float sum = (se[0] + se[1]) + (se[2] + se[3]);
        float r = m + logf(sum);
        if (A.lambda[h] != 0.f)
            r += A.lambda[h] * am[c] * erff(((float)(g0 + lane - c * kS) - 0.5f * kS) * A.inv2sigma[h]);
        sm.r12[lane][a] = r;
        __syncwarp();                                // kt is refilled for the next cell
    }
    __syncthreads();
    // ---- per row: shortlist by eq. (7), then the K best by eq. (12); ties go to the lower
    //      cell (the lower position in A), by rank counting over (row, cell) pairs
    const int ns = A.shortlist > 0 ? min(A.shortlist, nA) : nA;
    for (int e = t; e < kGroup * (kAmax / 32); e += kThreads) {
        (&sm.insl[0][0])[e] = 0u;
        (&sm.sel[0][0])[e] = 0u;
    }
    __syncthreads();
    for (int e = t; e < kGroup * nA; e += kThreads) {
        const int row = e / nA, a = e % nA;
        bool in = true;
        if (ns < nA) {
            const float ra = sm.r7[row][a];
            int rank = 0;
            for (int b = 0; b < nA; b++) {
                const float rb = sm.r7[row][b];
                rank += rb > ra || (rb == ra && b < a);
            }
            in = rank < ns;
        }
        if (in) atomicOr(&sm.insl[row][a >> 5], 1u << (a & 31));
    }
    __syncthreads();
    for (int e = t; e < kGroup * nA; e += kThreads) {
        const int row = e / nA, a = e % nA;
        if (!((sm.insl[row][a >> 5] >> (a & 31)) & 1u)) continue;
        const float ta = sm.r12[row][a];
        int rank = 0;
        for (int b = 0; b < nA; b++) {
            const float tb = sm.r12[row][b];
            rank += ((sm.insl[row][b >> 5] >> (b & 31)) & 1u) && (tb > ta || (tb == ta && b < a));
        }
        if (rank < A.K) atomicOr(&sm.sel[row][a >> 5], 1u << (a & 31));
    }
    __syncthreads();
    if (t < kGroup) {                                // row t writes its cells, ascending
        const int qr = g0 + t - A.q0;
        if (qr >= 0 && qr < A.Nq) {
            int32_t *out = idx + ((size_t)bh * A.Nq + qr) * A.K;
            int o = 0;
            for (int a = 0; a < nA && o < A.K; a++)
                if ((sm.sel[t][a >> 5] >> (a & 31)) & 1u) out[o++] = sm.acell[a];
            for (; o < A.K; o++) out[o] = -1;
        }
    }
}

}  // namespace

// Per-tile selection records for the fused kernel from a selection idx [B,H,Nq,K]: one
// CTA per 128-row tile; the union of the rows' cells goes into a bitmap over the cells,
// is compacted in ascending order, and each row marks the union positions of its cells.
// A union above 128 cells (impossible for cells of A_i when W + P + 10 <= 128) raises the
// check flag and is cut.
__global__ void __launch_bounds__(128) idx_tiles_kernel(const int32_t *__restrict__ idx, int Nq, int K, int C,
                                                        uint32_t *__restrict__ tiles, int *dev_flag) {
    extern __shared__ uint32_t bm[];             // bitmap over cells [ceil(C / 32)]
    __shared__ int ulist[128], wsum[4], s_tot;
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    const int bh = blockIdx.y, r0 = blockIdx.x * 128, row = r0 + t;
    const int nw = (C + 31) / 32;
    for (int e = t; e < nw; e += 128) bm[e] = 0u;
    if (t == 0) s_tot = 0;
    __syncthreads();
    const int32_t *mine = idx + ((size_t)bh * Nq + row) * K;
    if (row < Nq)
        for (int k = 0; k < K; k++) {
            const int c = mine[k];
            if (c >= 0 && c < C) atomicOr(&bm[c >> 5], 1u << (c & 31));
        }
    __syncthreads();
    // ascending compaction: thread t owns words [t * wpt, (t + 1) * wpt)
    const int wpt = (nw + 127) / 128;
    int cnt = 0;
    for (int e = t * wpt; e < min(nw, (t + 1) * wpt); e++) cnt += __popc(bm[e]);
    int incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(kFull, incl, o);
        if (lane >= o) incl += v;
    }
    if (lane == 31) wsum[warp] = incl;
    __syncthreads();
    int pos = incl - cnt;
    for (int k = 0; k < warp; k++) pos += wsum[k];
    if (t == 127) s_tot = pos + cnt;
    for (int e = t * wpt; e < min(nw, (t + 1) * wpt); e++)
        for (uint32_t w = bm[e]; w; w &= w - 1) {
            if (pos < 128) ulist[pos] = 32 * e + __ffs(w) - 1;
            pos++;
        }
    __syncthreads();
    const int total = s_tot, nU = min(total, 128);
    if (total > 128 && t == 0 && dev_flag) atomicExch(dev_flag, kFlagCheck);
    uint32_t mw[4] = {0u, 0u, 0u, 0u};
    if (row < Nq)
        for (int k = 0; k < K; k++) {
            const int c = mine[k];
            if (c < 0) continue;
            int lo = 0, hi = nU;                     // first union position >= c
            while (lo < hi) {
                const int mid = (lo + hi) >> 1;
                if (ulist[mid] < c) lo = mid + 1; else hi = mid;
            }
            if (lo < nU && ulist[lo] == c) mw[lo >> 5] |= 1u << (lo & 31);
        }
    uint32_t *rec = tiles + ((size_t)bh * gridDim.x + blockIdx.x) * kTileRecWords;
    *reinterpret_cast<uint4 *>(rec + kTileMaskOff + 4 * t) = make_uint4(mw[0], mw[1], mw[2], mw[3]);
    rec[kTileUlistOff + t] = t < nU ? (uint32_t)ulist[t] : 0xffffffffu;
    rec[kTileMrefOff + t] = 0x7fc00000u;          // no reference: running maximum
    if (t == 0) rec[kTileCountOff] = (uint32_t)nU;
}

cudaError_t launch_idx_tiles(const Dev &P, const int32_t *idx, uint32_t *tiles, int *dev_flag, cudaStream_t st) {
    if (P.Nq == 0) return cudaSuccess;
    const dim3 grid((P.Nq + 127) / 128, P.B * P.H);
    const size_t smem = (size_t)((P.C + 31) / 32) * 4;
    LaunchScope scope(kIdxTiles, st);
    idx_tiles_kernel<<<grid, 128, smem, st>>>(idx, P.Nq, P.K, P.C, tiles, dev_flag);
    return cudaGetLastError();
}

bool rerank_supported(const fs_params *p) {
    const int C = p->Nk / p->s;
    const int bound = p->W >= 0 ? p->W + p->P : C;
    return bound <= kAmax;
}

cudaError_t launch_rerank(const Dev &P, fs_dtype dt, const void *Q, const void *K, const float *kbar,
                          const float *amax, const int *exitn, int shortlist, int32_t *idx, cudaStream_t st) {
    if (P.Nq == 0) return cudaSuccess;
    RerankArgs A;
    A.Nq = P.Nq; A.Nk = P.Nk; A.q0 = P.q0; A.w = P.w; A.C = P.C; A.K = P.K; A.W = P.W; A.P = P.P;
    A.H = P.H; A.prune = P.prune; A.shortlist = shortlist; A.scale = P.scale;
    for (int h = 0; h < FS_MAX_HEADS; h++) {
        A.lambda[h] = P.lambda[h];
        A.inv2sigma[h] = P.inv2sigma[h];
    }
    const int g_first = P.q0 / kGroup, g_last = (P.q0 + P.Nq - 1) / kGroup;
    const dim3 grid(g_last - g_first + 1, P.B * P.H);
    const size_t smem = sizeof(RerankSmem);
    LaunchScope scope(kRerank, st);
    if (dt == FS_BF16) {
        cudaFuncSetAttribute(rerank_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        rerank_kernel<__nv_bfloat16><<<grid, kThreads, smem, st>>>(A, (const __nv_bfloat16 *)Q,
                                                                   (const __nv_bfloat16 *)K, kbar, amax, exitn, idx);
    } else {
        cudaFuncSetAttribute(rerank_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        rerank_kernel<float><<<grid, kThreads, smem, st>>>(A, (const float *)Q, (const float *)K, kbar, amax,
                                                           exitn, idx);
    }
    return cudaGetLastError();
}

}  // namespace fs
