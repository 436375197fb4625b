// Token-level rerank on the 5th-generation tensor cores (bf16), "FreeSolo" summary §3.4
// eq. (12), over the FS-L admitted sets of §3.3 eq. (8):
//   rt_ic = log sum_{j in I_c} exp(q_i.k_j / sqrt(d)) + lambda_h a_c erf((i - p_c) / (2 sigma_h)),
//   S_i   = the K cells of A_i with the largest rt_ic (ties: lower cell index).
//
// One CTA per 128 query rows of a (batch, head).  Warps 0-3 build U, the ordered union of
// the tile's admitted sets (the rows of a tile have at most five distinct prefixes), as
// the selection kernel does.  The TMA warp then gathers the keys of U two cells (64 keys)
// per chunk with 32-row boxes into a four-stage ring; the MMA warp computes
// S = Q K_chunk^T (M = 128, N = 64, fp32 in tensor memory, two S buffers); warps 0-3
// (thread = query row = TMEM lane) read each chunk's 64 scores, take each 32-column
// block's log-sum-exp (one exponential per score), add the prior and keep the result per
// (row, union position) in shared memory.  After the last chunk each thread keeps its
// row's admitted positions and finds the K-th largest by bisection on unique integer keys:
// the score as a 24-bit fixed-point fraction of the row's score range (about one float
// ulp), then (127 - position), so equal scores go to the lower cell.  Outputs: idx and/or
// the fused kernel's per-tile record (row masks over U, U, |U|), so the fused readout +
// window kernel can run on the reranked cells directly.
#include "tc_common.cuh"

namespace fs {

namespace {
constexpr int BM = 128, BN = 64, NSTAGE = 4, CPC = BN / kS;
constexpr int NSEL = 4, W_TMA = 4, W_MMA = 5, NWARPS = 6, NTHREADS = NWARPS * 32;
constexpr uint32_t TMEM_COLS = 128;                 // two S buffers of BN columns
constexpr int TILE_BYTES = BM * kD * 2, CELL_BYTES = kS * kD * 2;
constexpr int kSelBarrier = 1;                      // named barrier of the 128 row threads

template <int UM> struct RrSmem {
    __nv_bfloat16 q[BM * kD];                       // Q tile (NoPE), 1024-byte aligned
    __nv_bfloat16 k[NSTAGE][BN * kD];               // gathered keys, two cells per stage
    float rt[BM][UM + 1];                           // eq. (12) per (row, union position)
    int ulist[UM];
    float acell[UM];
    uint8_t amask[UM];                              // bit g: admitted for prefix n_min + g
    uint32_t admit[5][(UM + 31) / 32];
    int warp_cnt[4];
    int nU;
    uint64_t q_full, u_ready, drain;
    uint64_t s_full[2], s_free[2];
    uint64_t kv_full[NSTAGE], kv_empty[NSTAGE];
    uint32_t tmem_base;
    int abort;
};

struct RrArgs {
    int Nq, Nk, q0, w, C, K, W, P, H;
    int prune, has_prior;
    float scale, c_log2;                            // 1/sqrt(d); log2(e)/sqrt(d)
    float lambda[FS_MAX_HEADS];
    float inv2sigma[FS_MAX_HEADS];
};

__device__ __forceinline__ void rr_sync() {
    asm volatile("bar.sync %0, %1;" ::"n"(kSelBarrier), "n"(128) : "memory");
}

// U: the ordered union of the admitted sets (eq. (8)) of prefixes n_min .. n_max, built by
// the 128 row threads (eight consecutive cells per thread per round, one block-wide scan);
// also each member's admission bits per prefix, its a_c, and the per-prefix admission
// words.  Returns |U| (capped at UM; larger unions raise the device flag).
template <int UM>
__device__ int build_union(RrSmem<UM> &sm, const RrArgs &A, const int *ex, const float *am, int n_min,
                           int n_max, int t, int warp, int lane, int *dev_flag) {
    const int ng = n_max - n_min;   // <= 4
    int total = 0;
    for (int c0 = 0; c0 < n_max; c0 += 1024) {
        const int cb = c0 + 8 * t;
        int e8[8];
#pragma unroll
        for (int j = 0; j < 8; j++) e8[j] = (A.prune && cb + j < n_max) ? __ldg(ex + cb + j) : 0;
        uint32_t amk[8];
        int cnt = 0;
#pragma unroll
        for (int j = 0; j < 8; j++) {
            const int c = cb + j;
            amk[j] = 0;
#pragma unroll
            for (int g = 0; g <= 4; g++) {
                const int n = n_min + g;
                if (g <= ng && c < n && (!A.prune || c >= n - A.W || n < e8[j])) amk[j] |= 1u << g;
            }
            cnt += amk[j] != 0;
        }
        int incl = cnt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(kFull, incl, o);
            if (lane >= o) incl += y;
        }
        if (lane == 31) sm.warp_cnt[warp] = incl;
        rr_sync();
        int pos = total + incl - cnt, tot = 0;
        for (int k = 0; k < 4; k++) {
            if (k < warp) pos += sm.warp_cnt[k];
            tot += sm.warp_cnt[k];
        }
#pragma unroll
        for (int j = 0; j < 8; j++) {
            if (amk[j]) {
                if (pos < UM) {
                    sm.ulist[pos] = cb + j;
                    sm.amask[pos] = (uint8_t)amk[j];
                    sm.acell[pos] = A.has_prior ? __ldg(am + cb + j) : 0.f;
                }
                pos++;
            }
        }
        total += tot;
        rr_sync();
    }
    const int nU = min(total, UM);
    if (t == 0) {
        sm.nU = nU;
        if (total > UM && dev_flag) atomicExch(dev_flag, kFlagCheck);
    }
    constexpr int NW = (UM + 31) / 32;
    const uint32_t amk = t < nU ? sm.amask[t] : 0u;
#pragma unroll
    for (int g = 0; g < 5; g++) {
        const uint32_t word = __ballot_sync(kFull, (amk >> g) & 1u);
        if (lane == 0 && warp < NW) sm.admit[g][warp] = word;
    }
    rr_sync();
    return nU;
}

template <bool PRIOR, int UM>
__global__ void __launch_bounds__(NTHREADS, 2)
rerank_tc_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk32, const RrArgs A,
                 const float *__restrict__ amax, const int *__restrict__ exitn, int32_t *__restrict__ idx,
                 uint32_t *__restrict__ tiles, int *dev_flag) {
    extern __shared__ uint8_t smraw[];
    const uint32_t sbase = tc::smem_u32(smraw);
    RrSmem<UM> &sm = *reinterpret_cast<RrSmem<UM> *>(smraw + (((sbase + 1023u) & ~1023u) - sbase));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int bh = blockIdx.y, h = bh % A.H;
    const int r0 = blockIdx.x * BM;
    const int pb = A.q0 + r0;
    const int nrows = min(BM, A.Nq - r0);
    const int n_min = cand_count(pb, A.w, A.C);
    const int n_max = cand_count(pb + nrows - 1, A.w, A.C);
    const tc::Abort ab{dev_flag, &sm.abort};

    if (threadIdx.x == 0) {
        sm.abort = 0;
        tc::mbar_init(&sm.q_full, 1);
        tc::mbar_init(&sm.u_ready, 128);
        tc::mbar_init(&sm.drain, 1);
        for (int b = 0; b < 2; b++) {
            tc::mbar_init(&sm.s_full[b], 1);
            tc::mbar_init(&sm.s_free[b], NSEL);        // one arrival per row warp
        }
        for (int s = 0; s < NSTAGE; s++) {
            tc::mbar_init(&sm.kv_full[s], 1);
            tc::mbar_init(&sm.kv_empty[s], 1);
        }
        tc::fence_barrier_init();
    }
    if (warp == W_MMA) {
        tc::tmem_alloc(&sm.tmem_base, TMEM_COLS);
        tc::tmem_relinquish();
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem = sm.tmem_base;

    if (warp == W_TMA) {
        if (lane == 0) {
            tc::prefetch_tmap(&tq);
            tc::prefetch_tmap(&tk32);
            tc::mbar_expect_tx(&sm.q_full, TILE_BYTES);
            tc::tma_load_3d(sm.q, &tq, &sm.q_full, 0, r0, bh);
            int it = 0;
            if (tc::mbar_wait(&sm.u_ready, 0, ab)) {
                const int nU = sm.nU, nR = (nU + CPC - 1) / CPC;
                for (; it < nR; it++) {
                    const int s = it % NSTAGE;
                    if (!tc::mbar_wait(&sm.kv_empty[s], ((it / NSTAGE) & 1) ^ 1, ab)) break;
                    tc::mbar_expect_tx(&sm.kv_full[s], CPC * CELL_BYTES);
                    for (int j = 0; j < CPC; j++) {
                        const int u = CPC * it + j;
                        const int y = u < nU ? sm.ulist[u] * kS : A.Nk;   // past the end: zeros
                        tc::tma_load_3d(sm.k[s] + j * kS * kD, &tk32, &sm.kv_full[s], 0, y, bh);
                    }
                }
            }
            if (sm.abort) {   // let issued copies land before the CTA's memory is released
                for (int j = max(0, it - NSTAGE); j < it; j++) {
                    const uint64_t t0 = tc::globaltimer();
                    while (!tc::mbar_try_wait(&sm.kv_full[j % NSTAGE], (j / NSTAGE) & 1) &&
                           tc::globaltimer() - t0 < tc::kWaitLimitNs) {
                    }
                }
            }
        }
    } else if (warp == W_MMA) {
        if (lane == 0) {
            const uint32_t id_qk = tc::idesc_bf16(BM, BN, false, false);
            const uint64_t dq = tc::sdesc_sw128(tc::smem_u32(sm.q), 16, 1024);
            const uint64_t dk0 = tc::sdesc_sw128(tc::smem_u32(sm.k[0]), 16, 1024);
            constexpr uint32_t kStageStep = (BN * kD * 2) >> 4;
            bool ok = tc::mbar_wait(&sm.u_ready, 0, ab) && tc::mbar_wait(&sm.q_full, 0, ab);
            const int nR = ok ? (sm.nU + CPC - 1) / CPC : 0;
            int issued = 0;
            for (int c = 0; ok && c < nR; c++) {
                // buffer c mod 2 is free once the row threads have read chunk c - 2
                if (c >= 2 && !tc::mbar_wait(&sm.s_free[c & 1], ((c - 2) >> 1) & 1, ab)) { ok = false; break; }
                if (!tc::mbar_wait(&sm.kv_full[c % NSTAGE], (c / NSTAGE) & 1, ab)) { ok = false; break; }
                tc::tc_fence_after();
                const uint64_t db = dk0 + (uint64_t)((c % NSTAGE) * kStageStep);
#pragma unroll
                for (int kk = 0; kk < kD / 16; kk++)          // K steps of 16 columns = 32 bytes
                    tc::mma_ss(tmem + BN * (c & 1), dq + 2 * kk, db + 2 * kk, id_qk, kk > 0 ? 1u : 0u);
                tc::mma_commit(&sm.s_full[c & 1]);
                tc::mma_commit(&sm.kv_empty[c % NSTAGE]);
                issued++;
            }
            if (issued) {
                tc::mma_commit(&sm.drain);
                const uint64_t t0 = tc::globaltimer();
                while (!tc::mbar_try_wait(&sm.drain, 0) && tc::globaltimer() - t0 < tc::kWaitLimitNs) {
                }
            }
        }
    } else {
        const int t = threadIdx.x;                    // 0..127: union builder, then row t
        const int nU = build_union<UM>(sm, A, exitn + (size_t)bh * A.C, amax + (size_t)bh * A.C, n_min, n_max,
                                       t, warp, lane, dev_flag);
        tc::mbar_arrive(&sm.u_ready);
        const int nR = (nU + CPC - 1) / CPC;
        const int row = t, i = pb + row;
        const uint32_t trow = tmem + ((uint32_t)(warp * 32) << 16);
        const float lam = PRIOR ? A.lambda[h] : 0.f, i2s = PRIOR ? A.inv2sigma[h] : 0.f;
        bool ok = true;
        for (int it = 0; it < nR; it++) {
            if (!tc::mbar_wait(&sm.s_full[it & 1], (it >> 1) & 1, ab)) { ok = false; break; }
            tc::tc_fence_after();
            uint32_t sv[BN];
            tc::tmem_ld32(trow + BN * (it & 1), *reinterpret_cast<uint32_t(*)[32]>(&sv[0]));
            tc::tmem_ld32(trow + BN * (it & 1) + 32, *reinterpret_cast<uint32_t(*)[32]>(&sv[32]));
            tc::tmem_wait_ld();
            tc::tc_fence_before();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&sm.s_free[it & 1]);
#pragma unroll
            for (int b = 0; b < CPC; b++) {           // one cell: log-sum-exp of its 32 scores
                const int u = CPC * it + b;
                float a[4];
#pragma unroll
                for (int k = 0; k < 4; k++) a[k] = __uint_as_float(sv[32 * b + k]);
#pragma unroll
                for (int j = 4; j < 32; j += 2)
                    a[(j >> 1) & 3] = tc::max3(a[(j >> 1) & 3], __uint_as_float(sv[32 * b + j]),
                                               __uint_as_float(sv[32 * b + j + 1]));
                const float mx = fmaxf(fmaxf(a[0], a[1]), fmaxf(a[2], a[3]));
                const float nb = -mx * A.c_log2;
                const uint64_t c2 = tc::f2_pack(A.c_log2, A.c_log2), nb2 = tc::f2_pack(nb, nb);
                uint64_t ls[4];
#pragma unroll
                for (int k = 0; k < 4; k++) ls[k] = tc::f2_pack(0.f, 0.f);
#pragma unroll
                for (int e = 0; e < 16; e++) {
                    float x0, x1;
                    tc::f2_unpack(tc::f2_fma(tc::f2_pack(__uint_as_float(sv[32 * b + 2 * e]),
                                                         __uint_as_float(sv[32 * b + 2 * e + 1])), c2, nb2), x0, x1);
                    ls[e & 3] = tc::f2_add(ls[e & 3], tc::f2_pack(tc::ex2(x0), tc::ex2(x1)));
                }
                float s0, s1;
                tc::f2_unpack(tc::f2_add(tc::f2_add(ls[0], ls[1]), tc::f2_add(ls[2], ls[3])), s0, s1);
                float r = mx * A.scale + __logf(s0 + s1);
                if (u < nU) {
                    if (PRIOR) {
                        const float pc = (float)(sm.ulist[u] * kS) + 0.5f * kS;
                        r += lam * sm.acell[u] * erff(((float)i - pc) * i2s);
                    }
                    sm.rt[row][u] = r;
                }
            }
        }
        if (ok) {
            // this row's admitted positions -> keys -> the K best
            const int g = cand_count(i, A.w, A.C) - n_min;
            constexpr int NW = (UM + 31) / 32;
            uint32_t aw[NW];
#pragma unroll
            for (int b = 0; b < NW; b++) aw[b] = (row < nrows && g >= 0 && g <= 4) ? sm.admit[g][b] : 0u;
            int na = 0;
#pragma unroll
            for (int b = 0; b < NW; b++) na += __popc(aw[b]);
            // keys: the score as a 24-bit fixed-point fraction of this row's range of
            // admitted scores (resolution about one float ulp), then (127 - position):
            // unique, ordered by score and, between equal scores, by the lower cell
            float rmin = INFINITY, rmax = -INFINITY;
#pragma unroll
            for (int u = 0; u < UM; u++)
                if (u < nU && ((aw[u >> 5] >> (u & 31)) & 1u)) {
                    rmin = fminf(rmin, sm.rt[row][u]);
                    rmax = fmaxf(rmax, sm.rt[row][u]);
                }
            const float fscale = rmax > rmin ? 16777215.f / (rmax - rmin) : 0.f;
            uint32_t key[UM];
            uint32_t kmin = 0xffffffffu, kmax = 0u;
#pragma unroll
            for (int u = 0; u < UM; u++) {
                uint32_t k = 0u;
                if (u < nU && ((aw[u >> 5] >> (u & 31)) & 1u)) {
                    const uint32_t fx = (uint32_t)fminf((sm.rt[row][u] - rmin) * fscale, 16777215.f);
                    k = ((fx + 1u) << 7) | (uint32_t)(127 - u);
                    kmin = min(kmin, k);
                    kmax = max(kmax, k);
                }
                key[u] = k;
            }
            uint32_t tau = 1u;                        // selected: key >= tau (key 0: not admitted)
            if (na > A.K) {
                // bisection keeps count(key >= lo) >= K > count(key >= hi) and stops once the
                // bracket pins the K-th key to within one key; one pass then gives tau
                uint32_t lo = kmin, hi = kmax + 1u;
                int clo = na, chi = 0;
                while (clo > A.K + 1 && chi < A.K - 1 && hi - lo > 1u) {
                    const uint32_t mid = lo + ((hi - lo) >> 1);
                    int cp[4] = {0, 0, 0, 0};
#pragma unroll
                    for (int u = 0; u < UM; u++) cp[u & 3] += key[u] >= mid;
                    const int cnt = (cp[0] + cp[1]) + (cp[2] + cp[3]);
                    if (cnt >= A.K) {
                        lo = mid;
                        clo = cnt;
                    } else {
                        hi = mid;
                        chi = cnt;
                    }
                }
                if (clo == A.K) {
                    tau = lo;
                } else if (clo == A.K + 1) {          // the (K+1)-th key is the smallest >= lo
                    uint32_t m = 0xffffffffu;
#pragma unroll
                    for (int u = 0; u < UM; u++) m = key[u] >= lo ? min(m, key[u]) : m;
                    tau = m + 1u;
                } else {                               // count(key >= hi) = K - 1
                    uint32_t m = 0u;
#pragma unroll
                    for (int u = 0; u < UM; u++) m = key[u] < hi ? max(m, key[u]) : m;
                    tau = m;
                }
            }
            uint32_t mw[4] = {0u, 0u, 0u, 0u};        // selected union positions of this row
#pragma unroll
            for (int u = 0; u < UM; u++)
                if (key[u] >= tau && key[u] != 0u) mw[u >> 5] |= 1u << (u & 31);
            if (tiles) {   // compact record for the fused kernel: row masks | union | |U|
                uint32_t *rec = tiles + ((size_t)bh * gridDim.x + blockIdx.x) * kTileRecWords;
                *reinterpret_cast<uint4 *>(rec + kTileMaskOff + 4 * row) = make_uint4(mw[0], mw[1], mw[2], mw[3]);
                rec[kTileUlistOff + t] = t < nU ? (uint32_t)sm.ulist[t] : 0xffffffffu;
                rec[kTileMrefOff + row] = 0x7fc00000u;    // no reference: running maximum
                if (t == 0) rec[kTileCountOff] = (uint32_t)nU;
            }
            if (idx && row < nrows) {
                int32_t *out = idx + ((size_t)bh * A.Nq + r0 + row) * A.K;
                int o = 0;
#pragma unroll
                for (int u = 0; u < UM; u++)
                    if (((mw[u >> 5] >> (u & 31)) & 1u) && o < A.K) out[o++] = sm.ulist[u];
                for (; o < A.K; o++) out[o] = -1;
            }
        }
    }

    tc::tc_fence_before();
    __syncthreads();
    if (warp == W_MMA) {
        tc::tc_fence_after();
        tc::tmem_dealloc(tmem, TMEM_COLS);
    }
}

template <int UM>
cudaError_t launch_rr_um(const CUtensorMap &tq, const CUtensorMap &tk, const RrArgs &A, bool prior, dim3 grid,
                         const float *amax, const int *exitn, int32_t *idx, uint32_t *tiles, int *dev_flag,
                         cudaStream_t st) {
    const size_t smem = sizeof(RrSmem<UM>) + 1024;
    auto kern = prior ? rerank_tc_kernel<true, UM> : rerank_tc_kernel<false, UM>;
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    kern<<<grid, NTHREADS, smem, st>>>(tq, tk, A, amax, exitn, idx, tiles, dev_flag);
    return cudaGetLastError();
}
}  // namespace

// the tensor-core rerank takes bf16 inputs, every cell of A_i (no shortlist) and unions of
// at most 128 cells per tile (W + P + 10 with pruning, else every cell)
bool rerank_tc_supported(const fs_params *p, int shortlist) {
    if (p->dtype != FS_BF16) return false;
    const int C = p->Nk / p->s;
    const int admit = p->W >= 0 ? p->W + p->P : C;
    if (shortlist > 0 && shortlist < admit) return false;
    const int bound = p->W >= 0 ? p->W + p->P + 10 : C;
    return bound <= 128 && C <= 32768;
}

cudaError_t launch_rerank_tc(const Dev &P, const void *Q, const void *K, const float *amax, const int *exitn,
                             int32_t *idx, uint32_t *tiles, int *dev_flag, cudaStream_t st) {
    if (P.Nq == 0) return cudaSuccess;
    const int BH = P.B * P.H;
    CUtensorMap tq, tk32;
    if (!encode_tmap_3d_bf16(&tq, Q, kD, P.Nq, BH, kD, BM) || !encode_tmap_3d_bf16(&tk32, K, kD, P.Nk, BH, kD, kS))
        return cudaErrorInvalidValue;
    RrArgs A;
    A.Nq = P.Nq; A.Nk = P.Nk; A.q0 = P.q0; A.w = P.w; A.C = P.C; A.K = P.K;
    A.W = P.W; A.P = P.P; A.H = P.H; A.prune = P.prune; A.has_prior = P.has_prior;
    A.scale = P.scale;
    A.c_log2 = P.scale * 1.4426950408889634f;
    for (int hh = 0; hh < FS_MAX_HEADS; hh++) {
        A.lambda[hh] = P.lambda[hh];
        A.inv2sigma[hh] = P.inv2sigma[hh];
    }
    const dim3 grid((P.Nq + BM - 1) / BM, BH);
    const int bound = P.prune ? P.W + P.P + 10 : P.C;
    LaunchScope scope(kRerankTc, st);
    if (bound <= 80) return launch_rr_um<80>(tq, tk32, A, P.has_prior, grid, amax, exitn, idx, tiles, dev_flag, st);
    return launch_rr_um<128>(tq, tk32, A, P.has_prior, grid, amax, exitn, idx, tiles, dev_flag, st);
}

}  // namespace fs
