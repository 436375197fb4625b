// Local RoPE branch on the 5th-generation tensor cores, and the range combination,
// "FreeSolo" summary §3.2 eqs. (3)-(4) and §3.1 eq. (2) (bf16 inputs):
//   o_i^sr = softmax_{j in [i-w, i]}((R(i)q_i).(R(j)k_j) / sqrt(d)) V,
//   O_i    = o_i^sr + alpha_h o_i^lr        (alpha_h o_i^lr precomputed by the readout).
//
// One CTA per 128 query rows of a (batch, head); two CTAs share an SM.  Warp roles:
//   0-3  softmax: one query row per thread (its TMEM lane)
//   4    TMA: the Q tile once, then 128-key chunks of K and V (3-D maps, zero fill
//        outside [0, Nk)), two stages
//   5    MMA: S = Q K^T (M=128, N=128, K=64) into TMEM; O += P V with P read from TMEM
//        (M=128, N=64, K=128)
//   6-9  RoPE: rotate Q and each K chunk in shared memory (128-byte-swizzled layout the
//        TMA wrote), angles taken from the tile's first query position: by eq. (3) only
//        j - i matters, and offsets of at most w + 128 keep the angles exact.
// Per chunk: S lands in TMEM columns [0,128); the softmax threads take the row max over
// the band [i-w, i], rescale O in TMEM only when the max grows by more than 2^8 (lazy
// rescale), write P = exp2(S*scale*log2e - m) as bf16 pairs over S's first 64 columns,
// and the next MMA accumulates P V into O (columns [128,192)).  MMAs issued by one
// thread run in order, so the next S never overwrites P before P V has read it.
#include "tc_rope.cuh"

namespace fs {

namespace {
constexpr int BM = 128, BN = 128;
constexpr int NSTAGE = 2;
constexpr int W_TMA = 4, W_MMA = 5, W_ROT0 = 6, NWARPS = 10;
constexpr int NTHREADS = NWARPS * 32;
constexpr uint32_t TMEM_COLS = 256, S_COL = 0, O_COL = 128;
constexpr int TILE_BYTES = BM * kD * 2;      // one 128 x 64 bf16 box: 16 KiB

struct WinSmem {
    __nv_bfloat16 q[BM * kD];
    __nv_bfloat16 k[NSTAGE][BN * kD];
    __nv_bfloat16 v[NSTAGE][BN * kD];
    uint64_t q_full, q_ready, s_full, p_full, o_done, drain;
    uint64_t kv_full[NSTAGE], k_ready[NSTAGE], kv_empty[NSTAGE];
    uint32_t tmem_base;
    int abort;
};

struct WinArgs {
    int Nq, Nk, q0, w;
    float scale_log2e;       // log2(e) / sqrt(d)
    int rope_nb;             // rows of the chunk-base angle table
};

__device__ __forceinline__ bool in_band(int c, int clo, int chi) { return c >= clo && c <= chi; }
}  // namespace

__global__ void __launch_bounds__(NTHREADS, 2)
window_tc_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                 const __grid_constant__ CUtensorMap tv, const WinArgs A,
                 const float2 *__restrict__ rope_t, const float2 *__restrict__ rope_b,
                 const float *__restrict__ olr, __nv_bfloat16 *__restrict__ O, int *dev_flag) {
    extern __shared__ uint8_t smraw[];
    const uint32_t sbase = tc::smem_u32(smraw);
    WinSmem &sm = *reinterpret_cast<WinSmem *>(smraw + (((sbase + 1023u) & ~1023u) - sbase));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int bh = blockIdx.y;
    const int r0 = blockIdx.x * BM;
    const int pb = A.q0 + r0;                       // position of the tile's first query
    const int nrows = min(BM, A.Nq - r0);
    const int jbase = pb - A.w;                     // first key of chunk 0
    const int last = pb + nrows - 1;                // last key any row needs
    const int k_first = jbase < 0 ? (-jbase) / BN : 0;
    const int k_last = (last - jbase) / BN;
    const int nck = k_last - k_first + 1;
    const tc::Abort ab{dev_flag, &sm.abort};

    if (threadIdx.x == 0) {
        sm.abort = 0;
        tc::mbar_init(&sm.q_full, 1);
        tc::mbar_init(&sm.q_ready, 128);
        tc::mbar_init(&sm.s_full, 1);
        tc::mbar_init(&sm.p_full, 128);
        tc::mbar_init(&sm.o_done, 1);
        tc::mbar_init(&sm.drain, 1);
        for (int s = 0; s < NSTAGE; s++) {
            tc::mbar_init(&sm.kv_full[s], 1);
            tc::mbar_init(&sm.k_ready[s], 128);
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
            tc::prefetch_tmap(&tk);
            tc::prefetch_tmap(&tv);
            tc::mbar_expect_tx(&sm.q_full, TILE_BYTES);
            tc::tma_load_3d(sm.q, &tq, &sm.q_full, 0, r0, bh);
            int it = 0;
            for (; it < nck; it++) {
                const int s = it % NSTAGE;
                if (!tc::mbar_wait(&sm.kv_empty[s], ((it / NSTAGE) & 1) ^ 1, ab)) break;
                const int jc = jbase + BN * (k_first + it);
                tc::mbar_expect_tx(&sm.kv_full[s], 2 * TILE_BYTES);
                tc::tma_load_3d(sm.k[s], &tk, &sm.kv_full[s], 0, jc, bh);
                tc::tma_load_3d(sm.v[s], &tv, &sm.kv_full[s], 0, jc, bh);
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
    } else if (warp >= W_ROT0) {
        const int t = threadIdx.x - W_ROT0 * 32;
        if (tc::mbar_wait(&sm.q_full, 0, ab)) {
            tc::rotate_tile<128>(sm.q, sm.q, t, rope_t, nullptr);
            tc::fence_async_shared();
            tc::mbar_arrive(&sm.q_ready);
            for (int it = 0; it < nck; it++) {
                const int s = it % NSTAGE;
                if (!tc::mbar_wait(&sm.kv_full[s], (it / NSTAGE) & 1, ab)) break;
                tc::rotate_tile<128>(sm.k[s], sm.k[s], t, rope_t, rope_b + (size_t)(k_first + it) * 32);
                tc::fence_async_shared();
                tc::mbar_arrive(&sm.k_ready[s]);
            }
        }
    } else if (warp == W_MMA) {
        if (lane == 0) {
            const uint32_t id_qk = tc::idesc_bf16(BM, BN, false, false);
            const uint32_t id_pv = tc::idesc_bf16(BM, kD, false, true);
            const uint32_t qa = tc::smem_u32(sm.q);
            bool ok = tc::mbar_wait(&sm.q_ready, 0, ab);
            int issued = 0;
            for (int it = 0; ok && it <= nck; it++) {
                if (it < nck && !tc::mbar_wait(&sm.k_ready[it % NSTAGE], (it / NSTAGE) & 1, ab)) {
                    ok = false;
                    break;
                }
                if (it > 0) {   // O += P(it-1) V(it-1)
                    if (!tc::mbar_wait(&sm.p_full, (it - 1) & 1, ab)) { ok = false; break; }
                    tc::tc_fence_after();
                    const uint32_t vb = tc::smem_u32(sm.v[(it - 1) % NSTAGE]);
#pragma unroll
                    for (int kk = 0; kk < BN / 16; kk++)
                        tc::mma_ts(tmem + O_COL, tmem + S_COL + kk * 8,
                                   tc::sdesc_sw128(vb + kk * 2048, 16, 1024), id_pv,
                                   (it - 1 > 0 || kk > 0) ? 1u : 0u);
                    tc::mma_commit(&sm.kv_empty[(it - 1) % NSTAGE]);
                    issued++;
                }
                if (it < nck) {   // S = Q K(it)^T
                    tc::tc_fence_after();
                    const uint32_t kb = tc::smem_u32(sm.k[it % NSTAGE]);
#pragma unroll
                    for (int kk = 0; kk < kD / 16; kk++)
                        tc::mma_ss(tmem + S_COL, tc::sdesc_sw128(qa + kk * 32, 16, 1024),
                                   tc::sdesc_sw128(kb + kk * 32, 16, 1024), id_qk, kk > 0 ? 1u : 0u);
                    tc::mma_commit(&sm.s_full);
                    issued++;
                }
            }
            if (ok) tc::mma_commit(&sm.o_done);
            if (issued) {   // every MMA has finished before the tensor memory is released
                tc::mma_commit(&sm.drain);
                const uint64_t t0 = tc::globaltimer();
                while (!tc::mbar_try_wait(&sm.drain, 0) && tc::globaltimer() - t0 < tc::kWaitLimitNs) {
                }
            }
        }
    } else {
        // ---- softmax: thread = query row (TMEM lane warp*32 + lane)
        const int row = warp * 32 + lane;
        const int i = pb + row;
        const bool rvalid = row < nrows;
        const uint32_t trow = tmem + ((uint32_t)(warp * 32) << 16);
        float m_used = -INFINITY, l = 0.f;
        bool ok = true;
        for (int it = 0; it < nck; it++) {
            if (!tc::mbar_wait(&sm.s_full, it & 1, ab)) { ok = false; break; }
            tc::tc_fence_after();
            const int jc = jbase + BN * (k_first + it);
            int clo = max(-jc, i - A.w - jc), chi = min(i - jc, BN - 1);
            if (!rvalid) { clo = 1; chi = 0; }
            float mx = -INFINITY;
#pragma unroll
            for (int b = 0; b < BN / 32; b++) {
                uint32_t r[32];
                tc::tmem_ld32(trow + S_COL + 32 * b, r);
                tc::tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 32; e++)
                    if (in_band(32 * b + e, clo, chi)) mx = fmaxf(mx, __uint_as_float(r[e]));
            }
            mx *= A.scale_log2e;
            const bool grow = mx > m_used + 8.f;
            const float m_new = grow ? mx : m_used;
            const float corr = (grow && m_used != -INFINITY) ? tc::ex2(m_used - m_new) : 1.f;
            if (it > 0 && __any_sync(kFull, corr != 1.f)) {
#pragma unroll
                for (int b = 0; b < kD / 32; b++) {
                    uint32_t r[32];
                    tc::tmem_ld32(trow + O_COL + 32 * b, r);
                    tc::tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; e++) r[e] = __float_as_uint(__uint_as_float(r[e]) * corr);
                    tc::tmem_st32(trow + O_COL + 32 * b, r);
                }
                tc::tmem_wait_st();
            }
            l *= corr;
            m_used = m_new;
            const float msub = m_used == -INFINITY ? 0.f : m_used;
#pragma unroll
            for (int h2 = 0; h2 < 2; h2++) {
                uint32_t pk[32];
#pragma unroll
                for (int hb = 0; hb < 2; hb++) {
                    const int b = 2 * h2 + hb;
                    uint32_t r[32];
                    tc::tmem_ld32(trow + S_COL + 32 * b, r);
                    tc::tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 16; e++) {
                        const int c0 = 32 * b + 2 * e;
                        const float p0 = in_band(c0, clo, chi)
                                             ? tc::ex2(__uint_as_float(r[2 * e]) * A.scale_log2e - msub) : 0.f;
                        const float p1 = in_band(c0 + 1, clo, chi)
                                             ? tc::ex2(__uint_as_float(r[2 * e + 1]) * A.scale_log2e - msub) : 0.f;
                        l += p0 + p1;
                        pk[16 * hb + e] = tc::pack_bf16x2(p0, p1);
                    }
                }
                tc::tmem_st32(trow + S_COL + 32 * h2, pk);   // P keys [64 h2, 64 h2 + 64)
            }
            tc::tmem_wait_st();
            tc::tc_fence_before();
            tc::mbar_arrive(&sm.p_full);
        }
        if (ok && tc::mbar_wait(&sm.o_done, 0, ab)) {
            tc::tc_fence_after();
            uint32_t r[2][32];
            tc::tmem_ld32(trow + O_COL, r[0]);
            tc::tmem_ld32(trow + O_COL + 32, r[1]);
            tc::tmem_wait_ld();
            if (rvalid) {
                const size_t orow = ((size_t)bh * A.Nq + r0 + row) * kD;
                const float inv = 1.f / l;
                uint32_t outw[32];
#pragma unroll
                for (int e = 0; e < 32; e++) {
                    float o0 = __uint_as_float(r[e >> 4][(2 * e) & 31]) * inv;
                    float o1 = __uint_as_float(r[e >> 4][(2 * e + 1) & 31]) * inv;
                    if (olr) {
                        const float2 x = __ldg(reinterpret_cast<const float2 *>(olr + orow) + e);
                        o0 += x.x;
                        o1 += x.y;
                    }
                    outw[e] = tc::pack_bf16x2(o0, o1);
                }
                uint4 *dst = reinterpret_cast<uint4 *>(O + orow);
#pragma unroll
                for (int e = 0; e < 8; e++)
                    dst[e] = make_uint4(outw[4 * e], outw[4 * e + 1], outw[4 * e + 2], outw[4 * e + 3]);
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

// Angle tables for the window kernel, in double precision:
//   rope_t[t][m] = (cos, sin)(t theta_m),            t in [0, 128)
//   rope_b[k][m] = (cos, sin)((128 k - w) theta_m),  k in [0, nb)
__global__ void rope_table_kernel(float2 *rope_t, float2 *rope_b, int nb, int w, double base) {
    const int idx = blockIdx.x * blockDim.x + threadIdx.x;
    const int m = idx & 31, row = idx >> 5;
    if (row >= BM + nb) return;
    const double theta = pow(base, -2.0 * m / (double)kD);
    const double ang = (row < BM ? (double)row : (double)(128 * (row - BM) - w)) * theta;
    double s, c;
    sincos(ang, &s, &c);
    const float2 v = make_float2((float)c, (float)s);
    if (row < BM) rope_t[row * 32 + m] = v;
    else rope_b[(row - BM) * 32 + m] = v;
}

int rope_table_rows(int w) { return (w + BN - 1) / BN + 2; }

size_t window_tc_smem() { return sizeof(WinSmem) + 1024; }

cudaError_t launch_rope_table(int w, float rope_base, float2 *rope_t, float2 *rope_b, cudaStream_t st) {
    const int nb = rope_table_rows(w);
    const int n = (BM + nb) * 32;
    LaunchScope scope(kRopeTable, st);
    rope_table_kernel<<<(n + 255) / 256, 256, 0, st>>>(rope_t, rope_b, nb, w, (double)rope_base);
    return cudaGetLastError();
}

cudaError_t launch_window_tc(const Dev &P, const void *Q, const void *K, const void *V,
                             const float *olr, void *O, const float2 *rope_t, const float2 *rope_b,
                             int *dev_flag, cudaStream_t st) {
    if (P.Nq == 0) return cudaSuccess;
    const int BH = P.B * P.H;
    CUtensorMap tq, tk, tv;
    if (!encode_tmap_3d_bf16(&tq, Q, kD, P.Nq, BH, kD, BM) ||
        !encode_tmap_3d_bf16(&tk, K, kD, P.Nk, BH, kD, BN) ||
        !encode_tmap_3d_bf16(&tv, V, kD, P.Nk, BH, kD, BN))
        return cudaErrorInvalidValue;
    WinArgs A;
    A.Nq = P.Nq; A.Nk = P.Nk; A.q0 = P.q0; A.w = P.w;
    A.scale_log2e = P.scale * 1.4426950408889634f;
    A.rope_nb = rope_table_rows(P.w);
    const size_t smem = window_tc_smem();
    const dim3 grid((P.Nq + BM - 1) / BM, BH);
    LaunchScope scope(kWindowTc, st);
    cudaFuncSetAttribute(window_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    window_tc_kernel<<<grid, NTHREADS, smem, st>>>(tq, tk, tv, A, rope_t, rope_b, olr,
                                                   (__nv_bfloat16 *)O, dev_flag);
    return cudaGetLastError();
}

}  // namespace fs
