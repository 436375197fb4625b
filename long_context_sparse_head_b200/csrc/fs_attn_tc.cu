// Fused long-range readout + local window + combination on the 5th-generation tensor
// cores (bf16), "FreeSolo" summary §3.3 eq. (9), §3.2 eqs. (3)-(4), §3.1 eq. (2):
//   u_i    = softmax_{tokens of the cells in S_i}(q_i.k_j / sqrt(d)) V        (NoPE)
//   o_i^lr = RMSNorm(u_i)
//   o_i^sr = softmax_{j in [i-w, i]}((R(i)q_i).(R(j)k_j) / sqrt(d)) V       (RoPE)
//   O_i    = o_i^sr + alpha_h o_i^lr
// with S_i given by the selection kernel's per-tile record (union U of the tile's
// admitted cells and, per row, the positions in U it selected).
//
// One CTA per 128 query rows of a (batch, head); two CTAs per SM.  The readout runs over
// U (|U| <= 128, ascending), two cells (64 keys) per chunk, each cell fetched by its own
// 32-row TMA box; a row masks the cells it did not select (masked-dense on the tensor
// cores).  The readout's exponent reference is the row's bound from the record (an upper
// bound of its logits within 96 of their maximum, so every P is at most 1 and none
// underflows): no running maximum, no rescaling.  Then the window runs over 64-key chunks
// with a fixed reference or a running maximum.  Both softmaxes accumulate in tensor
// memory: three S buffers in columns [0,64), [64,128) and [128,192) (chunk c uses buffer
// c mod 3, and its P overwrites the first 32 columns of that buffer) and one O in
// [192,256).  The MMA warp keeps Q K^T two chunks ahead of P V, so a softmax warp that
// finishes early finds the next S ready while slower warps finish this chunk.  When the
// first window chunk arrives the readout is finished: the softmax threads read its O,
// keep alpha_h * RMSNorm(u) in registers (fp32), and the window's first P V overwrites O;
// the epilogue adds the two.  No intermediate leaves the SM.  The window, like the readout,
// subtracts a fixed per-row reference where one exists (|q_i| times the largest key norm
// of the band's cells, within 96 of the row's own logit), computed by the auxiliary warps
// while the readout runs; otherwise it keeps a running maximum with lazy rescaling.
//
// Warpgroup 0 (warps 0-3): softmax, thread = query row = TMEM lane; it holds a chunk's
// S row in registers (one TMEM wait per chunk), raised to 200 registers by setmaxnreg.
// Warpgroup 1 (lowered to 56): warp 4 TMA, warp 5 MMA, warps 6-7 auxiliary (stage U,
// rotate Q by its absolute positions).  The window's keys come pre-rotated (absolute
// positions, double-precision angles) from a workspace copy.
#include <algorithm>
#include <cstddef>

#include "tc_rope.cuh"

namespace fs {

namespace {
constexpr int BM = 128, BN = 64, NSTAGE = 4;
constexpr int UMAX = 128;                        // largest union of selected cells per tile
constexpr int CPC = BN / kS;                     // cells per readout chunk (2)
constexpr int NSOFT = 4, W_TMA = 4, W_MMA = 5, W_AUX0 = 6, NWARPS = 8, NAUX = 64;
constexpr int NTHREADS = NWARPS * 32;
constexpr int REGS_SOFTMAX = 200, REGS_PRODUCER = 56;   // 128 * (200 + 56) = 256 * 128
constexpr int NSBUF = 3;                        // S buffers (BN columns each) in tensor memory
constexpr uint32_t TMEM_COLS = 256, O_COL = NSBUF * BN;   // S at 0, BN, 2 BN; O at 192
constexpr int TILE_BYTES = BM * kD * 2;         // 128 x 64 bf16: 16 KiB
constexpr int CHUNK_BYTES = BN * kD * 2;        // 64 x 64 bf16: 8 KiB
constexpr int CELL_BYTES = kS * kD * 2;         // 32 x 64 bf16: 4 KiB
constexpr int kAuxBarrier = 1;                  // named barrier of the auxiliary threads

struct AttnSmem {
    __nv_bfloat16 qn[BM * kD];                  // Q as loaded (NoPE)
    __nv_bfloat16 qr[BM * kD];                  // Q rotated (RoPE)
    __nv_bfloat16 k[NSTAGE][BN * kD];
    __nv_bfloat16 v[NSTAGE][BN * kD];
    int ulist[UMAX];                            // union cells, ascending
    int nU;
    float wref[BM];                             // window reference per row (log2 units) or NaN
    float4 phead[BM];                           // split CTAs: per row (m, l) of both branches
    float amax_band;                            // largest a_c of the cells the band touches
    uint64_t q_full, q_ready, u_ready, w_ready, o_done, drain;
    uint64_t o_ready[2];                        // P V of chunk c completes phase c / 2 of [c % 2]
    uint64_t s_full[NSBUF], p_full[NSBUF];      // per S buffer
    uint64_t kv_full[NSTAGE], kv_empty[NSTAGE];
    uint32_t tmem_base;
    int abort;
};

struct AttnArgs {
    int Nq, Nk, q0, w, C, K, H;
    int kr0;                // first key of the rotated copy
    float scale_log2e;      // log2(e) / sqrt(d)
    float rms_eps;
    int nsplit;             // CTAs per tile (gridDim.z, one cluster); > 1: split and combined
    float alpha[FS_MAX_HEADS];
};

// A split CTA's partial state per row: m, l (log2 units) of the readout and the window
// (phead), then the readout's and the window's unnormalised O, 64 floats each, over the
// K / V stages (free once the last P V has completed): row r's 16-byte chunk q (0-15 the
// readout's, 16-31 the window's) at slot q ^ (r mod 8) of the row's 512 bytes, so that the
// rows a warp writes at once fall in different banks.
constexpr int kPartRowBytes = 2 * kD * 4;

__device__ __forceinline__ void aux_sync() {
    asm volatile("bar.sync %0, %1;" ::"n"(kAuxBarrier), "n"(NAUX) : "memory");
}
// Column validity of a chunk: every column (FULL), the columns of the selected cells
// (CELLS: 32-column block b valid iff bit b of sel), or a band of the window (BAND:
// lo <= j < lo + width).
enum ChunkKind { FULL = 0, CELLS = 1, BAND = 2 };

// One chunk of online softmax for this thread's row, on the S buffer at TMEM address tS
// (BN columns, read in one batch).  Invalid columns must contribute exp2(-inf) = 0: a
// BAND chunk sets them to -inf one by one; a CELLS chunk drops the 32-column block of an
// unselected cell from the max and adds an exponent bias of -inf to the whole block, so
// the exponentials of every kind of chunk share one body.  P = exp2(S*c - m) is written
// back as bf16 pairs over the buffer's first BN/2 columns.  The running max m (log2
// units) is raised only when a chunk exceeds it by more than 8 (lazy rescale of O); the
// factor O must be multiplied by is returned (1 when m stayed).  The arithmetic is paired
// (f32x2 FMA and add, three-input max) with independent partial accumulators.
__device__ __forceinline__ float softmax_chunk(uint32_t tS, int kind, uint32_t sel, int lo, int width,
                                               float c_log2, float &m_used, float &l) {
    uint32_t s[BN];
    tc::tmem_ld32(tS, *reinterpret_cast<uint32_t(*)[32]>(&s[0]));
    tc::tmem_ld32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(&s[32]));
    tc::tmem_wait_ld();
    if (kind == BAND) {
#pragma unroll
        for (int j = 0; j < BN; j++)
            if ((unsigned)(j - lo) >= (unsigned)width) s[j] = 0xff800000u;
    }
    float mx = -INFINITY;
    bool valid[BN / 32];
#pragma unroll
    for (int b = 0; b < BN / 32; b++) {           // block maximum: four three-input chains
        float a[4];
#pragma unroll
        for (int k = 0; k < 4; k++) a[k] = __uint_as_float(s[32 * b + k]);
#pragma unroll
        for (int j = 4; j < 32; j += 2)
            a[(j >> 1) & 3] = tc::max3(a[(j >> 1) & 3], __uint_as_float(s[32 * b + j]), __uint_as_float(s[32 * b + j + 1]));
        valid[b] = kind != CELLS || ((sel >> b) & 1u);
        mx = valid[b] ? tc::max3(mx, fmaxf(a[0], a[1]), fmaxf(a[2], a[3])) : mx;
    }
    mx *= c_log2;
    const bool grow = mx > m_used + 8.f;
    const float m_new = grow ? mx : m_used;
    const float corr = (grow && m_used != -INFINITY) ? tc::ex2(m_used - m_new) : 1.f;
    l *= corr;
    m_used = m_new;
    const float msub = m_used == -INFINITY ? 0.f : m_used;
    const uint64_t c2 = tc::f2_pack(c_log2, c_log2);
    uint64_t ls[4];
#pragma unroll
    for (int k = 0; k < 4; k++) ls[k] = tc::f2_pack(0.f, 0.f);
#pragma unroll
    for (int q = 0; q < BN / 32; q++) {              // P keys [32 q, 32 q + 32) -> 16 columns
        const float nb = valid[q] ? -msub : -INFINITY;
        const uint64_t nb2 = tc::f2_pack(nb, nb);
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; e++) {
            const int j = 32 * q + 2 * e;
            float x0, x1;
            tc::f2_unpack(tc::f2_fma(tc::f2_pack(__uint_as_float(s[j]), __uint_as_float(s[j + 1])), c2, nb2), x0, x1);
            const float p0 = tc::ex2(x0), p1 = tc::ex2(x1);
            ls[e & 3] = tc::f2_add(ls[e & 3], tc::f2_pack(p0, p1));
            pk[e] = tc::pack_bf16x2(p0, p1);
        }
        tc::tmem_st16(tS + 16 * q, pk);
    }
    float u, v;
    tc::f2_unpack(tc::f2_add(tc::f2_add(ls[0], ls[1]), tc::f2_add(ls[2], ls[3])), u, v);
    l += u + v;
    return corr;
}

// One readout chunk (two cells) against a fixed reference mref (log2 units, an upper
// bound of the row's logits, so every exponent is <= 0 and nothing is ever rescaled).
// Block b of 32 columns counts only if bit b of sel is set; otherwise its exponent bias is
// -inf and its P is 0.  P is written back as bf16 pairs over the buffer's first BN/2
// columns; l gathers the row sum.
__device__ __forceinline__ void softmax_chunk_fixed(uint32_t tS, uint32_t sel, float mref, float c_log2, float &l) {
    uint32_t s[BN];
    tc::tmem_ld32(tS, *reinterpret_cast<uint32_t(*)[32]>(&s[0]));
    tc::tmem_ld32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(&s[32]));
    tc::tmem_wait_ld();
    const uint64_t c2 = tc::f2_pack(c_log2, c_log2);
    uint64_t ls[4];
#pragma unroll
    for (int k = 0; k < 4; k++) ls[k] = tc::f2_pack(0.f, 0.f);
#pragma unroll
    for (int q = 0; q < BN / 32; q++) {
        const float nb = ((sel >> q) & 1u) ? -mref : -INFINITY;
        const uint64_t nb2 = tc::f2_pack(nb, nb);
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; e++) {
            const int j = 32 * q + 2 * e;
            float x0, x1;
            tc::f2_unpack(tc::f2_fma(tc::f2_pack(__uint_as_float(s[j]), __uint_as_float(s[j + 1])), c2, nb2), x0, x1);
            const float p0 = tc::ex2(x0), p1 = tc::ex2(x1);
            ls[e & 3] = tc::f2_add(ls[e & 3], tc::f2_pack(p0, p1));
            pk[e] = tc::pack_bf16x2(p0, p1);
        }
        tc::tmem_st16(tS + 16 * q, pk);
    }
    float u, v;
    tc::f2_unpack(tc::f2_add(tc::f2_add(ls[0], ls[1]), tc::f2_add(ls[2], ls[3])), u, v);
    l += u + v;
}

// One window chunk against a fixed reference (log2 units, an upper bound of the row's
// logits): a BAND chunk masks the columns outside lo <= j < lo + width with -inf, every
// exponent is then <= 0, and nothing is rescaled.  P goes to the buffer's first BN/2
// columns; l gathers the row sum.
__device__ __forceinline__ void softmax_chunk_band_fixed(uint32_t tS, int kind, int lo, int width, float ref,
                                                         float c_log2, float &l) {
    uint32_t s[BN];
    tc::tmem_ld32(tS, *reinterpret_cast<uint32_t(*)[32]>(&s[0]));
    tc::tmem_ld32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(&s[32]));
    tc::tmem_wait_ld();
    if (kind == BAND) {
#pragma unroll
        for (int j = 0; j < BN; j++)
            if ((unsigned)(j - lo) >= (unsigned)width) s[j] = 0xff800000u;
    }
    const uint64_t c2 = tc::f2_pack(c_log2, c_log2), nb2 = tc::f2_pack(-ref, -ref);
    uint64_t ls[4];
#pragma unroll
    for (int k = 0; k < 4; k++) ls[k] = tc::f2_pack(0.f, 0.f);
#pragma unroll
    for (int q = 0; q < BN / 32; q++) {
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; e++) {
            const int j = 32 * q + 2 * e;
            float x0, x1;
            tc::f2_unpack(tc::f2_fma(tc::f2_pack(__uint_as_float(s[j]), __uint_as_float(s[j + 1])), c2, nb2), x0, x1);
            const float p0 = tc::ex2(x0), p1 = tc::ex2(x1);
            ls[e & 3] = tc::f2_add(ls[e & 3], tc::f2_pack(p0, p1));
            pk[e] = tc::pack_bf16x2(p0, p1);
        }
        tc::tmem_st16(tS + 16 * q, pk);
    }
    float u, v;
    tc::f2_unpack(tc::f2_add(tc::f2_add(ls[0], ls[1]), tc::f2_add(ls[2], ls[3])), u, v);
    l += u + v;
}
}  // namespace

template <bool SPLIT>
__global__ void __launch_bounds__(NTHREADS, 2)
attn_tc_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk32,
               const __grid_constant__ CUtensorMap tv32, const __grid_constant__ CUtensorMap tkr64,
               const __grid_constant__ CUtensorMap tv64, const AttnArgs A,
               const uint32_t *__restrict__ tiles, const float2 *__restrict__ rope_lo,
               const float2 *__restrict__ rope_hi, __nv_bfloat16 *__restrict__ O, int *dev_flag,
               const __nv_bfloat16 *__restrict__ Kraw, const float *__restrict__ amax) {
    extern __shared__ uint8_t smraw[];
    const uint32_t sbase = tc::smem_u32(smraw);
    AttnSmem &sm = *reinterpret_cast<AttnSmem *>(smraw + (((sbase + 1023u) & ~1023u) - sbase));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int bh = blockIdx.y, h = bh % A.H;
    const int r0 = blockIdx.x * BM;
    const int pb = A.q0 + r0;
    const int nrows = min(BM, A.Nq - r0);
    const int jbase = pb - A.w;
    const int last = pb + nrows - 1;
    const int k_first = jbase < 0 ? (-jbase) / BN : 0;
    const int nW = (last - jbase) / BN - k_first + 1;    // window chunks
    // with nsplit > 1 this CTA takes the contiguous range [cb, ce) of the tile's chunk list
    // (readout chunks 0 .. nR-1, then window chunks nR .. nR+nW-1)
    const int S = SPLIT ? A.nsplit : 1, sidx = SPLIT ? (int)blockIdx.z : 0;
    auto chunk_range = [&](int nR, int &cb, int &ce) {
        const int T = nR + nW;
        cb = (int)((long long)T * sidx / S);
        ce = (int)((long long)T * (sidx + 1) / S);
    };
    const tc::Abort ab{dev_flag, &sm.abort};

    if (threadIdx.x == 0) {
        sm.abort = 0;
        tc::mbar_init(&sm.q_full, 1);
        tc::mbar_init(&sm.q_ready, NAUX);
        tc::mbar_init(&sm.u_ready, NAUX);
        tc::mbar_init(&sm.w_ready, NAUX);
        tc::mbar_init(&sm.o_ready[0], 1);
        tc::mbar_init(&sm.o_ready[1], 1);
        tc::mbar_init(&sm.o_done, 1);
        for (int b = 0; b < NSBUF; b++) {
            tc::mbar_init(&sm.s_full[b], 1);
            tc::mbar_init(&sm.p_full[b], NSOFT);       // one arrival per softmax warp
        }
        tc::mbar_init(&sm.drain, 1);
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
    griddep_wait();                             // the selection's tile records are complete

    if (warp >= NSOFT) {
        tc::regs_dec<REGS_PRODUCER>();
        if (warp == W_TMA) {
            if (lane == 0) {
                tc::prefetch_tmap(&tq);
                tc::prefetch_tmap(&tk32);
                tc::prefetch_tmap(&tv32);
                tc::prefetch_tmap(&tkr64);
                tc::prefetch_tmap(&tv64);
                tc::mbar_expect_tx(&sm.q_full, TILE_BYTES);
                tc::tma_load_3d(sm.qn, &tq, &sm.q_full, 0, r0, bh);
                int it = 0;
                if (tc::mbar_wait(&sm.u_ready, 0, ab)) {
                    const int nU = sm.nU, nR = (nU + CPC - 1) / CPC;
                    int cb, ce;
                    chunk_range(nR, cb, ce);
                    const int total = ce - cb;
                    for (; it < total; it++) {
                        const int s = it % NSTAGE, g = cb + it;
                        if (!tc::mbar_wait(&sm.kv_empty[s], ((it / NSTAGE) & 1) ^ 1, ab)) break;
                        if (g < nR) {           // two gathered cells; unused slots read zeros
                            tc::mbar_expect_tx(&sm.kv_full[s], 2 * CPC * CELL_BYTES);
                            for (int j = 0; j < CPC; j++) {
                                const int u = CPC * g + j;
                                const int y = u < nU ? sm.ulist[u] * kS : A.Nk;   // past the end: zeros
                                tc::tma_load_3d(sm.k[s] + j * kS * kD, &tk32, &sm.kv_full[s], 0, y, bh);
                                tc::tma_load_3d(sm.v[s] + j * kS * kD, &tv32, &sm.kv_full[s], 0, y, bh);
                            }
                        } else {                // BN consecutive keys of the band (K pre-rotated)
                            const int jc = jbase + BN * (k_first + g - nR);
                            tc::mbar_expect_tx(&sm.kv_full[s], 2 * CHUNK_BYTES);
                            tc::tma_load_3d(sm.k[s], &tkr64, &sm.kv_full[s], 0, jc - A.kr0, bh);
                            tc::tma_load_3d(sm.v[s], &tv64, &sm.kv_full[s], 0, jc, bh);
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
        } else if (warp >= W_AUX0) {
            const int t = threadIdx.x - W_AUX0 * 32;
            // ---- U and |U| from the selection kernel's record for this tile
            const uint32_t *rec = tiles + ((size_t)bh * gridDim.x + blockIdx.x) * kTileRecWords;
            for (int u = t; u < UMAX; u += NAUX) sm.ulist[u] = (int)__ldg(rec + kTileUlistOff + u);
            if (t == 0) sm.nU = min((int)__ldg(rec + kTileCountOff), UMAX);
            aux_sync();
            tc::mbar_arrive(&sm.u_ready);
            // ---- rotate Q by its absolute positions for the window
            if (tc::mbar_wait(&sm.q_full, 0, ab)) {
                const uint8_t *src = reinterpret_cast<const uint8_t *>(sm.qn);
                uint8_t *dst = reinterpret_cast<uint8_t *>(sm.qr);
#pragma unroll 2
                for (int j = 0; j < 1024 / NAUX; j++) {
                    const int item = t + NAUX * j, row = item >> 3, c = item & 7;
                    const int off = row * 128 + ((c ^ (row & 7)) << 4);   // 128-byte swizzle
                    float cs[4], sn[4];
                    rope_angles(pb + row, c, rope_lo, rope_hi, cs, sn);
                    *reinterpret_cast<uint4 *>(dst + off) =
                        rope_rotate8(*reinterpret_cast<const uint4 *>(src + off), cs, sn);
                }
                tc::fence_async_shared();
                tc::mbar_arrive(&sm.q_ready);
                // ---- window reference per row (log2 units).  Every window logit of row i is
                // at most |q_i| max_j |k_j| / sqrt(d) (Cauchy-Schwarz; rotations keep norms),
                // bounded by the largest a_c of the cells the tile's band touches; the
                // largest is at least the row's own logit q_i.k_i / sqrt(d) (key i is always
                // in its window, and R(i) cancels).  Within kMrefMaxGap the upper bound is the
                // reference; a band reaching past the last full cell (no a_c) gets none.
                const int c_lo = max(0, jbase) / kS, c_hi = (pb + nrows - 1) / kS;
                const bool band_ok = c_hi < A.C;
                if (t < 32) {
                    float am = 0.f;
                    if (band_ok)
                        for (int c = c_lo + t; c <= c_hi; c += 32) am = fmaxf(am, __ldg(amax + (size_t)bh * A.C + c));
                    am = warp_max(am);
                    if (t == 0) sm.amax_band = am;
                }
                aux_sync();
                const float cl2 = A.scale_log2e;
                for (int row = t; row < BM; row += NAUX) {
                    float ref = 0.f;
                    if (row < nrows) {
                        ref = __uint_as_float(0x7fc00000u);
                        if (band_ok) {
                            const uint8_t *qrow = reinterpret_cast<const uint8_t *>(sm.qn) + row * 128;
                            const uint4 *krow = reinterpret_cast<const uint4 *>(Kraw + ((size_t)bh * A.Nk + pb + row) * kD);
                            float qq = 0.f, qk = 0.f;
#pragma unroll
                            for (int j = 0; j < 8; j++) {
                                const uint4 qv = *reinterpret_cast<const uint4 *>(qrow + ((j ^ (row & 7)) << 4));
                                const uint4 kv = __ldg(krow + j);
                                const uint32_t q4[4] = {qv.x, qv.y, qv.z, qv.w}, k4[4] = {kv.x, kv.y, kv.z, kv.w};
#pragma unroll
                                for (int e = 0; e < 4; e++) {
                                    const float q0 = __uint_as_float(q4[e] << 16), q1 = __uint_as_float(q4[e] & 0xffff0000u);
                                    const float k0 = __uint_as_float(k4[e] << 16), k1 = __uint_as_float(k4[e] & 0xffff0000u);
                                    qq = fmaf(q0, q0, fmaf(q1, q1, qq));
                                    qk = fmaf(q0, k0, fmaf(q1, k1, qk));
                                }
                            }
                            const float ub = sqrtf(qq) * sm.amax_band * cl2;
                            if (ub - qk * cl2 <= kMrefMaxGap) ref = ub;
                        }
                    }
                    sm.wref[row] = ref;
                }
            }
            tc::mbar_arrive(&sm.w_ready);
        } else if (warp == W_MMA) {
            if (lane == 0) {
                const uint32_t id_qk = tc::idesc_bf16(BM, BN, false, false);
                const uint32_t id_pv = tc::idesc_bf16(BM, kD, false, true);
                // descriptors computed once; a byte offset o moves the address field by o >> 4
                const uint64_t dqn = tc::sdesc_sw128(tc::smem_u32(sm.qn), 16, 1024);
                const uint64_t dqr = tc::sdesc_sw128(tc::smem_u32(sm.qr), 16, 1024);
                const uint64_t dk0 = tc::sdesc_sw128(tc::smem_u32(sm.k[0]), 16, 1024);
                const uint64_t dv0 = tc::sdesc_sw128(tc::smem_u32(sm.v[0]), 16, 1024);
                constexpr uint32_t kStageStep = (BN * kD * 2) >> 4;
                bool ok = tc::mbar_wait(&sm.u_ready, 0, ab) && tc::mbar_wait(&sm.q_full, 0, ab);
                const int nR = ok ? (sm.nU + CPC - 1) / CPC : 0;
                int cb = 0, ce = 0;
                if (ok) chunk_range(nR, cb, ce);
                const int total = ce - cb;
                int issued = 0;
                // S(c) = Q K(c)^T into buffer c mod 3, with the NoPE or the rotated Q
                auto issue_qk = [&](int c) -> bool {
                    if (!tc::mbar_wait(&sm.kv_full[c % NSTAGE], (c / NSTAGE) & 1, ab)) return false;
                    const int g = cb + c;
                    if (g >= nR && (g == nR || c == 0) && !tc::mbar_wait(&sm.q_ready, 0, ab)) return false;
                    tc::tc_fence_after();
                    const uint64_t da = g < nR ? dqn : dqr;
                    const uint64_t db = dk0 + (uint64_t)((c % NSTAGE) * kStageStep);
#pragma unroll
                    for (int kk = 0; kk < kD / 16; kk++)      // K steps of 16 columns = 32 bytes
                        tc::mma_ss(tmem + BN * (c % NSBUF), da + 2 * kk, db + 2 * kk, id_qk, kk > 0 ? 1u : 0u);
                    tc::mma_commit(&sm.s_full[c % NSBUF]);
                    issued++;
                    return true;
                };
                if (ok && total > 0) ok = issue_qk(0);
                if (ok && total > 1) ok = issue_qk(1);
                for (int c = 0; ok && c < total; c++) {
                    // S(c+2) goes into the buffer of chunk c-1, whose P was consumed by a P V
                    // issued before this, while the softmax works on chunks c and c+1
                    if (c + 2 < total && !issue_qk(c + 2)) { ok = false; break; }
                    // O += P(c) V(c); the first chunk of each branch overwrites O
                    if (!tc::mbar_wait(&sm.p_full[c % NSBUF], (c / NSBUF) & 1, ab)) { ok = false; break; }
                    tc::tc_fence_after();
                    const bool first = c == 0 || cb + c == nR;
                    const uint64_t db = dv0 + (uint64_t)((c % NSTAGE) * kStageStep);
#pragma unroll
                    for (int kk = 0; kk < BN / 16; kk++)      // K steps of 16 keys = 2048 bytes
                        tc::mma_ts(tmem + O_COL, tmem + BN * (c % NSBUF) + 8 * kk, db + 128 * kk, id_pv,
                                   (!first || kk > 0) ? 1u : 0u);
                    tc::mma_commit(&sm.kv_empty[c % NSTAGE]);
                    tc::mma_commit(&sm.o_ready[c & 1]);
                    issued++;
                }
                if (ok) tc::mma_commit(&sm.o_done);
                if (issued) {
                    tc::mma_commit(&sm.drain);
                    const uint64_t t0 = tc::globaltimer();
                    while (!tc::mbar_try_wait(&sm.drain, 0) && tc::globaltimer() - t0 < tc::kWaitLimitNs) {
                    }
                }
            }
        }
        if (SPLIT) {                            // the softmax warps' two cluster barriers
            __syncwarp();
            tc::cluster_sync();
            tc::cluster_sync();
        }
    } else {
        tc::regs_inc<REGS_SOFTMAX>();
        // ---- softmax: thread = query row
        const int row = warp * 32 + lane;
        const int i = pb + row;
        const bool rvalid = row < nrows;
        const uint32_t trow = tmem + ((uint32_t)(warp * 32) << 16);
        const uint32_t *rec = tiles + ((size_t)bh * gridDim.x + blockIdx.x) * kTileRecWords;
        const uint4 m4 = __ldg(reinterpret_cast<const uint4 *>(rec + kTileMaskOff + 4 * row));
        const float mref = __uint_as_float(__ldg(rec + kTileMrefOff + row));
        // the readout runs against each row's fixed reference unless one of the warp's rows
        // has none; it then tracks a running maximum with lazy rescaling, as the window does
        const bool fixed = __all_sync(kFull, !isnan(mref));
        bool ok = tc::mbar_wait(&sm.u_ready, 0, ab);
        const int nR = ok ? (sm.nU + CPC - 1) / CPC : 0;
        int cb = 0, ce = 0;
        if (ok) chunk_range(nR, cb, ce);
        const int total = ce - cb;
        const int nread = max(0, min(ce, nR) - cb);     // this CTA's readout chunks come first
        float m_lr = fixed ? mref : -INFINITY, l_lr = 0.f, m_sr = -INFINITY, l_sr = 0.f;
        float4 *part_row = SPLIT ? reinterpret_cast<float4 *>(reinterpret_cast<uint8_t *>(sm.k) + row * kPartRowBytes)
                                 : nullptr;
        // O rescale, after the exponentials (S no longer occupies registers); the P V of the
        // previous chunk, which accumulates into the same O, must have finished.  Called only
        // after chunk it's S wait: that S was issued after the P V of chunk it - 3, which
        // shares o_ready[(it - 1) & 1], so the parity wait cannot match an older phase.
        auto rescale_o = [&](int it, float corr) -> bool {
            if (!tc::mbar_wait(&sm.o_ready[(it - 1) & 1], ((it - 1) >> 1) & 1, ab)) return false;
            tc::tc_fence_after();
#pragma unroll
            for (int b = 0; b < kD / 32; b++) {
                uint32_t r[32];
                tc::tmem_ld32(trow + O_COL + 32 * b, r);
                tc::tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 32; e++) r[e] = __float_as_uint(__uint_as_float(r[e]) * corr);
                tc::tmem_st32(trow + O_COL + 32 * b, r);
            }
            return true;
        };
        auto release = [&](int it) {            // P of chunk it is in tensor memory
            tc::tmem_wait_st();
            tc::tc_fence_before();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&sm.p_full[it % NSBUF]);
        };
        int it = 0;
        // ---- readout chunks (eq. (9)): two union cells each, the unselected ones masked
        for (; ok && it < nread; it++) {
            if (!tc::mbar_wait(&sm.s_full[it % NSBUF], (it / NSBUF) & 1, ab)) { ok = false; break; }
            tc::tc_fence_after();
            const int p0 = CPC * (cb + it);
            const int wsel = p0 >> 5;           // word of the row's union mask, in registers
            const uint32_t mw = wsel == 0 ? m4.x : wsel == 1 ? m4.y : wsel == 2 ? m4.z : m4.w;
            const uint32_t sel = (mw >> (p0 & 31)) & ((1u << CPC) - 1u);
            if (fixed) {
                softmax_chunk_fixed(trow + BN * (it % NSBUF), sel, mref, A.scale_log2e, l_lr);
            } else {
                const float corr = softmax_chunk(trow + BN * (it % NSBUF), CELLS, sel, 0, BN, A.scale_log2e, m_lr, l_lr);
                if (it > 0 && __any_sync(kFull, corr != 1.f) && !rescale_o(it, corr)) { ok = false; break; }
            }
            release(it);
        }
        float y[kD];                            // alpha_h RMSNorm(u), once the readout is done
#pragma unroll
        for (int e = 0; e < kD; e++) y[e] = 0.f;
        // the window runs against each row's fixed reference (from the auxiliary warps)
        // unless one of the warp's rows has none
        float wref = 0.f;
        if (ok && total > nread) {
            if (tc::mbar_wait(&sm.w_ready, 0, ab)) wref = sm.wref[row];
            else ok = false;
        }
        const bool wfixed = __all_sync(kFull, !isnan(wref));
        if (wfixed) m_sr = wref;
        // ---- window chunks (eqs. (3)-(4)): 64 consecutive keys of the band each
        for (; ok && it < total; it++) {
            const int g = cb + it;
            if (!tc::mbar_wait(&sm.s_full[it % NSBUF], (it / NSBUF) & 1, ab)) { ok = false; break; }
            tc::tc_fence_after();
            if (it == nread && nread > 0) {
                // readout done (its last P V may still run): take its O out of tensor memory
                // before the window's first P V overwrites it.  This chunk's S was issued
                // after the P V of chunk nread - 3, which shares the barrier of chunk nread - 1,
                // so the parity wait below cannot match an older phase.
                if (!tc::mbar_wait(&sm.o_ready[(nread - 1) & 1], ((nread - 1) >> 1) & 1, ab)) { ok = false; break; }
                tc::tc_fence_after();
                uint32_t a[kD];
                tc::tmem_ld32(trow + O_COL, *reinterpret_cast<uint32_t(*)[32]>(&a[0]));
                tc::tmem_ld32(trow + O_COL + 32, *reinterpret_cast<uint32_t(*)[32]>(&a[32]));
                tc::tmem_wait_ld();
                if (SPLIT) {                    // the readout's partial O, unnormalised, until the end
#pragma unroll
                    for (int e = 0; e < kD; e++) y[e] = __uint_as_float(a[e]);
                } else {                        // O_lr <- alpha_h RMSNorm(O_lr / l)
                    const float inv_l = l_lr > 0.f ? 1.f / l_lr : 0.f;
                    float ss = 0.f;
#pragma unroll
                    for (int e = 0; e < kD; e++) {
                        const float x = __uint_as_float(a[e]) * inv_l;
                        ss = fmaf(x, x, ss);
                    }
                    const float f = l_lr > 0.f ? A.alpha[h] * inv_l / sqrtf(ss * (1.f / kD) + A.rms_eps) : 0.f;
#pragma unroll
                    for (int e = 0; e < kD; e++) y[e] = __uint_as_float(a[e]) * f;
                }
            }
            const int jc = jbase + BN * (k_first + g - nR);
            const int clo = max(-jc, i - A.w - jc), chi = min(i - jc, BN - 1);
            const int width = rvalid ? max(0, chi - clo + 1) : 0;
            const int kind = __all_sync(kFull, clo <= 0 && chi >= BN - 1 && rvalid) ? FULL : BAND;
            if (wfixed) {
                softmax_chunk_band_fixed(trow + BN * (it % NSBUF), kind, clo, width, wref, A.scale_log2e, l_sr);
            } else {
                const float corr = softmax_chunk(trow + BN * (it % NSBUF), kind, 0u, clo, width, A.scale_log2e, m_sr,
                                                 l_sr);
                if (it > nread && __any_sync(kFull, corr != 1.f) && !rescale_o(it, corr)) { ok = false; break; }
            }
            release(it);
        }
        const bool done = ok && tc::mbar_wait(&sm.o_done, 0, ab);
        if (done) {
            tc::tc_fence_after();
            uint32_t a[kD];
            tc::tmem_ld32(trow + O_COL, *reinterpret_cast<uint32_t(*)[32]>(&a[0]));
            tc::tmem_ld32(trow + O_COL + 32, *reinterpret_cast<uint32_t(*)[32]>(&a[32]));
            tc::tmem_wait_ld();
            if (SPLIT) {
                // partial state of this CTA's chunks; a branch it had no chunk of stays empty.
                // O holds the window's sum if the CTA had window chunks, else the readout's
                // (which, with window chunks, was kept in y when the window began).
                const bool had_lr = cb < nR && ce > cb, had_sr = ce > nR && ce > cb;
                sm.phead[row] = make_float4(had_lr ? m_lr : -INFINITY, had_lr ? l_lr : 0.f, had_sr ? m_sr : -INFINITY,
                                            had_sr ? l_sr : 0.f);
#pragma unroll
                for (int q = 0; q < kD / 4; q++) {
                    const float4 v = make_float4(__uint_as_float(a[4 * q]), __uint_as_float(a[4 * q + 1]),
                                                 __uint_as_float(a[4 * q + 2]), __uint_as_float(a[4 * q + 3]));
                    const float4 yv = make_float4(y[4 * q], y[4 * q + 1], y[4 * q + 2], y[4 * q + 3]);
                    const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
                    part_row[q ^ (row & 7)] = !had_lr ? z : had_sr ? yv : v;
                    part_row[16 + (q ^ (row & 7))] = had_sr ? v : z;
                }
            } else if (rvalid) {
                const float inv = l_sr > 0.f ? 1.f / l_sr : 0.f;
                uint4 *dst = reinterpret_cast<uint4 *>(O + ((size_t)bh * A.Nq + r0 + row) * kD);
#pragma unroll
                for (int q = 0; q < 8; q++) {
                    uint32_t w4[4];
#pragma unroll
                    for (int e = 0; e < 4; e++) {
                        const int j = 8 * q + 2 * e;
                        w4[e] = tc::pack_bf16x2(fmaf(__uint_as_float(a[j]), inv, y[j]),
                                                fmaf(__uint_as_float(a[j + 1]), inv, y[j + 1]));
                    }
                    dst[q] = make_uint4(w4[0], w4[1], w4[2], w4[3]);
                }
            }
        }
        if (SPLIT && !done)                     // an aborted CTA contributes nothing (and sets the flag)
            sm.phead[row] = make_float4(-INFINITY, 0.f, -INFINITY, 0.f);
        if (SPLIT) {
            // the tile's S CTAs form one cluster: once every partial state is in place, CTA r
            // combines rows [r R, (r + 1) R) (R = ceil(128 / S)) from all S CTAs' shared memory:
            // the readout's partials merge into u (rescaled to the largest max) and RMSNorm
            // gives alpha_h o^lr, the window's merge into o^sr, and O = o^sr + alpha_h o^lr
            // (eq. (2)).  A softmax warp takes 4 rows at once: lane 8k + s reads split s's
            // (m, l) of row k; then, two rows at a time, every lane reads dimensions (2 lane,
            // 2 lane + 1) of the rows' partial O from every split before using any.  The
            // producer warps take part in both cluster barriers; the second keeps every CTA's
            // shared memory alive until all reads are done.
            __syncwarp();
            tc::cluster_sync();
            const int R = (BM + S - 1) / S;
            const int rlo = sidx * R, rhi = min(min(BM, nrows), rlo + R);
            const uint32_t hbase = tc::smem_u32(sm.phead), vbase = tc::smem_u32(sm.k);
            const int kk = lane >> 3, sp = lane & 7;
            for (int rw = rlo + 4 * warp; rw < rhi; rw += 4 * NSOFT) {
                float4 st = make_float4(-INFINITY, 0.f, -INFINITY, 0.f);
                if (sp < S && rw + kk < rhi)
                    st = tc::ld_cluster_f4(tc::cluster_map(hbase + (uint32_t)((rw + kk) * 16), (uint32_t)sp));
                float M_lr = st.x, M_sr = st.z;
#pragma unroll
                for (int o = 4; o > 0; o >>= 1) {       // maxima over the 8 lanes of a row
                    M_lr = fmaxf(M_lr, __shfl_xor_sync(kFull, M_lr, o));
                    M_sr = fmaxf(M_sr, __shfl_xor_sync(kFull, M_sr, o));
                }
                const float w_lr = st.y > 0.f ? exp2f(st.x - M_lr) : 0.f, w_sr = st.w > 0.f ? exp2f(st.z - M_sr) : 0.f;
                float L_lr = st.y * w_lr, L_sr = st.w * w_sr;
#pragma unroll
                for (int o = 4; o > 0; o >>= 1) {
                    L_lr += __shfl_xor_sync(kFull, L_lr, o);
                    L_sr += __shfl_xor_sync(kFull, L_sr, o);
                }
#pragma unroll
                for (int kb = 0; kb < 4; kb += 2) {     // two rows' loads in flight at a time
                    float2 x[2][8], z[2][8];
#pragma unroll
                    for (int k = 0; k < 2; k++) {
                        const int r = rw + kb + k;
                        const uint32_t ro = vbase + (uint32_t)(r * kPartRowBytes) + (uint32_t)((lane & 1) * 8);
                        const uint32_t cu = (uint32_t)(((lane >> 1) ^ (r & 7)) * 16);
#pragma unroll
                        for (int sx = 0; sx < 8; sx++) {
                            x[k][sx] = make_float2(0.f, 0.f);
                            z[k][sx] = make_float2(0.f, 0.f);
                            if (sx < S && r < rhi) {
                                x[k][sx] = tc::ld_cluster_f2(tc::cluster_map(ro + cu, (uint32_t)sx));
                                z[k][sx] = tc::ld_cluster_f2(tc::cluster_map(ro + 256u + cu, (uint32_t)sx));
                            }
                        }
                    }
#pragma unroll
                    for (int k = 0; k < 2; k++) {
                        const int r = rw + kb + k, src = 8 * (kb + k);
                        float u0 = 0.f, u1 = 0.f, o0 = 0.f, o1 = 0.f;
#pragma unroll
                        for (int sx = 0; sx < 8; sx++) {
                            const float wl = __shfl_sync(kFull, w_lr, src + sx), ws = __shfl_sync(kFull, w_sr, src + sx);
                            u0 = fmaf(x[k][sx].x, wl, u0);
                            u1 = fmaf(x[k][sx].y, wl, u1);
                            o0 = fmaf(z[k][sx].x, ws, o0);
                            o1 = fmaf(z[k][sx].y, ws, o1);
                        }
                        const float Ll = __shfl_sync(kFull, L_lr, src), Ls = __shfl_sync(kFull, L_sr, src);
                        float y0 = 0.f, y1 = 0.f;
                        if (Ll > 0.f) {
                            u0 /= Ll;
                            u1 /= Ll;
                            const float f = A.alpha[h] * rsqrtf(warp_sum(u0 * u0 + u1 * u1) * (1.f / kD) + A.rms_eps);
                            y0 = u0 * f;
                            y1 = u1 * f;
                        }
                        const float inv = Ls > 0.f ? 1.f / Ls : 0.f;
                        if (r < rhi)
                            *reinterpret_cast<uint32_t *>(O + ((size_t)bh * A.Nq + r0 + r) * kD + 2 * lane) =
                                tc::pack_bf16x2(o0 * inv + y0, o1 * inv + y1);
                    }
                }
            }
            __syncwarp();
            tc::cluster_sync();
        }
    }

    tc::tc_fence_before();
    __syncthreads();
    if (warp == W_MMA) {
        tc::tc_fence_after();
        tc::tmem_dealloc(tmem, TMEM_COLS);
    }
}

// CTAs per 128-row tile: 1 when the tiles fill the GPU; otherwise the tile's chunk list is
// split over up to 8 CTAs (about two CTAs per SM in all), one thread-block cluster, which
// combines its partial states itself.
int attn_splits(const fs_params *p) {
    const long long tiles = (long long)p->B * p->H * ((p->Nq + BM - 1) / BM);
    if (tiles <= 0 || tiles >= 148) return 1;
    return (int)std::min<long long>(8, std::max<long long>(1, (2 * 148) / tiles));
}

bool attn_tc_supported(const fs_params *p) {
    const int C = p->Nk / p->s;
    if (p->dtype != FS_BF16 || C > 32768) return false;
    const int bound = p->W >= 0 ? p->W + p->P + 10 : C;     // largest possible |U| per tile
    return bound <= UMAX;
}

cudaError_t launch_attn_tc(const Dev &P, const void *Q, const void *K, const void *V, const void *Krot,
                           const uint32_t *tiles, void *O, const float2 *rope_lo, const float2 *rope_hi,
                           int *dev_flag, int nsplit, const float *amax, cudaStream_t st) {
    if (P.Nq == 0) return cudaSuccess;
    const int BH = P.B * P.H;
    const int kr0 = rope_first_key(P);
    CUtensorMap tq, tk32, tv32, tkr64, tv64;
    if (!encode_tmap_3d_bf16(&tq, Q, kD, P.Nq, BH, kD, BM) ||
        !encode_tmap_3d_bf16(&tk32, K, kD, P.Nk, BH, kD, kS) ||
        !encode_tmap_3d_bf16(&tv32, V, kD, P.Nk, BH, kD, kS) ||
        !encode_tmap_3d_bf16(&tkr64, Krot, kD, P.Nk - kr0, BH, kD, BN) ||
        !encode_tmap_3d_bf16(&tv64, V, kD, P.Nk, BH, kD, BN))
        return cudaErrorInvalidValue;
    AttnArgs A;
    A.Nq = P.Nq; A.Nk = P.Nk; A.q0 = P.q0; A.w = P.w; A.C = P.C; A.K = P.K; A.H = P.H;
    A.kr0 = kr0;
    A.scale_log2e = P.scale * 1.4426950408889634f;
    A.rms_eps = P.rms_eps;
    for (int hh = 0; hh < FS_MAX_HEADS; hh++) A.alpha[hh] = P.alpha[hh];
    A.nsplit = std::min(std::max(nsplit, 1), 8);
    const size_t smem = sizeof(AttnSmem) + 1024;
    static_assert(sizeof(AttnSmem::k) + sizeof(AttnSmem::v) >= (size_t)BM * kPartRowBytes &&
                      offsetof(AttnSmem, v) == offsetof(AttnSmem, k) + sizeof(AttnSmem::k),
                  "the split partial states fit over the K / V stages");
    const int ntiles = (P.Nq + BM - 1) / BM;
    const dim3 grid(ntiles, BH, A.nsplit);
    LaunchScope scope(kAttnTc, st);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(NTHREADS);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;       // a split tile's CTAs: one cluster
    attr[1].val.clusterDim.x = 1;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = A.nsplit;
    cfg.attrs = attr;
    cfg.numAttrs = A.nsplit > 1 ? 2 : 1;
    auto kern = A.nsplit > 1 ? attn_tc_kernel<true> : attn_tc_kernel<false>;
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (cudaLaunchKernelEx(&cfg, kern, tq, tk32, tv32, tkr64, tv64, A, tiles, rope_lo, rope_hi, (__nv_bfloat16 *)O,
                           dev_flag, (const __nv_bfloat16 *)K, amax) != cudaSuccess)
        return cudaErrorLaunchFailure;
    return cudaGetLastError();
}

}  // namespace fs
