// Backward pass on the 5th-generation tensor cores (bf16), readout and window, "FreeSolo"
// summary §3.3 eq. (9) and §3.2 eqs. (3)-(4) with the selection held fixed.  The readout:
// for the rows of one 128-row tile of
// a (batch, head) and the union U of their selected cells (the tile record of the fused
// forward kernel, here built from idx):
//   u_i = sum_t pi_it v_t,  pi_i = softmax_t(s_it),  s_it = q_i.k_t / sqrt(d)  (t in cells(S_i))
//   y_i = u_i r_i,  r_i = (mean(u_i^2) + eps)^(-1/2),  O_i = o_i^sr + alpha_h y_i
// with upstream gradient g_i = dO_i:
//   du_i = r_i (alpha_h g_i - y_i (alpha_h g_i.y_i) / d),  D_i = du_i.u_i
//   dP_it = du_i.v_t,  dS_it = pi_it (dP_it - D_i) / sqrt(d)
//   dq_i += sum_t dS_it k_t,  dk_t += sum_i dS_it q_i,  dv_t += sum_i pi_it du_i,
//   and dO_i.y_i per row for dalpha_h.
// The readout is masked-dense over U, four cells (128 keys) per chunk; a row's unselected
// cells get pi = 0.  Three passes over the chunks:
//   A1  S = Q K^T, each row's largest selected logit (log2 units);
//   A2  S again, P = exp2(S c - m) into tensor memory, U += P V; then per row u, l, r, y,
//       du (bf16, into shared memory as an MMA operand), D and the row's log-sum-exp;
//   B   S and dP = du V^T; P and dS (bf16) into shared memory; dV = P^T du and
//       dK = dS^T Q for the chunk's 128 keys (added to the float32 dK, dV in global
//       memory with vector atomics: several tiles select the same cell); dQ += dS K
//       accumulated in tensor memory and added to dQ once per tile.
// The Q, du, P and dS tiles serve both as K-major operands ([rows][d or keys]) and, read
// the other way, as MN-major ones (the transposed products), in 128-byte-swizzled rows.
//
// The window's part (§3.2 eqs. (3)-(4)) is the same kernel over the band's keys instead of
// the cells (WIN): 128 consecutive keys per chunk from the rotated copy R(j) k_j, Q rotated
// in place by R(i), a row's valid keys [i - w, i], g = dO itself in place of du and
// D = dO.o^sr; dK and dQ are rotated back (R^T) before they are stored.  It runs first and
// stores dQ; the readout adds to it.
//
// Warps: 0-7 rows (warp w: rows 32 (w mod 4) .. + 31, keys 64 (w / 4) .. + 63 of every
// chunk; raised to 192 registers), 8-11 the dK / dV drain (lane = key of key block w - 8 of
// the chunk), 12 TMA, 13 MMA, 14 loads U (readout) or with 15 rotates Q (window; all
// lowered to 64 registers).
#include <cmath>

#include "tc_rope.cuh"

namespace fs {

namespace {
constexpr int BM = 128, BN = 128, CPC = BN / kS;        // rows per tile, keys (4 cells) per chunk
constexpr int UMAX = 128, NSTAGE = 3;
constexpr int NROWW = 8, W_EPI = 8, W_TMA = 12, W_MMA = 13, W_AUX = 14, NWARPS = 16;
constexpr int NTHREADS = NWARPS * 32;
constexpr int REGS_ROW = 192, REGS_OTHER = 64;           // 256 * 192 + 256 * 64 = 512 * 128
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t S_COL = 0, DP_COL = 128, U_COL = 256, DV_COL = 320, DK_COL = DV_COL + 64;
constexpr int TILE_BYTES = BM * kD * 2;                  // 128 rows x 64 bf16: 16 KiB

struct BtcSmem {
    __nv_bfloat16 q[BM * kD];                            // Q tile (NoPE), 128-byte swizzled rows
    __nv_bfloat16 du[BM * kD];                           // du (bf16), same layout
    __nv_bfloat16 k[NSTAGE][BN * kD];                    // chunk keys: 4 cells of 32 rows
    __nv_bfloat16 v[NSTAGE][BN * kD];
    __nv_bfloat16 p[2][BM * kD];                         // P, keys 0-63 | 64-127 of the chunk
    __nv_bfloat16 ds[2][BM * kD];                        // dS, same
    int ulist[UMAX];
    float xch[6][2][BM];                                 // exchanges between a row's two warps
    int nU;
    uint64_t q_full, q_rot, u_ready, du_ready, u_done, dq_done;
    uint64_t kv_full[NSTAGE], kv_empty[NSTAGE];
    uint64_t s_full[2], s_free[2];                       // passes A1 / A2: two S buffers
    uint64_t sd_full, sd_free, pds_full, pds_free, dkv_full, dkv_free;   // pass B
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
};

struct BtcArgs {
    int Nq, Nk, C, H, q0, w, kr0;
    float scale, c2;        // 1 / sqrt(d), log2(e) / sqrt(d)
    float rms_eps;
    float alpha[FS_MAX_HEADS];
};

// the two warps of a row quarter (w and w + 4) exchange one float per row
__device__ __forceinline__ float pair_sum(BtcSmem &sm, int slot, int half, int row, int quarter, float v,
                                          bool is_max) {
    sm.xch[slot][half][row] = v;
    asm volatile("bar.sync %0, 64;" ::"r"(1 + quarter) : "memory");
    const float o = sm.xch[slot][half ^ 1][row];
    return is_max ? fmaxf(v, o) : v + o;
}

// 16-byte chunk j of row r of a 128-byte-swizzled tile
__device__ __forceinline__ uint4 *sw_chunk(__nv_bfloat16 *tile, int r, int j) {
    return reinterpret_cast<uint4 *>(reinterpret_cast<uint8_t *>(tile) + r * 128 + ((j ^ (r & 7)) << 4));
}

__device__ __forceinline__ void red_add_v4(float *dst, float a, float b, float c, float d) {
    asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(dst), "f"(a), "f"(b), "f"(c), "f"(d)
                 : "memory");
}
}  // namespace

// WIN = false: the readout over the tile's cells (tk, tv: 32-row boxes of K, V; tg unused);
// WIN = true: the window over the band (tk: 128-row boxes of the rotated keys from kr0 on,
// tv: of V, tg: the dO tile)
template <bool WIN>
__global__ void __launch_bounds__(NTHREADS, 1)
bwd_tc_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tg,
              const __grid_constant__ CUtensorMap tk, const __grid_constant__ CUtensorMap tv, const BtcArgs A,
              const uint32_t *__restrict__ tiles, const __nv_bfloat16 *__restrict__ dO, float *__restrict__ dQ,
              float *__restrict__ dK, float *__restrict__ dV, float *__restrict__ dal,
              const float2 *__restrict__ rope_lo, const float2 *__restrict__ rope_hi, int *dev_flag) {
    extern __shared__ uint8_t smraw[];
    const uint32_t sbase = tc::smem_u32(smraw);
    BtcSmem &sm = *reinterpret_cast<BtcSmem *>(smraw + (((sbase + 1023u) & ~1023u) - sbase));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int bh = blockIdx.y, h = bh % A.H;
    const int r0 = blockIdx.x * BM;
    const int nrows = min(BM, A.Nq - r0);
    const uint32_t *rec = WIN ? nullptr : tiles + ((size_t)bh * gridDim.x + blockIdx.x) * kTileRecWords;
    const int pb = A.q0 + r0, jbase = pb - A.w, last = pb + nrows - 1;   // window: the tile's band
    const tc::Abort ab{dev_flag, &sm.abort};
    // chunks of the tile: four union cells each (readout), 128 band keys each (window)
    auto chunks = [&]() { return WIN ? (last - jbase) / BN + 1 : (sm.nU + CPC - 1) / CPC; };

    if (threadIdx.x == 0) {
        sm.abort = 0;
        tc::mbar_init(&sm.q_full, 1);
        tc::mbar_init(&sm.q_rot, 2);
        tc::mbar_init(&sm.u_ready, 1);
        tc::mbar_init(&sm.du_ready, NROWW);
        tc::mbar_init(&sm.u_done, 1);
        tc::mbar_init(&sm.dq_done, 1);
        for (int s = 0; s < NSTAGE; s++) {
            tc::mbar_init(&sm.kv_full[s], 1);
            tc::mbar_init(&sm.kv_empty[s], 1);
        }
        for (int b = 0; b < 2; b++) {
            tc::mbar_init(&sm.s_full[b], 1);
            tc::mbar_init(&sm.s_free[b], NROWW);
        }
        tc::mbar_init(&sm.sd_full, 1);
        tc::mbar_init(&sm.sd_free, NROWW);
        tc::mbar_init(&sm.pds_full, NROWW);
        tc::mbar_init(&sm.pds_free, 1);
        tc::mbar_init(&sm.dkv_full, 1);
        tc::mbar_init(&sm.dkv_free, 4);
        tc::mbar_init(&sm.drain, 1);
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

    if (warp >= NROWW) {
        tc::regs_dec<REGS_OTHER>();
        if (warp >= W_AUX) {
            if (!WIN) {
                if (warp == W_AUX) {
                    for (int u = lane; u < UMAX; u += 32) sm.ulist[u] = (int)__ldg(rec + kTileUlistOff + u);
                    if (lane == 0) sm.nU = min((int)__ldg(rec + kTileCountOff), UMAX);
                    __syncwarp();
                    if (lane == 0) tc::mbar_arrive(&sm.u_ready);
                }
            } else {
                if (warp == W_AUX && lane == 0) tc::mbar_arrive(&sm.u_ready);
                // rotate Q in place by its absolute positions (16-byte chunks, 128-byte swizzle)
                if (tc::mbar_wait(&sm.q_full, 0, ab)) {
                    const int t = threadIdx.x - W_AUX * 32;
                    uint8_t *qb = reinterpret_cast<uint8_t *>(sm.q);
#pragma unroll 2
                    for (int j = 0; j < BM * 8 / 64; j++) {
                        const int item = t + 64 * j, row = item >> 3, c = item & 7;
                        uint4 *ptr = reinterpret_cast<uint4 *>(qb + row * 128 + ((c ^ (row & 7)) << 4));
                        float cs[4], sn[4];
                        rope_angles(pb + row, c, rope_lo, rope_hi, cs, sn);
                        *ptr = rope_rotate8(*ptr, cs, sn);
                    }
                    tc::fence_async_shared();
                }
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(&sm.q_rot);
            }
        } else if (warp == W_TMA) {
            if (lane == 0) {
                tc::prefetch_tmap(&tq);
                tc::prefetch_tmap(&tk);
                tc::prefetch_tmap(&tv);
                tc::mbar_expect_tx(&sm.q_full, (WIN ? 2 : 1) * TILE_BYTES);
                tc::tma_load_3d(sm.q, &tq, &sm.q_full, 0, r0, bh);
                if (WIN) tc::tma_load_3d(sm.du, &tg, &sm.q_full, 0, r0, bh);   // g = dO
                int g = 0, total = 0;
                if (tc::mbar_wait(&sm.u_ready, 0, ab)) {
                    const int nU = WIN ? 0 : sm.nU, nC = chunks();
                    total = 3 * nC;                       // passes A1 (K only), A2, B
                    for (; g < total; g++) {
                        const int s = g % NSTAGE, c = g % nC;
                        const bool withv = g >= nC;
                        if (!tc::mbar_wait(&sm.kv_empty[s], ((g / NSTAGE) & 1) ^ 1, ab)) break;
                        tc::mbar_expect_tx(&sm.kv_full[s], (withv ? 2 : 1) * BN * kD * 2);
                        if (WIN) {                        // 128 band keys; before key 0: zeros
                            const int jc = jbase + BN * c;
                            tc::tma_load_3d(sm.k[s], &tk, &sm.kv_full[s], 0, jc - A.kr0, bh);
                            if (withv) tc::tma_load_3d(sm.v[s], &tv, &sm.kv_full[s], 0, jc, bh);
                        } else {
                            for (int j = 0; j < CPC; j++) {
                                const int u = CPC * c + j;
                                const int y = u < nU ? sm.ulist[u] * kS : A.Nk;   // past the end: zeros
                                tc::tma_load_3d(sm.k[s] + j * kS * kD, &tk, &sm.kv_full[s], 0, y, bh);
                                if (withv) tc::tma_load_3d(sm.v[s] + j * kS * kD, &tv, &sm.kv_full[s], 0, y, bh);
                            }
                        }
                    }
                }
                if (sm.abort) {   // let issued copies land before the CTA's memory is released
                    for (int j = max(0, g - NSTAGE); j < g; j++) {
                        const uint64_t t0 = tc::globaltimer();
                        while (!tc::mbar_try_wait(&sm.kv_full[j % NSTAGE], (j / NSTAGE) & 1) &&
                               tc::globaltimer() - t0 < tc::kWaitLimitNs) {
                        }
                    }
                }
            }
        } else if (warp == W_MMA) {
            if (lane == 0) {
                const uint32_t id_s = tc::idesc_bf16(BM, BN, false, false);     // S, dP: [rows x keys]
                const uint32_t id_kd = tc::idesc_bf16(BN, kD, true, true);      // dV, dK: [keys x d]
                const uint32_t id_pv = tc::idesc_bf16(BM, kD, false, true);     // U, dQ: [rows x d]
                const uint32_t aq = tc::smem_u32(sm.q), adu = tc::smem_u32(sm.du);
                const uint32_t ak0 = tc::smem_u32(sm.k[0]), av0 = tc::smem_u32(sm.v[0]);
                const uint32_t ap = tc::smem_u32(sm.p[0]), ads = tc::smem_u32(sm.ds[0]);
                constexpr uint32_t kStage = BN * kD * 2, kHalf = BM * kD * 2;
                bool ok = tc::mbar_wait(&sm.u_ready, 0, ab) && tc::mbar_wait(&sm.q_full, 0, ab) &&
                          (!WIN || tc::mbar_wait(&sm.q_rot, 0, ab));
                const int nC = ok ? chunks() : 0;
                int g = 0;                                // K / V load sequence
                int issued = 0;
                // [rows x keys] (+)= X [rows x 64] Y^T, X = Q or du (K-major), Y = the stage's K or V
                auto rows_keys = [&](uint32_t dcol, uint32_t ax, uint32_t ay) {
#pragma unroll 1
                    for (int kk = 0; kk < kD / 16; kk++)
                        tc::mma_ss(tmem + dcol, tc::sdesc_sw128(ax + 32 * kk, 16, 1024),
                                   tc::sdesc_sw128(ay + 32 * kk, 16, 1024), id_s, kk > 0 ? 1u : 0u);
                };
                // passes A1 and A2: S into buffer sc & 1; A2 adds P V into U
                for (int sc = 0; ok && sc < 2 * nC; sc++, g++) {
                    const int b = sc & 1, s = g % NSTAGE;
                    if (!tc::mbar_wait(&sm.kv_full[s], (g / NSTAGE) & 1, ab)) { ok = false; break; }
                    if (sc >= 2 && !tc::mbar_wait(&sm.s_free[b], ((sc - 2) >> 1) & 1, ab)) { ok = false; break; }
                    tc::tc_fence_after();
                    rows_keys(S_COL + 128 * b, aq, ak0 + s * kStage);
                    tc::mma_commit(&sm.s_full[b]);
                    issued++;
                    if (sc < nC) {
                        tc::mma_commit(&sm.kv_empty[s]);
                        continue;
                    }
                    // U += P V: P (bf16) in tensor memory, keys 0-63 at the buffer's column 0,
                    // keys 64-127 at its column 64; V MN-major, 16 keys (2048 bytes) per step
                    if (!tc::mbar_wait(&sm.s_free[b], (sc >> 1) & 1, ab)) { ok = false; break; }
                    tc::tc_fence_after();
#pragma unroll 1
                    for (int kk = 0; kk < BN / 16; kk++)
                        tc::mma_ts(tmem + U_COL, tmem + S_COL + 128 * b + 64 * (kk >> 2) + 8 * (kk & 3),
                                   tc::sdesc_sw128(av0 + s * kStage + 2048 * kk, 16, 1024), id_pv,
                                   (sc > nC || kk > 0) ? 1u : 0u);
                    tc::mma_commit(&sm.kv_empty[s]);
                }
                tc::mma_commit(&sm.u_done);
                // pass B
                auto issue_sdp = [&](int c) -> bool {
                    const int s = (g + c) % NSTAGE, gg = g + c;
                    if (!tc::mbar_wait(&sm.kv_full[s], (gg / NSTAGE) & 1, ab)) return false;
                    if (c > 0 && !tc::mbar_wait(&sm.sd_free, (c - 1) & 1, ab)) return false;
                    tc::tc_fence_after();
                    rows_keys(S_COL, aq, ak0 + s * kStage);
                    rows_keys(DP_COL, adu, av0 + s * kStage);
                    tc::mma_commit(&sm.sd_full);
                    return true;
                };
                if (ok && nC > 0) ok = tc::mbar_wait(&sm.du_ready, 0, ab) && issue_sdp(0);
                for (int c = 0; ok && c < nC; c++) {
                    const int s = (g + c) % NSTAGE;
                    if (c + 1 < nC && !issue_sdp(c + 1)) { ok = false; break; }
                    if (!tc::mbar_wait(&sm.pds_full, c & 1, ab)) { ok = false; break; }
                    if (c > 0 && !tc::mbar_wait(&sm.dkv_free, (c - 1) & 1, ab)) { ok = false; break; }
                    tc::tc_fence_after();
                    // dV = P^T du, dK = dS^T Q: [keys x d], K = rows, 16 rows (2048 bytes) per step;
                    // the A operand's two 64-key halves are 16 KiB apart (leading byte offset)
#pragma unroll 1
                    for (int kk = 0; kk < BM / 16; kk++) {
                        tc::mma_ss(tmem + DV_COL, tc::sdesc_sw128(ap + 2048 * kk, kHalf, 1024),
                                   tc::sdesc_sw128(adu + 2048 * kk, 16, 1024), id_kd, kk > 0 ? 1u : 0u);
                        tc::mma_ss(tmem + DK_COL, tc::sdesc_sw128(ads + 2048 * kk, kHalf, 1024),
                                   tc::sdesc_sw128(aq + 2048 * kk, 16, 1024), id_kd, kk > 0 ? 1u : 0u);
                    }
                    tc::mma_commit(&sm.dkv_full);
                    // dQ += dS K: [rows x d], K = keys; dS K-major (keys 0-63 in half 0, 64-127 in
                    // half 1, 32 bytes per step), K MN-major
#pragma unroll 1
                    for (int kk = 0; kk < BN / 16; kk++)
                        tc::mma_ss(tmem + U_COL, tc::sdesc_sw128(ads + kHalf * (kk >> 2) + 32 * (kk & 3), 16, 1024),
                                   tc::sdesc_sw128(ak0 + s * kStage + 2048 * kk, 16, 1024), id_pv,
                                   (c > 0 || kk > 0) ? 1u : 0u);
                    tc::mma_commit(&sm.pds_free);
                    tc::mma_commit(&sm.kv_empty[s]);
                }
                if (ok) tc::mma_commit(&sm.dq_done);
                if (issued) {       // every MMA done before tensor memory is released
                    tc::mma_commit(&sm.drain);
                    const uint64_t t0 = tc::globaltimer();
                    while (!tc::mbar_try_wait(&sm.drain, 0) && tc::globaltimer() - t0 < tc::kWaitLimitNs) {
                    }
                }
            }
        } else if (warp >= W_EPI && warp < W_EPI + 4) {
            // dK, dV of the chunk's cell (warp - W_EPI): lane = token of the cell
            const int e = warp - W_EPI;
            bool ok = tc::mbar_wait(&sm.u_ready, 0, ab);
            const int nU = ok && !WIN ? sm.nU : 0, nC = ok ? chunks() : 0;
            const uint32_t trow = tmem + ((uint32_t)(e * 32) << 16);
            for (int c = 0; ok && c < nC; c++) {
                if (!tc::mbar_wait(&sm.dkv_full, c & 1, ab)) { ok = false; break; }
                tc::tc_fence_after();
                int j = 0;                                   // this lane's key
                bool has = false;
                if (WIN) {
                    j = jbase + BN * c + 32 * e + lane;
                    has = j >= max(0, jbase) && j <= last;
                } else {
                    const int u = CPC * c + e;
                    has = u < nU;
                    if (has) j = sm.ulist[u] * kS + lane;
                }
                if (__any_sync(kFull, has)) {
                    const int jj = has ? j : 0;              // lanes without a key read position 0
                    const size_t key = (size_t)bh * A.Nk + (size_t)jj;
                    float *dv = dV + key * kD, *dk = dK + key * kD;
#pragma unroll 1
                    for (int b = 0; b < 2 * kD / 16; b++) {      // dV columns, then dK's, 16 at a time
                        uint32_t x[16];
                        tc::tmem_ld16(trow + DV_COL + 16 * b, x);   // DK_COL = DV_COL + 64
                        tc::tmem_wait_ld();
                        float y[16];
#pragma unroll
                        for (int q = 0; q < 16; q++) y[q] = __uint_as_float(x[q]);
                        if (WIN && b >= kD / 16) {           // dK_j = R(j)^T dK'_j, pairs 8 (b - 4) ..
#pragma unroll
                            for (int hc = 0; hc < 2; hc++) {
                                float cs[4], sn[4];
                                rope_angles(jj, 2 * (b - kD / 16) + hc, rope_lo, rope_hi, cs, sn);
#pragma unroll
                                for (int t = 0; t < 4; t++) {
                                    const float a0 = y[8 * hc + 2 * t], a1 = y[8 * hc + 2 * t + 1];
                                    y[8 * hc + 2 * t] = a0 * cs[t] + a1 * sn[t];
                                    y[8 * hc + 2 * t + 1] = -a0 * sn[t] + a1 * cs[t];
                                }
                            }
                        }
                        float *dst = (b < kD / 16 ? dv : dk - kD) + 16 * b;
                        if (has)
#pragma unroll
                            for (int q = 0; q < 4; q++)
                                red_add_v4(dst + 4 * q, y[4 * q], y[4 * q + 1], y[4 * q + 2], y[4 * q + 3]);
                    }
                }
                tc::tc_fence_before();
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(&sm.dkv_free);
            }
        }
    } else {
        tc::regs_inc<REGS_ROW>();
        const int quarter = warp & 3, half = warp >> 2;
        const int row = quarter * 32 + lane;
        const bool rvalid = row < nrows;
        const int i = pb + row;
        const uint32_t trow = tmem + ((uint32_t)(quarter * 32) << 16);
        const uint4 m4 = WIN ? make_uint4(0u, 0u, 0u, 0u)
                             : __ldg(reinterpret_cast<const uint4 *>(rec + kTileMaskOff + 4 * row));
        bool ok = tc::mbar_wait(&sm.u_ready, 0, ab);
        const int nC = ok ? chunks() : 0;
        // valid columns of this row among its half's 64 keys of chunk c: the selected cells
        // 4c + 2 half, + 1 (readout), or the keys of [i - w, i] at or after key 0 (window)
        auto colmask = [&](int c) -> uint64_t {
            if (!rvalid) return 0ull;
            if (WIN) {
                const int base = jbase + BN * c + 64 * half;
                const int lo = max(max(i - A.w - base, -base), 0), hi = min(i - base, 63);
                if (lo > hi) return 0ull;
                return (hi == 63 ? ~0ull : (2ull << hi) - 1ull) & ~((1ull << lo) - 1ull);
            }
            const int p0 = CPC * c + 2 * half;
            const int ws = p0 >> 5;
            const uint32_t mw = ws == 0 ? m4.x : ws == 1 ? m4.y : ws == 2 ? m4.z : m4.w;
            const uint32_t sel = (mw >> (p0 & 31)) & 3u;
            return ((sel & 1u) ? 0xffffffffull : 0ull) | ((sel & 2u) ? 0xffffffff00000000ull : 0ull);
        };
        const float c2 = A.c2;
        // ---- A1: the row's largest valid logit (log2 units)
        float m = -INFINITY;
        for (int c = 0; ok && c < nC; c++) {
            const int b = c & 1;
            if (!tc::mbar_wait(&sm.s_full[b], (c >> 1) & 1, ab)) { ok = false; break; }
            tc::tc_fence_after();
            uint32_t x[64];
            tc::tmem_ld32(trow + S_COL + 128 * b + 64 * half, *reinterpret_cast<uint32_t(*)[32]>(&x[0]));
            tc::tmem_ld32(trow + S_COL + 128 * b + 64 * half + 32, *reinterpret_cast<uint32_t(*)[32]>(&x[32]));
            tc::tmem_wait_ld();
            tc::tc_fence_before();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&sm.s_free[b]);
            const uint64_t vm = colmask(c);
            float mx = -INFINITY;
#pragma unroll
            for (int j = 0; j < 64; j++)
                if ((vm >> j) & 1ull) mx = fmaxf(mx, __uint_as_float(x[j]));
            m = fmaxf(m, mx * c2);
        }
        m = pair_sum(sm, 0, half, row, quarter, m, true);
        const float mb = m == -INFINITY ? 0.f : m;
        // ---- A2: P = exp2(S c - m) (valid columns) into tensor memory for U += P V
        float l = 0.f;
        for (int c = 0; ok && c < nC; c++) {
            const int sc = nC + c, b = sc & 1;
            if (!tc::mbar_wait(&sm.s_full[b], (sc >> 1) & 1, ab)) { ok = false; break; }
            tc::tc_fence_after();
            const uint64_t vm = colmask(c);
            const uint32_t tS = trow + S_COL + 128 * b + 64 * half;
            uint32_t x[64];
            tc::tmem_ld32(tS, *reinterpret_cast<uint32_t(*)[32]>(&x[0]));
            tc::tmem_ld32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(&x[32]));
            tc::tmem_wait_ld();
            uint32_t pk[32];
#pragma unroll
            for (int j = 0; j < 64; j += 2) {
                const float p0 = ((vm >> j) & 1ull) ? tc::ex2(fmaf(__uint_as_float(x[j]), c2, -mb)) : 0.f;
                const float p1 = ((vm >> (j + 1)) & 1ull) ? tc::ex2(fmaf(__uint_as_float(x[j + 1]), c2, -mb)) : 0.f;
                l += p0 + p1;
                pk[j >> 1] = tc::pack_bf16x2(p0, p1);
            }
            tc::tmem_st32(tS, *reinterpret_cast<uint32_t(*)[32]>(&pk[0]));
            tc::tmem_wait_st();
            tc::tc_fence_before();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&sm.s_free[b]);
        }
        l = pair_sum(sm, 1, half, row, quarter, l, false);
        // ---- row statistics (dimensions 32 half .. + 31 here): the branch's normalised output
        // o (u for the readout, o^sr for the window), then for the readout RMSNorm, du and
        // dO.y; D = du.u (readout) or dO.o^sr (window)
        float uu[32];
#pragma unroll
        for (int e = 0; e < 32; e++) uu[e] = 0.f;
        if (ok && tc::mbar_wait(&sm.u_done, 0, ab)) {
            tc::tc_fence_after();
            uint32_t ur[32];
            tc::tmem_ld32(trow + U_COL + 32 * half, ur);
            tc::tmem_wait_ld();
            const float inv_l = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
            for (int e = 0; e < 32; e++) uu[e] = __uint_as_float(ur[e]) * inv_l;
        } else {
            ok = false;
        }
        float g[32];
        {
            const uint4 *src = reinterpret_cast<const uint4 *>(dO + ((size_t)bh * A.Nq + r0 + (rvalid ? row : 0)) * kD + 32 * half);
#pragma unroll
            for (int q = 0; q < 4; q++) {
                const uint4 v = rvalid ? __ldg(src + q) : make_uint4(0u, 0u, 0u, 0u);
                const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int t = 0; t < 4; t++) {
                    g[8 * q + 2 * t] = __uint_as_float(w4[t] << 16);
                    g[8 * q + 2 * t + 1] = __uint_as_float(w4[t] & 0xffff0000u);
                }
            }
        }
        const bool has = l > 0.f;
        float D = 0.f;
        if (WIN) {
            float dsum = 0.f;
#pragma unroll
            for (int e = 0; e < 32; e++) dsum = fmaf(g[e], uu[e], dsum);
            D = pair_sum(sm, 4, half, row, quarter, dsum, false);
        } else {
            float ss = 0.f;
#pragma unroll
            for (int e = 0; e < 32; e++) ss = fmaf(uu[e], uu[e], ss);
            ss = pair_sum(sm, 2, half, row, quarter, ss, false);
            const float rin = rsqrtf(ss * (1.f / kD) + A.rms_eps);
            float gy = 0.f;
#pragma unroll
            for (int e = 0; e < 32; e++) gy = fmaf(g[e], uu[e] * rin, gy);
            gy = pair_sum(sm, 3, half, row, quarter, has ? gy : 0.f, false);
            const float a = A.alpha[h], dyy = a * gy;
            float dus[32], dsum = 0.f;
#pragma unroll
            for (int e = 0; e < 32; e++) {
                dus[e] = has ? rin * (a * g[e] - uu[e] * rin * dyy * (1.f / kD)) : 0.f;
                dsum = fmaf(dus[e], uu[e], dsum);
            }
            D = pair_sum(sm, 4, half, row, quarter, dsum, false);
#pragma unroll
            for (int q = 0; q < 4; q++) {      // 16-byte chunks 4 half .. 4 half + 3 of the row
                uint32_t w4[4];
#pragma unroll
                for (int t = 0; t < 4; t++) w4[t] = tc::pack_bf16x2(dus[8 * q + 2 * t], dus[8 * q + 2 * t + 1]);
                *sw_chunk(sm.du, row, 4 * half + q) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
            }
            if (half == 0 && rvalid) dal[(size_t)bh * A.Nq + r0 + row] = gy;
            tc::fence_async_shared();
        }
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&sm.du_ready);
        const float lse2 = has ? mb + log2f(l) : INFINITY;        // P = exp2(S c - lse2); none: 0
        // ---- B: P, dS for this row's 64 keys of each chunk
        for (int c = 0; ok && c < nC; c++) {
            if (!tc::mbar_wait(&sm.sd_full, c & 1, ab)) { ok = false; break; }
            tc::tc_fence_after();
            const uint64_t vm = colmask(c);
            uint32_t pk[32], dk[32];
#pragma unroll
            for (int hb = 0; hb < 2; hb++) {            // 32 keys at a time
                uint32_t x[32], y[32];
                tc::tmem_ld32(trow + S_COL + 64 * half + 32 * hb, x);
                tc::tmem_ld32(trow + DP_COL + 64 * half + 32 * hb, y);
                tc::tmem_wait_ld();
                const uint32_t vw = (uint32_t)(vm >> (32 * hb));
#pragma unroll
                for (int j = 0; j < 32; j += 2) {
                    const float p0 = ((vw >> j) & 1u) ? tc::ex2(fmaf(__uint_as_float(x[j]), c2, -lse2)) : 0.f;
                    const float p1 = ((vw >> (j + 1)) & 1u) ? tc::ex2(fmaf(__uint_as_float(x[j + 1]), c2, -lse2)) : 0.f;
                    const float d0 = p0 * (__uint_as_float(y[j]) - D) * A.scale;
                    const float d1 = p1 * (__uint_as_float(y[j + 1]) - D) * A.scale;
                    pk[16 * hb + (j >> 1)] = tc::pack_bf16x2(p0, p1);
                    dk[16 * hb + (j >> 1)] = tc::pack_bf16x2(d0, d1);
                }
            }
            tc::tc_fence_before();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&sm.sd_free);
            if (c > 0 && !tc::mbar_wait(&sm.pds_free, (c - 1) & 1, ab)) { ok = false; break; }
#pragma unroll
            for (int q = 0; q < 8; q++) {
                *sw_chunk(sm.p[half], row, q) = make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
                *sw_chunk(sm.ds[half], row, q) = make_uint4(dk[4 * q], dk[4 * q + 1], dk[4 * q + 2], dk[4 * q + 3]);
            }
            tc::fence_async_shared();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&sm.pds_full);
        }
        // ---- dQ: the window's, rotated back by R(i)^T, is stored; the readout's is added
        if (ok && nC > 0 && tc::mbar_wait(&sm.dq_done, 0, ab)) {
            tc::tc_fence_after();
            uint32_t qr[32];
            tc::tmem_ld32(trow + U_COL + 32 * half, qr);
            tc::tmem_wait_ld();
            if (rvalid) {
                float dq[32];
#pragma unroll
                for (int e = 0; e < 32; e++) dq[e] = __uint_as_float(qr[e]);
                float *dst = dQ + ((size_t)bh * A.Nq + r0 + row) * kD + 32 * half;
                if (WIN) {
#pragma unroll
                    for (int c4 = 0; c4 < 4; c4++) {   // pairs 16 half + 4 c4 .. + 3
                        float cs[4], sn[4];
                        rope_angles(i, 4 * half + c4, rope_lo, rope_hi, cs, sn);
#pragma unroll
                        for (int t = 0; t < 4; t++) {
                            const float a0 = dq[8 * c4 + 2 * t], a1 = dq[8 * c4 + 2 * t + 1];
                            dq[8 * c4 + 2 * t] = a0 * cs[t] + a1 * sn[t];
                            dq[8 * c4 + 2 * t + 1] = -a0 * sn[t] + a1 * cs[t];
                        }
                    }
#pragma unroll
                    for (int q = 0; q < 8; q++)
                        *reinterpret_cast<float4 *>(dst + 4 * q) = make_float4(dq[4 * q], dq[4 * q + 1], dq[4 * q + 2], dq[4 * q + 3]);
                } else {
#pragma unroll
                    for (int q = 0; q < 8; q++) {
                        float4 v = *reinterpret_cast<float4 *>(dst + 4 * q);
                        v.x += dq[4 * q];
                        v.y += dq[4 * q + 1];
                        v.z += dq[4 * q + 2];
                        v.w += dq[4 * q + 3];
                        *reinterpret_cast<float4 *>(dst + 4 * q) = v;
                    }
                }
            }
        } else if (WIN && rvalid) {               // no chunk ran (an aborted CTA): dQ defined anyway
            float *dst = dQ + ((size_t)bh * A.Nq + r0 + row) * kD + 32 * half;
#pragma unroll
            for (int q = 0; q < 8; q++) *reinterpret_cast<float4 *>(dst + 4 * q) = make_float4(0.f, 0.f, 0.f, 0.f);
        }
    }

    tc::tc_fence_before();
    __syncthreads();
    if (warp == W_MMA) {
        tc::tc_fence_after();
        tc::tmem_dealloc(tmem, TMEM_COLS);
    }
}

bool bwd_tc_supported(const fs_params *p) {
    if (p->dtype != FS_BF16) return false;
    const int C = p->Nk / p->s;
    const int bound = p->W >= 0 ? p->W + p->P + 10 : C;   // largest union of a tile's cells
    return bound <= UMAX && p->Nk < (1 << 30);
}

cudaError_t launch_bwd_tc(const fs_params *p, bool win, const void *Q, const void *K, const void *V,
                          const void *Krot, const uint32_t *tiles, const void *dO, float *dQ, float *dK, float *dV,
                          float *dal, const float2 *rope_lo, const float2 *rope_hi, int *dev_flag, cudaStream_t st) {
    if (p->Nq == 0) return cudaSuccess;
    const int BH = p->B * p->H;
    const int q0 = p->Nk - p->Nq, kr0 = q0 - p->w > 0 ? q0 - p->w : 0;
    CUtensorMap tq, tg, tk, tv;
    bool enc = encode_tmap_3d_bf16(&tq, Q, kD, p->Nq, BH, kD, BM);
    if (win)
        enc = enc && encode_tmap_3d_bf16(&tg, dO, kD, p->Nq, BH, kD, BM) &&
              encode_tmap_3d_bf16(&tk, Krot, kD, p->Nk - kr0, BH, kD, BN) &&
              encode_tmap_3d_bf16(&tv, V, kD, p->Nk, BH, kD, BN);
    else
        enc = enc && encode_tmap_3d_bf16(&tk, K, kD, p->Nk, BH, kD, kS) &&
              encode_tmap_3d_bf16(&tv, V, kD, p->Nk, BH, kD, kS);
    if (!enc) return cudaErrorInvalidValue;
    if (!win) tg = tq;                                     // unused
    BtcArgs A;
    A.Nq = p->Nq; A.Nk = p->Nk; A.C = p->Nk / p->s; A.H = p->H;
    A.q0 = q0; A.w = p->w; A.kr0 = kr0;
    A.scale = (float)(1.0 / std::sqrt((double)p->d));
    A.c2 = A.scale * 1.4426950408889634f;
    A.rms_eps = p->rms_eps;
    for (int hh = 0; hh < FS_MAX_HEADS; hh++) A.alpha[hh] = hh < p->H ? p->alpha[hh] : 0.f;
    const size_t smem = sizeof(BtcSmem) + 1024;
    const dim3 grid((p->Nq + BM - 1) / BM, BH);
    LaunchScope scope(win ? kBwdWindowTc : kBwdReadoutTc, st);
    auto kern = win ? bwd_tc_kernel<true> : bwd_tc_kernel<false>;
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    kern<<<grid, NTHREADS, smem, st>>>(tq, tg, tk, tv, A, tiles, (const __nv_bfloat16 *)dO, dQ, dK, dV, dal, rope_lo,
                                       rope_hi, dev_flag);
    return cudaGetLastError();
}

}  // namespace fs
