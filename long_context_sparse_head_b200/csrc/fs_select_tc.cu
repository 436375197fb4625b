// Long-range cell selection on the 5th-generation tensor cores (bf16 queries),
// "FreeSolo" summary §3.3 eqs. (7)-(8):
//   A_i  = Recent_W(C_i) u TopP_{c in C_i}(a_c)                       (FS-L pruning)
//   r_ic = q_i.kbar_c / sqrt(d) + lambda_h a_c erf((i - p_c) / (2 sigma_h)),  c in A_i
//   S_i  = the K cells of A_i with the largest r_ic (ties: lower cell index)
//
// One CTA per 128 query rows of a (batch, head).  The rows of a tile have at most five
// distinct candidate prefixes n (a prefix grows by one cell every s = 32 positions), so
// U = union of their admitted sets is at most W + P + 10 cells (<= 128 here).  Warps 0-3
// build U: with W >= 1, from the tile's TopP(n_min) list (tile-list kernel) below the
// recent range followed by that range; when decoding, from the exit-times kernel's list of
// the cells that are TopP members at an asked prefix plus the recent cells; otherwise by
// an ordered compaction of the TopP exit table.  Then they stage the fp32 mean keys of
// U as three bf16 parts hi + mid + lo (the split carries the fp32 mantissa, so the bf16
// tensor-core products sum to the fp32 dot product up to accumulation rounding), in the
// 128-byte-swizzled layout of a K-major MMA operand.  One thread issues
// S = Q (hi + mid + lo)^T (M = 128, N = |U| rounded up to 16) into tensor memory.  Each
// row thread then reads its row's scores (twice, 16 columns at a time: the admitted range,
// then the keys) and writes integer keys to shared memory, over Q and the mean-key parts:
// the score's 24-bit fixed-point place within the row's admitted range, above 7 bits of
// (127 - position).  Keys are unique, and among scores within 2^-24 of the row's range of
// each other the lower cell index wins, inside the near-tie tolerance of the selection
// check.  Eight warps then find each row's K-th largest key by bisection, two threads per
// row with half of its keys each; keys spread over one range per row separate in far
// fewer halvings than order-preserving bit patterns of the raw fp32 scores.
// Outputs: idx (selected cells per row, ascending, -1 padded) and/or, for the fused
// kernel, one compact record per tile: each row's selected union positions as a 128-bit
// mask, the union's cells and its size.
#include "tc_common.cuh"

namespace fs {

namespace {
constexpr int BM = 128, UMAX = 128;              // largest union; UM = 80 or UMAX per launch
// warps 0-3: union, staging, scores and keys (thread = row = TMEM lane); warps 0-7: the
// K-th search, two threads per row; warp 8: Q load, then the MMA
constexpr int NROWW = 4, NSRCHW = 8, W_MMA = 8, NWARPS = 9, NTHREADS = NWARPS * 32;
constexpr uint32_t TMEM_COLS = 128;
constexpr int TILE_BYTES = BM * kD * 2;
constexpr int kSelBarrier = 1;   // named barrier of the 128 row threads
constexpr int kSrchBarrier = 2;  // named barrier of the 256 search threads

template <int UM> struct SelSmem {       // UM: capacity of the union (a multiple of 16)
    __nv_bfloat16 q[BM * kD];              // Q tile (NoPE)
    __nv_bfloat16 kb[3][UM * kD];          // kbar of U as hi, mid, lo bf16 parts
    int ulist[UM];
    float acell[UM];                       // a_c of the union cells (prior, readout reference)
    uint8_t amask[UM];                     // bit g: admitted for prefix n_min + g
    uint32_t admit[5][(UM + 31) / 32];     // per prefix n_min + g: admitted union positions
    int warp_cnt[4];
    float amax_w[4];                       // per warp: largest a_c of its union positions
    int nU, ncand;
    uint64_t q_full, kb_ready, s_full, drain;
    uint4 hmask[BM][2];                    // per row and half: its selected union positions
    uint32_t tmem_base;
    int abort;
};

struct SelArgs {
    int Nq, Nk, q0, w, C, K, W, P, H;
    int tl_words;           // words per (b, h) of the member lists (with tlist)
    int tp_words;           // words per (b, h, tile) of the tiles' TopP lists (with tplist)
    int prune, has_prior;
    float scale;
};
// The eq. (7) prior's per-head parameters travel only with the instantiation that uses
// them: a kernel's argument block is copied at every launch, so the prior-free launch
// stays small.
struct SelPrior {
    float lambda[FS_MAX_HEADS];
    float inv2sigma[FS_MAX_HEADS];
};
template <bool PRIOR> struct SelArgsT : SelArgs {};
template <> struct SelArgsT<true> : SelArgs {
    SelPrior pr;
};

__device__ __forceinline__ void sel_sync() {
    asm volatile("bar.sync %0, %1;" ::"n"(kSelBarrier), "n"(NROWW * 32) : "memory");
}
__device__ __forceinline__ void srch_sync() {
    asm volatile("bar.sync %0, %1;" ::"n"(kSrchBarrier), "n"(NSRCHW * 32) : "memory");
}

// The rows' integer keys in shared memory, over the Q tile and the mean-key parts once the
// score MMA has read them: row r's 16-byte chunk c (keys 4c .. 4c + 3).  With UM = 80 a row
// takes 21 chunks (one of padding), so eight consecutive rows start in eight different
// bank groups; with UM = 128 (32 chunks, no room to pad) chunk c is stored at c ^ (r mod 8).
template <int UM> __device__ __forceinline__ int key_chunk(int r, int c) {
    if constexpr (UM == 128) return r * 32 + (c ^ (r & 7));
    else return r * (UM / 4 + 1) + c;
}
template <int UM> constexpr size_t key_bytes() { return (size_t)BM * (UM == 128 ? 32 : UM / 4 + 1) * 16; }
template <int UM> constexpr bool keys_fit() {
    return offsetof(SelSmem<UM>, kb) == sizeof(SelSmem<UM>::q) &&
           key_bytes<UM>() <= sizeof(SelSmem<UM>::q) + sizeof(SelSmem<UM>::kb);
}
static_assert(keys_fit<80>() && keys_fit<UMAX>(), "the keys fit over Q and the mean-key parts");

// K-th largest key of one row, by two threads (lanes l and l + 16 of a warp, each holding
// half of the row's keys): the bisection on c(x) = count(key >= x) with the stopping rule of
// the one-thread search, every count the sum of the two halves' (one shuffle).  The loop
// runs while any row of the warp is still searching; a finished row's threads take part in
// the shuffles without updating.  Writes the half's selected union positions.
template <int UM>
__device__ __forceinline__ void search_half(const uint4 *keys, uint4 (*hmask)[2], int K, int warp, int lane) {
    constexpr int HK = UM / 2, HC = HK / 4;     // keys and 16-byte chunks per half
    const int srow = 16 * warp + (lane & 15), half = lane >> 4;
    uint32_t key[HK];
#pragma unroll
    for (int j = 0; j < HC; j++) {
        const uint4 v = keys[key_chunk<UM>(srow, half * HC + j)];
        key[4 * j] = v.x; key[4 * j + 1] = v.y; key[4 * j + 2] = v.z; key[4 * j + 3] = v.w;
    }
    int nh = 0;
#pragma unroll
    for (int u = 0; u < HK; u++) nh += key[u] != 0u;
    const int na = nh + __shfl_xor_sync(kFull, nh, 16);
    uint32_t lo = 1u << 7, hi = (0x1000000u + 1u) << 7;
    int clo = na, chi = 0;
    const bool active = na > K;
    auto going = [&]() { return active && clo > K + 1 && chi < K - 1 && hi - lo > 1u; };
    while (__any_sync(kFull, going())) {
        const bool go = going();
        const uint32_t mid = lo + ((hi - lo) >> 1);
        int cp[4] = {0, 0, 0, 0};               // independent partial counts
#pragma unroll
        for (int u = 0; u < HK; u++) cp[u & 3] += key[u] >= mid;
        int cnt = (cp[0] + cp[1]) + (cp[2] + cp[3]);
        cnt += __shfl_xor_sync(kFull, cnt, 16);
        if (go) {
            if (cnt >= K) { lo = mid; clo = cnt; }
            else { hi = mid; chi = cnt; }
        }
    }
    // the bracket pins the K-th key: c(lo) = K, or the (K+1)-th key is the smallest >= lo, or
    // (c(hi) = K - 1) the K-th key is the largest < hi; both extremes over the row's halves
    uint32_t m0 = 0xffffffffu, m1 = 0u;
#pragma unroll
    for (int u = 0; u < HK; u++) {
        m0 = key[u] >= lo ? min(m0, key[u]) : m0;
        m1 = key[u] < hi ? max(m1, key[u]) : m1;
    }
    m0 = min(m0, __shfl_xor_sync(kFull, m0, 16));
    m1 = max(m1, __shfl_xor_sync(kFull, m1, 16));
    const uint32_t tau = !active ? 1u : clo == K ? lo : clo == K + 1 ? m0 + 1u : m1;
    uint32_t w[HK / 32 + 1];
#pragma unroll
    for (int b = 0; b <= HK / 32; b++) w[b] = 0u;
#pragma unroll
    for (int u = 0; u < HK; u++)
        if (key[u] >= tau && key[u] != 0u) w[u >> 5] |= 1u << (u & 31);
    // the half's bits at union positions half * HK + u, as a 128-bit mask
    uint32_t o[4] = {0u, 0u, 0u, 0u};
    if (half == 0) {
#pragma unroll
        for (int b = 0; b <= HK / 32; b++) o[b] = w[b];
    } else {
        constexpr int s0 = HK >> 5, sh = HK & 31;   // HK = 32 s0 + sh
#pragma unroll
        for (int b = 0; b <= HK / 32; b++) {
            if constexpr (sh == 0) {
                if (s0 + b < 4) o[s0 + b] |= w[b];
            } else {
                if (s0 + b < 4) o[s0 + b] |= w[b] << sh;
                if (s0 + b + 1 < 4) o[s0 + b + 1] |= w[b] >> (32 - sh);
            }
        }
    }
    hmask[srow][half] = make_uint4(o[0], o[1], o[2], o[3]);
}

__device__ __forceinline__ void split3(float x, __nv_bfloat16 &hi, __nv_bfloat16 &mid, __nv_bfloat16 &lo) {
    hi = __float2bfloat16_rn(x);
    const float r1 = x - __bfloat162float(hi);
    mid = __float2bfloat16_rn(r1);
    lo = __float2bfloat16_rn(r1 - __bfloat162float(mid));
}
}  // namespace

// UM = 80 (|U| <= 80: three CTAs of nine warps per SM, 72 registers a thread) or 128 (two
// CTAs per SM)
template <bool PRIOR, int UM>
__global__ void __launch_bounds__(NTHREADS, UM <= 80 ? 3 : 2)
select_tc_kernel(const __grid_constant__ CUtensorMap tq, const SelArgsT<PRIOR> A, const float *__restrict__ kbar,
                 const float *__restrict__ amax, const int *__restrict__ exitn,
                 int32_t *__restrict__ idx, uint32_t *__restrict__ tiles, int *dev_flag,
                 const int *__restrict__ tlist, const int *__restrict__ tplist) {
    extern __shared__ uint8_t smraw[];
    const uint32_t sbase = tc::smem_u32(smraw);
    SelSmem<UM> &sm = *reinterpret_cast<SelSmem<UM> *>(smraw + (((sbase + 1023u) & ~1023u) - sbase));
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
        tc::mbar_init(&sm.kb_ready, 128);
        tc::mbar_init(&sm.s_full, 1);
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
    griddep_wait();                             // the summaries and exit times are complete

    if (warp == W_MMA) {
        if (lane == 0) {
            tc::prefetch_tmap(&tq);
            tc::mbar_expect_tx(&sm.q_full, TILE_BYTES);
            tc::tma_load_3d(sm.q, &tq, &sm.q_full, 0, r0, bh);
            bool ok = tc::mbar_wait(&sm.kb_ready, 0, ab) && tc::mbar_wait(&sm.q_full, 0, ab);
            if (ok) {
                tc::tc_fence_after();
                const int N = max(16, (sm.nU + 15) & ~15);
                const uint32_t id = tc::idesc_bf16(BM, N, false, false);
                const uint32_t qa = tc::smem_u32(sm.q);
#pragma unroll
                for (int part = 0; part < 3; part++) {
                    const uint32_t kb = tc::smem_u32(sm.kb[part]);
#pragma unroll
                    for (int kk = 0; kk < kD / 16; kk++)
                        tc::mma_ss(tmem, tc::sdesc_sw128(qa + kk * 32, 16, 1024),
                                   tc::sdesc_sw128(kb + kk * 32, 16, 1024), id, (part | kk) ? 1u : 0u);
                }
                tc::mma_commit(&sm.s_full);
                tc::mma_commit(&sm.drain);
                const uint64_t t0 = tc::globaltimer();
                while (!tc::mbar_try_wait(&sm.drain, 0) && tc::globaltimer() - t0 < tc::kWaitLimitNs) {
                }
            }
        }
    } else if (warp >= NROWW) {
        // ---- helper warps: the K-th search of rows 16 (warp) .. 16 (warp) + 15, once the row
        // threads have written every row's keys
        srch_sync();
        search_half<UM>(reinterpret_cast<const uint4 *>(sm.q), sm.hmask, A.K, warp, lane);
        srch_sync();
    } else {
        const int t = threadIdx.x;     // 0..127: union builder, then the row this thread owns
        // ---- U: ordered union of the admitted sets of the tile's prefixes n_min..n_max
        const int *ex = exitn + (size_t)bh * A.C;
        const float *am = amax + (size_t)bh * A.C;
        const int ng = n_max - n_min;   // <= 4
        int total = 0;
        // admission bits of cell c (exit time e) for the prefixes n_min + g
        auto admit_bits = [&](int c, int e) {
            uint32_t m = 0;
#pragma unroll
            for (int g = 0; g <= 4; g++) {
                const int n = n_min + g;
                if (g <= ng && c < n && (!A.prune || c >= n - A.W || n < e)) m |= 1u << g;
            }
            return m;
        };
        if (tlist) {
            // decoding: the candidates are the cells listed as TopP members at an asked prefix
            // and the recent cells [n_min - W, n_max); listed cells older than that range are
            // ordered by counting, and the recent ones follow in index order
            const int *tl = tlist + (size_t)bh * A.tl_words;
            const int nl = min(__ldg(tl), A.tl_words - 1);
            const int rlo = max(0, n_min - A.W);
            int *cand = reinterpret_cast<int *>(sm.kb[0]);             // scratch until staging
            uint8_t *cmask = reinterpret_cast<uint8_t *>(sm.kb[1]);
            if (t == 0) sm.ncand = 0;
            sel_sync();
            for (int j = t; j < nl; j += 128) {
                const int c = __ldg(tl + 1 + j);
                if (c >= 0 && c < rlo) {
                    const uint32_t m = admit_bits(c, ex[c]);
                    if (m) {
                        const int slot = atomicAdd(&sm.ncand, 1);
                        cand[slot] = c;
                        cmask[slot] = (uint8_t)m;
                    }
                }
            }
            sel_sync();
            const int nc = sm.ncand;
            for (int j = t; j < nc; j += 128) {
                const int c = cand[j];
                int rank = 0;
                for (int x = 0; x < nc; x++) rank += cand[x] < c;
                if (rank < UM) {
                    sm.ulist[rank] = c;
                    sm.amask[rank] = cmask[j];
                    sm.acell[rank] = am[c];
                }
            }
            if (warp == 0) {
                int pos = nc;
                for (int c0 = rlo; c0 < n_max; c0 += 32) {
                    const int c = c0 + lane;
                    const uint32_t m = c < n_max ? admit_bits(c, __ldg(ex + c)) : 0u;
                    const unsigned bal = __ballot_sync(kFull, m != 0u);
                    const int p = pos + __popc(bal & ((1u << lane) - 1u));
                    if (m && p < UM) {
                        sm.ulist[p] = c;
                        sm.amask[p] = (uint8_t)m;
                        sm.acell[p] = am[c];
                    }
                    pos += __popc(bal);
                }
                if (lane == 0) sm.warp_cnt[0] = pos;
            }
            sel_sync();
            total = sm.warp_cnt[0];
            sel_sync();
        } else if (tplist) {
            // prefill with W >= 1: U is TopP(n_min) below the recent range, then the recent
            // range [n_min - W, n_max) itself (every cell there is recent for some prefix of
            // the tile); TopP(n_min) comes ascending from the tile-list kernel
            const int *lst = tplist + ((size_t)bh * gridDim.x + blockIdx.x) * A.tp_words;
            const int nl = min(__ldg(lst), A.tp_words - 1);
            const int rlo = max(0, n_min - A.W);
            if (t == 0) sm.ncand = 0;
            sel_sync();
            if (t < nl) {                       // members below rlo form a prefix of the list
                const bool below = __ldg(lst + 1 + t) < rlo;
                const bool next_below = t + 1 < nl && __ldg(lst + 2 + t) < rlo;
                if (below && !next_below) sm.ncand = t + 1;
            }
            sel_sync();
            const int nold = sm.ncand;
            total = nold + max(0, n_max - rlo);
            for (int u = t; u < min(total, UM); u += 128) {
                const int c = u < nold ? __ldg(lst + 1 + u) : rlo + (u - nold);
                sm.ulist[u] = c;
                sm.amask[u] = (uint8_t)admit_bits(c, __ldg(ex + c));
                sm.acell[u] = am[c];
            }
            sel_sync();
        } else {
            // 1024 cells per round, eight consecutive ones per thread: the exit times are
            // fetched with two 16-byte loads before any of them is used, then one block-wide
            // exclusive scan orders the members
            for (int c0 = 0; c0 < n_max; c0 += 1024) {
                const int cb = c0 + 8 * t;
                int e8[8];
                if (A.prune && cb + 8 <= n_max && (reinterpret_cast<uintptr_t>(ex + cb) & 15) == 0) {
                    const int4 x0 = __ldg(reinterpret_cast<const int4 *>(ex + cb));
                    const int4 x1 = __ldg(reinterpret_cast<const int4 *>(ex + cb) + 1);
                    e8[0] = x0.x; e8[1] = x0.y; e8[2] = x0.z; e8[3] = x0.w;
                    e8[4] = x1.x; e8[5] = x1.y; e8[6] = x1.z; e8[7] = x1.w;
                } else {
    #pragma unroll
                    for (int j = 0; j < 8; j++) e8[j] = (A.prune && cb + j < n_max) ? ex[cb + j] : 0;
                }
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
                sel_sync();
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
                            sm.acell[pos] = am[cb + j];
                        }
                        pos++;
                    }
                }
                total += tot;
                sel_sync();
            }
        }
        if (t == 0) {
            sm.nU = min(total, UM);
            if (total > UM && dev_flag) atomicExch(dev_flag, kFlagCheck);
        }
        sel_sync();
        const int nU = min(total, UM);
        constexpr int NW = (UM + 31) / 32;      // admission words
        {   // admission masks per prefix, one 32-position word per warp; the largest a_c of U
            const float au = warp_max(t < nU ? sm.acell[t] : 0.f);
            if (lane == 0) sm.amax_w[warp] = au;
            const uint32_t am = t < nU ? sm.amask[t] : 0u;
#pragma unroll
            for (int gg = 0; gg < 5; gg++) {
                const uint32_t word = __ballot_sync(kFull, (am >> gg) & 1u);
                if (lane == 0 && warp < NW) sm.admit[gg][warp] = word;
            }
        }
        // ---- kbar of U as three bf16 parts, row u = union position (zero rows pad to 16)
        const int N = max(16, (nU + 15) & ~15);
        if (t < N) {
            const float4 *src = reinterpret_cast<const float4 *>(kbar + ((size_t)bh * A.C + (t < nU ? sm.ulist[t] : 0)) * kD);
#pragma unroll
            for (int j = 0; j < 8; j++) {            // 16-byte chunk j = elements 8j..8j+7
                float x[8];
                if (t < nU) {
                    const float4 a = __ldg(src + 2 * j), b = __ldg(src + 2 * j + 1);
                    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w; x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
                } else {
#pragma unroll
                    for (int e = 0; e < 8; e++) x[e] = 0.f;
                }
                __align__(16) __nv_bfloat16 hi[8], mi[8], lo[8];
#pragma unroll
                for (int e = 0; e < 8; e++) split3(x[e], hi[e], mi[e], lo[e]);
                const int off = t * kD + ((j ^ (t & 7)) << 3);
                *reinterpret_cast<uint4 *>(&sm.kb[0][off]) = *reinterpret_cast<const uint4 *>(hi);
                *reinterpret_cast<uint4 *>(&sm.kb[1][off]) = *reinterpret_cast<const uint4 *>(mi);
                *reinterpret_cast<uint4 *>(&sm.kb[2][off]) = *reinterpret_cast<const uint4 *>(lo);
            }
        }
        tc::fence_async_shared();
        tc::mbar_arrive(&sm.kb_ready);

        // ---- this thread's row: scores -> admitted keys (to shared memory) -> K best (eight
        // warps, two threads per row) -> the row's record
        const int row = t;
        const int i = pb + row;
        const int n_r = cand_count(i, A.w, A.C);
        const int g = n_r - n_min;
        const bool ok = tc::mbar_wait(&sm.s_full, 0, ab) && (!tiles || tc::mbar_wait(&sm.q_full, 0, ab));
        const uint32_t trow = tmem + ((uint32_t)(warp * 32) << 16);
        float lam = 0.f, i2s = 0.f;
        if constexpr (PRIOR) {
            lam = A.pr.lambda[h];
            i2s = A.pr.inv2sigma[h];
        }
        uint32_t aw[NW];                            // admitted union positions of this row
#pragma unroll
        for (int b = 0; b < NW; b++) aw[b] = row < nrows ? sm.admit[g][b] : 0u;
        int na = 0;
#pragma unroll
        for (int b = 0; b < NW; b++) na += __popc(aw[b]);
        float qq = 0.f;                             // |q|^2 of this row, before the keys cover Q
        if (ok && tiles) {
            const uint8_t *qrow = reinterpret_cast<const uint8_t *>(sm.q) + row * 128;
#pragma unroll
            for (int j = 0; j < 8; j++) {
                const uint4 v = *reinterpret_cast<const uint4 *>(qrow + ((j ^ (row & 7)) << 4));
                const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int e = 0; e < 4; e++) {
                    const float lo = __uint_as_float(w4[e] << 16), hi = __uint_as_float(w4[e] & 0xffff0000u);
                    qq = fmaf(lo, lo, fmaf(hi, hi, qq));
                }
            }
        }
        // score r_ic of union position u from its raw product (the same arithmetic in both passes)
        auto score = [&](uint32_t raw, int u) {
            float sc = __uint_as_float(raw) * A.scale;
            if (PRIOR) {
                const float pc = (float)(sm.ulist[u] * kS) + 0.5f * kS;
                sc += lam * sm.acell[u] * erff(((float)i - pc) * i2s);
            }
            return sc;
        };
        float smax = -INFINITY;
        if (ok) {
            tc::tc_fence_after();
            // pass 1: the range of the admitted scores, 16 columns at a time
            float fmn[4], fmx[4];
#pragma unroll
            for (int k = 0; k < 4; k++) { fmn[k] = INFINITY; fmx[k] = -INFINITY; }
#pragma unroll
            for (int b = 0; b < UM / 16; b++) {
                if (16 * b < N) {
                    uint32_t r[16];
                    tc::tmem_ld16(trow + 16 * b, r);
                    tc::tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 16; e++) {
                        const int u = 16 * b + e;
                        const float sc = score(r[e], u);
                        const bool adm = (aw[u >> 5] >> (u & 31)) & 1u;
                        fmn[e & 3] = adm ? fminf(fmn[e & 3], sc) : fmn[e & 3];
                        fmx[e & 3] = adm ? fmaxf(fmx[e & 3], sc) : fmx[e & 3];
                    }
                }
            }
            const float mn = fminf(fminf(fmn[0], fmn[1]), fminf(fmn[2], fmn[3]));
            smax = fmaxf(fmaxf(fmx[0], fmx[1]), fmaxf(fmx[2], fmx[3]));
            const float span = smax - mn;
            const float q24 = span > 0.f ? 16777215.f / span : 0.f;
            // every row thread has read Q (and the MMA has read Q and the mean keys)
            sel_sync();
            // pass 2: integer keys, 1 + the score's 24-bit fixed-point place in the row's range,
            // then 7 bits of (127 - position); 0 for a cell that is not admitted (and for the
            // columns past N)
            uint4 *kdst = reinterpret_cast<uint4 *>(sm.q);
#pragma unroll
            for (int b = 0; b < UM / 16; b++) {
                uint32_t r[16];
                if (16 * b < N) {
                    tc::tmem_ld16(trow + 16 * b, r);
                    tc::tmem_wait_ld();
                }
#pragma unroll
                for (int e = 0; e < 16; e++) {
                    const int u = 16 * b + e;
                    uint32_t key = 0u;
                    if (16 * b < N) {
                        const bool adm = (aw[u >> 5] >> (u & 31)) & 1u;
                        const uint32_t fx = min(__float2uint_rz((score(r[e], u) - mn) * q24), 0xffffffu);
                        key = adm ? ((fx + 1u) << 7) | (uint32_t)(127 - u) : 0u;
                    }
                    r[e] = key;
                }
#pragma unroll
                for (int c = 0; c < 4; c++)
                    kdst[key_chunk<UM>(row, 4 * b + c)] = make_uint4(r[4 * c], r[4 * c + 1], r[4 * c + 2], r[4 * c + 3]);
            }
        } else {
            sel_sync();
        }
        srch_sync();
        search_half<UM>(reinterpret_cast<const uint4 *>(sm.q), sm.hmask, A.K, warp, lane);
        srch_sync();
        if (ok) {
            uint32_t mw[UMAX / 32];                 // selected union positions
            {
                const uint4 h0 = sm.hmask[row][0], h1 = sm.hmask[row][1];
                mw[0] = h0.x | h1.x; mw[1] = h0.y | h1.y; mw[2] = h0.z | h1.z; mw[3] = h0.w | h1.w;
            }
            if (tiles) {   // compact record for the fused kernel: row masks | union | |U| | reference
                // Readout reference (log2 units): every NoPE logit q.k_j / sqrt(d) of a selected
                // token is at most |q| max_{c in U} a_c / sqrt(d) (Cauchy-Schwarz), and the
                // largest is at least any selected cell's mean-key logit q.kbar_c / sqrt(d) (a
                // maximum is at least the mean).  The row's best admitted cell is always
                // selected; without the prior its eq. (7) score is that mean-key logit, with
                // the prior the selected cells' raw products are read again from tensor
                // memory.  Where the two bounds lie within kMrefMaxGap, the upper one serves
                // as the softmax's fixed reference (no running maximum).
                const float c = A.scale * 1.4426950408889634f;
                float lower = smax * 1.4426950408889634f;
                if (PRIOR) {
                    // warp-collective loads (.sync.aligned): every lane issues them
                    float dmax = -INFINITY;
#pragma unroll
                    for (int b = 0; b < UM / 16; b++) {
                        if (16 * b < N) {
                            uint32_t raw[16];
                            tc::tmem_ld16(trow + 16 * b, raw);
                            tc::tmem_wait_ld();
#pragma unroll
                            for (int e = 0; e < 16; e++) {
                                const int u = 16 * b + e;
                                if ((mw[u >> 5] >> (u & 31)) & 1u) dmax = fmaxf(dmax, __uint_as_float(raw[e]));
                            }
                        }
                    }
                    lower = dmax * c;
                }
                float mref = 0.f;
                if (na > 0) {
                    // |q| of this row (read from the tile before the keys covered it)
                    const float amx = fmaxf(fmaxf(sm.amax_w[0], sm.amax_w[1]), fmaxf(sm.amax_w[2], sm.amax_w[3]));
                    const float ub = sqrtf(qq) * amx * c;
                    mref = (ub - lower <= kMrefMaxGap) ? ub : __uint_as_float(0x7fc00000u);
                }
                uint32_t *rec = tiles + ((size_t)bh * gridDim.x + blockIdx.x) * kTileRecWords;
                *reinterpret_cast<uint4 *>(rec + kTileMaskOff + 4 * row) = make_uint4(mw[0], mw[1], mw[2], mw[3]);
                rec[kTileUlistOff + t] = t < nU ? (uint32_t)sm.ulist[t] : 0xffffffffu;
                rec[kTileMrefOff + row] = __float_as_uint(mref);
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

bool select_tc_supported(const fs_params *p) {
    if (p->dtype != FS_BF16) return false;
    const int C = p->Nk / p->s;
    const int bound = p->W >= 0 ? p->W + p->P + 10 : C;
    return bound <= UMAX;
}

namespace {
// the largest union a tile of this call can have (W + P + 10 with pruning, else C)
int union_bound(const Dev &P) { return P.prune ? P.W + P.P + 10 : P.C; }
// the erf prior is a separate instantiation: without it the unrolled score loop stays small
template <bool PRIOR, int UM>
cudaError_t launch_um(const CUtensorMap &tq, const SelArgsT<PRIOR> &A, dim3 grid, const float *kbar,
                      const float *amax, const int *exitn, int32_t *idx, uint32_t *tiles, int *dev_flag,
                      const int *tlist, const int *tplist, cudaStream_t st) {
    const size_t smem = sizeof(SelSmem<UM>) + 1024;
    auto kern = select_tc_kernel<PRIOR, UM>;
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    return launch_pdl(kern, grid, dim3(NTHREADS), smem, st, tq, A, kbar, amax, exitn, idx, tiles, dev_flag, tlist,
                      tplist);
}
template <bool PRIOR>
cudaError_t launch_sel(const Dev &P, const CUtensorMap &tq, const SelArgsT<PRIOR> &A, dim3 grid, const float *kbar,
                       const float *amax, const int *exitn, int32_t *idx, uint32_t *tiles, int *dev_flag,
                       const int *tlist, const int *tplist, cudaStream_t st) {
    if (union_bound(P) <= 80)
        return launch_um<PRIOR, 80>(tq, A, grid, kbar, amax, exitn, idx, tiles, dev_flag, tlist, tplist, st);
    return launch_um<PRIOR, UMAX>(tq, A, grid, kbar, amax, exitn, idx, tiles, dev_flag, tlist, tplist, st);
}
}  // namespace

cudaError_t launch_select_tc(const Dev &P, const void *Q, const float *kbar, const float *amax,
                             const int *exitn, int32_t *idx, uint32_t *tiles, int *dev_flag,
                             cudaStream_t st, const int *tlist, const int *tplist) {
    if (P.Nq == 0) return cudaSuccess;
    const int BH = P.B * P.H;
    CUtensorMap tq;
    if (!encode_tmap_3d_bf16(&tq, Q, kD, P.Nq, BH, kD, BM)) return cudaErrorInvalidValue;
    SelArgsT<true> A;
    A.Nq = P.Nq; A.Nk = P.Nk; A.q0 = P.q0; A.w = P.w; A.C = P.C; A.K = P.K;
    A.W = P.W; A.P = P.P; A.H = P.H; A.prune = P.prune; A.has_prior = P.has_prior;
    A.scale = P.scale;
    A.tl_words = exit_list_words(P.P);
    A.tp_words = tile_list_words(P);
    if (!P.prune) tlist = nullptr;
    if (tlist || A.tp_words == 0) tplist = nullptr;
    const dim3 grid((P.Nq + BM - 1) / BM, BH);
    LaunchScope scope(kSelectTc, st);
    if (!P.has_prior) {
        SelArgsT<false> A0;
        static_cast<SelArgs &>(A0) = A;         // the common part only
        return launch_sel<false>(P, tq, A0, grid, kbar, amax, exitn, idx, tiles, dev_flag, tlist, tplist, st);
    }
    for (int h = 0; h < FS_MAX_HEADS; h++) {
        A.pr.lambda[h] = P.lambda[h];
        A.pr.inv2sigma[h] = P.inv2sigma[h];
    }
    return launch_sel<true>(P, tq, A, grid, kbar, amax, exitn, idx, tiles, dev_flag, tlist, tplist, st);
}

}  // namespace fs
