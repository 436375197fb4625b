// FS-L streaming cache: the forward pass over a token stream with bounded state per head,
// "FreeSolo" summary, "Practical Implications" 3 (O((P+W)s + w + B + s)d token state per
// head) and §3.3 eq. (8).  Same arithmetic as the batch forward pass (§3.1 eq. (2), §3.2
// eqs. (3)-(4), §3.3 eqs. (5), (7), (9)); what differs is where the keys and values live.
//
// State of one (batch, head):
//   - a ring of the last R = roundup(max_block + w + 2s, s) tokens: raw keys, keys rotated
//     by their absolute positions (double-precision angles), values.  It holds the window
//     of every query still to come and the cells that are not candidates yet;
//   - M = W + P + 2 * ceil(max_block / s) + 4 cell slots: the candidate cells that a query
//     still to come may admit, each with its keys, values, mean key, max norm, and the
//     prefix at which it left TopP (never, while a member; c + 1 if it never entered).
//
// Why dropping cells is exact: a cell's rank by max norm among the prefix never improves
// as the prefix grows (cells only join), so once out of TopP it never returns, and once
// older than the W most recent candidates it never becomes recent again.  A cell is freed
// when no prefix that the next attend call can reach admits it.
//
// fs_cache_append: one CTA per (b, h).  New tokens go into the ring; then each cell that
// the new tokens make a candidate is processed in order: its max norm is computed, it joins
// TopP if it beats the weakest member (the weakest leaves at that prefix), and it takes a
// slot if some reachable prefix can admit it.  Keys, values and mean keys are copied into
// the slots last, in parallel.
// fs_cache_attend: one CTA per (query, b, h): admission and scores over the slots, top-K,
// NoPE readout over the selected cells' tokens, RMSNorm, RoPE window over the ring,
// combination.  CUDA cores: a decode step has a handful of queries per head.
#include <cmath>
#include <cstring>

#include "fs_common.cuh"

namespace fs {
namespace {

constexpr int kMaxBlock = 65536;
constexpr int kAppendThreads = 256, kAttendThreads = 128;
constexpr int kFlagOff = 0;                     // int error flag at the start of the cache
constexpr size_t kHeadBytes = 256;

size_t a256(size_t x) { return (x + 255) & ~size_t(255); }

// Byte layout of one (b, h) state block; the cache is a 256-byte header, then B*H blocks.
struct CacheGeom {
    int R, M, maxnew;
    size_t elem;
    size_t o_t, o_rk, o_rr, o_rv, o_cell, o_exit, o_a, o_kbar, o_ck, o_cv, bh_bytes;
};

CacheGeom cache_geom(const fs_params *p, int max_block) {
    CacheGeom g;
    g.R = ((max_block + p->w + 2 * kS + kS - 1) / kS) * kS;
    g.maxnew = (max_block + kS - 1) / kS + 1;   // cells that can become candidates per append
    g.M = p->W + p->P + 2 * g.maxnew + 2;
    g.elem = p->dtype == FS_BF16 ? 2 : 4;
    size_t off = 0;
    auto seg = [&](size_t bytes) {
        const size_t o = off;
        off += a256(bytes);
        return o;
    };
    g.o_t = seg(64);                                        // tokens appended so far (int64)
    g.o_rk = seg((size_t)g.R * kD * g.elem);                // ring: raw keys
    g.o_rr = seg((size_t)g.R * kD * g.elem);                // ring: rotated keys
    g.o_rv = seg((size_t)g.R * kD * g.elem);                // ring: values
    g.o_cell = seg((size_t)g.M * 4);                        // slot -> cell index (-1 free)
    g.o_exit = seg((size_t)g.M * 4);                        // prefix at which it left TopP
    g.o_a = seg((size_t)g.M * 4);                           // max key norm
    g.o_kbar = seg((size_t)g.M * kD * 4);                   // mean key (float32)
    g.o_ck = seg((size_t)g.M * kS * kD * g.elem);           // the cell's keys
    g.o_cv = seg((size_t)g.M * kS * kD * g.elem);           // the cell's values
    g.bh_bytes = off;
    return g;
}

struct CacheArgs {
    int R, M, maxnew, max_block;
    int w, K, W, P, H;
    int has_prior;
    double rope_base;
    float scale;       // 1 / sqrt(d)
    float rms_eps;
    size_t o_t, o_rk, o_rr, o_rv, o_cell, o_exit, o_a, o_kbar, o_ck, o_cv, bh_bytes;
    float alpha[FS_MAX_HEADS];
    float lambda[FS_MAX_HEADS];
    float inv2sigma[FS_MAX_HEADS];
};

// |C_i| for position i of an unbounded stream: cells with (c+1)s <= i - w
__device__ __forceinline__ int cand_count_ll(long long i, int w) {
    const long long lim = i - w;
    return lim < kS ? 0 : (int)(lim / kS);
}

// (cos, sin)(pos * theta_m), theta_m = base^(-2m/d), in double precision
__device__ __forceinline__ void rope_cs(long long pos, int m, double base, float &c, float &s) {
    const double theta = pow(base, -2.0 * m / (double)kD);
    double sn, cs;
    sincos((double)pos * theta, &sn, &cs);
    c = (float)cs;
    s = (float)sn;
}

struct Slots {   // pointers into one (b, h) block
    long long *t;
    uint8_t *rk, *rr, *rv;
    int *cell, *exit;
    float *a, *kbar;
    uint8_t *ck, *cv;
};
__device__ __forceinline__ Slots slots_of(uint8_t *cache, const CacheArgs &A, int bh) {
    uint8_t *b = cache + kHeadBytes + (size_t)bh * A.bh_bytes;
    Slots S;
    S.t = reinterpret_cast<long long *>(b + A.o_t);
    S.rk = b + A.o_rk; S.rr = b + A.o_rr; S.rv = b + A.o_rv;
    S.cell = reinterpret_cast<int *>(b + A.o_cell);
    S.exit = reinterpret_cast<int *>(b + A.o_exit);
    S.a = reinterpret_cast<float *>(b + A.o_a);
    S.kbar = reinterpret_cast<float *>(b + A.o_kbar);
    S.ck = b + A.o_ck; S.cv = b + A.o_cv;
    return S;
}

template <typename T>
__global__ void __launch_bounds__(kAppendThreads) cache_append_kernel(uint8_t *cache, const T *__restrict__ Kn,
                                                                      const T *__restrict__ Vn, int n_new,
                                                                      const CacheArgs A) {
    extern __shared__ int sh[];                  // slot of each new cell [maxnew], its norm [maxnew]
    int *s_slot = sh;
    float *s_a = reinterpret_cast<float *>(sh + A.maxnew);
    __shared__ int s_err;
    const int bh = blockIdx.x, t = threadIdx.x, lane = t & 31, warp = t >> 5;
    constexpr int NW = kAppendThreads / 32;
    const Slots S = slots_of(cache, A, bh);
    int *flag = reinterpret_cast<int *>(cache + kFlagOff);
    T *rk = reinterpret_cast<T *>(S.rk), *rr = reinterpret_cast<T *>(S.rr), *rv = reinterpret_cast<T *>(S.rv);
    T *ck = reinterpret_cast<T *>(S.ck), *cv = reinterpret_cast<T *>(S.cv);
    const long long t0 = *S.t, t1 = t0 + n_new;

    // 1. the new tokens into the ring: raw key, key rotated by its absolute position, value
    for (int item = t; item < n_new * (kD / 2); item += kAppendThreads) {
        const int j = item / (kD / 2), m = item % (kD / 2);
        const long long pos = t0 + j;
        const size_t src = ((size_t)bh * n_new + j) * kD + 2 * m;
        const size_t dst = (size_t)(pos % A.R) * kD + 2 * m;
        const float k0 = to_f<T>(Kn[src]), k1 = to_f<T>(Kn[src + 1]);
        float c, sn;
        rope_cs(pos, m, A.rope_base, c, sn);
        rk[dst] = Kn[src];
        rk[dst + 1] = Kn[src + 1];
        rr[dst] = from_f<T>(k0 * c - k1 * sn);
        rr[dst + 1] = from_f<T>(k0 * sn + k1 * c);
        rv[dst] = Vn[src];
        rv[dst + 1] = Vn[src + 1];
    }
    // cells nA .. nB-1 become candidates; a later attend reaches prefixes >= nlo
    const int nA = cand_count_ll(t0 - 1, A.w), nB = cand_count_ll(t1 - 1, A.w);
    const long long qlo = t1 - A.max_block;
    const int nlo = cand_count_ll(qlo < 0 ? 0 : qlo, A.w);
    const int nc = nB - nA;
    if (t == 0) s_err = (nc < 0 || nc > A.maxnew) ? 1 : 0;
    for (int k = t; k < A.maxnew; k += kAppendThreads) s_slot[k] = -1;
    // free the slots no reachable prefix admits (older than the recent W of prefix nlo, and
    // out of TopP by then)
    for (int x = t; x < A.M; x += kAppendThreads) {
        const int c = S.cell[x];
        if (c >= 0 && c < nlo - A.W && S.exit[x] <= nlo) S.cell[x] = -1;
    }
    __syncthreads();
    if (s_err) {
        if (t == 0) atomicExch(flag, kFlagCheck);
        return;
    }

    // 2. max key norm of each new candidate cell (eq. (5)): one warp per cell, lane = token
    for (int k = warp; k < nc; k += NW) {
        const long long pos = (long long)(nA + k) * kS + lane;
        const T *row = rk + (size_t)(pos % A.R) * kD;
        float ss = 0.f;
#pragma unroll 8
        for (int e = 0; e < kD; e++) {
            const float x = to_f<T>(row[e]);
            ss = fmaf(x, x, ss);
        }
        const float a = warp_max(sqrtf(ss));
        if (lane == 0) s_a[k] = a;
    }
    __syncthreads();

    // 3. TopP in cell order (one warp): cell c joins TopP at prefix c+1 iff TopP has fewer
    //    than P members or c beats the weakest member (larger a; a tie goes to the lower
    //    index, the member), which then leaves at prefix c+1.  A cell takes a slot if a
    //    reachable prefix can admit it.
    if (warp == 0) {
        for (int k = 0; k < nc; k++) {
            const int c = nA + k;
            const float ac = s_a[k];
            int cnt = 0, wc = -1, wx = -1;
            float wa = INFINITY;
            for (int x = lane; x < A.M; x += 32) {
                const int cx = S.cell[x];
                if (cx >= 0 && S.exit[x] == kNever) {
                    cnt++;
                    const float ax = S.a[x];
                    if (ax < wa || (ax == wa && cx > wc)) { wa = ax; wc = cx; wx = x; }
                }
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                cnt += __shfl_xor_sync(kFull, cnt, o);
                const float a2 = __shfl_xor_sync(kFull, wa, o);
                const int c2 = __shfl_xor_sync(kFull, wc, o), x2 = __shfl_xor_sync(kFull, wx, o);
                if (a2 < wa || (a2 == wa && c2 > wc)) { wa = a2; wc = c2; wx = x2; }
            }
            const bool enters = A.P > 0 && (cnt < A.P || ac > wa);
            if (enters && cnt >= A.P && lane == 0) {
                S.exit[wx] = c + 1;
                if (wc < nlo - A.W && c + 1 <= nlo) {        // nothing reachable admits it now
                    S.cell[wx] = -1;
                    if (wc >= nA) s_slot[wc - nA] = -1;      // a cell of this append: not copied
                }
            }
            __syncwarp();
            if (enters || c >= nlo - A.W) {
                int fx = -1;
                for (int base = 0; base < A.M && fx < 0; base += 32) {
                    const int x = base + lane;
                    const unsigned m = __ballot_sync(kFull, x < A.M && S.cell[x] < 0);
                    if (m) fx = base + __ffs(m) - 1;
                }
                if (fx < 0) {                                // cannot happen with M as sized
                    if (lane == 0) atomicExch(flag, kFlagCheck);
                    break;
                }
                if (lane == 0) {
                    S.cell[fx] = c;
                    S.exit[fx] = enters ? kNever : c + 1;
                    S.a[fx] = ac;
                    s_slot[k] = fx;
                }
            }
            __syncwarp();
        }
    }
    __syncthreads();

    // 4. keys, values and mean key of each kept new cell (one warp per cell, two dims a lane)
    for (int k = warp; k < nc; k += NW) {
        const int x = s_slot[k];
        if (x < 0) continue;
        const long long p0 = (long long)(nA + k) * kS;
        float s0 = 0.f, s1 = 0.f;
        for (int j = 0; j < kS; j++) {
            const size_t src = (size_t)((p0 + j) % A.R) * kD + 2 * lane;
            const size_t dst = ((size_t)x * kS + j) * kD + 2 * lane;
            const T k0 = rk[src], k1 = rk[src + 1];
            ck[dst] = k0;
            ck[dst + 1] = k1;
            cv[dst] = rv[src];
            cv[dst + 1] = rv[src + 1];
            s0 += to_f<T>(k0);
            s1 += to_f<T>(k1);
        }
        S.kbar[(size_t)x * kD + 2 * lane] = s0 * (1.f / kS);
        S.kbar[(size_t)x * kD + 2 * lane + 1] = s1 * (1.f / kS);
    }
    __syncthreads();
    if (t == 0) *S.t = t1;
}

// Online softmax state of one warp: running max m, sum l, and two output dims per lane.
struct Online {
    float m = -INFINITY, l = 0.f, a0 = 0.f, a1 = 0.f;
    // one 32-token block: sc = this lane's score (-inf if invalid), vrow(j) = value row of token j
    template <typename T> __device__ __forceinline__ void block(float sc, const T *v, size_t vstride, int lane) {
        const float mc = warp_max(sc);
        if (mc == -INFINITY) return;
        const float mn = fmaxf(m, mc);
        const float corr = m == -INFINITY ? 0.f : expf(m - mn);
        const float p = sc == -INFINITY ? 0.f : expf(sc - mn);
        l = l * corr + warp_sum(p);
        a0 *= corr;
        a1 *= corr;
#pragma unroll 8
        for (int j = 0; j < kS; j++) {
            const float pj = __shfl_sync(kFull, p, j);
            const T *vr = v + (size_t)j * vstride + 2 * lane;
            a0 = fmaf(pj, to_f<T>(vr[0]), a0);
            a1 = fmaf(pj, to_f<T>(vr[1]), a1);
        }
        m = mn;
    }
};

// q (shared, float) . key row (global, T), 64 dims
template <typename T> __device__ __forceinline__ float dot64(const float *q, const T *k) {
    float acc = 0.f;
#pragma unroll
    for (int c = 0; c < kD / Vec<T>::N; c++) {
        float x[Vec<T>::N];
        Vec<T>::load(k + c * Vec<T>::N, x);
#pragma unroll
        for (int e = 0; e < Vec<T>::N; e++) acc = fmaf(q[c * Vec<T>::N + e], x[e], acc);
    }
    return acc;
}

// Folds the four warps' online states into out[64] = acc / l (0 where nothing was attended).
__device__ __forceinline__ void fold_warps(const Online &o, float (*s_m)[4], float (*s_l)[4], float (*s_acc)[kD],
                                           float *out, int t, int warp, int lane) {
    if (lane == 0) {
        (*s_m)[warp] = o.m;
        (*s_l)[warp] = o.l;
    }
    s_acc[warp][2 * lane] = o.a0;
    s_acc[warp][2 * lane + 1] = o.a1;
    __syncthreads();
    if (t < kD) {
        float mx = -INFINITY;
        for (int w2 = 0; w2 < 4; w2++) mx = fmaxf(mx, (*s_m)[w2]);
        float num = 0.f, den = 0.f;
        if (mx != -INFINITY)
            for (int w2 = 0; w2 < 4; w2++) {
                if ((*s_m)[w2] == -INFINITY) continue;
                const float f = expf((*s_m)[w2] - mx);
                num = fmaf(s_acc[w2][t], f, num);
                den = fmaf((*s_l)[w2], f, den);
            }
        out[t] = den > 0.f ? num / den : 0.f;
    }
    __syncthreads();
}

template <typename T, bool PRIOR>
__global__ void __launch_bounds__(kAttendThreads) cache_attend_kernel(uint8_t *cache, const T *__restrict__ Qn,
                                                                      int n_q, int32_t *__restrict__ idx,
                                                                      T *__restrict__ O, const CacheArgs A) {
    extern __shared__ int shi[];                 // per slot: score, flags (1 admitted, 2 selected), cell
    float *s_score = reinterpret_cast<float *>(shi);
    int *s_flag = shi + A.M, *s_cell = shi + 2 * A.M, *s_list = shi + 3 * A.M;   // s_list: K slots
    __shared__ float s_qn[kD], s_qr[kD], s_u[kD], s_o[kD];
    __shared__ float s_m[4], s_l[4], s_acc[4][kD], s_ss[2];
    __shared__ int s_nsel;
    const int r = blockIdx.x, bh = blockIdx.y, h = bh % A.H;
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    const Slots S = slots_of(cache, A, bh);
    const long long tt = *S.t;
    if ((long long)n_q > tt) {                   // attending positions never appended
        if (t == 0) atomicExch(reinterpret_cast<int *>(cache + kFlagOff), kFlagCheck);
        return;
    }
    const long long i = tt - n_q + r;            // this query's position
    const int n = cand_count_ll(i, A.w);         // its prefix |C_i|
    const T *q = Qn + ((size_t)bh * n_q + r) * kD;
    if (t < kD / 2) {
        const float q0 = to_f<T>(q[2 * t]), q1 = to_f<T>(q[2 * t + 1]);
        float c, sn;
        rope_cs(i, t, A.rope_base, c, sn);
        s_qn[2 * t] = q0;
        s_qn[2 * t + 1] = q1;
        s_qr[2 * t] = q0 * c - q1 * sn;
        s_qr[2 * t + 1] = q0 * sn + q1 * c;
    }
    if (t == 0) s_nsel = 0;
    __syncthreads();

    // 1. admission (eq. (8)) and scores (eq. (7)) over the slots, one warp per slot
    for (int x = warp; x < A.M; x += kAttendThreads / 32) {
        const int c = S.cell[x];
        const bool adm = c >= 0 && c < n && (c >= n - A.W || n < S.exit[x]);
        float sc = 0.f;
        if (adm) {
            const float *kb = S.kbar + (size_t)x * kD;
            sc = warp_sum(fmaf(s_qn[2 * lane], kb[2 * lane], s_qn[2 * lane + 1] * kb[2 * lane + 1])) * A.scale;
            if (PRIOR) {
                const float dpos = (float)(i - (long long)c * kS) - 0.5f * kS;   // i - p_c
                sc += A.lambda[h] * S.a[x] * erff(dpos * A.inv2sigma[h]);
            }
        }
        if (lane == 0) {
            s_score[x] = sc;
            s_flag[x] = adm ? 1 : 0;
            s_cell[x] = c;
        }
    }
    __syncthreads();
    // 2. top-K: a slot is selected if fewer than K admitted slots rank above it (higher
    //    score, or equal score and lower cell)
    for (int x = t; x < A.M; x += kAttendThreads) {
        if (!(s_flag[x] & 1)) continue;
        const float sx = s_score[x];
        const int cx = s_cell[x];
        int rank = 0;
        for (int y = 0; y < A.M; y++)
            if (s_flag[y] & 1) {
                const float sy = s_score[y];
                rank += (sy > sx) || (sy == sx && s_cell[y] < cx);
            }
        if (rank < A.K) atomicOr(&s_flag[x], 2);
    }
    __syncthreads();
    for (int x = t; x < A.M; x += kAttendThreads) {   // selected slots in ascending cell order
        if (!(s_flag[x] & 2)) continue;
        int pos = 0;
        for (int y = 0; y < A.M; y++) pos += (s_flag[y] & 2) && s_cell[y] < s_cell[x];
        s_list[pos] = x;
        atomicAdd(&s_nsel, 1);
    }
    __syncthreads();
    const int nsel = s_nsel;
    if (idx && t < A.K) idx[((size_t)bh * n_q + r) * A.K + t] = t < nsel ? s_cell[s_list[t]] : -1;

    // 3. readout (eq. (9)): NoPE softmax over every token of the selected cells; warp w
    //    takes cells w, w+4, ...; lane = token for the scores, lane = dim pair for P V
    const T *ck = reinterpret_cast<const T *>(S.ck), *cv = reinterpret_cast<const T *>(S.cv);
    Online lr;
    for (int k = warp; k < nsel; k += kAttendThreads / 32) {
        const int x = s_list[k];
        const float sc = dot64<T>(s_qn, ck + ((size_t)x * kS + lane) * kD) * A.scale;
        lr.block<T>(sc, cv + (size_t)x * kS * kD, kD, lane);
    }
    fold_warps(lr, &s_m, &s_l, s_acc, s_u, t, warp, lane);
    if (t < kD) {                                 // RMSNorm (no gain), then alpha_h
        const float ss = warp_sum(s_u[t] * s_u[t]);
        if (lane == 0) s_ss[warp] = ss;
    }
    __syncthreads();
    const float f = nsel > 0 ? A.alpha[h] / sqrtf((s_ss[0] + s_ss[1]) * (1.f / kD) + A.rms_eps) : 0.f;

    // 4. window (eqs. (3)-(4)): keys max(0, i-w) .. i from the ring, rotated by their
    //    absolute positions; 32-token blocks split over the warps
    const T *rr = reinterpret_cast<const T *>(S.rr), *rv = reinterpret_cast<const T *>(S.rv);
    const long long jlo = i - A.w < 0 ? 0 : i - A.w;
    const int L = (int)(i - jlo) + 1;
    Online sr;
    for (int b = warp; b * kS < L; b += kAttendThreads / 32) {
        const long long j = jlo + (long long)b * kS + lane;
        const bool valid = j <= i;
        const long long jj = valid ? j : i;      // any ring row in range for the idle lanes
        const float sc = valid ? dot64<T>(s_qr, rr + (size_t)(jj % A.R) * kD) * A.scale : -INFINITY;
        // the 32 value rows of this block are not contiguous in the ring: gather per token
        const float mc = warp_max(sc);
        const float mn = fmaxf(sr.m, mc);
        const float corr = sr.m == -INFINITY ? 0.f : expf(sr.m - mn);
        const float p = valid ? expf(sc - mn) : 0.f;
        sr.l = sr.l * corr + warp_sum(p);
        sr.a0 *= corr;
        sr.a1 *= corr;
        for (int e = 0; e < kS; e++) {
            const float pe = __shfl_sync(kFull, p, e);
            const long long je = jlo + (long long)b * kS + e;
            if (je > i) break;
            const T *vr = rv + (size_t)(je % A.R) * kD + 2 * lane;
            sr.a0 = fmaf(pe, to_f<T>(vr[0]), sr.a0);
            sr.a1 = fmaf(pe, to_f<T>(vr[1]), sr.a1);
        }
        sr.m = mn;
    }
    fold_warps(sr, &s_m, &s_l, s_acc, s_o, t, warp, lane);

    // 5. O = o^sr + alpha_h RMSNorm(u)  (eq. (2))
    if (t < kD) O[((size_t)bh * n_q + r) * kD + t] = from_f<T>(s_o[t] + f * s_u[t]);
}

__global__ void cache_reset_kernel(uint8_t *cache, const CacheArgs A) {
    const Slots S = slots_of(cache, A, blockIdx.x);
    if (threadIdx.x == 0) *S.t = 0;
    if (blockIdx.x == 0 && threadIdx.x == 0) *reinterpret_cast<int *>(cache + kFlagOff) = kFlagOk;
    for (int x = threadIdx.x; x < A.M; x += blockDim.x) {
        S.cell[x] = -1;
        S.exit[x] = 0;
    }
}

}  // namespace
}  // namespace fs

using namespace fs;

namespace {

// The parameters a cache depends on; Nq and Nk play no part.
fs_status cache_validate(const fs_params *p, int max_block) {
    if (!p) return FS_ERR_INVALID_ARG;
    fs_params q = *p;
    q.Nq = 0;
    q.Nk = 0;
    const fs_status s = validate_params(&q);
    if (s != FS_OK) return s;
    if (p->W < 0 || p->P < 0) return FS_ERR_UNSUPPORTED;       // base FS: state grows with length
    if (max_block < 1 || max_block > kMaxBlock) return FS_ERR_INVALID_ARG;
    return FS_OK;
}

size_t cache_total(const fs_params *p, const CacheGeom &g) {
    return kHeadBytes + (size_t)p->B * p->H * g.bh_bytes;
}

CacheArgs cache_args(const fs_params *p, int max_block, const CacheGeom &g) {
    CacheArgs A;
    std::memset(&A, 0, sizeof(A));
    A.R = g.R; A.M = g.M; A.maxnew = g.maxnew; A.max_block = max_block;
    A.w = p->w; A.K = p->K; A.W = p->W; A.P = p->P; A.H = p->H;
    A.rope_base = (double)p->rope_base;
    A.scale = (float)(1.0 / std::sqrt((double)p->d));
    A.rms_eps = p->rms_eps;
    A.o_t = g.o_t; A.o_rk = g.o_rk; A.o_rr = g.o_rr; A.o_rv = g.o_rv; A.o_cell = g.o_cell;
    A.o_exit = g.o_exit; A.o_a = g.o_a; A.o_kbar = g.o_kbar; A.o_ck = g.o_ck; A.o_cv = g.o_cv;
    A.bh_bytes = g.bh_bytes;
    for (int h = 0; h < p->H; h++) {
        A.alpha[h] = p->alpha[h];
        A.lambda[h] = p->lambda ? p->lambda[h] : 0.f;
        A.inv2sigma[h] = p->lambda ? (float)(1.0 / (2.0 * (double)p->sigma[h])) : 0.f;
        if (A.lambda[h] != 0.f) A.has_prior = 1;
    }
    return A;
}

}  // namespace

extern "C" fs_status fs_cache_bytes(const fs_params *p, int max_block, size_t *bytes) {
    const fs_status s = cache_validate(p, max_block);
    if (s != FS_OK) return s;
    if (!bytes) return FS_ERR_INVALID_ARG;
    *bytes = cache_total(p, cache_geom(p, max_block));
    return FS_OK;
}

extern "C" fs_status fs_cache_reset(const fs_params *p, int max_block, void *cache, size_t cache_bytes,
                                    void *stream) {
    const fs_status s = cache_validate(p, max_block);
    if (s != FS_OK) return s;
    const CacheGeom g = cache_geom(p, max_block);
    if (!cache || cache_bytes < cache_total(p, g)) return FS_ERR_WORKSPACE;
    const CacheArgs A = cache_args(p, max_block, g);
    cache_reset_kernel<<<p->B * p->H, 256, 0, (cudaStream_t)stream>>>(static_cast<uint8_t *>(cache), A);
    return cudaGetLastError() == cudaSuccess ? FS_OK : FS_ERR_CUDA;
}

extern "C" fs_status fs_cache_append(const fs_params *p, int max_block, void *cache, size_t cache_bytes,
                                     const void *K_new, const void *V_new, int n_new, void *stream) {
    const fs_status s = cache_validate(p, max_block);
    if (s != FS_OK) return s;
    if (n_new < 0 || n_new > max_block) return FS_ERR_INVALID_ARG;
    const CacheGeom g = cache_geom(p, max_block);
    if (!cache || cache_bytes < cache_total(p, g)) return FS_ERR_WORKSPACE;
    if (n_new == 0) return FS_OK;
    if (!K_new || !V_new) return FS_ERR_INVALID_ARG;
    const CacheArgs A = cache_args(p, max_block, g);
    const size_t smem = (size_t)g.maxnew * 8;
    cudaStream_t st = (cudaStream_t)stream;
    LaunchScope scope(kCacheAppend, st);
    uint8_t *c = static_cast<uint8_t *>(cache);
    if (p->dtype == FS_BF16)
        cache_append_kernel<__nv_bfloat16><<<p->B * p->H, kAppendThreads, smem, st>>>(
            c, static_cast<const __nv_bfloat16 *>(K_new), static_cast<const __nv_bfloat16 *>(V_new), n_new, A);
    else
        cache_append_kernel<float><<<p->B * p->H, kAppendThreads, smem, st>>>(
            c, static_cast<const float *>(K_new), static_cast<const float *>(V_new), n_new, A);
    return cudaGetLastError() == cudaSuccess ? FS_OK : FS_ERR_CUDA;
}

namespace {
template <typename T>
cudaError_t attend_launch(const CacheArgs &A, uint8_t *c, const void *Q, int n_q, int32_t *idx, void *O,
                          int BH, cudaStream_t st) {
    const size_t smem = (size_t)(3 * A.M + kMaxK) * 4;
    const dim3 grid(n_q, BH);
    auto kern = A.has_prior ? cache_attend_kernel<T, true> : cache_attend_kernel<T, false>;
    if (smem > 48 * 1024) cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    kern<<<grid, kAttendThreads, smem, st>>>(c, static_cast<const T *>(Q), n_q, idx, static_cast<T *>(O), A);
    return cudaGetLastError();
}
}  // namespace

extern "C" fs_status fs_cache_attend(const fs_params *p, int max_block, void *cache, size_t cache_bytes,
                                     const void *Q_new, int n_q, int32_t *idx, void *O, void *stream) {
    const fs_status s = cache_validate(p, max_block);
    if (s != FS_OK) return s;
    if (n_q < 1 || n_q > max_block || !Q_new || !O) return FS_ERR_INVALID_ARG;
    const CacheGeom g = cache_geom(p, max_block);
    if (!cache || cache_bytes < cache_total(p, g)) return FS_ERR_WORKSPACE;
    const CacheArgs A = cache_args(p, max_block, g);
    cudaStream_t st = (cudaStream_t)stream;
    LaunchScope scope(kCacheAttend, st);
    uint8_t *c = static_cast<uint8_t *>(cache);
    const cudaError_t e = p->dtype == FS_BF16
                              ? attend_launch<__nv_bfloat16>(A, c, Q_new, n_q, idx, O, p->B * p->H, st)
                              : attend_launch<float>(A, c, Q_new, n_q, idx, O, p->B * p->H, st);
    return e == cudaSuccess ? FS_OK : FS_ERR_CUDA;
}

extern "C" fs_status fs_cache_status(void *cache, void *stream) {
    if (!cache) return FS_ERR_INVALID_ARG;
    cudaStream_t st = (cudaStream_t)stream;
    if (cudaStreamSynchronize(st) != cudaSuccess) return FS_ERR_CUDA;
    int flag = 0;
    if (cudaMemcpy(&flag, cache, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return FS_ERR_CUDA;
    if (flag == kFlagOk) return FS_OK;
    const int zero = 0;
    if (cudaMemcpy(cache, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess) return FS_ERR_CUDA;
    return flag == kFlagTimeout ? FS_ERR_TIMEOUT : FS_ERR_KERNEL_CHECK;
}
