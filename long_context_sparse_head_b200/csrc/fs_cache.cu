// FS-L streaming cache: the forward pass over a token stream with bounded state per head,
// "FreeSolo" summary, "Practical Implications" 3 (per-head memory bounded by
// O((P+W)s + w + B + s)·d) and §3.3 eq. (8).  Same arithmetic as the batch forward pass (§3.1 eq. (2), §3.2
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
// fs_cache_attend: kAttendParts CTAs per (query, b, h) (a decode step has a handful of
// queries per head, so the work of one is spread over several CTAs): part 0 runs the RoPE
// window over the ring; parts 1..kReadParts each run admission, scores and top-K over the
// slots, then the NoPE readout of every kReadParts-th selected cell.  Each writes a partial
// online-softmax state; the last part to finish combines them (RMSNorm of the readout,
// eq. (2)).  CUDA cores.
#include <cmath>
#include <cstring>

#include "fs_common.cuh"

namespace fs {
namespace {

constexpr int kMaxBlock = 65536;
constexpr int kAppendThreads = 256;
// Attend: each warp stages 32-token blocks of key and value rows in shared memory (input
// type, rows padded by 16 bytes against bank conflicts), double-buffered.
template <typename T> struct AttendCfg {
    static constexpr int kWarps = sizeof(T) == 2 ? 8 : 4;
    static constexpr int kThreads = kWarps * 32;
    static constexpr int kRowBytes = kD * (int)sizeof(T);
    static constexpr int kRowStride = kRowBytes + 16;
    static constexpr int kBlockBytes = kS * kRowStride;         // one 32-row block
    static constexpr int kWarpBytes = 4 * kBlockBytes;          // (K, V) x 2 buffers
};
// Attend runs as kAttendParts CTAs per (query, b, h): part 0 the window, parts 1..kReadParts
// the readout of every kReadParts-th selected cell; each writes a partial online-softmax
// state (m, l, then 64 unnormalised outputs) and the last to finish combines them.
constexpr int kReadParts = 4, kAttendParts = kReadParts + 1, kPartFloats = 4 + kD;
constexpr int kFlagOff = 0;                     // int error flag at the start of the cache
constexpr size_t kHeadBytes = 256;

size_t a256(size_t x) { return (x + 255) & ~size_t(255); }

// Byte layout of one (b, h) state block; the cache is a 256-byte header, then B*H blocks.
struct CacheGeom {
    int R, M, maxnew;
    size_t elem;
    size_t o_t, o_rk, o_rr, o_rv, o_cell, o_exit, o_a, o_kbar, o_ck, o_cv, o_part, o_cnt, bh_bytes;
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
    g.o_part = seg((size_t)max_block * kAttendParts * kPartFloats * 4);   // attend partial states
    g.o_cnt = seg((size_t)max_block * 4);                   // attend: parts done per query
    g.bh_bytes = off;
    return g;
}

struct CacheArgs {
    int R, M, maxnew, max_block;
    int w, K, W, P, H;
    int has_prior;
    double theta[kD / 2];   // RoPE frequencies base^(-2m/d), double precision
    float scale;       // 1 / sqrt(d)
    float rms_eps;
    size_t o_t, o_rk, o_rr, o_rv, o_cell, o_exit, o_a, o_kbar, o_ck, o_cv, o_part, o_cnt, bh_bytes;
    float alpha[FS_MAX_HEADS];
    float lambda[FS_MAX_HEADS];
    float inv2sigma[FS_MAX_HEADS];
};

// |C_i| for position i of an unbounded stream: cells with (c+1)s <= i - w
__device__ __forceinline__ int cand_count_ll(long long i, int w) {
    const long long lim = i - w;
    return lim < kS ? 0 : (int)(lim / kS);
}

__device__ __forceinline__ uint32_t tc_smem(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// (cos, sin)(pos * theta_m) in double precision, rounded to float.  The angle (up to
// ~1e9 rad) is first reduced to [-pi, pi] by Cody-Waite: 2 pi = kTwoPiHi + kTwoPiLo with
// kTwoPiHi holding 24 significant bits, so k * kTwoPiHi is exact for |k| < 2^29 and the
// reduced angle is good to ~1e-10 rad; sincos then works on a small argument.
__device__ __forceinline__ void rope_cs(long long pos, double theta, float &c, float &s) {
    constexpr double kTwoPiHi = 6.2831854820251465, kTwoPiLo = -1.748455600074497e-07;
    const double x = (double)pos * theta;
    const double k = rint(x * 0.15915494309189535);           // x / (2 pi), rounded
    const double r = fma(-k, kTwoPiLo, fma(-k, kTwoPiHi, x));
    double sn, cs;
    sincos(r, &sn, &cs);
    c = (float)cs;
    s = (float)sn;
}

struct Slots {   // pointers into one (b, h) block
    long long *t;
    uint8_t *rk, *rr, *rv;
    int *cell, *exit;
    float *a, *kbar;
    uint8_t *ck, *cv;
    float *part;
    int *cnt;
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
    S.part = reinterpret_cast<float *>(b + A.o_part);
    S.cnt = reinterpret_cast<int *>(b + A.o_cnt);
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
        rope_cs(pos, A.theta[m], c, sn);
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

// Copies a 32-row block (row r at rows(r)) into dst with cp.async: eight lanes per 128
// bytes of a row, so each instruction moves whole cache lines.
template <typename T, typename RowFn>
__device__ __forceinline__ void stage_block(uint8_t *dst, RowFn rows, int lane) {
    using C = AttendCfg<T>;
    constexpr int CPR = C::kRowBytes / 16;                       // 16-byte chunks per row
    const uint32_t base = tc_smem(dst);
#pragma unroll
    for (int k = 0; k < kS * CPR / 32; k++) {
        const int q = lane + 32 * k, row = q / CPR, c = q % CPR;
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(base + row * C::kRowStride + 16 * c),
                     "l"(reinterpret_cast<const uint8_t *>(rows(row)) + 16 * c)
                     : "memory");
    }
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N> __device__ __forceinline__ void cp_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// q (shared, float) . row (shared, T), 64 dims
template <typename T> __device__ __forceinline__ float dot64_smem(const float *q, const uint8_t *row) {
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int c = 0; c < AttendCfg<T>::kRowBytes / 16; c++) {
        const uint4 u = *reinterpret_cast<const uint4 *>(row + 16 * c);
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
        if (sizeof(T) == 2) {
#pragma unroll
            for (int e = 0; e < 4; e++) {
                acc[e] = fmaf(q[8 * c + 2 * e], __uint_as_float(w[e] << 16), acc[e]);
                acc[e] = fmaf(q[8 * c + 2 * e + 1], __uint_as_float(w[e] & 0xffff0000u), acc[e]);
            }
        } else {
#pragma unroll
            for (int e = 0; e < 4; e++) acc[e] = fmaf(q[4 * c + e], __uint_as_float(w[e]), acc[e]);
        }
    }
    return (acc[0] + acc[1]) + (acc[2] + acc[3]);
}

// Online softmax state of one warp: running max m, sum l, and two output dims per lane.
// add(): one 32-token block, lane j holding token j's score (-inf if invalid), the value
// rows staged at vb; lane = dim pair for P V.
struct Online {
    float m = -INFINITY, l = 0.f, a0 = 0.f, a1 = 0.f;
    template <typename T> __device__ __forceinline__ void add(float sc, const uint8_t *vb, int lane) {
        const float mc = warp_max(sc);
        if (mc == -INFINITY) return;
        const float mn = fmaxf(m, mc);
        const float corr = m == -INFINITY ? 0.f : expf(m - mn);
        const float p = sc == -INFINITY ? 0.f : expf(sc - mn);
        l = l * corr + warp_sum(p);
        float b0[2] = {a0 * corr, 0.f}, b1[2] = {a1 * corr, 0.f};   // two chains per dim
#pragma unroll 8
        for (int j = 0; j < kS; j++) {
            const float pj = __shfl_sync(kFull, p, j);
            const uint8_t *row = vb + j * AttendCfg<T>::kRowStride;
            float v0, v1;
            if (sizeof(T) == 2) {
                const uint32_t w = *reinterpret_cast<const uint32_t *>(row + 4 * lane);
                v0 = __uint_as_float(w << 16);
                v1 = __uint_as_float(w & 0xffff0000u);
            } else {
                const float2 f2 = *reinterpret_cast<const float2 *>(row + 8 * lane);
                v0 = f2.x;
                v1 = f2.y;
            }
            b0[j & 1] = fmaf(pj, v0, b0[j & 1]);
            b1[j & 1] = fmaf(pj, v1, b1[j & 1]);
        }
        a0 = b0[0] + b0[1];
        a1 = b1[0] + b1[1];
        m = mn;
    }
};

// Folds the NW warps' online states into out[64] = acc / l (0 where nothing was attended).
template <int NW>
__device__ __forceinline__ void fold_warps(const Online &o, float (*s_m)[NW], float (*s_l)[NW], float (*s_acc)[kD],
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
        for (int w2 = 0; w2 < NW; w2++) mx = fmaxf(mx, (*s_m)[w2]);
        float num = 0.f, den = 0.f;
        if (mx != -INFINITY)
            for (int w2 = 0; w2 < NW; w2++) {
                if ((*s_m)[w2] == -INFINITY) continue;
                const float f = expf((*s_m)[w2] - mx);
                num = fmaf(s_acc[w2][t], f, num);
                den = fmaf((*s_l)[w2], f, den);
            }
        out[t] = den > 0.f ? num / den : 0.f;
    }
    __syncthreads();
}

// Folds the NW warps' online states into one raw state: max m, sum l, and out[64] the
// outputs scaled to m (not divided by l); written to dst[0], dst[1], dst[4..68).
template <int NW>
__device__ __forceinline__ void fold_raw(const Online &o, float (*s_m)[NW], float (*s_l)[NW], float (*s_acc)[kD],
                                         float *dst, int t, int warp, int lane) {
    if (lane == 0) {
        (*s_m)[warp] = o.m;
        (*s_l)[warp] = o.l;
    }
    s_acc[warp][2 * lane] = o.a0;
    s_acc[warp][2 * lane + 1] = o.a1;
    __syncthreads();
    if (t < kD) {
        float mx = -INFINITY;
        for (int w2 = 0; w2 < NW; w2++) mx = fmaxf(mx, (*s_m)[w2]);
        float num = 0.f, den = 0.f;
        if (mx != -INFINITY)
            for (int w2 = 0; w2 < NW; w2++) {
                if ((*s_m)[w2] == -INFINITY) continue;
                const float f = expf((*s_m)[w2] - mx);
                num = fmaf(s_acc[w2][t], f, num);
                den = fmaf((*s_l)[w2], f, den);
            }
        dst[4 + t] = num;
        if (t == 0) {
            dst[0] = mx;
            dst[1] = den;
        }
    }
    __syncthreads();
}

template <typename T, bool PRIOR>
__global__ void __launch_bounds__(AttendCfg<T>::kThreads) cache_attend_kernel(uint8_t *cache, const T *__restrict__ Qn,
                                                                      int n_q, int32_t *__restrict__ idx,
                                                                      T *__restrict__ O, const CacheArgs A) {
    using Cfg = AttendCfg<T>;
    constexpr int NW = Cfg::kWarps, NT = Cfg::kThreads;
    // dynamic: per warp the staged (K, V) blocks x 2; per slot a sort key (0: not admitted;
    // else score order in the high word, lower cell first in the low word), its cell and a
    // selected flag; the selected slots [K]
    extern __shared__ __align__(16) uint8_t shb[];
    unsigned long long *s_key = reinterpret_cast<unsigned long long *>(shb + NW * Cfg::kWarpBytes);
    int *s_cell = reinterpret_cast<int *>(s_key + A.M), *s_sel = s_cell + A.M, *s_list = s_sel + A.M;
    __shared__ float s_qn[kD], s_qr[kD];
    __shared__ float s_m[NW], s_l[NW], s_acc[NW][kD], s_ss[2];
    __shared__ int s_last;
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
        rope_cs(i, A.theta[t], c, sn);
        s_qn[2 * t] = q0;
        s_qn[2 * t + 1] = q1;
        s_qr[2 * t] = q0 * c - q1 * sn;
        s_qr[2 * t + 1] = q0 * sn + q1 * c;
    }
    __syncthreads();

    const int part = blockIdx.z;      // 0: the window; 1..kReadParts: a share of the readout
    float *mypart = S.part + ((size_t)r * kAttendParts + part) * kPartFloats;
    uint8_t *wbuf = shb + warp * Cfg::kWarpBytes;              // (K, V) buffer b at 2 b Cfg::kBlockBytes
    if (part == 0) {
        // 4. window (eqs. (3)-(4)): keys max(0, i-w) .. i from the ring, rotated by their
        //    absolute positions; 32-token blocks split over the warps
        const T *rr = reinterpret_cast<const T *>(S.rr), *rv = reinterpret_cast<const T *>(S.rv);
        const long long jlo = i - A.w < 0 ? 0 : i - A.w;
        const int L = (int)(i - jlo) + 1;
        Online sr;
        {
            const int nblk = (L + kS - 1) / kS;
            const int nit = nblk > warp ? (nblk - warp + NW - 1) / NW : 0;   // blocks warp, warp + NW, ...
            const int ri = (int)(i % A.R);                        // ring row of the query's own token
            auto issue = [&](int k) {
                // ring row of token `row` of block k (no 64-bit modulo per row: one per block)
                const long long j0 = jlo + (long long)(warp + k * NW) * kS;
                const int r0 = (int)(j0 % A.R), last = (int)(i - j0);   // rows past `last` are past i
                auto row_of = [&](int row) {
                    if (row > last) return (size_t)ri * kD;           // past i: any row in range
                    const int rr0 = r0 + row;
                    return (size_t)(rr0 >= A.R ? rr0 - A.R : rr0) * kD;
                };
                uint8_t *b = wbuf + 2 * (k & 1) * Cfg::kBlockBytes;
                stage_block<T>(b, [&](int row) { return rr + row_of(row); }, lane);
                stage_block<T>(b + Cfg::kBlockBytes, [&](int row) { return rv + row_of(row); }, lane);
                cp_commit();
            };
            if (nit > 0) issue(0);
            for (int k = 0; k < nit; k++) {
                if (k + 1 < nit) {
                    issue(k + 1);
                    cp_wait<1>();
                } else {
                    cp_wait<0>();
                }
                __syncwarp();
                const uint8_t *b = wbuf + 2 * (k & 1) * Cfg::kBlockBytes;
                const long long j = jlo + (long long)(warp + k * NW) * kS + lane;
                const float sc = j <= i ? dot64_smem<T>(s_qr, b + lane * Cfg::kRowStride) * A.scale : -INFINITY;
                sr.add<T>(sc, b + Cfg::kBlockBytes, lane);
                __syncwarp();
            }
        }
        fold_raw<NW>(sr, &s_m, &s_l, s_acc, mypart, t, warp, lane);
    } else {
        // 1. admission (eq. (8)) and scores (eq. (7)) over the slots, one thread per slot (the
        //    mean-key loads of all slots are in flight together)
        for (int x = t; x < A.M; x += NT) {
            const int c = S.cell[x];
            const bool adm = c >= 0 && c < n && (c >= n - A.W || n < S.exit[x]);
            float sc = 0.f;
            if (adm) {
                const float4 *kb = reinterpret_cast<const float4 *>(S.kbar + (size_t)x * kD);
                float acc[4] = {0.f, 0.f, 0.f, 0.f};
    #pragma unroll
                for (int e = 0; e < kD / 4; e++) {
                    const float4 v = __ldg(kb + e);
                    acc[e & 3] = fmaf(s_qn[4 * e], v.x, fmaf(s_qn[4 * e + 1], v.y,
                                 fmaf(s_qn[4 * e + 2], v.z, fmaf(s_qn[4 * e + 3], v.w, acc[e & 3]))));
                }
                sc = ((acc[0] + acc[1]) + (acc[2] + acc[3])) * A.scale;
                if (PRIOR) {
                    const float dpos = (float)(i - (long long)c * kS) - 0.5f * kS;   // i - p_c
                    sc += A.lambda[h] * S.a[x] * erff(dpos * A.inv2sigma[h]);
                }
            }
            const uint32_t ob = __float_as_uint(sc);
            const uint32_t ok = (ob & 0x80000000u) ? ~ob : (ob | 0x80000000u);
            s_key[x] = adm ? ((unsigned long long)ok << 32) | (0xffffffffu - (uint32_t)c) : 0ull;
            s_cell[x] = c;
        }
        __syncthreads();
        // 2. top-K: a slot is selected if fewer than K admitted slots have a larger key (higher
        //    score, or equal score and lower cell): a branch-free count over the keys
        for (int x = t; x < A.M; x += NT) {
            const unsigned long long kx = s_key[x];
            int rank = 0;
    #pragma unroll 4
            for (int y = 0; y < A.M; y++) rank += s_key[y] > kx;
            s_sel[x] = kx != 0ull && rank < A.K;
        }
        __syncthreads();
        for (int x = t; x < A.M; x += NT) {   // selected slots in ascending cell order
            if (!s_sel[x]) continue;
            const int cx = s_cell[x];
            int pos = 0;
    #pragma unroll 4
            for (int y = 0; y < A.M; y++) pos += s_sel[y] & (s_cell[y] < cx);
            s_list[pos] = x;
        }
        __syncthreads();
        int nsel = 0;
        for (int y = 0; y < A.M; y++) nsel += s_sel[y];
        if (part == 1 && idx && t < A.K) idx[((size_t)bh * n_q + r) * A.K + t] = t < nsel ? s_cell[s_list[t]] : -1;

        // 3. readout (eq. (9)): NoPE softmax over this part's share of the selected cells
        //    (list positions part-1, part-1+kReadParts, ...), warp w taking every NW-th of
        //    them; lane = token for the scores, lane = dim pair for P V
        const T *ck = reinterpret_cast<const T *>(S.ck), *cv = reinterpret_cast<const T *>(S.cv);
        Online lr;
        {
            const int p0 = part - 1;
            const int nloc = nsel > p0 ? (nsel - p0 + kReadParts - 1) / kReadParts : 0;   // this part's cells
            const int nit = nloc > warp ? (nloc - warp + NW - 1) / NW : 0;
            auto issue = [&](int k) {
                const int x = s_list[p0 + kReadParts * (warp + k * NW)];
                uint8_t *b = wbuf + 2 * (k & 1) * Cfg::kBlockBytes;
                stage_block<T>(b, [&](int row) { return ck + ((size_t)x * kS + row) * kD; }, lane);
                stage_block<T>(b + Cfg::kBlockBytes, [&](int row) { return cv + ((size_t)x * kS + row) * kD; }, lane);
                cp_commit();
            };
            if (nit > 0) issue(0);
            for (int k = 0; k < nit; k++) {
                if (k + 1 < nit) {
                    issue(k + 1);
                    cp_wait<1>();
                } else {
                    cp_wait<0>();
                }
                __syncwarp();
                const uint8_t *b = wbuf + 2 * (k & 1) * Cfg::kBlockBytes;
                const float sc = dot64_smem<T>(s_qn, b + lane * Cfg::kRowStride) * A.scale;
                lr.add<T>(sc, b + Cfg::kBlockBytes, lane);
                __syncwarp();                                        // before the buffer is refilled
            }
        }
        fold_raw<NW>(lr, &s_m, &s_l, s_acc, mypart, t, warp, lane);
    }

    // 5. the last part to finish combines: u from the readout parts (rescaled to their
    //    largest max), RMSNorm, O = o^sr + alpha_h RMSNorm(u)  (eq. (2))
    __threadfence();
    __syncthreads();
    if (t == 0) s_last = atomicAdd(S.cnt + r, 1) == kAttendParts - 1;
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    const float *P0 = S.part + (size_t)r * kAttendParts * kPartFloats;
    float u = 0.f, o = 0.f, den = 0.f;
    if (t < kD) {
        float mx = -INFINITY;
        for (int pp = 1; pp <= kReadParts; pp++) mx = fmaxf(mx, __ldcg(P0 + pp * kPartFloats));
        float num = 0.f;
        if (mx != -INFINITY)
            for (int pp = 1; pp <= kReadParts; pp++) {
                const float mp = __ldcg(P0 + pp * kPartFloats);
                if (mp == -INFINITY) continue;
                const float fct = expf(mp - mx);
                num = fmaf(__ldcg(P0 + pp * kPartFloats + 4 + t), fct, num);
                den = fmaf(__ldcg(P0 + pp * kPartFloats + 1), fct, den);
            }
        u = den > 0.f ? num / den : 0.f;
        const float l0 = __ldcg(P0 + 1);
        o = l0 > 0.f ? __ldcg(P0 + 4 + t) / l0 : 0.f;
        const float ss = warp_sum(u * u);
        if (lane == 0) s_ss[warp] = ss;
    }
    __syncthreads();
    if (t < kD) {
        const float f = den > 0.f ? A.alpha[h] / sqrtf((s_ss[0] + s_ss[1]) * (1.f / kD) + A.rms_eps) : 0.f;
        O[((size_t)bh * n_q + r) * kD + t] = from_f<T>(o + f * u);
    }
    if (t == 0) S.cnt[r] = 0;                     // ready for the next call
}

__global__ void cache_reset_kernel(uint8_t *cache, const CacheArgs A) {
    const Slots S = slots_of(cache, A, blockIdx.x);
    if (threadIdx.x == 0) *S.t = 0;
    if (blockIdx.x == 0 && threadIdx.x == 0) *reinterpret_cast<int *>(cache + kFlagOff) = kFlagOk;
    for (int x = threadIdx.x; x < A.M; x += blockDim.x) {
        S.cell[x] = -1;
        S.exit[x] = 0;
    }
    for (int x = threadIdx.x; x < A.max_block; x += blockDim.x) S.cnt[x] = 0;
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
    for (int m = 0; m < kD / 2; m++) A.theta[m] = std::pow((double)p->rope_base, -2.0 * m / (double)p->d);
    A.scale = (float)(1.0 / std::sqrt((double)p->d));
    A.rms_eps = p->rms_eps;
    A.o_t = g.o_t; A.o_rk = g.o_rk; A.o_rr = g.o_rr; A.o_rv = g.o_rv; A.o_cell = g.o_cell;
    A.o_exit = g.o_exit; A.o_a = g.o_a; A.o_kbar = g.o_kbar; A.o_ck = g.o_ck; A.o_cv = g.o_cv;
    A.o_part = g.o_part; A.o_cnt = g.o_cnt;
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
    const size_t smem = (size_t)AttendCfg<T>::kWarps * AttendCfg<T>::kWarpBytes + (size_t)A.M * 16 + (size_t)kMaxK * 4;
    const dim3 grid(n_q, BH, kAttendParts);
    auto kern = A.has_prior ? cache_attend_kernel<T, true> : cache_attend_kernel<T, false>;
    if (smem > 48 * 1024) cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    kern<<<grid, AttendCfg<T>::kThreads, smem, st>>>(c, static_cast<const T *>(Q), n_q, idx, static_cast<T *>(O), A);
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
