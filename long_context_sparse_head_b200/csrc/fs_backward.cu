// Backward pass of eq. (2) ("FreeSolo" summary §3.1 eq. (2), §3.2 eqs. (3)-(4), §3.3
// eq. (9)) with the selection held fixed:
//   O_i = o_i^sr + alpha_h y_i,  y_i = RMSNorm(u_i) = u_i r_i,  r_i = (mean(u_i^2) + eps)^(-1/2)
//   window:  o^sr = sum_j p_j v_j,  p = softmax_j(l_ij),  l_ij = (R_i q_i).(R_j k_j)/sqrt(d)
//   readout: u = sum_t pi_t v_t,    pi = softmax_t(s_it),   s_it = q_i.k_t/sqrt(d), t in cells(S_i)
// For a softmax branch o = sum_j p_j v_j with output gradient g:
//   dv_j += p_j g,  dl_j = p_j (g.v_j - g.o),  dq += dl_j k_j / sqrt(d),  dk_j += dl_j q / sqrt(d)
// (the window's through the rotations: dq_i = R_i^T sum_j dl_ij k'_j, dk_j = R_j^T sum_i dl_ij q'_i),
// with g = dO for the window and g = du = r (dy - y (dy.y)/d), dy = alpha_h dO, for the readout;
// dalpha_h = sum_i dO_i.y_i.
//
// Kernels (CUDA cores, float32 throughout):
//   rotate_keys  k'_j = R_j k_j (absolute positions, double-precision angle tables)
//   win_rows     one warp per 32 query rows (lane = row), the band's keys staged in shared
//                memory: the window's log-sum-exp and g.o^sr, its part of dQ, rotated queries
//   lr_rows      one warp per query row, each selected cell staged in shared memory: the
//                readout's log-sum-exp, u, RMSNorm, du, g.u-term, its part of dQ, dalpha terms
//   window_kv    one warp per 32 keys (lane = key): dK, dV over the queries whose window
//                holds them; writes every key (zeros where none)
//   cells        cell -> rows lists by counting sort of idx (count, scan, fill)
//   readout_kv   one warp per cell (lane = token): adds the readout's dK, dV over the rows
//                that selected the cell
//   dalpha       per-head sum of the rows' dO.y
#include <cmath>
#include <type_traits>

#include "tc_rope.cuh"

namespace fs {
namespace {

struct BwdArgs {
    int B, H, Nq, Nk, C, w, K, q0;
    float scale, rms_eps;
    float alpha[FS_MAX_HEADS];
};

// Byte layout of the backward scratch (256-byte aligned segments).
struct BwdLayout {
    size_t flag, rope, krot, qrot, rowst, du, dal, cnt, off, fill, list, tiles, total;
};

size_t a256b(size_t x) { return (x + 255) & ~size_t(255); }

BwdLayout bwd_layout(const fs_params *p) {
    const size_t BH = (size_t)p->B * p->H, C = (size_t)(p->Nk / p->s), R = BH * p->Nq;
    BwdLayout L;
    size_t off = 0;
    auto seg = [&](size_t bytes) {
        const size_t o = off;
        off += a256b(bytes);
        return o;
    };
    L.flag = seg(256);                                                   // device error flag
    L.rope = seg((size_t)(kRopeLo + rope_hi_rows(p->Nk)) * 32 * 8);   // lo, hi angle tables
    L.krot = seg(BH * p->Nk * kD * 4);                                   // rotated keys, float
    L.qrot = seg(R * kD * 4);                                            // rotated queries
    L.rowst = seg(R * 4 * 4);                                            // lse_sr, D_sr, lse_lr, D_lr
    L.du = seg(R * kD * 4);                                              // readout output gradient
    L.dal = seg(R * 4);                                                  // dO.y per row
    L.cnt = seg((BH * C + 1) * 4);
    L.off = seg((BH * C + 1) * 4);
    L.fill = seg((BH * C + 1) * 4);
    L.list = seg(R * (size_t)(p->K > 0 ? p->K : 1) * 4);                 // rows of each cell
    L.tiles = seg(BH * (size_t)((p->Nq + 127) / 128) * kTileRecWords * 4);   // tile records (bf16)
    L.total = off;
    return L;
}

// (cos, sin)(pos theta_m) for pair m from the two-level tables
__device__ __forceinline__ float2 rope_cs_tab(int pos, int m, const float2 *__restrict__ lo, const float2 *__restrict__ hi) {
    const float2 a = __ldg(lo + (pos & (kRopeLo - 1)) * 32 + m), b = __ldg(hi + (pos / kRopeLo) * 32 + m);
    return make_float2(a.x * b.x - a.y * b.y, a.y * b.x + a.x * b.y);
}

template <typename T>
__global__ void bwd_rotate_keys_kernel(const T *__restrict__ K, float *__restrict__ krot, long long n_pairs, int Nk,
                                       const float2 *__restrict__ lo, const float2 *__restrict__ hi) {
    const long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (e >= n_pairs) return;
    const int m = (int)(e & 31);
    const int j = (int)((e >> 5) % Nk);
    const float2 cs = rope_cs_tab(j, m, lo, hi);
    const float k0 = to_f<T>(K[2 * e]), k1 = to_f<T>(K[2 * e + 1]);
    krot[2 * e] = k0 * cs.x - k1 * cs.y;
    krot[2 * e + 1] = k0 * cs.y + k1 * cs.x;
}

// ---- window rows: one warp per 32 consecutive query rows (lane = row); the keys of the
// warp's band [i0 - w, i0 + 31] pass through shared memory in 32-key tiles, read by every
// lane at once (broadcast).  Pass 1: log-sum-exp and D = dO.o^sr (online, as
// sum_j p_j (dO.v_j)); pass 2: dq' = sum_j dl_j k'_j.  Writes dQ (window part), the rotated
// queries and (lse_sr, D_sr).
constexpr int kWinWarps = 2;                  // 32 KB of static shared memory

template <typename T>
__device__ __forceinline__ void load_row64(const T *src, float *dst);
template <>
__device__ __forceinline__ void load_row64<float>(const float *src, float *dst) {
#pragma unroll
    for (int e = 0; e < kD / 4; e++) {
        const float4 x = __ldg(reinterpret_cast<const float4 *>(src) + e);
        dst[4 * e] = x.x; dst[4 * e + 1] = x.y; dst[4 * e + 2] = x.z; dst[4 * e + 3] = x.w;
    }
}
template <>
__device__ __forceinline__ void load_row64<__nv_bfloat16>(const __nv_bfloat16 *src, float *dst) {
#pragma unroll
    for (int e = 0; e < kD / 8; e++) {
        const uint4 x = __ldg(reinterpret_cast<const uint4 *>(src) + e);
        const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
        for (int k = 0; k < 4; k++) {
            dst[8 * e + 2 * k] = __uint_as_float(w[k] << 16);
            dst[8 * e + 2 * k + 1] = __uint_as_float(w[k] & 0xffff0000u);
        }
    }
}

// 32 rows x 64 of f32 from rows [j0, j0 + 32) of src (rows past `n` read as zeros) into a
// dense [32][64] tile; coalesced 16-byte loads
template <typename T>
__device__ __forceinline__ void stage_tile(const T *src, int j0, int n, float (*tile)[kD], int lane);
template <>
__device__ __forceinline__ void stage_tile<float>(const float *src, int j0, int n, float (*tile)[kD], int lane) {
#pragma unroll 4
    for (int q = lane; q < 32 * kD / 4; q += 32) {
        const int row = q >> 4, c4 = q & 15;
        const float4 x = j0 + row < n ? __ldg(reinterpret_cast<const float4 *>(src + (size_t)(j0 + row) * kD) + c4)
                                      : make_float4(0.f, 0.f, 0.f, 0.f);
        *reinterpret_cast<float4 *>(&tile[row][4 * c4]) = x;
    }
}
template <>
__device__ __forceinline__ void stage_tile<__nv_bfloat16>(const __nv_bfloat16 *src, int j0, int n, float (*tile)[kD],
                                                          int lane) {
#pragma unroll 4
    for (int q = lane; q < 32 * kD / 8; q += 32) {
        const int row = q >> 3, c8 = q & 7;
        const uint4 x = j0 + row < n ? __ldg(reinterpret_cast<const uint4 *>(src + (size_t)(j0 + row) * kD) + c8)
                                     : make_uint4(0u, 0u, 0u, 0u);
        const uint32_t w[4] = {x.x, x.y, x.z, x.w};
        float4 lo, hi;
        lo.x = __uint_as_float(w[0] << 16); lo.y = __uint_as_float(w[0] & 0xffff0000u);
        lo.z = __uint_as_float(w[1] << 16); lo.w = __uint_as_float(w[1] & 0xffff0000u);
        hi.x = __uint_as_float(w[2] << 16); hi.y = __uint_as_float(w[2] & 0xffff0000u);
        hi.z = __uint_as_float(w[3] << 16); hi.w = __uint_as_float(w[3] & 0xffff0000u);
        *reinterpret_cast<float4 *>(&tile[row][8 * c8]) = lo;
        *reinterpret_cast<float4 *>(&tile[row][8 * c8 + 4]) = hi;
    }
}

// a.b over 64 with a in registers and b a shared row read by every lane (broadcast)
__device__ __forceinline__ float dot_bcast(const float *a, const float *b) {
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int e = 0; e < kD / 4; e++) {
        const float4 x = *reinterpret_cast<const float4 *>(b + 4 * e);
        acc[0] = fmaf(a[4 * e], x.x, acc[0]);
        acc[1] = fmaf(a[4 * e + 1], x.y, acc[1]);
        acc[2] = fmaf(a[4 * e + 2], x.z, acc[2]);
        acc[3] = fmaf(a[4 * e + 3], x.w, acc[3]);
    }
    return (acc[0] + acc[1]) + (acc[2] + acc[3]);
}

template <typename T>
__global__ void __launch_bounds__(kWinWarps * 32) bwd_win_rows_kernel(
    const BwdArgs A, const T *__restrict__ Q, const T *__restrict__ V, const T *__restrict__ dO,
    const float *__restrict__ krot, const float2 *__restrict__ lo, const float2 *__restrict__ hi,
    float *__restrict__ dQ, float *__restrict__ qrot, float *__restrict__ rowst) {
    __shared__ __align__(16) float s_k[kWinWarps][32][kD];
    __shared__ __align__(16) float s_v[kWinWarps][32][kD];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int bh = blockIdx.y;
    const int r0 = (blockIdx.x * kWinWarps + warp) * 32;
    if (r0 >= A.Nq) return;                                   // warp-uniform
    const int r = r0 + lane;
    const bool valid = r < A.Nq;
    const int i = A.q0 + (valid ? r : A.Nq - 1);
    const size_t row = (size_t)bh * A.Nq + (valid ? r : A.Nq - 1);
    const size_t kb = (size_t)bh * A.Nk;
    float qr[kD], g[kD];
    load_row64<T>(Q + row * kD, qr);
#pragma unroll
    for (int m = 0; m < kD / 2; m++) {                        // q' = R_i q
        const float2 cs = rope_cs_tab(i, m, lo, hi);
        const float a = qr[2 * m], b = qr[2 * m + 1];
        qr[2 * m] = a * cs.x - b * cs.y;
        qr[2 * m + 1] = a * cs.y + b * cs.x;
    }
    if (valid) {
        float4 *d4 = reinterpret_cast<float4 *>(qrot + row * kD);
#pragma unroll
        for (int e = 0; e < kD / 4; e++) d4[e] = make_float4(qr[4 * e], qr[4 * e + 1], qr[4 * e + 2], qr[4 * e + 3]);
    }
    load_row64<T>(dO + row * kD, g);
    const int i0 = A.q0 + r0;
    const int jlo = max(0, i0 - A.w), jhi = min(A.q0 + A.Nq - 1, i0 + 31);
    float m = -INFINITY, l = 0.f, D = 0.f;
    for (int t0 = jlo; t0 <= jhi; t0 += 32) {                 // pass 1: statistics
        __syncwarp();
        stage_tile<float>(krot + kb * kD, t0, jhi + 1, s_k[warp], lane);
        stage_tile<T>(V + kb * kD, t0, jhi + 1, s_v[warp], lane);
        __syncwarp();
        const int nt = min(32, jhi + 1 - t0);
        for (int jj = 0; jj < nt; jj++) {
            const int j = t0 + jj;
            const float x = dot_bcast(qr, s_k[warp][jj]) * A.scale;
            const float dp = dot_bcast(g, s_v[warp][jj]);
            if (valid && j <= i && j >= i - A.w) {
                const float mn = fmaxf(m, x);
                const float corr = __expf(m - mn);           // 0 while m is -inf
                const float pj = __expf(x - mn);
                l = l * corr + pj;
                D = D * corr + pj * dp;
                m = mn;
            }
        }
    }
    const float lse = m + __logf(l), Dsr = D / l;
    float dq[kD];
#pragma unroll
    for (int e = 0; e < kD; e++) dq[e] = 0.f;
    for (int t0 = jlo; t0 <= jhi; t0 += 32) {                 // pass 2: dq' = sum_j dl_j k'_j
        __syncwarp();
        stage_tile<float>(krot + kb * kD, t0, jhi + 1, s_k[warp], lane);
        stage_tile<T>(V + kb * kD, t0, jhi + 1, s_v[warp], lane);
        __syncwarp();
        const int nt = min(32, jhi + 1 - t0);
        for (int jj = 0; jj < nt; jj++) {
            const int j = t0 + jj;
            const float x = dot_bcast(qr, s_k[warp][jj]) * A.scale;
            const float dp = dot_bcast(g, s_v[warp][jj]);
            const bool in = valid && j <= i && j >= i - A.w;
            const float dl = in ? __expf(x - lse) * (dp - Dsr) * A.scale : 0.f;
            const float *kr = s_k[warp][jj];
#pragma unroll
            for (int e = 0; e < kD / 4; e++) {
                const float4 k4 = *reinterpret_cast<const float4 *>(kr + 4 * e);
                dq[4 * e] = fmaf(dl, k4.x, dq[4 * e]);
                dq[4 * e + 1] = fmaf(dl, k4.y, dq[4 * e + 1]);
                dq[4 * e + 2] = fmaf(dl, k4.z, dq[4 * e + 2]);
                dq[4 * e + 3] = fmaf(dl, k4.w, dq[4 * e + 3]);
            }
        }
    }
    if (!valid) return;
#pragma unroll
    for (int mm = 0; mm < kD / 2; mm++) {                     // dq = R_i^T dq'
        const float2 cs = rope_cs_tab(i, mm, lo, hi);
        const float a = dq[2 * mm], b = dq[2 * mm + 1];
        dq[2 * mm] = a * cs.x + b * cs.y;
        dq[2 * mm + 1] = -a * cs.y + b * cs.x;
    }
    float4 *d4 = reinterpret_cast<float4 *>(dQ + row * kD);
#pragma unroll
    for (int e = 0; e < kD / 4; e++) d4[e] = make_float4(dq[4 * e], dq[4 * e + 1], dq[4 * e + 2], dq[4 * e + 3]);
    rowst[row * 4] = lse;
    rowst[row * 4 + 1] = Dsr;
}

// ---- readout rows: one warp per query row, lane m holding dimensions (2m, 2m + 1).  A
// cell's logits are formed as per-lane partial products over the lane's two dimensions,
// then a transposed butterfly sum hands lane t the total for token t (31 shuffles for 32
// tokens).  Pass 1: log-sum-exp and u; RMSNorm and du; pass 2: dq += sum_t dl_t k_t.  Adds
// the readout part to dQ; writes du, (lse_lr, D_lr) and the dalpha terms.
constexpr int kLrWarps = 4;

template <typename T>
__global__ void __launch_bounds__(kLrWarps * 32) bwd_lr_rows_kernel(
    const BwdArgs A, const T *__restrict__ Q, const T *__restrict__ K, const T *__restrict__ V,
    const int32_t *__restrict__ idx, const T *__restrict__ dO, float *__restrict__ dQ, float *__restrict__ rowst,
    float *__restrict__ du_out, float *__restrict__ dal) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int bh = blockIdx.y, h = bh % A.H;
    const int r = blockIdx.x * kLrWarps + warp;
    if (r >= A.Nq) return;                                    // warp-uniform
    const size_t row = (size_t)bh * A.Nq + r;
    const size_t kb = (size_t)bh * A.Nk;
    const int32_t *sel = idx + row * A.K;
    int ncell = 0;
    for (int e = 0; e < A.K; e++) ncell += (unsigned)sel[e] < (unsigned)A.C;
    float lse_lr = -INFINITY, D_lr = 0.f, gy = 0.f, du0 = 0.f, du1 = 0.f;
    if (ncell > 0) {
        const float2 q = ld_pair<T>(Q + row * kD + 2 * lane), g = ld_pair<T>(dO + row * kD + 2 * lane);
        float m = -INFINITY, l = 0.f, u0 = 0.f, u1 = 0.f;
        for (int e = 0; e < A.K; e++) {                       // pass 1: lse and u
            const int c = sel[e];
            if ((unsigned)c >= (unsigned)A.C) continue;
            const T *kc = K + (kb + (size_t)c * kS) * kD + 2 * lane;
            const T *vc = V + (kb + (size_t)c * kS) * kD + 2 * lane;
            float v[32];
#pragma unroll
            for (int t = 0; t < 32; t++) {
                const float2 k2 = ld_pair<T>(kc + t * kD);
                v[t] = fmaf(q.x, k2.x, q.y * k2.y);
            }
            const float x = transpose_sum32(v, lane) * A.scale;   // lane t: token t's logit
            const float mn = fmaxf(m, warp_max(x));
            const float corr = __expf(m - mn);
            const float pt = __expf(x - mn);
            l = l * corr + warp_sum(pt);
            u0 *= corr;
            u1 *= corr;
#pragma unroll
            for (int t = 0; t < 32; t++) {
                const float pe = __shfl_sync(kFull, pt, t);
                const float2 v2 = ld_pair<T>(vc + t * kD);
                u0 = fmaf(pe, v2.x, u0);
                u1 = fmaf(pe, v2.y, u1);
            }
            m = mn;
        }
        u0 /= l;
        u1 /= l;
        lse_lr = m + __logf(l);
        const float rin = rsqrtf(warp_sum(u0 * u0 + u1 * u1) * (1.f / kD) + A.rms_eps);
        const float y0 = u0 * rin, y1 = u1 * rin;
        gy = warp_sum(g.x * y0 + g.y * y1);
        const float a = A.alpha[h];
        const float dyy = a * gy;                             // dy.y with dy = alpha dO
        du0 = rin * (a * g.x - y0 * dyy * (1.f / kD));
        du1 = rin * (a * g.y - y1 * dyy * (1.f / kD));
        D_lr = warp_sum(du0 * u0 + du1 * u1);
        float dq0 = 0.f, dq1 = 0.f;
        for (int e = 0; e < A.K; e++) {                       // pass 2: dq += sum_t dl_t k_t
            const int c = sel[e];
            if ((unsigned)c >= (unsigned)A.C) continue;
            const T *kc = K + (kb + (size_t)c * kS) * kD + 2 * lane;
            const T *vc = V + (kb + (size_t)c * kS) * kD + 2 * lane;
            float2 k2[32];
            float v[32], w[32];
#pragma unroll
            for (int t = 0; t < 32; t++) {
                k2[t] = ld_pair<T>(kc + t * kD);
                const float2 v2 = ld_pair<T>(vc + t * kD);
                v[t] = fmaf(q.x, k2[t].x, q.y * k2[t].y);
                w[t] = fmaf(du0, v2.x, du1 * v2.y);
            }
            const float x = transpose_sum32(v, lane) * A.scale;
            const float dp = transpose_sum32(w, lane);
            const float dl = __expf(x - lse_lr) * (dp - D_lr) * A.scale;
#pragma unroll
            for (int t = 0; t < 32; t++) {
                const float de = __shfl_sync(kFull, dl, t);
                dq0 = fmaf(de, k2[t].x, dq0);
                dq1 = fmaf(de, k2[t].y, dq1);
            }
        }
        dQ[row * kD + 2 * lane] += dq0;
        dQ[row * kD + 2 * lane + 1] += dq1;
    }
    du_out[row * kD + 2 * lane] = du0;
    du_out[row * kD + 2 * lane + 1] = du1;
    if (lane == 0) {
        rowst[row * 4 + 2] = lse_lr;
        rowst[row * 4 + 3] = D_lr;
        dal[row] = gy;
    }
}

constexpr int kKvWarps = 2, kPad = kD + 1;   // 2 warps: 41 KB of static shared memory
constexpr int kRowBatch = 8;                  // query rows staged per round

// x = q.k, dp = g.v with q, g shared rows read by every lane (16-byte broadcasts) and k, v
// this lane's padded rows; four independent partial sums each
__device__ __forceinline__ void dot2_lane(const float *q, const float *g, const float *k, const float *v,
                                          float &x, float &dp) {
    float xa[4] = {0.f, 0.f, 0.f, 0.f}, pa[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int e = 0; e < kD; e += 4) {
        const float4 q4 = *reinterpret_cast<const float4 *>(q + e);
        const float4 g4 = *reinterpret_cast<const float4 *>(g + e);
        xa[0] = fmaf(q4.x, k[e], xa[0]);
        xa[1] = fmaf(q4.y, k[e + 1], xa[1]);
        xa[2] = fmaf(q4.z, k[e + 2], xa[2]);
        xa[3] = fmaf(q4.w, k[e + 3], xa[3]);
        pa[0] = fmaf(g4.x, v[e], pa[0]);
        pa[1] = fmaf(g4.y, v[e + 1], pa[1]);
        pa[2] = fmaf(g4.z, v[e + 2], pa[2]);
        pa[3] = fmaf(g4.w, v[e + 3], pa[3]);
    }
    x = (xa[0] + xa[1]) + (xa[2] + xa[3]);
    dp = (pa[0] + pa[1]) + (pa[2] + pa[3]);
}

// dv += a g, dk += b q (g, q shared rows, 16-byte broadcasts)
__device__ __forceinline__ void axpy2(float a, const float *g, float b, const float *q, float *dv, float *dk) {
#pragma unroll
    for (int e = 0; e < kD; e += 4) {
        const float4 g4 = *reinterpret_cast<const float4 *>(g + e);
        const float4 q4 = *reinterpret_cast<const float4 *>(q + e);
        dv[e] = fmaf(a, g4.x, dv[e]);
        dv[e + 1] = fmaf(a, g4.y, dv[e + 1]);
        dv[e + 2] = fmaf(a, g4.z, dv[e + 2]);
        dv[e + 3] = fmaf(a, g4.w, dv[e + 3]);
        dk[e] = fmaf(b, q4.x, dk[e]);
        dk[e + 1] = fmaf(b, q4.y, dk[e + 1]);
        dk[e + 2] = fmaf(b, q4.z, dk[e + 2]);
        dk[e + 3] = fmaf(b, q4.w, dk[e + 3]);
    }
}

// Window dK, dV: warp = 32 consecutive keys (lane = key j), over the queries i whose window
// [i - w, i] holds some key of the block; dK_j = R_j^T sum_i dl_ij q'_i.  Every key is written.
template <typename T>
__global__ void __launch_bounds__(kKvWarps * 32) bwd_window_kv_kernel(
    const BwdArgs A, const T *__restrict__ V, const T *__restrict__ dO, const float *__restrict__ krot,
    const float *__restrict__ qrot, const float *__restrict__ rowst, const float2 *__restrict__ lo,
    const float2 *__restrict__ hi, float *__restrict__ dK, float *__restrict__ dV) {
    __shared__ float s_k[kKvWarps][32][kPad], s_v[kKvWarps][32][kPad];
    __shared__ __align__(16) float s_qi[kKvWarps][kRowBatch][kD], s_gi[kKvWarps][kRowBatch][kD];
    __shared__ float4 s_st[kKvWarps][kRowBatch];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int bh = blockIdx.y;
    const int j0 = (blockIdx.x * kKvWarps + warp) * 32;
    if (j0 >= A.Nk) return;                                  // warp-uniform
    const int j = j0 + lane;
    const bool kv_ok = j < A.Nk;
    const size_t kb = (size_t)bh * A.Nk;
    for (int e = 0; e < kD; e++) {                           // this warp's 32 key / value rows
        s_k[warp][lane][e] = kv_ok ? krot[(kb + j) * kD + e] : 0.f;
        s_v[warp][lane][e] = kv_ok ? to_f<T>(V[(kb + j) * kD + e]) : 0.f;
    }
    float dk[kD], dv[kD];
#pragma unroll
    for (int e = 0; e < kD; e++) { dk[e] = 0.f; dv[e] = 0.f; }
    // queries at positions i in [j0, j0 + 31 + w] that exist, kRowBatch at a time
    const int ilo = max(j0, A.q0), ihi = min(j0 + 31 + A.w, A.q0 + A.Nq - 1);
    for (int ib = ilo; ib <= ihi; ib += kRowBatch) {
        const int nb = min(kRowBatch, ihi + 1 - ib);
        __syncwarp();
        for (int rr = 0; rr < nb; rr++) {
            const size_t row = (size_t)bh * A.Nq + (ib + rr - A.q0);
            const float2 q2 = *reinterpret_cast<const float2 *>(qrot + row * kD + 2 * lane);
            s_qi[warp][rr][2 * lane] = q2.x;
            s_qi[warp][rr][2 * lane + 1] = q2.y;
            s_gi[warp][rr][2 * lane] = to_f<T>(dO[row * kD + 2 * lane]);
            s_gi[warp][rr][2 * lane + 1] = to_f<T>(dO[row * kD + 2 * lane + 1]);
            if (lane == 0) s_st[warp][rr] = __ldg(reinterpret_cast<const float4 *>(rowst) + row);
        }
        __syncwarp();
        for (int rr = 0; rr < nb; rr++) {
            const int i = ib + rr;
            if (!kv_ok || j > i || j < i - A.w) continue;
            const float *qi = s_qi[warp][rr], *gi = s_gi[warp][rr];
            const float4 st = s_st[warp][rr];                // lse_sr, D_sr, ...
            float x, dp;
            dot2_lane(qi, gi, s_k[warp][lane], s_v[warp][lane], x, dp);
            const float pj = __expf(x * A.scale - st.x);
            const float dl = pj * (dp - st.y) * A.scale;
            axpy2(pj, gi, dl, qi, dv, dk);
        }
    }
    if (!kv_ok) return;
#pragma unroll
    for (int mm = 0; mm < kD / 2; mm++) {                    // R_j^T on each pair
        const float2 cs = rope_cs_tab(j, mm, lo, hi);
        const float a = dk[2 * mm], b = dk[2 * mm + 1];
        dk[2 * mm] = a * cs.x + b * cs.y;
        dk[2 * mm + 1] = -a * cs.y + b * cs.x;
    }
    float4 *dk4 = reinterpret_cast<float4 *>(dK + (kb + j) * kD), *dv4 = reinterpret_cast<float4 *>(dV + (kb + j) * kD);
#pragma unroll
    for (int e = 0; e < kD / 4; e++) {
        dk4[e] = make_float4(dk[4 * e], dk[4 * e + 1], dk[4 * e + 2], dk[4 * e + 3]);
        dv4[e] = make_float4(dv[4 * e], dv[4 * e + 1], dv[4 * e + 2], dv[4 * e + 3]);
    }
}

// cell -> rows lists: counts, exclusive scan, fill (order within a cell is irrelevant)
__global__ void bwd_count_kernel(const int32_t *__restrict__ idx, long long n, int K, int Nq, int C, int *cnt) {
    const long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (e >= n) return;
    const int c = idx[e];
    if ((unsigned)c >= (unsigned)C) return;           // -1 padding (and anything outside [0, C))
    const long long bh = e / ((long long)Nq * K);
    atomicAdd(&cnt[bh * C + c], 1);
}
__global__ void __launch_bounds__(1024) bwd_scan_kernel(const int *__restrict__ cnt, int *__restrict__ off, int n) {
    __shared__ int wsum[32];
    __shared__ int carry;
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    if (t == 0) carry = 0;
    __syncthreads();
    for (int base = 0; base < n; base += 1024) {
        const int v = base + t < n ? cnt[base + t] : 0;
        int incl = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(kFull, incl, o);
            if (lane >= o) incl += y;
        }
        if (lane == 31) wsum[warp] = incl;
        __syncthreads();
        int before = carry;
        for (int k = 0; k < warp; k++) before += wsum[k];
        if (base + t < n) off[base + t] = before + incl - v;
        __syncthreads();
        if (t == 1023) carry = before + incl;
        __syncthreads();
    }
    if (t == 0) off[n] = carry;
}
__global__ void bwd_fill_kernel(const int32_t *__restrict__ idx, long long n, int K, int Nq, int C,
                                const int *__restrict__ off, int *fill, int *list) {
    const long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (e >= n) return;
    const int c = idx[e];
    if ((unsigned)c >= (unsigned)C) return;           // -1 padding (and anything outside [0, C))
    const long long bh = e / ((long long)Nq * K);
    const int r = (int)((e / K) % Nq);
    const int pos = off[bh * C + c] + atomicAdd(&fill[bh * C + c], 1);
    list[pos] = r;
}

// Readout dK, dV: warp = one cell (lane = token), over the rows that selected it; adds to
// the window's values already in dK, dV.
template <typename T>
__global__ void __launch_bounds__(kKvWarps * 32) bwd_readout_kv_kernel(
    const BwdArgs A, const T *__restrict__ Q, const T *__restrict__ K, const T *__restrict__ V,
    const float *__restrict__ du, const float *__restrict__ rowst, const int *__restrict__ off,
    const int *__restrict__ list, float *__restrict__ dK, float *__restrict__ dV) {
    __shared__ float s_k[kKvWarps][32][kPad], s_v[kKvWarps][32][kPad];
    __shared__ __align__(16) float s_qi[kKvWarps][kRowBatch][kD], s_gi[kKvWarps][kRowBatch][kD];
    __shared__ int s_row[kKvWarps][kRowBatch];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int bh = blockIdx.y;
    const int c = blockIdx.x * kKvWarps + warp;
    if (c >= A.C) return;
    const int b0 = off[(size_t)bh * A.C + c], b1 = off[(size_t)bh * A.C + c + 1];
    if (b0 == b1) return;
    const size_t t = (size_t)bh * A.Nk + (size_t)c * kS + lane;
    for (int e = 0; e < kD; e++) {
        s_k[warp][lane][e] = to_f<T>(K[t * kD + e]);
        s_v[warp][lane][e] = to_f<T>(V[t * kD + e]);
    }
    float dk[kD], dv[kD];
#pragma unroll
    for (int e = 0; e < kD; e++) { dk[e] = 0.f; dv[e] = 0.f; }
    for (int qb = b0; qb < b1; qb += kRowBatch) {            // kRowBatch rows at a time
        const int nb = min(kRowBatch, b1 - qb);
        __syncwarp();
        for (int rr = 0; rr < nb; rr++) {
            const size_t row = (size_t)bh * A.Nq + list[qb + rr];
            const float2 d2 = *reinterpret_cast<const float2 *>(du + row * kD + 2 * lane);
            s_qi[warp][rr][2 * lane] = to_f<T>(Q[row * kD + 2 * lane]);
            s_qi[warp][rr][2 * lane + 1] = to_f<T>(Q[row * kD + 2 * lane + 1]);
            s_gi[warp][rr][2 * lane] = d2.x;
            s_gi[warp][rr][2 * lane + 1] = d2.y;
            if (lane == 0) s_row[warp][rr] = (int)(row - (size_t)bh * A.Nq);
        }
        __syncwarp();
        for (int rr = 0; rr < nb; rr++) {
            const float *qi = s_qi[warp][rr], *gi = s_gi[warp][rr];
            const float2 st = __ldg(reinterpret_cast<const float2 *>(rowst + ((size_t)bh * A.Nq + s_row[warp][rr]) * 4 + 2));
            float x, dp;
            dot2_lane(qi, gi, s_k[warp][lane], s_v[warp][lane], x, dp);
            const float pj = __expf(x * A.scale - st.x);     // st = (lse_lr, D_lr)
            const float dl = pj * (dp - st.y) * A.scale;
            axpy2(pj, gi, dl, qi, dv, dk);
        }
    }
    float4 *dk4 = reinterpret_cast<float4 *>(dK + t * kD), *dv4 = reinterpret_cast<float4 *>(dV + t * kD);
#pragma unroll
    for (int e = 0; e < kD / 4; e++) {
        const float4 a = dk4[e], b = dv4[e];
        dk4[e] = make_float4(a.x + dk[4 * e], a.y + dk[4 * e + 1], a.z + dk[4 * e + 2], a.w + dk[4 * e + 3]);
        dv4[e] = make_float4(b.x + dv[4 * e], b.y + dv[4 * e + 1], b.z + dv[4 * e + 2], b.w + dv[4 * e + 3]);
    }
}

// dalpha_h = sum over the rows of head h of dO.y (one CTA per head)
__global__ void __launch_bounds__(256) bwd_dalpha_kernel(const float *__restrict__ dal, int B, int H, int Nq,
                                                         float *__restrict__ dalpha) {
    __shared__ float ws[8];
    const int h = blockIdx.x, t = threadIdx.x;
    float acc = 0.f;
    for (long long e = t; e < (long long)B * Nq; e += 256) {
        const long long b = e / Nq, r = e % Nq;
        acc += dal[(b * H + h) * Nq + r];
    }
    acc = warp_sum(acc);
    if ((t & 31) == 0) ws[t >> 5] = acc;
    __syncthreads();
    if (t == 0) {
        float s = 0.f;
        for (int k = 0; k < 8; k++) s += ws[k];
        dalpha[h] = s;
    }
}

template <typename T>
fs_status run_backward(const fs_params *p, const T *Q, const T *K, const T *V, const int32_t *idx, const T *dO,
                       float *dQ, float *dK, float *dV, float *dalpha, uint8_t *ws, const BwdLayout &L,
                       cudaStream_t st) {
    BwdArgs A;
    A.B = p->B; A.H = p->H; A.Nq = p->Nq; A.Nk = p->Nk; A.C = p->Nk / p->s;
    A.w = p->w; A.K = p->K; A.q0 = p->Nk - p->Nq;
    A.scale = (float)(1.0 / std::sqrt((double)p->d));
    A.rms_eps = p->rms_eps;
    for (int h = 0; h < FS_MAX_HEADS; h++) A.alpha[h] = h < p->H ? p->alpha[h] : 0.f;
    const int BH = p->B * p->H;
    float2 *lo = reinterpret_cast<float2 *>(ws + L.rope), *hi = lo + kRopeLo * 32;
    float *krot = reinterpret_cast<float *>(ws + L.krot), *qrot = reinterpret_cast<float *>(ws + L.qrot);
    float *rowst = reinterpret_cast<float *>(ws + L.rowst), *du = reinterpret_cast<float *>(ws + L.du);
    float *dal = reinterpret_cast<float *>(ws + L.dal);
    int *cnt = reinterpret_cast<int *>(ws + L.cnt), *off = reinterpret_cast<int *>(ws + L.off);
    int *fill = reinterpret_cast<int *>(ws + L.fill), *list = reinterpret_cast<int *>(ws + L.list);
    auto ok = [] { return cudaGetLastError() == cudaSuccess; };
    if (std::is_same<T, __nv_bfloat16>::value && bwd_tc_supported(p)) {
        // bf16 with tiles of at most 128 distinct cells: both branches on the tensor cores.
        // The RoPE tables and the rotated keys (bf16, into the rotated-key segment); dK, dV
        // start at zero and take both branches' additions; the window stores dQ, the
        // readout adds to it and writes each row's dO.y.
        const Dev D = make_dev_params(p);
        void *krot16 = ws + L.krot;
        uint32_t *tiles = reinterpret_cast<uint32_t *>(ws + L.tiles);
        int *flag = reinterpret_cast<int *>(ws + L.flag);
        if (p->Nk > 0 && (launch_rope(D, p->rope_base, K, krot16, lo, hi, st) != cudaSuccess ||
                          cudaMemsetAsync(dK, 0, (size_t)BH * p->Nk * kD * 4, st) != cudaSuccess ||
                          cudaMemsetAsync(dV, 0, (size_t)BH * p->Nk * kD * 4, st) != cudaSuccess))
            return FS_ERR_CUDA;
        if (p->Nq > 0 &&
            (launch_bwd_tc(p, true, Q, K, V, krot16, nullptr, dO, dQ, dK, dV, dal, lo, hi, flag, st) != cudaSuccess ||
             launch_idx_tiles(D, idx, tiles, flag, st) != cudaSuccess ||
             launch_bwd_tc(p, false, Q, K, V, nullptr, tiles, dO, dQ, dK, dV, dal, lo, hi, flag, st) != cudaSuccess))
            return FS_ERR_CUDA;
        if (dalpha) {
            LaunchScope sc(kBwdDalpha, st);
            bwd_dalpha_kernel<<<p->H, 256, 0, st>>>(dal, p->B, p->H, p->Nq, dalpha);
            if (!ok()) return FS_ERR_CUDA;
        }
        return FS_OK;
    }
    if (launch_rope_abs_table(p->Nk, p->rope_base, lo, hi, st) != cudaSuccess) return FS_ERR_CUDA;
    if (p->Nk > 0) {
        const long long n_pairs = (long long)BH * p->Nk * (kD / 2);
        LaunchScope sc(kBwdRotate, st);
        bwd_rotate_keys_kernel<T><<<(unsigned)((n_pairs + 255) / 256), 256, 0, st>>>(K, krot, n_pairs, p->Nk, lo, hi);
        if (!ok()) return FS_ERR_CUDA;
    }
    if (p->Nq > 0) {
        LaunchScope sc(kBwdRows, st);
        const int nwin = (p->Nq + 32 * kWinWarps - 1) / (32 * kWinWarps);
        bwd_win_rows_kernel<T><<<dim3(nwin, BH), kWinWarps * 32, 0, st>>>(A, Q, V, dO, krot, lo, hi, dQ, qrot, rowst);
        if (!ok()) return FS_ERR_CUDA;
    }
    if (p->Nq > 0) {
        LaunchScope sc(kBwdLrRows, st);
        bwd_lr_rows_kernel<T><<<dim3((p->Nq + kLrWarps - 1) / kLrWarps, BH), kLrWarps * 32, 0, st>>>(
            A, Q, K, V, idx, dO, dQ, rowst, du, dal);
        if (!ok()) return FS_ERR_CUDA;
    }
    if (p->Nk > 0) {
        LaunchScope sc(kBwdWindowKv, st);
        const int nblk = (p->Nk + 32 * kKvWarps - 1) / (32 * kKvWarps);
        bwd_window_kv_kernel<T><<<dim3(nblk, BH), kKvWarps * 32, 0, st>>>(A, V, dO, krot, qrot, rowst, lo, hi, dK, dV);
        if (!ok()) return FS_ERR_CUDA;
    }
    const long long nsel = (long long)BH * p->Nq * p->K;
    if (nsel > 0 && A.C > 0) {
        const int ncell = BH * A.C;
        {
            LaunchScope sc(kBwdCells, st);
            if (cudaMemsetAsync(cnt, 0, (size_t)ncell * 4, st) != cudaSuccess ||
                cudaMemsetAsync(fill, 0, (size_t)ncell * 4, st) != cudaSuccess)
                return FS_ERR_CUDA;
            const unsigned g = (unsigned)((nsel + 255) / 256);
            bwd_count_kernel<<<g, 256, 0, st>>>(idx, nsel, p->K, p->Nq, A.C, cnt);
            bwd_scan_kernel<<<1, 1024, 0, st>>>(cnt, off, ncell);
            bwd_fill_kernel<<<g, 256, 0, st>>>(idx, nsel, p->K, p->Nq, A.C, off, fill, list);
            if (!ok()) return FS_ERR_CUDA;
        }
        LaunchScope sc(kBwdReadoutKv, st);
        bwd_readout_kv_kernel<T><<<dim3((A.C + kKvWarps - 1) / kKvWarps, BH), kKvWarps * 32, 0, st>>>(
            A, Q, K, V, du, rowst, off, list, dK, dV);
        if (!ok()) return FS_ERR_CUDA;
    }
    if (dalpha) {
        LaunchScope sc(kBwdDalpha, st);
        bwd_dalpha_kernel<<<p->H, 256, 0, st>>>(dal, p->B, p->H, p->Nq, dalpha);
        if (!ok()) return FS_ERR_CUDA;
    }
    return FS_OK;
}

}  // namespace
}  // namespace fs

using namespace fs;

extern "C" fs_status fs_backward_workspace_size(const fs_params *p, size_t *bytes) {
    const fs_status s = validate_params(p);
    if (s != FS_OK) return s;
    if (!bytes) return FS_ERR_INVALID_ARG;
    *bytes = bwd_layout(p).total;
    return FS_OK;
}

extern "C" fs_status fs_backward(const fs_params *p, const void *Q, const void *K, const void *V, const int32_t *idx,
                                 const void *dO, float *dQ, float *dK, float *dV, float *dalpha, void *bws,
                                 size_t bws_bytes, void *stream) {
    const fs_status s = validate_params(p);
    if (s != FS_OK) return s;
    if ((p->Nq > 0 && (!Q || !dO || !dQ || (p->K > 0 && !idx))) || (p->Nk > 0 && (!K || !V || !dK || !dV)))
        return FS_ERR_INVALID_ARG;
    const BwdLayout L = bwd_layout(p);
    if (!bws || bws_bytes < L.total) return FS_ERR_WORKSPACE;
    cudaStream_t st = (cudaStream_t)stream;
    uint8_t *ws = static_cast<uint8_t *>(bws);
    if (p->dtype == FS_BF16)
        return run_backward<__nv_bfloat16>(p, static_cast<const __nv_bfloat16 *>(Q), static_cast<const __nv_bfloat16 *>(K),
                                           static_cast<const __nv_bfloat16 *>(V), idx,
                                           static_cast<const __nv_bfloat16 *>(dO), dQ, dK, dV, dalpha, ws, L, st);
    return run_backward<float>(p, static_cast<const float *>(Q), static_cast<const float *>(K),
                               static_cast<const float *>(V), idx, static_cast<const float *>(dO), dQ, dK, dV,
                               dalpha, ws, L, st);
}
