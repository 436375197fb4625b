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
//   rows         one warp per query row: both branches' softmax statistics, o^sr, u, y, du,
//                the per-row terms the key kernels need (log-sum-exps, g.o), dQ, dalpha terms
//   window_kv    one warp per 32 keys (lane = key): dK, dV over the queries whose window
//                holds them; writes every key (zeros where none)
//   cells        cell -> rows lists by counting sort of idx (count, scan, fill)
//   readout_kv   one warp per cell (lane = token): adds the readout's dK, dV over the rows
//                that selected the cell
//   dalpha       per-head sum of the rows' dO.y
#include <cmath>

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
    size_t rope, krot, qrot, rowst, du, dal, cnt, off, fill, list, total;
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

// lane j's dot product of the shared 64-vector v with the 64 floats (or T) at row
template <typename R> __device__ __forceinline__ float dot_row(const float *v, const R *row) {
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int e = 0; e < kD; e++) acc[e & 3] = fmaf(v[e], to_f<R>(row[e]), acc[e & 3]);
    return (acc[0] + acc[1]) + (acc[2] + acc[3]);
}
template <> __device__ __forceinline__ float dot_row<float>(const float *v, const float *row) {
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    const float4 *r4 = reinterpret_cast<const float4 *>(row);
#pragma unroll
    for (int e = 0; e < kD / 4; e++) {
        const float4 x = __ldg(r4 + e);
        acc[0] = fmaf(v[4 * e], x.x, acc[0]);
        acc[1] = fmaf(v[4 * e + 1], x.y, acc[1]);
        acc[2] = fmaf(v[4 * e + 2], x.z, acc[2]);
        acc[3] = fmaf(v[4 * e + 3], x.w, acc[3]);
    }
    return (acc[0] + acc[1]) + (acc[2] + acc[3]);
}

constexpr int kRowWarps = 8;

template <typename T>
__global__ void __launch_bounds__(kRowWarps * 32) bwd_rows_kernel(
    const BwdArgs A, const T *__restrict__ Q, const T *__restrict__ K, const T *__restrict__ V,
    const int32_t *__restrict__ idx, const T *__restrict__ dO, const float *__restrict__ krot,
    const float2 *__restrict__ lo, const float2 *__restrict__ hi, float *__restrict__ dQ, float *__restrict__ qrot,
    float *__restrict__ rowst, float *__restrict__ du_out, float *__restrict__ dal) {
    __shared__ float s_q[kRowWarps][kD], s_qr[kRowWarps][kD], s_g[kRowWarps][kD], s_du[kRowWarps][kD];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int bh = blockIdx.y, h = bh % A.H;
    const int r = blockIdx.x * kRowWarps + warp;
    if (r >= A.Nq) return;                                   // warp-uniform
    const size_t row = (size_t)bh * A.Nq + r;
    const int i = A.q0 + r;
    const size_t kb = (size_t)bh * A.Nk;
    // lane m holds the pair (2m, 2m+1) of q, R_i q and dO
    const float q0 = to_f<T>(Q[row * kD + 2 * lane]), q1 = to_f<T>(Q[row * kD + 2 * lane + 1]);
    const float2 cs = rope_cs_tab(i, lane, lo, hi);
    const float qr0 = q0 * cs.x - q1 * cs.y, qr1 = q0 * cs.y + q1 * cs.x;
    const float g0 = to_f<T>(dO[row * kD + 2 * lane]), g1 = to_f<T>(dO[row * kD + 2 * lane + 1]);
    s_q[warp][2 * lane] = q0; s_q[warp][2 * lane + 1] = q1;
    s_qr[warp][2 * lane] = qr0; s_qr[warp][2 * lane + 1] = qr1;
    s_g[warp][2 * lane] = g0; s_g[warp][2 * lane + 1] = g1;
    qrot[row * kD + 2 * lane] = qr0;
    qrot[row * kD + 2 * lane + 1] = qr1;
    __syncwarp();

    // ---- window: statistics and o^sr (lane = key for the logits, lane = pair for p V)
    const int jlo = max(0, i - A.w), L = i - jlo + 1;
    float m = -INFINITY, l = 0.f, o0 = 0.f, o1 = 0.f;
    for (int b = 0; b * 32 < L; b++) {
        const int j = jlo + 32 * b + lane;
        const bool ok = j <= i;
        const float x = ok ? dot_row<float>(s_qr[warp], krot + (kb + j) * kD) * A.scale : -INFINITY;
        const float mn = fmaxf(m, warp_max(x));
        const float corr = m == -INFINITY ? 0.f : __expf(m - mn);
        const float pj = ok ? __expf(x - mn) : 0.f;
        l = l * corr + warp_sum(pj);
        o0 *= corr;
        o1 *= corr;
        const int nb = min(32, L - 32 * b);
        for (int e = 0; e < nb; e++) {
            const float pe = __shfl_sync(kFull, pj, e);
            const T *vr = V + (kb + jlo + 32 * b + e) * kD + 2 * lane;
            o0 = fmaf(pe, to_f<T>(vr[0]), o0);
            o1 = fmaf(pe, to_f<T>(vr[1]), o1);
        }
        m = mn;
    }
    o0 /= l;
    o1 /= l;
    const float lse_sr = m + __logf(l);
    const float D_sr = warp_sum(g0 * o0 + g1 * o1);
    // dq' = sum_j dl_j k'_j
    float dq0 = 0.f, dq1 = 0.f;
    for (int b = 0; b * 32 < L; b++) {
        const int j = jlo + 32 * b + lane;
        const bool ok = j <= i;
        float dl = 0.f;
        if (ok) {
            const float x = dot_row<float>(s_qr[warp], krot + (kb + j) * kD) * A.scale;
            const float pj = __expf(x - lse_sr);
            const float dp = dot_row<T>(s_g[warp], V + (kb + j) * kD);
            dl = pj * (dp - D_sr) * A.scale;
        }
        const int nb = min(32, L - 32 * b);
        for (int e = 0; e < nb; e++) {
            const float de = __shfl_sync(kFull, dl, e);
            const float *kr = krot + (kb + jlo + 32 * b + e) * kD + 2 * lane;
            dq0 = fmaf(de, kr[0], dq0);
            dq1 = fmaf(de, kr[1], dq1);
        }
    }
    // rotate back: R_i^T
    float dqa = dq0 * cs.x + dq1 * cs.y, dqb = -dq0 * cs.y + dq1 * cs.x;

    // ---- readout over the selected cells' tokens (NoPE)
    const int32_t *sel = idx + row * A.K;
    int ncell = 0;
    for (int e = 0; e < A.K; e++) ncell += (unsigned)sel[e] < (unsigned)A.C;
    float lse_lr = -INFINITY, D_lr = 0.f, gy = 0.f;
    float du0 = 0.f, du1 = 0.f;
    if (ncell > 0) {
        m = -INFINITY; l = 0.f;
        float u0 = 0.f, u1 = 0.f;
        for (int e = 0; e < A.K; e++) {
            const int c = sel[e];
            if ((unsigned)c >= (unsigned)A.C) continue;
            const size_t t0 = kb + (size_t)c * kS;
            const float x = dot_row<T>(s_q[warp], K + (t0 + lane) * kD) * A.scale;
            const float mn = fmaxf(m, warp_max(x));
            const float corr = m == -INFINITY ? 0.f : __expf(m - mn);
            const float pj = __expf(x - mn);
            l = l * corr + warp_sum(pj);
            u0 *= corr;
            u1 *= corr;
            for (int t = 0; t < kS; t++) {
                const float pe = __shfl_sync(kFull, pj, t);
                const T *vr = V + (t0 + t) * kD + 2 * lane;
                u0 = fmaf(pe, to_f<T>(vr[0]), u0);
                u1 = fmaf(pe, to_f<T>(vr[1]), u1);
            }
            m = mn;
        }
        u0 /= l;
        u1 /= l;
        lse_lr = m + __logf(l);
        const float ss = warp_sum(u0 * u0 + u1 * u1);
        const float rin = rsqrtf(ss * (1.f / kD) + A.rms_eps);
        const float y0 = u0 * rin, y1 = u1 * rin;
        gy = warp_sum(g0 * y0 + g1 * y1);
        const float a = A.alpha[h];
        const float dyy = a * gy;                                // dy.y with dy = alpha dO
        du0 = rin * (a * g0 - y0 * dyy * (1.f / kD));
        du1 = rin * (a * g1 - y1 * dyy * (1.f / kD));
        D_lr = warp_sum(du0 * u0 + du1 * u1);
        s_du[warp][2 * lane] = du0;
        s_du[warp][2 * lane + 1] = du1;
        __syncwarp();
        for (int e = 0; e < A.K; e++) {
            const int c = sel[e];
            if ((unsigned)c >= (unsigned)A.C) continue;
            const size_t t0 = kb + (size_t)c * kS;
            const float x = dot_row<T>(s_q[warp], K + (t0 + lane) * kD) * A.scale;
            const float pj = __expf(x - lse_lr);
            const float dp = dot_row<T>(s_du[warp], V + (t0 + lane) * kD);
            const float dl = pj * (dp - D_lr) * A.scale;
            for (int t = 0; t < kS; t++) {
                const float de = __shfl_sync(kFull, dl, t);
                const T *kr = K + (t0 + t) * kD + 2 * lane;
                dqa = fmaf(de, to_f<T>(kr[0]), dqa);
                dqb = fmaf(de, to_f<T>(kr[1]), dqb);
            }
        }
    }
    dQ[row * kD + 2 * lane] = dqa;
    dQ[row * kD + 2 * lane + 1] = dqb;
    du_out[row * kD + 2 * lane] = du0;
    du_out[row * kD + 2 * lane + 1] = du1;
    if (lane == 0) {
        reinterpret_cast<float4 *>(rowst)[row] = make_float4(lse_sr, D_sr, lse_lr, D_lr);
        dal[row] = gy;
    }
}

constexpr int kKvWarps = 2, kPad = kD + 1;   // 2 warps: 33 KB of static shared memory

// Window dK, dV: warp = 32 consecutive keys (lane = key j), over the queries i whose window
// [i - w, i] holds some key of the block; dK_j = R_j^T sum_i dl_ij q'_i.  Every key is written.
template <typename T>
__global__ void __launch_bounds__(kKvWarps * 32) bwd_window_kv_kernel(
    const BwdArgs A, const T *__restrict__ V, const T *__restrict__ dO, const float *__restrict__ krot,
    const float *__restrict__ qrot, const float *__restrict__ rowst, const float2 *__restrict__ lo,
    const float2 *__restrict__ hi, float *__restrict__ dK, float *__restrict__ dV) {
    __shared__ float s_k[kKvWarps][32][kPad], s_v[kKvWarps][32][kPad];
    __shared__ float s_qi[kKvWarps][kD], s_gi[kKvWarps][kD];
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
    // queries at positions i in [j0, j0 + 31 + w] that exist
    const int ilo = max(j0, A.q0), ihi = min(j0 + 31 + A.w, A.q0 + A.Nq - 1);
    for (int i = ilo; i <= ihi; i++) {
        const size_t row = (size_t)bh * A.Nq + (i - A.q0);
        __syncwarp();
        s_qi[warp][2 * lane] = qrot[row * kD + 2 * lane];
        s_qi[warp][2 * lane + 1] = qrot[row * kD + 2 * lane + 1];
        s_gi[warp][2 * lane] = to_f<T>(dO[row * kD + 2 * lane]);
        s_gi[warp][2 * lane + 1] = to_f<T>(dO[row * kD + 2 * lane + 1]);
        __syncwarp();
        const float4 st = __ldg(reinterpret_cast<const float4 *>(rowst) + row);   // lse_sr, D_sr, ...
        if (!kv_ok || j > i || j < i - A.w) continue;
        float x = 0.f, dp = 0.f;
#pragma unroll
        for (int e = 0; e < kD; e++) {
            x = fmaf(s_qi[warp][e], s_k[warp][lane][e], x);
            dp = fmaf(s_gi[warp][e], s_v[warp][lane][e], dp);
        }
        const float pj = __expf(x * A.scale - st.x);
        const float dl = pj * (dp - st.y) * A.scale;
#pragma unroll
        for (int e = 0; e < kD; e++) {
            dv[e] = fmaf(pj, s_gi[warp][e], dv[e]);
            dk[e] = fmaf(dl, s_qi[warp][e], dk[e]);
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
    __shared__ float s_qi[kKvWarps][kD], s_gi[kKvWarps][kD];
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
    for (int q = b0; q < b1; q++) {
        const size_t row = (size_t)bh * A.Nq + list[q];
        __syncwarp();
        s_qi[warp][2 * lane] = to_f<T>(Q[row * kD + 2 * lane]);
        s_qi[warp][2 * lane + 1] = to_f<T>(Q[row * kD + 2 * lane + 1]);
        s_gi[warp][2 * lane] = du[row * kD + 2 * lane];
        s_gi[warp][2 * lane + 1] = du[row * kD + 2 * lane + 1];
        __syncwarp();
        const float4 st = __ldg(reinterpret_cast<const float4 *>(rowst) + row);   // ..., lse_lr, D_lr
        float x = 0.f, dp = 0.f;
#pragma unroll
        for (int e = 0; e < kD; e++) {
            x = fmaf(s_qi[warp][e], s_k[warp][lane][e], x);
            dp = fmaf(s_gi[warp][e], s_v[warp][lane][e], dp);
        }
        const float pj = __expf(x * A.scale - st.z);
        const float dl = pj * (dp - st.w) * A.scale;
#pragma unroll
        for (int e = 0; e < kD; e++) {
            dv[e] = fmaf(pj, s_gi[warp][e], dv[e]);
            dk[e] = fmaf(dl, s_qi[warp][e], dk[e]);
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
    if (launch_rope_abs_table(p->Nk, p->rope_base, lo, hi, st) != cudaSuccess) return FS_ERR_CUDA;
    if (p->Nk > 0) {
        const long long n_pairs = (long long)BH * p->Nk * (kD / 2);
        LaunchScope sc(kBwdRotate, st);
        bwd_rotate_keys_kernel<T><<<(unsigned)((n_pairs + 255) / 256), 256, 0, st>>>(K, krot, n_pairs, p->Nk, lo, hi);
        if (!ok()) return FS_ERR_CUDA;
    }
    if (p->Nq > 0) {
        LaunchScope sc(kBwdRows, st);
        bwd_rows_kernel<T><<<dim3((p->Nq + kRowWarps - 1) / kRowWarps, BH), kRowWarps * 32, 0, st>>>(
            A, Q, K, V, idx, dO, krot, lo, hi, dQ, qrot, rowst, du, dal);
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
