// RoPE for the tensor-core window (bf16), "FreeSolo" summary §3.2 eq. (3): the keys any
// window will read are rotated once per call, by their absolute positions, into a
// workspace copy; the window kernel then feeds them to the tensor cores as they are.
//
// Angles: pos * theta_m with theta_m = base^(-2m/d) (interleaved pairs (2m, 2m+1)).  An
// fp32 product pos * theta_m would be off by ~0.03 rad at pos ~ 2^18, so the angle is
// split as pos = 1024 a + b and the two tables
//   lo[b][m] = (cos, sin)(b theta_m),  hi[a][m] = (cos, sin)(1024 a theta_m)
// are computed in double precision; (cos, sin)(pos theta_m) is their complex product in
// fp32 (error ~1e-7, far below the bf16 rounding of the rotated values).
#include <cmath>

#include "tc_rope.cuh"

namespace fs {

__global__ void rope_abs_table_kernel(float2 *lo, float2 *hi, int n_hi, double base) {
    const int idx = blockIdx.x * blockDim.x + threadIdx.x;
    const int m = idx & 31, row = idx >> 5;
    if (row >= kRopeLo + n_hi) return;
    const double theta = pow(base, -2.0 * m / (double)kD);
    const double pos = row < kRopeLo ? (double)row : (double)kRopeLo * (double)(row - kRopeLo);
    double s, c;
    sincos(pos * theta, &s, &c);
    const float2 v = make_float2((float)c, (float)s);
    if (row < kRopeLo) lo[row * 32 + m] = v;
    else hi[(row - kRopeLo) * 32 + m] = v;
}

// Krot[bh][j - kr0] = R(j) K[bh][j] for j in [kr0, Nk); one thread per 16-byte chunk (four
// pairs) of a key row: coalesced 16-byte loads and stores, HBM-bound.
__global__ void __launch_bounds__(256) rope_keys_kernel(const __nv_bfloat16 *__restrict__ K,
                                                        __nv_bfloat16 *__restrict__ Krot, long long n_items,
                                                        int Nk, int kr0, const float2 *__restrict__ lo,
                                                        const float2 *__restrict__ hi) {
    const long long item = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (item >= n_items) return;
    const int rows = Nk - kr0;
    const int c = (int)(item & 7);
    const long long rr = item >> 3;                 // row within the rotated range, over all heads
    const long long bh = rr / rows;
    const int j = kr0 + (int)(rr - bh * rows);
    const uint4 x = __ldg(reinterpret_cast<const uint4 *>(K + ((size_t)bh * Nk + j) * kD) + c);
    float cs[4], sn[4];
    rope_angles(j, c, lo, hi, cs, sn);
    reinterpret_cast<uint4 *>(Krot + (size_t)rr * kD)[c] = rope_rotate8(x, cs, sn);
}

// Calls that rotate few keys (decoding: the window of a few queries) build the tables and
// rotate the keys in one launch.  The table threads fill every lo row and the hi rows from
// the first rotated key's on; the key threads take (cos, sin)(j theta_m) directly in
// double precision, so they do not wait for the tables.
struct RopeTheta {
    double t[kD / 2];
};
__global__ void __launch_bounds__(256) rope_small_kernel(const __nv_bfloat16 *__restrict__ K,
                                                         __nv_bfloat16 *__restrict__ Krot, long long n_items,
                                                         int Nk, int kr0, float2 *lo, float2 *hi, int hi0,
                                                         int n_hi, const RopeTheta th) {
    const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    const int n_tab = (kRopeLo + n_hi) * 32;
    if (idx < n_tab) {
        const int m = (int)(idx & 31), row = (int)(idx >> 5);
        const double pos = row < kRopeLo ? (double)row : (double)kRopeLo * (double)(hi0 + row - kRopeLo);
        double s, c;
        sincos(pos * th.t[m], &s, &c);
        const float2 v = make_float2((float)c, (float)s);
        if (row < kRopeLo) lo[row * 32 + m] = v;
        else hi[(hi0 + row - kRopeLo) * 32 + m] = v;
        return;
    }
    const long long item = idx - n_tab;
    if (item >= n_items) return;
    const int rows = Nk - kr0;
    const int c = (int)(item & 7);
    const long long rr = item >> 3;
    const long long bh = rr / rows;
    const int j = kr0 + (int)(rr - bh * rows);
    const uint4 x = __ldg(reinterpret_cast<const uint4 *>(K + ((size_t)bh * Nk + j) * kD) + c);
    float cs[4], sn[4];
#pragma unroll
    for (int e = 0; e < 4; e++) {
        double s, co;
        sincos((double)j * th.t[4 * c + e], &s, &co);
        cs[e] = (float)co;
        sn[e] = (float)s;
    }
    reinterpret_cast<uint4 *>(Krot + (size_t)rr * kD)[c] = rope_rotate8(x, cs, sn);
}

int rope_hi_rows(int Nk) { return Nk / kRopeLo + 2; }

cudaError_t launch_rope_abs_table(int Nk, float rope_base, float2 *lo, float2 *hi, cudaStream_t st) {
    const int n_hi = rope_hi_rows(Nk);
    const int n = (kRopeLo + n_hi) * 32;
    LaunchScope scope(kRopeTable, st);
    rope_abs_table_kernel<<<(n + 255) / 256, 256, 0, st>>>(lo, hi, n_hi, (double)rope_base);
    return cudaGetLastError();
}

cudaError_t launch_rope_keys(const Dev &P, const void *K, void *Krot, const float2 *lo, const float2 *hi,
                             cudaStream_t st) {
    const int kr0 = rope_first_key(P);
    const long long n_items = (long long)P.B * P.H * (P.Nk - kr0) * 8;
    if (n_items == 0) return cudaSuccess;
    LaunchScope scope(kRopeKeys, st);
    rope_keys_kernel<<<(unsigned)((n_items + 255) / 256), 256, 0, st>>>(
        (const __nv_bfloat16 *)K, (__nv_bfloat16 *)Krot, n_items, P.Nk, kr0, lo, hi);
    return cudaGetLastError();
}

// At most this many rotated key rows per head take the one-launch path.
constexpr int kRopeSmallRows = 2048;

cudaError_t launch_rope(const Dev &P, float rope_base, const void *K, void *Krot, float2 *lo, float2 *hi,
                        cudaStream_t st) {
    const int kr0 = rope_first_key(P);
    if (P.Nk - kr0 > kRopeSmallRows) {
        if (launch_rope_abs_table(P.Nk, rope_base, lo, hi, st) != cudaSuccess) return cudaErrorLaunchFailure;
        return launch_rope_keys(P, K, Krot, lo, hi, st);
    }
    RopeTheta th;
    for (int m = 0; m < kD / 2; m++) th.t[m] = std::pow((double)rope_base, -2.0 * m / (double)kD);
    const int hi0 = kr0 / kRopeLo, n_hi = rope_hi_rows(P.Nk) - hi0;
    const long long n_items = (long long)P.B * P.H * (P.Nk - kr0) * 8;
    const long long n = (long long)(kRopeLo + n_hi) * 32 + n_items;
    LaunchScope scope(kRopeKeys, st);
    rope_small_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>((const __nv_bfloat16 *)K, (__nv_bfloat16 *)Krot,
                                                                   n_items, P.Nk, kr0, lo, hi, hi0, n_hi, th);
    return cudaGetLastError();
}
}  // namespace fs
