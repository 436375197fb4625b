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

}  // namespace fs
