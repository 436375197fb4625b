// RoPE rotation of a 128 x 64 bf16 tile held in shared memory in the 128-byte-swizzled
// layout a TMA box of 64 bf16 columns produces ("FreeSolo" summary §3.2 eq. (3); pairs
// (2m, 2m+1) rotated by angle * theta_m, theta_m = base^(-2m/d)).
#pragma once

#include "tc_common.cuh"

namespace fs {
namespace tc {

// Rotate the 128 x 64 bf16 tile `src` into `tile` (may be the same buffer).  128-byte
// swizzle: logical 16-byte chunk c of row r sits at chunk c ^ (r & 7).  Row r, pair m is
// rotated by angle (r + base_k) * theta_m: rt[r][m] holds (cos, sin)(r theta_m) and rb[m]
// (or null for base 0) (cos, sin)(base_k theta_m).  Thread t of NT threads.
template <int NT>
__device__ __forceinline__ void rotate_tile(const __nv_bfloat16 *src, __nv_bfloat16 *tile, int t,
                                            const float2 *__restrict__ rt, const float2 *__restrict__ rb) {
    uint8_t *base = reinterpret_cast<uint8_t *>(tile);
    const uint8_t *sbase = reinterpret_cast<const uint8_t *>(src);
#pragma unroll 2
    for (int j = 0; j < 1024 / NT; j++) {
        const int item = t + NT * j;
        const int row = item >> 3, c = item & 7;
        const int off = row * 128 + ((c ^ (row & 7)) << 4);
        uint4 *p = reinterpret_cast<uint4 *>(base + off);
        const uint4 x = *reinterpret_cast<const uint4 *>(sbase + off);
        const float4 *tr = reinterpret_cast<const float4 *>(rt + row * 32 + 4 * c);
        float4 a01 = __ldg(tr), a23 = __ldg(tr + 1);
        float cs[4] = {a01.x, a01.z, a23.x, a23.z}, sn[4] = {a01.y, a01.w, a23.y, a23.w};
        if (rb) {
            const float4 *tb = reinterpret_cast<const float4 *>(rb + 4 * c);
            float4 b01 = __ldg(tb), b23 = __ldg(tb + 1);
            const float cb[4] = {b01.x, b01.z, b23.x, b23.z}, sb[4] = {b01.y, b01.w, b23.y, b23.w};
#pragma unroll
            for (int e = 0; e < 4; e++) {
                const float c2 = cs[e] * cb[e] - sn[e] * sb[e];
                const float s2 = sn[e] * cb[e] + cs[e] * sb[e];
                cs[e] = c2;
                sn[e] = s2;
            }
        }
        uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
        for (int e = 0; e < 4; e++) {
            const float x0 = __uint_as_float(w[e] << 16), x1 = __uint_as_float(w[e] & 0xffff0000u);
            w[e] = pack_bf16x2(x0 * cs[e] - x1 * sn[e], x0 * sn[e] + x1 * cs[e]);
        }
        *p = make_uint4(w[0], w[1], w[2], w[3]);
    }
}

}  // namespace tc

// Absolute-position RoPE angles: pos = kRopeLo * a + b, (cos, sin)(pos theta_m) is the
// complex product of lo[b][m] and hi[a][m] (both computed in double precision).
constexpr int kRopeLo = 1024;

// (cos, sin) of pos * theta_m for the four pairs m = 4c .. 4c+3 of 16-byte chunk c.
__device__ __forceinline__ void rope_angles(int pos, int c, const float2 *__restrict__ lo,
                                            const float2 *__restrict__ hi, float (&cs)[4], float (&sn)[4]) {
    const float4 *tl = reinterpret_cast<const float4 *>(lo + (pos & (kRopeLo - 1)) * 32 + 4 * c);
    const float4 *th = reinterpret_cast<const float4 *>(hi + (pos / kRopeLo) * 32 + 4 * c);
    const float4 a01 = __ldg(tl), a23 = __ldg(tl + 1), b01 = __ldg(th), b23 = __ldg(th + 1);
    const float ca[4] = {a01.x, a01.z, a23.x, a23.z}, sa[4] = {a01.y, a01.w, a23.y, a23.w};
    const float cb[4] = {b01.x, b01.z, b23.x, b23.z}, sb[4] = {b01.y, b01.w, b23.y, b23.w};
#pragma unroll
    for (int e = 0; e < 4; e++) {
        cs[e] = ca[e] * cb[e] - sa[e] * sb[e];
        sn[e] = sa[e] * cb[e] + ca[e] * sb[e];
    }
}

// Rotate the four bf16 pairs of a 16-byte chunk: (x0, x1) -> (x0 c - x1 s, x0 s + x1 c).
__device__ __forceinline__ uint4 rope_rotate8(uint4 x, const float (&cs)[4], const float (&sn)[4]) {
    uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
    for (int e = 0; e < 4; e++) {
        const float x0 = __uint_as_float(w[e] << 16), x1 = __uint_as_float(w[e] & 0xffff0000u);
        w[e] = tc::pack_bf16x2(x0 * cs[e] - x1 * sn[e], x0 * sn[e] + x1 * cs[e]);
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
}

// First key any window of this problem reads: keys [max(0, q0 - w), Nk) are rotated.
__host__ __device__ inline int rope_first_key(const Dev &P) { return P.q0 - P.w > 0 ? P.q0 - P.w : 0; }

}  // namespace fs
