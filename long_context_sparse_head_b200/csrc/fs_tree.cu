// FS-B selection ("FreeSolo" summary §3.4, eqs. (10)-(11)): beam search over two causal
// forests of balanced trees.
//   forest 0 holds every cell in time order (admitted set A^0_i = C_i, eq. (10));
//   forest 1 the cells with a_c >= tau_h in time order (A^tau_i, eq. (10)).
// Over a forest's sequence there is one balanced binary tree per aligned block of 2^k
// entries, every k; a query whose prefix holds m entries searches the trees of the set
// bits of m (those a binary counter holds after m insertions: the growing archive).
// A tree's leaves are its block's cells sorted by a 16-bit code (the signs of the first
// 16 coordinates of kbar_c, coordinate 0 the most significant bit; ties by time): level
// k's order is the stable merge of level k-1's two halves, i.e. the radix order.  Node v
// of the complete binary tree over that order stores
//   mu_v = mean kbar_c, rho_v = max ||kbar_c - mu_v||, A_v = max a_c, p_v^min = min p_c
// over its leaves, and eq. (11) scores it for query i:
//   U_v = (q_i.mu_v + c ||q_i|| rho_v) / sqrt(d) + lambda_h A_v erf((i - p_v^min) / (2 sigma_h)).
// Beam search of width beta per forest: start from the prefix's roots (keep the beta best),
// then replace every internal node of the beam by its two children and keep the beta best
// (U descending, ties to the lower p_v^min), until the beam holds only leaves.  S_i = the K
// best cells by eq. (7) among both beams' leaves (a leaf's U_v is its eq. (7) score),
// ascending, -1 padded.
//
// Kernels: prep (codes, admitted prefix counts, sequences; one CTA per head), merge (one
// launch per level; each entry's place by binary search in the other half), node
// statistics (bottom-up means, max norms and first cells per tree, then radii with one
// thread per leaf), search (one warp per query row; a right child's q.mu is
// 2 q.mu_parent - q.mu_left, so an expansion reads one mean).
#include <algorithm>
#include <cmath>

#include "fs_common.cuh"

namespace fs {

namespace {

constexpr int kTreeMagic = 0x46534254;
constexpr int kMaxBeam = FS_TREE_MAX_BEAM;
constexpr int kCodeBits = 16;
constexpr int kSearchWarps = 4;
constexpr int kCandCap = 2 * kMaxBeam + 32;   // children of a full beam, or the roots

// A forest buffer is laid out for a capacity of C cells (the largest count whose forest
// fits in the buffer's bytes); the cells built so far may be fewer.  Header words: magic,
// has_tau, capacity, levels, B*H, cells built, error (a failed append check).
enum { kHdrMagic = 0, kHdrTau, kHdrCap, kHdrLevels, kHdrBH, kHdrCells, kHdrError };

struct ForestGeom {
    int BH, C, L;           // C: capacity (layout stride)
    size_t hdr, nseq, nprev, seq, admp, code, ord, mu, meta, total;
};

size_t al256(size_t x) { return (x + 255) & ~size_t(255); }

ForestGeom forest_geom(int BHn, int Ccap) {
    ForestGeom g;
    g.BH = BHn;
    g.C = Ccap;
    g.L = 0;
    while (g.L < 31 && (1LL << g.L) <= g.C) g.L++;
    const size_t BH = g.BH, C = g.C, L = g.L > 0 ? g.L : 1;
    size_t off = 0;
    auto seg = [&](size_t bytes) {
        const size_t o = off;
        off += al256(bytes);
        return o;
    };
    g.hdr = seg(16 * 4);
    g.nseq = seg(BH * 2 * 4);
    g.nprev = seg(BH * 2 * 4);              // sequence lengths before the last build / append
    g.seq = seg(BH * 2 * C * 4);
    g.admp = seg(BH * (C + 1) * 4);
    g.code = seg(BH * C * 4);
    g.ord = seg(BH * 2 * L * C * 4);
    g.mu = seg(BH * 2 * L * 2 * C * kD * 4);
    g.meta = seg(BH * 2 * L * 2 * C * 16);
    g.total = off;
    return g;
}

// Device view of a forest buffer.
struct Forest {
    int *hdr, *nseq, *nprev, *seq, *admp;
    uint32_t *code;
    int *ord;
    float *mu;
    float4 *meta;       // (rho, A, pmin as int bits, 0)
    int C, L;
    __device__ __forceinline__ size_t lvl(int bh, int f, int k) const {
        return ((size_t)(bh * 2 + f) * L + k);
    }
};

Forest forest_view(void *buf, const ForestGeom &g) {
    uint8_t *b = static_cast<uint8_t *>(buf);
    Forest F;
    F.hdr = reinterpret_cast<int *>(b + g.hdr);
    F.nseq = reinterpret_cast<int *>(b + g.nseq);
    F.nprev = reinterpret_cast<int *>(b + g.nprev);
    F.seq = reinterpret_cast<int *>(b + g.seq);
    F.admp = reinterpret_cast<int *>(b + g.admp);
    F.code = reinterpret_cast<uint32_t *>(b + g.code);
    F.ord = reinterpret_cast<int *>(b + g.ord);
    F.mu = reinterpret_cast<float *>(b + g.mu);
    F.meta = reinterpret_cast<float4 *>(b + g.meta);
    F.C = g.C;
    F.L = g.L;
    return F;
}

// codes, sequences and admitted prefix counts of one (b, h); 1024 threads
struct TauArgs {
    float tau[FS_MAX_HEADS];
};

// cells [prev, Cn) of one (b, h): codes, sequences, admitted prefix counts (continuing the
// scan at admp[prev]).  An append (prev > 0) first checks that the forest was built for
// these sizes, these thresholds' presence and at least prev cells; a mismatch is recorded
// in the header and reported by the search.
__global__ void __launch_bounds__(1024) tree_prep_kernel(Forest F, const float *__restrict__ kbar,
                                                         const float *__restrict__ amax, int H, int has_tau,
                                                         const TauArgs T, int Cn, int prev) {
    __shared__ int wsum[32];
    __shared__ int carry;
    const int bh = blockIdx.x, t = threadIdx.x, lane = t & 31, warp = t >> 5;
    const int C = F.C;                             // capacity: the layout's stride
    const float tau = has_tau ? T.tau[bh % H] : 0.f;
    if (t == 0) {
        carry = 0;
        if (prev > 0) {
            const bool ok = F.hdr[kHdrMagic] == kTreeMagic && F.hdr[kHdrTau] == has_tau && F.hdr[kHdrCap] == C &&
                            F.hdr[kHdrLevels] == F.L && F.hdr[kHdrBH] == (int)gridDim.x && F.hdr[kHdrCells] >= prev;
            if (!ok) atomicOr(F.hdr + kHdrError, kFlagCheck);
            carry = ok ? F.admp[(size_t)bh * (C + 1) + prev] : 0;
        }
        F.nprev[bh * 2 + 0] = prev;
        F.nprev[bh * 2 + 1] = carry;
    }
    __syncthreads();
    for (int base = prev; base < Cn; base += 1024) {
        const int c = base + t;
        int adm = 0;
        if (c < Cn) {
            const float *kb = kbar + ((size_t)bh * Cn + c) * kD;      // caller's arrays: [B*H, Cn]
            uint32_t code = 0;
#pragma unroll
            for (int b = 0; b < kCodeBits; b++) code = (code << 1) | (kb[b] > 0.f ? 1u : 0u);
            F.code[(size_t)bh * C + c] = code;
            F.seq[((size_t)bh * 2 + 0) * C + c] = c;
            adm = has_tau && amax[(size_t)bh * Cn + c] >= tau;
        }
        int incl = adm;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(kFull, incl, o);
            if (lane >= o) incl += y;
        }
        if (lane == 31) wsum[warp] = incl;
        __syncthreads();
        int before = carry;
        for (int k = 0; k < warp; k++) before += wsum[k];
        const int excl = before + incl - adm;
        if (c < Cn) {
            F.admp[(size_t)bh * (C + 1) + c] = excl;
            if (adm) F.seq[((size_t)bh * 2 + 1) * C + excl] = c;
        }
        __syncthreads();
        if (t == 1023) carry = excl + adm;
        __syncthreads();
    }
    if (t == 0) {
        F.admp[(size_t)bh * (C + 1) + Cn] = carry;
        F.nseq[bh * 2 + 0] = Cn;
        F.nseq[bh * 2 + 1] = carry;
    }
}

// Header of a finished build or append (one thread, after every other kernel of it).
__global__ void tree_header_kernel(Forest F, int BH, int has_tau, int Cn, int full) {
    F.hdr[kHdrMagic] = kTreeMagic;
    F.hdr[kHdrTau] = has_tau;
    F.hdr[kHdrCap] = F.C;
    F.hdr[kHdrLevels] = F.L;
    F.hdr[kHdrBH] = BH;
    F.hdr[kHdrCells] = Cn;
    if (full) F.hdr[kHdrError] = 0;
}

__device__ __forceinline__ unsigned long long sort_key(const Forest &F, int bh, int cell) {
    return ((unsigned long long)F.code[(size_t)bh * F.C + cell] << 32) | (unsigned)cell;
}

// level k's leaf order: level 0 copies the sequence; level k >= 1 merges the two sorted
// halves of each block (an entry's place = its index in its half + the number of keys
// below it in the other half).  Only the blocks completed since the previous build are
// done: entry positions base + r, base = the first position of a new block, r < span.
__global__ void tree_merge_kernel(Forest F, int BH, int k, int span) {
    const long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    const int C = F.C;
    if (e >= (long long)BH * 2 * span) return;
    const int bhf = (int)(e / span), bh = bhf >> 1, f = bhf & 1;
    const int pos = ((F.nprev[bhf] >> k) << k) + (int)(e % span);
    const int n = F.nseq[bhf];
    if (pos >= ((n >> k) << k)) return;
    int *out = F.ord + F.lvl(bh, f, k) * C;
    if (k == 0) {
        out[pos] = F.seq[(size_t)bhf * C + pos];
        return;
    }
    const int *in = F.ord + F.lvl(bh, f, k - 1) * C;
    const int hlen = 1 << (k - 1);
    const int blk = pos >> k, half = (pos >> (k - 1)) & 1, a = pos & (hlen - 1);
    const int cell = in[pos];
    const unsigned long long key = sort_key(F, bh, cell);
    const int *other = in + ((size_t)(2 * blk + (half ^ 1)) << (k - 1));
    int lo = 0, hi = hlen;                      // keys of the other half below `key`
    while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (sort_key(F, bh, other[mid]) < key) lo = mid + 1;
        else hi = mid;
    }
    out[(blk << k) + a + lo] = cell;
}

// Node statistics of level k, in two passes.
// (1) tree_up_kernel: bottom-up over each tree's depths.  A leaf holds its cell's kbar_c,
//     a_c and index; an internal node's mean is the average of its two children's (they
//     cover equally many leaves), its max norm and first cell the larger / smaller of
//     theirs; every radius starts at 0.  Work items are subtrees of at most 128 leaves,
//     one warp each (grid-stride): depths k down to d0 = max(0, k - 7); for k > 7 a second
//     launch takes each tree's top depths d0 - 1 .. 0 (at most 63 nodes), again one warp.
//     A warp takes four nodes of a depth at a time, their loads issued together.
// (2) tree_radius_kernel: rho_v = max ||kbar_c - mu_v|| over v's leaves.  One thread per
//     leaf holds its kbar_c and walks the depths above it; a node of fewer than 32 leaves
//     lies inside one warp and takes a butterfly maximum, a larger one a warp maximum and
//     an atomic maximum on the radius's bits (non-negative floats order as integers, so
//     the result does not depend on the order).
constexpr int kUpThreads = 256, kUpSubK = 7, kUpBatch = 4, kUpMaxBlocks = 148 * 8;

__device__ __forceinline__ size_t node_index(const Forest &F, int bh, int f, int k, int blk, int v) {
    return F.lvl(bh, f, k) * 2 * (size_t)F.C + ((size_t)blk << (k + 1)) + v;
}

// top == 0: items are (tree, subtree rooted at depth d0); top == 1: items are trees, and the
// warp fills depths d0 - 1 .. 0.  The trees are those completed since the previous build:
// blocks nprev >> k + r, r < per, below nseq >> k.
__global__ void __launch_bounds__(kUpThreads) tree_up_kernel(Forest F, const float *__restrict__ kbar,
                                                             const float *__restrict__ amax, int BH, int k, int top,
                                                             int per, int Cn) {
    const int lane = threadIdx.x & 31;
    const int C = F.C;
    const int d0 = k > kUpSubK ? k - kUpSubK : 0;
    const int subs = top ? 1 : 1 << d0;                     // items per tree
    const long long items = (long long)BH * 2 * per * subs;
    const long long nwarps = (long long)gridDim.x * (kUpThreads / 32);
    for (long long it = ((long long)blockIdx.x * kUpThreads + threadIdx.x) >> 5; it < items; it += nwarps) {
        const long long tree = it / subs;
        const int sub = (int)(it - tree * subs);
        const int bhf = (int)(tree / per), bh = bhf >> 1, f = bhf & 1;
        const int blk = (F.nprev[bhf] >> k) + (int)(tree % per);
        if (blk >= (F.nseq[bhf] >> k)) continue;             // uniform across the warp
        const int *ord = F.ord + F.lvl(bh, f, k) * C + ((size_t)blk << k);
        const float *kb = kbar + (size_t)bh * Cn * kD;         // caller's arrays: [B*H, Cn]
        const int t_hi = top ? d0 - 1 : k, t_lo = top ? 0 : d0;
        for (int t = t_hi; t >= t_lo; t--) {
            // nodes of this item at depth t: [v_first, v_first + n)
            const int n = top ? 1 << t : 1 << (t - d0);
            const int v_first = top ? 1 << t : ((1 << d0) + sub) << (t - d0);
            for (int i0 = 0; i0 < n; i0 += kUpBatch) {
                float2 m[kUpBatch];
                float A[kUpBatch];
                int pmin[kUpBatch];
#pragma unroll
                for (int u = 0; u < kUpBatch; u++) {
                    const int v = v_first + i0 + u;
                    if (i0 + u >= n) continue;
                    if (t == k) {
                        const int c = ord[v - (1 << k)];
                        m[u] = *reinterpret_cast<const float2 *>(kb + (size_t)c * kD + 2 * lane);
                        A[u] = amax[(size_t)bh * Cn + c];
                        pmin[u] = c;
                    } else {
                        const size_t nl = node_index(F, bh, f, k, blk, 2 * v), nr = nl + 1;   // children
                        const float2 a = *reinterpret_cast<const float2 *>(F.mu + nl * kD + 2 * lane);
                        const float2 b = *reinterpret_cast<const float2 *>(F.mu + nr * kD + 2 * lane);
                        m[u] = make_float2(0.5f * (a.x + b.x), 0.5f * (a.y + b.y));
                        const float4 ml = F.meta[nl], mr = F.meta[nr];
                        A[u] = fmaxf(ml.y, mr.y);
                        pmin[u] = min(__float_as_int(ml.z), __float_as_int(mr.z));
                    }
                }
#pragma unroll
                for (int u = 0; u < kUpBatch; u++) {
                    if (i0 + u >= n) continue;
                    const size_t ni = node_index(F, bh, f, k, blk, v_first + i0 + u);
                    *reinterpret_cast<float2 *>(F.mu + ni * kD + 2 * lane) = m[u];
                    if (lane == 0) F.meta[ni] = make_float4(0.f, A[u], __int_as_float(pmin[u]), 0.f);
                }
            }
            __syncwarp();
        }
    }
}

__global__ void __launch_bounds__(256) tree_radius_kernel(Forest F, const float *__restrict__ kbar, int BH, int k,
                                                          int per, int Cn) {
    const int lane = threadIdx.x & 31;
    const int C = F.C;
    const long long per_bhf = (long long)per << k;          // leaf slots per (bh, f): new trees only
    const long long id = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if ((id & ~31LL) >= (long long)BH * 2 * per_bhf) return;   // whole warps only
    const bool live = id < (long long)BH * 2 * per_bhf;
    const int bhf = live ? (int)(id / per_bhf) : 0, bh = bhf >> 1, f = bhf & 1;
    const long long r = live ? id % per_bhf : 0;
    const int blk = (F.nprev[bhf] >> k) + (int)(r >> k), j = (int)(r & ((1 << k) - 1));
    const bool have = live && blk < (F.nseq[bhf] >> k);
    float x[kD];
    if (have) {
        const int c = F.ord[F.lvl(bh, f, k) * C + ((size_t)blk << k) + j];
        const float4 *src = reinterpret_cast<const float4 *>(kbar + ((size_t)bh * Cn + c) * kD);
#pragma unroll
        for (int q = 0; q < kD / 4; q++) {
            const float4 v = __ldg(src + q);
            x[4 * q] = v.x; x[4 * q + 1] = v.y; x[4 * q + 2] = v.z; x[4 * q + 3] = v.w;
        }
    }
    for (int t = k - 1; t >= 0; t--) {
        const int sz = 1 << (k - t);                         // leaves per node at depth t
        const int v = (1 << t) + (j >> (k - t));
        const size_t ni = have ? node_index(F, bh, f, k, blk, v) : 0;
        float d2 = 0.f;
        if (have) {
            const float4 *mu = reinterpret_cast<const float4 *>(F.mu + ni * kD);
#pragma unroll
            for (int q = 0; q < kD / 4; q++) {
                const float4 m = mu[q];
                const float a = x[4 * q] - m.x, b = x[4 * q + 1] - m.y, c = x[4 * q + 2] - m.z, e = x[4 * q + 3] - m.w;
                d2 = fmaf(a, a, fmaf(b, b, fmaf(c, c, fmaf(e, e, d2))));
            }
        }
        // trees never straddle a warp (sizes are powers of two), and a tree missing from
        // the sequence is missing for all of its lanes, so `have` is uniform per node
        const int span = sz < 32 ? sz : 32;
        for (int o = 1; o < span; o <<= 1) d2 = fmaxf(d2, __shfl_xor_sync(kFull, d2, o));
        if (have && (lane & (span - 1)) == 0) {
            const float rho = sqrtf(d2);
            if (sz <= 32) F.meta[ni].x = rho;                // the node lies inside this warp
            else atomicMax(reinterpret_cast<int *>(&F.meta[ni].x), __float_as_int(rho));
        }
    }
}

struct SearchArgs {
    int Nq, H, w, K, q0, beam;
    int cells;              // C = floor(Nk / s) of the call (at most the forest's capacity)
    float scale, c_explore;
    float lambda[FS_MAX_HEADS], inv2sigma[FS_MAX_HEADS];
};

struct SearchSmem {
    float q[kD];
    float U[kCandCap];
    int ref[kCandCap];      // level << 26 | node slot
    int pmin[kCandCap];
    float dot[kCandCap];    // q . mu_v
    float bU[kMaxBeam];
    int bref[kMaxBeam], bpmin[kMaxBeam];
    float bdot[kMaxBeam];
    float rU[2 * kMaxBeam];  // leaves both beams end on
    int rcell[2 * kMaxBeam];
};

__device__ __forceinline__ bool beats(float Ua, int pa, float Ub, int pb) {
    return Ua > Ub || (Ua == Ub && pa < pb);
}

// Bitonic sort of the warp's 32E entries (entry i = e*32 + lane: score U, tie key pm, ref),
// better first (beats()).  Partners closer than 32 are exchanged by shuffles, the others
// within the lane's registers.
template <int E>
__device__ __forceinline__ void warp_sort(float (&U)[E], int (&pm)[E], int (&rf)[E], int lane) {
    constexpr int P = 32 * E;
#pragma unroll
    for (int k = 2; k <= P; k <<= 1) {
#pragma unroll
        for (int d = k >> 1; d > 0; d >>= 1) {
            if (d >= 32) {
#pragma unroll
                for (int e = 0; e < E; e++) {
                    const int f = e ^ (d >> 5);
                    if (f <= e) continue;              // each pair once, from its lower entry
                    const bool desc = ((e * 32 + lane) & k) == 0;   // better to the lower index
                    if (beats(U[f], pm[f], U[e], pm[e]) == desc) {
                        const float tu = U[e]; U[e] = U[f]; U[f] = tu;
                        const int tp = pm[e]; pm[e] = pm[f]; pm[f] = tp;
                        const int tr = rf[e]; rf[e] = rf[f]; rf[f] = tr;
                    }
                }
            } else {
#pragma unroll
                for (int e = 0; e < E; e++) {
                    const float Ub = __shfl_xor_sync(kFull, U[e], d);
                    const int pb = __shfl_xor_sync(kFull, pm[e], d);
                    const int rb = __shfl_xor_sync(kFull, rf[e], d);
                    const bool lower = (lane & d) == 0, desc = ((e * 32 + lane) & k) == 0;
                    const bool better = beats(Ub, pb, U[e], pm[e]);
                    if ((lower == desc) ? better : !better) {
                        U[e] = Ub;
                        pm[e] = pb;
                        rf[e] = rb;
                    }
                }
            }
        }
    }
}

// The beam: the nb = min(n, beta) best of the n candidates in S.U/S.pmin/S.ref, sorted,
// into S.bU/S.bpmin/S.bref (entries past n are padding that never wins)
template <int E, typename Smem>
__device__ __forceinline__ void beam_cut(Smem &S, int n, int nb, int lane) {
    float U[E];
    int pm[E], rf[E];
#pragma unroll
    for (int e = 0; e < E; e++) {
        const int i = e * 32 + lane;
        U[e] = i < n ? S.U[i] : -INFINITY;
        pm[e] = i < n ? S.pmin[i] : 0x7fffffff;
        rf[e] = i < n ? i : 0;                        // the candidate's index
    }
    warp_sort<E>(U, pm, rf, lane);
#pragma unroll
    for (int e = 0; e < E; e++) {
        const int i = e * 32 + lane;
        if (i < nb) {
            S.bU[i] = U[e];
            S.bpmin[i] = pm[e];
            S.bref[i] = S.ref[rf[e]];
            S.bdot[i] = S.dot[rf[e]];
        }
    }
}

// eq. (11) for one node (lane-local: the whole dot product in this lane)
// eq. (11) for a node whose q . mu_v is known (meta loads only)
template <bool PRIOR>
__device__ __forceinline__ float node_U_dot(const Forest &F, size_t lvl_base, int node, float dot, float qn,
                                            const SearchArgs &A, int h, int i, int *pmin_out) {
    const float4 mt = __ldg(F.meta + lvl_base + node);
    const int pmin = __float_as_int(mt.z);
    *pmin_out = pmin;
    float U = (dot + A.c_explore * qn * mt.x) * A.scale;
    if (PRIOR) U += A.lambda[h] * mt.y * erff(((float)i - ((float)pmin + 0.5f) * kS) * A.inv2sigma[h]);
    return U;
}

template <bool PRIOR>
__device__ __forceinline__ float node_U(const Forest &F, size_t lvl_base, int node, const float *q, float qn,
                                        const SearchArgs &A, int h, int i, int *pmin_out, float *dot_out) {
    const size_t ni = lvl_base + node;
    const float4 *mu = reinterpret_cast<const float4 *>(F.mu + ni * kD);
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int e = 0; e < kD / 4; e++) {
        const float4 x = __ldg(mu + e);
        acc[0] = fmaf(q[4 * e], x.x, acc[0]);
        acc[1] = fmaf(q[4 * e + 1], x.y, acc[1]);
        acc[2] = fmaf(q[4 * e + 2], x.z, acc[2]);
        acc[3] = fmaf(q[4 * e + 3], x.w, acc[3]);
    }
    const float dot = (acc[0] + acc[1]) + (acc[2] + acc[3]);
    *dot_out = dot;
    return node_U_dot<PRIOR>(F, lvl_base, node, dot, qn, A, h, i, pmin_out);
}

// beam search on one forest for a prefix of m entries; appends the final leaves to the
// result list (returns the new count)
template <bool PRIOR>
__device__ int search_forest(const Forest &F, SearchSmem &S, int bh, int f, int m, float qn, const SearchArgs &A,
                             int h, int i, int nres, int lane, int ncells, int *dev_flag) {
    if (m <= 0) return nres;
    const int C = F.C;
    // roots: the set bits of m
    int ncand = 0;
    {
        const int k = lane;
        const bool root = k < F.L && ((m >> k) & 1);
        const unsigned bal = __ballot_sync(kFull, root);
        if (root) {
            const int slot = __popc(bal >> (k + 1));      // high bits first
            const int node = (((m >> k) - 1) << (k + 1)) + 1;
            int pm;
            float dt;
            S.U[slot] = node_U<PRIOR>(F, F.lvl(bh, f, k) * 2 * C, node, S.q, qn, A, h, i, &pm, &dt);
            S.dot[slot] = dt;
            S.ref[slot] = (k << 26) | node;
            S.pmin[slot] = pm;
        }
        ncand = __popc(bal);
    }
    __syncwarp();
    for (int guard = 0; guard < 64; guard++) {
        // keep the beam best candidates (a warp-wide bitonic sort of the candidates)
        const int nb = min(ncand, A.beam);
        if (ncand <= 32) beam_cut<1>(S, ncand, nb, lane);
        else if (ncand <= 64) beam_cut<2>(S, ncand, nb, lane);
        else beam_cut<4>(S, ncand, nb, lane);
        __syncwarp();
        // expand every internal node
        int cnt0 = 0, cnt1 = 0;
        bool int0 = false, int1 = false;
        if (lane < nb) {
            const int k = S.bref[lane] >> 26, v = (S.bref[lane] & ((1 << 26) - 1)) & ((2 << k) - 1);
            int0 = v < (1 << k);
            cnt0 = int0 ? 2 : 1;
        }
        if (lane + 32 < nb) {
            const int k = S.bref[lane + 32] >> 26, v = (S.bref[lane + 32] & ((1 << 26) - 1)) & ((2 << k) - 1);
            int1 = v < (1 << k);
            cnt1 = int1 ? 2 : 1;
        }
        if (!__any_sync(kFull, int0 || int1)) {
            for (int j = lane; j < nb; j += 32) {          // all leaves: the result
                const int k = S.bref[j] >> 26, node = S.bref[j] & ((1 << 26) - 1);
                const int blk = node >> (k + 1), v = node & ((2 << k) - 1);
                int cell = F.ord[F.lvl(bh, f, k) * C + ((size_t)blk << k) + (v - (1 << k))];
                if ((unsigned)cell >= (unsigned)ncells) {  // a forest not built from these summaries
                    atomicOr(dev_flag, kFlagCheck);
                    cell = -1;
                }
                S.rcell[nres + j] = cell;
                S.rU[nres + j] = S.bU[j];
            }
            __syncwarp();
            return nres + nb;
        }
        int inc0 = cnt0, inc1 = cnt1;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y0 = __shfl_up_sync(kFull, inc0, o), y1 = __shfl_up_sync(kFull, inc1, o);
            if (lane >= o) { inc0 += y0; inc1 += y1; }
        }
        const int tot0 = __shfl_sync(kFull, inc0, 31), tot1 = __shfl_sync(kFull, inc1, 31);
        const int pos0 = inc0 - cnt0, pos1 = tot0 + inc1 - cnt1;
        for (int half = 0; half < 2; half++) {
            const int j = lane + 32 * half;
            if (j >= nb) continue;
            const int ref = S.bref[j];
            const int k = ref >> 26, node = ref & ((1 << 26) - 1);
            const int v = node & ((2 << k) - 1);
            const int o = half ? pos1 : pos0;
            if (v >= (1 << k)) {                            // a leaf stays
                S.U[o] = S.bU[j];
                S.ref[o] = ref;
                S.pmin[o] = S.bpmin[j];
                S.dot[o] = S.bdot[j];
            } else {
                const size_t base = F.lvl(bh, f, k) * 2 * C;
                const int c0 = node + v, c1 = node + v + 1;  // heap children 2v, 2v + 1
                int p0, p1;
                // left child from its mean; the right child's mean is 2 mu_v - mu_left (both
                // halves hold 2^(depth) leaves), so its dot needs no load of its mean
                float d0;
                S.U[o] = node_U<PRIOR>(F, base, c0, S.q, qn, A, h, i, &p0, &d0);
                S.dot[o] = d0;
                S.ref[o] = (k << 26) | c0;
                S.pmin[o] = p0;
                const float d1 = 2.f * S.bdot[j] - d0;
                S.U[o + 1] = node_U_dot<PRIOR>(F, base, c1, d1, qn, A, h, i, &p1);
                S.dot[o + 1] = d1;
                S.ref[o + 1] = (k << 26) | c1;
                S.pmin[o + 1] = p1;
            }
        }
        ncand = tot0 + tot1;
        __syncwarp();
    }
    return nres;                                           // unreachable: depth < 64
}

template <typename T, bool PRIOR>
__global__ void __launch_bounds__(kSearchWarps * 32) tree_search_kernel(Forest F, const T *__restrict__ Q,
                                                                        SearchArgs A, int32_t *__restrict__ idx,
                                                                        int *dev_flag) {
    __shared__ SearchSmem smem[kSearchWarps];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    SearchSmem &S = smem[warp];
    const int bh = blockIdx.y, h = bh % A.H;
    const int r = blockIdx.x * kSearchWarps + warp;
    if (r >= A.Nq) return;
    const size_t row = (size_t)bh * A.Nq + r;
    int32_t *out = idx + row * A.K;
    if (F.hdr[kHdrMagic] != kTreeMagic || F.hdr[kHdrCap] != F.C || F.hdr[kHdrLevels] != F.L ||
        F.hdr[kHdrBH] != (int)gridDim.y || F.hdr[kHdrCells] != A.cells || F.hdr[kHdrError] != 0) {
        for (int j = lane; j < A.K; j += 32) out[j] = -1;
        if (lane == 0) atomicOr(dev_flag, kFlagCheck);
        return;
    }
    const int i = A.q0 + r;
    const float q0 = to_f<T>(Q[row * kD + 2 * lane]), q1 = to_f<T>(Q[row * kD + 2 * lane + 1]);
    S.q[2 * lane] = q0;
    S.q[2 * lane + 1] = q1;
    const float qn = sqrtf(warp_sum(q0 * q0 + q1 * q1));
    __syncwarp();
    const int n = cand_count(i, A.w, A.cells);
    int nres = search_forest<PRIOR>(F, S, bh, 0, n, qn, A, h, i, 0, lane, n, dev_flag);
    const int n0 = nres;
    if (F.hdr[kHdrTau] && n > 0) {
        const int m = F.admp[(size_t)bh * (F.C + 1) + n];
        nres = search_forest<PRIOR>(F, S, bh, 1, m, qn, A, h, i, nres, lane, n, dev_flag);
    }
    // a cell both beams reached counts once (forest 0's copy)
    for (int j = n0 + lane; j < nres; j += 32) {
        bool dup = false;
        for (int x = 0; x < n0; x++) dup |= S.rcell[x] == S.rcell[j];
        if (dup) S.rcell[j] = -1;
    }
    __syncwarp();
    // the K best by eq. (7) (U desc, cell asc), written in ascending cell order; the
    // candidate arrays are free now: S.ref holds each result's rank
    int nsel = 0;
    for (int j = 0; j < nres; j++) nsel += S.rcell[j] >= 0;
    nsel = min(nsel, A.K);
    for (int j = lane; j < nres; j += 32) {
        const int cj = S.rcell[j];
        int rank = 0x7fffffff;
        if (cj >= 0) {
            const float Uj = S.rU[j];
            rank = 0;
            for (int x = 0; x < nres; x++) rank += S.rcell[x] >= 0 && beats(S.rU[x], S.rcell[x], Uj, cj);
        }
        S.ref[j] = rank;
    }
    __syncwarp();
    for (int j = lane; j < nres; j += 32) {
        const int cj = S.rcell[j];
        if (S.ref[j] >= A.K) continue;
        int pos = 0;
        for (int x = 0; x < nres; x++) pos += S.ref[x] < A.K && S.rcell[x] < cj;
        out[pos] = cj;
    }
    for (int j = nsel + lane; j < A.K; j += 32) out[j] = -1;
}

}  // namespace

size_t forest_bytes(const fs_params *p) { return forest_geom(p->B * p->H, p->Nk / p->s).total; }

// The capacity of a forest buffer of `bytes`: the largest cell count whose layout fits
// (the layout grows strictly with the count), or -1 if not even p's cells fit.
int forest_capacity(const fs_params *p, size_t bytes) {
    const int BH = p->B * p->H, C = p->Nk / p->s;
    const long long kMax = 1 << 26;
    auto fits = [&](long long c) { return forest_geom(BH, (int)c).total <= bytes; };
    if (!fits(C)) return -1;
    long long lo = C, step = C > 0 ? C : 1;       // lo fits; grow until lo + step does not
    while (lo < kMax && fits(std::min(lo + step, kMax))) {
        lo = std::min(lo + step, kMax);
        step *= 2;
    }
    long long hi = std::min(lo + step, kMax);      // lo fits, hi may not
    while (lo < hi) {
        const long long mid = lo + (hi - lo + 1) / 2;
        if (fits(mid)) lo = mid;
        else hi = mid - 1;
    }
    return (int)lo;
}

cudaError_t launch_tree_build(const fs_params *p, const float *kbar, const float *amax, const float *tau,
                              void *forest, size_t bytes, int prev, cudaStream_t st) {
    const int cap = forest_capacity(p, bytes);
    if (cap < 0) return cudaErrorInvalidValue;
    const ForestGeom g = forest_geom(p->B * p->H, cap);
    const Forest F = forest_view(forest, g);
    const int Cn = p->Nk / p->s;
    TauArgs T;
    for (int h = 0; h < FS_MAX_HEADS; h++) T.tau[h] = tau && h < p->H ? tau[h] : 0.f;
    {
        LaunchScope sc(kTreePrep, st);
        tree_prep_kernel<<<g.BH, 1024, 0, st>>>(F, kbar, amax, p->H, tau != nullptr, T, Cn, prev);
        if (cudaGetLastError() != cudaSuccess) return cudaErrorLaunchFailure;
    }
    const int fresh = Cn - prev;                 // cells since the previous build
    for (int k = 0; k < g.L; k++) {
        LaunchScope sc(kTreeMerge, st);
        const int span = fresh + (1 << k);       // entries of the blocks completed since then
        const long long nent = (long long)g.BH * 2 * span;
        tree_merge_kernel<<<(unsigned)((nent + 255) / 256), 256, 0, st>>>(F, g.BH, k, span);
        if (cudaGetLastError() != cudaSuccess) return cudaErrorLaunchFailure;
    }
    for (int k = 0; k < g.L; k++) {
        LaunchScope sc(kTreeNodes, st);
        const int per = (fresh >> k) + 1;        // trees per (bh, f) completed since then, at most
        const int d0 = k > kUpSubK ? k - kUpSubK : 0;
        const long long items = (long long)g.BH * 2 * per << d0;
        const long long blocks = std::min<long long>(kUpMaxBlocks, (items + kUpThreads / 32 - 1) / (kUpThreads / 32));
        tree_up_kernel<<<(unsigned)blocks, kUpThreads, 0, st>>>(F, kbar, amax, g.BH, k, 0, per, Cn);
        if (cudaGetLastError() != cudaSuccess) return cudaErrorLaunchFailure;
        if (d0 > 0) {                           // the top depths of each tree, after its subtrees
            const long long trees = (long long)g.BH * 2 * per;
            const long long tb = std::min<long long>(kUpMaxBlocks, (trees + kUpThreads / 32 - 1) / (kUpThreads / 32));
            tree_up_kernel<<<(unsigned)tb, kUpThreads, 0, st>>>(F, kbar, amax, g.BH, k, 1, per, Cn);
            if (cudaGetLastError() != cudaSuccess) return cudaErrorLaunchFailure;
        }
        if (k > 0) {
            const long long leaves = (long long)g.BH * 2 * ((long long)per << k);
            tree_radius_kernel<<<(unsigned)((leaves + 255) / 256), 256, 0, st>>>(F, kbar, g.BH, k, per, Cn);
            if (cudaGetLastError() != cudaSuccess) return cudaErrorLaunchFailure;
        }
    }
    tree_header_kernel<<<1, 1, 0, st>>>(F, g.BH, tau != nullptr, Cn, prev == 0);
    return cudaGetLastError();
}

cudaError_t launch_tree_search(const fs_params *p, const Dev &D, const void *Q, const void *forest, size_t bytes,
                               int beam, float c_explore, int32_t *idx, int *dev_flag, cudaStream_t st) {
    const int cap = forest_capacity(p, bytes);
    if (cap < 0) return cudaErrorInvalidValue;
    const ForestGeom g = forest_geom(p->B * p->H, cap);
    const Forest F = forest_view(const_cast<void *>(forest), g);
    SearchArgs A;
    A.Nq = p->Nq; A.H = p->H; A.w = p->w; A.K = p->K; A.q0 = p->Nk - p->Nq; A.beam = beam;
    A.cells = p->Nk / p->s;
    A.scale = D.scale;
    A.c_explore = c_explore;
    for (int h = 0; h < FS_MAX_HEADS; h++) {
        A.lambda[h] = D.lambda[h];
        A.inv2sigma[h] = D.inv2sigma[h];
    }
    const dim3 grid((p->Nq + kSearchWarps - 1) / kSearchWarps, g.BH);
    LaunchScope sc(kTreeSearch, st);
    if (p->dtype == FS_BF16) {
        auto kern = D.has_prior ? tree_search_kernel<__nv_bfloat16, true> : tree_search_kernel<__nv_bfloat16, false>;
        kern<<<grid, kSearchWarps * 32, 0, st>>>(F, static_cast<const __nv_bfloat16 *>(Q), A, idx, dev_flag);
    } else {
        auto kern = D.has_prior ? tree_search_kernel<float, true> : tree_search_kernel<float, false>;
        kern<<<grid, kSearchWarps * 32, 0, st>>>(F, static_cast<const float *>(Q), A, idx, dev_flag);
    }
    return cudaGetLastError();
}

}  // namespace fs
