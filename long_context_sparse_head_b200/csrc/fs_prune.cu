// FS-L prefix pruning support, "FreeSolo" summary §3.3 eq. (8).
//
// A_i keeps the P candidates of largest a_c among the prefix C_i = cells [0, n).  As n
// grows a cell's rank (how many prefix cells beat it: larger a_c, ties to the lower
// index) never decreases, so each cell c is in TopP(n) exactly for c < n < exit(c), with
//   exit(c) = max(c + 1, 1 + index of the P-th cell (in index order) that beats c),
// or "never" if fewer than P cells beat it.  This kernel tabulates exit(c) once per
// head; the selection kernels then test membership of any prefix in O(1).
//
// One warp per cell scans the head's a values 256 at a time (eight independent coalesced
// loads per lane in flight, L2-resident), counting beating cells with a ballot per
// 32-cell block in index order, and stops at the P-th.  The cells with the largest a scan
// the whole head, so the kernel's time is set by those scans' round trips to L2.
#include "fs_common.cuh"

namespace fs {

namespace {
constexpr int kScanBlocks = 8;                   // 32-cell blocks loaded per round trip
}

__global__ void __launch_bounds__(256) exit_times_kernel(const float *__restrict__ amax,
                                                         int *__restrict__ exitn,
                                                         long long ncell, int C, int P) {
    griddep_wait();
    const long long cell = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (cell >= ncell) return;
    const int lane = threadIdx.x & 31;
    const long long bh = cell / C;
    const int c = (int)(cell - bh * C);
    const float *a = amax + bh * C;
    const float ac = a[c];
    int ex = kNever;
    if (P <= 0) {
        ex = c + 1;
    } else {
        int count = 0;
        bool found = false;
        for (int base = 0; base < C && !found; base += 32 * kScanBlocks) {
            float b[kScanBlocks];
#pragma unroll
            for (int k = 0; k < kScanBlocks; k++) {
                const int cp = base + 32 * k + lane;
                b[k] = cp < C ? __ldg(a + cp) : 0.f;
            }
#pragma unroll
            for (int k = 0; k < kScanBlocks; k++) {
                const int cp = base + 32 * k + lane;
                const bool beats = cp < C && cp != c && ((b[k] > ac) || (b[k] == ac && cp < c));
                unsigned m = __ballot_sync(kFull, beats);
                const int pc = __popc(m);
                if (!found && count + pc >= P) {
                    for (int r = P - count; r > 1; r--) m &= m - 1;   // drop lower set bits
                    const int cP = base + 32 * k + __ffs(m) - 1;      // the P-th beating cell
                    ex = max(c + 1, cP + 1);
                    found = true;
                }
                count += pc;
            }
        }
    }
    if (lane == 0) exitn[cell] = ex;
}

// Exit times for a call whose queries span few prefixes (decode: Nq queries cover about
// Nq / s + 1 prefixes of an archive of C cells).  Only prefixes n in [n_lo, n_hi] are
// ever asked, so the table only has to be right there: TopP(n_lo) comes from a radix
// select over [0, n_lo), and each later prefix n adds the one cell c = n - 1, which
// enters TopP(n) iff it beats the weakest member (larger a; a tie goes to the lower
// index, i.e. to the member), evicting that member at n.  Members get exit = the prefix
// that evicts them (never, if none in range); every other cell gets c + 1, which makes
// c < n < exit(c) false for every n >= n_lo.  One CTA per (b, h).
namespace {
constexpr int kRangeThreads = 1024;
constexpr int kRangeMaxSteps = 128;              // largest n_hi - n_lo this kernel takes
constexpr int kEqCap = 512;                      // cells equal to the threshold ranked directly

// order-preserving integer key of a float (larger float, larger key)
__device__ __forceinline__ uint32_t order_key(float a) {
    const uint32_t b = __float_as_uint(a);
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
}  // namespace

__global__ void __launch_bounds__(kRangeThreads) topp_range_kernel(const float *__restrict__ amax,
                                                                   int *__restrict__ exitn, int C, int P,
                                                                   int n_lo, int n_hi, int *__restrict__ tlist,
                                                                   int tl_words) {
    extern __shared__ uint32_t list[];           // TopP members: keys [P], then cells [P]
    __shared__ int hist[256];
    __shared__ int wsum[kRangeThreads / 32];
    __shared__ uint32_t s_prefix;
    __shared__ int s_remaining, s_count, s_neq;
    __shared__ int eq_list[kEqCap];              // cells whose key equals tau
    uint32_t *lkey = list;
    int *lidx = reinterpret_cast<int *>(list + P);
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    const float *a = amax + (size_t)blockIdx.x * C;
    int *ex = exitn + (size_t)blockIdx.x * C;
    int *tl = tlist ? tlist + (size_t)blockIdx.x * tl_words : nullptr;   // [0] count, then cells
    griddep_wait();
    for (int c = t; c < C; c += kRangeThreads) ex[c] = c + 1;
    const int n0 = min(n_lo, C), m0 = min(P, n0);  // |TopP(n0)| = m0
    if (t == 0) s_count = 0;
    __syncthreads();
    if (m0 > 0) {
        // key tau of the m0-th largest a in [0, n0), and how many cells with key tau
        // belong to TopP (the lowest-indexed ones)
        const bool all = m0 == n0;
        uint32_t tau = 0;
        int remaining = m0;
        if (!all) {
            uint32_t mask = 0;
            for (int shift = 24; shift >= 0; shift -= 8) {
                for (int i = t; i < 256; i += kRangeThreads) hist[i] = 0;
                __syncthreads();
                for (int c = t; c < n0; c += kRangeThreads) {
                    const uint32_t k = order_key(__ldg(a + c));
                    if ((k & mask) == tau) atomicAdd(&hist[(k >> shift) & 255], 1);
                }
                __syncthreads();
                if (warp == 0) {   // lane l holds digits 255 - 8l down to 248 - 8l
                    int h[8], sum = 0;
#pragma unroll
                    for (int j = 0; j < 8; j++) {
                        h[j] = hist[255 - 8 * lane - j];
                        sum += h[j];
                    }
                    int incl = sum;
#pragma unroll
                    for (int o = 1; o < 32; o <<= 1) {
                        const int v = __shfl_up_sync(kFull, incl, o);
                        if (lane >= o) incl += v;
                    }
                    const int excl = incl - sum;
                    if (excl < remaining && remaining <= incl) {
                        int cum = excl, d = 255 - 8 * lane;
#pragma unroll
                        for (int j = 0; j < 8; j++) {
                            if (cum + h[j] >= remaining) {
                                d = 255 - 8 * lane - j;
                                break;
                            }
                            cum += h[j];
                        }
                        s_prefix = tau | ((uint32_t)d << shift);
                        s_remaining = remaining - cum;
                    }
                }
                __syncthreads();
                tau = s_prefix;
                remaining = s_remaining;
                mask |= 255u << shift;
                __syncthreads();
            }
        }
        // members of TopP(n0): every cell whose key beats tau, and the `remaining` lowest-
        // indexed cells whose key equals tau.  One pass lists the equal ones (usually a
        // handful), which are then ranked by index; with very many equal keys they are
        // taken in rounds of kRangeThreads cells in index order instead.
        auto add_member = [&](int c, uint32_t k) {
            const int slot = atomicAdd(&s_count, 1);
            lkey[slot] = k;
            lidx[slot] = c;
            ex[c] = kNever;
            if (tl) tl[1 + slot] = c;
        };
        if (t == 0) s_neq = 0;
        __syncthreads();
        for (int c = t; c < n0; c += kRangeThreads) {
            const uint32_t k = order_key(__ldg(a + c));
            if (all || k > tau) {
                add_member(c, k);
            } else if (k == tau) {
                const int e = atomicAdd(&s_neq, 1);
                if (e < kEqCap) eq_list[e] = c;
            }
        }
        __syncthreads();
        const int neq = s_neq;
        if (neq <= kEqCap) {
            for (int j = t; j < neq; j += kRangeThreads) {
                const int c = eq_list[j];
                int rank = 0;
                for (int x = 0; x < neq; x++) rank += eq_list[x] < c;
                if (rank < remaining) add_member(c, tau);
            }
        } else {
            int eq_before = 0;
            for (int base = 0; base < n0; base += kRangeThreads) {
                const int c = base + t;
                const bool eq = c < n0 && order_key(__ldg(a + c)) == tau;
                const unsigned bal = __ballot_sync(kFull, eq);
                if (lane == 0) wsum[warp] = __popc(bal);
                __syncthreads();
                int before = eq_before + __popc(bal & ((1u << lane) - 1u)), tot = 0;
                for (int w2 = 0; w2 < kRangeThreads / 32; w2++) {
                    if (w2 < warp) before += wsum[w2];
                    tot += wsum[w2];
                }
                if (eq && before < remaining) add_member(c, tau);
                eq_before += tot;
                __syncthreads();
            }
        }
    }
    __syncthreads();
    if (warp == 0) {   // prefixes n0 + 1 .. n_hi, one joining cell each
        int cnt = s_count, nl = s_count;        // members now; cells listed
        for (int n = n0 + 1; n <= n_hi && n <= C; n++) {
            const int c = n - 1;
            const uint32_t kc = order_key(__ldg(a + c));
            if (cnt < P) {                       // fewer than P cells yet: all are members
                if (lane == 0) {
                    lkey[cnt] = kc;
                    lidx[cnt] = c;
                    ex[c] = kNever;
                    if (tl) tl[1 + nl] = c;
                }
                nl++;
                cnt++;
                __syncwarp();
                continue;
            }
            uint32_t wk = 0xffffffffu;           // weakest: smallest key, then highest cell
            int wi = -1, ws = -1;
            for (int j = lane; j < cnt; j += 32) {
                const uint32_t kj = lkey[j];
                const int ij = lidx[j];
                if (kj < wk || (kj == wk && ij > wi)) { wk = kj; wi = ij; ws = j; }
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                const uint32_t k2 = __shfl_xor_sync(kFull, wk, o);
                const int i2 = __shfl_xor_sync(kFull, wi, o), s2 = __shfl_xor_sync(kFull, ws, o);
                if (k2 < wk || (k2 == wk && i2 > wi)) { wk = k2; wi = i2; ws = s2; }
            }
            if (kc > wk && lane == 0) {          // c enters TopP(n), the weakest leaves at n
                ex[wi] = n;
                lkey[ws] = kc;
                lidx[ws] = c;
                ex[c] = kNever;
                if (tl) tl[1 + nl] = c;
            }
            nl += kc > wk;
            __syncwarp();
        }
        if (tl && lane == 0) tl[0] = nl;
    }
}

// TopP(n_min) of each 128-query tile (n_min = the candidate count of its first row): the
// cells c < n_min with exit(c) > n_min, ascending, count first.  With W >= 1 the union of a
// tile's admitted sets is exactly these members below n_min - W followed by the recent
// range [n_min - W, n_max), so the selection builds it without scanning the prefix.  One
// warp per (b, h, tile); eight coalesced exit-time loads per lane in flight.
namespace {
constexpr int kListWarps = 4;
}
__global__ void __launch_bounds__(kListWarps * 32) tile_lists_kernel(const int *__restrict__ exitn, int C, int q0,
                                                                      int w, int ntiles, long long ntot, int P,
                                                                      int *__restrict__ lists, int words) {
    griddep_wait();
    const long long id = (long long)blockIdx.x * kListWarps + (threadIdx.x >> 5);
    if (id >= ntot) return;
    const int lane = threadIdx.x & 31;
    const long long bh = id / ntiles;
    const int t = (int)(id - bh * ntiles);
    const int n = cand_count(q0 + 128 * t, w, C);
    const int *ex = exitn + bh * C;
    int *out = lists + id * words;
    int cnt = 0;
    for (int base = 0; base < n; base += 32 * kScanBlocks) {
        int e[kScanBlocks];
#pragma unroll
        for (int k = 0; k < kScanBlocks; k++) {
            const int c = base + 32 * k + lane;
            e[k] = c < n ? __ldg(ex + c) : 0;
        }
#pragma unroll
        for (int k = 0; k < kScanBlocks; k++) {
            const int c = base + 32 * k + lane;
            const bool in = c < n && e[k] > n;
            const unsigned m = __ballot_sync(kFull, in);
            const int pos = cnt + __popc(m & ((1u << lane) - 1u));
            if (in && pos < P) out[1 + pos] = c;
            cnt += __popc(m);
        }
    }
    if (lane == 0) out[0] = min(cnt, P);
}

int tile_list_words(const Dev &P) {
    if (!P.prune || P.W < 1 || P.Nq <= 0 || exit_list_mode(P) || P.W + P.P + 10 > 128) return 0;
    return 1 + (P.P > 0 ? P.P : 0);
}

cudaError_t launch_tile_lists(const Dev &P, const int *exitn, int *lists, cudaStream_t st) {
    const int words = tile_list_words(P);
    const int ntiles = (P.Nq + 127) / 128;
    const long long ntot = (long long)P.B * P.H * ntiles;
    if (words == 0 || ntot == 0) return cudaSuccess;
    LaunchScope scope(kTileLists, st);
    return launch_pdl(tile_lists_kernel, dim3((unsigned)((ntot + kListWarps - 1) / kListWarps)), dim3(kListWarps * 32),
                      0, st, exitn, P.C, P.q0, P.w, ntiles, ntot, P.P, lists, words);
}

bool exit_list_mode(const Dev &P) {
    if (!(P.P > 0 && P.Nq > 0 && P.B * P.H * P.C > 0)) return false;
    const int n_lo = cand_count(P.q0, P.w, P.C), n_hi = cand_count(P.q0 + P.Nq - 1, P.w, P.C);
    return n_hi - n_lo <= kRangeMaxSteps;
}

int exit_list_words(int P) { return 1 + (P > 0 ? P : 0) + kRangeMaxSteps; }

cudaError_t launch_exit_times(const Dev &P, const float *amax, int *exitn, cudaStream_t st, int *tlist) {
    const long long ncell = (long long)P.B * P.H * P.C;
    if (ncell == 0) return cudaSuccess;
    if (P.P > 0 && P.Nq > 0) {
        const int n_lo = cand_count(P.q0, P.w, P.C), n_hi = cand_count(P.q0 + P.Nq - 1, P.w, P.C);
        if (n_hi - n_lo <= kRangeMaxSteps) {
            LaunchScope scope(kExitTimes, st);
            return launch_pdl(topp_range_kernel, dim3((unsigned)(P.B * P.H)), dim3(kRangeThreads), (size_t)P.P * 8,
                              st, amax, exitn, P.C, P.P, n_lo, n_hi, tlist, exit_list_words(P.P));
        }
    }
    const int warps = 8;
    const long long blocks = (ncell + warps - 1) / warps;
    LaunchScope scope(kExitTimes, st);
    return launch_pdl(exit_times_kernel, dim3((unsigned)blocks), dim3(warps * 32), 0, st, amax, exitn, ncell, P.C, P.P);
}

}  // namespace fs
