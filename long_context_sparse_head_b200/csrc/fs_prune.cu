// FS-L prefix pruning support, "FreeSolo" summary §3.3 eq. (8).
//
// A_i keeps the P candidates of largest a_c among the prefix C_i = cells [0, n).  As n
// grows a cell's rank (how many prefix cells beat it: larger a_c, ties to the lower
// index) never decreases, so each cell c is in TopP(n) exactly for c < n < exit(c), with
//   exit(c) = max(c + 1, 1 + index of the P-th cell (in index order) that beats c),
// or "never" if fewer than P cells beat it.  This kernel tabulates exit(c) once per
// head; the selection kernels then test membership of any prefix in O(1).
//
// One warp per cell scans the head's a values 32 at a time (coalesced, L2-resident),
// counting beating cells with a ballot, and stops at the P-th.
#include "fs_common.cuh"

namespace fs {

__global__ void __launch_bounds__(256) exit_times_kernel(const float *__restrict__ amax,
                                                         int *__restrict__ exitn,
                                                         long long ncell, int C, int P) {
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
        for (int base = 0; base < C; base += 32) {
            const int cp = base + lane;
            bool beats = false;
            if (cp < C && cp != c) {
                const float b = a[cp];
                beats = (b > ac) || (b == ac && cp < c);
            }
            unsigned m = __ballot_sync(kFull, beats);
            const int pc = __popc(m);
            if (count + pc >= P) {
                for (int k = P - count; k > 1; k--) m &= m - 1;   // drop lower set bits
                const int cP = base + __ffs(m) - 1;                 // the P-th beating cell
                ex = max(c + 1, cP + 1);
                break;
            }
            count += pc;
        }
    }
    if (lane == 0) exitn[cell] = ex;
}

cudaError_t launch_exit_times(const Dev &P, const float *amax, int *exitn, cudaStream_t st) {
    const long long ncell = (long long)P.B * P.H * P.C;
    if (ncell == 0) return cudaSuccess;
    const int warps = 8;
    const long long blocks = (ncell + warps - 1) / warps;
    LaunchScope scope(kExitTimes, st);
    exit_times_kernel<<<(unsigned)blocks, warps * 32, 0, st>>>(amax, exitn, ncell, P.C, P.P);
    return cudaGetLastError();
}

}  // namespace fs
