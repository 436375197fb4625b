// fs_select_topk_noalloc: the long-range cell selection of fs_select_topk for callers
// that cannot allocate device memory.
//
// Some callers have no way to hand this library a workspace: programs that run inside a
// fixed device-memory budget planned before they start, plugins whose host framework owns
// every device allocation, and latency-critical loops where cudaMalloc/cudaFree would
// stall on a device-wide synchronization.  For them the one scratch buffer selection needs
// (the TopP exit table, one int per cell) lives in a fixed-size array compiled into the
// library.  Every GPU that loads the library holds that array until the process exits.
#include <mutex>

#include "fs_common.cuh"

// Scratch for fs_select_topk_noalloc: the TopP exit table of up to FS_NOALLOC_MAX_CELLS
// cells (B * H * floor(Nk / s)), 4 MiB.  Shared by every call on a device.
static __device__ __align__(256) int fs_noalloc_exit_table[FS_NOALLOC_MAX_CELLS];

namespace fs {
namespace {

constexpr int kMaxDevices = 128;
std::mutex g_mu;
int *g_table[kMaxDevices];      // device address of the array, per device (host stand-in
                                // `fs_noalloc_exit_table` is not a device address)

// Set-up, once per device, with that device current: look up the array's device address.
fs_status table_for_current_device(int **out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return FS_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_table[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, fs_noalloc_exit_table) != cudaSuccess || !p) return FS_ERR_CUDA;
        g_table[dev] = static_cast<int *>(p);
    }
    *out = g_table[dev];
    return FS_OK;
}

}  // namespace
}  // namespace fs

using namespace fs;

extern "C" fs_status fs_select_topk_noalloc(const fs_params *p, const void *Q, const float *kbar,
                                            const float *amax, int32_t *idx, void *stream) {
    fs_status s = validate_params(p);
    if (s != FS_OK) return s;
    if (p->Nq == 0 || p->K == 0) return FS_OK;
    if (!Q || !idx) return FS_ERR_INVALID_ARG;
    const Dev D = make_dev_params(p);
    const bool prune = p->W >= 0;
    if (prune && (long long)p->B * p->H * (p->Nk / p->s) > FS_NOALLOC_MAX_CELLS)
        return FS_ERR_UNSUPPORTED;                    // the exit table would not fit
    cudaStream_t st = (cudaStream_t)stream;
    if (D.C == 0 || !params_have_long_range(p))
        return cudaMemsetAsync(idx, 0xff, (size_t)p->B * p->H * p->Nq * p->K * 4, st) == cudaSuccess
                   ? FS_OK : FS_ERR_CUDA;
    if (!kbar || !amax) return FS_ERR_INVALID_ARG;
    int *exitn = nullptr;
    if ((s = table_for_current_device(&exitn)) != FS_OK) return s;
    // every entry the selection reads is written by this call's exit-time pass first, so
    // nothing in the shared array needs clearing between calls
    if (prune && launch_exit_times(D, amax, exitn, st) != cudaSuccess) return FS_ERR_CUDA;
    // same kernels as fs_select_topk; with no workspace there is no device error flag
    return launch_selection(p, D, Q, kbar, amax, exitn, idx, nullptr, st) == cudaSuccess ? FS_OK
                                                                                          : FS_ERR_CUDA;
}
