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
// Device error word of the calls on this device: a kernel that gives up a bounded wait or
// finds its inputs inconsistent records it here (0 = none).  Zero when the library's
// module is loaded; sticky until fs_sync_status(NULL, ...) reads and clears it.
static __device__ __align__(256) int fs_noalloc_status_word;

namespace fs {
namespace {

constexpr int kMaxDevices = 128;
std::mutex g_mu;
// Device addresses of the two arrays, per device.  In host code the names above are
// host-side stand-ins, not device addresses, so every kernel gets these instead.
struct Scratch {
    int *table = nullptr;
    int *status = nullptr;
};
Scratch g_scratch[kMaxDevices];

bool stream_capturing(cudaStream_t st) {
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    // a query that fails (e.g. the legacy stream while another stream captures) is taken
    // as "capturing": the cached addresses are used, no symbol is looked up
    if (cudaStreamIsCapturing(st, &cs) != cudaSuccess) return true;
    return cs != cudaStreamCaptureStatusNone;
}

// Set-up with the device current: look up the arrays' device addresses.  Outside stream
// capture this is repeated on every call (a host-side query, not an allocation), so a
// device reset that reloads the library's module cannot leave a stale address behind;
// inside a capture the addresses found by an earlier call on this device are used.
fs_status scratch_for_current_device(cudaStream_t st, Scratch *out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return FS_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_mu);
    Scratch &s = g_scratch[dev];
    if (!s.table || !stream_capturing(st)) {
        void *t = nullptr, *f = nullptr;
        if (cudaGetSymbolAddress(&t, fs_noalloc_exit_table) != cudaSuccess || !t) return FS_ERR_CUDA;
        if (cudaGetSymbolAddress(&f, fs_noalloc_status_word) != cudaSuccess || !f) return FS_ERR_CUDA;
        s.table = static_cast<int *>(t);
        s.status = static_cast<int *>(f);
    }
    *out = s;
    return FS_OK;
}

}  // namespace

// The status word of the no-allocation calls on the current device, read and cleared;
// called by fs_sync_status(NULL, ...) after the stream has drained.  Devices on which no
// such call was made report kFlagOk without touching the GPU.
fs_status noalloc_take_status() {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return FS_ERR_CUDA;
    int *word = nullptr;
    {
        std::lock_guard<std::mutex> lk(g_mu);
        if (!g_scratch[dev].table) return FS_OK;
        void *f = nullptr;
        if (cudaGetSymbolAddress(&f, fs_noalloc_status_word) != cudaSuccess || !f) return FS_ERR_CUDA;
        g_scratch[dev].status = word = static_cast<int *>(f);
    }
    int flag = kFlagOk;
    if (cudaMemcpy(&flag, word, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return FS_ERR_CUDA;
    if (flag == kFlagOk) return FS_OK;
    const int zero = kFlagOk;
    if (cudaMemcpy(word, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess) return FS_ERR_CUDA;
    return flag == kFlagTimeout ? FS_ERR_TIMEOUT : FS_ERR_KERNEL_CHECK;
}

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
    Scratch sc;
    if ((s = scratch_for_current_device(st, &sc)) != FS_OK) return s;
    // every entry of the exit table the selection reads is written by this call's
    // exit-time pass first, so nothing in the shared array needs clearing between calls
    if (prune && launch_exit_times(D, amax, sc.table, st) != cudaSuccess) return FS_ERR_CUDA;
    // same kernels as fs_select_topk; their device error flag is the status word, read by
    // fs_sync_status(NULL, stream)
    return launch_selection(p, D, Q, kbar, amax, sc.table, idx, sc.status, st) == cudaSuccess ? FS_OK
                                                                                             : FS_ERR_CUDA;
}
