// Launch counting and optional per-kernel device timing (measurement support only).
#include <atomic>
#include <mutex>
#include <vector>

#include "tc_common.cuh"

namespace fs {
namespace {

std::atomic<long long> g_launches{0};
std::atomic<int> g_timing{0};
std::mutex g_mu;

struct Pending { int id; cudaEvent_t a, b; };
std::vector<Pending> g_pending;      // recorded, not yet read
std::vector<cudaEvent_t> g_free;     // reusable events
long long g_count[kNumKernels];
double g_ms[kNumKernels];

cudaEvent_t take_event() {
    if (!g_free.empty()) {
        cudaEvent_t e = g_free.back();
        g_free.pop_back();
        return e;
    }
    cudaEvent_t e = nullptr;
    if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
    return e;
}

const char *const kNames[kNumKernels] = {"cell_summaries", "exit_times", "select_topk",
                                         "readout", "window_combine", "rope_table",
                                         "window_tc", "attn_tc", "select_tc", "rope_keys",
                                         "cache_append", "cache_attend", "rerank", "idx_tiles",
                                         "bwd_rotate", "bwd_win_rows", "bwd_window_kv", "bwd_cells",
                                         "bwd_readout_kv", "bwd_dalpha", "tree_prep", "tree_merge",
                                         "tree_nodes", "tree_search", "bwd_lr_rows", "rerank_tc", "readout_rows",
                                         "tile_lists", "bwd_readout_tc", "bwd_window_tc"};
}  // namespace

LaunchScope::LaunchScope(int id_, cudaStream_t st_) : id(id_), st(st_), slot(-1) {
    g_launches.fetch_add(1, std::memory_order_relaxed);
    if (!g_timing.load(std::memory_order_relaxed)) return;
    std::lock_guard<std::mutex> lk(g_mu);
    Pending p{id, take_event(), take_event()};
    if (!p.a || !p.b) return;
    cudaEventRecord(p.a, st);
    slot = (int)g_pending.size();
    g_pending.push_back(p);
}

LaunchScope::~LaunchScope() {
    if (slot < 0) return;
    std::lock_guard<std::mutex> lk(g_mu);
    if (slot < (int)g_pending.size()) cudaEventRecord(g_pending[slot].b, st);
}

}  // namespace fs

using namespace fs;

namespace fs {
namespace {
// waits (bounded) on a barrier nothing arrives at: the wait runs out and records the timeout
__global__ void selftest_wait_kernel(int *dev_flag) {
    __shared__ uint64_t bar;
    __shared__ int abort_word;
    if (threadIdx.x == 0) {
        abort_word = 0;
        tc::mbar_init(&bar, 1);
        tc::fence_barrier_init();
    }
    __syncthreads();
    const tc::Abort ab{dev_flag, &abort_word};
    if (threadIdx.x == 0) (void)tc::mbar_wait(&bar, 0, ab);
}
}  // namespace
}  // namespace fs

extern "C" fs_status fs_selftest_timeout(void *ws, void *stream) {
    if (!ws) return FS_ERR_INVALID_ARG;
    selftest_wait_kernel<<<1, 32, 0, (cudaStream_t)stream>>>(static_cast<int *>(ws));
    return cudaGetLastError() == cudaSuccess ? FS_OK : FS_ERR_CUDA;
}

extern "C" long long fs_launch_count(void) { return g_launches.load(); }

extern "C" fs_status fs_timing_enable(int on) {
    g_timing.store(on ? 1 : 0);
    return FS_OK;
}

extern "C" int fs_kernel_times(int max_ids, long long *launches, double *ms) {
    std::lock_guard<std::mutex> lk(g_mu);
    for (const Pending &p : g_pending) {
        float t = 0.f;
        if (cudaEventSynchronize(p.b) == cudaSuccess && cudaEventElapsedTime(&t, p.a, p.b) == cudaSuccess) {
            g_count[p.id] += 1;
            g_ms[p.id] += t;
        }
        g_free.push_back(p.a);
        g_free.push_back(p.b);
    }
    g_pending.clear();
    for (int i = 0; i < kNumKernels && i < max_ids; i++) {
        if (launches) launches[i] = g_count[i];
        if (ms) ms[i] = g_ms[i];
        g_count[i] = 0;
        g_ms[i] = 0.0;
    }
    return kNumKernels;
}

extern "C" const char *fs_kernel_name(int id) {
    return (id >= 0 && id < kNumKernels) ? kNames[id] : nullptr;
}
