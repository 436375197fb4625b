// Shared definitions of the FreeSolo CUDA library (sm_100a).
#pragma once

#include <utility>

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "freesolo.h"

namespace fs {

constexpr int kD = 64;          // head dim supported by the kernels
constexpr int kS = 32;          // cell size supported by the kernels
constexpr int kMaxK = 64;       // largest top-K
constexpr int kMaxAdmit = 2048; // largest W + P
constexpr unsigned kFull = 0xffffffffu;

// Never-leaves sentinel of the TopP exit table.
constexpr int kNever = 0x7fffffff;

// Kernel-side copy of the parameters (passed by value).
struct Dev {
    int B, H, Nq, Nk, C;       // C = floor(Nk / s)
    int w, K, W, P;
    int prune;                 // 0: base FS (A_i = C_i)
    int has_prior;             // lambda given and not all zero
    int q0;                    // position of query row 0 = Nk - Nq
    float scale;               // 1 / sqrt(d)
    float rms_eps;
    float theta[kD / 2];       // RoPE frequencies base^(-2m/d)
    float alpha[FS_MAX_HEADS];
    float lambda[FS_MAX_HEADS];
    float inv2sigma[FS_MAX_HEADS];  // 1 / (2 sigma_h)
};

// Workspace layout (byte offsets from ws; each segment 256-byte aligned).
struct WsLayout {
    size_t flag, exitn, kbar, amax, idx, olr, rope, tiles, rope_abs, krot, tlist, tplist, total;
};

// Per-tile selection record passed from the tensor-core selection kernel to the fused
// attention kernel (128 query rows, union of at most 128 cells), in 32-bit words:
// [0, 512) row masks [128][4] (bit u of a row: union position u selected), [512, 640)
// union cells ascending (0xffffffff past |U|), [640] |U|, [644, 772) per row a float
// softmax reference for the readout in log2 units (an upper bound of every logit of the
// row's selected tokens that lies within 96 of their largest one), or NaN where none was
// found (the readout then tracks a running maximum).  3088 bytes, 16-byte multiple.
constexpr int kTileMaskOff = 0, kTileUlistOff = 512, kTileCountOff = 640, kTileMrefOff = 644,
              kTileRecWords = 772;
// Largest gap (log2 units) between a row's readout reference and its largest selected
// logit: p = 2^(x - ref) then stays a normal float for the row's heaviest tokens.
constexpr float kMrefMaxGap = 96.f;

// Device error flag codes (first int of the workspace).
enum : int { kFlagOk = 0, kFlagTimeout = 1, kFlagCheck = 2 };

// Candidate count |C_i| for key-index position i: cells with (c+1)s <= i - w.
__host__ __device__ inline int cand_count(int i, int w, int C) {
    int lim = i - w;
    if (lim < kS) return 0;
    int n = lim / kS;
    return n < C ? n : C;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(kFull, v, o);
    return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(kFull, v, o));
    return v;
}

// Load VEC consecutive elements (16 bytes) and widen to float.
template <typename T> struct Vec;
template <> struct Vec<float> {
    static constexpr int N = 4;
    __device__ __forceinline__ static void load(const float *p, float *o) {
        float4 v = __ldg(reinterpret_cast<const float4 *>(p));
        o[0] = v.x; o[1] = v.y; o[2] = v.z; o[3] = v.w;
    }
};
template <> struct Vec<__nv_bfloat16> {
    static constexpr int N = 8;
    __device__ __forceinline__ static void load(const __nv_bfloat16 *p, float *o) {
        uint4 v = __ldg(reinterpret_cast<const uint4 *>(p));
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int e = 0; e < 4; e++) {
            o[2 * e] = __uint_as_float(w[e] << 16);
            o[2 * e + 1] = __uint_as_float(w[e] & 0xffff0000u);
        }
    }
};

template <typename T> __device__ __forceinline__ float to_f(T x);
template <> __device__ __forceinline__ float to_f<float>(float x) { return x; }
template <> __device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 x) {
    return __bfloat162float(x);
}

// Two consecutive elements p[0], p[1] as floats (8- or 4-byte load).
template <typename T> __device__ __forceinline__ float2 ld_pair(const T *p);
template <> __device__ __forceinline__ float2 ld_pair<float>(const float *p) {
    return __ldg(reinterpret_cast<const float2 *>(p));
}
template <> __device__ __forceinline__ float2 ld_pair<__nv_bfloat16>(const __nv_bfloat16 *p) {
    return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(p));
}

// Transposed butterfly sum: lane t receives the sum over the warp of v[t] (31 shuffles for
// 32 values per lane; each step keeps the half whose index bit matches the lane's bit).
__device__ __forceinline__ float transpose_sum32(float (&v)[32], int lane) {
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
        const bool up = lane & o;
#pragma unroll
        for (int k = 0; k < o; k++) {
            const float send = up ? v[k] : v[k + o];
            const float keep = up ? v[k + o] : v[k];
            v[k] = keep + __shfl_xor_sync(kFull, send, o);
        }
    }
    return v[0];
}
template <typename T> __device__ __forceinline__ T from_f(float x);
template <> __device__ __forceinline__ float from_f<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

// ---- kernel ids for the diagnostics (fs_kernel_times) ----
enum KernelId : int {
    kSummaries = 0, kExitTimes, kSelect, kReadout, kWindow, kRopeTable, kWindowTc, kAttnTc,
    kSelectTc, kRopeKeys, kCacheAppend, kCacheAttend, kRerank, kIdxTiles, kBwdRotate, kBwdRows,
    kBwdWindowKv, kBwdCells, kBwdReadoutKv, kBwdDalpha, kTreePrep, kTreeMerge, kTreeNodes, kTreeSearch,
    kBwdLrRows, kRerankTc, kReadoutRows, kTileLists, kBwdReadoutTc, kBwdWindowTc, kNumKernels
};

// Brackets one kernel launch: counts it and, when timing is on, records events around it.
// Programmatic dependent launch: a kernel launched this way may be scheduled as soon as
// every CTA of the previous kernel on the stream has exited, so its launch and prologue
// overlap that kernel's completion.  It must execute griddep_wait() (which returns once
// the previous kernel has completed and its writes are visible) before it reads anything
// an earlier kernel wrote or writes anything an earlier kernel reads.  griddep_wait() is a
// no-op in a kernel launched without the attribute.
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                       Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

struct LaunchScope {
    LaunchScope(int id, cudaStream_t st);
    ~LaunchScope();
    int id;
    cudaStream_t st;
    int slot;
};

// ---- argument checks shared by the entry points (defined in fs_api.cu) ----
fs_status validate_params(const fs_params *p);
Dev make_dev_params(const fs_params *p);
bool params_have_long_range(const fs_params *p);

// ---- launchers (one per kernel file) ----
cudaError_t launch_summaries(const Dev &P, fs_dtype dt, const void *K, float *kbar,
                             float *amax, cudaStream_t st);
// exit times; for a call whose queries span few prefixes (decoding) the table is only right
// at the asked prefixes, and with tlist the kernel also lists, per (b, h), the cells that are
// TopP members at one of them: tlist[0] = their count, then the cells (unordered)
bool exit_list_mode(const Dev &P);
int exit_list_words(int P);                      // per (b, h)
cudaError_t launch_exit_times(const Dev &P, const float *amax, int *exitn, cudaStream_t st,
                              int *tlist = nullptr);
// TopP(n_min) of every 128-query tile, from the exit table: per (b, h, tile) tile_list_words
// ints, the count then the member cells ascending.  Used when the call is not decoding-
// shaped, pruning is on with W >= 1 and the tensor-core selection applies (0 words else).
int tile_list_words(const Dev &P);
cudaError_t launch_tile_lists(const Dev &P, const int *exitn, int *lists, cudaStream_t st);
// eq. (12) token-level rerank of the selection (CUDA cores, |A_i| <= 128)
bool rerank_supported(const fs_params *p);
cudaError_t launch_rerank(const Dev &P, fs_dtype dt, const void *Q, const void *K, const float *kbar,
                          const float *amax, const int *exitn, int shortlist, int32_t *idx, cudaStream_t st);
// eq. (12) rerank on the tensor cores (bf16, all of A_i): idx and/or per-tile records
bool rerank_tc_supported(const fs_params *p, int shortlist);
cudaError_t launch_rerank_tc(const Dev &P, const void *Q, const void *K, const float *amax, const int *exitn,
                             int32_t *idx, uint32_t *tiles, int *dev_flag, cudaStream_t st);
// per-tile selection records (the fused kernel's input) from a selection idx
cudaError_t launch_idx_tiles(const Dev &P, const int32_t *idx, uint32_t *tiles, int *dev_flag, cudaStream_t st);
cudaError_t launch_select(const Dev &P, fs_dtype dt, const void *Q, const float *kbar,
                          const float *amax, const int *exitn, int32_t *idx, cudaStream_t st);
cudaError_t launch_readout(const Dev &P, fs_dtype dt, const void *Q, const void *K,
                           const void *V, const int32_t *idx, float *olr, cudaStream_t st);
// the same, one warp per row (for selections that differ across a group's rows)
cudaError_t launch_readout_rows(const Dev &P, fs_dtype dt, const void *Q, const void *K,
                                const void *V, const int32_t *idx, float *olr, cudaStream_t st);
cudaError_t launch_window(const Dev &P, fs_dtype dt, const void *Q, const void *K,
                          const void *V, const float *olr, void *O, cudaStream_t st);
// tensor-core window (bf16): angle tables, then the kernel
int rope_table_rows(int w);
cudaError_t launch_rope_table(int w, float rope_base, float2 *rope_t, float2 *rope_b, cudaStream_t st);
cudaError_t launch_window_tc(const Dev &P, const void *Q, const void *K, const void *V,
                             const float *olr, void *O, const float2 *rope_t, const float2 *rope_b,
                             int *dev_flag, cudaStream_t st);
// absolute-position RoPE tables and the rotated copy of the keys the windows read
int rope_hi_rows(int Nk);
cudaError_t launch_rope_abs_table(int Nk, float rope_base, float2 *lo, float2 *hi, cudaStream_t st);
cudaError_t launch_rope_keys(const Dev &P, const void *K, void *Krot, const float2 *lo, const float2 *hi,
                             cudaStream_t st);
// the RoPE tables and the rotated keys of a call: two launches, or one when few keys rotate
cudaError_t launch_rope(const Dev &P, float rope_base, const void *K, void *Krot, float2 *lo, float2 *hi,
                        cudaStream_t st);
// tensor-core selection (bf16): scores against the bf16x3 split of the mean keys
bool select_tc_supported(const fs_params *p);
// (tlist: the exit-times kernel's member lists, when it wrote them: the union is then built
// from them and the recent cells instead of a scan of the whole exit table)
cudaError_t launch_select_tc(const Dev &P, const void *Q, const float *kbar, const float *amax,
                             const int *exitn, int32_t *idx, uint32_t *tiles, int *dev_flag,
                             cudaStream_t st, const int *tlist = nullptr, const int *tplist = nullptr);
// selection with whichever kernel applies (tensor cores for bf16 when supported)
cudaError_t launch_selection(const fs_params *p, const Dev &D, const void *Q, const float *kbar,
                             const float *amax, const int *exitn, int32_t *idx, int *dev_flag,
                             cudaStream_t st, const int *tplist = nullptr);
// status word of fs_select_topk_noalloc on the current device, read and cleared
fs_status noalloc_take_status();
// FS-B (eqs. (10)-(11)): forest buffer size, build (tau: host [H] or NULL), search
size_t forest_bytes(const fs_params *p);
// a forest buffer's layout is that of its capacity, the largest cell count whose forest fits
// in its bytes (-1: not even p's cells fit); prev: cells already built (0: a full build)
int forest_capacity(const fs_params *p, size_t bytes);
cudaError_t launch_tree_build(const fs_params *p, const float *kbar, const float *amax, const float *tau,
                              void *forest, size_t bytes, int prev, cudaStream_t st);
cudaError_t launch_tree_search(const fs_params *p, const Dev &D, const void *Q, const void *forest, size_t bytes,
                               int beam, float c_explore, int32_t *idx, int *dev_flag, cudaStream_t st);
// fused tensor-core readout + window + combine (bf16, internally selected cells)
bool attn_tc_supported(const fs_params *p);
// decoding shapes (fewer tiles than SMs): the tile's chunks split over nsplit CTAs, one
// thread-block cluster that combines its partial states in shared memory
// backward on the tensor cores (bf16; unions of at most 128 cells per tile): the window's
// part (win: stores dQ; Krot = the rotated keys from rope_first_key on, bf16) or the
// readout's (tiles from idx; adds to dQ; writes dO.y per row to dal); both add to dK, dV
bool bwd_tc_supported(const fs_params *p);
cudaError_t launch_bwd_tc(const fs_params *p, bool win, const void *Q, const void *K, const void *V,
                          const void *Krot, const uint32_t *tiles, const void *dO, float *dQ, float *dK, float *dV,
                          float *dal, const float2 *rope_lo, const float2 *rope_hi, int *dev_flag, cudaStream_t st);
int attn_splits(const fs_params *p);
// amax: the cell summaries' max key norms (the window's fixed reference)
cudaError_t launch_attn_tc(const Dev &P, const void *Q, const void *K, const void *V, const void *Krot,
                           const uint32_t *tiles, void *O, const float2 *rope_lo, const float2 *rope_hi,
                           int *dev_flag, int nsplit, const float *amax, cudaStream_t st);

}  // namespace fs
