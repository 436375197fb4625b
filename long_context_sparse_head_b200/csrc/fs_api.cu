// C ABI of the FreeSolo forward pass (declared in include/freesolo.h): argument checks,
// workspace layout and the launch sequence
//   summaries (eq. (5)) -> TopP exit table (eq. (8)) -> selection (eq. (7))
//   -> readout (eq. (9)) -> window + combine (eqs. (2)-(4)).
#include <algorithm>
#include <cmath>
#include <cstring>

#include "tc_rope.cuh"

namespace fs {
namespace {

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

size_t esize(fs_dtype t) { return t == FS_BF16 ? 2 : 4; }

fs_status validate(const fs_params *p) {
    if (!p) return FS_ERR_INVALID_ARG;
    if (p->B < 1 || p->H < 1 || p->Nq < 0 || p->Nk < 0 || p->Nq > p->Nk) return FS_ERR_INVALID_ARG;
    if (p->d <= 0 || p->s <= 0 || p->w < 0 || p->K < 0) return FS_ERR_INVALID_ARG;
    if ((p->W < 0) != (p->P < 0)) return FS_ERR_INVALID_ARG;     // both off or both on
    if (p->dtype != FS_BF16 && p->dtype != FS_F32) return FS_ERR_INVALID_ARG;
    if (!p->alpha) return FS_ERR_INVALID_ARG;
    if (!(p->rope_base > 0.f) || !(p->rms_eps >= 0.f)) return FS_ERR_INVALID_ARG;
    if (p->lambda) {
        if (!p->sigma) return FS_ERR_INVALID_ARG;
        for (int h = 0; h < p->H && h < FS_MAX_HEADS; h++)
            if (!(p->lambda[h] >= 0.f) || !(p->sigma[h] > 0.f)) return FS_ERR_INVALID_ARG;
    }
    if (p->d != kD || p->s != kS || p->w % kS != 0) return FS_ERR_UNSUPPORTED;
    if (p->K > kMaxK || p->H > FS_MAX_HEADS) return FS_ERR_UNSUPPORTED;
    if (p->W >= 0 && (long long)p->W + p->P > kMaxAdmit) return FS_ERR_UNSUPPORTED;
    if ((long long)p->B * p->H > 65535 || p->Nk > (1 << 30)) return FS_ERR_UNSUPPORTED;
    return FS_OK;
}

Dev make_dev(const fs_params *p) {
    Dev D;
    std::memset(&D, 0, sizeof(D));
    D.B = p->B; D.H = p->H; D.Nq = p->Nq; D.Nk = p->Nk; D.C = p->Nk / p->s;
    D.w = p->w; D.K = p->K; D.W = p->W; D.P = p->P;
    D.prune = (p->W >= 0);
    D.q0 = p->Nk - p->Nq;
    D.scale = (float)(1.0 / std::sqrt((double)p->d));
    D.rms_eps = p->rms_eps;
    for (int m = 0; m < kD / 2; m++)
        D.theta[m] = (float)std::pow((double)p->rope_base, -2.0 * m / (double)p->d);
    D.has_prior = 0;
    for (int h = 0; h < p->H; h++) {
        D.alpha[h] = p->alpha[h];
        D.lambda[h] = p->lambda ? p->lambda[h] : 0.f;
        D.inv2sigma[h] = p->lambda ? (float)(1.0 / (2.0 * (double)p->sigma[h])) : 0.f;
        if (D.lambda[h] != 0.f) D.has_prior = 1;
    }
    return D;
}

WsLayout layout(const fs_params *p) {
    const size_t BH = (size_t)p->B * p->H, C = (size_t)(p->Nk / p->s);
    WsLayout L;
    size_t off = 0;
    L.flag = off;  off += 256;
    L.exitn = off; off += align256(BH * C * 4);
    L.kbar = off;  off += align256(BH * C * kD * 4);
    L.amax = off;  off += align256(BH * C * 4);
    L.idx = off;   off += align256(BH * (size_t)p->Nq * p->K * 4);
    L.olr = off;   off += align256(BH * (size_t)p->Nq * kD * 4);
    L.rope = off;  off += align256((size_t)(128 + rope_table_rows(p->w)) * 32 * 8);
    L.tiles = off; off += align256(BH * (size_t)((p->Nq + 127) / 128) * kTileRecWords * 4);
    L.rope_abs = off; off += align256((size_t)(kRopeLo + rope_hi_rows(p->Nk)) * 32 * 8);
    const int kr0 = p->Nk - p->Nq - p->w > 0 ? p->Nk - p->Nq - p->w : 0;   // first rotated key
    L.krot = off;  off += align256(BH * (size_t)(p->Nk - kr0) * kD * 2);
    L.tlist = off; off += align256(BH * (size_t)exit_list_words(p->P) * 4);   // TopP member lists (decoding)
    const Dev D = make_dev(p);
    L.tplist = off; off += align256(BH * (size_t)((p->Nq + 127) / 128) * tile_list_words(D) * 4);   // tiles' TopP
    L.total = off;
    return L;
}

template <typename X> X *at(void *ws, size_t off) {
    return reinterpret_cast<X *>(static_cast<uint8_t *>(ws) + off);
}

fs_status cuda_status(cudaError_t e) { return e == cudaSuccess ? FS_OK : FS_ERR_CUDA; }

// Does any query row have a long-range candidate?
bool has_long_range(const fs_params *p) {
    if (p->K == 0 || p->Nq == 0) return false;
    return cand_count(p->Nk - 1, p->w, p->Nk / p->s) > 0;
}

// A second stream forked from `st` for launches independent of the chain on `st`, joined
// back before the first launch that needs them.  The side stream and its two events are
// created once per host thread and device and kept (creating them per call costs more
// host time than a short step runs on the GPU); being per thread, two threads that call
// the library concurrently never share them.  If they cannot be created, the launches go
// to `st` in order.
struct ForkRes {
    cudaStream_t side = nullptr;
    cudaEvent_t fork = nullptr, join = nullptr;
    bool ok = false, tried = false;
};
constexpr int kForkDevices = 64;
thread_local ForkRes tl_fork[kForkDevices];

struct Fork {
    ForkRes *r = nullptr;
    cudaStream_t open(cudaStream_t st) {
        int dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kForkDevices) return st;
        ForkRes &x = tl_fork[dev];
        if (!x.tried) {
            x.tried = true;
            x.ok = cudaStreamCreateWithFlags(&x.side, cudaStreamNonBlocking) == cudaSuccess &&
                   cudaEventCreateWithFlags(&x.fork, cudaEventDisableTiming) == cudaSuccess &&
                   cudaEventCreateWithFlags(&x.join, cudaEventDisableTiming) == cudaSuccess;
        }
        if (!x.ok || cudaEventRecord(x.fork, st) != cudaSuccess || cudaStreamWaitEvent(x.side, x.fork, 0) != cudaSuccess)
            return st;
        r = &x;
        return x.side;
    }
    bool close(cudaStream_t st, cudaStream_t used) {
        if (used == st || !r) return true;
        return cudaEventRecord(r->join, r->side) == cudaSuccess && cudaStreamWaitEvent(st, r->join, 0) == cudaSuccess;
    }
};

// per_row_readout: the caller's idx differs across the rows of a group (FS-B), so the
// readout runs one warp per row instead of staging each group's union of cells.
fs_status run_forward(const fs_params *p, const void *Q, const void *K, const void *V,
                      const float *kbar, const float *amax, const int32_t *idx, void *O,
                      void *ws, cudaStream_t st, bool per_row_readout = false) {
    const Dev D = make_dev(p);
    const WsLayout L = layout(p);
    const float *olr = nullptr;
    const bool fused = has_long_range(p) && !idx && attn_tc_supported(p) && select_tc_supported(p);
    if (fused) {   // bf16: selection, then one tensor-core kernel for readout + window + combine
        // the RoPE tables and the rotated keys depend on K only: they run beside the
        // summaries -> exit times -> selection chain
        Fork fk;
        const cudaStream_t rs = fk.open(st);
        float2 *lo = at<float2>(ws, L.rope_abs), *hi = lo + kRopeLo * 32;
        void *krot = at<void>(ws, L.krot);
        if (launch_rope(D, p->rope_base, K, krot, lo, hi, rs) != cudaSuccess) return FS_ERR_CUDA;
        if (!kbar) {
            float *kb = at<float>(ws, L.kbar), *am = at<float>(ws, L.amax);
            if (launch_summaries(D, p->dtype, K, kb, am, st) != cudaSuccess) return FS_ERR_CUDA;
            kbar = kb;
            amax = am;
        }
        int *exitn = at<int>(ws, L.exitn);
        int *tlist = D.prune && exit_list_mode(D) ? at<int>(ws, L.tlist) : nullptr;
        if (D.prune && launch_exit_times(D, amax, exitn, st, tlist) != cudaSuccess) return FS_ERR_CUDA;
        int *tplist = tile_list_words(D) > 0 ? at<int>(ws, L.tplist) : nullptr;
        if (tplist && launch_tile_lists(D, exitn, tplist, st) != cudaSuccess) return FS_ERR_CUDA;
        uint32_t *tiles = at<uint32_t>(ws, L.tiles);
        if (launch_select_tc(D, Q, kbar, amax, exitn, nullptr, tiles, at<int>(ws, L.flag), st, tlist, tplist) !=
            cudaSuccess)
            return FS_ERR_CUDA;
        if (!fk.close(st, rs)) return FS_ERR_CUDA;
        return cuda_status(launch_attn_tc(D, Q, K, V, krot, tiles, O, lo, hi, at<int>(ws, L.flag),
                                          attn_splits(p), amax, st));
    }
    if (has_long_range(p)) {
        const int32_t *sel = idx;
        if (!sel) {
            if (!kbar) {
                float *kb = at<float>(ws, L.kbar), *am = at<float>(ws, L.amax);
                if (launch_summaries(D, p->dtype, K, kb, am, st) != cudaSuccess) return FS_ERR_CUDA;
                kbar = kb;
                amax = am;
            }
            int *exitn = at<int>(ws, L.exitn);
            if (D.prune && launch_exit_times(D, amax, exitn, st) != cudaSuccess) return FS_ERR_CUDA;
            int32_t *wsidx = at<int32_t>(ws, L.idx);
            if (launch_selection(p, D, Q, kbar, amax, exitn, wsidx, at<int>(ws, L.flag), st) != cudaSuccess)
                return FS_ERR_CUDA;
            sel = wsidx;
        }
        float *o = at<float>(ws, L.olr);
        const cudaError_t e = per_row_readout ? launch_readout_rows(D, p->dtype, Q, K, V, sel, o, st)
                                              : launch_readout(D, p->dtype, Q, K, V, sel, o, st);
        if (e != cudaSuccess) return FS_ERR_CUDA;
        olr = o;
    }
    if (p->dtype == FS_BF16) {
        float2 *rt = at<float2>(ws, L.rope), *rb = rt + 128 * 32;
        if (launch_rope_table(p->w, p->rope_base, rt, rb, st) != cudaSuccess) return FS_ERR_CUDA;
        return cuda_status(launch_window_tc(D, Q, K, V, olr, O, rt, rb, at<int>(ws, L.flag), st));
    }
    return cuda_status(launch_window(D, p->dtype, Q, K, V, olr, O, st));
}

}  // namespace

fs_status validate_params(const fs_params *p) { return validate(p); }

cudaError_t launch_selection(const fs_params *p, const Dev &D, const void *Q, const float *kbar,
                             const float *amax, const int *exitn, int32_t *idx, int *dev_flag,
                             cudaStream_t st, const int *tplist) {
    if (select_tc_supported(p))
        return launch_select_tc(D, Q, kbar, amax, exitn, idx, nullptr, dev_flag, st, nullptr, tplist);
    return launch_select(D, p->dtype, Q, kbar, amax, exitn, idx, st);
}
Dev make_dev_params(const fs_params *p) { return make_dev(p); }
bool params_have_long_range(const fs_params *p) { return has_long_range(p); }

}  // namespace fs

using namespace fs;

extern "C" fs_status fs_workspace_size(const fs_params *p, size_t *bytes) {
    fs_status s = validate(p);
    if (s != FS_OK) return s;
    if (!bytes) return FS_ERR_INVALID_ARG;
    *bytes = layout(p).total;
    return FS_OK;
}

extern "C" fs_status fs_cell_summaries(const fs_params *p, const void *K, float *kbar,
                                       float *amax, void *stream) {
    fs_status s = validate(p);
    if (s != FS_OK) return s;
    if (p->Nk / p->s == 0) return FS_OK;
    if (!K || !kbar || !amax) return FS_ERR_INVALID_ARG;
    return cuda_status(launch_summaries(make_dev(p), p->dtype, K, kbar, amax, (cudaStream_t)stream));
}

extern "C" fs_status fs_select_topk(const fs_params *p, const void *Q, const float *kbar,
                                    const float *amax, int32_t *idx, void *ws, size_t ws_bytes,
                                    void *stream) {
    fs_status s = validate(p);
    if (s != FS_OK) return s;
    if (p->Nq == 0 || p->K == 0) return FS_OK;
    if (!Q || !idx) return FS_ERR_INVALID_ARG;
    const WsLayout L = layout(p);
    if (!ws || ws_bytes < L.total) return FS_ERR_WORKSPACE;
    cudaStream_t st = (cudaStream_t)stream;
    const Dev D = make_dev(p);
    if (D.C == 0 || !has_long_range(p)) {
        return cuda_status(cudaMemsetAsync(idx, 0xff, (size_t)p->B * p->H * p->Nq * p->K * 4, st));
    }
    if (!kbar || !amax) return FS_ERR_INVALID_ARG;
    int *exitn = at<int>(ws, L.exitn);
    if (D.prune && launch_exit_times(D, amax, exitn, st) != cudaSuccess) return FS_ERR_CUDA;
    int *tplist = select_tc_supported(p) && tile_list_words(D) > 0 ? at<int>(ws, L.tplist) : nullptr;
    if (tplist && launch_tile_lists(D, exitn, tplist, st) != cudaSuccess) return FS_ERR_CUDA;
    return cuda_status(launch_selection(p, D, Q, kbar, amax, exitn, idx, at<int>(ws, L.flag), st, tplist));
}

extern "C" fs_status fs_select_topk_rerank(const fs_params *p, const void *Q, const void *K, const float *kbar,
                                           const float *amax, int shortlist, int32_t *idx, void *ws,
                                           size_t ws_bytes, void *stream) {
    fs_status s = validate(p);
    if (s != FS_OK) return s;
    if (shortlist < 0) return FS_ERR_INVALID_ARG;
    if (!rerank_supported(p)) return FS_ERR_UNSUPPORTED;
    if (p->Nq == 0 || p->K == 0) return FS_OK;
    if (!Q || !K || !idx) return FS_ERR_INVALID_ARG;
    const WsLayout L = layout(p);
    if (!ws || ws_bytes < L.total) return FS_ERR_WORKSPACE;
    cudaStream_t st = (cudaStream_t)stream;
    const Dev D = make_dev(p);
    if (D.C == 0 || !has_long_range(p)) {
        return cuda_status(cudaMemsetAsync(idx, 0xff, (size_t)p->B * p->H * p->Nq * p->K * 4, st));
    }
    if (!kbar || !amax) return FS_ERR_INVALID_ARG;
    int *exitn = at<int>(ws, L.exitn);
    if (D.prune && launch_exit_times(D, amax, exitn, st) != cudaSuccess) return FS_ERR_CUDA;
    if (rerank_tc_supported(p, shortlist))        // bf16, all of A_i: the tensor-core kernel
        return cuda_status(launch_rerank_tc(D, Q, K, amax, exitn, idx, nullptr, at<int>(ws, L.flag), st));
    return cuda_status(launch_rerank(D, p->dtype, Q, K, kbar, amax, exitn, shortlist, idx, st));
}

extern "C" fs_status fs_forward_rerank(const fs_params *p, const void *Q, const void *K, const void *V,
                                       const float *kbar, const float *amax, int shortlist, int32_t *idx,
                                       void *O, void *ws, size_t ws_bytes, void *stream) {
    fs_status s = validate(p);
    if (s != FS_OK) return s;
    if (shortlist < 0) return FS_ERR_INVALID_ARG;
    if (!rerank_supported(p)) return FS_ERR_UNSUPPORTED;
    if (p->Nq == 0) return FS_OK;
    if (!Q || !K || !V || !O) return FS_ERR_INVALID_ARG;
    if ((kbar == nullptr) != (amax == nullptr)) return FS_ERR_INVALID_ARG;
    const WsLayout L = layout(p);
    if (!ws || ws_bytes < L.total) return FS_ERR_WORKSPACE;
    cudaStream_t st = (cudaStream_t)stream;
    if (!has_long_range(p)) {                      // window only; no cells to select
        if (idx && p->K > 0 &&
            cudaMemsetAsync(idx, 0xff, (size_t)p->B * p->H * p->Nq * p->K * 4, st) != cudaSuccess)
            return FS_ERR_CUDA;
        return run_forward(p, Q, K, V, nullptr, nullptr, nullptr, O, ws, st);
    }
    const Dev D = make_dev(p);
    if (!kbar) {
        float *kb = at<float>(ws, L.kbar), *am = at<float>(ws, L.amax);
        if (launch_summaries(D, p->dtype, K, kb, am, st) != cudaSuccess) return FS_ERR_CUDA;
        kbar = kb;
        amax = am;
    }
    int *exitn = at<int>(ws, L.exitn);
    if (D.prune && launch_exit_times(D, amax, exitn, st) != cudaSuccess) return FS_ERR_CUDA;
    int32_t *sel = idx ? idx : at<int32_t>(ws, L.idx);
    if (attn_tc_supported(p) && rerank_tc_supported(p, shortlist)) {
        // bf16, all of A_i: the tensor-core rerank writes the fused kernel's tile records
        uint32_t *tiles = at<uint32_t>(ws, L.tiles);
        if (launch_rerank_tc(D, Q, K, amax, exitn, idx, tiles, at<int>(ws, L.flag), st) != cudaSuccess)
            return FS_ERR_CUDA;
        float2 *lo = at<float2>(ws, L.rope_abs), *hi = lo + kRopeLo * 32;
        void *krot = at<void>(ws, L.krot);
        if (launch_rope(D, p->rope_base, K, krot, lo, hi, st) != cudaSuccess) return FS_ERR_CUDA;
        return cuda_status(launch_attn_tc(D, Q, K, V, krot, tiles, O, lo, hi, at<int>(ws, L.flag),
                                          attn_splits(p), amax, st));
    }
    if (launch_rerank(D, p->dtype, Q, K, kbar, amax, exitn, shortlist, sel, st) != cudaSuccess) return FS_ERR_CUDA;
    if (attn_tc_supported(p)) {                    // bf16: the fused tensor-core readout + window
        uint32_t *tiles = at<uint32_t>(ws, L.tiles);
        if (launch_idx_tiles(D, sel, tiles, at<int>(ws, L.flag), st) != cudaSuccess) return FS_ERR_CUDA;
        float2 *lo = at<float2>(ws, L.rope_abs), *hi = lo + kRopeLo * 32;
        void *krot = at<void>(ws, L.krot);
        if (launch_rope(D, p->rope_base, K, krot, lo, hi, st) != cudaSuccess) return FS_ERR_CUDA;
        return cuda_status(launch_attn_tc(D, Q, K, V, krot, tiles, O, lo, hi, at<int>(ws, L.flag),
                                          attn_splits(p), amax, st));
    }
    return run_forward(p, Q, K, V, kbar, amax, sel, O, ws, st);
}

extern "C" fs_status fs_forest_bytes(const fs_params *p, size_t *bytes) {
    fs_status s = validate(p);
    if (s != FS_OK) return s;
    if (!bytes) return FS_ERR_INVALID_ARG;
    *bytes = forest_bytes(p);
    return FS_OK;
}

extern "C" fs_status fs_forest_build(const fs_params *p, const float *kbar, const float *amax, const float *tau,
                                     void *forest, size_t forest_bytes_, void *stream) {
    fs_status s = validate(p);
    if (s != FS_OK) return s;
    if (!forest || forest_bytes_ < forest_bytes(p)) return FS_ERR_WORKSPACE;
    if (p->Nk / p->s > 0 && (!kbar || !amax)) return FS_ERR_INVALID_ARG;
    if (tau)
        for (int h = 0; h < p->H; h++)
            if (std::isnan(tau[h])) return FS_ERR_INVALID_ARG;
    return cuda_status(launch_tree_build(p, kbar, amax, tau, forest, forest_bytes_, 0, (cudaStream_t)stream));
}

extern "C" fs_status fs_forest_append(const fs_params *p, int prev_cells, const float *kbar, const float *amax,
                                      const float *tau, void *forest, size_t forest_bytes_, void *stream) {
    fs_status s = validate(p);
    if (s != FS_OK) return s;
    const int C = p->Nk / p->s;
    if (prev_cells < 0 || prev_cells > C) return FS_ERR_INVALID_ARG;
    if (!forest || forest_bytes_ < forest_bytes(p)) return FS_ERR_WORKSPACE;
    if (C > 0 && (!kbar || !amax)) return FS_ERR_INVALID_ARG;
    if (tau)
        for (int h = 0; h < p->H; h++)
            if (std::isnan(tau[h])) return FS_ERR_INVALID_ARG;
    return cuda_status(launch_tree_build(p, kbar, amax, tau, forest, forest_bytes_, prev_cells, (cudaStream_t)stream));
}

extern "C" fs_status fs_select_topk_tree(const fs_params *p, const void *Q, const void *forest,
                                         size_t forest_bytes_, int beam, float c_explore, int32_t *idx,
                                         void *ws, size_t ws_bytes, void *stream) {
    fs_status s = validate(p);
    if (s != FS_OK) return s;
    if (beam < 1 || beam > FS_TREE_MAX_BEAM || !(c_explore >= 0.f) || std::isinf(c_explore)) return FS_ERR_INVALID_ARG;
    if (p->Nq == 0 || p->K == 0) return FS_OK;
    if (!Q || !idx) return FS_ERR_INVALID_ARG;
    if (!forest || forest_bytes_ < forest_bytes(p)) return FS_ERR_WORKSPACE;
    if (!ws || ws_bytes < layout(p).total) return FS_ERR_WORKSPACE;
    const Dev D = make_dev(p);
    return cuda_status(launch_tree_search(p, D, Q, forest, forest_bytes_, beam, c_explore, idx,
                                          at<int>(ws, layout(p).flag), (cudaStream_t)stream));
}

extern "C" fs_status fs_forward_tree(const fs_params *p, const void *Q, const void *K, const void *V,
                                     const float *tau, int beam, float c_explore, int32_t *idx, void *O,
                                     void *ws, size_t ws_bytes, void *forest, size_t forest_bytes_,
                                     void *stream) {
    fs_status s = validate(p);
    if (s != FS_OK) return s;
    if (beam < 1 || beam > FS_TREE_MAX_BEAM || !(c_explore >= 0.f) || std::isinf(c_explore)) return FS_ERR_INVALID_ARG;
    if (p->Nq == 0) return FS_OK;
    if (!Q || !K || !V || !O) return FS_ERR_INVALID_ARG;
    const WsLayout L = layout(p);
    if (!ws || ws_bytes < L.total) return FS_ERR_WORKSPACE;
    if (!forest || forest_bytes_ < forest_bytes(p)) return FS_ERR_WORKSPACE;
    if (tau)
        for (int h = 0; h < p->H; h++)
            if (std::isnan(tau[h])) return FS_ERR_INVALID_ARG;
    cudaStream_t st = (cudaStream_t)stream;
    if (!has_long_range(p)) {                      // window only; no cells to select
        if (idx && p->K > 0 &&
            cudaMemsetAsync(idx, 0xff, (size_t)p->B * p->H * p->Nq * p->K * 4, st) != cudaSuccess)
            return FS_ERR_CUDA;
        return run_forward(p, Q, K, V, nullptr, nullptr, nullptr, O, ws, st);
    }
    const Dev D = make_dev(p);
    float *kb = at<float>(ws, L.kbar), *am = at<float>(ws, L.amax);
    if (launch_summaries(D, p->dtype, K, kb, am, st) != cudaSuccess) return FS_ERR_CUDA;
    if (launch_tree_build(p, kb, am, tau, forest, forest_bytes_, 0, st) != cudaSuccess) return FS_ERR_CUDA;
    int32_t *sel = idx ? idx : at<int32_t>(ws, L.idx);
    if (launch_tree_search(p, D, Q, forest, forest_bytes_, beam, c_explore, sel, at<int>(ws, L.flag), st) !=
        cudaSuccess)
        return FS_ERR_CUDA;
    // FS-B rows of one query tile pick cells across the whole prefix (their union is not
    // bounded like FS-L's), so the readout gathers per row: the readout kernel on the
    // selection, then the tensor-core window + combine
    return run_forward(p, Q, K, V, kb, am, sel, O, ws, st, true);
}

extern "C" fs_status fs_forward(const fs_params *p, const void *Q, const void *K, const void *V,
                                const float *kbar, const float *amax, const int32_t *idx, void *O,
                                void *ws, size_t ws_bytes, void *stream) {
    fs_status s = validate(p);
    if (s != FS_OK) return s;
    if (p->Nq == 0) return FS_OK;
    if (!Q || !K || !V || !O) return FS_ERR_INVALID_ARG;
    if ((kbar == nullptr) != (amax == nullptr)) return FS_ERR_INVALID_ARG;
    if (!ws || ws_bytes < layout(p).total) return FS_ERR_WORKSPACE;
    return run_forward(p, Q, K, V, kbar, amax, idx, O, ws, (cudaStream_t)stream);
}

namespace {
struct HostScratch { size_t q, k, v, o, ws, total; };
HostScratch host_scratch(const fs_params *p) {
    const size_t e = esize(p->dtype), BH = (size_t)p->B * p->H;
    HostScratch h;
    size_t off = 0;
    h.q = off;  off += align256(BH * p->Nq * kD * e);
    h.k = off;  off += align256(BH * p->Nk * kD * e);
    h.v = off;  off += align256(BH * p->Nk * kD * e);
    h.o = off;  off += align256(BH * p->Nq * kD * e);
    h.ws = off; off += layout(p).total;
    h.total = off;
    return h;
}
}  // namespace

extern "C" fs_status fs_host_scratch_size(const fs_params *p, size_t *bytes) {
    fs_status s = validate(p);
    if (s != FS_OK) return s;
    if (!bytes) return FS_ERR_INVALID_ARG;
    *bytes = host_scratch(p).total;
    return FS_OK;
}

namespace {
// Streams and events of one pipelined host call; released when the call has been enqueued
// (the runtime defers the release until the enqueued work completes).
struct HostPipe {
    cudaStream_t in = nullptr, out = nullptr;
    cudaEvent_t ev[2 * 64 + 2] = {};
    int nev = 0;
    ~HostPipe() {
        for (int i = 0; i < nev; i++) cudaEventDestroy(ev[i]);
        if (in) cudaStreamDestroy(in);
        if (out) cudaStreamDestroy(out);
    }
    cudaEvent_t event() {
        if (nev >= (int)(sizeof(ev) / sizeof(ev[0]))) return nullptr;
        if (cudaEventCreateWithFlags(&ev[nev], cudaEventDisableTiming) != cudaSuccess) return nullptr;
        return ev[nev++];
    }
};
}  // namespace

extern "C" fs_status fs_forward_host(const fs_params *p, const void *hQ, const void *hK,
                                     const void *hV, void *hO, void *dscratch,
                                     size_t scratch_bytes, void *stream) {
    fs_status s = validate(p);
    if (s != FS_OK) return s;
    if (p->Nq == 0) return FS_OK;
    if (!hQ || !hK || !hV || !hO) return FS_ERR_INVALID_ARG;
    const HostScratch h = host_scratch(p);
    if (!dscratch || scratch_bytes < h.total) return FS_ERR_WORKSPACE;
    cudaStream_t st = (cudaStream_t)stream;
    const size_t e = esize(p->dtype);
    uint8_t *dQ = at<uint8_t>(dscratch, h.q), *dK = at<uint8_t>(dscratch, h.k);
    uint8_t *dV = at<uint8_t>(dscratch, h.v), *dO = at<uint8_t>(dscratch, h.o);
    void *ws = at<void>(dscratch, h.ws);
    // Heads are independent, so the call runs as a pipeline over about 16 chunks (heads of
    // one batch entry, or whole batch entries): chunk c's inputs copy in (stream `in`) while
    // chunk c-1 computes (the caller's stream) and chunk c-2's output copies out (stream
    // `out`).  Each direction is one plain async copy per buffer and chunk.  The copy in is
    // the bound; what the pipeline cannot hide is the last chunk's compute and copy out,
    // so more chunks shorten the tail.
    constexpr int kChunks = 16;
    const int per_b = p->B >= kChunks ? 1 : kChunks / p->B;             // chunks per batch entry
    const int hc = (p->H + per_b - 1) / per_b;                          // heads per chunk
    const int bc = p->B >= kChunks ? (p->B + kChunks - 1) / kChunks : 1; // batch entries per chunk
    HostPipe pp;
    if (cudaStreamCreateWithFlags(&pp.in, cudaStreamNonBlocking) != cudaSuccess ||
        cudaStreamCreateWithFlags(&pp.out, cudaStreamNonBlocking) != cudaSuccess)
        return FS_ERR_CUDA;
    cudaEvent_t start = pp.event();
    if (!start || cudaEventRecord(start, st) != cudaSuccess || cudaStreamWaitEvent(pp.in, start, 0) != cudaSuccess)
        return FS_ERR_CUDA;                          // earlier work on `stream` may still use the scratch
    for (int b = 0; b < p->B; b += bc) {
        for (int h0 = 0; h0 < p->H; h0 += hc) {
            const int nb = std::min(bc, p->B - b), nh = std::min(hc, p->H - h0);
            fs_params sub = *p;
            sub.B = nb;
            sub.H = nh;
            sub.alpha = p->alpha + h0;
            sub.lambda = p->lambda ? p->lambda + h0 : nullptr;
            sub.sigma = p->sigma ? p->sigma + h0 : nullptr;
            const size_t hb = (size_t)b * p->H + h0;            // first (b, h) of the chunk
            const size_t qoff = hb * p->Nq * kD * e, koff = hb * p->Nk * kD * e;
            const size_t qbytes = (size_t)nb * nh * p->Nq * kD * e, kbytes = (size_t)nb * nh * p->Nk * kD * e;
            cudaEvent_t in_done = pp.event(), fwd_done = pp.event();
            if (!in_done || !fwd_done) return FS_ERR_CUDA;
            if (cudaMemcpyAsync(dQ + qoff, static_cast<const uint8_t *>(hQ) + qoff, qbytes, cudaMemcpyHostToDevice, pp.in) != cudaSuccess ||
                cudaMemcpyAsync(dK + koff, static_cast<const uint8_t *>(hK) + koff, kbytes, cudaMemcpyHostToDevice, pp.in) != cudaSuccess ||
                cudaMemcpyAsync(dV + koff, static_cast<const uint8_t *>(hV) + koff, kbytes, cudaMemcpyHostToDevice, pp.in) != cudaSuccess ||
                cudaEventRecord(in_done, pp.in) != cudaSuccess || cudaStreamWaitEvent(st, in_done, 0) != cudaSuccess)
                return FS_ERR_CUDA;
            s = run_forward(&sub, dQ + qoff, dK + koff, dV + koff, nullptr, nullptr, nullptr, dO + qoff, ws, st);
            if (s != FS_OK) return s;
            if (cudaEventRecord(fwd_done, st) != cudaSuccess || cudaStreamWaitEvent(pp.out, fwd_done, 0) != cudaSuccess ||
                cudaMemcpyAsync(static_cast<uint8_t *>(hO) + qoff, dO + qoff, qbytes, cudaMemcpyDeviceToHost, pp.out) != cudaSuccess)
                return FS_ERR_CUDA;
        }
    }
    cudaEvent_t all_out = pp.event();                 // the caller's stream joins the copies out
    if (!all_out || cudaEventRecord(all_out, pp.out) != cudaSuccess || cudaStreamWaitEvent(st, all_out, 0) != cudaSuccess)
        return FS_ERR_CUDA;
    return FS_OK;
}

extern "C" fs_status fs_sync_status(void *ws, void *stream) {
    cudaStream_t st = (cudaStream_t)stream;
    if (cudaStreamSynchronize(st) != cudaSuccess) return FS_ERR_CUDA;
    if (!ws) return noalloc_take_status();      // fs_select_topk_noalloc's status word
    int flag = 0;
    if (cudaMemcpy(&flag, ws, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return FS_ERR_CUDA;
    if (flag != kFlagOk) {
        const int zero = 0;
        if (cudaMemcpy(ws, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess) return FS_ERR_CUDA;
        return flag == kFlagTimeout ? FS_ERR_TIMEOUT : FS_ERR_KERNEL_CHECK;
    }
    return FS_OK;
}

extern "C" const char *fs_status_string(fs_status s) {
    switch (s) {
    case FS_OK: return "ok";
    case FS_ERR_INVALID_ARG: return "invalid argument";
    case FS_ERR_UNSUPPORTED: return "unsupported size or option";
    case FS_ERR_WORKSPACE: return "workspace missing or too small";
    case FS_ERR_CUDA: return "CUDA error";
    case FS_ERR_TIMEOUT: return "a kernel gave up a bounded wait";
    case FS_ERR_KERNEL_CHECK: return "a kernel's consistency check failed";
    }
    return "unknown status";
}
