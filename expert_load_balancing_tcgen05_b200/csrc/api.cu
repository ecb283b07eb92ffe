// C ABI of libmoeroute: argument validation on the host, then stream-ordered
// launches.  No allocation, no synchronisation (except moe_workspace_status).
#include <stddef.h>
#include <stdio.h>
#include <stdlib.h>

#include "common.cuh"

namespace moe {
int route_epl(int N);
bool gate_tc_supported(int N);
bool gate_tc_can_fuse(int N, int K, int fn, int n_groups, int group_topn);
cudaError_t launch_gate_tc(const void* x, const void* W, const float* off, const float* bias, int T, int d, int N,
                           int K, int fn, int n_groups, int topk_groups, int group_topn, int renorm, float scale,
                           bool fused, bool bias_in_logits, float* scores, int32_t* idx, float* w, int32_t* err,
                           int max_ctas, int32_t* tile_counts, cudaStream_t st);
cudaError_t launch_gate_simt(const void* x, const void* W, int dtype, const float* off, const float* logit_bias,
                             int T, int d, int N, int fn, float* scores, cudaStream_t st);
cudaError_t launch_bias_update_ema(const int32_t* counts, int N, int64_t total, float u, float alpha, float* ema,
                                   float* bias, cudaStream_t st);
size_t capacity_workspace_bytes(int64_t T, int K, int N);
cudaError_t launch_route_capacity(const float* scores, const float* bias, int T, int N, int K, int n_groups,
                                  int topk_groups, int group_topn, int renorm, float route_scale, long long C,
                                  int32_t* idx, float* w, long long* info, void* ws, cudaStream_t st);
cudaError_t launch_route_balanced(int64_t T, int K, int N, float scale, int32_t* idx, float* w, cudaStream_t st);
cudaError_t launch_route_topk(const float* scores, const float* bias, int T, int N, int K, int n_groups,
                              int topk_groups, int group_topn, int renorm, float route_scale, int32_t* idx,
                              float* w, cudaStream_t st);
cudaError_t launch_load_stats(const int32_t* idx, int64_t T, int K, int N, const int32_t* replica_slot,
                              int n_slots, int32_t* slot_idx, int32_t* counts, int32_t* offsets, int32_t* rank,
                              const float* scores, int score_fn, moe_stats* stats, void* ws, cudaStream_t st,
                              const int32_t* tile_counts = nullptr);
cudaError_t run_lookback_timeout_probe(void* ws, int32_t* err_out, cudaStream_t st);
cudaError_t launch_replica_plan(const int32_t* counts, int N, int R, int32_t* replica_slot, cudaStream_t st);
cudaError_t launch_bias_update(const int32_t* counts, int N, int64_t total, float u, int mode, float* bias,
                               cudaStream_t st);
cudaError_t launch_dispatch(const void* x, int dtype, int64_t T, int d, int K, const int32_t* slot_idx,
                            const int32_t* offsets, const int32_t* rank, void* rows, uint8_t* rows_fp8,
                            float* scales, int32_t* pos, int32_t* row_src, cudaStream_t st);
cudaError_t launch_combine(const void* y, int dtype, int64_t T, int d, int K, const int32_t* pos,
                           const float* w, void* out, cudaStream_t st);
}  // namespace moe

namespace moe_host {
static thread_local int64_t g_launches = 0;
void note_launch(int n) { g_launches += n; }

int sm_count() {
    static int cache[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    if (cache[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
        cache[dev] = n;
    }
    return cache[dev];
}
}  // namespace moe_host

using namespace moe;

static inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Whether the GEMM epilogue selects (instead of a separate selection kernel).
// The epilogue's selection is serial per token row; it pays off only when it
// overlaps the next tile's main loop, i.e. when every CTA runs several tiles.
// MOE_FUSED_SELECT=0/1 forces either path (tuning and tests).
static bool use_fused_select(int T) {
    const char* e = getenv("MOE_FUSED_SELECT");
    if (e != nullptr && e[0] == '0') return false;
    if (e != nullptr && e[0] == '1') return true;
    const int tiles = (T + 127) / 128;
    return tiles >= 3 * moe_host::sm_count();
}
static inline moe_status cuda_status(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

static moe_status check_route_cfg(const moe_route_cfg* c) {
    if (c == nullptr) return MOE_ERR_INVALID;
    if (c->T < 0 || c->N <= 0 || c->K <= 0 || c->K > c->N || c->K > 32) return MOE_ERR_INVALID;
    if (c->score_fn != MOE_SOFTMAX && c->score_fn != MOE_SIGMOID) return MOE_ERR_INVALID;
    if (c->bias_mode != 0 && c->bias_mode != 1) return MOE_ERR_INVALID;
    if (c->gate_max_ctas < 0) return MOE_ERR_INVALID;
    if (c->n_groups <= 0 || c->N % c->n_groups != 0 || c->n_groups > 32) return MOE_ERR_INVALID;
    const int gsize = c->N / c->n_groups;
    if (c->n_groups > 1) {
        if (c->topk_groups <= 0 || c->topk_groups > c->n_groups) return MOE_ERR_INVALID;
        if ((int64_t)c->topk_groups * gsize < c->K) return MOE_ERR_INVALID;
        if (c->group_topn <= 0 || c->group_topn > gsize) return MOE_ERR_INVALID;
    }
    if ((int64_t)c->T * c->K >= (int64_t)1 << 31) return MOE_ERR_INVALID;
    const int epl = route_epl(c->N);
    if (epl == 0) return MOE_ERR_UNSUPPORTED;
    if (c->n_groups > 1) {
        if (gsize % epl != 0) return MOE_ERR_UNSUPPORTED;
        const int lpg = gsize / epl;
        if (lpg & (lpg - 1)) return MOE_ERR_UNSUPPORTED;
    }
    return MOE_OK;
}

extern "C" {

size_t moe_workspace_bytes(int64_t T, int32_t K, int32_t N, int32_t n_slots) {
    if (T < 0 || K <= 0 || N <= 0 || n_slots < N) return 0;
    return ws_layout(T, K, N, n_slots).total;
}

moe_status moe_route(const moe_route_cfg* cfg, const void* x, const void* w_gate, const float* logit_offset,
                     const float* bias, float* scores, int32_t* topk_idx, float* topk_w, void* ws,
                     size_t ws_bytes, moe_stream_t stream) {
    moe_status s = check_route_cfg(cfg);
    if (s != MOE_OK) return s;
    const moe_route_cfg& c = *cfg;
    if (topk_idx == nullptr || topk_w == nullptr) return MOE_ERR_INVALID;
    if (scores != nullptr && !aligned16(scores)) return MOE_ERR_INVALID;
    const int eff_topk_groups = c.n_groups > 1 ? c.topk_groups : 1;
    const bool bias_in_logits = c.bias_mode == 1;
    if (bias_in_logits && x == nullptr) return MOE_ERR_INVALID;  // the bias needs the logits
    const float* sel_bias = bias_in_logits ? nullptr : bias;
    const bool tensor_core = x != nullptr && c.in_dtype == MOE_BF16 && gate_tc_supported(c.N);
    const bool fused = tensor_core && gate_tc_can_fuse(c.N, c.K, c.score_fn, c.n_groups, c.group_topn) &&
                       (scores == nullptr || use_fused_select(c.T));
    if (scores == nullptr && !fused) return MOE_ERR_INVALID;  // the scores carry the selection's input
    if (c.T == 0) return MOE_OK;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (x != nullptr) {
        if (w_gate == nullptr || ws == nullptr || !aligned16(ws)) return MOE_ERR_INVALID;
        if (c.d <= 0 || c.N > MAX_N) return MOE_ERR_INVALID;
        if (ws_bytes < moe_workspace_bytes(c.T, c.K, c.N, c.N)) return MOE_ERR_INVALID;
        if (c.in_dtype != MOE_F32 && c.in_dtype != MOE_BF16) return MOE_ERR_INVALID;
        WsHeader* hdr = reinterpret_cast<WsHeader*>(static_cast<char*>(ws) + ws_layout(c.T, c.K, c.N, c.N).header);
        cudaError_t e;
        if (tensor_core) {
            if (c.d % 8 != 0 || !aligned16(x) || !aligned16(w_gate)) return MOE_ERR_INVALID;
            e = launch_gate_tc(x, w_gate, logit_offset, bias, c.T, c.d, c.N, c.K, c.score_fn, c.n_groups,
                               eff_topk_groups, c.group_topn, c.renorm ? 1 : 0, c.route_scale, fused,
                               bias_in_logits, scores, topk_idx, topk_w, &hdr->gate_err, c.gate_max_ctas, nullptr,
                               st);
            if (e != cudaSuccess) return MOE_ERR_CUDA;
            if (fused) return MOE_OK;
        } else {
            e = launch_gate_simt(x, w_gate, c.in_dtype, logit_offset, bias_in_logits ? bias : nullptr, c.T, c.d, c.N,
                                 c.score_fn, scores, st);
        }
        if (e != cudaSuccess) return MOE_ERR_CUDA;
    }
    return cuda_status(launch_route_topk(scores, sel_bias, c.T, c.N, c.K, c.n_groups, eff_topk_groups,
                                         c.group_topn, c.renorm ? 1 : 0, c.route_scale, topk_idx, topk_w, st));
}

moe_status moe_route_tiles(const moe_route_cfg* cfg, const void* x, const void* w_gate, const float* logit_offset,
                           const float* bias, int32_t* topk_idx, float* topk_w, int32_t* tile_counts, void* ws,
                           size_t ws_bytes, moe_stream_t stream) {
    moe_status s = check_route_cfg(cfg);
    if (s != MOE_OK) return s;
    const moe_route_cfg& c = *cfg;
    if (x == nullptr || w_gate == nullptr || ws == nullptr || !aligned16(ws)) return MOE_ERR_INVALID;
    if (c.T > 0 && (topk_idx == nullptr || topk_w == nullptr || tile_counts == nullptr)) return MOE_ERR_INVALID;
    if (c.d <= 0 || c.in_dtype != MOE_BF16) return c.in_dtype == MOE_F32 ? MOE_ERR_UNSUPPORTED : MOE_ERR_INVALID;
    if (!gate_tc_supported(c.N) || !gate_tc_can_fuse(c.N, c.K, c.score_fn, c.n_groups, c.group_topn))
        return MOE_ERR_UNSUPPORTED;
    if (c.d % 8 != 0 || !aligned16(x) || !aligned16(w_gate)) return MOE_ERR_INVALID;
    if (ws_bytes < moe_workspace_bytes(c.T, c.K, c.N, c.N)) return MOE_ERR_INVALID;
    if (c.T == 0) return MOE_OK;
    WsHeader* hdr = reinterpret_cast<WsHeader*>(static_cast<char*>(ws) + ws_layout(c.T, c.K, c.N, c.N).header);
    const int eff_topk_groups = c.n_groups > 1 ? c.topk_groups : 1;
    return cuda_status(launch_gate_tc(x, w_gate, logit_offset, bias, c.T, c.d, c.N, c.K, c.score_fn, c.n_groups,
                                      eff_topk_groups, c.group_topn, c.renorm ? 1 : 0, c.route_scale, /*fused=*/true,
                                      c.bias_mode == 1, nullptr, topk_idx, topk_w, &hdr->gate_err, c.gate_max_ctas,
                                      tile_counts, reinterpret_cast<cudaStream_t>(stream)));
}

moe_status moe_load_stats(const int32_t* topk_idx, int64_t T, int32_t K, int32_t N, const int32_t* replica_slot,
                          int32_t n_slots, int32_t* slot_idx, int32_t* counts, int32_t* offsets, int32_t* rank,
                          const float* scores, int32_t score_fn, moe_stats* stats, void* ws, size_t ws_bytes,
                          moe_stream_t stream) {
    if (T < 0 || K <= 0 || K > 32 || N <= 0 || n_slots < N || n_slots > MAX_SLOTS) return MOE_ERR_INVALID;
    if (T * (int64_t)K >= ((int64_t)1 << 31)) return MOE_ERR_INVALID;
    if (counts == nullptr || offsets == nullptr || ws == nullptr || !aligned16(ws)) return MOE_ERR_INVALID;
    if (T > 0 && (topk_idx == nullptr || rank == nullptr)) return MOE_ERR_INVALID;  // empty batch: may be NULL
    if (replica_slot == nullptr && n_slots != N) return MOE_ERR_INVALID;
    if (scores != nullptr && (N > MAX_N || (score_fn != MOE_SOFTMAX && score_fn != MOE_SIGMOID)))
        return MOE_ERR_INVALID;
    if (ws_bytes < moe_workspace_bytes(T, K, N, n_slots)) return MOE_ERR_INVALID;
    return cuda_status(launch_load_stats(topk_idx, T, K, N, replica_slot, n_slots, slot_idx, counts, offsets, rank,
                                         scores, score_fn, stats, ws, reinterpret_cast<cudaStream_t>(stream)));
}

moe_status moe_load_stats_tiles(const int32_t* topk_idx, int64_t T, int32_t K, int32_t N,
                                const int32_t* tile_counts, const int32_t* replica_slot, int32_t n_slots,
                                int32_t* slot_idx, int32_t* counts, int32_t* offsets, int32_t* rank, moe_stats* stats,
                                void* ws, size_t ws_bytes, moe_stream_t stream) {
    if (T < 0 || K <= 0 || K > 32 || N <= 0 || n_slots < N || n_slots > MAX_SLOTS) return MOE_ERR_INVALID;
    if (T * (int64_t)K >= ((int64_t)1 << 31)) return MOE_ERR_INVALID;
    if (counts == nullptr || offsets == nullptr || ws == nullptr || !aligned16(ws)) return MOE_ERR_INVALID;
    if (T > 0 && (topk_idx == nullptr || rank == nullptr || tile_counts == nullptr)) return MOE_ERR_INVALID;
    if (replica_slot == nullptr && n_slots != N) return MOE_ERR_INVALID;
    if (ws_bytes < moe_workspace_bytes(T, K, N, n_slots)) return MOE_ERR_INVALID;
    return cuda_status(launch_load_stats(topk_idx, T, K, N, replica_slot, n_slots, slot_idx, counts, offsets, rank,
                                         nullptr, MOE_SIGMOID, stats, ws, reinterpret_cast<cudaStream_t>(stream),
                                         tile_counts));
}

size_t moe_capacity_workspace_bytes(int64_t T, int32_t K, int32_t N) {
    if (T < 0 || K <= 0 || N <= 0) return 0;
    return capacity_workspace_bytes(T, K, N);
}

// ceil(1.25 * T*K/N) = ceil(5*T*K / (4*N)), exact in integers (T*K < 2^31
// for every routed problem, so 5*T*K fits easily in 64 bits)
int64_t moe_capacity_limit(int64_t T, int32_t K, int32_t N) {
    if (T < 0 || K <= 0 || N <= 0) return -1;
    const int64_t num = 5 * T * (int64_t)K, den = 4 * (int64_t)N;
    return (num + den - 1) / den;
}

moe_status moe_route_capacity(const moe_route_cfg* cfg, const float* scores, const float* bias, int64_t capacity,
                              int32_t* topk_idx, float* topk_w, moe_capacity_info* info, void* ws,
                              size_t ws_bytes, moe_stream_t stream) {
    moe_status s = check_route_cfg(cfg);
    if (s != MOE_OK) return s;
    const moe_route_cfg& c = *cfg;
    if (c.K > 16) return MOE_ERR_INVALID;
    if (capacity < 0) capacity = moe_capacity_limit(c.T, c.K, c.N);  // the page's 1.25 factor
    if (c.T > 0 && (scores == nullptr || topk_idx == nullptr || topk_w == nullptr)) return MOE_ERR_INVALID;
    if (scores != nullptr && !aligned16(scores)) return MOE_ERR_INVALID;
    if (ws == nullptr || !aligned16(ws) || ws_bytes < moe_capacity_workspace_bytes(c.T, c.K, c.N)) return MOE_ERR_INVALID;
    // the counters are always written: to info, or else to the workspace header
    static_assert(sizeof(moe_capacity_info) == 4 * sizeof(long long), "info layout");
    long long* inf = info != nullptr ? reinterpret_cast<long long*>(info)
                                     : reinterpret_cast<WsHeader*>(static_cast<char*>(ws) +
                                                                   ws_layout(c.T, c.K, c.N, c.N).header)->cap_info;
    const int eff_topk_groups = c.n_groups > 1 ? c.topk_groups : 1;
    return cuda_status(launch_route_capacity(scores, c.bias_mode == 1 ? nullptr : bias, (int)c.T, c.N, c.K,
                                             c.n_groups, eff_topk_groups, c.group_topn, c.renorm ? 1 : 0,
                                             c.route_scale, capacity, topk_idx, topk_w, inf, ws,
                                             reinterpret_cast<cudaStream_t>(stream)));
}

moe_status moe_route_balanced(int64_t T, int32_t K, int32_t N, float route_scale, int32_t* topk_idx,
                              float* topk_w, moe_stream_t stream) {
    if (T < 0 || K <= 0 || N <= 0 || K > N || T * (int64_t)K >= ((int64_t)1 << 31)) return MOE_ERR_INVALID;
    if (T > 0 && (topk_idx == nullptr || topk_w == nullptr)) return MOE_ERR_INVALID;
    if (T == 0) return MOE_OK;
    return cuda_status(launch_route_balanced(T, K, N, route_scale, topk_idx, topk_w,
                                             reinterpret_cast<cudaStream_t>(stream)));
}

moe_status moe_bias_update_ema(const int32_t* counts, int32_t N, int64_t total_assignments, float u, float alpha,
                               float* load_ema, float* bias, moe_stream_t stream) {
    if (counts == nullptr || load_ema == nullptr || bias == nullptr || N <= 0 || total_assignments <= 0 ||
        !(alpha >= 0.f && alpha < 1.f))
        return MOE_ERR_INVALID;
    return cuda_status(launch_bias_update_ema(counts, N, total_assignments, u, alpha, load_ema, bias,
                                              reinterpret_cast<cudaStream_t>(stream)));
}

moe_status moe_replica_plan(const int32_t* counts, int32_t N, int32_t n_replicas, int32_t* replica_slot,
                            moe_stream_t stream) {
    if (counts == nullptr || replica_slot == nullptr || N <= 0 || N > 12 * 1024 || n_replicas < 0 ||
        n_replicas > N)
        return MOE_ERR_INVALID;
    return cuda_status(launch_replica_plan(counts, N, n_replicas, replica_slot, reinterpret_cast<cudaStream_t>(stream)));
}

moe_status moe_bias_update(const int32_t* counts, int32_t N, int64_t total_assignments, float u, int32_t mode,
                           float* bias, moe_stream_t stream) {
    if (counts == nullptr || bias == nullptr || N <= 0 || total_assignments <= 0 || (mode != 0 && mode != 1))
        return MOE_ERR_INVALID;
    return cuda_status(
        launch_bias_update(counts, N, total_assignments, u, mode, bias, reinterpret_cast<cudaStream_t>(stream)));
}

moe_status moe_dispatch(const void* x, int32_t x_dtype, int64_t T, int32_t d, int32_t K, const int32_t* slot_idx,
                        const int32_t* offsets, const int32_t* rank, void* rows, uint8_t* rows_fp8, float* scales,
                        int32_t* pos, int32_t* row_src, moe_stream_t stream) {
    if (T < 0 || d <= 0 || K <= 0 || K > 32) return MOE_ERR_INVALID;
    if (T * (int64_t)K >= ((int64_t)1 << 31)) return MOE_ERR_INVALID;
    if (x_dtype != MOE_BF16 && x_dtype != MOE_F32) return MOE_ERR_INVALID;
    const int epv = x_dtype == MOE_BF16 ? 8 : 4;
    if (d % epv != 0) return MOE_ERR_INVALID;
    if (T == 0) return MOE_OK;  // empty batch: nothing is read or written, buffers may be NULL
    if (x == nullptr || slot_idx == nullptr || offsets == nullptr || rank == nullptr) return MOE_ERR_INVALID;
    if ((rows_fp8 == nullptr) != (scales == nullptr)) return MOE_ERR_INVALID;
    if (rows_fp8 != nullptr && (d % 128 != 0 || (reinterpret_cast<uintptr_t>(rows_fp8) & 7u) ||
                                (reinterpret_cast<uintptr_t>(scales) & 3u)))
        return MOE_ERR_INVALID;
    if (!aligned16(x) || (rows != nullptr && !aligned16(rows))) return MOE_ERR_INVALID;
    return cuda_status(launch_dispatch(x, x_dtype, T, d, K, slot_idx, offsets, rank, rows, rows_fp8, scales, pos,
                                       row_src, reinterpret_cast<cudaStream_t>(stream)));
}

moe_status moe_combine(const void* y, int32_t dtype, int64_t T, int32_t d, int32_t K, const int32_t* pos,
                       const float* w, void* out, moe_stream_t stream) {
    if (T < 0 || d <= 0 || K <= 0 || K > 32) return MOE_ERR_INVALID;
    if (T * (int64_t)K >= ((int64_t)1 << 31)) return MOE_ERR_INVALID;
    if (dtype != MOE_BF16 && dtype != MOE_F32) return MOE_ERR_INVALID;
    const int epv = dtype == MOE_BF16 ? 8 : 4;
    if (d % epv != 0) return MOE_ERR_INVALID;
    if (T == 0) return MOE_OK;  // empty batch: buffers may be NULL
    if (y == nullptr || pos == nullptr || w == nullptr || out == nullptr) return MOE_ERR_INVALID;
    if (!aligned16(y) || !aligned16(out)) return MOE_ERR_INVALID;
    return cuda_status(launch_combine(y, dtype, T, d, K, pos, w, out, reinterpret_cast<cudaStream_t>(stream)));
}

moe_status moe_workspace_status(void* ws, moe_stream_t stream) {
    if (ws == nullptr || !aligned16(ws)) return MOE_ERR_INVALID;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    struct {
        WsHeader h;
        ScanCtl c;
    } w;
    static_assert(sizeof(w) == sizeof(WsHeader) + sizeof(ScanCtl), "header and control are adjacent");
    if (cudaMemcpyAsync(&w, ws, sizeof(w), cudaMemcpyDeviceToHost, st) != cudaSuccess) return MOE_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return MOE_ERR_CUDA;
    const int32_t scan = w.c.sticky | w.c.err;
    moe_status r = MOE_OK;
    if ((w.h.gate_err & 1) || (scan & 1)) r = MOE_ERR_TIMEOUT;
    else if (scan & 6) r = MOE_ERR_INVALID;  // an expert id out of range, or overlapping calls on one workspace
    if (w.h.gate_err || w.c.sticky) {
        const int32_t z = 0;
        char* base = static_cast<char*>(ws);
        if (cudaMemcpyAsync(base + offsetof(WsHeader, gate_err), &z, sizeof(z), cudaMemcpyHostToDevice, st) !=
                cudaSuccess ||
            cudaMemcpyAsync(base + sizeof(WsHeader) + offsetof(ScanCtl, sticky), &z, sizeof(z),
                            cudaMemcpyHostToDevice, st) != cudaSuccess)
            return MOE_ERR_CUDA;
        if (cudaStreamSynchronize(st) != cudaSuccess) return MOE_ERR_CUDA;
    }
    return r;
}

moe_status moe_selftest_wait_timeout(void* ws, size_t ws_bytes, moe_stream_t stream) {
    if (ws == nullptr || !aligned16(ws) || ws_bytes < moe_workspace_bytes(2 * LS_BLOCK, 1, 8, 8)) return MOE_ERR_INVALID;
    int32_t err = 0;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (run_lookback_timeout_probe(ws, &err, st) != cudaSuccess) return MOE_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return MOE_ERR_CUDA;
    return (err & 1) ? MOE_ERR_TIMEOUT : MOE_OK;
}

int64_t moe_launch_count(int32_t reset) {
    const int64_t v = moe_host::g_launches;
    if (reset) moe_host::g_launches = 0;
    return v;
}

const char* moe_status_str(moe_status s) {
    switch (s) {
        case MOE_OK: return "ok";
        case MOE_ERR_INVALID: return "invalid argument";
        case MOE_ERR_UNSUPPORTED: return "unsupported shape or dtype";
        case MOE_ERR_CUDA: return "CUDA error";
        case MOE_ERR_TIMEOUT: return "bounded device wait timed out";
    }
    return "unknown status";
}

const char* moe_version(void) { return "moeroute 0.1 sm_100a"; }

}  // extern "C"
