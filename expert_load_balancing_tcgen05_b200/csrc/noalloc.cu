// moe_load_stats_noalloc: the load-statistics pipeline with its scratch in a
// fixed device array owned by this library instead of a caller workspace.
//
// For callers that cannot allocate device memory at the point of the call:
// code running under a framework that owns the whole device memory pool,
// real-time or embedded callers whose memory is fixed at start-up, and
// host code (callbacks, plugins) where a cudaMalloc would block or is not
// allowed.  They still pass their inputs and outputs; only the scratch is
// supplied here.
//
// The array is a file-scope __device__ variable: every GPU that loads the
// library holds MOE_NOALLOC_SCRATCH_BYTES of it until the process exits.  In
// host code its name is only a host-side stand-in, so the device address is
// taken with cudaGetSymbolAddress once per device (with that device current)
// and cached for the life of the process (a cudaDeviceReset reloads the
// module at a new address; the cache is not refreshed).  All calls share the
// array and it keeps the last call's contents.  The load-statistics kernel
// leaves its control words (tile ticket, finished-block count, error words,
// call epoch) reset when its last block finishes, but a call must not depend
// on the previous one having ended cleanly, so every call here first clears,
// on its own stream, the control block, look-back flags and per-block count
// words of its layout (about 1.2 MB for the largest workload here).  Two calls whose kernels overlap on the GPU race on the
// array; the caller must serialise them.
#include <mutex>

#include "common.cuh"

namespace moe {
cudaError_t launch_load_stats(const int32_t* idx, int64_t T, int K, int N, const int32_t* replica_slot,
                              int n_slots, int32_t* slot_idx, int32_t* counts, int32_t* offsets, int32_t* rank,
                              const float* scores, int score_fn, moe_stats* stats, void* ws, cudaStream_t st,
                              const int32_t* tile_counts = nullptr);
}

static __device__ __align__(256) unsigned char g_noalloc_scratch[MOE_NOALLOC_SCRATCH_BYTES];

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_dev[kMaxDevices] = {nullptr};

// Device address of the scratch array on the current device (set-up on first use).
cudaError_t scratch_address(void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_mu);
    if (g_scratch_dev[dev] == nullptr) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return e;
        g_scratch_dev[dev] = p;
    }
    *out = g_scratch_dev[dev];
    return cudaSuccess;
}
}  // namespace

extern "C" moe_status moe_load_stats_noalloc(const int32_t* topk_idx, int64_t T, int32_t K, int32_t N,
                                             const int32_t* replica_slot, int32_t n_slots, int32_t* slot_idx,
                                             int32_t* counts, int32_t* offsets, int32_t* rank, const float* scores,
                                             int32_t score_fn, moe_stats* stats, moe_stream_t stream) {
    if (T < 0 || K <= 0 || K > 32 || N <= 0 || n_slots < N || n_slots > moe::MAX_SLOTS) return MOE_ERR_INVALID;
    if (T * (int64_t)K >= ((int64_t)1 << 31)) return MOE_ERR_INVALID;
    if (counts == nullptr || offsets == nullptr) return MOE_ERR_INVALID;
    if (T > 0 && (topk_idx == nullptr || rank == nullptr)) return MOE_ERR_INVALID;
    if (replica_slot == nullptr && n_slots != N) return MOE_ERR_INVALID;
    if (scores != nullptr && (N > moe::MAX_N || (score_fn != MOE_SOFTMAX && score_fn != MOE_SIGMOID)))
        return MOE_ERR_INVALID;
    // the problem must fit the fixed scratch array
    if (moe_workspace_bytes(T, K, N, n_slots) > (size_t)MOE_NOALLOC_SCRATCH_BYTES) return MOE_ERR_UNSUPPORTED;
    void* ws = nullptr;
    if (scratch_address(&ws) != cudaSuccess) return MOE_ERR_CUDA;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    // the control block, the look-back flags and the per-block count words
    // start at zero: the epoch restarts at 0 and no word carries its tag
    // (about 1.2 MB for the largest workload here)
    const moe::WsLayout L = moe::ws_layout(T, K, N, n_slots);
    if (cudaMemsetAsync(static_cast<char*>(ws) + L.ctl, 0, L.hs_partial - L.ctl, st) != cudaSuccess)
        return MOE_ERR_CUDA;
    const cudaError_t e = moe::launch_load_stats(topk_idx, T, K, N, replica_slot, n_slots, slot_idx, counts, offsets,
                                                 rank, scores, score_fn, stats, ws, st);
    return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
