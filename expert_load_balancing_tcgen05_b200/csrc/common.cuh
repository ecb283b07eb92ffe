// Shared device/host helpers of libmoeroute (sm_100a only).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/moe_route.h"

#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ < 1000)
#error "libmoeroute targets sm_100a (B200) only"
#endif

namespace moe {

constexpr unsigned FULL = 0xffffffffu;

// ---------------------------------------------------------------------------
// Workspace layout (all regions 256-byte aligned).  The header holds the
// error words and the scan's tile ticket; the rest is per-call scratch.
// ---------------------------------------------------------------------------
struct WsHeader {
    int32_t gate_err;       // set by the gate GEMM when a barrier wait runs out
    int32_t scan_err;       // set by the offsets scan (look-back) or a bad id
    uint32_t scan_ticket;   // dynamic tile counter of the look-back scan
    int32_t pad[61];
};
static_assert(sizeof(WsHeader) == 256, "header is 256 bytes");

constexpr int HIST_THREADS = 256;              // 8 warps
constexpr int HIST_WARPS = HIST_THREADS / 32;
constexpr int HIST_ITEMS_PER_WARP = 512;       // 16 chunks of 32 assignments
constexpr int HIST_BLOCK = HIST_WARPS * HIST_ITEMS_PER_WARP;  // 4096 assignments per block
constexpr int MAX_SLOTS = 2048;                // smem: 8 warps x 2048 x 4 B = 64 KB
constexpr int SCAN_THREADS = 256;
constexpr int SCAN_ITEMS = 8;
constexpr int SCAN_TILE = SCAN_THREADS * SCAN_ITEMS;  // 2048 values per look-back tile
constexpr int HS_BLOCKS = 256;                 // blocks of the score-entropy pass
constexpr int MAX_N = 1024;                    // experts supported by selection / stats

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

struct WsLayout {
    size_t header = 0, blk_counts = 0, blk_base = 0, scan_status = 0, hs_partial = 0, total = 0;
    int64_t nblk = 0, L = 0, n_tiles = 0;
};

inline WsLayout ws_layout(int64_t T, int32_t K, int32_t N, int32_t n_slots) {
    WsLayout w;
    int64_t A = T * (int64_t)K;
    w.nblk = (A + HIST_BLOCK - 1) / HIST_BLOCK;
    if (w.nblk < 1) w.nblk = 1;
    w.L = w.nblk * (int64_t)n_slots;
    w.n_tiles = (w.L + SCAN_TILE - 1) / SCAN_TILE;
    size_t off = 0;
    w.header = off;      off += align256(sizeof(WsHeader));
    w.blk_counts = off;  off += align256(sizeof(int32_t) * (size_t)w.L);
    w.blk_base = off;    off += align256(sizeof(int32_t) * (size_t)w.L);
    w.scan_status = off; off += align256(sizeof(uint64_t) * (size_t)w.n_tiles);
    w.hs_partial = off;  off += align256(sizeof(double) * (size_t)HS_BLOCKS * (size_t)(N > 0 ? N : 1));
    w.total = off;
    return w;
}

// ---------------------------------------------------------------------------
// Bounded waiting.  Every spin in the library gives up after about a second
// of wall time (%globaltimer), records an error and lets the kernel finish.
// ---------------------------------------------------------------------------
constexpr uint64_t WAIT_LIMIT_NS = 1000000000ull;

__device__ __forceinline__ uint64_t globaltimer() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ int ld_volatile_i32(const int32_t* p) {
    return *reinterpret_cast<const volatile int32_t*>(p);
}

__device__ __forceinline__ uint64_t ld_acquire_u64(const uint64_t* p) {
    uint64_t v;
    asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void st_release_u64(uint64_t* p, uint64_t v) {
    asm volatile("st.release.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

__device__ __forceinline__ unsigned lanemask_lt() {
    unsigned m;
    asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
    return m;
}

}  // namespace moe

// Host-side launch accounting (per calling thread).
namespace moe_host {
void note_launch(int n = 1);
int sm_count();
}  // namespace moe_host
