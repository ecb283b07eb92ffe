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
// Workspace layout (regions 256-byte aligned):
//   header   256 B   gate error word (moe_route)
//   ctl       64 B   per-call control of the load-statistics pass: tile
//                    ticket, finished-block counter, error bits
//   flags   4*nblk   look-back status per block (look-back kernel): bit 31 |
//                    call epoch << 2 | state (state 1 aggregate, 2 prefix);
//                    a word without this call's tag means "none"
//   agg     nblk x n_slots int32   per-block slot counts (look-back kernel), or
//                    the chain-free kernel's count words [block][slot]: bit 31
//                    (ready) | bit 30 (bad id seen) | count
//   pre     nblk x n_slots int32   per-block inclusive prefix over blocks
//   hs      HS_BLOCKS x N double   score-entropy partial column sums
// The layout depends on the problem size, so one call's flags can lie where
// another call's count words go.  Invariant: no call leaves a flagged word
// behind -- the last block of every load-statistics call, once no block
// reads them any more, clears that call's look-back flags or count words,
// resets the ticket and finished counter and advances the epoch.  The
// workspace is zero-filled once by its owner before first use; the error
// words are sticky until moe_workspace_status reads them.
// ---------------------------------------------------------------------------
struct WsHeader {
    int32_t gate_err;       // bit 0: a barrier wait of the gate GEMM ran out
    int32_t pad0;
    long long cap_info[4];  // capacity routing counters when the caller passes none
    int32_t pad[54];
};
static_assert(sizeof(WsHeader) == 256, "header is 256 bytes");

struct ScanCtl {
    uint32_t ticket;        // next block index to hand out
    uint32_t done;          // blocks finished
    int32_t err;            // this call: bit 0 look-back wait ran out; bit 1 expert id out of range;
                            // bit 2 a ticket past the grid (control words left set by an overlapping call)
    int32_t sticky;         // all calls since the last moe_workspace_status
    uint32_t epoch;         // calls completed; tags this call's look-back flags
    int32_t pad[11];
};
static_assert(sizeof(ScanCtl) == 64, "control block is 64 bytes");

constexpr int LS_THREADS = 256;                // 8 warps
constexpr int LS_WARPS = LS_THREADS / 32;
constexpr int LS_CHUNKS = 8;                   // 32-assignment chunks per warp
constexpr int LS_BLOCK = LS_WARPS * LS_CHUNKS * 32;  // 2048 assignments per block
constexpr int MAX_SLOTS = 2048;                // smem: 8 warps x 2048 x 4 B = 64 KB
constexpr int LS_SLOTS_PER_THREAD = MAX_SLOTS / LS_THREADS;
constexpr int HS_BLOCKS = 256;                 // blocks of the score-entropy pass
constexpr int V2_MAX_BLOCKS = 320;             // largest grid of the chain-free load-statistics kernel
constexpr int V2_WAVE = 148;                   // preferred grid: one block per SM of a B200
constexpr int MAX_N = 1024;                    // experts supported by selection / stats

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

struct WsLayout {
    size_t header = 0, ctl = 0, flags = 0, agg = 0, pre = 0, hs_partial = 0, total = 0, ctl_bytes = 0;
    int64_t nblk = 0;
};

inline WsLayout ws_layout(int64_t T, int32_t K, int32_t N, int32_t n_slots) {
    WsLayout w;
    const int64_t A = T * (int64_t)K;
    w.nblk = (A + LS_BLOCK - 1) / LS_BLOCK;
    if (w.nblk < 1) w.nblk = 1;
    const size_t cells = (size_t)w.nblk * (size_t)n_slots;
    size_t off = 0;
    w.header = off;      off += align256(sizeof(WsHeader));
    w.ctl = off;
    w.flags = off + sizeof(ScanCtl);
    w.ctl_bytes = sizeof(ScanCtl) + sizeof(uint32_t) * (size_t)w.nblk;
    off += align256(w.ctl_bytes);
    // (the chain-free kernel's count words, one per block of >= 2048
    // assignments and slot, fit the agg region)
    w.agg = off;         off += align256(sizeof(int32_t) * cells);
    w.pre = off;         off += align256(sizeof(int32_t) * cells);
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

__device__ __forceinline__ uint32_t ld_acquire_u32(const uint32_t* p) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void st_release_u32(uint32_t* p, uint32_t v) {
    asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
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
