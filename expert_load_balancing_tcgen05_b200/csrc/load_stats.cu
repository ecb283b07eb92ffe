// Load histogram, expert offsets, stable in-expert ranks, load statistics,
// replica plan and bias update.
//
// The histogram is the bincount of the chosen experts ("MoE Routing Entropy
// vs Expert Saturation", section "Concrete Implementation"); statistics are
// those of "A minimal experiment in expert-load imbalance" (total, max,
// max/mean, capacity = max * N), the std/mean monitor of "DeepSeek V4 MoE
// load balancing" (deployment and monitoring section) and the Shannon
// entropy of "The Mathematics" section.  Offsets give the expert-contiguous
// layout that dispatch and combine use ("DeepSeek V4 MoE load balancing",
// DeepEP section).
//
// One stream, no host synchronisation: the optional score-entropy column
// sums, then one single-pass kernel (histogram, look-back, ranks, offsets,
// statistics; see load_stats_kernel).
#include <math.h>
#include <string.h>

#include "common.cuh"

namespace moe {

// ---------------------------------------------------------------------------
// Block-wide exclusive scan of one int per thread (any multiple of 32 threads).
// ---------------------------------------------------------------------------
__device__ __forceinline__ int block_exclusive_scan(int v, int& total, int* sm /*[33]*/) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int y = __shfl_up_sync(FULL, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) sm[warp] = x;
    __syncthreads();
    if (warp == 0) {
        const int nw = blockDim.x >> 5;
        int w = lane < nw ? sm[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int y = __shfl_up_sync(FULL, w, o);
            if (lane >= o) w += y;
        }
        if (lane < nw) sm[lane] = w;  // inclusive over warps
    }
    __syncthreads();
    total = sm[(blockDim.x >> 5) - 1];
    const int warp_excl = warp ? sm[warp - 1] : 0;
    __syncthreads();
    return warp_excl + x - v;
}

__device__ double block_sum_d(double v, double* sm) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(FULL, v, o);
    __syncthreads();
    if (lane == 0) sm[warp] = v;
    __syncthreads();
    double r = 0.0;
    for (int w = 0; w < nw; ++w) r += sm[w];  // same order in every thread
    return r;
}

__device__ double block_max_d(double v, double* sm) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) v = fmax(v, __shfl_xor_sync(FULL, v, o));
    __syncthreads();
    if (lane == 0) sm[warp] = v;
    __syncthreads();
    double r = sm[0];
    for (int w = 1; w < nw; ++w) r = fmax(r, sm[w]);
    return r;
}

__device__ __forceinline__ int ld_volatile(const int32_t* p) { return *reinterpret_cast<const volatile int32_t*>(p); }

// ---------------------------------------------------------------------------
// Single-pass load statistics.
//
// Each block takes the next ticket b and the assignments [b*2048, (b+1)*2048).
//  1. slot of every assignment (replica remap), warp-private shared-memory
//     histograms and the stable rank of each assignment inside its warp's
//     chunk run (warp_slot_rank: peers with the same slot, rank = peers
//     before me + what the warp saw earlier);
//  2. per-slot prefix over the block's warps and the block's slot counts,
//     published as the block aggregate (flag 1);
//  3. decoupled look-back over earlier blocks' vectors (aggregate or
//     inclusive prefix) gives, per slot, the count of all earlier
//     assignments; the block publishes its inclusive prefix (flag 2);
//  4. rank = earlier blocks + earlier warps + within the warp: the
//     assignment's place in its slot's segment;
//  5. the block with the last ticket turns its inclusive prefix (the
//     totals) into counts, offsets (exclusive scan over slots) and the
//     statistics; the last block to finish resets the control words.
// Every spin is bounded; on expiry the error bit is set and the kernel goes on.
// ---------------------------------------------------------------------------
// counts, offsets and statistics from the totals (the last block's
// inclusive prefix over blocks); one combined block reduction for the stats
// tot: the totals, in global memory (read through L2) or, when tot_shared,
// in this block's shared memory; err_word (may be null) holds the call's
// error bits, or'ed with local_err
__device__ __forceinline__ void finish_totals(const int32_t* tot, bool tot_shared, int n_slots, int64_t A,
                                              int32_t* __restrict__ counts, int32_t* __restrict__ offsets,
                                              moe_stats* stats, const double* __restrict__ hs_partial, int hs_blocks,
                                              int N, int64_t T, const int32_t* err_word, int local_err, int* s_scan,
                                              double* s_red, int* s_cnt) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    int c8[LS_SLOTS_PER_THREAD];
#pragma unroll
    for (int j = 0; j < LS_SLOTS_PER_THREAD; ++j) {
        const int e = tid * LS_SLOTS_PER_THREAD + j;
        c8[j] = e < n_slots ? (tot_shared ? tot[e] : __ldcg(tot + e)) : 0;
    }
    __syncthreads();  // every total read before s_cnt (which may alias tot) is written
    int tsum = 0;
#pragma unroll
    for (int j = 0; j < LS_SLOTS_PER_THREAD; ++j) tsum += c8[j];
    int total_i;
    int run = block_exclusive_scan(tsum, total_i, s_scan);
#pragma unroll
    for (int j = 0; j < LS_SLOTS_PER_THREAD; ++j) {
        const int e = tid * LS_SLOTS_PER_THREAD + j;
        if (e < n_slots) {
            offsets[e] = run;
            counts[e] = c8[j];
            s_cnt[e] = c8[j];
        }
        run += c8[j];
    }
    if (tid == 0) offsets[n_slots] = total_i;  // T*K less the dropped assignments
    if (stats == nullptr) return;
    __syncthreads();  // s_cnt complete
    const double total = (double)total_i;
    const double mean = n_slots > 0 ? total / (double)n_slots : 0.0;
    double mx = 0.0, var = 0.0, H = 0.0, Hs = 0.0;
    // one slot per thread (strided), so the fp64 log2 work is spread over the block
    for (int e = tid; e < n_slots; e += LS_THREADS) {
        {
            const double c = (double)s_cnt[e];
            mx = fmax(mx, c);
            var += (c - mean) * (c - mean);
            if (c > 0.0) {
                const double pr = c / total;
                H -= pr * log2(pr);
            }
        }
    }
    if (hs_partial != nullptr) {
        for (int e = tid; e < N; e += LS_THREADS) {
            double m = 0.0;
            for (int q = 0; q < hs_blocks; ++q) m += hs_partial[(int64_t)q * N + e];
            m /= (double)T;
            if (m > 0.0) Hs -= m * log2(m);
        }
    }
    // one reduction round for (max, var, H, Hs): warp butterflies, then warp 0
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
        mx = fmax(mx, __shfl_xor_sync(FULL, mx, o));
        var += __shfl_xor_sync(FULL, var, o);
        H += __shfl_xor_sync(FULL, H, o);
        Hs += __shfl_xor_sync(FULL, Hs, o);
    }
    if (lane == 0) { s_red[warp] = mx; s_red[8 + warp] = var; s_red[16 + warp] = H; s_red[24 + warp] = Hs; }
    __syncthreads();
    if (tid < 4) {
        // the warps' partials in the same order in every thread; the fields
        // are split over four threads so the divisions and the square root
        // do not run one after another
        double rmx = s_red[0], rvar = 0.0, rH = 0.0, rHs = 0.0;
        for (int w = 0; w < LS_WARPS; ++w) {
            rmx = fmax(rmx, s_red[w]);
            rvar += s_red[8 + w];
            rH += s_red[16 + w];
            rHs += s_red[24 + w];
        }
        if (tid == 0) {
            const int err = (err_word != nullptr ? ld_volatile(err_word) : 0) | local_err;
            stats->status = err == 0 ? MOE_OK : ((err & 1) ? MOE_ERR_TIMEOUT : MOE_ERR_INVALID);
            stats->n_slots = n_slots;
            stats->total = (int64_t)total_i;
            stats->max_load = (int64_t)rmx;
            stats->mean = mean;
        } else if (tid == 1) {
            stats->imbalance = mean > 0.0 ? rmx / mean : 0.0;
            stats->capacity_fixed = rmx * (double)n_slots;
            stats->capacity_125 = 1.25 * mean;
        } else if (tid == 2) {
            rvar /= (double)(n_slots > 0 ? n_slots : 1);
            stats->std_over_mean = mean > 0.0 ? sqrt(rvar) / mean : 0.0;
        } else {
            stats->entropy_load_bits = rH;
            stats->entropy_score_bits = hs_partial != nullptr ? rHs : NAN;
        }
    }
}

constexpr uint32_t FLAG_AGG = 1, FLAG_PREFIX = 2;

// Place of each lane's assignment among the warp's assignments to the same
// slot so far (the warp's running histogram `my`, in shared memory), in lane
// order.  The lanes holding the same slot are found by one ballot per bit of
// the slot (nbits = bits of n_slots - 1) instead of __match_any_sync, whose
// cost grows with the number of distinct values; the lowest of them adds the
// group's size to the histogram with one shared-memory atomic.  Lanes with
// slot < 0 get an unused value.  Call with the whole warp, chunks in order:
// the leader's atomic returns before the warp-wide shuffle of its result, so
// a later chunk's atomic on the same slot always sees it.
// The lanes holding `slot` (bit-sliced ballots), for warp_slot_rank and the
// chain-free kernel's interleaved chunks.
__device__ __forceinline__ unsigned slot_peers(int slot, int nbits) {
    unsigned peers = __ballot_sync(FULL, slot >= 0);
    if (slot < 0) peers = ~peers;
#pragma unroll
    for (int bit = 0; bit < 11; ++bit) {
        if (bit < nbits) {
            const unsigned B = __ballot_sync(FULL, (slot >> bit) & 1);
            peers &= ((slot >> bit) & 1) ? B : ~B;
        }
    }
    return peers;
}

__device__ __forceinline__ int warp_slot_rank(int slot, int nbits, int32_t* my, int lane) {
    unsigned peers = __ballot_sync(FULL, slot >= 0);
    if (slot < 0) peers = ~peers;
#pragma unroll
    for (int bit = 0; bit < 11; ++bit) {
        if (bit < nbits) {
            const unsigned B = __ballot_sync(FULL, (slot >> bit) & 1);
            peers &= ((slot >> bit) & 1) ? B : ~B;
        }
    }
    const int before = __popc(peers & lanemask_lt());
    const int leader = __ffs(peers) - 1;
    int seen = 0;
    if (slot >= 0 && lane == leader) seen = atomicAdd(my + slot, __popc(peers));
    seen = __shfl_sync(FULL, seen, leader);
    return seen + before;
}

// Block end: the last block to finish folds this call's error bits into the
// sticky word and resets the control words for the next call.
// Every block calls it (whole block, uniformly) as its last step.  The last
// to finish -- no block reads the look-back flags any more -- clears the
// call's flags, so that no flagged word outlives its call (the workspace
// layout depends on the problem size, and another call's count words may
// land where these flags were), folds the call's error bits into the sticky
// word and resets the control words.
__device__ __forceinline__ void block_done(ScanCtl* ctl, uint32_t* flags, int64_t nblk) {
    __shared__ int s_last_lb;
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        s_last_lb = atomicAdd(&ctl->done, 1u) == (uint32_t)(nblk - 1);
    }
    __syncthreads();
    if (s_last_lb) {
        __threadfence();
        for (int64_t i = threadIdx.x; i < nblk; i += blockDim.x) flags[i] = 0u;
        if (threadIdx.x == 0) {
            ctl->sticky |= ctl->err;
            ctl->err = 0;
            ctl->done = 0;
            ctl->ticket = 0;
            ctl->epoch = ctl->epoch + 1;
        }
    }
}

__device__ __forceinline__ uint32_t flag_tag(uint32_t epoch) { return 0x80000000u | ((epoch & 0x1FFFFFFFu) << 2); }
// state of a flag word for the call tagged `tag`: 0 unless the word carries the tag
__device__ __forceinline__ uint32_t flag_state(uint32_t f, uint32_t tag) { return (f & ~3u) == tag ? (f & 3u) : 0u; }

__global__ void __launch_bounds__(LS_THREADS) load_stats_kernel(
    const int32_t* __restrict__ idx, int64_t A, int K, int N, const int32_t* __restrict__ replica_slot,
    int n_slots, int32_t* __restrict__ slot_out, int32_t* __restrict__ rank_out, int32_t* __restrict__ counts,
    int32_t* __restrict__ offsets, moe_stats* stats, const double* __restrict__ hs_partial, int hs_blocks,
    int64_t T, ScanCtl* ctl, uint32_t* flags, int32_t* agg, int32_t* pre, int64_t nblk, uint32_t ticket_base) {
    extern __shared__ int32_t sm_dyn[];
    int32_t* wh = sm_dyn;                          // [LS_WARPS][n_slots]
    int32_t* ex = sm_dyn + LS_WARPS * n_slots;     // [n_slots] earlier-block counts
    __shared__ uint32_t s_b, s_tag;
    __shared__ int s_scan[33];
    __shared__ int s_win[3];
    __shared__ double s_red[32];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    if (tid == 0) {
        s_b = ticket_base + atomicAdd(&ctl->ticket, 1u);
        s_tag = flag_tag(ld_volatile(reinterpret_cast<const int32_t*>(&ctl->epoch)));
    }
    for (int i = tid; i < LS_WARPS * n_slots; i += LS_THREADS) wh[i] = 0;
    __syncthreads();
    const int64_t b = s_b;
    const uint32_t tag = s_tag;
    if (b >= nblk) {
        // a ticket past the grid: the control words were not reset (two calls
        // overlapped on one workspace).  Write nothing; report it (bit 2).
        if (tid == 0) atomicOr(&ctl->err, 4);
        block_done(ctl, flags, nblk);
        return;
    }

    // 1. slots, warp histograms, in-warp stable ranks (all loads issued first)
    int32_t* my = wh + warp * n_slots;
    const int nbits = n_slots > 1 ? 32 - __clz(n_slots - 1) : 0;
    const int64_t base_a = b * LS_BLOCK + (int64_t)warp * (LS_CHUNKS * 32);
    int slot_r[LS_CHUNKS], rank_r[LS_CHUNKS];
#pragma unroll
    for (int j = 0; j < LS_CHUNKS; ++j) {
        const int64_t a = base_a + j * 32 + lane;
        slot_r[j] = a < A ? __ldg(idx + a) : -1;
    }
    int bad = 0;
#pragma unroll
    for (int j = 0; j < LS_CHUNKS; ++j) {
        const int64_t a = base_a + j * 32 + lane;
        int slot = slot_r[j];
        if (a < A) {
            if (slot < 0) {
                slot = -1;  // dropped by the capacity limit: no slot, rank -1
            } else if (slot >= N) {
                bad = 1;
                slot = -1;
            } else if (replica_slot != nullptr) {
                const int r = __ldg(replica_slot + slot);
                if (r >= 0 && ((a / K) & 1)) slot = r;
                if (slot >= n_slots) { bad = 1; slot = -1; }
            }
        }
        rank_r[j] = warp_slot_rank(slot, nbits, my, lane);
        slot_r[j] = slot;
    }
    if (bad) atomicOr(&ctl->err, 2);
    __syncthreads();

    // 2. per-slot exclusive prefix over warps; block aggregate
    int my_agg[LS_SLOTS_PER_THREAD];
#pragma unroll
    for (int j = 0; j < LS_SLOTS_PER_THREAD; ++j) {
        const int e = tid + j * LS_THREADS;
        my_agg[j] = 0;
        if (e < n_slots) {
            int run = 0;
#pragma unroll
            for (int w = 0; w < LS_WARPS; ++w) {
                const int c = wh[w * n_slots + e];
                wh[w * n_slots + e] = run;
                run += c;
            }
            my_agg[j] = run;
            agg[b * n_slots + e] = run;
            if (b == 0) pre[e] = run;
        }
    }
    __threadfence();
    __syncthreads();
    if (tid == 0) st_release_u32(flags + b, tag | (b == 0 ? FLAG_PREFIX : FLAG_AGG));

    // 3. look-back over earlier blocks, 32 at a time: warp 0 reads a window of
    //    32 predecessor flags at once, finds the nearest inclusive prefix and
    //    waits (bounded) only for the blocks above it to publish their
    //    aggregates; then every thread adds, for its slots, the window's
    //    aggregates and that prefix with independent loads.
    int excl[LS_SLOTS_PER_THREAD];
#pragma unroll
    for (int j = 0; j < LS_SLOTS_PER_THREAD; ++j) excl[j] = 0;
    if (b > 0) {
        int64_t hi = b - 1;
        bool timed_out = false;
        while (hi >= 0) {
            if (warp == 0) {
                const int64_t p = hi - lane;
                uint64_t t0 = 0;
                int stop = 32, ready = 0;
                while (true) {
                    const uint32_t f = p >= 0 ? flag_state(ld_acquire_u32(flags + p), tag) : FLAG_PREFIX;
                    const unsigned pm = __ballot_sync(FULL, f == FLAG_PREFIX);
                    const unsigned zm = __ballot_sync(FULL, f == 0);
                    stop = pm ? __ffs(pm) - 1 : 32;               // nearest prefix (lane 0 = block hi)
                    const unsigned need = stop == 32 ? FULL : ((1u << stop) - 1u);
                    if (!(zm & need)) { ready = 1; break; }
                    // lane 0's clock decides for the whole warp, so the warp leaves together
                    int give_up = 0;
                    if (lane == 0) {
                        if (t0 == 0) t0 = globaltimer();
                        else give_up = globaltimer() - t0 > WAIT_LIMIT_NS;
                    }
                    if (__shfl_sync(FULL, give_up, 0)) break;
                    __nanosleep(32);
                }
                if (lane == 0) {
                    s_win[0] = stop;
                    // a window that reaches below block 0 ends at the virtual prefix there
                    s_win[1] = (stop < 32 && hi - stop >= 0) ? 1 : 0;
                    s_win[2] = ready;
                }
            }
            __syncthreads();
            const int stop = s_win[0], has_pre = s_win[1];
            if (!s_win[2]) timed_out = true;
            // the window's blocks hi, hi-1, ..., hi-nagg+1 give aggregates; block
            // hi-stop (if real) its prefix.  L2-coherent loads (ld.cg), all
            // issued before the first is used: one L2 latency per window.
            const int nagg = (int)(stop < hi + 1 ? stop : hi + 1);
#pragma unroll
            for (int j = 0; j < LS_SLOTS_PER_THREAD; ++j) {
                const int e = tid + j * LS_THREADS;
                if (e >= n_slots) continue;
                int v32[32];
#pragma unroll
                for (int l = 0; l < 32; ++l) v32[l] = l < nagg ? __ldcg(agg + (hi - l) * n_slots + e) : 0;
                int acc = has_pre ? __ldcg(pre + (hi - stop) * n_slots + e) : 0;
#pragma unroll
                for (int l = 0; l < 32; ++l) acc += v32[l];
                excl[j] += acc;
            }
            const bool done = stop < 32 || !s_win[2];
            __syncthreads();  // s_win is rewritten by the next window
            if (done) break;
            hi -= 32;
        }
        if (timed_out && tid == 0) atomicOr(&ctl->err, 1);
#pragma unroll
        for (int j = 0; j < LS_SLOTS_PER_THREAD; ++j) {
            const int e = tid + j * LS_THREADS;
            if (e < n_slots) pre[b * n_slots + e] = excl[j] + my_agg[j];
        }
        __threadfence();
    }
#pragma unroll
    for (int j = 0; j < LS_SLOTS_PER_THREAD; ++j) {
        const int e = tid + j * LS_THREADS;
        if (e < n_slots) ex[e] = excl[j];
    }
    __syncthreads();
    if (tid == 0 && b > 0) st_release_u32(flags + b, tag | FLAG_PREFIX);

    // 4. in-expert ranks (and the slots, stored here rather than in the
    //    histogram loop so that no store sits between its chunks)
#pragma unroll
    for (int j = 0; j < LS_CHUNKS; ++j) {
        const int64_t a = base_a + j * 32 + lane;
        if (a < A) {
            rank_out[a] = slot_r[j] >= 0 ? ex[slot_r[j]] + my[slot_r[j]] + rank_r[j] : -1;
            if (slot_out != nullptr) slot_out[a] = slot_r[j];
        }
    }

    // 5. the block with the last ticket holds the totals in its inclusive
    //    prefix: it writes counts, offsets and statistics while the other
    //    blocks still write ranks; the last block to finish resets the
    //    control words for the next call
    if (b == nblk - 1 && counts != nullptr) {  // (the bounded-wait self-test passes no outputs)
        __syncthreads();
        // the warp histograms are no longer needed: they hold the counts for the statistics
        finish_totals(pre + b * n_slots, false, n_slots, A, counts, offsets, stats, hs_partial, hs_blocks, N, T,
                      &ctl->err, 0, s_scan, s_red, wh);
    }
    block_done(ctl, flags, nblk);
}

// ---------------------------------------------------------------------------
// Load statistics without a look-back chain (problems up to ~2.6M
// assignments).  Block b takes assignments [b*BPB, (b+1)*BPB), BPB = 8 warps x
// C chunks of 32 (one wave of at most ~320 blocks):
//  1. slots, warp histograms and in-warp stable ranks, as above;
//  2. per-slot prefix over the block's warps; the block's per-slot counts are
//     published as 32-bit words with bit 31 set, so a word is its own ready
//     flag: no separate flag and no fence on the normal path (a word without
//     bit 31 -- zero, or the look-back kernel's counts, which never have it
//     -- reads as "not yet");
//  3. each block sums, per slot, the words of ALL earlier blocks (laid out
//     [block][slot], so a warp reads one 128-byte line per earlier block; 32
//     loads in flight, a bounded re-poll of any word not yet ready): the
//     count of every earlier assignment in that slot, without waiting on
//     inclusive prefixes;
//  4. rank = earlier blocks + earlier warps + within the warp;
//  5. the last block's sums plus its own counts are the totals: counts,
//     offsets, statistics.  The last block to finish -- no block reads the
//     words any more -- clears this call's words, so no ready word outlives
//     its call, and resets the control words.
// A one-block problem shares nothing with other blocks: it publishes nothing,
// waits for nothing and leaves the control words untouched (error bits go to
// the sticky word directly).
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t ld_relaxed_u32(const uint32_t* p) {
    uint32_t v;
    asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void st_relaxed_u32(uint32_t* p, uint32_t v) {
    asm volatile("st.relaxed.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

constexpr uint32_t WORD_READY = 0x80000000u;  // a published per-block count: bit 31 | bit 30 | count
constexpr uint32_t WORD_BAD = 0x40000000u;    // the publishing block saw an expert id out of range
constexpr uint32_t WORD_COUNT = 0x3fffffffu;

template <int C>
__global__ void __launch_bounds__(LS_THREADS, 1) load_stats_v2_kernel(
    const int32_t* __restrict__ idx, int64_t A, int K, int N, const int32_t* __restrict__ replica_slot,
    int n_slots, int32_t* __restrict__ slot_out, int32_t* __restrict__ rank_out, int32_t* __restrict__ counts,
    int32_t* __restrict__ offsets, moe_stats* stats, const double* __restrict__ hs_partial, int hs_blocks,
    int64_t T, ScanCtl* ctl, uint32_t* aggw, int nblk, int block_base, const int32_t* __restrict__ tile_counts) {
    // Each SM runs one block of this kernel once, so its instructions are
    // fetched cold: the loops stay rolled (their bodies then run from the
    // instruction cache) and the block's ids, slots and ranks live in shared
    // memory rather than in fully unrolled registers.
    constexpr int BPB = LS_WARPS * C * 32;
    extern __shared__ int32_t sm_dyn[];
    int32_t* wh = sm_dyn;                       // [LS_WARPS][n_slots]
    int32_t* ex = sm_dyn + LS_WARPS * n_slots;  // [n_slots] earlier-block counts
    int32_t* s_slot = ex + n_slots;             // [BPB] this block's expert ids, then slots
    int32_t* s_rank = s_slot + BPB;             // [BPB] in-warp ranks
    int32_t* s_rep = s_rank + BPB;              // [N] replica slot of each expert (with replicas)
    __shared__ int s_err;
    __shared__ int s_scan[33];
    __shared__ double s_red[32];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int b = block_base + (int)blockIdx.x;  // block_base > 0 only in the bounded-wait self-test
    const bool multi = nblk > 1;
    const int64_t a0 = (int64_t)b * BPB;  // count words: aggw[block * n_slots + slot]

    // the block's expert ids (eight independent loads per thread in flight)
#pragma unroll 8
    for (int v = tid; v < BPB; v += LS_THREADS) s_slot[v] = a0 + v < A ? __ldg(idx + a0 + v) : -1;
    if (replica_slot != nullptr)
        for (int e = tid; e < N; e += LS_THREADS) s_rep[e] = __ldg(replica_slot + e);
    if (tid == 0) s_err = 0;
    for (int i = tid; i < LS_WARPS * n_slots; i += LS_THREADS) wh[i] = 0;
    // the gate epilogue's per-tile histograms (tiles of 128 tokens, aligned to
    // this block, split by token parity) give the block's counts without its
    // indices: publish them at once
    const bool pre_published = tile_counts != nullptr && multi;
    int tc_agg[LS_SLOTS_PER_THREAD];
    if (pre_published) {
        const int64_t tok0 = (int64_t)b * (BPB / K);
        const int64_t ntiles = (T + 127) / 128;
        const int64_t j0 = tok0 / 128;
        const int64_t j1 = min(ntiles, j0 + (int64_t)(BPB / K) / 128);
        // replica slot -> the expert it copies (ex[] is free until step 3)
        for (int i = tid; i < n_slots - N; i += LS_THREADS) ex[i] = -1;
        __syncthreads();
        if (replica_slot != nullptr)
            for (int e = tid; e < N; e += LS_THREADS) {
                const int r = __ldg(replica_slot + e);
                if (r >= N && r < n_slots) ex[r - N] = e;
            }
        __syncthreads();
#pragma unroll 1
        for (int j = 0; j < LS_SLOTS_PER_THREAD; ++j) {
            const int e = tid + j * LS_THREADS;
            int c = 0;
            if (e < n_slots) {
                const int src = e < N ? e : ex[e - N];
                const bool has_rep = e < N && replica_slot != nullptr && __ldg(replica_slot + e) >= 0;
                if (src >= 0)
                    for (int64_t q = j0; q < j1; ++q) {
                        const int32_t* tq = tile_counts + q * 2 * N;
                        if (e < N) c += __ldg(tq + src) + (has_rep ? 0 : __ldg(tq + N + src));
                        else c += __ldg(tq + N + src);
                    }
                if (b < nblk - 1) st_relaxed_u32(aggw + (int64_t)b * n_slots + e, WORD_READY | (uint32_t)c);
            }
            tc_agg[j] = c;
        }
    }
    __syncthreads();

    // 1. slots, warp histograms, in-warp stable ranks: four chunks of 32 per
    //    step, their ballot chains independent; the leaders' atomics on the
    //    warp's running histogram are issued in chunk order, so a later
    //    chunk's atomic on a slot always sees the earlier chunks' counts
    int32_t* my = wh + warp * n_slots;
    const int nbits = n_slots > 1 ? 32 - __clz(n_slots - 1) : 0;
    int bad = 0;
#pragma unroll 1
    for (int j0 = 0; j0 < C; j0 += 4) {
        int sl[4];
        unsigned pe[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int li = warp * (C * 32) + (j0 + u) * 32 + lane;
            const int64_t a = a0 + li;
            int slot = s_slot[li];
            if (a < A) {
                if (slot < 0) {
                    slot = -1;  // dropped by the capacity limit: no slot, rank -1
                } else if (slot >= N) {
                    bad = 1;
                    slot = -1;
                } else if (replica_slot != nullptr) {
                    const int r = s_rep[slot];
                    if (r >= 0 && ((a / K) & 1)) slot = r;
                    if (slot >= n_slots) { bad = 1; slot = -1; }
                }
            }
            sl[u] = slot;
            pe[u] = slot_peers(slot, nbits);
        }
        int seen[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            seen[u] = 0;
            if (sl[u] >= 0 && lane == __ffs(pe[u]) - 1) seen[u] = atomicAdd(my + sl[u], __popc(pe[u]));
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int li = warp * (C * 32) + (j0 + u) * 32 + lane;
            s_rank[li] = __shfl_sync(FULL, seen[u], __ffs(pe[u]) - 1) + __popc(pe[u] & lanemask_lt());
            s_slot[li] = sl[u];
        }
    }
    if (__any_sync(FULL, bad) && lane == 0) atomicOr(&s_err, 2);
    __syncthreads();
    const int blk_err = s_err;  // the published counts carry it (WORD_BAD) to later blocks

    // 2. per-slot exclusive prefix over warps; the block's counts, published
    int my_agg[LS_SLOTS_PER_THREAD];
#pragma unroll
    for (int j = 0; j < LS_SLOTS_PER_THREAD; ++j) {
        const int e = tid + j * LS_THREADS;
        my_agg[j] = 0;
        if (e < n_slots) {
            int run = 0;
#pragma unroll
            for (int w = 0; w < LS_WARPS; ++w) {
                const int c = wh[w * n_slots + e];
                wh[w * n_slots + e] = run;
                run += c;
            }
            my_agg[j] = run;
            if (pre_published) {
                if (tc_agg[j] != run) atomicOr(&s_err, 2);  // the tile histograms do not match the indices
            } else if (multi && b < nblk - 1) {
                st_relaxed_u32(aggw + (int64_t)b * n_slots + e, WORD_READY | (blk_err ? WORD_BAD : 0u) | (uint32_t)run);
            }
        }
    }

    // 3. counts of all earlier blocks, per slot: a warp reads one 128-byte line
    //    per earlier block (words [block][slot]), up to 64 blocks in flight at
    //    once; the words not ready yet are re-read together, round by round
    constexpr int PB = 64;
    int excl[LS_SLOTS_PER_THREAD];
    bool timed_out = false, pred_bad = false;
#pragma unroll 1
    for (int j = 0; j < LS_SLOTS_PER_THREAD; ++j) {
        excl[j] = 0;
        const int e = tid + j * LS_THREADS;
        if (e >= n_slots || b == 0) continue;
        uint64_t t0 = 0;
        int acc = 0;
#pragma unroll 1
        for (int q0 = 0; q0 < b; q0 += PB) {
            uint32_t w[PB];
#pragma unroll
            // first pass: plain L2 loads (ld.global.cg), all in flight; only a
            // word not yet ready is re-read with the relaxed loads below
            for (int u = 0; u < PB; ++u)
                w[u] = q0 + u < b ? __ldcg(aggw + (int64_t)(q0 + u) * n_slots + e) : WORD_READY;
            bool pending = false;
#pragma unroll
            for (int u = 0; u < PB; ++u) pending |= !(w[u] & WORD_READY);
            // bounded rounds: every word not ready yet is re-read (all in
            // flight), until each is ready or the wait limit has passed
            while (pending && !timed_out) {
                if (t0 == 0) t0 = globaltimer();
                else if (globaltimer() - t0 > WAIT_LIMIT_NS) { timed_out = true; break; }
                __nanosleep(64);
#pragma unroll
                for (int u = 0; u < PB; ++u)
                    if (!(w[u] & WORD_READY)) w[u] = ld_relaxed_u32(aggw + (int64_t)(q0 + u) * n_slots + e);
                pending = false;
#pragma unroll
                for (int u = 0; u < PB; ++u) pending |= !(w[u] & WORD_READY);
            }
#pragma unroll
            for (int u = 0; u < PB; ++u) {
                if (w[u] & WORD_READY) {
                    acc += (int)(w[u] & WORD_COUNT);
                    pred_bad |= (w[u] & WORD_BAD) != 0;
                }
            }
        }
        excl[j] = acc;
    }
    if (pred_bad) atomicOr(&s_err, 2);
    if (timed_out) atomicOr(&s_err, 1);
#pragma unroll
    for (int j = 0; j < LS_SLOTS_PER_THREAD; ++j) {
        const int e = tid + j * LS_THREADS;
        if (e < n_slots) ex[e] = excl[j];
    }
    __syncthreads();

    // 4. in-expert ranks, and the slots
#pragma unroll 4
    for (int j = 0; j < C; ++j) {
        const int li = warp * (C * 32) + j * 32 + lane;
        const int64_t a = a0 + li;
        if (a < A) {
            const int sl = s_slot[li];
            rank_out[a] = sl >= 0 ? ex[sl] + my[sl] + s_rank[li] : -1;
            if (slot_out != nullptr) slot_out[a] = sl;
        }
    }

    // 5. the last block: totals = earlier blocks + its own counts
    if (b == nblk - 1 && counts != nullptr) {
        // errors: this block's, its predecessors' bad ids (carried in their
        // counts), and whatever else other blocks have recorded by now (the
        // workspace status has every one)
        const int other_err = multi ? ld_volatile(&ctl->err) : 0;  // its latency overlaps the totals
        __syncthreads();  // ranks read ex and my before wh is reused for the totals
        const int local_err = s_err;
#pragma unroll
        for (int j = 0; j < LS_SLOTS_PER_THREAD; ++j) {
            const int e = tid + j * LS_THREADS;
            if (e < n_slots) wh[e] = excl[j] + my_agg[j];
        }
        __syncthreads();
        finish_totals(wh, true, n_slots, A, counts, offsets, stats, hs_partial, hs_blocks, N, T, nullptr,
                      local_err | other_err, s_scan, s_red, wh);
    }
    if (multi) {
        __syncthreads();
        if (tid == 0 && s_err) atomicOr(&ctl->err, s_err);  // bad ids, timeouts, histogram mismatch
        __syncthreads();
        // the last block to finish clears this call's count words (no block
        // reads them any more) and resets the control words
        __shared__ int s_last;
        if (tid == 0) {
            __threadfence();
            s_last = atomicAdd(&ctl->done, 1u) == (uint32_t)(nblk - 1);
        }
        __syncthreads();
        if (s_last) {
            __threadfence();
            // (the region starts 256-byte aligned: 16-byte stores, then the tail)
            const int64_t nw = (int64_t)(nblk - 1) * n_slots;
            uint4* aw4 = reinterpret_cast<uint4*>(aggw);
            for (int64_t i = tid; i < nw / 4; i += LS_THREADS) aw4[i] = make_uint4(0u, 0u, 0u, 0u);
            for (int64_t i = (nw / 4) * 4 + tid; i < nw; i += LS_THREADS) aggw[i] = 0u;
            if (tid == 0) {
                ctl->sticky |= ctl->err;
                ctl->err = 0;
                ctl->done = 0;
                ctl->ticket = 0;
                ctl->epoch = ctl->epoch + 1;
            }
        }
    } else if (tid == 0 && s_err != 0) {
        atomicOr(&ctl->sticky, s_err);  // read and cleared by moe_workspace_status
    }
}

// ---------------------------------------------------------------------------
// score entropy, pass 1: per-block column sums (double) of per-token
// normalised scores (softmax rows as they are, sigmoid rows / their sum).
// Fixed token-to-block assignment, fixed reduction order: deterministic.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) score_colsum_kernel(const float* __restrict__ s, int64_t T, int N,
                                                           int fn, double* __restrict__ partial) {
    extern __shared__ double cs[];  // [8][N]
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int per_lane = (N + 31) / 32;  // <= 32
    double acc[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) acc[i] = 0.0;
    for (int64_t t = (int64_t)blockIdx.x * 8 + warp; t < T; t += (int64_t)gridDim.x * 8) {
        const float* row = s + t * N;
        double rs = 1.0;
        if (fn == MOE_SIGMOID) {
            double part = 0.0;
            for (int e = lane; e < N; e += 32) part += (double)row[e];
#pragma unroll
            for (int o = 16; o >= 1; o >>= 1) part += __shfl_xor_sync(FULL, part, o);
            rs = part;
        }
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            const int e = lane + 32 * i;
            if (i < per_lane && e < N) acc[i] += (double)row[e] / rs;
        }
    }
#pragma unroll
    for (int i = 0; i < 32; ++i) {
        const int e = lane + 32 * i;
        if (i < per_lane && e < N) cs[warp * N + e] = acc[i];
    }
    __syncthreads();
    for (int e = threadIdx.x; e < N; e += blockDim.x) {
        double v = 0.0;
        for (int w = 0; w < 8; ++w) v += cs[w * N + e];
        partial[(int64_t)blockIdx.x * N + e] = v;
    }
}

// ---------------------------------------------------------------------------
// replica plan and bias update: one block each
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(1024) replica_plan_kernel(const int32_t* __restrict__ counts, int N,
                                                            int R, int32_t* __restrict__ replica_slot) {
    extern __shared__ int32_t c[];
    for (int e = threadIdx.x; e < N; e += blockDim.x) c[e] = counts[e];
    __syncthreads();
    for (int e = threadIdx.x; e < N; e += blockDim.x) {
        const int ce = c[e];
        int rank = 0;
        for (int f = 0; f < N; ++f) rank += (c[f] > ce) || (c[f] == ce && f < e);
        replica_slot[e] = rank < R ? N + rank : -1;
    }
}

__global__ void __launch_bounds__(1024) bias_update_kernel(const int32_t* __restrict__ counts, int N,
                                                           int64_t total, float u, int mode,
                                                           float* __restrict__ bias) {
    for (int e = threadIdx.x; e < N; e += blockDim.x) {
        const int64_t c = counts[e];
        if (mode == 0) {
            const int64_t lhs = c * (int64_t)N;
            const int sgn = (lhs > total) - (lhs < total);
            bias[e] = __fsub_rn(bias[e], __fmul_rn(u, (float)sgn));
        } else {
            const float target = (float)((double)total / (double)N);
            const float err = __fsub_rn((float)c, target);
            const float sgn = (float)((err > 0.f) - (err < 0.f));
            const float a = __fmul_rn(u, sgn);
            const float r = __fdiv_rn(fabsf(err), target);
            bias[e] = __fsub_rn(bias[e], __fmul_rn(a, r));
        }
    }
}

// smoothed-load bias step: ema = fp32(fp32(alpha*ema) + fp32((1-alpha)*c)),
// b -= fp32(u * sign(ema - fp32(total/N)))
__global__ void __launch_bounds__(1024) bias_update_ema_kernel(const int32_t* __restrict__ counts, int N,
                                                               int64_t total, float u, float alpha,
                                                               float* __restrict__ ema, float* __restrict__ bias) {
    const float mean = (float)((double)total / (double)N);
    const float beta = __fsub_rn(1.f, alpha);
    for (int e = threadIdx.x; e < N; e += blockDim.x) {
        const float v = __fadd_rn(__fmul_rn(alpha, ema[e]), __fmul_rn(beta, (float)counts[e]));
        ema[e] = v;
        const float sgn = (float)((v > mean) - (v < mean));
        bias[e] = __fsub_rn(bias[e], __fmul_rn(u, sgn));
    }
}

// forcible balancing: expert (t*K + k) mod N, weight scale / K
__global__ void __launch_bounds__(256) route_balanced_kernel(int64_t A, int K, int N, float w,
                                                             int32_t* __restrict__ idx, float* __restrict__ wout) {
    for (int64_t a = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; a < A; a += (int64_t)gridDim.x * blockDim.x) {
        idx[a] = (int32_t)(a % N);
        wout[a] = w;
    }
}

// ---------------------------------------------------------------------------
// host launchers
// ---------------------------------------------------------------------------
cudaError_t launch_load_stats(const int32_t* idx, int64_t T, int K, int N, const int32_t* replica_slot,
                              int n_slots, int32_t* slot_idx, int32_t* counts, int32_t* offsets,
                              int32_t* rank, const float* scores, int score_fn, moe_stats* stats,
                              void* ws, cudaStream_t st, const int32_t* tile_counts) {
    const WsLayout L = ws_layout(T, K, N, n_slots);
    char* w = static_cast<char*>(ws);
    ScanCtl* ctl = reinterpret_cast<ScanCtl*>(w + L.ctl);
    uint32_t* flags = reinterpret_cast<uint32_t*>(w + L.flags);
    int32_t* agg = reinterpret_cast<int32_t*>(w + L.agg);
    int32_t* pre = reinterpret_cast<int32_t*>(w + L.pre);
    double* partial = reinterpret_cast<double*>(w + L.hs_partial);
    const int64_t A = T * K;
    cudaError_t e;
    const double* part = nullptr;
    if (stats != nullptr && scores != nullptr && T > 0) {
        const size_t csm = sizeof(double) * 8 * (size_t)N;
        if (csm > 48 * 1024) {
            e = cudaFuncSetAttribute(score_colsum_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)csm);
            if (e != cudaSuccess) return e;
        }
        score_colsum_kernel<<<HS_BLOCKS, 256, csm, st>>>(scores, T, N, score_fn, partial);
        moe_host::note_launch();
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        part = partial;
    }
    const size_t lsm = sizeof(int32_t) * (LS_WARPS + 1) * (size_t)n_slots;
    // problems of up to V2_MAX_BLOCKS blocks of 2048, 4096 or 8192 assignments
    // run without a look-back chain; larger ones use the look-back kernel
    // the smallest blocks (1024, 2048, 4096 or 8192 assignments) that still
    // fit one block per SM, or, beyond that, up to V2_MAX_BLOCKS blocks of 8192
    int chunks = 32;
    for (int c = 8; c <= 32; c *= 2)
        if (A <= (int64_t)V2_WAVE * LS_THREADS * c) { chunks = c; break; }
    const int64_t nb2 = (A + (int64_t)LS_THREADS * chunks - 1) / ((int64_t)LS_THREADS * chunks);
    if (nb2 <= V2_MAX_BLOCKS) {
        const int nb = nb2 < 1 ? 1 : (int)nb2;
        uint32_t* aggw = reinterpret_cast<uint32_t*>(agg);  // one ready-flagged count word per (block, slot)
        auto kern = chunks == 8 ? load_stats_v2_kernel<8>
                                : (chunks == 16 ? load_stats_v2_kernel<16> : load_stats_v2_kernel<32>);
        // + ids/slots, ranks and the replica map
        const size_t lsm2 = lsm + sizeof(int32_t) * (2 * (size_t)LS_THREADS * chunks + (size_t)N);
        if (lsm2 > 48 * 1024) {
            e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)lsm2);
            if (e != cudaSuccess) return e;
        }
        // the tile histograms serve when a block is a whole number of 128-token tiles
        const int bpb = LS_THREADS * chunks;
        const bool tiles_ok = tile_counts != nullptr && bpb % K == 0 && (bpb / K) % 128 == 0;
        kern<<<nb, LS_THREADS, lsm2, st>>>(idx, A, K, N, replica_slot, n_slots, slot_idx, rank, counts, offsets, stats,
                                          part, HS_BLOCKS, T, ctl, aggw, nb, 0, tiles_ok ? tile_counts : nullptr);
        moe_host::note_launch();
        return cudaGetLastError();
    }
    if (lsm > 48 * 1024) {
        e = cudaFuncSetAttribute(load_stats_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)lsm);
        if (e != cudaSuccess) return e;
    }
    load_stats_kernel<<<(unsigned)L.nblk, LS_THREADS, lsm, st>>>(idx, A, K, N, replica_slot, n_slots, slot_idx, rank,
                                                                  counts, offsets, stats, part, HS_BLOCKS, T, ctl,
                                                                  flags, agg, pre, L.nblk, 0u);
    moe_host::note_launch();
    return cudaGetLastError();
}

// Self-test of the bounded waits of both load-statistics kernels: a
// two-block problem (no assignments, 8 slots) of which only the second block
// is launched, so block 0 never publishes (its look-back flag, or its ready
// count words, never appear).  Each probe block must give up after the wait
// limit, set the timeout bit and finish.  Returns the error bits of the two
// probes and'ed (bit 0 set only if both waits ran out).
cudaError_t run_lookback_timeout_probe(void* ws, int32_t* err_out, cudaStream_t st) {
    const WsLayout L = ws_layout(2 * LS_BLOCK, 1, 8, 8);
    char* w = static_cast<char*>(ws);
    ScanCtl* ctl = reinterpret_cast<ScanCtl*>(w + L.ctl);
    int32_t bits = ~0;
    for (int probe = 0; probe < 2; ++probe) {
        // ticket, finished count and error words start at zero; the epoch
        // stays, so flags left by earlier calls are stale (count words are
        // cleared by every call's last block)
        cudaError_t e = cudaMemsetAsync(ctl, 0, 4 * sizeof(int32_t), st);
        if (e != cudaSuccess) return e;
        const size_t smem = sizeof(int32_t) * (LS_WARPS + 1) * 8 + (probe == 1 ? sizeof(int32_t) * (2 * LS_BLOCK + 8) : 0);
        if (probe == 0)
            load_stats_kernel<<<1, LS_THREADS, smem, st>>>(
                nullptr, 0, 1, 8, nullptr, 8, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, 0, 0, ctl,
                reinterpret_cast<uint32_t*>(w + L.flags), reinterpret_cast<int32_t*>(w + L.agg),
                reinterpret_cast<int32_t*>(w + L.pre), /*nblk=*/2, /*ticket_base=*/1u);
        else
            load_stats_v2_kernel<8><<<1, LS_THREADS, smem, st>>>(
                nullptr, 0, 1, 8, nullptr, 8, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, 0, 0, ctl,
                reinterpret_cast<uint32_t*>(w + L.agg), /*nblk=*/2, /*block_base=*/1, nullptr);
        moe_host::note_launch();
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        ScanCtl h;
        if ((e = cudaMemcpyAsync(&h, ctl, sizeof(h), cudaMemcpyDeviceToHost, st)) != cudaSuccess) return e;
        if ((e = cudaStreamSynchronize(st)) != cudaSuccess) return e;
        // the look-back probe's block is also the last to finish (it folds err
        // into sticky); the other probe's finished count stops short of 2
        bits &= h.err | h.sticky;
        // leave the workspace as a finished call does: counters zero, next
        // epoch (the probe's own flags become stale), error words cleared
        ScanCtl z;
        memset(&z, 0, sizeof(z));
        z.epoch = h.epoch + 1;
        if ((e = cudaMemcpyAsync(ctl, &z, sizeof(z), cudaMemcpyHostToDevice, st)) != cudaSuccess) return e;
        // no flag of the probe outlives it (its block published one)
        if ((e = cudaMemsetAsync(w + L.flags, 0, sizeof(uint32_t) * (size_t)L.nblk, st)) != cudaSuccess) return e;
        if ((e = cudaStreamSynchronize(st)) != cudaSuccess) return e;
    }
    *err_out = bits;
    return cudaSuccess;
}

cudaError_t launch_replica_plan(const int32_t* counts, int N, int R, int32_t* replica_slot, cudaStream_t st) {
    replica_plan_kernel<<<1, 1024, sizeof(int32_t) * (size_t)N, st>>>(counts, N, R, replica_slot);
    moe_host::note_launch();
    return cudaGetLastError();
}

cudaError_t launch_bias_update_ema(const int32_t* counts, int N, int64_t total, float u, float alpha, float* ema,
                                   float* bias, cudaStream_t st) {
    bias_update_ema_kernel<<<1, 1024, 0, st>>>(counts, N, total, u, alpha, ema, bias);
    moe_host::note_launch();
    return cudaGetLastError();
}

cudaError_t launch_route_balanced(int64_t T, int K, int N, float scale, int32_t* idx, float* w, cudaStream_t st) {
    const int64_t A = T * K;
    long long blocks = (A + 255) / 256;
    const long long cap = (long long)moe_host::sm_count() * 16;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    route_balanced_kernel<<<(unsigned)blocks, 256, 0, st>>>(A, K, N, scale / (float)K, idx, w);
    moe_host::note_launch();
    return cudaGetLastError();
}

cudaError_t launch_bias_update(const int32_t* counts, int N, int64_t total, float u, int mode, float* bias,
                               cudaStream_t st) {
    bias_update_kernel<<<1, 1024, 0, st>>>(counts, N, total, u, mode, bias);
    moe_host::note_launch();
    return cudaGetLastError();
}

}  // namespace moe
