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
// Pipeline (one stream, no host synchronisation):
//   hist_rank     per 4096-assignment block: slot remap, warp-private
//                 shared-memory histograms, stable in-block rank via
//                 __match_any_sync; writes per-block counts expert-major.
//   scan          single-pass decoupled look-back exclusive scan over the
//                 expert-major per-block counts -> every (expert, block) base.
//   finalize      in-expert rank = base - offset + in-block rank; offsets and
//                 counts.
//   score_entropy optional: per-block column sums of normalised scores.
//   stats         one block: moments, entropy, capacities, status.
#include <math.h>

#include "common.cuh"

namespace moe {

// ---------------------------------------------------------------------------
// hist_rank
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(HIST_THREADS) hist_rank_kernel(
    const int32_t* __restrict__ idx, int64_t A, int K, int N, const int32_t* __restrict__ replica_slot,
    int n_slots, int32_t* __restrict__ slot_out, int32_t* __restrict__ rank_out,
    int32_t* __restrict__ blk_counts, int64_t nblk, WsHeader* hdr, uint64_t* scan_status,
    int64_t n_tiles) {
    extern __shared__ int32_t wh[];  // [HIST_WARPS][n_slots]
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t blk = blockIdx.x;

    // this call's scan state starts clean (the scan runs after this kernel)
    if (blk == 0) {
        for (int64_t i = threadIdx.x; i < n_tiles; i += blockDim.x) scan_status[i] = 0;
        if (threadIdx.x == 0) { hdr->scan_ticket = 0; hdr->scan_err = 0; }
    }
    for (int i = threadIdx.x; i < HIST_WARPS * n_slots; i += blockDim.x) wh[i] = 0;
    __syncthreads();

    int32_t* my = wh + warp * n_slots;
    constexpr int CH = HIST_ITEMS_PER_WARP / 32;
    int slot_r[CH], rank_r[CH];
    const int64_t base_a = blk * HIST_BLOCK + (int64_t)warp * HIST_ITEMS_PER_WARP;
#pragma unroll
    for (int j = 0; j < CH; ++j) {
        const int64_t a = base_a + j * 32 + lane;
        int slot = -1;
        if (a < A) {
            int e = __ldg(idx + a);
            if (e < 0 || e >= N) {
                atomicOr(&hdr->scan_err, 2);  // invalid expert id: not counted
            } else {
                slot = e;
                if (replica_slot != nullptr) {
                    const int r = __ldg(replica_slot + e);
                    const int64_t t = a / K;
                    if (r >= 0 && (t & 1)) slot = r;
                    if (slot >= n_slots) { atomicOr(&hdr->scan_err, 2); slot = -1; }
                }
            }
            if (slot_out != nullptr) slot_out[a] = slot;
        }
        const unsigned peers = __match_any_sync(FULL, slot);
        const int before = __popc(peers & lanemask_lt());
        const int seen = (slot >= 0) ? my[slot] : 0;
        __syncwarp();
        if (slot >= 0 && before == 0) my[slot] = seen + __popc(peers);
        __syncwarp();
        slot_r[j] = slot;
        rank_r[j] = seen + before;
    }
    __syncthreads();
    // per slot: exclusive prefix over warps (stable order) and the block total
    for (int e = threadIdx.x; e < n_slots; e += blockDim.x) {
        int run = 0;
#pragma unroll
        for (int w = 0; w < HIST_WARPS; ++w) {
            const int c = wh[w * n_slots + e];
            wh[w * n_slots + e] = run;
            run += c;
        }
        blk_counts[(int64_t)e * nblk + blk] = run;
    }
    __syncthreads();
#pragma unroll
    for (int j = 0; j < CH; ++j) {
        const int64_t a = base_a + j * 32 + lane;
        if (a < A) rank_out[a] = slot_r[j] >= 0 ? rank_r[j] + my[slot_r[j]] : -1;
    }
}

// ---------------------------------------------------------------------------
// Decoupled look-back exclusive scan (single pass).  Tile status words pack
// (flag << 32) | value: flag 1 = tile aggregate, flag 2 = inclusive prefix.
// Tiles are taken from a ticket counter so a tile only ever waits on tiles
// already held by running blocks.
// ---------------------------------------------------------------------------
constexpr uint64_t FLAG_AGG = 1ull << 32, FLAG_PREFIX = 2ull << 32;

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

__global__ void __launch_bounds__(SCAN_THREADS) scan_lookback_kernel(
    const int32_t* __restrict__ in, int32_t* __restrict__ out, int64_t L, uint64_t* status,
    WsHeader* hdr) {
    __shared__ int sm[33];
    __shared__ uint32_t s_tile;
    __shared__ int s_prefix;
    if (threadIdx.x == 0) s_tile = atomicAdd(&hdr->scan_ticket, 1u);
    __syncthreads();
    const int64_t tile = s_tile;
    const int64_t base = tile * SCAN_TILE + (int64_t)threadIdx.x * SCAN_ITEMS;
    int v[SCAN_ITEMS];
    int sum = 0;
#pragma unroll
    for (int i = 0; i < SCAN_ITEMS; ++i) {
        v[i] = (base + i < L) ? __ldg(in + base + i) : 0;
        sum += v[i];
    }
    int total;
    const int excl = block_exclusive_scan(sum, total, sm);
    if (threadIdx.x == 0) {
        int prefix = 0;
        if (tile == 0) {
            st_release_u64(status, FLAG_PREFIX | (uint32_t)total);
        } else {
            st_release_u64(status + tile, FLAG_AGG | (uint32_t)total);
            int64_t p = tile - 1;
            uint64_t t0 = 0;
            bool timed_out = false;
            while (p >= 0) {
                const uint64_t s = ld_acquire_u64(status + p);
                const uint64_t flag = s & (3ull << 32);
                if (flag == 0) {
                    if (t0 == 0) t0 = globaltimer();
                    else if (globaltimer() - t0 > WAIT_LIMIT_NS) { timed_out = true; break; }
                    __nanosleep(64);
                    continue;
                }
                prefix += (int)(uint32_t)s;
                if (flag == FLAG_PREFIX) break;
                --p;
            }
            if (timed_out) atomicOr(&hdr->scan_err, 1);
            // publish even on a timeout so later tiles do not wait in turn
            st_release_u64(status + tile, FLAG_PREFIX | (uint32_t)(prefix + total));
        }
        s_prefix = prefix;
    }
    __syncthreads();
    int run = s_prefix + excl;
#pragma unroll
    for (int i = 0; i < SCAN_ITEMS; ++i) {
        if (base + i < L) out[base + i] = run;
        run += v[i];
    }
}

// ---------------------------------------------------------------------------
// finalize: in-expert rank, offsets, counts
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) finalize_kernel(
    const int32_t* __restrict__ slot_in, const int32_t* __restrict__ idx, const int32_t* __restrict__ replica_slot,
    int K, int64_t A, int n_slots, int64_t nblk, const int32_t* __restrict__ blk_base,
    int32_t* __restrict__ rank, int32_t* __restrict__ offsets, int32_t* __restrict__ counts) {
    if (blockIdx.x == 0) {
        for (int e = threadIdx.x; e <= n_slots; e += blockDim.x) {
            const int off = e < n_slots ? blk_base[(int64_t)e * nblk] : (int)A;
            offsets[e] = off;
            if (e < n_slots) {
                const int nxt = e + 1 < n_slots ? blk_base[(int64_t)(e + 1) * nblk] : (int)A;
                counts[e] = nxt - off;
            }
        }
    }
    for (int64_t a = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; a < A;
         a += (int64_t)gridDim.x * blockDim.x) {
        int slot;
        if (slot_in != nullptr) {
            slot = slot_in[a];
        } else {
            slot = idx[a];
            if (replica_slot != nullptr && slot >= 0) {
                const int r = replica_slot[slot];
                if (r >= 0 && ((a / K) & 1)) slot = r;
            }
        }
        const int r = rank[a];
        if (slot < 0 || slot >= n_slots || r < 0) continue;
        const int64_t blk = a / HIST_BLOCK;
        rank[a] = blk_base[(int64_t)slot * nblk + blk] - blk_base[(int64_t)slot * nblk] + r;
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
// stats: one block
// ---------------------------------------------------------------------------
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

__global__ void __launch_bounds__(1024) stats_kernel(const int32_t* __restrict__ counts, int n_slots,
                                                     const double* __restrict__ partial, int n_part,
                                                     int N, int64_t T, const WsHeader* hdr,
                                                     moe_stats* out) {
    __shared__ double sm[32];
    double tot = 0.0, mx = 0.0;
    for (int e = threadIdx.x; e < n_slots; e += blockDim.x) {
        tot += (double)counts[e];
        mx = fmax(mx, (double)counts[e]);
    }
    tot = block_sum_d(tot, sm);
    mx = block_max_d(mx, sm);
    const double mean = n_slots > 0 ? tot / (double)n_slots : 0.0;
    double var = 0.0, H = 0.0;
    for (int e = threadIdx.x; e < n_slots; e += blockDim.x) {
        const double c = (double)counts[e];
        var += (c - mean) * (c - mean);
        if (c > 0.0) {
            const double p = c / tot;
            H -= p * log2(p);
        }
    }
    var = block_sum_d(var, sm) / (double)(n_slots > 0 ? n_slots : 1);
    H = block_sum_d(H, sm);
    double Hs = NAN;
    if (partial != nullptr) {
        double h = 0.0;
        for (int e = threadIdx.x; e < N; e += blockDim.x) {
            double m = 0.0;
            for (int b = 0; b < n_part; ++b) m += partial[(int64_t)b * N + e];
            m /= (double)T;
            if (m > 0.0) h -= m * log2(m);
        }
        Hs = block_sum_d(h, sm);
    }
    if (threadIdx.x == 0) {
        const int err = hdr->scan_err;
        out->status = err == 0 ? MOE_OK : ((err & 1) ? MOE_ERR_TIMEOUT : MOE_ERR_INVALID);
        out->n_slots = n_slots;
        out->total = (int64_t)tot;
        out->max_load = (int64_t)mx;
        out->mean = mean;
        out->imbalance = mean > 0.0 ? mx / mean : 0.0;
        out->std_over_mean = mean > 0.0 ? sqrt(var) / mean : 0.0;
        out->entropy_load_bits = H;
        out->entropy_score_bits = Hs;
        out->capacity_fixed = mx * (double)n_slots;
        out->capacity_125 = 1.25 * mean;
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

// ---------------------------------------------------------------------------
// host launchers
// ---------------------------------------------------------------------------
cudaError_t launch_load_stats(const int32_t* idx, int64_t T, int K, int N, const int32_t* replica_slot,
                              int n_slots, int32_t* slot_idx, int32_t* counts, int32_t* offsets,
                              int32_t* rank, const float* scores, int score_fn, moe_stats* stats,
                              void* ws, cudaStream_t st) {
    const WsLayout L = ws_layout(T, K, N, n_slots);
    char* w = static_cast<char*>(ws);
    WsHeader* hdr = reinterpret_cast<WsHeader*>(w + L.header);
    int32_t* blk_counts = reinterpret_cast<int32_t*>(w + L.blk_counts);
    int32_t* blk_base = reinterpret_cast<int32_t*>(w + L.blk_base);
    uint64_t* status = reinterpret_cast<uint64_t*>(w + L.scan_status);
    double* partial = reinterpret_cast<double*>(w + L.hs_partial);
    const int64_t A = T * K;

    const size_t hsm = sizeof(int32_t) * HIST_WARPS * (size_t)n_slots;
    cudaError_t e;
    if (hsm > 48 * 1024) {
        e = cudaFuncSetAttribute(hist_rank_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)hsm);
        if (e != cudaSuccess) return e;
    }
    hist_rank_kernel<<<(unsigned)L.nblk, HIST_THREADS, hsm, st>>>(
        idx, A, K, N, replica_slot, n_slots, slot_idx, rank, blk_counts, L.nblk, hdr, status, L.n_tiles);
    moe_host::note_launch();
    if ((e = cudaGetLastError()) != cudaSuccess) return e;

    scan_lookback_kernel<<<(unsigned)L.n_tiles, SCAN_THREADS, 0, st>>>(blk_counts, blk_base, L.L,
                                                                       status, hdr);
    moe_host::note_launch();
    if ((e = cudaGetLastError()) != cudaSuccess) return e;

    long long fb = (A + 255) / 256;
    const long long cap = (long long)moe_host::sm_count() * 8;
    if (fb > cap) fb = cap;
    if (fb < 1) fb = 1;
    finalize_kernel<<<(unsigned)fb, 256, 0, st>>>(slot_idx, idx, replica_slot, K, A, n_slots, L.nblk,
                                                  blk_base, rank, offsets, counts);
    moe_host::note_launch();
    if ((e = cudaGetLastError()) != cudaSuccess) return e;

    if (stats != nullptr) {
        const double* part = nullptr;
        if (scores != nullptr) {
            const size_t csm = sizeof(double) * 8 * (size_t)N;
            if (csm > 48 * 1024) {
                e = cudaFuncSetAttribute(score_colsum_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)csm);
                if (e != cudaSuccess) return e;
            }
            score_colsum_kernel<<<HS_BLOCKS, 256, csm, st>>>(scores, T, N, score_fn, partial);
            moe_host::note_launch();
            if ((e = cudaGetLastError()) != cudaSuccess) return e;
            part = partial;
        }
        stats_kernel<<<1, 1024, 0, st>>>(counts, n_slots, part, HS_BLOCKS, N, T, hdr, stats);
        moe_host::note_launch();
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    return cudaSuccess;
}

cudaError_t launch_replica_plan(const int32_t* counts, int N, int R, int32_t* replica_slot, cudaStream_t st) {
    replica_plan_kernel<<<1, 1024, sizeof(int32_t) * (size_t)N, st>>>(counts, N, R, replica_slot);
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
