// Capacity-limited routing ("MoE Routing Entropy vs Expert Saturation",
// section "Production Testing": a hard token capacity per expert of
// 1.25 * T*K/N; the excess goes to secondary candidate experts ranked by the
// bias-adjusted key).
//
//   1. capacity_candidates_kernel: each token's 2K best kept experts; the
//      first K are the plain selection, the next K its secondaries;
//   2. load statistics of the primaries: stable in-expert ranks in flat
//      (t, k) order and counts c1; a primary is kept iff its rank < C;
//   3. capacity_reroute_kernel: token t's j-th overflowed slot (k order)
//      points at secondary j;
//   4. load statistics of the reroutes alone (every other slot marked -1):
//      their stable ranks per expert, again in flat order;
//   5. capacity_finalize_kernel: a reroute is kept iff its rank is below the
//      room its expert has left, C - min(c1, C); the rest are dropped (index
//      -1, weight 0); weights are recomputed from the unbiased scores of the
//      token's kept experts.
// Ranks from a stable scan make every decision equal to the sequential walk
// over the assignments in flat order, with no atomics deciding anything.
#include "common.cuh"

namespace moe {

cudaError_t launch_capacity_candidates(const float* scores, const float* bias, int T, int N, int K, int n_groups,
                                       int topk_groups, int group_topn, int32_t* idx, int32_t* second,
                                       long long* info, long long capacity, cudaStream_t st);
cudaError_t launch_load_stats(const int32_t* idx, int64_t T, int K, int N, const int32_t* replica_slot,
                              int n_slots, int32_t* slot_idx, int32_t* counts, int32_t* offsets,
                              int32_t* rank, const float* scores, int score_fn, moe_stats* stats,
                              void* ws, cudaStream_t st, const int32_t* tile_counts = nullptr);

constexpr int CAP_THREADS = 256;
constexpr int CAP_KMAX = 16;

__device__ __forceinline__ long long block_sum_ll(long long v, long long* sm /*[CAP_THREADS/32]*/) {
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(FULL, v, o);
    if ((threadIdx.x & 31) == 0) sm[threadIdx.x >> 5] = v;
    __syncthreads();
    long long r = 0;
    if (threadIdx.x == 0)
        for (int w = 0; w < CAP_THREADS / 32; ++w) r += sm[w];
    return r;
}

// one thread per token: overflowed primaries (rank >= C) take the token's
// secondaries in order
__global__ void __launch_bounds__(CAP_THREADS) capacity_reroute_kernel(const int32_t* __restrict__ rank1,
                                                                       const int32_t* __restrict__ second,
                                                                       int64_t T, int K, long long C,
                                                                       int32_t* __restrict__ re_idx,
                                                                       long long* __restrict__ info) {
    __shared__ long long sm[CAP_THREADS / 32];
    long long over = 0;
    for (int64_t t0 = (int64_t)blockIdx.x * CAP_THREADS; t0 < T; t0 += (int64_t)gridDim.x * CAP_THREADS) {
        const int64_t t = t0 + threadIdx.x;
        if (t < T) {
            int j = 0;
            for (int k = 0; k < K; ++k) {
                const int64_t a = t * K + k;
                int32_t e2 = -1;
                if (rank1[a] >= C) {
                    e2 = second[t * K + j];
                    ++j;
                    ++over;
                }
                re_idx[a] = e2;
            }
        }
    }
    const long long tot = block_sum_ll(over, sm);
    if (threadIdx.x == 0 && tot != 0) atomicAdd(reinterpret_cast<unsigned long long*>(info + 1),
                                                 (unsigned long long)tot);
}

__global__ void __launch_bounds__(CAP_THREADS) capacity_finalize_kernel(
    const float* __restrict__ scores, int N, const int32_t* __restrict__ rank1, const int32_t* __restrict__ re_idx,
    const int32_t* __restrict__ rank2, const int32_t* __restrict__ counts1, int64_t T, int K, long long C,
    int renorm, float route_scale, int32_t* __restrict__ idx, float* __restrict__ w, long long* __restrict__ info) {
    __shared__ long long sm[CAP_THREADS / 32];
    long long rer = 0, drop = 0;
    for (int64_t t0 = (int64_t)blockIdx.x * CAP_THREADS; t0 < T; t0 += (int64_t)gridDim.x * CAP_THREADS) {
        const int64_t t = t0 + threadIdx.x;
        if (t >= T) continue;
        int fin[CAP_KMAX];
        float sv[CAP_KMAX];
        float ssum = 0.f;
        bool first = true;
#pragma unroll
        for (int k = 0; k < CAP_KMAX; ++k) {
            if (k >= K) break;
            const int64_t a = t * K + k;
            int e = idx[a];
            if (rank1[a] >= C) {
                const int e2 = re_idx[a];
                e = -1;
                if (e2 >= 0) {
                    const long long room = C - (long long)min((long long)counts1[e2], C);
                    if ((long long)rank2[a] < room) e = e2;
                }
                if (e >= 0) ++rer;
                else ++drop;
            }
            fin[k] = e;
            sv[k] = e >= 0 ? __ldg(scores + t * N + e) : 0.f;
            if (e >= 0) {
                ssum = first ? sv[k] : __fadd_rn(ssum, sv[k]);
                first = false;
            }
        }
#pragma unroll
        for (int k = 0; k < CAP_KMAX; ++k) {
            if (k >= K) break;
            const int64_t a = t * K + k;
            idx[a] = fin[k];
            float v = 0.f;
            if (fin[k] >= 0) v = __fmul_rn(renorm ? __fdiv_rn(sv[k], ssum) : sv[k], route_scale);
            w[a] = v;
        }
    }
    const long long r = block_sum_ll(rer, sm);
    __syncthreads();
    const long long d = block_sum_ll(drop, sm);
    if (threadIdx.x == 0) {
        if (r != 0) atomicAdd(reinterpret_cast<unsigned long long*>(info + 2), (unsigned long long)r);
        if (d != 0) atomicAdd(reinterpret_cast<unsigned long long*>(info + 3), (unsigned long long)d);
    }
}

// Workspace: the load-statistics workspace, then second, rank1, re_idx and
// rank2 ([T*K] int32 each), then counts1, counts2 and offsets ([N+1] int32
// each).  Regions 256-byte aligned.
struct CapLayout {
    size_t ls = 0, second = 0, rank1 = 0, re_idx = 0, rank2 = 0, c1 = 0, c2 = 0, off = 0, total = 0;
};

inline CapLayout cap_layout(int64_t T, int K, int N) {
    CapLayout L;
    const size_t tk = align256(sizeof(int32_t) * (size_t)T * (size_t)K);
    const size_t nn = align256(sizeof(int32_t) * ((size_t)N + 1));
    size_t off = align256(ws_layout(T, K, N, N).total);
    L.second = off; off += tk;
    L.rank1 = off;  off += tk;
    L.re_idx = off; off += tk;
    L.rank2 = off;  off += tk;
    L.c1 = off;     off += nn;
    L.c2 = off;     off += nn;
    L.off = off;    off += nn;
    L.total = off;
    return L;
}

size_t capacity_workspace_bytes(int64_t T, int K, int N) { return cap_layout(T, K, N).total; }

static unsigned cap_blocks(int64_t T) {
    long long b = (T + CAP_THREADS - 1) / CAP_THREADS;
    const long long cap = (long long)moe_host::sm_count() * 8;
    if (b > cap) b = cap;
    if (b < 1) b = 1;
    return (unsigned)b;
}

cudaError_t launch_route_capacity(const float* scores, const float* bias, int T, int N, int K, int n_groups,
                                  int topk_groups, int group_topn, int renorm, float route_scale, long long C,
                                  int32_t* idx, float* w, long long* info, void* ws, cudaStream_t st) {
    const CapLayout L = cap_layout(T, K, N);
    char* b = static_cast<char*>(ws);
    int32_t* second = reinterpret_cast<int32_t*>(b + L.second);
    int32_t* rank1 = reinterpret_cast<int32_t*>(b + L.rank1);
    int32_t* re_idx = reinterpret_cast<int32_t*>(b + L.re_idx);
    int32_t* rank2 = reinterpret_cast<int32_t*>(b + L.rank2);
    int32_t* c1 = reinterpret_cast<int32_t*>(b + L.c1);
    int32_t* c2 = reinterpret_cast<int32_t*>(b + L.c2);
    int32_t* offs = reinterpret_cast<int32_t*>(b + L.off);
    cudaError_t e = launch_capacity_candidates(scores, bias, T, N, K, n_groups, topk_groups, group_topn, idx,
                                               second, info, C, st);
    if (e != cudaSuccess || T == 0) return e;
    if ((e = launch_load_stats(idx, T, K, N, nullptr, N, nullptr, c1, offs, rank1, nullptr, 0, nullptr, ws, st)) !=
        cudaSuccess)
        return e;
    const unsigned nb = cap_blocks(T);
    capacity_reroute_kernel<<<nb, CAP_THREADS, 0, st>>>(rank1, second, T, K, C, re_idx, info);
    moe_host::note_launch();
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if ((e = launch_load_stats(re_idx, T, K, N, nullptr, N, nullptr, c2, offs, rank2, nullptr, 0, nullptr, ws,
                               st)) != cudaSuccess)
        return e;
    capacity_finalize_kernel<<<nb, CAP_THREADS, 0, st>>>(scores, N, rank1, re_idx, rank2, c1, T, K, C, renorm,
                                                         route_scale, idx, w, info);
    moe_host::note_launch();
    return cudaGetLastError();
}

}  // namespace moe
