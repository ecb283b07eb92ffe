// Bias-adjusted, group-limited top-K selection and combine weights.
//
// Group-limited routing follows "DeepSeek-V3 Group-Limited Expert Routing"
// (sections 1 and 3: score the groups, keep the best topk_groups, choose the
// top-K among their experts only); the bias joins the affinity for the choice
// only ("DeepSeek V4 MoE load balancing", aux-loss-free section); weights are
// the renormalised unbiased scores ("MoE Routing Entropy vs Expert
// Saturation", section "Concrete Implementation").
//
// One warp per token.  Lane l holds EPL consecutive experts [l*EPL, l*EPL+EPL)
// in registers, so a group of gsize experts spans LPG = gsize/EPL lanes and
// every reduction is a butterfly of shuffles; nothing goes through shared
// memory.  The order (key desc, index asc) is total, so the result is unique.
#include <math.h>

#include "common.cuh"
#include "select.cuh"

namespace moe {

int route_epl(int N);


// Warp-wide argmax over lanes [base, base+width) by (key desc, idx asc);
// `width` a power of two; all lanes of the span end with the winner.
__device__ __forceinline__ void argmax_span(float& k, int& i, int width) {
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) {
        if (off >= width) continue;
        float ok = __shfl_xor_sync(FULL, k, off);
        int oi = __shfl_xor_sync(FULL, i, off);
        if (beats(ok, oi, k, i)) { k = ok; i = oi; }
    }
}

template <int EPL>
__device__ __forceinline__ void load_row(const float* __restrict__ row, int lane, int N, float (&v)[EPL]) {
    const int e0 = lane * EPL;
    if constexpr (EPL % 4 == 0) {
        if (e0 < N) {
#pragma unroll
            for (int q = 0; q < EPL / 4; ++q) {
                float4 f = __ldg(reinterpret_cast<const float4*>(row + e0) + q);
                v[4 * q + 0] = f.x; v[4 * q + 1] = f.y; v[4 * q + 2] = f.z; v[4 * q + 3] = f.w;
            }
        } else {
#pragma unroll
            for (int i = 0; i < EPL; ++i) v[i] = 0.f;
        }
    } else {
#pragma unroll
        for (int i = 0; i < EPL; ++i) v[i] = (e0 + i < N) ? __ldg(row + e0 + i) : 0.f;
    }
}

// Mask of this lane's experts that are candidates: all of them without
// groups; with groups, those of the topk_groups best groups, a group's score
// being the fp32 sum, largest first, of its group_topn largest keys.
template <int EPL>
__device__ __forceinline__ unsigned kept_experts(const float (&key)[EPL], unsigned exist, int lane, int e0,
                                                 int n_groups, int topk_groups, int group_topn, int lpg) {
    if (n_groups <= 1) return exist;
    unsigned left = exist;
    float gsum = 0.f;
    for (int r = 0; r < group_topn; ++r) {
        float bk = -INFINITY;
        int bi = 0x7fffffff;
#pragma unroll
        for (int i = 0; i < EPL; ++i)
            if (((left >> i) & 1u) && beats(key[i], e0 + i, bk, bi)) { bk = key[i]; bi = e0 + i; }
        argmax_span(bk, bi, lpg);
        if (bi >= e0 && bi < e0 + EPL) left &= ~(1u << (bi - e0));
        gsum = (r == 0) ? bk : __fadd_rn(gsum, bk);
    }
    // rank of my group among all groups by (score desc, group asc)
    const int g = lane / lpg;
    int rank = 0;
    for (int h = 0; h < n_groups; ++h) {
        float gh = __shfl_sync(FULL, gsum, h * lpg);
        if (h != g && beats(gh, h, gsum, g)) ++rank;
    }
    return rank < topk_groups ? exist : 0u;
}

template <int EPL>
__global__ void __launch_bounds__(256) route_topk_kernel(
    const float* __restrict__ scores, const float* __restrict__ bias, int T, int N, int K,
    int n_groups, int topk_groups, int group_topn, int lpg, int renorm, float route_scale,
    int32_t* __restrict__ topk_idx, float* __restrict__ topk_w) {
    const int lane = threadIdx.x & 31;
    const int warps_per_block = blockDim.x >> 5;
    const int e0 = lane * EPL;

    // bias for this lane's experts stays in registers across tokens
    float b[EPL];
#pragma unroll
    for (int i = 0; i < EPL; ++i) b[i] = (bias != nullptr && e0 + i < N) ? __ldg(bias + e0 + i) : 0.f;
    unsigned exist = 0;
#pragma unroll
    for (int i = 0; i < EPL; ++i) if (e0 + i < N) exist |= 1u << i;

    for (int t = blockIdx.x * warps_per_block + (threadIdx.x >> 5); t < T;
         t += gridDim.x * warps_per_block) {
        float s[EPL], key[EPL];
        load_row<EPL>(scores + (size_t)t * N, lane, N, s);
#pragma unroll
        for (int i = 0; i < EPL; ++i) key[i] = __fadd_rn(s[i], b[i]);

        unsigned avail = kept_experts<EPL>(key, exist, lane, e0, n_groups, topk_groups, group_topn, lpg);

        // K rounds of warp argmax over the available candidates
        float ssum = 0.f, my_s = 0.f;
        int my_idx = 0;
        for (int k = 0; k < K; ++k) {
            float bk = -INFINITY, bs = 0.f;
            int bi = 0x7fffffff;
#pragma unroll
            for (int i = 0; i < EPL; ++i)
                if (((avail >> i) & 1u) && beats(key[i], e0 + i, bk, bi)) { bk = key[i]; bi = e0 + i; bs = s[i]; }
            float wk = bk;
            int wi = bi;
            argmax_span(wk, wi, 32);
            const int owner = wi / EPL;
            const float ws = __shfl_sync(FULL, bs, owner);
            if (lane == owner) avail &= ~(1u << (wi - e0));
            ssum = (k == 0) ? ws : __fadd_rn(ssum, ws);
            if (lane == k) { my_s = ws; my_idx = wi; }
        }
        if (lane < K) {
            float v = renorm ? __fdiv_rn(my_s, ssum) : my_s;
            topk_idx[(size_t)t * K + lane] = my_idx;
            topk_w[(size_t)t * K + lane] = __fmul_rn(v, route_scale);
        }
    }
}


// Ranked candidates for capacity-limited routing ("MoE Routing Entropy vs
// Expert Saturation", section "Production Testing": the excess goes to
// secondary candidates).  One warp per token, 2K rounds of warp argmax by
// (key desc, index asc) over the kept groups' experts: rounds 0..K-1 are the
// selection (idx, in order), rounds K..2K-1 the secondaries (second, -1 once
// the kept experts run out).  Block 0 also resets the capacity counters.
template <int EPL>
__global__ void __launch_bounds__(256) capacity_candidates_kernel(
    const float* __restrict__ scores, const float* __restrict__ bias, int T, int N, int K, int n_groups,
    int topk_groups, int group_topn, int lpg, int32_t* __restrict__ idx, int32_t* __restrict__ second,
    long long* __restrict__ info, long long capacity) {
    const int lane = threadIdx.x & 31;
    const int warps_per_block = blockDim.x >> 5;
    const int e0 = lane * EPL;
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        info[0] = capacity;
        info[1] = 0;
        info[2] = 0;
        info[3] = 0;
    }
    float b[EPL];
#pragma unroll
    for (int i = 0; i < EPL; ++i) b[i] = (bias != nullptr && e0 + i < N) ? __ldg(bias + e0 + i) : 0.f;
    unsigned exist = 0;
#pragma unroll
    for (int i = 0; i < EPL; ++i) if (e0 + i < N) exist |= 1u << i;

    for (int t = blockIdx.x * warps_per_block + (threadIdx.x >> 5); t < T; t += gridDim.x * warps_per_block) {
        float s[EPL], key[EPL];
        load_row<EPL>(scores + (size_t)t * N, lane, N, s);
#pragma unroll
        for (int i = 0; i < EPL; ++i) key[i] = __fadd_rn(s[i], b[i]);
        unsigned avail = kept_experts<EPL>(key, exist, lane, e0, n_groups, topk_groups, group_topn, lpg);
        int my_idx = -1;
        for (int r = 0; r < 2 * K; ++r) {
            float bk = -INFINITY;
            int bi = 0x7fffffff;
#pragma unroll
            for (int i = 0; i < EPL; ++i)
                if (((avail >> i) & 1u) && beats(key[i], e0 + i, bk, bi)) { bk = key[i]; bi = e0 + i; }
            argmax_span(bk, bi, 32);
            if (bi == 0x7fffffff) break;  // no kept expert left (uniform across the warp)
            if (lane == bi / EPL) avail &= ~(1u << (bi - e0));
            if (lane == r) my_idx = bi;
        }
        if (lane < K) idx[(size_t)t * K + lane] = my_idx;
        else if (lane < 2 * K) second[(size_t)t * K + (lane - K)] = my_idx;
    }
}

cudaError_t launch_capacity_candidates(const float* scores, const float* bias, int T, int N, int K, int n_groups,
                                       int topk_groups, int group_topn, int32_t* idx, int32_t* second,
                                       long long* info, long long capacity, cudaStream_t st) {
    const int epl = route_epl(N);
    const int gsize = N / n_groups;
    const int lpg = n_groups > 1 ? gsize / epl : 32;
    long long blocks = ((long long)T + 7) / 8;
    const long long cap = (long long)moe_host::sm_count() * 8;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
#define MOE_CAND_CASE(E)                                                                               \
    case E:                                                                                            \
        capacity_candidates_kernel<E><<<(unsigned)blocks, 256, 0, st>>>(                               \
            scores, bias, T, N, K, n_groups, topk_groups, group_topn, lpg, idx, second, info, capacity); \
        break;
    switch (epl) {
        MOE_CAND_CASE(1)
        MOE_CAND_CASE(2)
        MOE_CAND_CASE(4)
        MOE_CAND_CASE(8)
        MOE_CAND_CASE(16)
        default: return cudaErrorInvalidValue;
    }
#undef MOE_CAND_CASE
    moe_host::note_launch();
    return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Warp-per-token selection.  Lane l owns experts [l*EPL, l*EPL + EPL)
// (EPL = N/32), so an expert group of 32 spans G = 32/EPL consecutive lanes;
// the lane's bias values live in registers for the whole kernel.
//   1. keys = fp32(s + b); each lane's two largest keys (t1 >= t2);
//   2. with groups: the group's two largest keys by a butterfly over its G
//      lanes, group score fp32(t1 + t2) (or t1), group ranks from the
//      scores of all groups (shuffles); lanes of groups not kept drop out;
//   3. theta = the ceil(K/2)-th largest t2 over the kept lanes (ceil(K/2)
//      rounds of a warp max-reduction, redux.sync, on order-preserving
//      integer images of the keys).  At least ceil(K/2) kept lanes hold two
//      keys >= theta, so at least K kept keys are >= theta and the K best
//      keys are all >= theta;
//   4. the survivors (kept keys >= theta; typically K to K+4) are moved
//      through a per-warp shared list, in expert order, to one per lane;
//   5. K rounds of a warp max-reduction (redux.sync) over the survivors'
//      order-preserving key images pick the choices in (key desc, index asc)
//      order -- among equal keys the lowest lane, which holds the lowest
//      index; lane k takes the k-th choice, and lanes 0..K-1 write the
//      outputs, the weights from the unbiased scores summed in k order.  A
//      token with more than 32 survivors takes K rounds of a warp argmax over
//      its survivors in registers instead.
// The result is the plain definition's: the survivors contain the K best
// kept keys and the ranking is the (key desc, index asc) order.
// ---------------------------------------------------------------------------
constexpr int SW_THREADS = 256;

// order-preserving image of a float key in the unsigned integers (-0 and +0,
// equal as keys, share one image)
__device__ __forceinline__ uint32_t ord_key(float f) {
    const uint32_t u = __float_as_uint(f == 0.f ? 0.f : f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

template <int EPL>
__global__ void __launch_bounds__(SW_THREADS, 3) route_select_warp_kernel(
    const float* __restrict__ scores, const float* __restrict__ bias, int T, int K, int grouped, int topk_groups,
    int group_topn, int renorm, float route_scale, int32_t* __restrict__ topk_idx, float* __restrict__ topk_w) {
    constexpr int N = 32 * EPL;
    constexpr int G = 32 / EPL;  // lanes per group of 32 experts
    __shared__ float l_key[SW_THREADS / 32][32], l_s[SW_THREADS / 32][32];
    __shared__ int l_idx[SW_THREADS / 32][32];
    const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
    const int e0 = lane * EPL;
    float b[EPL];
#pragma unroll
    for (int i = 0; i < EPL; ++i) b[i] = bias != nullptr ? __ldg(bias + e0 + i) : 0.f;
    const int rounds = (K + 1) >> 1;
    const int warps = gridDim.x * (SW_THREADS / 32);

    // the next token's row is loaded while the current one is ranked
    float nv[EPL];
    int64_t t = (int64_t)blockIdx.x * (SW_THREADS / 32) + wib;
    if (t < T) load_row<EPL>(scores + t * N, lane, N, nv);
    for (; t < T; t += warps) {
        float sv[EPL], kv[EPL];
#pragma unroll
        for (int i = 0; i < EPL; ++i) sv[i] = nv[i];
        if (t + warps < T) load_row<EPL>(scores + (t + warps) * N, lane, N, nv);
#pragma unroll
        for (int i = 0; i < EPL; ++i) kv[i] = __fadd_rn(sv[i], b[i]);
        // 1. the lane's two largest keys (a NaN key enters neither)
        float t1 = -INFINITY, t2 = -INFINITY;
#pragma unroll
        for (int i = 0; i < EPL; ++i) {
            t2 = fmaxf(t2, fminf(t1, kv[i]));
            t1 = fmaxf(t1, kv[i]);
        }
        // 2. groups: the group's top two over its lanes, scores, ranks
        bool kept = true;
        if (grouped) {
            float g1 = t1, g2 = t2;
#pragma unroll
            for (int o = 1; o < G; o <<= 1) {
                const float h1 = __shfl_xor_sync(FULL, g1, o), h2 = __shfl_xor_sync(FULL, g2, o);
                const float lo = fminf(g1, h1);
                g1 = fmaxf(g1, h1);
                g2 = fmaxf(lo, fmaxf(g2, h2));
            }
            const float gs = group_topn == 1 ? g1 : __fadd_rn(g1, g2);
            const int g = lane / G;
            int rank = 0;
#pragma unroll
            for (int h = 0; h < EPL; ++h) {  // EPL = number of groups of 32
                const float gh = __shfl_sync(FULL, gs, h * G);
                rank += (h != g && beats(gh, h, gs, g)) ? 1 : 0;
            }
            kept = rank < topk_groups;
        }
        // 3. theta: the ceil(K/2)-th largest t2 over the kept lanes
        uint32_t u2 = kept ? ord_key(t2) : 0u, th_u = 0u;
        for (int r = 0; r < rounds; ++r) {
            th_u = __reduce_max_sync(FULL, u2);
            if (u2 == th_u) u2 = 0u;
        }
        // 4. survivors, compacted in expert order, one per lane.  For a key
        //    that is not NaN, ord_key(k) >= th_u is k >= th_f with th_f the
        //    float whose image th_u is (-inf when no lane had a value left)
        const float th_f = th_u == 0u ? -INFINITY
                                      : __uint_as_float((th_u & 0x80000000u) ? (th_u & 0x7fffffffu) : ~th_u);
        unsigned m = 0;
        if (kept) {
#pragma unroll
            for (int i = 0; i < EPL; ++i) m |= (kv[i] >= th_f ? 1u : 0u) << i;
        }
        const int cnt = __popc(m);
        const int total = __reduce_add_sync(FULL, (unsigned)cnt);
        int my_i = 0;
        float my_s = 0.f;
        if (total <= 32) {
            int off = cnt;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(FULL, off, o);
                if (lane >= o) off += y;
            }
            off -= cnt;
#pragma unroll
            for (int i = 0; i < EPL; ++i) {  // predicated stores, no branches
                if ((m >> i) & 1u) {
                    l_key[wib][off] = kv[i];
                    l_s[wib][off] = sv[i];
                    l_idx[wib][off] = e0 + i;
                }
                off += (int)((m >> i) & 1u);
            }
            __syncwarp();
            const bool has = lane < total;
            uint32_t uk = has ? ord_key(l_key[wib][lane]) : 0u;
            const int ci = has ? l_idx[wib][lane] : 0;
            const float cs = has ? l_s[wib][lane] : 0.f;
            __syncwarp();
            // 5. K rounds: the largest key; among equal keys the lowest lane,
            //    which holds the lowest index (the list is in expert order)
            int winner_k = 0;
            for (int k = 0; k < K; ++k) {
                const uint32_t mx = __reduce_max_sync(FULL, uk);
                const unsigned tie = __ballot_sync(FULL, uk == mx && has);
                const int w = __ffs(tie) - 1;
                if (lane == w) uk = 0u;
                if (lane == k) winner_k = w;
            }
            my_i = __shfl_sync(FULL, ci, winner_k);
            my_s = __shfl_sync(FULL, cs, winner_k);
        } else {
            // more survivors than lanes: K rounds of a warp argmax over them
            for (int k = 0; k < K; ++k) {
                float bk = -INFINITY, bs = 0.f;
                int bi = 0x7fffffff;
#pragma unroll
                for (int i = 0; i < EPL; ++i)
                    if (((m >> i) & 1u) && beats(kv[i], e0 + i, bk, bi)) { bk = kv[i]; bi = e0 + i; bs = sv[i]; }
                float wk = bk;
                int wi = bi;
                argmax_span(wk, wi, 32);
                const int owner = wi / EPL;
                const float ws = __shfl_sync(FULL, bs, owner);
                if (lane == owner) m &= ~(1u << (wi - e0));
                if (lane == k) { my_i = wi; my_s = ws; }
            }
        }
        // outputs: lane k holds the k-th choice; weights from the unbiased
        // scores summed in k order
        float sk[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) sk[k] = __shfl_sync(FULL, my_s, k);
        float ssum = sk[0];
#pragma unroll
        for (int k = 1; k < 8; ++k)
            if (k < K) ssum = __fadd_rn(ssum, sk[k]);
        if (lane < K) {
            const float wv = renorm ? __fdiv_rn(my_s, ssum) : my_s;
            topk_idx[t * K + lane] = my_i;
            topk_w[t * K + lane] = __fmul_rn(wv, route_scale);
        }
    }
}

// Elements per lane for N experts; 0 if unsupported.
int route_epl(int N) {
    if (N <= 32) return 1;
    if (N == 64) return 2;
    if (N == 128) return 4;
    if (N == 256) return 8;
    if (N == 512) return 16;
    return 0;
}

// The warp-per-token kernel covers N in {64, 128, 256, 512}, K <= 8, and
// either one group or groups of exactly 32 experts with a group score of the
// top one or two keys.
static bool select_warp_ok(int N, int K, int n_groups, int group_topn) {
    if (!(N == 64 || N == 128 || N == 256 || N == 512) || K > 8) return false;
    return n_groups == 1 || (N / n_groups == 32 && group_topn >= 1 && group_topn <= 2);
}

cudaError_t launch_route_topk(const float* scores, const float* bias, int T, int N, int K,
                              int n_groups, int topk_groups, int group_topn, int renorm,
                              float route_scale, int32_t* idx, float* w, cudaStream_t st) {
    if (select_warp_ok(N, K, n_groups, group_topn)) {
        // one wave of resident blocks (three per SM at this kernel's registers); each warp
        // walks its tokens with the next row's load in flight
        long long blocks = ((long long)T + SW_THREADS / 32 - 1) / (SW_THREADS / 32);
        const long long cap = (long long)moe_host::sm_count() * 3;
        if (blocks > cap) blocks = cap;
        if (blocks < 1) blocks = 1;
        const int grouped = n_groups > 1 ? 1 : 0;
#define MOE_SELW(E)                                                                                            \
    route_select_warp_kernel<E><<<(unsigned)blocks, SW_THREADS, 0, st>>>(scores, bias, T, K, grouped, topk_groups, \
                                                                         group_topn, renorm, route_scale, idx, w)
        switch (N) {
            case 64: MOE_SELW(2); break;
            case 128: MOE_SELW(4); break;
            case 256: MOE_SELW(8); break;
            default: MOE_SELW(16); break;
        }
#undef MOE_SELW
        moe_host::note_launch();
        return cudaGetLastError();
    }
    const int epl = route_epl(N);
    const int gsize = N / n_groups;
    const int lpg = n_groups > 1 ? gsize / epl : 32;
    const int threads = 256;
    const int wpb = threads / 32;
    long long blocks = ((long long)T + wpb - 1) / wpb;
    const long long cap = (long long)moe_host::sm_count() * 8;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
#define MOE_ROUTE_CASE(E)                                                                     \
    case E:                                                                                   \
        route_topk_kernel<E><<<(unsigned)blocks, threads, 0, st>>>(                          \
            scores, bias, T, N, K, n_groups, topk_groups, group_topn, lpg, renorm, route_scale, \
            idx, w);                                                                          \
        break;
    switch (epl) {
        MOE_ROUTE_CASE(1)
        MOE_ROUTE_CASE(2)
        MOE_ROUTE_CASE(4)
        MOE_ROUTE_CASE(8)
        MOE_ROUTE_CASE(16)
        default: return cudaErrorInvalidValue;
    }
#undef MOE_ROUTE_CASE
    moe_host::note_launch();
    return cudaGetLastError();
}

}  // namespace moe
