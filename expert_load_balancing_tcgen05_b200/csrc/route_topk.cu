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

namespace moe {

struct Cand {
    float key;
    int idx;
    float s;
};

__device__ __forceinline__ bool beats(float ka, int ia, float kb, int ib) {
    return (ka > kb) || (ka == kb && ia < ib);
}

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

        unsigned avail = exist;
        if (n_groups > 1) {
            // group score: fp32 sum, largest first, of the group's group_topn largest keys
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
            if (rank >= topk_groups) avail = 0;
        }

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

// Elements per lane for N experts; 0 if unsupported.
int route_epl(int N) {
    if (N <= 32) return 1;
    if (N == 64) return 2;
    if (N == 128) return 4;
    if (N == 256) return 8;
    if (N == 512) return 16;
    return 0;
}

cudaError_t launch_route_topk(const float* scores, const float* bias, int T, int N, int K,
                              int n_groups, int topk_groups, int group_topn, int renorm,
                              float route_scale, int32_t* idx, float* w, cudaStream_t st) {
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
