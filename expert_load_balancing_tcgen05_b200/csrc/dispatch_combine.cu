// Dispatch (token rows -> expert-contiguous buffer, optional FP8 e4m3 copy
// with one fp32 scale per row and 128-channel block) and combine (weighted
// gather-sum back to token order).  "DeepSeek V4 MoE load balancing", DeepEP
// section: dispatch sends each token to its experts, combine brings the
// results back; FP8 on dispatch, BF16 on combine.
//
// Both are pure HBM streams.  One warp owns one token: it reads the token's
// row once with 16-byte vector loads and writes it K times (dispatch), or
// reads K expert rows and writes one (combine).  Every warp-wide access is a
// contiguous 512-byte span, so HBM sees full lines; the row destinations
// come from pos = offsets[slot] + rank, computed once per token by K lanes.
// An assignment dropped by the capacity limit (slot < 0) has pos -1 and no
// row of its own (dispatch parks its copy in the unused last row of the
// buffer); combine skips it.
#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include "common.cuh"

namespace moe {

constexpr int DC_THREADS = 256;
constexpr int DC_WARPS = DC_THREADS / 32;
// combine runs 4-warp blocks: finer blocks spread its warps evenly over the SMs
// (at 4096 tokens, 8-warp blocks land 3 or 4 per SM)
constexpr int CB_THREADS = 128;
constexpr int CB_WARPS = CB_THREADS / 32;

__device__ __forceinline__ void ld_vec(const void* p, uint4& v) {
    v = __ldg(reinterpret_cast<const uint4*>(p));
}

// streaming store: the dispatch buffer is not re-read by this kernel
__device__ __forceinline__ void st_vec(void* p, const uint4& v) {
    __stcs(reinterpret_cast<uint4*>(p), v);
}

__device__ __forceinline__ void unpack(const uint4& v, float (&f)[8]) {  // bf16 x 8
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        float2 t = __bfloat1622float2(h[i]);
        f[2 * i] = t.x;
        f[2 * i + 1] = t.y;
    }
}

__device__ __forceinline__ void unpack(const uint4& v, float (&f)[4]) {  // fp32 x 4
    f[0] = __uint_as_float(v.x); f[1] = __uint_as_float(v.y);
    f[2] = __uint_as_float(v.z); f[3] = __uint_as_float(v.w);
}

// e4m3 with round-to-nearest-even and saturation to +-448 (cvt.rn.satfinite)
__device__ __forceinline__ uint16_t to_e4m3x2(float a, float b) {
    __nv_fp8x2_storage_t r = __nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3);
    return (uint16_t)r;
}

// EPV: elements per 16-byte vector (8 bf16, 4 fp32).  VPB = vectors per
// 128-channel block (16 or 32 lanes).  KMAX >= K bounds the fully unrolled
// destination loop so the K row positions live in registers.
template <int EPV, bool FP8, int KMAX>
__global__ void __launch_bounds__(DC_THREADS) dispatch_kernel(
    const char* __restrict__ x, int64_t T, int d, int K, const int32_t* __restrict__ slot_idx,
    const int32_t* __restrict__ offsets, const int32_t* __restrict__ rank, char* __restrict__ rows,
    uint8_t* __restrict__ rows_fp8, float* __restrict__ scales, int32_t* __restrict__ pos_out,
    int32_t* __restrict__ row_src) {
    constexpr int VPB = 128 / EPV;
    const int lane = threadIdx.x & 31;
    const int64_t row_bytes = (int64_t)d * (16 / EPV);
    const int nvec = d / EPV;
    const int nblk128 = d / 128;
    for (int64_t t = (int64_t)blockIdx.x * DC_WARPS + (threadIdx.x >> 5); t < T;
         t += (int64_t)gridDim.x * DC_WARPS) {
        int my_pos = 0;
        if (lane < K) {
            const int64_t a = t * K + lane;
            const int sl = __ldg(slot_idx + a);
            const int q = sl >= 0 ? __ldg(offsets + sl) + __ldg(rank + a) : -1;
            if (pos_out) pos_out[a] = q;
            if (row_src && q >= 0) row_src[q] = (int32_t)t;
            // a dropped assignment's copy goes to the last row, which is past
            // the kept rows whenever anything was dropped: the store loop
            // stays free of per-row tests
            my_pos = q >= 0 ? q : (int)(T * K - 1);
        }
        int p[KMAX];
#pragma unroll
        for (int k = 0; k < KMAX; ++k) p[k] = __shfl_sync(FULL, my_pos, k);
        const char* src = x + t * row_bytes;
        // 4 vectors per lane in flight per step
        for (int v0 = 0; v0 < nvec; v0 += 32 * 4) {
            uint4 val[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int v = v0 + u * 32 + lane;
                if (v < nvec) ld_vec(src + (int64_t)v * 16, val[u]);
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int v = v0 + u * 32 + lane;
                if (rows != nullptr && v < nvec) {
#pragma unroll
                    for (int k = 0; k < KMAX; ++k) {
                        if (k >= K) break;
                        st_vec(rows + (int64_t)p[k] * row_bytes + (int64_t)v * 16, val[u]);
                    }
                }
                if constexpr (FP8) {
                    // the whole warp takes part in the shuffles; lanes past the row idle
                    float f[EPV];
                    if (v < nvec) unpack(val[u], f);
                    else {
#pragma unroll
                        for (int i = 0; i < EPV; ++i) f[i] = 0.f;
                    }
                    float amax = 0.f;
#pragma unroll
                    for (int i = 0; i < EPV; ++i) amax = fmaxf(amax, fabsf(f[i]));
#pragma unroll
                    for (int o = VPB / 2; o >= 1; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(FULL, amax, o));
                    if (v < nvec) {
                        const float inv = amax > 0.f ? __fdiv_rn(448.f, amax) : 0.f;
                        uint16_t q[EPV / 2];
#pragma unroll
                        for (int i = 0; i < EPV / 2; ++i)
                            q[i] = to_e4m3x2(__fmul_rn(f[2 * i], inv), __fmul_rn(f[2 * i + 1], inv));
                        const float sc = __fdiv_rn(amax, 448.f);
                        const int blk = v / VPB;
#pragma unroll
                        for (int k = 0; k < KMAX; ++k) {
                            if (k >= K) break;
                            uint8_t* dst = rows_fp8 + (int64_t)p[k] * d + (int64_t)v * EPV;
                            if constexpr (EPV == 8) {
                                uint2 pk = make_uint2((uint32_t)q[0] | ((uint32_t)q[1] << 16),
                                                      (uint32_t)q[2] | ((uint32_t)q[3] << 16));
                                __stcs(reinterpret_cast<uint2*>(dst), pk);
                            } else {
                                __stcs(reinterpret_cast<uint32_t*>(dst), (uint32_t)q[0] | ((uint32_t)q[1] << 16));
                            }
                            if ((lane % VPB) == 0) scales[(int64_t)p[k] * nblk128 + blk] = sc;
                        }
                    }
                }
            }
        }
    }
}

template <int EPV>
__global__ void __launch_bounds__(CB_THREADS) combine_kernel(const char* __restrict__ y, int64_t T, int d,
                                                             int K, const int32_t* __restrict__ pos,
                                                             const float* __restrict__ w,
                                                             char* __restrict__ out) {
    __shared__ int s_pos[CB_WARPS][32];
    __shared__ float s_w[CB_WARPS][32];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t row_bytes = (int64_t)d * (16 / EPV);
    const int nvec = d / EPV;
    for (int64_t t = (int64_t)blockIdx.x * CB_WARPS + warp; t < T; t += (int64_t)gridDim.x * CB_WARPS) {
        int my_pos = -1;
        float my_w = 0.f;
        if (lane < K) {
            my_pos = __ldg(pos + t * K + lane);
            my_w = __ldg(w + t * K + lane);
        }
        // the token's kept assignments (pos >= 0; dropped ones have no row)
        // moved to the front in k order, so the sum runs over them alone
        const unsigned live = __ballot_sync(FULL, my_pos >= 0);
        const int Kl = __popc(live);
        if (live != ((K >= 32) ? FULL : ((1u << K) - 1u))) {
            if (my_pos >= 0) {
                const int r = __popc(live & lanemask_lt());
                s_pos[warp][r] = my_pos;
                s_w[warp][r] = my_w;
            }
            __syncwarp();
            my_pos = lane < Kl ? s_pos[warp][lane] : 0;
            my_w = lane < Kl ? s_w[warp][lane] : 0.f;
            __syncwarp();
        }
        for (int v0 = 0; v0 < nvec; v0 += 64) {
            float acc[2][EPV];
#pragma unroll
            for (int u = 0; u < 2; ++u)
#pragma unroll
                for (int i = 0; i < EPV; ++i) acc[u][i] = 0.f;
            for (int k0 = 0; k0 < Kl; k0 += 4) {
                uint4 val[4][2];
                float wk[4];
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    const int k = k0 + kk;
                    const int pk = __shfl_sync(FULL, my_pos, k & 31);
                    wk[kk] = __shfl_sync(FULL, my_w, k & 31);
#pragma unroll
                    for (int u = 0; u < 2; ++u) {
                        const int v = v0 + u * 32 + lane;
                        if (k < Kl && v < nvec) ld_vec(y + (int64_t)pk * row_bytes + (int64_t)v * 16, val[kk][u]);
                    }
                }
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    if (k0 + kk >= Kl) break;
#pragma unroll
                    for (int u = 0; u < 2; ++u) {
                        const int v = v0 + u * 32 + lane;
                        if (v < nvec) {
                            float f[EPV];
                            unpack(val[kk][u], f);
#pragma unroll
                            for (int i = 0; i < EPV; ++i) acc[u][i] = __fmaf_rn(wk[kk], f[i], acc[u][i]);
                        }
                    }
                }
            }
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const int v = v0 + u * 32 + lane;
                if (v >= nvec) continue;
                uint4 o;
                if constexpr (EPV == 8) {
                    __nv_bfloat162 h[4];
#pragma unroll
                    for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(acc[u][2 * i], acc[u][2 * i + 1]);
                    o = *reinterpret_cast<uint4*>(h);
                } else {
                    o = make_uint4(__float_as_uint(acc[u][0]), __float_as_uint(acc[u][1]),
                                   __float_as_uint(acc[u][2]), __float_as_uint(acc[u][3]));
                }
                st_vec(out + t * row_bytes + (int64_t)v * 16, o);
            }
        }
    }
}

// one warp per token; grid capped at 64 blocks per SM (grid-stride beyond)
static unsigned token_blocks(int64_t T, int warps_per_block) {
    long long b = (T + warps_per_block - 1) / warps_per_block;
    const long long cap = (long long)moe_host::sm_count() * 64;
    if (b > cap) b = cap;
    if (b < 1) b = 1;
    return (unsigned)b;
}

cudaError_t launch_dispatch(const void* x, int dtype, int64_t T, int d, int K, const int32_t* slot_idx,
                            const int32_t* offsets, const int32_t* rank, void* rows, uint8_t* rows_fp8,
                            float* scales, int32_t* pos, int32_t* row_src, cudaStream_t st) {
    const unsigned nb = token_blocks(T, DC_WARPS);
    const char* xc = static_cast<const char*>(x);
    char* rc = static_cast<char*>(rows);
    const bool fp8 = rows_fp8 != nullptr;
#define MOE_DISPATCH(EPV, F8, KM)                                                              \
    dispatch_kernel<EPV, F8, KM><<<nb, DC_THREADS, 0, st>>>(xc, T, d, K, slot_idx, offsets, rank, rc, \
                                                            rows_fp8, scales, pos, row_src)
    const bool small_k = K <= 8;
    if (dtype == MOE_BF16) {
        if (fp8) { if (small_k) MOE_DISPATCH(8, true, 8); else MOE_DISPATCH(8, true, 32); }
        else     { if (small_k) MOE_DISPATCH(8, false, 8); else MOE_DISPATCH(8, false, 32); }
    } else {
        if (fp8) { if (small_k) MOE_DISPATCH(4, true, 8); else MOE_DISPATCH(4, true, 32); }
        else     { if (small_k) MOE_DISPATCH(4, false, 8); else MOE_DISPATCH(4, false, 32); }
    }
#undef MOE_DISPATCH
    moe_host::note_launch();
    return cudaGetLastError();
}

cudaError_t launch_combine(const void* y, int dtype, int64_t T, int d, int K, const int32_t* pos,
                           const float* w, void* out, cudaStream_t st) {
    const unsigned nb = token_blocks(T, CB_WARPS);
    if (dtype == MOE_BF16)
        combine_kernel<8><<<nb, CB_THREADS, 0, st>>>(static_cast<const char*>(y), T, d, K, pos, w,
                                                     static_cast<char*>(out));
    else
        combine_kernel<4><<<nb, CB_THREADS, 0, st>>>(static_cast<const char*>(y), T, d, K, pos, w,
                                                     static_cast<char*>(out));
    moe_host::note_launch();
    return cudaGetLastError();
}

}  // namespace moe
