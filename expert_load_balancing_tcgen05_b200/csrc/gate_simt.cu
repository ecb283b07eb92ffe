// Gate logits and scores on CUDA cores, for fp32 inputs (and for bf16
// expert counts the tensor-core kernel has no tile for).
//
// h[t,e] = sum_j x[t,j] * W[e,j] + off[e] (+ b[e] when the bias joins the
// logits) ("MoE Routing Entropy vs Expert
// Saturation", section "The Mathematics": h = x . W_g with the nn.Linear gate
// of section "Concrete Implementation"); then softmax over the experts (same
// section) or sigmoid ("DeepSeek V4 MoE load balancing", token routing).
//
// One warp per token: the lanes stride over the hidden dimension for each
// expert (coalesced reads of x and W rows), a shuffle butterfly completes the
// dot product, lane e%32 keeps h_e, and the nonlinearity is a warp
// reduction.  fp32 accumulation.
#include <cuda_bf16.h>
#include <math.h>

#include "common.cuh"

namespace moe {

template <typename TIn>
__device__ __forceinline__ float to_f(TIn v);
template <>
__device__ __forceinline__ float to_f<float>(float v) { return v; }
template <>
__device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 v) { return __bfloat162float(v); }

template <typename TIn>
__global__ void __launch_bounds__(256) gate_simt_kernel(const TIn* __restrict__ x, const TIn* __restrict__ W,
                                                        const float* __restrict__ off,
                                                        const float* __restrict__ logit_bias, int T, int d, int N,
                                                        int fn, float* __restrict__ scores) {
    const int lane = threadIdx.x & 31;
    const int wpb = blockDim.x >> 5;
    for (int t = blockIdx.x * wpb + (threadIdx.x >> 5); t < T; t += gridDim.x * wpb) {
        const TIn* xr = x + (size_t)t * d;
        float h[MAX_N / 32];
#pragma unroll
        for (int i = 0; i < MAX_N / 32; ++i) h[i] = -INFINITY;
        for (int e = 0; e < N; ++e) {
            const TIn* wr = W + (size_t)e * d;
            float acc = 0.f;
            for (int j = lane; j < d; j += 32) acc = fmaf(to_f(xr[j]), to_f(wr[j]), acc);
#pragma unroll
            for (int o = 16; o >= 1; o >>= 1) acc += __shfl_xor_sync(FULL, acc, o);
            if (off != nullptr) acc += off[e];
            if (logit_bias != nullptr) acc += logit_bias[e];
            // lane e%32 keeps h_e in register slot e/32 (unrolled select keeps h in registers)
#pragma unroll
            for (int i = 0; i < MAX_N / 32; ++i)
                if (i == (e >> 5) && lane == (e & 31)) h[i] = acc;
        }
        float* out = scores + (size_t)t * N;
        if (fn == MOE_SIGMOID) {
#pragma unroll
            for (int i = 0; i < MAX_N / 32; ++i) {
                const int e = i * 32 + lane;
                if (e < N) out[e] = 1.f / (1.f + expf(-h[i]));
            }
        } else {
            float m = -INFINITY;
#pragma unroll
            for (int i = 0; i < MAX_N / 32; ++i) if (i * 32 + lane < N) m = fmaxf(m, h[i]);
#pragma unroll
            for (int o = 16; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(FULL, m, o));
            float sum = 0.f;
#pragma unroll
            for (int i = 0; i < MAX_N / 32; ++i) {
                const int e = i * 32 + lane;
                if (e < N) { h[i] = expf(h[i] - m); sum += h[i]; }
            }
#pragma unroll
            for (int o = 16; o >= 1; o >>= 1) sum += __shfl_xor_sync(FULL, sum, o);
            const float inv = 1.f / sum;
#pragma unroll
            for (int i = 0; i < MAX_N / 32; ++i) {
                const int e = i * 32 + lane;
                if (e < N) out[e] = h[i] * inv;
            }
        }
    }
}

cudaError_t launch_gate_simt(const void* x, const void* W, int dtype, const float* off, const float* logit_bias,
                             int T, int d, int N, int fn, float* scores, cudaStream_t st) {
    long long blocks = ((long long)T + 7) / 8;
    const long long cap = (long long)moe_host::sm_count() * 8;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    if (dtype == MOE_F32)
        gate_simt_kernel<float><<<(unsigned)blocks, 256, 0, st>>>(
            static_cast<const float*>(x), static_cast<const float*>(W), off, logit_bias, T, d, N, fn, scores);
    else
        gate_simt_kernel<__nv_bfloat16><<<(unsigned)blocks, 256, 0, st>>>(
            static_cast<const __nv_bfloat16*>(x), static_cast<const __nv_bfloat16*>(W), off, logit_bias, T, d, N,
            fn, scores);
    moe_host::note_launch();
    return cudaGetLastError();
}

}  // namespace moe
