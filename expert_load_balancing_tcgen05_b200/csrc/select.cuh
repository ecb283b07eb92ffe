// Device helpers shared by the selection paths (the stand-alone selection
// kernel and the GEMM epilogue): the (key desc, index asc) order, the score
// nonlinearity, and an 8-entry sorted candidate list.
#pragma once

#include <math.h>

#include "common.cuh"

namespace moe {

__device__ __forceinline__ bool beats(float ka, int ia, float kb, int ib) {
    return (ka > kb) || (ka == kb && ia < ib);
}

// The sigmoid used by every path that writes or selects on scores, so the
// written scores are exactly the values selected on.
__device__ __forceinline__ float sigmoid_f(float h) { return __fdividef(1.f, 1.f + __expf(-h)); }

// Sorted (key desc, index asc) list of the 8 best candidates seen so far.
// Candidates must be offered in ascending expert index: an equal key then
// always lands behind the entries already held (they have lower indices).
// The insertion is branch-free: the new entry's place is the number of
// entries that stay ahead of it, and every slot picks its new content from
// (itself, its upper neighbour, the newcomer) independently.
struct Top8 {
    float k[8], s[8];
    int i[8];
    __device__ __forceinline__ void init() {
#pragma unroll
        for (int j = 0; j < 8; ++j) { k[j] = -INFINITY; s[j] = 0.f; i[j] = 0x7fffffff; }
    }
    __device__ __forceinline__ void offer(float key, int e, float sv) {
        int pos = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) pos += (k[j] >= key) ? 1 : 0;
#pragma unroll
        for (int j = 7; j > 0; --j) {
            const bool put = j == pos, shift = j > pos;
            k[j] = put ? key : (shift ? k[j - 1] : k[j]);
            s[j] = put ? sv : (shift ? s[j - 1] : s[j]);
            i[j] = put ? e : (shift ? i[j - 1] : i[j]);
        }
        if (pos == 0) { k[0] = key; s[0] = sv; i[0] = e; }
    }
    // weights from the unbiased scores of the first K entries, sum in k order
    __device__ __forceinline__ void write(int K, int renorm, float scale, int32_t* idx, float* w) const {
        float ssum = s[0];
#pragma unroll
        for (int k = 1; k < 8; ++k)
            if (k < K) ssum = __fadd_rn(ssum, s[k]);
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            if (k < K) {
                const float wv = renorm ? __fdiv_rn(s[k], ssum) : s[k];
                idx[k] = i[k];
                w[k] = __fmul_rn(wv, scale);
            }
        }
    }
};

}  // namespace moe
