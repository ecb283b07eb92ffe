// Gate GEMM on the 5th-generation tensor cores (tcgen05 + TMEM), fed by TMA,
// with the score nonlinearity fused into the epilogue.
//
//   h[t,e] = sum_j x[t,j] * W[e,j] + off[e]        (bf16 in, fp32 accumulate)
//   s[t,e] = sigmoid(h) | softmax_e(h)             (fp32 out)
//
// "MoE Routing Entropy vs Expert Saturation", section "The Mathematics"
// (h = x . W_g, softmax) with the nn.Linear(hidden, N, bias=False) gate of
// section "Concrete Implementation"; sigmoid gating from "DeepSeek V4 MoE
// load balancing" (token routing section).
//
// Design (one CTA per SM, persistent over 128-token tiles):
//   warp 0      TMA producer: x tile [128 x 64] and the whole W slice
//               [N x 64] per k-step into a STAGES-deep ring of 128B-swizzled
//               shared-memory buffers (no multicast).
//   warp 1      allocates TMEM (2 x N fp32 columns: double-buffered
//               accumulators) and issues tcgen05.mma.cta_group::1.kind::f16
//               M=128, N=BN, K=16 from one elected thread; tcgen05.commit
//               frees ring slots and signals a finished accumulator.
//   warps 2..5  epilogue: tcgen05.ld rows out of TMEM (thread = token row),
//               add the logit offset, apply the nonlinearity (softmax has the
//               whole row in one thread) and store fp32 scores; then release
//               the accumulator so the next tile's MMAs overlap this work.
// Every barrier wait is bounded: on expiry the kernel records the error in
// the workspace, drains its own copies and MMAs, frees TMEM and returns.
#include <cuda.h>
#include <math.h>

#include "common.cuh"

namespace moe {
namespace tc {

constexpr int BM = 128;
constexpr int BK = 64;                 // 64 bf16 = 128 bytes = one swizzle row
constexpr int THREADS = 192;
constexpr uint32_t A_STAGE_BYTES = BM * BK * 2;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// Bounded wait for the phase of `parity` to complete.  False on timeout
// (recorded in the global error word) or, when `watch` is set, as soon as
// another role has given up.
__device__ __noinline__ bool mbar_wait(uint32_t bar, uint32_t parity, int32_t* err, bool watch = true) {
    for (int i = 0; i < 256; ++i)
        if (mbar_try(bar, parity)) return true;
    const uint64_t t0 = globaltimer();
    while (true) {
        if (mbar_try(bar, parity)) return true;
        if (watch && ld_volatile_i32(err) != 0) return false;
        if (globaltimer() - t0 > WAIT_LIMIT_NS) {
            atomicOr(err, 1);
            return false;
        }
    }
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int c0, int c1, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(bar)
        : "memory");
}

// Shared-memory matrix descriptor: K-major operand, 128-byte swizzle,
// 8-row core-matrix groups 1024 bytes apart (SBO), sm_100 descriptor version.
__device__ __forceinline__ uint64_t sdesc(uint32_t saddr) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)1u << 16;                 // leading byte offset (unused for swizzled K-major)
    d |= (uint64_t)(1024u >> 4) << 32;       // stride byte offset
    d |= (uint64_t)1u << 46;                 // descriptor version
    d |= (uint64_t)2u << 61;                 // SWIZZLE_128B
    return d;
}

// Instruction descriptor: bf16 x bf16 -> fp32, both K-major, M=128, N=BN.
template <int BN>
__device__ __forceinline__ constexpr uint32_t idesc() {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);
}

__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t id, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a), "l"(b), "r"(id), "r"(acc)
        : "memory");
}

__device__ __forceinline__ void mma_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                 : "memory");
}

__device__ __forceinline__ void fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
          "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),
          "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),
          "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

template <int BN>
struct Cfg {
    static constexpr int STAGES = BN >= 256 ? 4 : (BN >= 128 ? 6 : 8);
    static constexpr uint32_t B_STAGE_BYTES = BN * BK * 2;
    static constexpr uint32_t STAGE_BYTES = A_STAGE_BYTES + B_STAGE_BYTES;
    static constexpr int TMEM_COLS = 2 * BN;  // 128, 256 or 512: powers of two
    static constexpr size_t SMEM_BYTES =
        1024 /*alignment slack*/ + (size_t)STAGES * STAGE_BYTES + 8 * (2 * STAGES + 5) + 16 + 4 * BN;
};

template <int BN>
__global__ void __launch_bounds__(THREADS, 1) gate_tc_kernel(const __grid_constant__ CUtensorMap tmA,
                                                             const __grid_constant__ CUtensorMap tmB, int T,
                                                             int d, int fn, const float* __restrict__ off,
                                                             float* __restrict__ scores, int32_t* err,
                                                             int num_tiles) {
    using C = Cfg<BN>;
    constexpr int STAGES = C::STAGES;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sA = smem;
    uint8_t* sB = smem + (size_t)STAGES * A_STAGE_BYTES;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + (size_t)STAGES * C::STAGE_BYTES);
    // bars: full[STAGES], empty[STAGES], tfull[2], tempty[2], done
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * STAGES + 5);
    float* off_s = reinterpret_cast<float*>(tmem_slot + 4);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t full0 = smem_u32(bars), empty0 = smem_u32(bars + STAGES);
    const uint32_t tfull0 = smem_u32(bars + 2 * STAGES), tempty0 = smem_u32(bars + 2 * STAGES + 2);
    const uint32_t done_bar = smem_u32(bars + 2 * STAGES + 4);
    const int num_kb = (d + BK - 1) / BK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) { mbar_init(full0 + 8 * s, 1); mbar_init(empty0 + 8 * s, 1); }
        for (int a = 0; a < 2; ++a) { mbar_init(tfull0 + 8 * a, 1); mbar_init(tempty0 + 8 * a, 4); }
        mbar_init(done_bar, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(C::TMEM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    for (int i = threadIdx.x; i < BN; i += blockDim.x) off_s[i] = off != nullptr ? off[i] : 0.f;
    fence_before();
    __syncthreads();
    fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            uint32_t it = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
                for (int kb = 0; kb < num_kb; ++kb, ++it) {
                    const uint32_t s = it % STAGES, ph = (it / STAGES) & 1;
                    if (!mbar_wait(empty0 + 8 * s, ph ^ 1, err)) { ok = false; break; }
                    mbar_expect_tx(full0 + 8 * s, C::STAGE_BYTES);
                    tma_load_2d(smem_u32(sA + (size_t)s * A_STAGE_BYTES), &tmA, kb * BK, tile * BM, full0 + 8 * s);
                    tma_load_2d(smem_u32(sB + (size_t)s * C::B_STAGE_BYTES), &tmB, kb * BK, 0, full0 + 8 * s);
                }
            }
            // drain: the last load issued into each ring slot has landed
            const uint32_t first = it > (uint32_t)STAGES ? it - STAGES : 0;
            for (uint32_t j = first; j < it; ++j) {
                const uint32_t s = j % STAGES, ph = (j / STAGES) & 1;
                if (!mbar_wait(full0 + 8 * s, ph, err, /*watch=*/false)) break;
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            uint32_t it = 0, local = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x, ++local) {
                const uint32_t a = local & 1, aph = (local >> 1) & 1;
                if (!mbar_wait(tempty0 + 8 * a, aph ^ 1, err)) { ok = false; break; }
                fence_after();
                const uint32_t d_tmem = tmem_base + a * BN;
                for (int kb = 0; kb < num_kb; ++kb, ++it) {
                    const uint32_t s = it % STAGES, ph = (it / STAGES) & 1;
                    if (!mbar_wait(full0 + 8 * s, ph, err)) { ok = false; break; }
                    fence_after();
                    const uint32_t a_addr = smem_u32(sA + (size_t)s * A_STAGE_BYTES);
                    const uint32_t b_addr = smem_u32(sB + (size_t)s * C::B_STAGE_BYTES);
#pragma unroll
                    for (int k = 0; k < BK / 16; ++k)
                        mma_bf16(d_tmem, sdesc(a_addr + 32 * k), sdesc(b_addr + 32 * k), idesc<BN>(),
                                 (kb > 0 || k > 0) ? 1u : 0u);
                    mma_commit(empty0 + 8 * s);
                }
                if (ok) mma_commit(tfull0 + 8 * a);
            }
            // drain: every MMA this thread issued has completed
            mma_commit(done_bar);
            mbar_wait(done_bar, 0, err, /*watch=*/false);
        }
    } else {
        // ------------------------------------------------------------ epilogue
        const int q = warp & 3;              // TMEM lane quarter this warp may access
        const int row = q * 32 + lane;
        uint32_t local = 0;
        for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++local) {
            const uint32_t a = local & 1, aph = (local >> 1) & 1;
            // one lane waits, the warp follows its verdict together (tcgen05.ld is warp-collective)
            int ok = 1;
            if (lane == 0) ok = mbar_wait(tfull0 + 8 * a, aph, err) ? 1 : 0;
            ok = __shfl_sync(FULL, ok, 0);
            if (!ok) break;
            fence_after();
            const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + a * BN;
            const int64_t grow = (int64_t)tile * BM + row;
            float* out = scores + grow * BN;
            const bool live = grow < T;
            float v[32];
            if (fn == MOE_SIGMOID) {
#pragma unroll 1
                for (int c0 = 0; c0 < BN; c0 += 32) {
                    tmem_ld32(taddr + c0, v);
#pragma unroll
                    for (int i = 0; i < 32; ++i) v[i] = 1.f / (1.f + expf(-(v[i] + off_s[c0 + i])));
                    if (live) {
#pragma unroll
                        for (int i = 0; i < 32; i += 4)
                            *reinterpret_cast<float4*>(out + c0 + i) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
                    }
                }
            } else {
                float m = -INFINITY;
#pragma unroll 1
                for (int c0 = 0; c0 < BN; c0 += 32) {
                    tmem_ld32(taddr + c0, v);
#pragma unroll
                    for (int i = 0; i < 32; ++i) m = fmaxf(m, v[i] + off_s[c0 + i]);
                }
                float sum = 0.f;
#pragma unroll 1
                for (int c0 = 0; c0 < BN; c0 += 32) {
                    tmem_ld32(taddr + c0, v);
#pragma unroll
                    for (int i = 0; i < 32; ++i) sum += expf(v[i] + off_s[c0 + i] - m);
                }
                const float inv = 1.f / sum;
#pragma unroll 1
                for (int c0 = 0; c0 < BN; c0 += 32) {
                    tmem_ld32(taddr + c0, v);
#pragma unroll
                    for (int i = 0; i < 32; ++i) v[i] = expf(v[i] + off_s[c0 + i] - m) * inv;
                    if (live) {
#pragma unroll
                        for (int i = 0; i < 32; i += 4)
                            *reinterpret_cast<float4*>(out + c0 + i) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
                    }
                }
            }
            fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(tempty0 + 8 * a);
        }
    }

    fence_before();
    __syncthreads();
    fence_after();
    if (warp == 1) {
        __syncwarp();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(C::TMEM_COLS)
                     : "memory");
    }
}

}  // namespace tc

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (fn == nullptr) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

// 2-D bf16 map over a row-major [rows, cols] matrix, box [box_rows, 64], 128B swizzle.
static bool make_map(CUtensorMap* m, const void* base, int64_t rows, int64_t cols, int box_rows) {
    EncodeTiledFn enc = encode_fn();
    if (enc == nullptr) return false;
    cuuint64_t gdim[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t gstride[1] = {(cuuint64_t)cols * 2};
    cuuint32_t box[2] = {(cuuint32_t)tc::BK, (cuuint32_t)box_rows};
    cuuint32_t estride[2] = {1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), gdim, gstride, box, estride,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

bool gate_tc_supported(int N) { return N == 64 || N == 128 || N == 256; }

template <int BN>
static cudaError_t launch_bn(const void* x, const void* W, const float* off, int T, int d, int fn, float* scores,
                             int32_t* err, cudaStream_t st) {
    CUtensorMap ma, mb;
    if (!make_map(&ma, x, T, d, tc::BM) || !make_map(&mb, W, BN, d, BN)) return cudaErrorInvalidValue;
    const size_t smem = tc::Cfg<BN>::SMEM_BYTES;
    cudaError_t e = cudaFuncSetAttribute(tc::gate_tc_kernel<BN>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int num_tiles = (T + tc::BM - 1) / tc::BM;
    int grid = moe_host::sm_count();
    if (grid > num_tiles) grid = num_tiles;
    if (grid < 1) grid = 1;
    tc::gate_tc_kernel<BN><<<grid, tc::THREADS, smem, st>>>(ma, mb, T, d, fn, off, scores, err, num_tiles);
    moe_host::note_launch();
    return cudaGetLastError();
}

cudaError_t launch_gate_tc(const void* x, const void* W, const float* off, int T, int d, int N, int fn,
                           float* scores, int32_t* err, cudaStream_t st) {
    switch (N) {
        case 64: return launch_bn<64>(x, W, off, T, d, fn, scores, err, st);
        case 128: return launch_bn<128>(x, W, off, T, d, fn, scores, err, st);
        case 256: return launch_bn<256>(x, W, off, T, d, fn, scores, err, st);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace moe
