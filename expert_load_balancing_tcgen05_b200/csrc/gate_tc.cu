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
//               [N x 64] per k-block into a 192 KB ring of 128B-swizzled
//               shared-memory slots of one or two k-blocks (no multicast).
//   warp 1      allocates TMEM (2 x N fp32 columns: double-buffered
//               accumulators) and issues tcgen05.mma.cta_group::1.kind::f16
//               M=128, N=BN, K=16 from one elected thread; tcgen05.commit
//               frees ring slots and signals a finished accumulator.
//   warps 2..9  epilogue, two warps per TMEM lane quarter, each owning half
//               the columns: tcgen05.ld rows out of TMEM (thread = token
//               row), add the logit offset, apply the nonlinearity (softmax
//               exchanges the halves' max and sum) and store fp32 scores, or
//               select in place; then release the accumulator so the next
//               tile's MMAs overlap this work.
// The N = 256 variant further down runs the same roles on a pair of CTAs.
// Every barrier wait is bounded: on expiry the kernel records the error in
// the workspace, drains its own copies and MMAs, frees TMEM and returns.
#include <cuda.h>
#include <cuda_fp16.h>
#include <math.h>
#include <stdlib.h>

#include "common.cuh"
#include "select.cuh"

namespace moe {
namespace tc {

constexpr int BM = 128;
constexpr int BK = 64;                 // 64 bf16 = 128 bytes = one swizzle row
constexpr int EPI_WARPS = 8;             // two per TMEM lane quarter, each owning half the columns
constexpr int THREADS = 64 + 32 * EPI_WARPS;
constexpr int EPI_THREADS = 32 * EPI_WARPS;
constexpr uint32_t A_KB_BYTES = BM * BK * 2;  // one k-block of the x tile

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

// 8 columns: the fused epilogue's selection loops walk a chunk in these
// pieces so that their (rolled) bodies stay small enough for the instruction
// cache -- each offer into the sorted list unrolls to dozens of instructions
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, float (&v)[8]) {
    uint32_t r[8];
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
                 : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(r[i]);
}

template <int BN>
struct Cfg {
    // a ring slot holds KPS consecutive k-blocks (fewer, larger waits and
    // commits per MMA; the x rows come in 256-byte runs); 192 KB of ring
    static constexpr int KPS = BN >= 256 ? 1 : 2;
    static constexpr int STAGES = (BN >= 256 ? 4 : (BN >= 128 ? 6 : 8)) / KPS;
    static constexpr uint32_t B_KB_BYTES = BN * BK * 2;
    static constexpr uint32_t KB_BYTES = A_KB_BYTES + B_KB_BYTES;
    static constexpr int TMEM_COLS = 2 * BN;  // 128, 256 or 512: powers of two
    // epilogue exchange (per token row): 2 x 2 reduction floats, up to 8 group
    // scores and 8 group second-largest keys, one 8-entry candidate list
    // (key, score, index); the wait verdicts; the tile's expert histogram by
    // token parity (2 x BN counts).  The scores-only epilogue uses the space
    // of the lists, histogram and second-largest keys as its store staging.
    static constexpr size_t XCH_LISTS = (size_t)BM * (3 * 8 + 8) * 4 + 2 * BN * 4;
    static constexpr size_t XCH_STAGE = (size_t)EPI_WARPS * 32 * 20 * 4;
    static constexpr size_t XCH_BYTES = (size_t)BM * (4 + 8) * 4 + 2 * EPI_WARPS * 4 + 16 +
                                        (XCH_LISTS > XCH_STAGE ? XCH_LISTS : XCH_STAGE);
    static constexpr size_t SMEM_BYTES = 1024 /*alignment slack*/ + (size_t)STAGES * KPS * KB_BYTES +
                                         8 * (2 * STAGES + 5) + 16 + 2 * 4 * BN + XCH_BYTES;
};

// Epilogue parameters.  `fused` = select in the epilogue (write topk_idx /
// topk_w directly); otherwise only the scores are written.
struct Epi {
    const float* off;   // [N] logit offsets or null
    const float* bias;  // [N] selection bias or null
    float* scores;      // [T, N] or null (fused only)
    int32_t* idx;       // [T, K]
    float* w;           // [T, K]
    int32_t* tile_counts;  // [ceil(T/128)][2][N] per-tile histogram of the chosen experts by token parity, or null
    int T, fn, K, n_groups, topk_groups, group_topn, renorm, fused;
    int bias_in_logits;  // the bias joins the logit offset; the selection key is the score itself
    float scale;
};

__device__ __forceinline__ void store32(float* dst, const float (&v)[32]) {
#pragma unroll
    for (int i = 0; i < 32; i += 4) *reinterpret_cast<float4*>(dst + i) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
}

__device__ __forceinline__ void store8(float* dst, const float (&v)[8]) {
    *reinterpret_cast<float4*>(dst) = make_float4(v[0], v[1], v[2], v[3]);
    *reinterpret_cast<float4*>(dst + 4) = make_float4(v[4], v[5], v[6], v[7]);
}

// Named barrier over the epilogue warps only.
__device__ __forceinline__ void epi_sync() { asm volatile("bar.sync 1, %0;" ::"n"(EPI_THREADS) : "memory"); }

// Shared-memory exchange between the two warps that own one token row.
struct Xch {
    float* red;   // [2][2][BM]: per half, per round (max, then sum)
    float* gs;    // [BM][8]: group scores
    float* lk;    // [BM][8]: the second half's candidate list
    float* ls;    // [BM][8]
    int* li;      // [BM][8]
    int* agree;   // [2][EPI_WARPS]: per tile parity, each warp's wait verdict
    int* hist;    // [2][BN]: the tile's chosen experts counted by token parity (fused, tile_counts given)
    float* gt2;   // [BM][8]: each group's second-largest key
    float* stage;  // [EPI_WARPS][32][20], 16-byte aligned: scores-only epilogue, aliases lk..gt2
};

// The exchange, carved from shared memory at `base` (4-byte aligned).
template <int BN>
__device__ __forceinline__ Xch carve_xch(float* base) {
    Xch x;
    x.red = base;
    x.gs = x.red + 4 * BM;
    x.agree = reinterpret_cast<int*>(x.gs + 8 * BM);
    float* q = reinterpret_cast<float*>(x.agree + 2 * EPI_WARPS);
    q = reinterpret_cast<float*>((reinterpret_cast<uintptr_t>(q) + 15) & ~uintptr_t(15));
    x.lk = q;
    x.ls = x.lk + 8 * BM;
    x.li = reinterpret_cast<int*>(x.ls + 8 * BM);
    x.hist = x.li + 8 * BM;
    x.gt2 = reinterpret_cast<float*>(x.hist + 2 * BN);
    x.stage = q;
    return x;
}

// One 32-column chunk of scores for the warp's 32 consecutive token rows
// (this lane's row in v), written through the warp's [32][20] staging tile
// 16 columns at a time: each store instruction then writes 64 contiguous
// bytes of 8 rows, not 16 bytes of 32 rows (a quarter of the L2 write
// requests).  Rows at or past T are not written.
template <int BN>
__device__ __forceinline__ void store_chunk_staged(const Epi& p, int64_t grow, int c, const float (&v)[32],
                                                   float* stage, int lane) {
    const int64_t r0 = grow - lane;
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
        float* mine = stage + lane * 20;
#pragma unroll
        for (int q = 0; q < 4; ++q)
            *reinterpret_cast<float4*>(mine + 4 * q) =
                make_float4(v[16 * hh + 4 * q], v[16 * hh + 4 * q + 1], v[16 * hh + 4 * q + 2], v[16 * hh + 4 * q + 3]);
        __syncwarp();
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int r = 8 * i + (lane >> 2), cq = lane & 3;
            const float4 val = *reinterpret_cast<const float4*>(stage + r * 20 + 4 * cq);
            if (r0 + r < (int64_t)p.T)
                *reinterpret_cast<float4*>(p.scores + (r0 + r) * BN + 32 * c + 16 * hh + 4 * cq) = val;
        }
        __syncwarp();
    }
}

// One group (every expert a candidate): the fused selection over this half's
// columns.  Pass A computes each 8-column piece's values and keys (writing the
// scores when they are wanted) and keeps the r = ceil(K/2) largest of the
// pieces' second-largest keys; the halves exchange theirs, and theta, the r-th
// largest of them over the whole row, bounds the K-th best key from below (at
// least r pieces hold two keys >= theta).  Pass B offers, from the same values,
// only the keys >= theta, in rounds of one per lane (lanes are rows with
// different survivors).  `value` turns a raw accumulator column into the score.
template <int BN, typename F>
__device__ __forceinline__ void one_group_select(const Epi& p, uint32_t taddr, int row, int h, int c_lo, float* srow,
                                                 const float* bias_s, float* xg, Top8& top, F value) {
    constexpr int NQ = 4 * (BN / 64);  // 8-column pieces in a half row
    const int r = (p.K + 1) >> 1;
    float b4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};  // descending
#pragma unroll 1
    for (int q = 0; q < NQ; ++q) {
        const int col0 = 32 * c_lo + 8 * q;
        float v8[8];
        tmem_ld8(taddr + col0, v8);
        float t1 = -INFINITY, t2 = -INFINITY;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            v8[i] = value(v8[i], col0 + i);
            const float k = __fadd_rn(v8[i], bias_s[col0 + i]);
            t2 = fmaxf(t2, fminf(t1, k));
            t1 = fmaxf(t1, k);
        }
        if (srow) store8(srow + col0, v8);
        float x = t2;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float hi = fmaxf(b4[j], x);
            x = fminf(b4[j], x);
            b4[j] = hi;
        }
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) xg[row * 8 + h * 4 + j] = b4[j];
    epi_sync();
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        float x = xg[row * 8 + (1 - h) * 4 + j];
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
            const float hi = fmaxf(b4[jj], x);
            x = fminf(b4[jj], x);
            b4[jj] = hi;
        }
    }
    float theta = b4[0];
#pragma unroll
    for (int j = 1; j < 4; ++j)
        if (j < r) theta = b4[j];
#pragma unroll 1
    for (int q = 0; q < NQ; ++q) {
        const int col0 = 32 * c_lo + 8 * q;
        float v8[8], k8[8];
        tmem_ld8(taddr + col0, v8);
        unsigned m = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            v8[i] = value(v8[i], col0 + i);
            k8[i] = __fadd_rn(v8[i], bias_s[col0 + i]);
            if (!(k8[i] < theta)) m |= 1u << i;  // a NaN key is offered
        }
        while (__any_sync(0xffffffffu, m != 0)) {
            if (m != 0) {
                const int i = __ffs(m) - 1;
                m &= m - 1;
                float kk = k8[0], sv = v8[0];
#pragma unroll
                for (int j = 1; j < 8; ++j)
                    if (i == j) { kk = k8[j]; sv = v8[j]; }
                top.offer(kk, col0 + i, sv);
            }
        }
    }
}

// One token row (this thread's TMEM lane) of one finished tile.  The two
// warps of a lane quarter split the columns: half h owns chunks
// [h*NC/2, (h+1)*NC/2) of 32 columns.  Softmax exchanges the row max and sum;
// grouped selection exchanges group scores; half 1 hands its top-8 to half 0,
// which merges and writes the row's choice.  Every epilogue thread executes
// the same sequence of epi_sync() calls.
template <int BN, bool FUSED>
__device__ __forceinline__ void epilogue_row(const Epi& p, uint32_t taddr, int row, int h, int64_t grow,
                                             const float* off_s, const float* bias_s, const Xch& x) {
    constexpr int NC = BN / 32, NCH = NC / 2;
    const int c_lo = h * NCH;
    const int lane = threadIdx.x & 31, warp_in_epi = (int)(threadIdx.x >> 5) - 2;  // epilogue warps are 2..
    const bool live = grow < p.T;
    float* srow = (p.scores != nullptr && live) ? p.scores + grow * BN : nullptr;
    float v[32];
    Top8 top;
    top.init();
    if (p.fn == MOE_SIGMOID) {
        if (FUSED && p.n_groups > 1) {
            // one expert group per 32-column chunk: group score = sum of its top-n
            // keys; each 8-column piece's second-largest key also goes to shared
            // memory (rounded down to half precision: still a lower bound) for
            // the bound below, in the merge lists' space (idle until the merge)
            __half* piece_t2 = reinterpret_cast<__half*>(x.lk) + row * 32;
#pragma unroll 1
            for (int cc = 0; cc < NCH; ++cc) {
                const int c = c_lo + cc;
                tmem_ld32(taddr + 32 * c, v);
                float a1[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY}, a2[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    v[i] = sigmoid_f(__fadd_rn(v[i], off_s[32 * c + i]));
                    const float key = __fadd_rn(v[i], bias_s[32 * c + i]);
                    a2[i >> 3] = fmaxf(a2[i >> 3], fminf(a1[i >> 3], key));  // a NaN key enters none
                    a1[i >> 3] = fmaxf(a1[i >> 3], key);
                }
                float t1 = -INFINITY, t2 = -INFINITY;
#pragma unroll
                for (int pc = 0; pc < 4; ++pc) {
                    t2 = fmaxf(t2, fminf(t1, a1[pc]));
                    t1 = fmaxf(t1, a1[pc]);
                    t2 = fmaxf(t2, fminf(t1, a2[pc]));
                    t1 = fmaxf(t1, a2[pc]);
                    piece_t2[4 * c + pc] = __float2half_rd(a2[pc]);
                }
                x.gs[row * 8 + c] = p.group_topn == 1 ? t1 : __fadd_rn(t1, t2);
                x.gt2[row * 8 + c] = t2;
                if (srow) store32(srow + 32 * c, v);
            }
            epi_sync();
            float gs[NC];
#pragma unroll
            for (int c = 0; c < NC; ++c) gs[c] = x.gs[row * 8 + c];
            unsigned keep = 0;
#pragma unroll
            for (int c = 0; c < NC; ++c) {
                int rank = 0;
#pragma unroll
                for (int c2 = 0; c2 < NC; ++c2) rank += (c2 != c && beats(gs[c2], c2, gs[c], c)) ? 1 : 0;
                if (rank < p.topk_groups) keep |= 1u << c;
            }
            // A lower bound on the row's K-th best kept key: every kept group
            // holds two keys at or above its second largest, so with
            // 2 * topk_groups >= K the K best keys are all at or above the
            // smallest kept second-largest key.  Only those candidates are
            // offered (lanes are token rows with different kept groups, so
            // offering every kept column would run every column in every warp).
            float t0 = INFINITY;
#pragma unroll
            for (int c = 0; c < NC; ++c)
                if ((keep >> c) & 1u) t0 = fminf(t0, x.gt2[row * 8 + c]);
            if (2 * p.topk_groups < p.K || !(t0 < INFINITY)) t0 = -INFINITY;
            // A second bound, tighter when one group holds most of the best keys:
            // the ceil(K/2)-th largest second-largest key over the kept groups'
            // 8-column pieces (at least that many pieces hold two keys at or
            // above it).  Both bound the K-th best key, so their maximum does.
            {
                float b4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};  // descending
#pragma unroll
                for (int c = 0; c < NC; ++c) {
                    if (!((keep >> c) & 1u)) continue;
#pragma unroll
                    for (int pc = 0; pc < 4; ++pc) {
                        float xv = __half2float(piece_t2[4 * c + pc]);
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            const float hi = fmaxf(b4[j], xv);
                            xv = fminf(b4[j], xv);
                            b4[j] = hi;
                        }
                    }
                }
                const int r = (p.K + 1) >> 1;
                float thp = b4[0];
#pragma unroll
                for (int j = 1; j < 4; ++j)
                    if (j < r) thp = b4[j];
                t0 = fmaxf(t0, thp);
            }
            epi_sync();  // every row's pieces are read before the merge lists reuse their space
#pragma unroll 1
            for (int cc = 0; cc < NCH; ++cc) {
                const int c = c_lo + cc;
                const bool kc = (keep >> c) & 1u;
                if (!__any_sync(0xffffffffu, kc)) continue;
#pragma unroll 1
                for (int q = 0; q < 4; ++q) {
                    float v8[8], k8[8];
                    tmem_ld8(taddr + 32 * c + 8 * q, v8);  // warp-collective: every lane loads every piece
                    unsigned m = 0;
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const int col = 32 * c + 8 * q + i;
                        v8[i] = sigmoid_f(__fadd_rn(v8[i], off_s[col]));
                        k8[i] = __fadd_rn(v8[i], bias_s[col]);
                        if (kc && !(k8[i] < t0)) m |= 1u << i;  // a NaN key is offered, as without the bound
                    }
                    // survivors in ascending column order, one per lane per round
                    while (__any_sync(0xffffffffu, m != 0)) {
                        if (m != 0) {
                            const int i = __ffs(m) - 1;
                            m &= m - 1;
                            float kk = k8[0], sv = v8[0];
#pragma unroll
                            for (int j = 1; j < 8; ++j)
                                if (i == j) { kk = k8[j]; sv = v8[j]; }
                            top.offer(kk, 32 * c + 8 * q + i, sv);
                        }
                    }
                }
            }
        } else if constexpr (FUSED) {
            one_group_select<BN>(p, taddr, row, h, c_lo, srow, bias_s, x.gs, top,
                                 [&](float a, int col) { return sigmoid_f(__fadd_rn(a, off_s[col])); });
        } else {
#pragma unroll 1
            for (int cc = 0; cc < NCH; ++cc) {
                const int c = c_lo + cc;
                tmem_ld32(taddr + 32 * c, v);
#pragma unroll
                for (int i = 0; i < 32; ++i) v[i] = sigmoid_f(__fadd_rn(v[i], off_s[32 * c + i]));
                if (p.scores != nullptr) store_chunk_staged<BN>(p, grow, c, v, x.stage + warp_in_epi * (32 * 20), lane);
            }
        }
    } else {
        // softmax over the whole row: exchange the halves' max, then their sums
        float m = -INFINITY;
#pragma unroll 1
        for (int cc = 0; cc < NCH; ++cc) {
            const int c = c_lo + cc;
            tmem_ld32(taddr + 32 * c, v);
#pragma unroll
            for (int i = 0; i < 32; ++i) m = fmaxf(m, v[i] + off_s[32 * c + i]);
        }
        x.red[(h * 2 + 0) * BM + row] = m;
        epi_sync();
        m = fmaxf(x.red[0 * BM + row], x.red[2 * BM + row]);
        float sum = 0.f;
#pragma unroll 1
        for (int cc = 0; cc < NCH; ++cc) {
            const int c = c_lo + cc;
            tmem_ld32(taddr + 32 * c, v);
#pragma unroll
            for (int i = 0; i < 32; ++i) sum += expf(__fsub_rn(__fadd_rn(v[i], off_s[32 * c + i]), m));
        }
        x.red[(h * 2 + 1) * BM + row] = sum;
        epi_sync();
        const float inv = 1.f / (x.red[1 * BM + row] + x.red[3 * BM + row]);
        if constexpr (FUSED) {
            one_group_select<BN>(p, taddr, row, h, c_lo, srow, bias_s, x.gs, top, [&](float a, int col) {
                return __fmul_rn(expf(__fsub_rn(__fadd_rn(a, off_s[col]), m)), inv);
            });
        } else {
#pragma unroll 1
            for (int cc = 0; cc < NCH; ++cc) {
                const int c = c_lo + cc;
                tmem_ld32(taddr + 32 * c, v);
#pragma unroll
                for (int i = 0; i < 32; ++i) v[i] = __fmul_rn(expf(__fsub_rn(__fadd_rn(v[i], off_s[32 * c + i]), m)), inv);
                if (p.scores != nullptr) store_chunk_staged<BN>(p, grow, c, v, x.stage + warp_in_epi * (32 * 20), lane);
            }
        }
    }
    if constexpr (!FUSED) return;
    // half 1 hands its list to half 0; its indices are all above half 0's,
    // so offering them in list order keeps (key desc, index asc)
    if (h == 1) {
#pragma unroll
        for (int j = 0; j < 8; ++j) { x.lk[row * 8 + j] = top.k[j]; x.ls[row * 8 + j] = top.s[j]; x.li[row * 8 + j] = top.i[j]; }
    }
    epi_sync();
    if (h == 0) {
#pragma unroll
        for (int j = 0; j < 8; ++j) top.offer(x.lk[row * 8 + j], x.li[row * 8 + j], x.ls[row * 8 + j]);
        if (live) {
            top.write(p.K, p.renorm, p.scale, p.idx + grow * p.K, p.w + grow * p.K);
            if (p.tile_counts != nullptr) {
                int* hp = x.hist + (int)(grow & 1) * BN;
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    if (k < p.K && (unsigned)top.i[k] < (unsigned)BN) atomicAdd(hp + top.i[k], 1);
            }
        }
    }
}

// After a fused tile's rows: its histogram to global memory (tile index
// `tile`, skipped past the last token), and cleared for the next tile.  Every
// epilogue thread calls it; the named barrier orders the rows' counts first.
template <int BN>
__device__ __forceinline__ void flush_tile_hist(const Epi& p, const Xch& x, int64_t tile) {
    epi_sync();
    const int et = (int)threadIdx.x - 64;  // epilogue threads are warps 2..
    int32_t* dst = tile * BM < (int64_t)p.T ? p.tile_counts + tile * 2 * BN : nullptr;
    for (int i = et; i < 2 * BN; i += EPI_THREADS) {
        if (dst != nullptr) dst[i] = x.hist[i];
        x.hist[i] = 0;
    }
}

template <int BN, bool FUSED>
__global__ void __launch_bounds__(THREADS, 1) gate_tc_kernel(const __grid_constant__ CUtensorMap tmA,
                                                             const __grid_constant__ CUtensorMap tmB, int d,
                                                             const Epi p, int32_t* err, int num_tiles) {
    using C = Cfg<BN>;
    constexpr int STAGES = C::STAGES, KPS = C::KPS;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sA = smem;                                          // [STAGES * KPS][128 x 64] bf16
    uint8_t* sB = smem + (size_t)STAGES * KPS * A_KB_BYTES;      // [STAGES * KPS][BN x 64] bf16
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + (size_t)STAGES * KPS * C::KB_BYTES);
    // bars: full[STAGES], empty[STAGES], tfull[2], tempty[2], done
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * STAGES + 5);
    float* off_s = reinterpret_cast<float*>(tmem_slot + 4);
    float* bias_s = off_s + BN;
    const Xch xch = carve_xch<BN>(bias_s + BN);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t full0 = smem_u32(bars), empty0 = smem_u32(bars + STAGES);
    const uint32_t tfull0 = smem_u32(bars + 2 * STAGES), tempty0 = smem_u32(bars + 2 * STAGES + 2);
    const uint32_t done_bar = smem_u32(bars + 2 * STAGES + 4);
    const int num_kb = (d + BK - 1) / BK;
    for (int i = threadIdx.x; i < 2 * BN; i += blockDim.x) xch.hist[i] = 0;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) { mbar_init(full0 + 8 * s, 1); mbar_init(empty0 + 8 * s, 1); }
        for (int a = 0; a < 2; ++a) { mbar_init(tfull0 + 8 * a, 1); mbar_init(tempty0 + 8 * a, EPI_WARPS); }
        mbar_init(done_bar, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(C::TMEM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    for (int i = threadIdx.x; i < BN; i += blockDim.x) {
        const float o = p.off != nullptr ? p.off[i] : 0.f;
        const float b = p.bias != nullptr ? p.bias[i] : 0.f;
        off_s[i] = p.bias_in_logits ? __fadd_rn(o, b) : o;
        bias_s[i] = p.bias_in_logits ? 0.f : b;
    }
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
                for (int kb = 0; kb < num_kb; kb += KPS, ++it) {
                    const int nk = min(KPS, num_kb - kb);
                    const uint32_t s = it % STAGES, ph = (it / STAGES) & 1;
                    if (!mbar_wait(empty0 + 8 * s, ph ^ 1, err)) { ok = false; break; }
                    mbar_expect_tx(full0 + 8 * s, nk * C::KB_BYTES);
#pragma unroll
                    for (int j = 0; j < KPS; ++j) {
                        if (j >= nk) break;
                        const size_t slot = (size_t)s * KPS + j;
                        tma_load_2d(smem_u32(sA + slot * A_KB_BYTES), &tmA, (kb + j) * BK, tile * BM, full0 + 8 * s);
                        tma_load_2d(smem_u32(sB + slot * C::B_KB_BYTES), &tmB, (kb + j) * BK, 0, full0 + 8 * s);
                    }
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
                for (int kb = 0; kb < num_kb; kb += KPS, ++it) {
                    const int nk = min(KPS, num_kb - kb);
                    const uint32_t s = it % STAGES, ph = (it / STAGES) & 1;
                    if (!mbar_wait(full0 + 8 * s, ph, err)) { ok = false; break; }
                    fence_after();
#pragma unroll
                    for (int j = 0; j < KPS; ++j) {
                        if (j >= nk) break;
                        const size_t slot = (size_t)s * KPS + j;
                        const uint32_t a_addr = smem_u32(sA + slot * A_KB_BYTES);
                        const uint32_t b_addr = smem_u32(sB + slot * C::B_KB_BYTES);
#pragma unroll
                        for (int k = 0; k < BK / 16; ++k)
                            mma_bf16(d_tmem, sdesc(a_addr + 32 * k), sdesc(b_addr + 32 * k), idesc<BN>(),
                                     (kb + j > 0 || k > 0) ? 1u : 0u);
                    }
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
        const int h = (warp - 2) >> 2;       // which half of the columns
        const int row = q * 32 + lane;
        uint32_t local = 0;
        for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++local) {
            const uint32_t a = local & 1, aph = (local >> 1) & 1;
            // one lane per warp waits; the epilogue warps then agree on one verdict
            // (tcgen05.ld is warp-collective and the halves meet at named barriers,
            // so either every epilogue warp processes the tile or none does)
            const int ew = warp - 2;
            if (lane == 0) xch.agree[a * EPI_WARPS + ew] = mbar_wait(tfull0 + 8 * a, aph, err) ? 1 : 0;
            epi_sync();
            int ok = 1;
#pragma unroll
            for (int w = 0; w < EPI_WARPS; ++w) ok &= xch.agree[a * EPI_WARPS + w];
            if (!ok) break;
            fence_after();
            const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + a * BN;
            const int64_t grow = (int64_t)tile * BM + row;
            epilogue_row<BN, FUSED>(p, taddr, row, h, grow, off_s, bias_s, xch);
            fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(tempty0 + 8 * a);
            if (FUSED && p.tile_counts != nullptr) flush_tile_hist<BN>(p, xch, tile);
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


// ===========================================================================
// Two-SM variant (N = 256): a cluster of two CTAs computes a 256-token tile
// with tcgen05.mma.cta_group::2 (M = 256 across the pair, N = 256).  Each CTA
// loads its own 128 token rows of x and its own half (128 experts) of W per
// k-block, 32 KB per SM instead of 48 KB: half the W traffic from L2 and a
// third less shared-memory traffic per MMA.  The ring has three slots of two
// k-blocks each (64 KB per slot): one wait, eight MMAs and one commit per
// slot, and each token row arrives in 256-byte runs.  The leader CTA (rank 0) owns the full barriers (both CTAs' TMA
// loads complete on them), issues the MMAs, and multicasts its commits to
// both CTAs' barriers; each CTA's TMEM receives its own 128 rows x 256
// columns and each CTA runs the same epilogue on them.
// ===========================================================================
constexpr int PAIR_KPS = 2;                              // k-blocks per ring slot
constexpr int PAIR_STAGES = 3;
constexpr uint32_t PAIR_KB_BYTES = 2u * BM * BK * 2;     // one k-block of A rows + B half, per CTA
struct PairCfg {
    static constexpr int BN = 256;
    static constexpr int TMEM_COLS = 2 * BN;
    static constexpr size_t XCH_BYTES = Cfg<256>::XCH_BYTES;
    static constexpr size_t SMEM_BYTES = 1024 + (size_t)PAIR_STAGES * PAIR_KPS * PAIR_KB_BYTES +
                                         8 * (2 * PAIR_STAGES + 5) + 16 + 2 * 4 * BN + XCH_BYTES;
};

__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

// address of the same shared-memory object in CTA `rank` of the cluster
__device__ __forceinline__ uint32_t map_to(uint32_t saddr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
    return r;
}

__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release;\n\tbarrier.cluster.wait.acquire;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}

// TMA load into this CTA's shared memory whose completion is counted on the
// leader CTA's barrier (cluster address).
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap* map, int c0, int c1,
                                                 uint32_t bar_cluster) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(bar_cluster)
        : "memory");
}

__device__ __forceinline__ void mma_bf16_pair(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t id, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a), "l"(b), "r"(id), "r"(acc)
        : "memory");
}

// commit this thread's MMAs to the barrier at `bar` in both CTAs of the pair
__device__ __forceinline__ void mma_commit_pair(uint32_t bar) {
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(bar),
        "h"((uint16_t)3)
        : "memory");
}

__device__ __forceinline__ void mma_commit_pair_local(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}

// bf16 x bf16 -> fp32, K-major, M = 256 (pair), N = 256
__device__ __forceinline__ constexpr uint32_t idesc_pair() {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(256 >> 3) << 17) | ((uint32_t)(256 >> 4) << 24);
}

template <bool FUSED>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(THREADS, 1)
    gate_tc_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, int d,
                        const Epi p, int32_t* err, int num_pairs) {
    constexpr int BN = 256, STAGES = PAIR_STAGES, KPS = PAIR_KPS;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sA = smem;                                          // [STAGES * KPS][128 x 64] bf16, 128B swizzle
    uint8_t* sB = smem + (size_t)STAGES * KPS * A_KB_BYTES;      // [STAGES * KPS][128 x 64] bf16 (this CTA's experts)
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + (size_t)STAGES * KPS * PAIR_KB_BYTES);
    // bars: full[STAGES] (leader), empty[STAGES], tfull[2], tempty[2] (leader), done (leader)
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * STAGES + 5);
    float* off_s = reinterpret_cast<float*>(tmem_slot + 4);
    float* bias_s = off_s + BN;
    const Xch xch = carve_xch<BN>(bias_s + BN);
    for (int i = threadIdx.x; i < 2 * BN; i += blockDim.x) xch.hist[i] = 0;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_rank();
    const bool leader = rank == 0;
    const int cluster = blockIdx.x >> 1, nclusters = gridDim.x >> 1;
    const uint32_t full0 = smem_u32(bars), empty0 = smem_u32(bars + STAGES);
    const uint32_t tfull0 = smem_u32(bars + 2 * STAGES), tempty0 = smem_u32(bars + 2 * STAGES + 2);
    const uint32_t done_bar = smem_u32(bars + 2 * STAGES + 4);
    const int num_kb = (d + BK - 1) / BK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) { mbar_init(full0 + 8 * s, 1); mbar_init(empty0 + 8 * s, 1); }
        for (int a = 0; a < 2; ++a) { mbar_init(tfull0 + 8 * a, 1); mbar_init(tempty0 + 8 * a, 2 * EPI_WARPS); }
        mbar_init(done_bar, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(PairCfg::TMEM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
    }
    for (int i = threadIdx.x; i < BN; i += blockDim.x) {
        const float o = p.off != nullptr ? p.off[i] : 0.f;
        const float b = p.bias != nullptr ? p.bias[i] : 0.f;
        off_s[i] = p.bias_in_logits ? __fadd_rn(o, b) : o;
        bias_s[i] = p.bias_in_logits ? 0.f : b;
    }
    fence_before();
    cluster_sync();  // both CTAs' barriers exist before any cross-CTA arrival
    fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------------------ producer (both CTAs)
        if (lane == 0) {
            uint32_t it = 0;
            bool ok = true;
            for (int tp = cluster; tp < num_pairs && ok; tp += nclusters) {
                const int m0 = tp * 2 * BM + (int)rank * BM;
                for (int kb = 0; kb < num_kb; kb += KPS, ++it) {
                    const int nk = min(KPS, num_kb - kb);
                    const uint32_t s = it % STAGES, ph = (it / STAGES) & 1;
                    if (!mbar_wait(empty0 + 8 * s, ph ^ 1, err)) { ok = false; break; }
                    const uint32_t fb = map_to(full0 + 8 * s, 0);
                    if (leader) mbar_expect_tx(full0 + 8 * s, 2 * nk * PAIR_KB_BYTES);
#pragma unroll
                    for (int j = 0; j < KPS; ++j) {
                        if (j >= nk) break;
                        const size_t slot = (size_t)s * KPS + j;
                        tma_load_2d_pair(smem_u32(sA + slot * A_KB_BYTES), &tmA, (kb + j) * BK, m0, fb);
                        tma_load_2d_pair(smem_u32(sB + slot * A_KB_BYTES), &tmB, (kb + j) * BK, (int)rank * BM, fb);
                    }
                }
            }
            // drain: this CTA's last loads into each slot have landed (the leader sees all of them)
            if (leader) {
                const uint32_t first = it > (uint32_t)STAGES ? it - STAGES : 0;
                for (uint32_t j = first; j < it; ++j) {
                    const uint32_t s = j % STAGES, ph = (j / STAGES) & 1;
                    if (!mbar_wait(full0 + 8 * s, ph, err, /*watch=*/false)) break;
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer (leader only)
        if (leader && lane == 0) {
            uint32_t it = 0, local = 0;
            bool ok = true;
            for (int tp = cluster; tp < num_pairs && ok; tp += nclusters, ++local) {
                const uint32_t a = local & 1, aph = (local >> 1) & 1;
                if (!mbar_wait(tempty0 + 8 * a, aph ^ 1, err)) { ok = false; break; }
                fence_after();
                const uint32_t d_tmem = tmem_base + a * BN;
                for (int kb = 0; kb < num_kb; kb += KPS, ++it) {
                    const int nk = min(KPS, num_kb - kb);
                    const uint32_t s = it % STAGES, ph = (it / STAGES) & 1;
                    if (!mbar_wait(full0 + 8 * s, ph, err)) { ok = false; break; }
                    fence_after();
#pragma unroll
                    for (int j = 0; j < KPS; ++j) {
                        if (j >= nk) break;
                        const size_t slot = (size_t)s * KPS + j;
                        const uint32_t a_addr = smem_u32(sA + slot * A_KB_BYTES);
                        const uint32_t b_addr = smem_u32(sB + slot * A_KB_BYTES);
#pragma unroll
                        for (int k = 0; k < BK / 16; ++k)
                            mma_bf16_pair(d_tmem, sdesc(a_addr + 32 * k), sdesc(b_addr + 32 * k), idesc_pair(),
                                          (kb + j > 0 || k > 0) ? 1u : 0u);
                    }
                    mma_commit_pair(empty0 + 8 * s);
                }
                if (ok) mma_commit_pair(tfull0 + 8 * a);
            }
            mma_commit_pair_local(done_bar);
            mbar_wait(done_bar, 0, err, /*watch=*/false);
        }
    } else {
        // ------------------------------------------------------------ epilogue (both CTAs)
        const int q = warp & 3;
        const int h = (warp - 2) >> 2;
        const int row = q * 32 + lane;
        const uint32_t tempty_leader0 = map_to(tempty0, 0);
        uint32_t local = 0;
        for (int tp = cluster; tp < num_pairs; tp += nclusters, ++local) {
            const uint32_t a = local & 1, aph = (local >> 1) & 1;
            const int ew = warp - 2;
            if (lane == 0) xch.agree[a * EPI_WARPS + ew] = mbar_wait(tfull0 + 8 * a, aph, err) ? 1 : 0;
            epi_sync();
            int ok = 1;
#pragma unroll
            for (int w = 0; w < EPI_WARPS; ++w) ok &= xch.agree[a * EPI_WARPS + w];
            if (!ok) break;
            fence_after();
            const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + a * BN;
            const int64_t grow = (int64_t)tp * 2 * BM + (int64_t)rank * BM + row;
            epilogue_row<BN, FUSED>(p, taddr, row, h, grow, off_s, bias_s, xch);
            fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(tempty_leader0 + 8 * a);
            if (FUSED && p.tile_counts != nullptr) flush_tile_hist<BN>(p, xch, (int64_t)tp * 2 + rank);
        }
    }

    // both CTAs finished with TMEM and the leader's MMAs are drained before
    // either CTA frees its half of the accumulators
    fence_before();
    __syncthreads();
    cluster_sync();
    fence_after();
    if (warp == 1) {
        __syncwarp();
        asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                     "r"(PairCfg::TMEM_COLS)
                     : "memory");
    }
}


// ===========================================================================
// Split-K variant for batches with fewer 256-token tiles than CTA pairs:
// clusters of 2 * S CTAs (S = 2..4 pairs), each taking its tiles one after
// another.  For every tile, pair p (cluster ranks
// 2p and 2p + 1, a tcgen05 CTA pair) runs the same producer / MMA roles as the
// kernel above over its own range of k-blocks into its own TMEM.  Then the
// pairs p >= 1 copy their accumulators into their idle TMA rings, every
// thread of the cluster meets at a cluster barrier, and pair 0 adds the other
// pairs' partial sums (read over distributed shared memory, in pair order, so
// the result does not depend on timing) into its TMEM and runs the usual
// epilogue.  No atomics, no waits on other CTAs beyond the cluster barriers,
// which every thread reaches on every path.
// ===========================================================================
// staged partial sums, as float4 pieces [chunk of 32 columns][piece of 4][row]:
// the 32 rows of a warp's piece are 512 contiguous bytes, so both the staging
// stores and the remote loads of the fold move whole lines
__device__ __forceinline__ uint32_t split_piece(int c, int q, int row) { return (uint32_t)((c * 8 + q) * 128 + row); }

__device__ __forceinline__ void mma_commit_pair_mask(uint32_t bar, uint16_t mask) {
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(bar),
        "h"(mask)
        : "memory");
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float (&v)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
        "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])), "r"(__float_as_uint(v[3])),
        "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])), "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])),
        "r"(__float_as_uint(v[8])), "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])),
        "r"(__float_as_uint(v[11])), "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])),
        "r"(__float_as_uint(v[14])), "r"(__float_as_uint(v[15])), "r"(__float_as_uint(v[16])),
        "r"(__float_as_uint(v[17])), "r"(__float_as_uint(v[18])), "r"(__float_as_uint(v[19])),
        "r"(__float_as_uint(v[20])), "r"(__float_as_uint(v[21])), "r"(__float_as_uint(v[22])),
        "r"(__float_as_uint(v[23])), "r"(__float_as_uint(v[24])), "r"(__float_as_uint(v[25])),
        "r"(__float_as_uint(v[26])), "r"(__float_as_uint(v[27])), "r"(__float_as_uint(v[28])),
        "r"(__float_as_uint(v[29])), "r"(__float_as_uint(v[30])), "r"(__float_as_uint(v[31]))
        : "memory");
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ float4 ld_dsmem_f4(uint32_t cluster_addr) {
    float4 r;
    asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(r.x), "=f"(r.y), "=f"(r.z), "=f"(r.w)
                 : "r"(cluster_addr)
                 : "memory");
    return r;
}

template <bool FUSED>
__global__ void __launch_bounds__(THREADS, 1)
    gate_tc_split_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, int d,
                         const Epi p, int32_t* err, int num_pairs, int splits) {
    constexpr int BN = 256, STAGES = PAIR_STAGES, KPS = PAIR_KPS, NCH = BN / 64;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sA = smem;
    uint8_t* sB = smem + (size_t)STAGES * KPS * A_KB_BYTES;
    float4* stage = reinterpret_cast<float4*>(smem);  // partial sums (split_piece order), while the ring is idle
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + (size_t)STAGES * KPS * PAIR_KB_BYTES);
    // bars: full[STAGES] (pair leader), empty[STAGES], tfull, (unused), (unused), (unused), done
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * STAGES + 5);
    float* off_s = reinterpret_cast<float*>(tmem_slot + 4);
    float* bias_s = off_s + BN;
    const Xch xch = carve_xch<BN>(bias_s + BN);
    for (int i = threadIdx.x; i < 2 * BN; i += blockDim.x) xch.hist[i] = 0;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_rank();
    const uint32_t prank = rank & 1u, pair_leader = rank & ~1u;
    const int pr = (int)(rank >> 1);  // this pair's share of each tile's k-blocks
    const bool leader = prank == 0;
    const int cluster = (int)blockIdx.x / (2 * splits), nclusters = (int)gridDim.x / (2 * splits);
    const uint32_t full0 = smem_u32(bars), empty0 = smem_u32(bars + STAGES);
    const uint32_t tfull0 = smem_u32(bars + 2 * STAGES);
    const uint32_t done_bar = smem_u32(bars + 2 * STAGES + 4);
    const int num_kb = (d + BK - 1) / BK;
    const int nslots = (num_kb + KPS - 1) / KPS;
    const int kb_lo = (pr * nslots / splits) * KPS;
    const int kb_hi = min(num_kb, ((pr + 1) * nslots / splits) * KPS);
    const uint16_t pair_mask = (uint16_t)(3u << pair_leader);

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) { mbar_init(full0 + 8 * s, 1); mbar_init(empty0 + 8 * s, 1); }
        mbar_init(tfull0, 1);
        mbar_init(done_bar, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(PairCfg::TMEM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
    }
    for (int i = threadIdx.x; i < BN; i += blockDim.x) {
        const float o = p.off != nullptr ? p.off[i] : 0.f;
        const float b = p.bias != nullptr ? p.bias[i] : 0.f;
        off_s[i] = p.bias_in_logits ? __fadd_rn(o, b) : o;
        bias_s[i] = p.bias_in_logits ? 0.f : b;
    }
    fence_before();
    cluster_sync();  // every CTA's barriers exist before any cross-CTA arrival
    fence_after();
    const uint32_t tmem_base = *tmem_slot;

    // The cluster walks its tiles one after another; every thread of every
    // CTA takes the same iterations and meets the two cluster barriers of each
    // (a role that has given up on a wait does nothing more but still meets
    // them), so the accumulator and the staged partials are never overwritten
    // while still being read.
    uint32_t it = 0;   // ring slot sequence (producer and MMA issuer)
    bool ok = true;    // this thread's waits have all succeeded
    uint32_t local = 0;
    for (int tp = cluster; tp < num_pairs; tp += nclusters, ++local) {
        int epi_ok = 0;
        if (warp == 0) {
            // -------------------------------------------------------- producer (every CTA)
            if (lane == 0 && ok) {
                const int m0 = tp * 2 * BM + (int)prank * BM;
                for (int kb = kb_lo; kb < kb_hi; kb += KPS, ++it) {
                    const int nk = min(KPS, kb_hi - kb);
                    const uint32_t s = it % STAGES, ph = (it / STAGES) & 1;
                    if (!mbar_wait(empty0 + 8 * s, ph ^ 1, err)) { ok = false; break; }
                    const uint32_t fb = map_to(full0 + 8 * s, pair_leader);
                    if (leader) mbar_expect_tx(full0 + 8 * s, 2 * nk * PAIR_KB_BYTES);
#pragma unroll
                    for (int j = 0; j < KPS; ++j) {
                        if (j >= nk) break;
                        const size_t slot = (size_t)s * KPS + j;
                        tma_load_2d_pair(smem_u32(sA + slot * A_KB_BYTES), &tmA, (kb + j) * BK, m0, fb);
                        tma_load_2d_pair(smem_u32(sB + slot * A_KB_BYTES), &tmB, (kb + j) * BK, (int)prank * BM,
                                         fb);
                    }
                }
            }
        } else if (warp == 1) {
            // -------------------------------------------------------- MMA issuer (pair leaders)
            if (leader && lane == 0 && ok) {
                for (int kb = kb_lo; kb < kb_hi; kb += KPS, ++it) {
                    const int nk = min(KPS, kb_hi - kb);
                    const uint32_t s = it % STAGES, ph = (it / STAGES) & 1;
                    if (!mbar_wait(full0 + 8 * s, ph, err)) { ok = false; break; }
                    fence_after();
#pragma unroll
                    for (int j = 0; j < KPS; ++j) {
                        if (j >= nk) break;
                        const size_t slot = (size_t)s * KPS + j;
                        const uint32_t a_addr = smem_u32(sA + slot * A_KB_BYTES);
                        const uint32_t b_addr = smem_u32(sB + slot * A_KB_BYTES);
#pragma unroll
                        for (int k = 0; k < BK / 16; ++k)
                            mma_bf16_pair(tmem_base, sdesc(a_addr + 32 * k), sdesc(b_addr + 32 * k), idesc_pair(),
                                          (kb + j > kb_lo || k > 0) ? 1u : 0u);
                    }
                    mma_commit_pair_mask(empty0 + 8 * s, pair_mask);
                }
                if (ok) mma_commit_pair_mask(tfull0, pair_mask);
            }
        } else {
            // -------------------------------------------------------- epilogue warps: the accumulator
            const int q = warp & 3, h = (warp - 2) >> 2, row = q * 32 + lane, ew = warp - 2;
            if (lane == 0) xch.agree[ew] = (ok && mbar_wait(tfull0, local & 1, err)) ? 1 : 0;
            epi_sync();
            epi_ok = 1;
#pragma unroll
            for (int w = 0; w < EPI_WARPS; ++w) epi_ok &= xch.agree[w];
            epi_sync();  // every warp has read the verdicts before the next tile's are written
            if (!epi_ok) ok = false;
            fence_after();
            if (epi_ok && pr != 0) {
                // this pair's partial sums into the idle ring (rows padded against bank conflicts)
                const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16);
#pragma unroll 1
                for (int cc = 0; cc < NCH; ++cc) {
                    const int c = h * NCH + cc;
                    float v[32];
                    tmem_ld32(taddr + 32 * c, v);
#pragma unroll
                    for (int qq = 0; qq < 8; ++qq)
                        stage[split_piece(c, qq, row)] =
                            make_float4(v[4 * qq], v[4 * qq + 1], v[4 * qq + 2], v[4 * qq + 3]);
                }
            }
        }

        // every partial of this tile is staged before pair 0 reads it
        fence_before();
        __syncthreads();
        cluster_sync();
        fence_after();

        if (warp >= 2 && pr == 0 && epi_ok) {
            const int q = warp & 3, h = (warp - 2) >> 2, row = q * 32 + lane;
            const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16);
            // the other pairs' partial sums, in pair order, added into this CTA's accumulator
#pragma unroll 1
            for (int cc = 0; cc < NCH; ++cc) {
                const int c = h * NCH + cc;
                float v[32];
                tmem_ld32(taddr + 32 * c, v);
                const uint32_t src = smem_u32(stage + split_piece(c, 0, row));
                // two pairs' pieces in flight at once, added in pair order
                for (int p2 = 1; p2 < splits; p2 += 2) {
                    const bool two = p2 + 1 < splits;
                    const uint32_t peer_a = map_to(src, 2u * (uint32_t)p2 + prank);
                    const uint32_t peer_b = map_to(src, 2u * (uint32_t)(two ? p2 + 1 : p2) + prank);
                    float4 fa[8], fb[8];
#pragma unroll
                    for (int qq = 0; qq < 8; ++qq) {
                        fa[qq] = ld_dsmem_f4(peer_a + 16u * 128u * (uint32_t)qq);
                        fb[qq] = ld_dsmem_f4(peer_b + 16u * 128u * (uint32_t)qq);
                    }
#pragma unroll
                    for (int qq = 0; qq < 8; ++qq) {
                        v[4 * qq] += fa[qq].x;
                        v[4 * qq + 1] += fa[qq].y;
                        v[4 * qq + 2] += fa[qq].z;
                        v[4 * qq + 3] += fa[qq].w;
                    }
                    if (two) {
#pragma unroll
                        for (int qq = 0; qq < 8; ++qq) {
                            v[4 * qq] += fb[qq].x;
                            v[4 * qq + 1] += fb[qq].y;
                            v[4 * qq + 2] += fb[qq].z;
                            v[4 * qq + 3] += fb[qq].w;
                        }
                    }
                }
                tmem_st32(taddr + 32 * c, v);
            }
            const int64_t grow = (int64_t)tp * 2 * BM + (int64_t)prank * BM + row;
            epilogue_row<BN, FUSED>(p, taddr, row, h, grow, off_s, bias_s, xch);
            if (FUSED && p.tile_counts != nullptr) flush_tile_hist<BN>(p, xch, (int64_t)tp * 2 + prank);
        }

        // pair 0 has read every partial and finished with the accumulators
        // before the next tile's loads and MMAs reuse the ring and TMEM
        fence_before();
        __syncthreads();
        cluster_sync();
        fence_after();
    }

    // the MMA issuers' MMAs are complete before TMEM is freed
    if (warp == 1 && leader && lane == 0) {
        mma_commit_pair_local(done_bar);
        mbar_wait(done_bar, 0, err, /*watch=*/false);
    }
    fence_before();
    __syncthreads();
    cluster_sync();
    fence_after();
    if (warp == 1) {
        __syncwarp();
        asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                     "r"(PairCfg::TMEM_COLS)
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

// The epilogue can select when the groups are whole 32-column chunks (or
// there is one group) and K fits its 8-entry list.
bool gate_tc_can_fuse(int N, int K, int fn, int n_groups, int group_topn) {
    if (K > 8) return false;
    if (n_groups == 1) return true;
    return fn == MOE_SIGMOID && N / n_groups == 32 && group_topn >= 1 && group_topn <= 2;
}

// Launch configuration of the split-K pair kernel: one tile per cluster of
// 2 * splits CTAs.
static cudaLaunchConfig_t split_config(int num_pairs, int splits, size_t smem, cudaStream_t st,
                                       cudaLaunchAttribute* attr) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(num_pairs * 2 * splits), 1, 1);
    cfg.blockDim = dim3(tc::THREADS, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)(2 * splits);
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cfg;
}

// How many CTA pairs share each tile's k-blocks, from the batch shape and the
// device alone (so that the result does not depend on an SM budget): 1 unless
// at least half of the device's CTA pairs would otherwise sit idle; at most 4
// (clusters of 8 CTAs), at least two ring slots of k-blocks per pair, and no
// more than lets one cluster per tile be resident at once (on a B200 with this
// kernel's shared memory: 74 clusters of 2 CTAs, 33 of 4, 22 of 6, 15 of 8).
// MOE_GATE_SPLIT=0 turns it off.
static int split_resident(int splits, bool fused, size_t smem) {
    static int resident[2][5] = {};  // [fused][splits]: clusters that fit at once (-1: none)
    int& r = resident[fused ? 1 : 0][splits];
    if (r == 0) {
        auto kern = fused ? tc::gate_tc_split_kernel<true> : tc::gate_tc_split_kernel<false>;
        cudaLaunchAttribute attr[1];
        cudaLaunchConfig_t cfg = split_config(1, splits, smem, nullptr, attr);
        int n = 0;
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess ||
            cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess)
            n = 0;
        r = n > 0 ? n : -1;
    }
    return r;
}

static int choose_splits(int num_pairs, int num_kb, bool fused, size_t smem) {
    const char* env = getenv("MOE_GATE_SPLIT");
    if (env != nullptr && env[0] == '0') return 1;
    const int device_pairs = moe_host::sm_count() / 2;
    if (num_pairs < 1 || 2 * num_pairs > device_pairs) return 1;
    const int nslots = (num_kb + tc::PAIR_KPS - 1) / tc::PAIR_KPS;
    int s = device_pairs / num_pairs;
    if (s > 4) s = 4;
    while (s >= 2 && nslots < 2 * s) --s;
    while (s >= 2 && split_resident(s, fused, smem) < num_pairs) --s;  // every tile's cluster at once
    return s < 2 ? 1 : s;
}

static cudaError_t launch_pair(const void* x, const void* W, int T, int d, const tc::Epi& p, int32_t* err,
                               int max_ctas, cudaStream_t st) {
    CUtensorMap ma, mb;
    if (!make_map(&ma, x, T, d, tc::BM) || !make_map(&mb, W, 256, d, tc::BM)) return cudaErrorInvalidValue;
    const size_t smem = tc::PairCfg::SMEM_BYTES;
    const int num_pairs = (T + 2 * tc::BM - 1) / (2 * tc::BM);
    int clusters = moe_host::sm_count() / 2;
    if (max_ctas > 0 && clusters > max_ctas / 2) clusters = max_ctas / 2;
    int splits = choose_splits(num_pairs, (d + tc::BK - 1) / tc::BK, p.fused != 0, smem);
    if (splits > 1 && max_ctas > 0 && max_ctas < 2 * splits) splits = 1;  // a budget below one cluster
    if (splits > 1) {
        // clusters: one per tile, within the SM budget and what fits at once;
        // each walks its tiles in turn, so the result is the same for any count
        int ncl = num_pairs;
        if (max_ctas > 0 && ncl > max_ctas / (2 * splits)) ncl = max_ctas / (2 * splits);
        const int res = split_resident(splits, p.fused != 0, smem);
        if (ncl > res) ncl = res;
        if (ncl < 1) ncl = 1;
        auto skern = p.fused ? tc::gate_tc_split_kernel<true> : tc::gate_tc_split_kernel<false>;
        cudaError_t e = cudaFuncSetAttribute(skern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        cudaLaunchAttribute attr[1];
        cudaLaunchConfig_t cfg = split_config(ncl, splits, smem, st, attr);
        e = cudaLaunchKernelEx(&cfg, skern, ma, mb, d, p, err, num_pairs, splits);
        moe_host::note_launch();
        if (e != cudaSuccess) return e;
        return cudaGetLastError();
    }
    auto kern = p.fused ? tc::gate_tc_pair_kernel<true> : tc::gate_tc_pair_kernel<false>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    if (clusters > num_pairs) clusters = num_pairs;
    if (clusters < 1) clusters = 1;
    kern<<<2 * clusters, tc::THREADS, smem, st>>>(ma, mb, d, p, err, num_pairs);
    moe_host::note_launch();
    return cudaGetLastError();
}

template <int BN>
static cudaError_t launch_bn(const void* x, const void* W, int T, int d, const tc::Epi& p, int32_t* err,
                             int max_ctas, cudaStream_t st) {
    CUtensorMap ma, mb;
    if (!make_map(&ma, x, T, d, tc::BM) || !make_map(&mb, W, BN, d, BN)) return cudaErrorInvalidValue;
    const size_t smem = tc::Cfg<BN>::SMEM_BYTES;
    auto kern = p.fused ? tc::gate_tc_kernel<BN, true> : tc::gate_tc_kernel<BN, false>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int num_tiles = (T + tc::BM - 1) / tc::BM;
    int grid = moe_host::sm_count();
    if (max_ctas > 0 && grid > max_ctas) grid = max_ctas;
    if (grid > num_tiles) grid = num_tiles;
    if (grid < 1) grid = 1;
    kern<<<grid, tc::THREADS, smem, st>>>(ma, mb, d, p, err, num_tiles);
    moe_host::note_launch();
    return cudaGetLastError();
}

cudaError_t launch_gate_tc(const void* x, const void* W, const float* off, const float* bias, int T, int d, int N,
                           int K, int fn, int n_groups, int topk_groups, int group_topn, int renorm, float scale,
                           bool fused, bool bias_in_logits, float* scores, int32_t* idx, float* w, int32_t* err,
                           int max_ctas, int32_t* tile_counts, cudaStream_t st) {
    tc::Epi p;
    p.tile_counts = fused ? tile_counts : nullptr;
    p.bias_in_logits = bias_in_logits ? 1 : 0;
    p.off = off; p.bias = bias; p.scores = scores; p.idx = idx; p.w = w;
    p.T = T; p.fn = fn; p.K = K; p.n_groups = n_groups; p.topk_groups = topk_groups; p.group_topn = group_topn;
    p.renorm = renorm; p.fused = fused ? 1 : 0; p.scale = scale;
    switch (N) {
        case 64: return launch_bn<64>(x, W, T, d, p, err, max_ctas, st);
        case 128: return launch_bn<128>(x, W, T, d, p, err, max_ctas, st);
        case 256: {
            const char* e = getenv("MOE_GATE_PAIR");
            const bool pair = e == nullptr || e[0] != '0';
            return pair ? launch_pair(x, W, T, d, p, err, max_ctas, st)
                        : launch_bn<256>(x, W, T, d, p, err, max_ctas, st);
        }
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace moe
