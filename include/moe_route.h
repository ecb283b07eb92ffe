/*
 * moe_route.h -- C ABI of libmoeroute.so, the B200 (sm_100a) MoE routing hot
 * path: gate GEMM + score nonlinearity, bias-adjusted group-limited top-K with
 * combine weights, load histogram and statistics, bias update, and the
 * expert-contiguous dispatch / weighted combine permutation.
 *
 * Conventions for every call
 *  - All array arguments are DEVICE pointers to dense row-major arrays owned
 *    by the caller.  The library never allocates, frees or synchronises; every
 *    call only enqueues kernels on `stream` and returns.  Results are ready
 *    when the stream reaches them.
 *  - Arguments are validated on the host before any launch; a bad argument
 *    returns MOE_ERR_INVALID (or MOE_ERR_UNSUPPORTED for a valid shape this
 *    build has no kernel for) and enqueues nothing.  A failed launch returns
 *    MOE_ERR_CUDA.  Nothing aborts or traps.
 *  - Device-side waits (TMA/MMA barriers in the gate GEMM, the look-back of
 *    the offsets scan) are bounded.  A wait that runs out sets an error word
 *    in the workspace (sticky until read) and the kernel returns early; read
 *    it with moe_workspace_status().  The load-statistics struct also
 *    carries the status of its own call.
 *  - 16-byte alignment is required for x, w_gate, rows, y and out.
 *  - Flat assignment counts must satisfy T*K < 2^31.
 *
 * Sources (web pages on MoE load balancing), cited per call below:
 *  [ENT] "MoE Routing Entropy vs Expert Saturation: Optimizing DeepSeek V4
 *        Load Balancing" (dailyaiworld.com)
 *  [HD]  "DeepSeek V4 MoE load balancing" (blog.hotdry.top)
 *  [GL]  "DeepSeek-V3 Group-Limited Expert Routing" (cnnetsun.cn)
 *  [MIN] "A minimal experiment in expert-load imbalance" (tech-blog-chi)
 */
#ifndef MOE_ROUTE_H_
#define MOE_ROUTE_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* cudaStream_t without pulling in the CUDA headers. */
typedef struct CUstream_st* moe_stream_t;

typedef enum {
    MOE_OK = 0,
    MOE_ERR_INVALID = 1,     /* bad argument; nothing enqueued */
    MOE_ERR_UNSUPPORTED = 2, /* valid but not implemented for this shape / dtype */
    MOE_ERR_CUDA = 3,        /* a CUDA call failed */
    MOE_ERR_TIMEOUT = 4      /* a bounded device-side wait ran out */
} moe_status;

typedef enum { MOE_SOFTMAX = 0, MOE_SIGMOID = 1 } moe_score_fn;
typedef enum { MOE_F32 = 0, MOE_BF16 = 1 } moe_dtype;

/* Routing configuration ([ENT] "Concrete Implementation" router arguments;
 * [GL] section 3 Gate arguments n_groups / topk_groups). */
typedef struct {
    int32_t T;            /* tokens */
    int32_t d;            /* hidden size (gate GEMM contraction length) */
    int32_t N;            /* routed experts */
    int32_t K;            /* experts per token */
    int32_t score_fn;     /* moe_score_fn */
    int32_t n_groups;     /* expert groups (1 = no group limit); N % n_groups == 0 */
    int32_t topk_groups;  /* groups kept per token */
    int32_t group_topn;   /* group score = sum of this many largest keys (2) */
    int32_t renorm;       /* 1: weights = s_k / sum of chosen s; 0: weights = s_k */
    float route_scale;    /* weights are multiplied by this (2.5 for V3 routing) */
    int32_t in_dtype;     /* moe_dtype of x and w_gate */
    int32_t bias_mode;    /* 0: bias only in the selection key (aux-loss-free routing);
                             1: bias added to the logits before the nonlinearity, so it
                                also shapes the weights ([ENT] "Concrete Implementation":
                                the router adds its expert biases to the raw logits);
                                needs x */
    int32_t gate_max_ctas; /* at most this many CTAs (SMs) for the tensor-core gate GEMM,
                              0 = all SMs; a smaller budget leaves SMs to work running
                              beside it on another stream (e.g. the previous batch's
                              dispatch).  The scores do not depend on the budget, except
                              that a budget smaller than one cluster of the small-batch
                              split of the k-blocks over CTA pairs (4 to 8 CTAs) turns
                              the split off, which changes the fp32 summation order */
} moe_route_cfg;

/* Load statistics of one histogram, written to device memory.
 * [MIN] "Run the example": total, max, mean, imbalance = max / mean (0 when
 * mean is 0), capacity_fixed = max * n_slots.  [HD] "Deployment parameters
 * and monitoring": std_over_mean (population std).  [ENT] "The Mathematics":
 * entropy_load_bits = -sum p log2 p over p = count / total;
 * "Concrete Implementation": entropy_score_bits = entropy of the batch-mean
 * routing distribution (NaN when no scores were given);
 * "Production Testing": capacity_125 = 1.25 * mean. */
typedef struct {
    int32_t status;       /* MOE_OK, or MOE_ERR_TIMEOUT if the offsets scan gave up */
    int32_t n_slots;
    int64_t total;
    int64_t max_load;
    double mean;
    double imbalance;
    double std_over_mean;
    double entropy_load_bits;
    double entropy_score_bits;
    double capacity_fixed;
    double capacity_125;
} moe_stats;

/* Bytes of workspace the calls below need for T tokens, K choices, N experts
 * and n_slots histogram slots (n_slots >= N; N + replicas).  One workspace
 * may serve every call on one stream; calls that overlap on the GPU need
 * their own workspaces.  Zero-fill it once before its first use; every call
 * leaves it ready for the next one, so no per-call initialisation is needed.
 * A workspace must start on a 16-byte boundary (the calls that take one
 * return MOE_ERR_INVALID otherwise). */
size_t moe_workspace_bytes(int64_t T, int32_t K, int32_t N, int32_t n_slots);

/*
 * moe_route -- gate GEMM, score nonlinearity, selection and combine weights.
 *
 * Gate ([ENT] "The Mathematics": h = x . W_g; "Concrete Implementation":
 * nn.Linear(hidden, N, bias=False)):
 *   h[t,e] = sum_j x[t,j] * w_gate[e,j] + logit_offset[e]
 *   x [T,d], w_gate [N,d] in cfg->in_dtype, d % 8 == 0 for bf16.  bf16 with
 *   N in {64, 128, 256}: tcgen05 tensor-core GEMM with fp32 accumulation
 *   (N = 256 on a 2-SM CTA pair; environment variable MOE_GATE_PAIR=0 uses
 *   one CTA per 128-token tile instead); other N, and fp32 inputs:
 *   CUDA-core GEMM with fp32 accumulation.  logit_offset [N] fp32 or NULL.
 * Shapes: N <= 32 or N in {64, 128, 256, 512}; K <= min(N, 32); groups of
 * N / n_groups experts (n_groups <= 32), a size of max(N / 32, 1) times a
 * power of two.  Other valid shapes return MOE_ERR_UNSUPPORTED.
 * Scores, fused into the GEMM epilogue, written to scores [T,N] fp32:
 *   softmax over N ([ENT] softmax equation) or sigmoid ([HD] "Token routing").
 *   If x == NULL the call skips the GEMM and reads `scores` as input instead.
 *   With bf16 inputs, N in {64, 128, 256}, K <= 8 and either one group or
 *   sigmoid scores in groups of 32 experts with group_topn <= 2, the
 *   selection below can also run inside the GEMM epilogue (no scores round
 *   trip); `scores` may then be NULL, and with `scores` given the library
 *   picks the faster of the two for the batch size (environment variable
 *   MOE_FUSED_SELECT=0/1 forces one).  Otherwise `scores` is required.
 * Selection ([HD] "Auxiliary-loss-free load balancing": the bias steers only
 * the choice; [GL] sections 1 and 3: group-limited routing):
 *   key = fp32(s + bias) (bias [N] fp32 or NULL); with n_groups > 1 the
 *   topk_groups groups with the best fp32 sum of their group_topn largest
 *   keys are kept and the rest excluded; the K best keys among the kept
 *   experts are chosen.  Order: key descending, ties to the lower index.
 *   topk_idx [T,K] int32 in that order.  Keys must be finite (scores and
 *   bias finite, hence no NaN or infinite key): the pages define no order
 *   for NaN, and with a non-finite key the choice is unspecified -- an
 *   entry may even hold an id outside [0, N), which the load statistics
 *   reject (an id >= N: stats->status = MOE_ERR_INVALID; a negative id
 *   counts as dropped; either way slot -1 and nothing dispatched for it).
 *   No path reads or writes out of bounds.
 * Weights ([ENT] "Concrete Implementation" renormalisation; [HD] weighted
 * combine by affinity): from the UNBIASED scores,
 *   topk_w[t,k] = fp32(fp32(s_k / fp32-sum-in-k-order) * route_scale)
 *   (renorm = 1) or fp32(s_k * route_scale) (renorm = 0).
 * ws: workspace of moe_workspace_bytes() bytes (error word of the GEMM).
 */
moe_status moe_route(const moe_route_cfg* cfg, const void* x, const void* w_gate,
                     const float* logit_offset, const float* bias, float* scores,
                     int32_t* topk_idx, float* topk_w, void* ws, size_t ws_bytes,
                     moe_stream_t stream);

/*
 * moe_route_tiles -- moe_route with the selection in the GEMM epilogue and
 * the load histogram counted there too, per tile ([GL] section 6: fuse the
 * routing computation with the dispatch path; the scores never reach
 * memory).
 * Same routing as moe_route (the tensor-core gate with the epilogue
 * selection: bf16, N in {64, 128, 256}, K <= 8, one group or sigmoid groups
 * of 32 experts with group_topn <= 2; otherwise MOE_ERR_UNSUPPORTED).  No
 * scores are written.  Additionally, for every tile of 128 tokens,
 *   tile_counts[j][p][e] = #{(t,k) : t in [128j, 128j+128), t % 2 == p,
 *                           topk_idx[t,k] == e}
 * (tile_counts int32 [ceil(T/128)][2][N]): the tile's expert histogram split
 * by token parity, so that per-slot counts with replicas (odd tokens of a
 * replicated expert go to its replica) follow without the indices.
 * moe_load_stats_tiles takes them.
 */
moe_status moe_route_tiles(const moe_route_cfg* cfg, const void* x, const void* w_gate,
                           const float* logit_offset, const float* bias, int32_t* topk_idx,
                           float* topk_w, int32_t* tile_counts, void* ws, size_t ws_bytes,
                           moe_stream_t stream);

/*
 * moe_route_balanced -- "forcible load balancing": the top-K output replaced
 * by an exactly balanced one, an upper bound for balance experiments
 * (MindIE expert_parallelism_load_balancer page, forcible load balancing).
 *   topk_idx[t,k] = (t*K + k) mod N,  topk_w[t,k] = route_scale / K
 * Every expert gets T*K/N assignments (+-1); a token's K experts are
 * distinct (K <= N).
 */
moe_status moe_route_balanced(int64_t T, int32_t K, int32_t N, float route_scale, int32_t* topk_idx,
                              float* topk_w, moe_stream_t stream);

/*
 * moe_route_capacity -- capacity-limited selection ([ENT] "Production
 * Testing": a hard token capacity per expert, 1.25 * T*K/N, with the excess
 * routed to secondary candidate experts by the bias-adjusted ranking).
 *   Candidates of token t: the experts of its kept groups ranked by (key
 *   desc, index asc), key = fp32(s + bias) as in moe_route (the key is s
 *   itself when cfg->bias_mode = 1 or bias is NULL); the first K are
 *   moe_route's choice, in its order.
 *   1. In flat order a = t*K + k a primary is kept while its expert has kept
 *      fewer than `capacity`; the others overflow.
 *   2. Token t's j-th overflowed slot (in k order) moves to its candidate
 *      K + j, if it has one; in flat order again such a reroute is kept while
 *      its expert holds fewer than `capacity` in all.  Everything else is
 *      dropped: topk_idx = -1, topk_w = 0 (one reroute round).
 *   3. Weights as in moe_route, over the token's kept slots in k order.
 * scores [T,N] fp32 (moe_route's scores), bias [N] fp32 or NULL; cfg gives T,
 * N, K (<= 16), the groups, renorm and route_scale (d, score_fn, in_dtype are
 * not used).  capacity >= 0 sets the per-expert limit; capacity < 0 takes
 * the page's rule, moe_capacity_limit(T, K, N) = ceil(1.25 * T*K/N).
 * topk_idx, topk_w [T,K] out; info (device, may be NULL) receives the
 * capacity and the overflow / reroute / drop counts.  ws: a zero-filled
 * workspace of moe_capacity_workspace_bytes() bytes, kept between calls,
 * on a 16-byte boundary.
 * Six launches (candidates, two load-statistics passes, reroute, finalize);
 * every decision comes from stable ranks, so the result equals the
 * sequential walk and is deterministic.
 */
typedef struct moe_capacity_info {
    int64_t capacity;
    int64_t n_overflow;  /* primaries over the capacity */
    int64_t n_rerouted;  /* of those, kept on a secondary expert */
    int64_t n_dropped;   /* n_overflow - n_rerouted */
} moe_capacity_info;

size_t moe_capacity_workspace_bytes(int64_t T, int32_t K, int32_t N);

/* The per-expert token capacity of [ENT] "Production Testing": a capacity
 * factor of 1.25 over the balanced load, ceil(1.25 * T*K / N), computed
 * exactly in integers as ceil(5*T*K / (4*N)).  Returns -1 for T < 0, K <= 0
 * or N <= 0. */
int64_t moe_capacity_limit(int64_t T, int32_t K, int32_t N);

moe_status moe_route_capacity(const moe_route_cfg* cfg, const float* scores, const float* bias,
                              int64_t capacity, int32_t* topk_idx, float* topk_w,
                              moe_capacity_info* info, void* ws, size_t ws_bytes,
                              moe_stream_t stream);

/*
 * moe_load_stats -- load histogram, expert offsets, stable in-expert ranks
 * and load statistics.
 *
 * slot(t,k) = topk_idx[t,k], or, when replica_slot [N] is given (a replica
 * slot id in [N, n_slots) or -1 per expert), the replica slot for odd t and
 * the original for even t ([HD] redundant experts for prefill; [GL] section
 * 2).  slot_idx [T,K] receives slot(t,k) (may be NULL).
 * A negative topk_idx entry is an assignment dropped by the capacity limit
 * (moe_route_capacity): it has slot -1 and rank -1 and counts nowhere.
 * counts [n_slots]: c_e = #{(t,k) : slot = e}  ([ENT] bincount).
 * offsets [n_slots + 1]: exclusive prefix of counts; offsets[n_slots] = the
 *   kept assignments (T*K less the dropped ones).
 * rank [T,K]: number of earlier flat assignments (t',k') < (t,k) with the
 *   same slot -- the row's place inside its expert's segment.
 * stats (device, may be NULL): see moe_stats.  scores [T,N] fp32 (may be
 *   NULL) adds entropy_score_bits, with score_fn telling softmax rows
 *   (used as they are) from sigmoid rows (normalised per token).
 * One single-pass kernel.  Up to about 2.6M assignments (T*K): one wave of
 * blocks of 2048, 4096 or 8192 assignments; each block publishes its
 * per-slot counts as words tagged with the call, and sums the tagged counts
 * of all earlier blocks for its ranks (no chain of prefixes); the last block
 * writes counts, offsets and stats.  Larger problems: blocks of 2048
 * assignments with a decoupled look-back over earlier blocks' count vectors.
 * Either way the waits are bounded (stats->status = MOE_ERR_TIMEOUT on
 * expiry).
 */
moe_status moe_load_stats(const int32_t* topk_idx, int64_t T, int32_t K, int32_t N,
                          const int32_t* replica_slot, int32_t n_slots, int32_t* slot_idx,
                          int32_t* counts, int32_t* offsets, int32_t* rank,
                          const float* scores, int32_t score_fn, moe_stats* stats, void* ws,
                          size_t ws_bytes, moe_stream_t stream);

/*
 * moe_load_stats_tiles -- moe_load_stats (without the score entropy) for a
 * routing made by moe_route_tiles, taking its per-tile histograms
 * tile_counts [ceil(T/128)][2][N] as well as topk_idx.  Results are those of
 * moe_load_stats.  Where a block of the statistics kernel is a whole number
 * of 128-token tiles (K dividing 16, and up to about 2.6M assignments) the
 * block's per-slot counts come from the tile histograms, so it publishes them
 * to the later blocks before reading a single index; its own count of the
 * indices is then checked against them (a mismatch: stats->status or
 * moe_workspace_status MOE_ERR_INVALID).  Otherwise the histograms are not
 * read.
 */
moe_status moe_load_stats_tiles(const int32_t* topk_idx, int64_t T, int32_t K, int32_t N,
                                const int32_t* tile_counts, const int32_t* replica_slot,
                                int32_t n_slots, int32_t* slot_idx, int32_t* counts, int32_t* offsets,
                                int32_t* rank, moe_stats* stats, void* ws, size_t ws_bytes,
                                moe_stream_t stream);

/*
 * moe_replica_plan -- replica slots for the n_replicas hottest experts.
 * Experts ranked by (count desc, index asc); the j-th gets slot N + j, the
 * rest -1.  counts [N] int32 (a histogram over the N experts), replica_slot
 * [N] int32 out.  ([HD] "Auxiliary-loss-free load balancing": hot experts
 * get copies in prefill; [GL] section 2: 32 redundant experts.)
 * n_replicas in [0, N].
 */
moe_status moe_replica_plan(const int32_t* counts, int32_t N, int32_t n_replicas,
                            int32_t* replica_slot, moe_stream_t stream);

/*
 * moe_bias_update -- per-expert routing bias step, in place on bias [N].
 * ([HD] "Auxiliary-loss-free load balancing": lower the bias of overloaded
 * experts, raise it for underloaded ones.)
 *   mode 0: b_e = fp32(b_e - fp32(u * sign(c_e - total/N))), the sign taken
 *           exactly on integers (c_e * N against total), sign(0) = 0.
 *   mode 1: the proportional rule of [ENT] "Concrete Implementation" with
 *           u as bias_decay: target = total / N, err = c_e - target,
 *           b_e -= u * sign(err) * (|err| / target), every op fp32.
 * counts [N] int32; total_assignments = T*K (> 0).
 */
moe_status moe_bias_update(const int32_t* counts, int32_t N, int64_t total_assignments,
                           float u, int32_t mode, float* bias, moe_stream_t stream);

/*
 * moe_bias_update_ema -- the sign-rule bias step on a smoothed load ([HD]
 * "Auxiliary-loss-free load balancing": a moving average smooths the load
 * statistics before the bias is adjusted).  In place on load_ema [N] and
 * bias [N] (fp32, caller-owned state; start load_ema at 0 or at a first
 * histogram):
 *   load_ema_e = fp32(fp32(alpha * load_ema_e) + fp32((1 - alpha) * c_e))
 *   b_e        = fp32(b_e - fp32(u * sign(load_ema_e - fp32(total / N))))
 * alpha in [0, 1); alpha = 0 is the plain sign rule on this step's counts.
 */
moe_status moe_bias_update_ema(const int32_t* counts, int32_t N, int64_t total_assignments, float u,
                               float alpha, float* load_ema, float* bias, moe_stream_t stream);

/*
 * moe_dispatch -- scatter token rows into the expert-contiguous buffer
 * ([HD] "DeepEP": dispatch sends each token to its experts; FP8 dispatch).
 *   pos[t,k] = offsets[slot_idx[t,k]] + rank[t,k]
 *   rows[pos[t,k], :] = x[t, :]          (x_dtype, [T*K, d]; may be NULL)
 *   row_src[pos[t,k]] = t               ([T*K] int32; may be NULL)
 *   pos [T,K] int32 (may be NULL)
 * FP8 copy (rows_fp8 [T*K, d] e4m3 bytes and scales [T*K, d/128] fp32, both
 * NULL or both set; needs d % 128 == 0): per row and 128-channel block,
 *   amax = max|v|, inv = amax > 0 ? fp32(448 / amax) : 0,
 *   q = e4m3_rn_satfinite(fp32(v * inv)), scale = fp32(amax / 448).
 * slot_idx, offsets, rank as produced by moe_load_stats.  d % 8 == 0
 * (bf16) or d % 4 == 0 (fp32).
 * T = 0: nothing is read or written and every buffer may be NULL.
 * Dropped assignments (slot_idx < 0, from moe_route_capacity) get pos = -1
 * and no row; the buffers still hold T*K rows, and the rows from
 * offsets[n_slots] on are scratch (the dropped copies land in the last one).
 */
moe_status moe_dispatch(const void* x, int32_t x_dtype, int64_t T, int32_t d, int32_t K,
                        const int32_t* slot_idx, const int32_t* offsets, const int32_t* rank,
                        void* rows, uint8_t* rows_fp8, float* scales, int32_t* pos,
                        int32_t* row_src, moe_stream_t stream);

/*
 * moe_combine -- weighted gather-sum of expert outputs back to token order
 * ([HD] "Token routing": outputs summed weighted by affinity; "DeepEP":
 * combine, BF16).
 *   out[t, :] = sum_{k=0..K-1, pos[t,k] >= 0} w[t,k] * y[pos[t,k], :]
 * accumulated in fp32 in k order, rounded once to the output dtype (pos < 0:
 * an assignment dropped by the capacity limit, skipped).  T = 0: buffers may
 * be NULL.
 * y [T*K, d] and out [T, d] in `dtype`; pos [T,K] int32, w [T,K] fp32.
 */
moe_status moe_combine(const void* y, int32_t dtype, int64_t T, int32_t d, int32_t K,
                       const int32_t* pos, const float* w, void* out, moe_stream_t stream);

/*
 * moe_load_stats_noalloc -- moe_load_stats without a caller workspace.  The
 * pages have no counterpart: this is a library convenience.
 *
 * For callers that cannot allocate device memory where they call: a
 * framework that owns the whole device memory pool, real-time or embedded
 * code whose memory is fixed at start-up, host callbacks and plugins where a
 * cudaMalloc would block or is not allowed.  Arguments and results are those
 * of moe_load_stats; the scratch comes from a fixed device array inside this
 * library of MOE_NOALLOC_SCRATCH_BYTES bytes, which every GPU that loads the
 * library holds until the process exits.  The call allocates nothing.
 *  - Returns MOE_ERR_UNSUPPORTED, enqueuing nothing, when the problem needs
 *    more scratch than that (moe_workspace_bytes(T, K, N, n_slots) larger
 *    than MOE_NOALLOC_SCRATCH_BYTES, 4 MiB; the largest routing workload
 *    here, T = 131072 tokens, K = 8, 288 slots, needs 1,706,496 bytes).
 *  - The first call on a device looks up the array's device address (with
 *    that device current) and caches it for the life of the process; make
 *    that first call before any stream capture.  The cached address does
 *    not survive cudaDeviceReset (the library's device module is reloaded
 *    at a new address): do not call this entry point after a device reset.
 *  - All calls share the one array, which keeps the last call's contents.
 *    Every call first clears, on its stream, the part that must start at
 *    zero (the scan's control words, look-back flags and per-block count
 *    words: at most about 1.2 MB for the largest workload here), so a call never depends on how the
 *    previous one ended.  Calls whose kernels
 *    overlap on the GPU -- different streams, or threads, using the same
 *    device -- race on the array: the caller must serialise them.
 * The load status of the call is in stats->status, as for moe_load_stats.
 */
#define MOE_NOALLOC_SCRATCH_BYTES (4u << 20)
moe_status moe_load_stats_noalloc(const int32_t* topk_idx, int64_t T, int32_t K, int32_t N,
                                  const int32_t* replica_slot, int32_t n_slots, int32_t* slot_idx,
                                  int32_t* counts, int32_t* offsets, int32_t* rank,
                                  const float* scores, int32_t score_fn, moe_stats* stats,
                                  moe_stream_t stream);

/* Synchronises `stream`, reads and clears the workspace's sticky device
 * error words: MOE_OK, MOE_ERR_TIMEOUT if a bounded wait ran out, or
 * MOE_ERR_INVALID if an expert id was out of range or two load-statistics
 * calls overlapped on the workspace, since the last check.
 * (The calls that synchronise are this one and moe_selftest_wait_timeout.) */
moe_status moe_workspace_status(void* ws, moe_stream_t stream);

/* Self-test of the bounded device waits: runs each load-statistics kernel's
 * wait for an earlier block (the look-back, and the read of earlier blocks'
 * tagged counts) on a two-block problem whose first block never runs.  Each
 * wait must give up after about one second, record the timeout and return,
 * and the CUDA context stays usable.  Returns MOE_ERR_TIMEOUT when both waits
 * ran out as designed (the expected result), MOE_OK if not.  Synchronises
 * `stream`; ws needs moe_workspace_bytes(4096, 1, 8, 8) bytes; the
 * workspace's error words are cleared afterwards. */
moe_status moe_selftest_wait_timeout(void* ws, size_t ws_bytes, moe_stream_t stream);

/* Kernel launches issued by this library on the calling thread since the
 * last reset (for launch accounting). */
int64_t moe_launch_count(int32_t reset);

const char* moe_status_str(moe_status s);
const char* moe_version(void);

#ifdef __cplusplus
}
#endif
#endif /* MOE_ROUTE_H_ */
