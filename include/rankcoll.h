/*
 * rankcoll.h -- C ABI of librankcoll: collective reductions over p simulated
 * ranks whose buffers all live in one GPU's memory (sm_100a, B200).
 *
 * Every rank is a separate device buffer.  A call takes host arrays of p
 * device pointers (one per rank), a per-rank element count, a dtype, a
 * reduction op, an fp32 scale and a CUDA stream.  All work runs in this
 * library's own CUDA kernels, enqueued on the caller's stream.
 *
 * Sources, cited as page title and section:
 *  [SEM]  "分布式训练/推理" (llm-from-scratch, chapter 7), section
 *         "通信原语：rank、world size 和 collective operations" -- the primitive
 *         table (broadcast, reduce with sum/min/max, all-gather, reduce-scatter,
 *         all-reduce), y = sum_r x_r, the four-rank worked example, and
 *         all_reduce = reduce_scatter + all_gather.
 *  [API]  same page, "PyTorch distributed：代码里真正发生了什么" -- all_reduce
 *         works in place; reduce_scatter takes a world_size x k input and a
 *         separate k output; all_gather writes a separate full output.
 *  [AVG]  same page, "数据并行：切 batch，复制模型" -- the gradient average
 *         g = (1/p) sum_r grad L_r (ReduceOp.AVG), here `scale` = 1/p.
 *  [FSDP] same page, "FSDP 的执行顺序：常驻 shard，计算前 gather，反向后 scatter" --
 *         all_gather of parameter shards, reduce_scatter of (1/N_d) sum of grads.
 *  [COLL] "LLM Parallelism 基础", sections "AllReduce" and "其他 Collective" --
 *         Reduce (result on one process), Broadcast, AllGather, ReduceScatter.
 *  [RING] same page, section "Ring AllReduce" -- N chunks; reduce-scatter phase
 *         of N-1 steps (send one chunk to the next card, which accumulates);
 *         all-gather phase of N-1 steps (forward the finished chunk, receiver
 *         overwrites); 2(N-1) steps; card 0 ends the first phase holding chunk 0.
 *  [DDP]  "分布式训练/推理", section "数据并行：切 batch，复制模型" -- naive DDP
 *         all-reduces every gradient after backward (many calls, all exposed);
 *         one flattened all-reduce saves calls but waits for the last gradient;
 *         per-parameter hooks all-reduce each gradient as soon as it is ready
 *         and hide communication under the rest of backward; measure the
 *         communication left exposed after backward.
 *  [ZERO] "分布式训练/推理", section "显存账：不同数据并行的局限性" -- ZeRO-1
 *         shards the optimizer state (Adam moments, fp32 master weights) while
 *         every rank keeps full parameters; section "DDP 模型训练示例" -- the
 *         ShardedOptimizer averages the gradients, runs AdamW on the parameters
 *         its rank owns and hands every rank the owner's parameters.  The page
 *         names torch.optim.AdamW without printing it (see rc_adamw_step).
 *  [A2A]  "分布式训练/推理", primitive table -- all-to-all: every rank sends a
 *         different slice to every rank (MoE token routing); section "从路由结果
 *         到专家输出" -- dispatch towards the experts and combine back, split
 *         counts tell the receiver how much arrives; section "为什么 top-k 和 EP
 *         degree 会直接放大通信" -- payload t*k*h*b per rank and phase.
 *  [P2P]  "分布式训练/推理", section "从单卡到多卡：瓶颈从 HBM 扩展到互联" -- past
 *         one GPU the ranks' data crosses NVLink/NVSwitch, a transfer costs
 *         alpha + bytes/bandwidth; section "通信原语：rank、world size 和
 *         collective operations" -- a rank is usually one GPU or one process;
 *         section "PyTorch distributed：代码里真正发生了什么" -- the collective
 *         library turns a collective into GPU kernels that move data between
 *         GPUs; section "Ring all-reduce 的带宽账" -- T_AR = 2(N-1)/N * S/W.
 *  [HIER] "大模型并行的最小闭环：集合通信、TP、FSDP/ZeRO-3 到权重分片", log excerpt
 *         "分层 AllReduce + SHARP", steps 1-6 -- intra-node AllReduce, one
 *         representative per node, the node results added together, intra-node
 *         broadcast.
 *
 * Result contract (identical bits on every call, checked against an
 * independent CPU implementation):
 *  - Chunk length C = ceil(n/p); element i lies in chunk c = i / C.  Every
 *    reducing call folds the ranks of element i in the order the ring of
 *    [RING] produces: x_{(c+1)%p}, then x_{(c+2)%p}, ..., last x_{c}, starting
 *    from the first operand (no identity element).
 *  - fp32 and bf16 inputs accumulate in fp32 (IEEE round-to-nearest-even,
 *    no fused multiply-add, no flush to zero); `scale` is one fp32 multiply
 *    after the fold; a bf16 output is one round-to-nearest-even at the end.
 *  - int32 SUM wraps (two's complement).  MAX / MIN are compare-selects
 *    (acc = v > acc ? v : acc), so a tie keeps the earlier operand.
 *  - `scale` must be 1.0f unless op is RC_SUM on a floating type.
 *
 * Common argument rules:
 *  - p in [1, 16].  n = per-rank length of the full vector (elements).
 *    n == 0 returns RC_OK and launches nothing.
 *  - Pointer arrays are host memory owned by the caller, read only during the
 *    call (their contents are copied into kernel parameters).  Device buffers
 *    belong to the caller and must stay valid until the stream work is done.
 *  - Aliasing: output buffers must not overlap each other.  An output may
 *    overlap an input only when both describe the same elements at the same
 *    addresses (e.g. in-place all_reduce recv[r] == send[r], or a
 *    reduce_scatter output recv[r] == send[r] + r*(n/p) with equal element
 *    sizes).  Any other overlap returns RC_ERR_INVALID_ARG.
 *  - Pointers need no particular alignment; 16-byte aligned buffers (and
 *    chunk lengths that keep 16-byte alignment) take the vectorised path.
 *  - Calls are asynchronous and stream-ordered.  Argument errors are reported
 *    before anything is enqueued.  A failed launch returns RC_ERR_CUDA.
 *    Faults that happen later on the device surface through rc_stream_status.
 *  - Thread safety: calls may come from several host threads.  Calls that
 *    use the library workspace (see each function) share it per (device,
 *    stream), so calls on one stream are safe; the workspace of a stream is
 *    grown in stream order.
 */
#ifndef RANKCOLL_H
#define RANKCOLL_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    RC_OK = 0,
    RC_ERR_INVALID_ARG = 1, /* bad pointer, size, dtype/op combination, alias */
    RC_ERR_UNSUPPORTED = 2, /* valid request this build does not implement    */
    RC_ERR_CUDA = 3,        /* a CUDA runtime call or launch failed           */
    RC_ERR_TIMEOUT = 4      /* a bounded device-side wait gave up             */
} rc_status;

typedef enum { RC_FP32 = 0, RC_BF16 = 1, RC_INT32 = 2 } rc_dtype;
typedef enum { RC_SUM = 0, RC_MAX = 1, RC_MIN = 2 } rc_op;
typedef enum { RC_RING_LITERAL = 0, RC_RING_ONESHOT = 1 } rc_ring_variant;
typedef enum { RC_HIER_FUSED = 0, RC_HIER_STAGED = 1 } rc_hier_variant;

/* Same type as cudaStream_t; NULL is the legacy default stream. */
typedef struct CUstream_st *rc_stream_t;

/*
 * all-reduce [SEM] [COLL] [AVG]: recv[r][i] = cast(scale * fold_r send[r][i])
 * for every rank r.  send, recv: p device pointers to n elements of dt.
 * One kernel launch: each element is read once per rank and written once per
 * rank.  In place (recv[r] == send[r]) is allowed.
 */
rc_status rc_all_reduce(const void *const *send, void *const *recv, int p, size_t n,
                        rc_dtype dt, rc_op op, float scale, rc_stream_t stream);

/*
 * reduce-scatter [SEM] [API] [FSDP]: rank r receives elements [r*m, (r+1)*m)
 * of the all-reduce result, m = n/p, cast to out_dt.  send: p pointers to n
 * elements of in_dt; recv: p pointers to m elements of out_dt.  n % p != 0
 * is RC_ERR_INVALID_ARG.  (in_dt, out_dt) may be equal, or fp32->bf16 (the
 * fused gradient path: scale 1/p and the bf16 cast in the same kernel), or
 * bf16->fp32.  int32 only to int32.
 */
rc_status rc_reduce_scatter(const void *const *send, void *const *recv, int p, size_t n,
                            rc_dtype in_dt, rc_dtype out_dt, rc_op op, float scale,
                            rc_stream_t stream);

/*
 * all-gather [SEM] [API] [FSDP]: recv[q][r*m + j] = send[r][j] for every q;
 * m = n/p.  send: p pointers to m elements; recv: p pointers to n elements.
 * A byte copy (any dt).  If recv[q] + r*m*size == send[r] that slot is left
 * as is.  Aligned data moves by bulk copies global -> shared -> global.
 */
rc_status rc_all_gather(const void *const *send, void *const *recv, int p, size_t n,
                        rc_dtype dt, rc_stream_t stream);

/*
 * reduce [SEM] [COLL]: only the root receives the all-reduce result:
 * recv_root[i] = cast(scale * fold_r send[r][i]).  root in [0, p) names the
 * receiving rank (the fold order does not depend on it); recv_root may be
 * send[root] (in place).
 */
rc_status rc_reduce(const void *const *send, void *recv_root, int p, int root, size_t n,
                    rc_dtype dt, rc_op op, float scale, rc_stream_t stream);

/*
 * broadcast [SEM] [COLL]: recv[q][i] = send_root[i] for every q.  root in
 * [0, p); if recv[root] == send_root the root's copy is skipped.
 */
rc_status rc_broadcast(const void *send_root, void *const *recv, int p, int root, size_t n,
                       rc_dtype dt, rc_stream_t stream);

/*
 * ring all-reduce [RING]: same result bits as rc_all_reduce.
 *  RC_RING_LITERAL executes the 2(p-1) steps: reduce-scatter step k, every
 *   rank r sends chunk (r-k-1) mod p to rank r+1, which folds it with its own
 *   chunk; all-gather step k, rank r forwards chunk (r-k) mod p to rank r+1,
 *   which overwrites.  Partials are fp32 (int32 for int32) between steps.
 *   One launch; each thread block runs all 2(p-1) steps on one offset range
 *   of every chunk.  16-byte aligned buffers whose chunk length keeps that
 *   alignment: the block's thread groups are the p ranks and each step's
 *   messages cross link buffers in the block's shared memory (a store by the
 *   sender, a barrier, a load by the receiver), so device memory sees every
 *   input read once and every output written once, and no workspace is used.
 *   Other buffers: partials are kept in the receivers' recv buffers when dt
 *   is fp32/int32, in the library workspace (2 * p * C * 4 bytes) when dt is
 *   bf16.
 *  RC_RING_ONESHOT reads all p ranks directly (the rc_all_reduce kernel).
 */
rc_status rc_ring_all_reduce(const void *const *send, void *const *recv, int p, size_t n,
                             rc_dtype dt, rc_op op, float scale, rc_ring_variant variant,
                             rc_stream_t stream);

/*
 * ring all-reduce that allocates nothing.  The pages have no counterpart of
 * this entry point; it exists for callers that cannot allocate device memory
 * at call time: code whose device memory is owned entirely by another
 * allocator (a framework's caching allocator that must remain the only one),
 * code that must not stall on cudaMalloc/cudaFree (both can synchronise the
 * device), and code running where allocation is not allowed.
 *
 * Same arguments, result bits and literal schedule as rc_ring_all_reduce with
 * RC_RING_LITERAL, executed by the kernel that passes every message through
 * device memory (partials stored by the sender and loaded by the receiver
 * at each step).  For bf16 the fp32 partials live in a fixed scratch array
 * inside this library (16 MiB of device memory, held by every GPU that loads
 * the library until the process exits) instead of the library workspace, so
 * bf16 calls need 2 * p * ceil(n/p) <= 4,194,304; larger requests return
 * RC_ERR_INVALID_ARG with the limit in rc_last_error.  fp32 and int32 keep
 * their partials in recv and use no scratch.
 *  - The first call on a device looks up the scratch array's device address
 *    (once per device, that device current); make that first call before any
 *    stream capture.  rc_finalize forgets the looked-up addresses; a device
 *    reset (cudaDeviceReset) must come after rc_finalize.
 *  - All calls share the one array and it keeps the last call's contents;
 *    calls whose kernels overlap on the GPU (for example on two streams) race
 *    on it.  Nothing in it needs clearing: every partial is written before it
 *    is read.
 *  - Calls no cudaMalloc, cudaFree or allocating library routine.
 */
rc_status rc_ring_all_reduce_noalloc(const void *const *send, void *const *recv, int p, size_t n,
                                     rc_dtype dt, rc_op op, float scale, rc_stream_t stream);

/*
 * hierarchical all-reduce [HIER]: ranks form p/group_size contiguous groups
 * of group_size.  (1) each group's ranks are folded in ring order over the
 * group (chunk length ceil(n/group_size)); (2) the groups' results are folded
 * in ring order over the groups (chunk length ceil(n/(p/group_size))); (3)
 * scale and cast once, and every rank receives the result.  group_size must
 * divide p.  Result bits differ from rc_all_reduce by rounding only (equal
 * for int32, MAX, MIN).
 *  RC_HIER_FUSED: one launch, group results in registers.
 *  RC_HIER_STAGED: three launches (intra-group reduce to fp32 workspace,
 *   leader sum, broadcast); workspace (p/group_size + 1) * n * 4 bytes.
 */
rc_status rc_hier_all_reduce(const void *const *send, void *const *recv, int p, int group_size,
                             size_t n, rc_dtype dt, rc_op op, float scale,
                             rc_hier_variant variant, rc_stream_t stream);

/*
 * All-to-all with split counts [A2A] (MoE dispatch; the combine is the same
 * call with the transposed counts).  counts is a host array of p*p element
 * counts, row-major: counts[r*p + q] elements go from rank r to rank q.
 *  send[r]: rank r's outgoing blocks in destination order q = 0..p-1
 *           (sum_q counts[r*p+q] elements), read.
 *  recv[q]: rank q's incoming blocks in source order r = 0..p-1
 *           (sum_r counts[r*p+q] elements), written.
 * Block (r, q) is copied bit for bit from send[r] + sum_{q'<q} counts[r*p+q']
 * to recv[q] + sum_{r'<r} counts[r'*p+q].  Any dtype (elements are copied).
 * No send buffer may overlap a receive buffer; receive buffers must not
 * overlap one another.  All counts zero: RC_OK, nothing launched.
 */
rc_status rc_all_to_all_v(const void *const *send, void *const *recv, int p, const size_t *counts,
                          rc_dtype dt, rc_stream_t stream);

/* Equal splits: n elements per rank (n % p == 0), counts[r*p+q] = n/p, i.e.
 * recv[q][r*(n/p) + j] = send[r][q*(n/p) + j]. */
rc_status rc_all_to_all(const void *const *send, void *const *recv, int p, size_t n, rc_dtype dt,
                        rc_stream_t stream);

/*
 * Gradient bucketing for data parallelism [DDP] -- a host-side runtime over
 * rc_all_reduce; no kernels of its own.
 *
 * Every simulated rank keeps its gradients in one flat device buffer of
 * sum(numel) elements of dt; tensor t occupies the same element range
 * [off_t, off_t + numel[t]) of every rank's buffer, tensors in the order
 * their gradients become ready.  Buckets are runs of consecutive whole
 * tensors: a bucket takes tensors in order and closes as soon as it holds at
 * least bucket_bytes (bucket_bytes = 0: one bucket per tensor; SIZE_MAX: one
 * bucket for all).  A bucket is reduced by one in-place rc_all_reduce of its
 * slice of every rank's buffer (op SUM, `scale`, e.g. 1/p for the average),
 * so its fold order is that of an all-reduce of the slice.
 */
typedef struct rc_bucketer rc_bucketer;

/* The bucket plan alone (host only, no GPU): bucket_of[t] receives tensor
 * t's bucket index, *nbuckets the count.  elem_bytes > 0. */
rc_status rc_plan_buckets(int ntensors, const size_t *numel, size_t elem_bytes, size_t bucket_bytes,
                          int *bucket_of, int *nbuckets);

/* Create a bucketer for p flat gradient buffers (device memory of the
 * current device, each checked like rc_check_buffer).  The buffers and the
 * communication stream `comm` must outlive the bucketer.  dt RC_INT32
 * requires scale == 1. */
rc_status rc_bucketer_create(rc_bucketer **out, void *const *flat, int p, int ntensors,
                             const size_t *numel, size_t bucket_bytes, rc_dtype dt, float scale,
                             rc_stream_t comm);

/* Inspect the plan: the number of buckets, and bucket k's tensors
 * [first_tensor, end_tensor) and element range (any output may be NULL). */
rc_status rc_bucketer_num_buckets(const rc_bucketer *b, int *nbuckets);
rc_status rc_bucketer_bucket(const rc_bucketer *b, int k, int *first_tensor, int *end_tensor,
                             size_t *first_elem, size_t *nelem);

/* Tensor t's gradients are complete on every rank in the order of stream
 * `producer`: records an event there and makes `comm` wait for it; when t
 * completes its bucket, enqueues the bucket's all-reduce on `comm`.  A tensor
 * marked twice in one step returns RC_ERR_INVALID_ARG. */
rc_status rc_bucketer_ready(rc_bucketer *b, int tensor, rc_stream_t producer);

/* End of the step: `consumer` waits for every all-reduce enqueued so far and
 * the bucketer resets for the next step.  RC_ERR_INVALID_ARG if a bucket was
 * incomplete (a tensor never marked ready; that bucket was not reduced). */
rc_status rc_bucketer_flush(rc_bucketer *b, rc_stream_t consumer);

/* Release the bucketer's events and memory (NULL is a no-op).  Call it after
 * the work it enqueued has been waited for. */
rc_status rc_bucketer_destroy(rc_bucketer *b);

/* AdamW hyperparameters of one optimizer step [ZERO]. */
typedef struct rc_adamw_hparams {
  float lr;
  float beta1;
  float beta2;
  float eps;
  float weight_decay;
  int64_t step; /* t >= 1: the index of this step (bias corrections use it) */
} rc_adamw_hparams;

/*
 * One AdamW step on n elements, in place: [ZERO] names torch.optim.AdamW; the
 * update is AdamW's published definition (decoupled weight decay,
 * bias-corrected moments), evaluated in binary32 with one rounding per
 * operation in exactly this order:
 *   theta <- theta * (1 - lr*wd)
 *   m     <- beta1*m + (1 - beta1)*g
 *   v     <- beta2*v + (1 - beta2)*(g*g)
 *   mhat  <- m / (1 - beta1^t);   vhat <- v / (1 - beta2^t)
 *   theta <- theta - lr * (mhat / (sqrt(vhat) + eps))
 * The scalars 1 - lr*wd, 1 - beta1, 1 - beta2, 1 - beta1^t, 1 - beta2^t are
 * binary64 expressions (C library pow) rounded to binary32 once.
 *  param, exp_avg, exp_avg_sq: n fp32 each, read and written.
 *  grad: n elements of grad_dt (RC_FP32 or RC_BF16, widened exactly), read.
 *  The four buffers must not overlap.  hp->step < 1, a NULL hp or another
 *  grad_dt return RC_ERR_INVALID_ARG.
 */
rc_status rc_adamw_step(float *param, float *exp_avg, float *exp_avg_sq, const void *grad,
                        rc_dtype grad_dt, size_t n, const rc_adamw_hparams *hp, rc_stream_t stream);

/*
 * ZeRO-1 sharded optimizer step [ZERO], [FSDP], [AVG], fused with its
 * collectives in one pass over p simulated ranks (n % p == 0, m = n/p):
 *   g[i]         = scale * (fold of grads[0..p-1][i] in the ring order of
 *                  chunk c = i / m), fp32 accumulate  (the reduce-scatter:
 *                  rank c owns shard c; scale is typically 1/p)
 *   shard c      : rc_adamw_step's update of master[c][j], exp_avg[c][j],
 *                  exp_avg_sq[c][j] with g[c*m + j], j < m
 *   params[q][i] = cast_param(master[c][i - c*m]) for every rank q (the
 *                  all-gather; bf16 is round-to-nearest-even)
 * Bit-identical to rc_reduce_scatter (fp32 out) + rc_adamw_step per shard +
 * rc_all_gather.
 *  grads[r]: n elements of grad_dt (RC_FP32 / RC_BF16), read.
 *  params[q]: n elements of param_dt (RC_FP32 / RC_BF16), written.
 *  master[r], exp_avg[r], exp_avg_sq[r]: m fp32 each (rank r's shard), read
 *  and written.  Output and state buffers must not overlap one another.
 */
rc_status rc_zero1_step(const void *const *grads, void *const *params, float *const *master,
                        float *const *exp_avg, float *const *exp_avg_sq, int p, size_t n,
                        rc_dtype grad_dt, rc_dtype param_dt, float scale,
                        const rc_adamw_hparams *hp, rc_stream_t stream);

/*
 * Rank view [P2P]: one rank's share of a collective, for rank-per-GPU
 * execution -- one process per GPU, each reaching the other ranks' buffers
 * through peer mappings (rc_ipc_import).  The pointer arrays hold the p
 * ranks' buffers as the calling process addresses them: its own buffer at
 * index `rank`, the other ranks' mapped buffers elsewhere.  A pointer may
 * live on another device when the current device can access that device's
 * memory (an imported mapping always can).
 *
 * Calling a rank-view function once for every rank 0..p-1 gives exactly the
 * bits of the corresponding whole collective above (same chunks, same fold
 * order).  The functions do not synchronise the ranks: the caller must make
 * every rank's inputs complete before any rank's call runs, and every rank's
 * call complete before the outputs are read or the inputs reused (for
 * example: synchronise the stream, then a host barrier among the processes).
 * Validation is as for the whole collective.
 */

/* Chunk `rank` of the all-reduce (elements [rank*C, min((rank+1)*C, n)),
 * C = ceil(n/p)): read from the p send buffers, folded in the ring order,
 * scaled, written to the same elements of all p recv buffers.  Traffic per
 * rank: (p-1)/p * n elements read from peers and as many written to them.
 * (The pull form of the one-shot all-reduce, where a rank reads the whole
 * vector from every peer and writes only its own output, is
 * rc_reduce(send, recv_own, p, root = rank, ...).) */
rc_status rc_rank_all_reduce(const void *const *send, void *const *recv, int p, int rank, size_t n,
                             rc_dtype dt, rc_op op, float scale, rc_stream_t stream);

/* recv_own (n/p elements of out_dt) = shard `rank` of the reduce-scatter,
 * read from chunk `rank` of the p send buffers (n elements each, n % p == 0).
 * recv_own may be send[rank] + rank*(n/p) with equal element sizes. */
rc_status rc_rank_reduce_scatter(const void *const *send, void *recv_own, int p, int rank, size_t n,
                                 rc_dtype in_dt, rc_dtype out_dt, rc_op op, float scale,
                                 rc_stream_t stream);

/* recv_own (n elements) = the concatenation of the p shards send[0..p-1]
 * (n/p elements each): every rank pulls the others' shards.  If
 * recv_own + rank*(n/p) == send[rank] the own shard is left in place. */
rc_status rc_rank_all_gather(const void *const *send, void *recv_own, int p, int rank, size_t n,
                             rc_dtype dt, rc_stream_t stream);

/* Step `step` in [0, 2(p-1)) of the literal ring all-reduce [RING], as
 * executed by receiving rank `rank` (p >= 2), which pulls from its
 * predecessor r = rank-1 mod p:
 *  - reduce-scatter step k = step < p-1, chunk c = (rank-k-2) mod p:
 *    partial_rank[c] = msg (+) send[rank][chunk c], where msg is
 *    send[r][chunk c] at k = 0 and r's partial of chunk c after; at
 *    k = p-2 (c == rank) recv[rank][chunk rank] = cast(scale * acc) instead.
 *  - all-gather step k = step - (p-1), chunk c = (rank-k-1) mod p:
 *    recv[rank][chunk c] = recv[r][chunk c].
 * Partials are fp32 (int32 for int32).  For fp32 and int32 they live in the
 * receiver's recv buffer (chunk c); for bf16 in ws[rank], 2*C floats per
 * rank (C = ceil(n/p)), slot step%2.  ws may be NULL unless dt is bf16.
 * Step s of every rank must be complete before any rank starts step s+1;
 * all steps of all ranks give exactly rc_ring_all_reduce(..., LITERAL). */
rc_status rc_rank_ring_step(const void *const *send, void *const *recv, void *const *ws, int p, int rank,
                            int step, size_t n, rc_dtype dt, rc_op op, float scale, rc_stream_t stream);

/*
 * Peer mappings between processes (CUDA IPC) [P2P].  rc_ipc_export describes
 * a device buffer so that another process can map it; rc_ipc_import maps
 * such a description into the calling process (enabling peer access from the
 * current device when the buffer lives on another one) and returns the
 * buffer's address there; rc_ipc_release unmaps it.  The handle is plain
 * bytes and may travel through any channel (a torch.distributed object
 * gather, a file, a socket).
 *
 * A buffer inside a larger allocation (a caching allocator's block) is
 * exported as that allocation plus an offset; importing maps the whole
 * allocation once per process (several imports of buffers in one allocation
 * share the mapping, reference-counted) and returns base + offset.  The
 * exporting process must keep the allocation alive until every importer has
 * released it.  A process cannot import its own export (RC_ERR_INVALID_ARG):
 * use the buffer's own address.
 */
typedef struct {
  unsigned char ipc[64];  /* the driver's IPC handle of the containing allocation */
  uint64_t offset;        /* buffer address - allocation base */
  uint64_t bytes;         /* buffer length */
  int32_t device;         /* exporting device ordinal (in the exporter's numbering) */
  int32_t pid;            /* exporting process */
} rc_ipc_handle;

/* [ptr, ptr+bytes) must be device memory of the current device inside one
 * allocation (rc_check_buffer). */
rc_status rc_ipc_export(const void *ptr, size_t bytes, rc_ipc_handle *out);

/* *ptr = the exported buffer's address in this process. */
rc_status rc_ipc_import(const rc_ipc_handle *h, void **ptr);

/* Drop one import of the buffer at ptr (an address rc_ipc_import returned);
 * the allocation's mapping is closed with its last import.  Synchronises
 * nothing: the caller makes sure no work on the mapping is pending. */
rc_status rc_ipc_release(void *ptr);

/*
 * Plain device copy dst[0, bytes) = src[0, bytes) with this library's
 * streaming kernel: the measured copy roofline the collectives are compared
 * against.  src and dst must not overlap.
 */
rc_status rc_copy(const void *src, void *dst, size_t bytes, rc_stream_t stream);

/* Validate a device range without launching anything: RC_OK when
 * [ptr, ptr + bytes) is device (or managed) memory of the current device
 * inside a single allocation, RC_ERR_INVALID_ARG otherwise (message in
 * rc_last_error).  Every collective runs this check on each buffer. */
rc_status rc_check_buffer(const void *ptr, size_t bytes);

/* Grow the workspace of the current device to at least `bytes` now, so that
 * later calls do not allocate (a call under stream capture cannot).
 * Stream-ordered: the growth waits for the workspace's last user if that was
 * another stream, and the old block is freed in `stream`'s order.  This is
 * why it takes a stream, unlike a size-only reservation: the workspace is
 * allocated with cudaMallocAsync, and growing it must not free a block that
 * work still queued on another stream is using.  Pass 0 for the legacy
 * default stream.
 * A block that a stream capture has used is never freed before rc_finalize:
 * the captured graph holds its address and may be replayed after a later
 * call grew the workspace, so growth retires such a block (it stays
 * allocated, see rc_workspace_bytes) instead of freeing it.  Call
 * rc_finalize only when no graph that captured a call of this library will
 * be launched again. */
rc_status rc_reserve_workspace(size_t bytes, rc_stream_t stream);

/* Bytes of the current device's workspace: *live = the block calls use now,
 * *retired = blocks kept alive for captured graphs (freed by rc_finalize). */
rc_status rc_workspace_bytes(size_t *live, size_t *retired);

/* Synchronise `stream`, then report: RC_ERR_CUDA for an asynchronous CUDA
 * error, RC_ERR_TIMEOUT if a bounded device wait of this library gave up
 * since the last call (the flag is cleared), else RC_OK. */
rc_status rc_stream_status(rc_stream_t stream);

/* Failure-path self test: launches one kernel whose single thread waits on a
 * barrier phase that nothing completes.  The wait is bounded like every wait
 * in this library: after limit_ns (0 < limit_ns <= 1e9) it gives up, records
 * the event and returns, so the context stays usable and the next
 * rc_stream_status(stream) returns RC_ERR_TIMEOUT. */
rc_status rc_probe_bounded_wait(uint64_t limit_ns, rc_stream_t stream);

/* Static description of a status code. */
const char *rc_status_string(rc_status status);

/* Text of the last error raised on the calling host thread ("" if none). */
const char *rc_last_error(void);

/* Number of kernels this library has launched in this process. */
uint64_t rc_launch_count(void);

/* Free every workspace, retired blocks included (synchronises the devices
 * that own one), and forget the fixed scratch's looked-up addresses. */
rc_status rc_finalize(void);

/* Library version, major*10000 + minor*100 + patch. */
int rc_version(void);

#ifdef __cplusplus
}
#endif

#endif /* RANKCOLL_H */
