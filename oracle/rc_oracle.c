/*
 * rc_oracle.c -- plain, slow, single-threaded CPU oracle for the simulated-rank
 * collectives.  TEST INFRASTRUCTURE ONLY: it exists to check the CUDA library.
 * Only tests/, __graft_entry__.smoke() and bench.py's cpu_baseline /
 * reference leg may load it.  It shares no code, header, table or constant
 * with the CUDA library (collective_rc_all_b200/csrc) and never calls it.
 *
 * Sources (page title, section):
 *  [P2-SEM]  "分布式训练/推理" (llm-from-scratch ch. 7), section
 *            "通信原语：rank、world size 和 collective operations": primitive
 *            table (broadcast, reduce with sum/min/max, all-gather,
 *            reduce-scatter, all-reduce), the equation y = sum_r x_r, the worked
 *            example x_r = [0,1,2,3]+r -> [6,10,14,18], and the identity
 *            all_reduce = reduce_scatter + all_gather.
 *  [P2-API]  same page, "PyTorch distributed：代码里真正发生了什么": all_reduce is
 *            in place, reduce_scatter / all_gather write a separate output;
 *            reduce_scatter input is world_size x k per rank.
 *  [P2-DP]   same page, "数据并行：切 batch，复制模型": g = (1/p) sum_r grad L_r,
 *            ReduceOp.AVG (a scale applied to the sum).
 *  [P2-FSDP] same page, "FSDP 的执行顺序": all_gather of W_i shards before the
 *            module, reduce_scatter of (1/N_d) sum_r grad W^(r) after backward.
 *  [P4-COLL] "LLM Parallelism 基础", sections "AllReduce" and "其他 Collective":
 *            Reduce/Broadcast/AllGather/ReduceScatter semantics and
 *            "AllReduce = Reduce + Broadcast" in effect.
 *  [P4-RING] same page, "Ring AllReduce": N chunks, phase 1 reduce-scatter (each
 *            card sends one chunk to the next card, which accumulates it into its
 *            own matching chunk; after N-1 steps card 0 holds chunk 0 ...),
 *            phase 2 all-gather (each card forwards its finished chunk to the
 *            next card, which overwrites), 2(N-1) steps in total.
 *  [P2-ZERO] "分布式训练/推理", sections "DDP 模型训练示例" (ShardedOptimizer:
 *            average the gradients, run AdamW on the parameters this rank owns,
 *            broadcast every parameter from its owner) and "显存账：不同数据并行的
 *            局限性" (ZeRO-1 shards the optimizer state: the Adam moments and the
 *            fp32 master weights).  The pages name torch.optim.AdamW without
 *            printing it; the update below is AdamW's published definition.
 *  [P2-A2A]  "分布式训练/推理", primitive table: all-to-all -- every rank sends a
 *            different slice to every rank (MoE token routing); section "从路由
 *            结果到专家输出" (dispatch = the exchange towards the experts, combine
 *            = the way back; split counts tell a receiver how much arrives) and
 *            section "为什么 top-k 和 EP degree 会直接放大通信" (payload t*k*h*b
 *            per phase, of which t*k*h*b*(p-1)/p leaves the rank when routing is
 *            balanced).
 *  [P1-HIER] "大模型并行的最小闭环：集合通信、TP、FSDP/ZeRO-3 到权重分片", log excerpt
 *            "分层 AllReduce + SHARP": 2 nodes x 4 GPUs, B per GPU; step 1 intra-node
 *            AllReduce, step 2 one representative (GPU0) per node, step 3 uplink B
 *            per node, step 4 switch computes A+B, step 5 downlink, step 6
 *            intra-node broadcast; traffic B x N = 32 MB inside a node, B instead
 *            of B x N across nodes.
 *
 * Readings taken where the pages are silent (each one is listed in the design
 * notes with its reason):
 *  R1 reduction order: every reducing collective folds ranks in the order the
 *     literal ring of [P4-RING] produces.  Chunk size C = ceil(n/p); element i
 *     is in chunk c = i / C; chunk c is folded as
 *       acc = x_{(c+1)%p}; acc = acc (+) x_{(c+2)%p}; ... ; acc = acc (+) x_{c}.
 *  R2 floating point: fp32 accumulation in IEEE binary32 round-to-nearest-even;
 *     bf16 inputs are widened exactly; `scale` is one fp32 multiply after the
 *     fold; bf16 outputs are one round-half-to-even narrowing at the end.
 *  R3 the fold starts from the first operand (never from 0), so -0 survives.
 *  R4 int32 SUM wraps (two's complement); MAX/MIN are compare-selects
 *     acc = (v > acc) ? v : acc and acc = (v < acc) ? v : acc.
 *  R5 hierarchical groups are contiguous blocks of G ranks; the intra-group
 *     step is a ring over the group (so its order is R1 with q = G); the
 *     leader (local rank 0) sums the group results in ring order over the
 *     groups (q = p/G); scale and cast happen once, after the leader sum.
 *  R6 AdamW (rco_adamw): binary32, each operation rounded once, in the order
 *     written there; the scalars 1 - lr*wd, 1 - beta1, 1 - beta2, 1 - beta1^t
 *     and 1 - beta2^t are evaluated in binary64 (the C library's pow) and
 *     rounded to binary32 once.
 *
 * Build: gcc -O2 -std=c11 -ffp-contract=off -fno-fast-math (oracle/build.py).
 * x86-64 float arithmetic is SSE binary32, so every `float` operation below is
 * one correctly rounded IEEE operation.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* Codes of the oracle's own interface (mirrored by oracle/__init__.py). */
#define RCO_F32 0
#define RCO_BF16 1
#define RCO_I32 2

#define RCO_SUM 0
#define RCO_MAX 1
#define RCO_MIN 2

#define RCO_OK 0
#define RCO_EINVAL 1
#define RCO_ENOMEM 2

/* ------------------------------------------------------------------------ */
/* bf16 <-> fp32 from the IEEE-754 definitions.                              */
/* bf16 is the top half of a binary32.  Narrowing keeps the top 16 bits and   */
/* rounds on the 16 dropped bits: up when they exceed one half, to the even   */
/* neighbour when they are exactly one half.  A carry out of the mantissa     */
/* moves into the exponent, which is the correct rounded value (up to inf).  */
/* NaN stays NaN (quiet bit forced so that truncation cannot make it inf).   */
/* ------------------------------------------------------------------------ */
uint16_t rco_f32_to_bf16(float f)
{
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    if ((u & 0x7f800000u) == 0x7f800000u && (u & 0x007fffffu) != 0u)
        return (uint16_t)((u >> 16) | 0x0040u);
    uint32_t hi = u >> 16;
    uint32_t lo = u & 0xffffu;
    if (lo > 0x8000u || (lo == 0x8000u && (hi & 1u) != 0u))
        hi += 1u;
    return (uint16_t)hi;
}

float rco_bf16_to_f32(uint16_t h)
{
    uint32_t u = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

void rco_f32_to_bf16_n(const float *x, uint16_t *y, size_t n)
{
    for (size_t i = 0; i < n; ++i)
        y[i] = rco_f32_to_bf16(x[i]);
}

static size_t dt_size(int dt)
{
    return dt == RCO_BF16 ? 2u : 4u;
}

static int dt_valid(int dt) { return dt == RCO_F32 || dt == RCO_BF16 || dt == RCO_I32; }
static int op_valid(int op) { return op == RCO_SUM || op == RCO_MAX || op == RCO_MIN; }

/* A value being reduced: fp32 for the float types, int32 for int32. */
typedef struct {
    float f;
    int32_t i;
} acc_t;

static acc_t load_elem(const void *base, size_t i, int dt)
{
    acc_t a = {0.0f, 0};
    if (dt == RCO_F32) {
        a.f = ((const float *)base)[i];
    } else if (dt == RCO_BF16) {
        a.f = rco_bf16_to_f32(((const uint16_t *)base)[i]);
    } else {
        a.i = ((const int32_t *)base)[i];
    }
    return a;
}

/* acc (+) v for one element, [P2-SEM] "sum、min、max" and readings R2, R4. */
static acc_t combine(acc_t acc, acc_t v, int is_int, int op)
{
    if (is_int) {
        if (op == RCO_SUM)
            acc.i = (int32_t)((uint32_t)acc.i + (uint32_t)v.i);
        else if (op == RCO_MAX)
            acc.i = (v.i > acc.i) ? v.i : acc.i;
        else
            acc.i = (v.i < acc.i) ? v.i : acc.i;
    } else {
        if (op == RCO_SUM)
            acc.f = acc.f + v.f;
        else if (op == RCO_MAX)
            acc.f = (v.f > acc.f) ? v.f : acc.f;
        else
            acc.f = (v.f < acc.f) ? v.f : acc.f;
    }
    return acc;
}

/* Final step of every reducing collective: one fp32 multiply by `scale`,
 * then the cast to the output type (reading R2).  int32 is stored as is. */
static void store_result(void *base, size_t i, int out_dt, acc_t acc, float scale)
{
    if (out_dt == RCO_I32) {
        ((int32_t *)base)[i] = acc.i;
        return;
    }
    float y = acc.f * scale;
    if (out_dt == RCO_F32)
        ((float *)base)[i] = y;
    else
        ((uint16_t *)base)[i] = rco_f32_to_bf16(y);
}

/* Argument rules shared by every reducing entry point. */
static int check_reduce_args(int p, int in_dt, int out_dt, int op, float scale)
{
    if (p < 1 || p > 64 || !dt_valid(in_dt) || !dt_valid(out_dt) || !op_valid(op))
        return RCO_EINVAL;
    if ((in_dt == RCO_I32) != (out_dt == RCO_I32))
        return RCO_EINVAL;
    if ((in_dt == RCO_I32 || op != RCO_SUM) && scale != 1.0f)
        return RCO_EINVAL;
    return RCO_OK;
}

/* ------------------------------------------------------------------------ */
/* The direct definition: y[i] = cast(scale * fold over ranks in ring order) */
/* (reading R1).                                                              */
/* ------------------------------------------------------------------------ */
static acc_t fold_ring_order(const void *const *x, int q, size_t n, size_t i, int dt, int op)
{
    size_t C = (n + (size_t)q - 1) / (size_t)q; /* chunk length */
    size_t c = i / C;                           /* chunk that holds element i */
    int is_int = (dt == RCO_I32);
    int r = (int)((c + 1) % (size_t)q);
    acc_t acc = load_elem(x[r], i, dt);
    for (int k = 1; k < q; ++k) {
        r = (int)((c + 1 + (size_t)k) % (size_t)q);
        acc = combine(acc, load_elem(x[r], i, dt), is_int, op);
    }
    return acc;
}

/* all-reduce [P2-SEM], [P4-COLL]: every rank receives y. */
int rco_all_reduce(const void *const *send, void *const *recv, int p, size_t n,
                   int dt, int op, float scale)
{
    int e = check_reduce_args(p, dt, dt, op, scale);
    if (e)
        return e;
    if (n == 0)
        return RCO_OK;
    float *yf = NULL;
    int32_t *yi = NULL;
    /* Results go to a private buffer first, so in-place calls read unmodified
     * inputs for every element. */
    if (dt == RCO_I32)
        yi = (int32_t *)malloc(n * sizeof(int32_t));
    else
        yf = (float *)malloc(n * sizeof(float));
    if (!yf && !yi)
        return RCO_ENOMEM;
    for (size_t i = 0; i < n; ++i) {
        acc_t a = fold_ring_order(send, p, n, i, dt, op);
        if (yi)
            yi[i] = a.i;
        else
            yf[i] = a.f;
    }
    for (int r = 0; r < p; ++r) {
        for (size_t i = 0; i < n; ++i) {
            acc_t a = {0.0f, 0};
            if (yi)
                a.i = yi[i];
            else
                a.f = yf[i];
            store_result(recv[r], i, dt, a, scale);
        }
    }
    free(yf);
    free(yi);
    return RCO_OK;
}

/* reduce-scatter [P2-SEM], [P2-API], [P2-FSDP]: rank r keeps elements
 * [r*m, (r+1)*m) of the reduced vector, m = n/p, cast to out_dt. */
int rco_reduce_scatter(const void *const *send, void *const *recv, int p, size_t n,
                       int in_dt, int out_dt, int op, float scale)
{
    int e = check_reduce_args(p, in_dt, out_dt, op, scale);
    if (e)
        return e;
    if (n % (size_t)p != 0)
        return RCO_EINVAL;
    size_t m = n / (size_t)p;
    for (int r = 0; r < p; ++r) {
        for (size_t j = 0; j < m; ++j) {
            size_t i = (size_t)r * m + j;
            acc_t a = fold_ring_order(send, p, n, i, in_dt, op);
            store_result(recv[r], j, out_dt, a, scale);
        }
    }
    return RCO_OK;
}

/* all-gather [P2-SEM], [P2-FSDP]: out_q[r*m + j] = in_r[j] for every q. */
int rco_all_gather(const void *const *send, void *const *recv, int p, size_t n, int dt)
{
    if (p < 1 || p > 64 || !dt_valid(dt) || n % (size_t)p != 0)
        return RCO_EINVAL;
    size_t m = n / (size_t)p, s = dt_size(dt);
    for (int q = 0; q < p; ++q)
        for (int r = 0; r < p; ++r)
            memmove((char *)recv[q] + (size_t)r * m * s, send[r], m * s);
    return RCO_OK;
}

/* reduce [P2-SEM] "结果到一个 rank", [P4-COLL]: only the root receives y. */
int rco_reduce(const void *const *send, void *recv_root, int p, int root, size_t n,
               int dt, int op, float scale)
{
    int e = check_reduce_args(p, dt, dt, op, scale);
    if (e)
        return e;
    if (root < 0 || root >= p)
        return RCO_EINVAL;
    void *one[1] = {recv_root};
    /* identical to all-reduce restricted to one output buffer */
    if (n == 0)
        return RCO_OK;
    float *yf = NULL;
    int32_t *yi = NULL;
    if (dt == RCO_I32)
        yi = (int32_t *)malloc(n * sizeof(int32_t));
    else
        yf = (float *)malloc(n * sizeof(float));
    if (!yf && !yi)
        return RCO_ENOMEM;
    for (size_t i = 0; i < n; ++i) {
        acc_t a = fold_ring_order(send, p, n, i, dt, op);
        if (yi)
            yi[i] = a.i;
        else
            yf[i] = a.f;
    }
    for (size_t i = 0; i < n; ++i) {
        acc_t a = {0.0f, 0};
        if (yi)
            a.i = yi[i];
        else
            a.f = yf[i];
        store_result(one[0], i, dt, a, scale);
    }
    free(yf);
    free(yi);
    return RCO_OK;
}

/* broadcast [P2-SEM], [P4-COLL]: every rank receives the root's tensor. */
int rco_broadcast(const void *send_root, void *const *recv, int p, int root, size_t n, int dt)
{
    if (p < 1 || p > 64 || !dt_valid(dt) || root < 0 || root >= p)
        return RCO_EINVAL;
    for (int q = 0; q < p; ++q)
        memmove(recv[q], send_root, n * dt_size(dt));
    return RCO_OK;
}

/* Reduced values at selected indices only: out[j] = y[idx[j]] in out_dt.
 * Lets tests check full-size GPU results on samples. */
int rco_reduce_at(const void *const *send, int p, size_t n, int in_dt, int out_dt,
                  int op, float scale, const uint64_t *idx, size_t k, void *out)
{
    int e = check_reduce_args(p, in_dt, out_dt, op, scale);
    if (e)
        return e;
    for (size_t j = 0; j < k; ++j) {
        if (idx[j] >= n)
            return RCO_EINVAL;
        acc_t a = fold_ring_order(send, p, n, (size_t)idx[j], in_dt, op);
        store_result(out, j, out_dt, a, scale);
    }
    return RCO_OK;
}

/* ------------------------------------------------------------------------ */
/* Literal ring all-reduce [P4-RING], simulated step by step.               */
/*                                                                          */
/* Rank r works on a private copy w_r of its data (fp32 for float types,     */
/* int32 for int32).  Reduce-scatter step k (k = 0..q-2): every rank r sends */
/* chunk (r-k-1) mod q of w_r to rank r+1; the receiver folds the message    */
/* with its own matching chunk:  w_{r+1}[c] = msg (+) w_{r+1}[c].  After q-1 */
/* steps rank r holds the finished chunk r.  It applies scale and the cast   */
/* to its output buffer.  All-gather step k: rank r sends chunk (r-k) mod q  */
/* of its output to rank r+1, which overwrites its own copy.                 */
/* All q sends of one step are taken from the state before that step         */
/* (messages are copied out first), as on a real ring.                       */
/*                                                                          */
/* msgs_elems[r] (if not NULL, length q) counts elements rank r sent;        */
/* *steps_out (if not NULL) counts communication steps.                      */
/* ------------------------------------------------------------------------ */
static size_t chunk_begin(size_t C, size_t n, size_t c)
{
    size_t b = c * C;
    return b < n ? b : n;
}

static int ring_core(const void *const *x, int q, size_t n, int dt, int op,
                     acc_t *out_acc /* n values, the reduced vector as fp32/int32 */,
                     uint64_t *msgs_elems, uint64_t *steps_out)
{
    size_t C = (n + (size_t)q - 1) / (size_t)q;
    int is_int = (dt == RCO_I32);
    acc_t **w = (acc_t **)calloc((size_t)q, sizeof(acc_t *));
    acc_t **msg = (acc_t **)calloc((size_t)q, sizeof(acc_t *));
    int ok = (w != NULL && msg != NULL);
    for (int r = 0; ok && r < q; ++r) {
        w[r] = (acc_t *)malloc((n ? n : 1) * sizeof(acc_t));
        msg[r] = (acc_t *)malloc((C ? C : 1) * sizeof(acc_t));
        ok = (w[r] != NULL && msg[r] != NULL);
    }
    if (!ok) {
        for (int r = 0; w && msg && r < q; ++r) {
            free(w[r]);
            free(msg[r]);
        }
        free(w);
        free(msg);
        return RCO_ENOMEM;
    }
    for (int r = 0; r < q; ++r)
        for (size_t i = 0; i < n; ++i)
            w[r][i] = load_elem(x[r], i, dt);
    uint64_t steps = 0;

    /* phase 1: reduce-scatter, q-1 steps */
    for (int k = 0; k < q - 1; ++k) {
        for (int r = 0; r < q; ++r) { /* every rank packs its message */
            size_t c = (size_t)(((r - k - 1) % q + q) % q);
            size_t b = chunk_begin(C, n, c), e = chunk_begin(C, n, c + 1);
            for (size_t i = b; i < e; ++i)
                msg[r][i - b] = w[r][i];
            if (msgs_elems)
                msgs_elems[r] += (uint64_t)(e - b);
        }
        for (int r = 0; r < q; ++r) { /* rank r+1 folds what rank r sent */
            int d = (r + 1) % q;
            size_t c = (size_t)(((r - k - 1) % q + q) % q);
            size_t b = chunk_begin(C, n, c), e = chunk_begin(C, n, c + 1);
            for (size_t i = b; i < e; ++i)
                w[d][i] = combine(msg[r][i - b], w[d][i], is_int, op);
        }
        ++steps;
    }
    /* rank r now owns the reduced chunk r; hand the owners' chunks out */
    for (int r = 0; r < q; ++r) {
        size_t b = chunk_begin(C, n, (size_t)r), e = chunk_begin(C, n, (size_t)r + 1);
        for (size_t i = b; i < e; ++i)
            out_acc[i] = w[r][i];
    }
    for (int r = 0; r < q; ++r) {
        free(w[r]);
        free(msg[r]);
    }
    free(w);
    free(msg);
    if (steps_out)
        *steps_out += steps;
    return RCO_OK;
}

int rco_ring_all_reduce(const void *const *send, void *const *recv, int p, size_t n,
                        int dt, int op, float scale, uint64_t *msgs_elems, uint64_t *steps_out)
{
    int e = check_reduce_args(p, dt, dt, op, scale);
    if (e)
        return e;
    if (n == 0)
        return RCO_OK;
    size_t C = (n + (size_t)p - 1) / (size_t)p, s = dt_size(dt);
    acc_t *red = (acc_t *)malloc(n * sizeof(acc_t));
    char **out = (char **)calloc((size_t)p, sizeof(char *));
    if (!red || !out) {
        free(red);
        free(out);
        return RCO_ENOMEM;
    }
    e = ring_core(send, p, n, dt, op, red, msgs_elems, steps_out);
    if (e) {
        free(red);
        free(out);
        return e;
    }
    /* owners apply scale + cast into their own output copies (private buffers
     * so an in-place call cannot disturb the simulation) */
    for (int r = 0; r < p; ++r) {
        out[r] = (char *)malloc(n * s);
        if (!out[r]) {
            for (int t = 0; t < r; ++t)
                free(out[t]);
            free(out);
            free(red);
            return RCO_ENOMEM;
        }
        size_t b = chunk_begin(C, n, (size_t)r), en = chunk_begin(C, n, (size_t)r + 1);
        for (size_t i = b; i < en; ++i)
            store_result(out[r], i, dt, red[i], scale);
    }
    /* phase 2: all-gather, p-1 steps, receiver overwrites */
    char *msg = (char *)malloc((C ? C : 1) * s * (size_t)p);
    if (!msg) {
        for (int r = 0; r < p; ++r)
            free(out[r]);
        free(out);
        free(red);
        return RCO_ENOMEM;
    }
    for (int k = 0; k < p - 1; ++k) {
        for (int r = 0; r < p; ++r) {
            size_t c = (size_t)(((r - k) % p + p) % p);
            size_t b = chunk_begin(C, n, c), en = chunk_begin(C, n, c + 1);
            memcpy(msg + (size_t)r * C * s, out[r] + b * s, (en - b) * s);
            if (msgs_elems)
                msgs_elems[r] += (uint64_t)(en - b);
        }
        for (int r = 0; r < p; ++r) {
            int d = (r + 1) % p;
            size_t c = (size_t)(((r - k) % p + p) % p);
            size_t b = chunk_begin(C, n, c), en = chunk_begin(C, n, c + 1);
            memcpy(out[d] + b * s, msg + (size_t)r * C * s, (en - b) * s);
        }
        if (steps_out)
            *steps_out += 1;
    }
    for (int r = 0; r < p; ++r) {
        memcpy(recv[r], out[r], n * s);
        free(out[r]);
    }
    free(msg);
    free(out);
    free(red);
    return RCO_OK;
}

/* ------------------------------------------------------------------------ */
/* Hierarchical all-reduce [P1-HIER], simulated phase by phase (reading R5). */
/*                                                                          */
/* traffic (if not NULL, 4 entries, in elements of the input type):         */
/*   [0] data entering the intra-group step, summed over groups (B x N per  */
/*       node in the page's example)                                        */
/*   [1] uplink volume per group: one leader sends one vector (B)           */
/*   [2] cross-group volume per group if every rank went across (B x N)     */
/*   [3] intra-group broadcast volume, summed over groups                   */
/* ------------------------------------------------------------------------ */
int rco_hier_all_reduce(const void *const *send, void *const *recv, int p, int G, size_t n,
                        int dt, int op, float scale, uint64_t *traffic)
{
    int e = check_reduce_args(p, dt, dt, op, scale);
    if (e)
        return e;
    if (G < 1 || p % G != 0)
        return RCO_EINVAL;
    if (n == 0)
        return RCO_OK;
    int ng = p / G;
    int is_int = (dt == RCO_I32);
    acc_t **S = (acc_t **)calloc((size_t)ng, sizeof(acc_t *));
    if (!S)
        return RCO_ENOMEM;
    for (int g = 0; g < ng; ++g) {
        S[g] = (acc_t *)malloc(n * sizeof(acc_t));
        if (!S[g]) {
            for (int t = 0; t < g; ++t)
                free(S[t]);
            free(S);
            return RCO_ENOMEM;
        }
    }
    /* step 1: intra-group all-reduce as a ring over the group's G ranks; the
     * leader (local rank 0) keeps the group result S_g */
    for (int g = 0; g < ng; ++g) {
        e = ring_core(send + (size_t)g * (size_t)G, G, n, dt, op, S[g], NULL, NULL);
        if (e) {
            for (int t = 0; t < ng; ++t)
                free(S[t]);
            free(S);
            return e;
        }
        if (traffic)
            traffic[0] += (uint64_t)G * n;
    }
    /* steps 2-5: each group's leader sends S_g up; the groups' results are
     * combined in ring order over the ng groups (for two groups: A + B) */
    if (traffic) {
        traffic[1] += (uint64_t)n;
        traffic[2] += (uint64_t)G * n;
    }
    size_t Cg = (n + (size_t)ng - 1) / (size_t)ng;
    acc_t *T = (acc_t *)malloc(n * sizeof(acc_t));
    if (!T) {
        for (int t = 0; t < ng; ++t)
            free(S[t]);
        free(S);
        return RCO_ENOMEM;
    }
    for (size_t i = 0; i < n; ++i) {
        size_t c = i / Cg;
        int g = (int)((c + 1) % (size_t)ng);
        acc_t acc = S[g][i];
        for (int k = 1; k < ng; ++k) {
            g = (int)((c + 1 + (size_t)k) % (size_t)ng);
            acc = combine(acc, S[g][i], is_int, op);
        }
        T[i] = acc;
    }
    /* step 6: every leader broadcasts the final vector inside its group;
     * scale and cast are applied once */
    for (int r = 0; r < p; ++r)
        for (size_t i = 0; i < n; ++i)
            store_result(recv[r], i, dt, T[i], scale);
    if (traffic)
        traffic[3] += (uint64_t)(p - ng) * n;
    free(T);
    for (int g = 0; g < ng; ++g)
        free(S[g]);
    free(S);
    return RCO_OK;
}

/* ------------------------------------------------------------------------ */
/* AdamW, one step on n elements [P2-ZERO], in place.                        */
/* Definition (decoupled weight decay, bias-corrected moments), step t >= 1:  */
/*   theta <- theta * (1 - lr*wd)                                            */
/*   m     <- beta1*m + (1 - beta1)*g                                        */
/*   v     <- beta2*v + (1 - beta2)*(g*g)                                    */
/*   mhat  <- m / (1 - beta1^t)          vhat <- v / (1 - beta2^t)            */
/*   theta <- theta - lr * (mhat / (sqrt(vhat) + eps))                       */
/* Reading R6: every line is evaluated left to right in binary32, one        */
/* rounding per operation; the five scalars in parentheses that do not       */
/* involve m, v, g or theta are binary64 expressions rounded once.            */
/* g is fp32 (grad_dt RCO_F32) or bf16 bits (RCO_BF16), widened exactly.      */
int rco_adamw(float *theta, float *m, float *v, const void *g, int grad_dt, size_t n,
              float lr, float beta1, float beta2, float eps, float wd, int64_t t)
{
    if (t < 1 || (grad_dt != RCO_F32 && grad_dt != RCO_BF16))
        return RCO_EINVAL;
    const float decay = (float)(1.0 - (double)lr * (double)wd);
    const float omb1 = (float)(1.0 - (double)beta1);
    const float omb2 = (float)(1.0 - (double)beta2);
    const float bc1 = (float)(1.0 - pow((double)beta1, (double)t));
    const float bc2 = (float)(1.0 - pow((double)beta2, (double)t));
    for (size_t i = 0; i < n; ++i) {
        float gi = grad_dt == RCO_F32 ? ((const float *)g)[i]
                                      : rco_bf16_to_f32(((const uint16_t *)g)[i]);
        float th = theta[i] * decay;
        float mi = beta1 * m[i] + omb1 * gi;
        float vi = beta2 * v[i] + omb2 * (gi * gi);
        float mhat = mi / bc1;
        float vhat = vi / bc2;
        float den = sqrtf(vhat) + eps;
        th = th - lr * (mhat / den);
        theta[i] = th;
        m[i] = mi;
        v[i] = vi;
    }
    return RCO_OK;
}

/* ------------------------------------------------------------------------ */
/* all-to-all with split counts [P2-A2A].                                     */
/* counts[r*p + q] = elements rank r sends to rank q.  Rank r's send buffer   */
/* holds its p outgoing blocks in destination order q = 0..p-1; rank q's      */
/* receive buffer holds its p incoming blocks in source order r = 0..p-1:     */
/*   send offset of block (r,q) = sum_{q' < q} counts[r*p + q']                */
/*   recv offset of block (r,q) = sum_{r' < r} counts[r'*p + q]                */
/* Each block is copied bit for bit.  traffic (optional, 2 counters, bytes):  */
/* [0] blocks that stay on their rank (r == q), [1] blocks that cross ranks.  */
int rco_all_to_all_v(const void *const *send, void *const *recv, int p, const uint64_t *counts,
                     int esz, uint64_t *traffic)
{
    if (p < 1 || p > 64 || (esz != 1 && esz != 2 && esz != 4 && esz != 8) || !counts)
        return RCO_EINVAL;
    for (int r = 0; r < p; ++r) {
        for (int q = 0; q < p; ++q) {
            uint64_t soff = 0, roff = 0;
            for (int k = 0; k < q; ++k)
                soff += counts[(size_t)r * p + k];
            for (int k = 0; k < r; ++k)
                roff += counts[(size_t)k * p + q];
            uint64_t c = counts[(size_t)r * p + q];
            memcpy((char *)recv[q] + roff * (uint64_t)esz, (const char *)send[r] + soff * (uint64_t)esz,
                   c * (uint64_t)esz);
            if (traffic)
                traffic[r == q ? 0 : 1] += c * (uint64_t)esz;
        }
    }
    return RCO_OK;
}
