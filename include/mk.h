/*
 * mk.h -- C ABI of the B200 persistent decode megakernel.
 *
 * One call of mk_decode_step runs the single-token decode step of a
 * Llama-style decoder for up to max_batch independent sequences as ONE
 * persistent kernel launch on a B200 (sm_100a); mk_generate runs a prompt
 * and a greedy generation in one launch.  Inside the launch, a static task
 * graph built by mk_create splits the rows of every matrix-vector op into
 * per-SM tasks, each bumping its op's event counter in global memory (no
 * grid-wide barrier between layers).  A task starts when its inputs exist:
 * by default the workers poll the step-tagged activation words they read;
 * with MK_FLAG_EVENT_WAIT a scheduler warp per SM first waits for the
 * dependency's counter to reach its threshold.  A loader warp per SM streams
 * the weights of upcoming tasks into paged shared memory ahead of their
 * dependencies, and worker warps run the fused task bodies.
 *
 * Where the operations are defined (reference pages on the persistent
 * decode megakernel topic):
 *  - task / event model (a task runs on one SM, bumps its triggering event
 *    when done; a task may start once its dependent event has fired, i.e.
 *    its counter reached the threshold): "显著提升小LLM的性能，所有kernel集成一个
 *    巨大kernel！" (zejuncao.github.io, 2025-06-26), Figure 2 and Figure 3 text;
 *  - worker loop (fetch task, run, notify) and scheduler warps: same page,
 *    MPK runtime section; warp specialisation: zizhi168.cn/news/174794,
 *    section 2.2;
 *  - fused ops of one decoder layer and the model tail: the Hazy megakernel
 *    news page (sfrk.com.cn/ruanjian/202506/86466), paragraph listing the
 *    fused instructions, and the MPK walkthrough's per-layer *_layer calls
 *    (zizhi168.cn/news/174794, section 3.3.1);
 *  - paged shared memory with early weight preload: the Hazy page, paragraph
 *    on static plans and paged shared memory.
 *
 * Conventions for every entry point:
 *  - Pointers documented "device" must be device pointers of the current
 *    CUDA device; "host" pointers are ordinary host memory.
 *  - The caller owns every weight, KV-cache, token, position and output
 *    buffer and keeps it alive while a context that uses it exists; the
 *    library never frees them.  The library owns its scratch (activations,
 *    partial results, event counters, task tables, error word, trace).
 *  - Return value: MK_OK (0) or one of the MK_ERR_* codes below;
 *    mk_status_string() names them.  Invalid arguments are reported
 *    synchronously with MK_ERR_INVALID and nothing is launched.
 */
#ifndef MK_H
#define MK_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* A cudaStream_t (NULL = the legacy default stream). */
typedef struct CUstream_st *mk_stream_t;

enum mk_status {
    MK_OK = 0,
    MK_ERR_INVALID = 1,  /* bad argument or unsupported shape             */
    MK_ERR_CUDA = 2,     /* a CUDA runtime call failed                     */
    MK_ERR_TIMEOUT = 3,  /* a device-side wait exceeded timeout_ns         */
    MK_ERR_OOM = 4,      /* device or pinned host allocation failed        */
    MK_ERR_STATE = 5     /* context unusable after an earlier device error */
};

enum mk_flags {
    MK_FLAG_TRACE = 1,          /* record a per-task timing trace (globaltimer) */
    MK_FLAG_NO_L2_PREFETCH = 2, /* no L2 prefetch whatever l2_lookahead_kb says */
    /* Gate every task on its dependency's event counter (a scheduler warp
     * spins until counter >= threshold * epoch, the scheduling of MPK's
     * event model, "显著提升小LLM的性能..." page, Figure 3 text).  Without
     * it tasks wait on their inputs directly: every activation is stored
     * with the step's tag in the same 64-bit word and readers poll the tags.
     * Results are identical either way; the counters are bumped either way. */
    MK_FLAG_EVENT_WAIT = 4,
    /* Stream every weight page through shared memory only.  By default the
     * pages of the matrix-vector ops whose rows are multiples of 2048
     * columns (hidden, n_q_heads*head_dim or ffn of 2048, 4096 or 8192) are
     * copied on from the shared-memory ring into tensor memory as soon as
     * they land, which frees the ring for further prefetch (7 pages of
     * 64 KB buffered per SM instead of 3); mk_create then keeps those
     * weights in a library-owned copy laid out for that copy. */
    MK_FLAG_NO_TMEM_RING = 8,
    /* Run steps on the batched tensor-core kernel even with max_batch = 1,
     * which mk_prefill needs (contexts with max_batch > 1 always use it).
     * See "Batched steps" below. */
    MK_FLAG_ROWS = 16,
    /* Work items of the attention op (scaled dot-product attention over the
     * KV cache, split into chunks of positions whose partial softmax states
     * are merged exactly -- the chunked attention of the Flash-Decoding
     * scheme the "Mirage Persistent Kernel" page's attention tasks follow).
     * With MK_FLAG_ATTN_KV_ITEMS an item is (sequence, KV head, chunk) and
     * computes every q head that shares the KV head (up to 512 / head_dim
     * of them: a larger group is split), reading each K/V page once; with
     * MK_FLAG_ATTN_Q_ITEMS an item is (sequence, q head, chunk).  Neither:
     * KV-head items when a full cache would need more chunks per q head
     * (ceil(max_seq / 1024)) than the SMs give (SMs / (max_batch *
     * n_q_heads)), else q-head items.  Both: MK_ERR_INVALID.  The batched
     * kernel always uses KV-head items. */
    MK_FLAG_ATTN_KV_ITEMS = 32,
    MK_FLAG_ATTN_Q_ITEMS = 64
};

/* Upper bounds of the shapes the kernel tiles. */
#define MK_MAX_BATCH 16
#define MK_MAX_K 14336      /* max of n_q_heads*head_dim and ffn */
#define MK_MAX_HIDDEN 4096
#define MK_MAX_HEAD_DIM 128

/*
 * Model shape and run options.
 *  hidden: multiple of 8, at most MK_MAX_HIDDEN; ffn, n_q_heads*head_dim:
 *  multiples of 8, at most MK_MAX_K.  head_dim: 64 or 128; n_q_heads /
 *  n_kv_heads: 1, 2, 4 or 8.  max_seq: KV capacity per sequence (positions
 *  0..max_seq-1).  max_batch: 1..MK_MAX_BATCH (above 1 see "Batched
 *  steps").  rms_eps > 0, rope_theta > 1.
 *  attn_chunks: most split-K chunks per attention item (see
 *  MK_FLAG_ATTN_KV_ITEMS; a step uses ceil(context / 1024) of them, so
 *  contexts up to 1024 positions need no merge); 0 picks min(SMs /
 *  (max_batch * items per chunk), ceil(max_seq / 1024)), items per chunk
 *  being n_q_heads or n_q_heads / heads per item.  At most 4096 and chunks *
 *  heads per item * (head_dim + 2) <= 8192.
 *  timeout_ns: bound on every device-side wait; 0 means 2 s.
 *  l2_lookahead_kb: how far (KiB of weights per SM) the loader bulk-
 *  prefetches into L2 beyond the pages it has copied into shared memory;
 *  0 (the default) means none -- every distance measured slower.
 *  poll_ns: pause (ns) between two polls of a task's not yet ready input
 *  words; 0 polls back to back.
 */
typedef struct mk_config {
    int layers, hidden, n_q_heads, n_kv_heads, head_dim, ffn, vocab;
    int max_seq, max_batch;
    float rope_theta, rms_eps;
    int flags;
    int attn_chunks;
    long long timeout_ns;
    int l2_lookahead_kb;
    int poll_ns;
} mk_config;

/*
 * Weights, all bf16, row-major, 16-byte aligned, in device memory.  The
 * per-layer members are HOST arrays of `layers` device pointers (copied by
 * mk_create; the arrays themselves may be freed after it returns).
 *   embed      [vocab][hidden]
 *   lm_head    [vocab][hidden]          (may equal embed: tied head)
 *   final_norm [hidden]
 *   attn_norm, mlp_norm  [layers] -> [hidden]        RMSNorm gains
 *   wq [layers] -> [n_q_heads*head_dim][hidden]
 *   wk, wv [layers] -> [n_kv_heads*head_dim][hidden]
 *   wo [layers] -> [hidden][n_q_heads*head_dim]
 *   wg, wu [layers] -> [ffn][hidden]    (gate, up)
 *   wd [layers] -> [hidden][ffn]        (down)
 */
typedef struct mk_weights {
    const void *embed, *lm_head, *final_norm;
    const void *const *attn_norm, *const *mlp_norm;
    const void *const *wq, *const *wk, *const *wv, *const *wo;
    const void *const *wg, *const *wu, *const *wd;
} mk_weights;

/*
 * KV cache: per layer, device bf16 [max_batch][n_kv_heads][max_seq][head_dim]
 * (keys stored after RoPE).  k, v are HOST arrays of `layers` device
 * pointers.  Sequence b of a step uses batch slot b.
 */
typedef struct mk_kv {
    void *const *k, *const *v;
} mk_kv;

typedef struct mk_ctx mk_ctx;

/*
 * Validate the shape, build the static task graph for this device (one
 * persistent CTA per SM), allocate scratch and upload the tables.  Blocks
 * the host.  *out receives the context (NULL on error).
 * The graph is MPK's compile step done once on the host: every op split into
 * tasks, one event per op whose threshold is the number of tasks that
 * trigger it ("显著提升小LLM的性能..." page, Figure 2 text on tasks and
 * events; the MPK walkthrough zizhi168.cn/news/174794, section 3.3.2 on
 * task-graph generation by compile()), with the tasks placed in static per-SM queues (the Hazy page,
 * sfrk.com.cn/ruanjian/202506/86466, paragraph on the per-SM execution plan).
 * The device must be compute capability 10.0 (B200; the library holds sm_100a
 * code only), support cooperative launches and offer the kernel's shared
 * memory per block: any other device gives MK_ERR_INVALID
 * (mk_device_supported states the rule).
 * The q/k/v and gate/up matrices are copied into a library-owned layout
 * (rows in the order the kernel streams them, so every task reads one
 * contiguous range); unless MK_FLAG_NO_TMEM_RING is set, so are the other
 * matrices whose pages pass through tensor memory (O-projection, down
 * projection, LM head, in the TMEM page order).  Later changes to copied
 * caller buffers are not seen, and device memory grows by their size.  The
 * embedding table (also when tied to the LM head), the RMSNorm gains and
 * the KV cache are always used in place.
 * Errors: MK_ERR_INVALID (shape or pointer checks), MK_ERR_OOM, MK_ERR_CUDA.
 */
int mk_create(const mk_config *cfg, const mk_weights *w, const mk_kv *kv, mk_ctx **out);

/*
 * One decode step for sequences 0..batch-1, enqueued on `stream` (one
 * kernel launch; asynchronous).  The step is the decoder layer sequence of
 * the Hazy megakernel page (sfrk.com.cn/ruanjian/202506/86466, paragraph
 * listing the fused instructions: RMSNorm + QKV + RoPE, attention and its
 * reduction, O-projection + residual, RMSNorm + gate/up + SiLU, down +
 * residual) and of the MPK walkthrough's per-layer *_layer calls
 * (zizhi168.cn/news/174794, section 3.3.1), ending in the final RMSNorm, the
 * LM head and argmax (same walkthrough, the argmax_partial / argmax_reduce
 * layers).
 *   tokens    device int32 [batch]: input token of each sequence.
 *   positions device int32 [batch]: position of that token; its K/V entry
 *             is written at that slot of every layer's cache and attention
 *             covers positions 0..positions[b].
 *   logits_out   device float [batch][vocab], or NULL to skip writing.
 *   next_tok_out device int32 [batch]: argmax of each row of logits
 *                (lowest index on ties).
 * 1 <= batch <= max_batch.  A token outside [0, vocab) or a position
 * outside [0, max_seq) is detected on the device: the step then does no
 * work and the context reports MK_ERR_INVALID from mk_sync.  A device
 * timeout is reported as MK_ERR_TIMEOUT by mk_sync.  After a device error
 * every call returns MK_ERR_STATE until mk_reset.
 * Not thread-safe with respect to the same context.
 */
int mk_decode_step(mk_ctx *ctx, const int32_t *tokens, const int32_t *positions, int batch,
                   float *logits_out, int32_t *next_tok_out, mk_stream_t stream);

/*
 * Prompt and greedy generation in one launch (MPK's once-per-generation
 * mode: the persistent kernel keeps running while the tokens are produced,
 * "显著提升小LLM的性能..." page, section on the decode loop and its step
 * tensor).  Step s decodes one token per sequence at positions[b] + s,
 * writing that K/V slot: for s < n_prompt the prompt's token tokens[s][b],
 * afterwards step s-1's argmax.  The steps run back to back inside the
 * kernel: each step's next token is published on the device and feeds the
 * next step's embedding, and the next step's weights stream into shared
 * memory while the current step's LM head finishes.  (The prompt is fed
 * one token per step, like the decode steps, not as a multi-token
 * contraction.)
 *   tokens             device int32 [n_prompt][batch]: the prompt (n_prompt
 *                      = 1: just the first step's token).
 *   positions          device int32 [batch]: the first step's positions.
 *   n_steps            steps to run, n_prompt..max_seq; positions[b] +
 *                      n_steps must not exceed max_seq and every prompt
 *                      token must lie in [0, vocab) (checked on the device:
 *                      MK_ERR_INVALID from mk_sync, nothing run).
 *   eos                a sequence stops at the first eos it generates
 *                      (steps >= n_prompt - 1; < 0: never); once every
 *                      sequence has stopped the launch ends.
 *   tokens_out         device int32 [n_steps][batch]: step s's argmax for
 *                      sequence b (eos after the sequence stopped); the
 *                      generated tokens start at row n_prompt - 1; rows of
 *                      steps not run (early stop) are left untouched.
 *   next_tok_out       device int32 [batch]: the last step's argmax.
 * Logits are not written.  Errors as for mk_decode_step.
 */
int mk_generate(mk_ctx *ctx, const int32_t *tokens, int n_prompt, const int32_t *positions, int batch,
                int n_steps, int32_t eos, int32_t *tokens_out, int32_t *next_tok_out, mk_stream_t stream);

/*
 * Batched steps.  A context created with max_batch > 1 (or MK_FLAG_ROWS)
 * runs every step on a second persistent kernel: one kernel step takes up to
 * 16 rows -- a row is one token of one sequence -- and every matrix op is a
 * contraction of the weights with those rows on the tcgen05 tensor cores
 * (M = 128 weight rows, N = 32: each row's fp32 input enters as its bf16
 * high part and bf16 remainder; fp32 accumulation in tensor memory), so the
 * weights are read once per kernel step whatever the number of rows.  The
 * matrices are copied into a library-owned tile layout at create time.
 * Shape limits: hidden, n_q_heads*head_dim, n_kv_heads*head_dim and ffn
 * multiples of 128; n_q_heads / n_kv_heads = 1, 2 or 4 with (n_q_heads /
 * n_kv_heads) * head_dim <= 512; attn_chunks: chunks of at least 4096
 * positions per (row, KV head), default ceil(max_seq / 4096).
 * MK_FLAG_EVENT_WAIT (tasks always wait on event counters here),
 * mk_generate, mk_get_sm_stats and mk_debug_withhold_event are not
 * available on such contexts (MK_ERR_INVALID); mk_read_buffer offers
 * MK_BUF_HIDDEN as float [16][hidden].  With MK_FLAG_TRACE the trace
 * records mean: t_ready the scheduler saw the dependency met, t_wait the
 * MMA issuer began the task's pages, t_start the compute warps began,
 * t_input the first accumulator (or the attention queries) was in hand,
 * t_done the epilogue was done, t_end the completion was posted.
 *
 * mk_decode_step on such a context: sequence b (b < batch) is a row at its
 * own position, in KV slot b; any mix of positions.
 *
 * mk_prefill: a prompt of n_tokens tokens of the sequence in KV slot `slot`,
 * at positions start_pos .. start_pos + n_tokens - 1, in ONE launch: kernel
 * steps of 16 consecutive tokens, each a contraction over its 16 rows with
 * causal attention (a token attends to the slot's positions up to its own,
 * the prompt's earlier tokens included), the LM head only for the step that
 * holds the last token (the MPK walkthrough, zizhi168.cn/news/174794, feeds
 * the prompt through its decode loop one token per step; this is the same
 * computation with the prompt's tokens sharing each weight read).
 *   tokens        device int32 [n_tokens]
 *   logits_out    device float [vocab] for the last token, or NULL
 *   next_tok_out  device int32 [1]: argmax of the last token's logits
 * Positions beyond max_seq, a slot >= max_batch or a context without the
 * batched kernel give MK_ERR_INVALID synchronously; a token outside [0,
 * vocab) is reported by mk_sync.
 */
int mk_prefill(mk_ctx *ctx, const int32_t *tokens, int n_tokens, int slot, int start_pos, float *logits_out,
               int32_t *next_tok_out, mk_stream_t stream);

/* Wait for `stream`, then return the device status of the context
 * (MK_OK, MK_ERR_INVALID, MK_ERR_TIMEOUT) or MK_ERR_CUDA. */
int mk_sync(mk_ctx *ctx, mk_stream_t stream);

/* Clear the device error state, the event counters and the tagged
 * activations, and restart the step count (blocks the host; no step may be
 * in flight).  Also turns off the mk_debug_withhold_event hook.  The
 * context is usable again afterwards (also after MK_ERR_TIMEOUT or
 * MK_ERR_INVALID from the device).  Errors: MK_ERR_INVALID (ctx NULL),
 * MK_ERR_CUDA (a CUDA call failed). */
int mk_reset(mk_ctx *ctx);

/* Wait for the device, then free the context's scratch and library-owned
 * weight copies (blocks the host).  Caller buffers are not touched.  NULL is
 * accepted.  Always returns MK_OK. */
int mk_destroy(mk_ctx *ctx);

/* A static description of a status code ("unknown status" for codes this
 * header does not define); never NULL, never to be freed. */
const char *mk_status_string(int status);

/* ---- introspection (tests, tracing) ------------------------------------ */

typedef struct mk_info {
    int num_sms;        /* persistent CTAs = SMs used */
    int num_tasks;
    int num_events;
    int num_ops;
    int attn_chunks;
    int max_queue;      /* longest per-SM task queue */
    int page_bytes, num_pages;
    long long steps_run; /* decode steps enqueued since create/reset (mk_generate adds n_steps) */
    unsigned int err_code, err_info; /* device error word (0 = none); err_info = which wait << 24 | detail */
    unsigned int err_task;           /* task id the device error was raised in (0xffffffff: none) */
    int attn_heads;                  /* q heads per attention item (MK_FLAG_ATTN_KV_ITEMS) */
} mk_info;

/* Sizes of the context's task graph and its device error word (copied
 * from the device: call after mk_sync for the status of finished steps).
 * Errors: MK_ERR_INVALID (ctx or out NULL), MK_ERR_CUDA. */
int mk_get_info(mk_ctx *ctx, mk_info *out);

/* Copy the first n event counters (uint32) and thresholds to host (either
 * pointer may be NULL).  After s successful steps every counter equals
 * threshold * s (mod 2^32).  Blocks the host.  Errors: MK_ERR_INVALID (ctx
 * NULL, n < 0 or n > num_events), MK_ERR_CUDA. */
int mk_get_event_counts(mk_ctx *ctx, uint32_t *counts_out, uint32_t *thresholds_out, int n);

/* Scratch buffers readable after a step (host copy, blocks the host):
 * MK_BUF_HIDDEN float [max_batch][hidden] residual stream after the last
 * layer; MK_BUF_Q float [max_batch][nq*head_dim] last layer's q before RoPE
 * (the attention tasks rotate it);
 * MK_BUF_ATTN float [max_batch][nq*head_dim] last layer's attention output;
 * MK_BUF_ACT float [max_batch][ffn] last layer's SiLU(gate)*up. */
enum mk_buffer { MK_BUF_HIDDEN = 0, MK_BUF_Q = 1, MK_BUF_ATTN = 2, MK_BUF_ACT = 3 };
/* Copies the first `count` floats of buffer `which` to host_out.
 * Batched contexts (max_batch > 1 or MK_FLAG_ROWS) have MK_BUF_HIDDEN only
 * (float [16][hidden]: the residual stream after the last layer, one row
 * per row of the last kernel step).  Errors:
 * MK_ERR_INVALID (ctx or host_out NULL, unknown or unavailable buffer,
 * count beyond its size), MK_ERR_CUDA. */
int mk_read_buffer(mk_ctx *ctx, int which, float *host_out, size_t count);

/* Per-task trace of the last step (MK_FLAG_TRACE).  Records are
 * mk_trace_rec [num_tasks], indexed by task id. */
typedef struct mk_trace_rec {
    unsigned long long t_ready;  /* globaltimer ns: the dependency was seen met (the
                                    scheduler saw the event fire; without
                                    MK_FLAG_EVENT_WAIT: every input word the
                                    task reads carried this step's tag) */
    unsigned long long t_start;  /* workers passed the dependency (loads that do not
                                    depend on it may start earlier); without
                                    MK_FLAG_EVENT_WAIT equal to t_ready */
    unsigned long long t_input;  /* the task's input vector is loaded (and normalised) */
    unsigned long long t_done;   /* all rows computed, before the task-end barrier */
    unsigned long long t_end;    /* workers finished and posted the completion */
    unsigned long long t_wait;   /* ns worker thread 0 spent waiting for pages */
    int sm;                      /* CTA that ran it */
    int kind;                    /* op kind (MK_OP_*) */
    int layer;
    int trig_event;
} mk_trace_rec;
enum mk_op_kind { MK_OP_QKV = 0, MK_OP_ATTN = 1, MK_OP_OPROJ = 2, MK_OP_GATEUP = 3,
                  MK_OP_DOWN = 4, MK_OP_LMHEAD = 5 };
/* Copies the first n records.  Errors: MK_ERR_INVALID (ctx or host_out
 * NULL, n < 0 or n > num_tasks, or the context was created without
 * MK_FLAG_TRACE), MK_ERR_CUDA. */
int mk_get_trace(mk_ctx *ctx, mk_trace_rec *host_out, int n);

/* Per-SM time accounting of the last step (MK_FLAG_TRACE): uint64
 * [num_sms][16] = {loader ns waiting for a free page, pages issued, loader
 * ns total, worker ns waiting for loaded pages, worker ns waiting for the
 * scheduler, worker ns in worker barriers, worker ns total, scheduler ns
 * waiting on event counters, worker ns in task prologues (waiting for and
 * loading the input vector, RMSNorm), worker ns in row-per-warp dot
 * products, worker ns in per-tile reductions and epilogues, worker ns in
 * task ends (barrier, completion post, argmax), tasks run, worker ns in
 * attention combine/merge tails, worker ns in the first page of each
 * column-split task, worker ns in its later pages}.  Worker figures are
 * those of thread 0 and some phases overlap the waits they contain.  Copies
 * the first n values.  Errors: MK_ERR_INVALID (ctx or host_out NULL, n < 0
 * or n > num_sms * 16, or no MK_FLAG_TRACE), MK_ERR_CUDA. */
int mk_get_sm_stats(mk_ctx *ctx, uint64_t *host_out, int n);

/* Static task graph as built by mk_create (host copy).  task_out: int32
 * [num_tasks][8] = {kind, layer, dep_event (-1 none), trig_event, begin,
 * end, sm, slot}; queue_out: int32 [num_tasks] task ids grouped by SM in
 * execution order; qoff_out: int32 [num_sms+1] offsets into queue_out.
 * Any of the arrays may be NULL; the sizes are in mk_get_info.  No device
 * access.  Errors: MK_ERR_INVALID (ctx NULL). */
int mk_get_graph(mk_ctx *ctx, int32_t *task_out, int32_t *queue_out, int32_t *qoff_out);

/* Host-only planning (no GPU needed): build the task graph for `cfg` on a
 * machine with `num_sms` SMs and return its sizes in *info (num_tasks,
 * num_events, num_ops, attn_chunks, max_queue, page sizes), then fill the
 * arrays as mk_get_graph does (any of them may be NULL) plus thresholds_out
 * uint32 [num_events] and the per-task weight bytes bytes_out int64
 * [num_tasks].  Used to test the graph builder without a device.  Errors:
 * MK_ERR_INVALID (cfg NULL, a shape or option mk_create would refuse,
 * num_sms outside 1..1024). */
int mk_plan(const mk_config *cfg, int num_sms, mk_info *info,
            int32_t *task_out, int32_t *queue_out, int32_t *qoff_out,
            uint32_t *thresholds_out, int64_t *bytes_out);

/* Host-only (no GPU needed): whether mk_create and mk_decode_step_static
 * accept a device with compute capability major.minor, cooperative-launch
 * support (0 / 1) and `smem_optin_bytes` of opt-in shared memory per block
 * (cudaDeviceProp.sharedMemPerBlockOptin), for the batched kernel (batched
 * != 0: max_batch > 1 or MK_FLAG_ROWS) or the batch-1 kernel.  The library
 * holds arch-specific sm_100a code, which runs on compute capability 10.0
 * only.  Returns MK_OK or MK_ERR_INVALID; both entry points make exactly
 * this check on the current device before anything else touches it. */
int mk_device_supported(int major, int minor, int cooperative_launch, size_t smem_optin_bytes,
                        int batched);

/* ---- decode without allocating --------------------------------------- */

/*
 * For callers that cannot allocate device memory where they decode (an
 * arena that owns all device memory, an allocation-free serving loop):
 * mk_decode_step_static runs the same decode step as mk_decode_step without
 * a context and without allocating anything.  The pages describing this
 * method have no counterpart of it; it is an addition of this library.
 *
 * Its scratch (task tables, RoPE table, activations, attention partials,
 * counters, error word) lives in one fixed device array of
 * MK_STATIC_SCRATCH_BYTES that every GPU which loads the library holds
 * until the process exits.  Shapes whose scratch does not fit are rejected
 * with MK_ERR_INVALID (the 1B shape needs about 3.2 MiB at max_seq 560 and
 * 8.0 MiB at max_seq 16640).
 * Every call shares that array and leaves its last contents there: calls
 * on the same device that overlap on the GPU (several streams or host
 * threads) race.  Each device has its own array; the host-side staging of
 * the tables is serialised by a lock, so host threads driving different
 * devices do not interfere.  The first call on a device looks up the
 * array's address and sets up the kernel for that device; a call whose shape
 * differs from the previous call's on that device (its sizes, or the
 * attention items its flags choose: MK_FLAG_ATTN_KV_ITEMS) uploads new task
 * and RoPE tables, and a call whose weight or KV pointers differ uploads a new layer
 * table -- both synchronise the stream, so make such calls outside stream
 * capture (the first call on a device included).  The tables carry a key
 * that the kernel compares with the key its launch was set up with: a
 * launch set up for tables that have been replaced since (a replay of an
 * earlier launch) runs nothing and reports MK_ERR_INVALID through
 * status_out.
 * MK_FLAG_TRACE is not supported here.
 *
 * Weights come already in the kernel's streaming layout (mk_create makes
 * this copy itself; this entry point cannot allocate one):
 *   qkv [layers] -> bf16 [(n_q_heads + 2*n_kv_heads)*head_dim][hidden]:
 *       the wq rows, then the wk rows, then the wv rows (one buffer);
 *   gu  [layers] -> bf16 [2*ffn][hidden]: for each j < ffn/8, gate rows
 *       8j..8j+7 then up rows 8j..8j+7;
 *   the other members as in mk_weights.
 * tokens, positions, logits_out, next_tok_out, stream: as mk_decode_step.
 * status_out: device int32 [1] or NULL; receives the step's device status
 * (MK_OK, MK_ERR_INVALID for an out-of-range token/position,
 * MK_ERR_TIMEOUT) in stream order.
 */
#define MK_STATIC_SCRATCH_BYTES (8u << 20)

typedef struct mk_packed_weights {
    const void *embed, *lm_head, *final_norm;
    const void *const *attn_norm, *const *mlp_norm;
    const void *const *qkv, *const *wo, *const *gu, *const *wd;
} mk_packed_weights;

int mk_decode_step_static(const mk_config *cfg, const mk_packed_weights *w, const mk_kv *kv,
                          const int32_t *tokens, const int32_t *positions, int batch,
                          float *logits_out, int32_t *next_tok_out, int32_t *status_out,
                          mk_stream_t stream);

/* Test hook: overwrite the threshold of one event (simulates a graph
 * whose event can never fire; the next step then ends in MK_ERR_TIMEOUT).
 * Blocks the host. */
int mk_debug_set_threshold(mk_ctx *ctx, int event, uint32_t threshold);

/* Test hook for the tagged-input waits: from the next step on, the tasks
 * that trigger `event` store their outputs with a stale tag, so the tasks
 * reading them wait until timeout_ns and the step ends in MK_ERR_TIMEOUT
 * (every wait is bounded; nothing faults).  event = -1 turns it off;
 * mk_reset turns it off too.  Host-side only (applies to later launches). */
int mk_debug_withhold_event(mk_ctx *ctx, int event);

#ifdef __cplusplus
}
#endif
#endif /* MK_H */
