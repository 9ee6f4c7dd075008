// mk_internal.h -- layout of the task graph and the kernel parameters,
// shared by the host runtime (mk_runtime.cpp, mk_graph.cpp) and the
// persistent kernel (mk_kernel.cu).  Not part of the public ABI.
#pragma once

#include <stdint.h>
#include <stddef.h>
#include <vector_types.h>   // float2

#if defined(__CUDACC__)
#define MK_HD __host__ __device__
#else
#define MK_HD
#endif

namespace mk {

// ---- CTA shape ---------------------------------------------------------------
// Three warpgroups: two of workers, one of control warps (loader, scheduler
// and two idle warps).  The CTA launches at kLaunchRegs registers per thread
// (65536 / 384, rounded down to 8); setmaxnreg then moves registers from the
// control warpgroup to the workers.  The shares must add up to the launch
// total exactly or setmaxnreg.inc would wait forever:
//   256 * kWorkerRegs + 128 * kControlRegs == 384 * kLaunchRegs.
constexpr int kWorkerWarps = 8;                     // run task bodies
constexpr int kWorkerThreads = kWorkerWarps * 32;   // 256
constexpr int kLoaderWarp = kWorkerWarps;           // streams weight pages
constexpr int kSchedWarp = kWorkerWarps + 1;        // waits on events (when gating by events)
constexpr int kStashWarp = kWorkerWarps + 2;        // moves landed weight pages into tensor memory
constexpr int kThreads = (kWorkerWarps + 4) * 32;   // 384
constexpr int kLaunchRegs = 168;
constexpr int kWorkerRegs = 224;
constexpr int kControlRegs = 56;
static_assert(kWorkerThreads * kWorkerRegs + (kThreads - kWorkerThreads) * kControlRegs ==
                  kThreads * kLaunchRegs,
              "register split must equal the launch allocation");

// ---- tiling ------------------------------------------------------------------
constexpr int kTileRows = 8;        // output rows per GEMV tile
constexpr int kPageRowsMax = 16;    // rows one page holds at most (a 16-row unit)
constexpr int kPageBytes = 65536;   // one shared-memory page
constexpr int kNumPages = 3;        // pages in the per-SM ring
constexpr int kVecMax = 7;          // 16-byte vectors per thread per row (K <= 7*8*256)
constexpr int kMaxK = kVecMax * 8 * kWorkerThreads;  // 14336
constexpr int kMaxBatch = 1;        // sequences per step (MK_MAX_BATCH)
// Attention chunking: a sequence's positions are split into at most NC
// chunks of at least this many positions (shorter contexts use fewer chunks;
// one chunk needs no merge).
constexpr int kAttnChunkPositions = 1024;
// q heads of one attention item, times head_dim, at most (the item's
// per-warp softmax states and queries live in the shared staging area).
constexpr int kAttnHeadDims = 512;
constexpr int kMaxHeadDim = 256;
constexpr long long kL2Lookahead = 0;  // default L2 prefetch distance beyond the ring (0: off; measured no gain)
constexpr int kStageFloats = 8192;  // shared staging: a GEMV input vector, or attention partials
// Tensor memory as a second level of the weight ring: the whole 512-column
// allocation of the SM, as kTmemSlots slots of one 64 KB page each (a page of
// 16 rows of 2048 bf16 columns occupies 128 lanes x 128 columns).
constexpr int kTmemCols = 512;
constexpr int kTmemSlots = 4;
constexpr int kTmemSlotCols = kTmemCols / kTmemSlots;

// ---- ops ---------------------------------------------------------------------
enum OpKind : int32_t { OP_QKV = 0, OP_ATTN = 1, OP_OPROJ = 2, OP_GATEUP = 3, OP_DOWN = 4, OP_LMHEAD = 5 };

// One task: a contiguous range of tiles of one op (GEMV ops), or one
// attention work item (b, q head, chunk), assigned to one SM.
struct Task {
    int32_t kind;
    int32_t layer;
    int32_t dep;      // event waited on (-1: none)
    int32_t trig;     // event bumped when done
    int32_t begin;    // first tile (GEMV) / item index (ATTN)
    int32_t end;      // one past the last tile / item
    int32_t sm;       // CTA whose queue holds it
    int32_t slot;     // index of the task within its op
};
static_assert(sizeof(Task) == 32, "Task is 8 int32");

// Device pointers of one layer (bf16 as uint16_t on the host side).
//  qkv: library-owned [(nq + 2 nkv) d][H]: the q rows, then the k rows,
//       then the v rows (each in the caller's order), so a QKV task's
//       rows are one contiguous range.
//  gu:  library-owned [2F][H] in gate/up tile order: 4 gate rows, then the
//       4 up rows with the same indices.
//  wo, wd: the caller's matrices, read in place.
struct LayerW {
    const uint16_t *qkv, *gu, *wo, *wd;
    const uint16_t *g_attn, *g_mlp;
    uint16_t *kc, *vc;
};

// Sizes derived from the model shape.
struct Shape {
    int L, H, nq, nkv, d, F, V, S, Bmax, NC;
    int tmem;         // 1: GEMV pages of 2048-column rows pass through tensor memory
                      //    (weights in the TMEM page order, tasks start on page boundaries)
    int G;            // nq / nkv
    int HA;           // q heads per attention item: 1, or a divisor of G (the
                      //  q heads of one KV head share the item's K/V pages)
    int QD, KD;       // nq*d, nkv*d
    float theta, eps;
};

// Tile counts of each op (identical on host and device).
//  QKV:    (nq + 2 nkv) * d / 8 tiles of 8 rows (q, then k, then v rows;
//          RoPE is applied by the attention tasks, so no tile needs its
//          rotation partner rows and 8-row tiles balance the SMs)
//  GATEUP: F / 8 pair tiles of 16 rows (8 gate rows + the same 8 up rows)
//  OPROJ, DOWN: H / 8 tiles of 8 rows; LMHEAD: ceil(V / 8) tiles of 8 rows
struct OpTiles {
    int qkv;
    int oproj;
    int gateup;
    int down;
    int lmhead;
    int attn_items;   // Bmax * (nq / HA) * NC
};

MK_HD inline OpTiles op_tiles(const Shape &s) {
    OpTiles t;
    t.qkv = (s.QD + 2 * s.KD) / 8;
    t.oproj = s.H / 8;
    t.gateup = s.F / 8;
    t.down = s.H / 8;
    t.lmhead = (s.V + 7) / 8;
    t.attn_items = s.Bmax * (s.nq / s.HA) * s.NC;
    return t;
}

// Reduction dimension (columns) of a GEMV op.
MK_HD inline int op_k(const Shape &s, int kind) {
    return kind == OP_OPROJ ? s.QD : (kind == OP_DOWN ? s.F : s.H);
}

// Row offset of tile `tile` in its op's weight buffer (rows of tiles are
// contiguous and in tile order) -- also the rows of tiles [0, tile).
MK_HD inline long long tile_row_offset(const Shape &s, int kind, int tile) {
    (void)s;
    return kind == OP_GATEUP ? 16LL * tile : 8LL * tile;
}

MK_HD inline int tile_rows(const Shape &s, int kind, int tile) {
    return (int)(tile_row_offset(s, kind, tile + 1) - tile_row_offset(s, kind, tile));
}

// GEMVs with K <= kRowK run one row per warp with the whole input vector in
// registers; K = 2 or 4 x kRowK run one 2048-column segment of a row per
// warp; other K split columns across all worker threads.
constexpr int kRowK = 2048;
MK_HD inline bool rows_gemv(int K) { return K <= kRowK || K == 2 * kRowK || K == 4 * kRowK; }
constexpr int kMaxHidden = 4096;   // MK_MAX_HIDDEN: the largest hidden size the tests cover

// GEMV ops whose pages are 16 "page rows" of 2048 columns (K = 2048, 4096,
// 8192): with Shape::tmem these pages are staged in tensor memory, and the
// weights are stored in the TMEM page order (tmem_page_src below).
MK_HD inline bool tmem_page_op(const Shape &s, int kind) {
    const int K = op_k(s, kind);
    return s.tmem && kind != OP_ATTN && K % kRowK == 0 && rows_gemv(K);
}

// The TMEM page order.  A page of 16 page rows (each 2048 bf16 = 256
// vectors of 16 bytes) is stored as 16 blocks of 4 KB; tcgen05.cp of block c
// (128x256b, no swizzle, stride offset 128 B, leading offset 2048 B) puts
// the 16-byte pieces at 512p + 16L and 2048 + 512p + 16L of the block into
// TMEM lane 32p + L, columns 8c..8c+3 and 8c+4..8c+7.  Block c holds page
// row (c / 8) * 8 + p + 4 * ((c / 4) % 2), vectors L + 32 * (2 * (c % 4) + q)
// for the piece q, so that worker warp w reads page rows w and 8 + w (the
// rows the shared-memory path gives it) as 32 consecutive columns each from
// its own lane quarter (w % 4), lane L getting vectors L, L + 32, ..., L + 224
// in order -- and rows 0..7 sit in the first 32 KB (a trailing 8-row page is
// one half-size copy).
// tmem_page_src: the source (page row, vector) of destination vector u
// (0..4095) of a page.
MK_HD inline void tmem_page_src(int u, int &row, int &vec) {
    const int c = u >> 8, q = (u >> 7) & 1, p = (u >> 5) & 3, L = u & 31;
    row = (c >> 3) * 8 + p + 4 * ((c >> 2) & 1);
    vec = L + 32 * (2 * (c & 3) + q);
}

// Rows of one page: the largest power of two <= 16 whose rows (K bf16 each)
// fit in a page (16 for K <= 2048: one page holds a whole 16-row unit).
MK_HD inline int rows_per_page(int K) {
    int r = kPageBytes / (2 * K);
    int p = 1;
    while (p * 2 <= r && p * 2 <= kPageRowsMax) p *= 2;
    return p;
}

// KV-head attention items score positions with the queries in registers:
// a warp's lanes are (position p, dim group g) pairs, NG = HA * d / 64
// groups of NS = 8 / HA 16-byte chunks of the K row each (every lane holds
// its chunks' slices of all HA queries: 64 floats).  Lane (p, g) reads its
// chunks starting at attn_kv_rot(p, g, ...) (mod NS) so that the 8 lanes of
// every quarter-warp hit 8 different bank groups (chunk index mod 8; K rows
// are 128 or 256 bytes apart).
MK_HD inline int attn_kv_rot(int p, int g, int ng, int ns, int d) {
    return ((p % (8 / ng)) * (d / 64) + (g * ns) / 8) % ns;
}

// Attention positions per page (K block and V block of `n` positions).
MK_HD inline int attn_pos_per_page(int d) { return kPageBytes / (4 * d); }

// ---- tagged activations -------------------------------------------------------
// Every activation one task hands to another lives in a "tagged" buffer: one
// 64-bit word per fp32 value, the value's bits in the low half and the step
// tag (the launch's epoch) in the high half, written with one 64-bit store.
// A consumer polls the words it needs until every tag equals the current
// epoch, so the data carries its own readiness: no fence, counter or extra
// copy sits between a producer's store and the consumer's read.  Each layer
// owns its own buffers (nothing is overwritten within a step), so a word's tag
// is either this step's or an older one.
// The vectors every SM reads whole (the two residual streams, the attention
// output and SiLU(gate) * up) can be written kReplicas times, SM i reading
// copy i % kReplicas, so that the 148 readers spread over more L2 lines.
// Measured: 8 copies are slower than one (the extra stores cost more than
// the readers gain), so kReplicas is 1.
//   xa: residual after the O-projection   [R][Bmax][H]
//   xb: residual after the down projection [R][Bmax][H] (layer L-1: final hidden)
//   q:  queries before RoPE                [Bmax][nq * d]
//   kn: the new position's key before RoPE; vn: its value rounded to bf16
//                                          [Bmax][nkv * d]
//   part: split-K attention partials, per q head and chunk o[d], m, l
//                                          [Bmax][nq][NC][d + 2]
//   attn: merged attention output          [R][Bmax][nq * d]
//   act:  SiLU(gate) * up                  [R][Bmax][F]
constexpr int kReplicas = 1;
struct TagLayout {
    size_t xa, xb, q, kn, vn, part, attn, act;   // word offsets within a layer's block
    size_t rep_h, rep_qd, rep_f;                 // distance between copies (words)
    size_t layer;                                // words per layer
};

MK_HD inline TagLayout tag_layout(const Shape &s) {
    TagLayout t;
    const size_t B = (size_t)s.Bmax;
    t.rep_h = B * s.H;
    t.rep_qd = B * s.QD;
    t.rep_f = B * s.F;
    size_t o = 0;
    t.xa = o; o += kReplicas * t.rep_h;
    t.xb = o; o += kReplicas * t.rep_h;
    t.q = o; o += B * s.QD;
    t.kn = o; o += B * s.KD;
    t.vn = o; o += B * s.KD;
    t.part = o; o += B * s.nq * (size_t)s.NC * (s.d + 2);
    t.attn = o; o += kReplicas * t.rep_qd;
    t.act = o; o += kReplicas * t.rep_f;
    t.layer = (o + 1) & ~(size_t)1;   // keep every block 16-byte aligned
    return t;
}

// Device-side error word (mapped pinned host memory).
struct ErrWord {
    uint32_t code;    // MK_ERR_* (0 = none)
    uint32_t task;    // task id where it happened (or 0xffffffff)
    uint32_t where;   // which wait: 1 dep event, 2 ready, 3 page full, 4 page empty,
                      // 5 worker barrier, 6 input check, 7 drain
    uint32_t info;    // extra (event index, bad value)
};

// Per-SM wait accounting (trace mode), in globaltimer ns unless noted.
enum StatSlot {
    ST_LOADER_EMPTY = 0,  // loader waiting for a free page
    ST_LOADER_PAGES = 1,  // pages issued (count)
    ST_LOADER_TOTAL = 2,  // loader role start to end
    ST_WORKER_FULL = 3,   // worker warp 0 waiting for a loaded page
    ST_WORKER_READY = 4,  // worker warp 0 waiting for the scheduler
    ST_WORKER_SYNC = 5,   // worker warp 0 in worker barriers
    ST_WORKER_TOTAL = 6,  // worker role start to end
    ST_SCHED_DEP = 7,     // scheduler waiting on event counters
    ST_WORKER_PROLOGUE = 8,  // worker warp 0: task start to its first page (input load, norm)
    ST_WORKER_DOT = 9,       // worker warp 0: dot products on loaded pages
    ST_WORKER_EPI = 10,      // worker warp 0: per-tile reductions and epilogues
    ST_WORKER_END = 11,      // worker warp 0: task end (barrier, fence, event, merges)
    ST_WORKER_TASKS = 12,    // tasks run (count)
    ST_WORKER_ATTN_TAIL = 13, // worker warp 0: attention combine, partial write and merge
    kStatSlots = 16
};

struct TraceRec {
    unsigned long long t_ready, t_start, t_input, t_done, t_end, t_wait;
    int32_t sm, kind, layer, trig;
};
static_assert(sizeof(TraceRec) == 64, "trace record layout");

struct Params {
    Shape s;
    // graph
    const Task *qtasks;          // [num_tasks] the tasks in queue order, `sm` holding the task id
    const int32_t *qoff;         // [num_sms + 1]
    const uint32_t *thresholds;  // [num_events]
    uint32_t *events;            // [num_events]
    uint32_t *lm_cnt;            // [1]
    uint32_t *epoch;             // [1]: steps completed
    uint32_t *done_cnt;          // [1]: CTAs that have read the epoch
    uint32_t *abort_flag;        // [1]
    int num_lm_tasks;
    // model
    const LayerW *layers;
    const uint16_t *embed, *lm_head, *g_final;
    const float2 *rope;          // [S][d/2] (cos, sin)
    // step inputs / outputs
    const int32_t *tokens, *positions;
    int batch;
    float *logits;               // may be null
    int32_t *next_tok;
    // generation (once-per-generation launch): n_steps decode steps back to
    // back, each step's argmax the next step's token
    int n_steps;                 // 1 for a single decode step
    int n_prompt;                // steps 0 .. n_prompt-1 take their token from `tokens` ([n_prompt][batch])
    int32_t eos;                 // a sequence stops at its first eos (-1: never)
    int32_t *tokens_out;         // [n_steps][batch] generated tokens (null: single step)
    uint64_t *tok_tag;           // [Bmax][2] tagged words: next step's token, sequence done
    // scratch
    uint64_t *tag;               // [L][TagLayout::layer] tagged activations
    TagLayout tl;
    float *amax_val;             // [Bmax][num_lm_tasks]
    int32_t *amax_idx;           // [Bmax][num_lm_tasks]
    // control
    ErrWord *err;                // device view of mapped host memory
    TraceRec *trace;             // null unless tracing
    unsigned long long *sm_stats; // [num_sms][kStatSlots] wait times (ns), null unless tracing
    unsigned long long timeout_ns;
    long long l2_lookahead;      // bytes the L2 prefetch runs ahead of the ring (0: off)
    int event_wait;              // 1: the scheduler gates tasks on event counters
    int debug_withhold;          // test hook: tasks triggering this event write stale tags (-1: off)
    unsigned int poll_ns;        // pause between polls of stale input words
    // tables shared between calls (the no-allocation entry point): the key
    // of the tables currently uploaded, and the key this launch was built
    // for; a mismatch refuses the step (MK_ERR_INVALID).  Null: no check.
    const uint64_t *table_key;
    uint64_t expect_key;
};

// ---- host planning -------------------------------------------------------------
struct Plan {
    Shape s;
    int num_sms = 0;
    int num_events = 0;
    int num_ops = 0;
    int max_queue = 0;
    int num_lm_tasks = 0;
    // tasks in op order; queue grouped by SM
    Task *tasks = nullptr; int num_tasks = 0;
    int32_t *queue = nullptr;
    int32_t *qoff = nullptr;
    uint32_t *thresholds = nullptr;
    int64_t *bytes = nullptr;    // weight bytes per task (attention: estimate)
};

// Build the plan into caller-sized storage.  plan_sizes() returns the
// element counts needed; plan_build() fills arrays of at least those sizes.
struct PlanSizes { int num_tasks, num_events, num_ops; };
PlanSizes plan_sizes(const Shape &s, int num_sms);
void plan_build(const Shape &s, int num_sms, Plan &p);

// Default number of attention chunks for a shape on `num_sms` SMs.
// Attention planning (mk_graph.cpp): sets s.HA and s.NC from the config
// (flags MK_FLAG_ATTN_KV_ITEMS / MK_FLAG_ATTN_Q_ITEMS, attn_chunks) and the
// SM count; false when the chunk partials of an item's heads would not fit
// the merge's staging area.
bool plan_attention(Shape &s, int num_sms, int flags, int attn_chunks);

}  // namespace mk
