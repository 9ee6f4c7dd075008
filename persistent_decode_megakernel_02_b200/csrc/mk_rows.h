// mk_rows.h -- the batched ("rows") decode step on tcgen05 tensor cores:
// task graph, weight/activation layouts and kernel parameters, shared by the
// host runtime (mk_runtime.cpp, mk_rows_graph.cpp) and the kernel
// (mk_rows.cu).  Not part of the public ABI.
//
// One kernel step processes up to kRows rows; a row is one token of one
// sequence: (token, position, KV slot).  Independent sequences of a batch
// are rows of different slots; the tokens of a prompt are rows of one slot
// at consecutive positions (causal: a row attends to its slot's positions
// up to its own, including those of earlier rows of the same step).  Every
// matrix-vector product of the step is then a real contraction of the
// weights with kRows input vectors: D[128 weight rows][N] += W[128][K] .
// X[K][N] on the tensor cores (tcgen05.mma kind::f16, M = 128, N = 2 kRows:
// every input vector enters as its bf16 high part and its bf16 remainder,
// so the products keep ~16 significant bits of the fp32 activations; the
// accumulator is fp32 in tensor memory).
#pragma once

#include <stdint.h>
#include <stddef.h>

#include "mk_internal.h"

namespace mk {

constexpr int kRows = 16;                    // rows per kernel step (MK_MAX_BATCH)
constexpr int kRowsN = 2 * kRows;            // MMA N: high and low halves of every row
constexpr int kRTile = 128;                  // weight rows per tile (MMA M)
constexpr int kRSlab = 128;                  // reduction columns per page
constexpr int kRPageBytes = kRTile * kRSlab * 2;   // 32 KB of weights per page
constexpr int kRSlabBytes = kRowsN * kRSlab * 2;   // 8 KB of activations per page
constexpr int kRStages = 5;                  // pages in flight per SM
constexpr int kRAccCols = kRowsN;            // TMEM columns of one accumulator
constexpr int kRTmemCols = 64;               // two accumulators (double buffer)

// Ops of the rows step, in queue order within a layer.
enum ROp : int32_t { ROP_EMBED = 0, ROP_QKV = 1, ROP_ATTN = 2, ROP_OPROJ = 3, ROP_GATEUP = 4,
                     ROP_DOWN = 5, ROP_LMHEAD = 6 };

// Events: EMBED, then 5 per layer, then LMHEAD.
MK_HD inline int rev_embed() { return 0; }
MK_HD inline int rev_op(int layer, int op) { return 1 + 5 * layer + (op - ROP_QKV); }
MK_HD inline int rev_lm(const Shape &s) { return 1 + 5 * s.L; }
MK_HD inline int rnum_events(const Shape &s) { return 2 + 5 * s.L; }

// Geometry of a GEMV op: `tiles` tiles of 128 weight rows, each `slabs`
// pages of 128 reduction columns; a page p is tile p / slabs, slab p % slabs.
struct RGemv {
    int tiles, slabs, K;
};
MK_HD inline RGemv rgemv(const Shape &s, int op) {
    RGemv g;
    switch (op) {
    case ROP_QKV: g.tiles = (s.QD + 2 * s.KD) / kRTile; g.K = s.H; break;
    case ROP_OPROJ: g.tiles = s.H / kRTile; g.K = s.QD; break;
    case ROP_GATEUP: g.tiles = 2 * s.F / kRTile; g.K = s.H; break;   // 64 gate + the 64 matching up rows
    case ROP_DOWN: g.tiles = s.H / kRTile; g.K = s.F; break;
    default: g.tiles = (s.V + kRTile - 1) / kRTile; g.K = s.H; break;  // ROP_LMHEAD
    }
    g.slabs = g.K / kRSlab;
    return g;
}

// Layout of a weight page (tile i, slab j; 32 KB): the K-major canonical
// layout of tcgen05 without swizzle, 16-byte core-matrix rows of 8 bf16:
// element (m, k) at byte (k / 8) * 2048 + (m / 8) * 128 + (m % 8) * 16 +
// (k % 8) * 2 -- leading byte offset 2048 (next 8 columns), stride byte
// offset 128 (next 8 rows).  One MMA (K = 16) reads 4 KB from column 16 kk.
MK_HD inline size_t rpage_elem(int m, int k) {
    return (size_t)(k >> 3) * 1024 + (size_t)(m >> 3) * 64 + (size_t)(m & 7) * 8 + (size_t)(k & 7);
}
// Layout of an activation slab (128 columns of the kRowsN MMA columns, 8 KB):
// element (n, k) at byte (k / 8) * 512 + (n / 8) * 128 + (n % 8) * 16 +
// (k % 8) * 2 -- leading byte offset 512, stride byte offset 128.  Column n
// < kRows is row n's high half, n >= kRows row n - kRows's low half.
MK_HD inline size_t rslab_elem(int n, int k) {
    return (size_t)(k >> 3) * 256 + (size_t)(n >> 3) * 64 + (size_t)(n & 7) * 8 + (size_t)(k & 7);
}
// Index (bf16 elements) of input column k, MMA column n, in an activation
// buffer of K columns (K / 128 slabs back to back).
MK_HD inline size_t rx_elem(int n, int k) {
    return (size_t)(k / kRSlab) * (kRSlabBytes / 2) + rslab_elem(n, k % kRSlab);
}

// Attention positions per page (K block then V block).
MK_HD inline int rattn_pos_per_page(int d) { return kRPageBytes / (4 * d); }
// A row's positions are split into chunks of at least this many (one
// attention item each); contexts up to this long need no merge.  Longer
// chunks measured faster at the batched workloads' positions (<= ~2200):
// batch 16, 1024 / 2048 / 4096 positions: 1.816 / 1.652 / 1.591 ms/step --
// a merge costs chunk 0's item a wait for the slowest chunk and an extra
// pass, more than the longer items cost in balance.
constexpr int kRAttnChunk = 4096;

// Per-layer device buffers of the rows step.
//  xq, xo, xg, xd: the bf16 high/low inputs of QKV (rmsnorm gain folded in,
//    the 1/rms scale applied in the epilogue), OPROJ, GATEUP, DOWN
//    [K / 128 slabs][8 KB]
//  xa, xb: fp32 residual stream after OPROJ and DOWN [kRows][H]
//  ssq, ssg: per tile of the producing op, per row, the sum of squares of
//    the residual stream that feeds QKV (written by the previous layer's
//    DOWN or EMBED) and GATEUP (written by OPROJ) [H / 128][kRows]
//  q: rotated queries, scaled by 1/sqrt(d) [kRows][nq * d] fp32
//  part: tagged attention partials [kRows][nkv][NC][G * (d + 2)]
//  acc_*: split-tile accumulators [tiles][128][kRows] fp32 (zero between
//    uses), cnt_*: pages accumulated per tile (epoch-scaled) [tiles]
//  rdy_*: per input slab of the op, the releases of its writers so far
//    (epoch-scaled) [K / 128]: a GEMV task's pages start on a slab as soon
//    as that slab is written, not when the whole producing op is done
struct RLayerBuf {
    uint16_t *xq, *xo, *xg, *xd;
    float *xa, *xb;
    float *ssq, *ssg;
    float *q;
    uint64_t *part;
    float *acc[4];          // QKV, OPROJ, GATEUP, DOWN (index: rgemv_slot)
    uint32_t *cnt[4];
    uint32_t *rdy[4];       // per input slab of QKV, OPROJ, GATEUP, DOWN: writers that have
                            //  released it (epoch-scaled: rslab_writers(op) per step)
};

// Index of a layer's GEMV op in RLayerBuf::acc / cnt (the attention op sits
// between QKV and OPROJ in the op order, so the op values are not it).
MK_HD inline int rgemv_slot(int op) {
    return op == ROP_QKV ? 0 : op == ROP_OPROJ ? 1 : op == ROP_GATEUP ? 2 : 3;
}

// Releases of one input slab (128 columns) of a GEMV op per step: one
// producing tile for the QKV, gate/up and LM-head inputs (a residual
// tile of the down projection, the O-projection or the embedding); two
// gate/up tiles of 64 outputs, one release per writer warp each, for the
// down projection's; one per row and KV head covering the slab for the
// O-projection's (the attention output: every chunk-0 item of a (row, KV
// head) releases, active or not, so the count is the same every step).
MK_HD inline uint32_t rslab_writers(const Shape &s, int op) {
    if (op == ROP_DOWN) return 4u;
    if (op != ROP_OPROJ) return 1u;
    const int gd = s.G * s.d;
    return (uint32_t)kRows * (uint32_t)(gd >= kRSlab ? 1 : kRSlab / gd);
}

// Device pointers of one layer's weights (library copies in the page
// layout) and caches.
struct RLayerW {
    const uint16_t *qkv, *wo, *gu, *wd;   // pages of tiles in order (tile-major, slab-minor)
    const uint16_t *g_attn, *g_mlp;       // RMSNorm gains (caller's)
    uint16_t *kc, *vc;                    // caller's caches [max_batch][nkv][max_seq][d]
};

// Rows of one kernel step: token, position, KV slot, and `pre`: how many of
// the row's positions were written before this launch (they stream through
// the page ring ahead of the step; the rest are read after the step's QKV).
struct RRow {
    int32_t tok, pos, slot, pre;
};

struct RParams {
    Shape s;
    // graph (tasks in queue order, `sm` holding the task id)
    const Task *qtasks;
    const int32_t *qoff;
    const uint32_t *thresholds;
    uint32_t *events;
    uint32_t *lm_cnt, *epoch, *done_cnt, *abort_flag;
    int num_lm_tasks;
    // model
    const RLayerW *layers;
    const uint16_t *embed;      // caller's [V][H] (row lookups)
    const uint16_t *lm;         // library copy in the page layout
    const uint16_t *g_final;
    const float2 *rope;         // [S][d/2] (cos, sin)
    // launch: n_total rows in n_steps kernel steps of up to kRows each.
    //  decode (positions != null): row b = tokens[b] at positions[b], slot b;
    //  prompt (positions == null): row i = tokens[i] at pf_start + i, slot
    //  pf_slot (consecutive positions of one sequence).
    const int32_t *tokens;
    const int32_t *positions;
    int n_total;
    int pf_slot, pf_start;
    int n_steps;
    int lm_from;                // the LM head runs for steps >= lm_from only
    int out_row0;               // outputs: rows >= out_row0 of the last step, at index r - out_row0
    float *logits;              // [rows out][V] or null
    int32_t *next_tok;          // [rows out]
    // scratch
    const RLayerBuf *buf;       // [L]
    uint16_t *xlm;              // LM-head input [H / 128][8 KB]
    float *sslm;                // [H / 128][kRows]
    uint32_t *rdy_lm;           // LM-head input slab releases (epoch-scaled) [H / 128]
    float *x0;                  // embedding rows [kRows][H] fp32
    float *lm_acc;              // [tiles][128][kRows]
    uint32_t *lm_tcnt;          // [tiles]
    float *amax_val;            // [kRows][num_lm_tasks]
    int32_t *amax_idx;
    ErrWord *err;
    TraceRec *trace;            // per-task timestamps of the last step (MK_FLAG_TRACE), or null:
                                //  t_ready: the scheduler saw the dependency met; t_wait: the MMA
                                //  issuer began the task's pages; t_start: the compute warps began;
                                //  t_input: first accumulator (or attention queries) in hand;
                                //  t_done: epilogue done; t_end: completion posted
    unsigned long long *sm_stats;   // [num_sms][16] ns spent per wait kind (MK_FLAG_TRACE), or null: RStat
    unsigned long long timeout_ns;
};

// Per-SM time accounting of the batched step (MK_FLAG_TRACE), ns.
enum RStat {
    RS_LOAD_SLOT = 0,    // loader waiting for a free page slot
    RS_LOAD_TOTAL = 1,
    RS_SCHED_DEP = 2,    // scheduler waiting on event counters
    RS_SCHED_SLAB = 3,   // scheduler waiting for a free activation slab slot
    RS_MMA_PAGE = 4,     // MMA issuer waiting for a weight page
    RS_MMA_SLAB = 5,     // MMA issuer waiting for an activation slab
    RS_MMA_ACC = 6,      // MMA issuer waiting for a free accumulator
    RS_MMA_TOTAL = 7,
    RS_CMP_READY = 8,    // compute warp 0 waiting for the scheduler
    RS_CMP_ACC = 9,      // compute warp 0 waiting for an accumulator
    RS_CMP_KV = 10,      // compute warp 0 waiting for a K/V page
    RS_CMP_ATTN = 11,    // compute warp 0 in attention items (all of it)
    RS_CMP_EPI = 12,     // compute warp 0 in GEMV tasks, accumulator waits excluded
    RS_CMP_TOTAL = 13,
    RS_CMP_SYNC = 14,    // compute warp 0 in group barriers
    kRStats = 16
};

MK_HD inline int rrows_in_step(const RParams &p, int step) {
    const int n = p.n_total - step * kRows;
    return n < kRows ? n : kRows;
}
#if defined(__CUDACC__)
__device__ __forceinline__ RRow rrow(const RParams &p, int step, int r) {
    RRow w;
    if (p.positions) {
        w.tok = p.tokens[r];
        w.pos = p.positions[r];
        w.slot = r;
        w.pre = w.pos;
    } else {
        const int i = step * kRows + r;
        w.tok = p.tokens[i];
        w.pos = p.pf_start + i;
        w.slot = p.pf_slot;
        w.pre = p.pf_start;
    }
    return w;
}
#endif

// Host planning of the rows graph (see mk_rows_graph.cpp).
PlanSizes rplan_sizes(const Shape &s, int num_sms);
void rplan_build(const Shape &s, int num_sms, Plan &p);

}  // namespace mk
