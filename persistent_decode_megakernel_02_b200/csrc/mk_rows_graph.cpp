// mk_rows_graph.cpp -- host-side builder of the rows step's static task
// graph (the batched step on tensor cores, mk_rows.cu).
//
// The same task/event model as the batch-1 graph (mk_graph.cpp; MPK's
// tasks and events, "显著提升小LLM的性能，所有kernel集成一个巨大kernel！",
// Figure 2 / Figure 3 text): one event per op, threshold = the number of
// tasks that trigger it, static per-SM queues in op order.  What differs is
// the unit of work of a matrix op: a page of 128 weight rows x 128 reduction
// columns, one 128 x N x 128 tensor-core contraction.  An op's pages (tile
// by tile, the reduction columns of a tile in order) are cut into one
// contiguous range per SM, of equal size +-1, so every op spreads over every
// SM whatever its shape; a tile whose pages land on several SMs is summed in
// global memory and finished by the last of them (mk_rows.cu).
//
// No heap allocation: the caller sizes the arrays with rplan_sizes().
#include "mk_rows.h"

namespace mk {

namespace {

constexpr int kMaxSms = 1024;

int gemv_tasks(const Shape &s, int op, int num_sms) {
    const RGemv g = rgemv(s, op);
    const int pages = g.tiles * g.slabs;
    return pages < num_sms ? pages : num_sms;
}

int attn_items(const Shape &s) { return kRows * s.nkv * s.NC; }

struct RBuilder {
    const Shape &s;
    Plan &p;
    int64_t load[kMaxSms];
    int order[kMaxSms];
    int nt = 0;

    RBuilder(const Shape &s_, Plan &p_) : s(s_), p(p_) {
        for (int i = 0; i < p.num_sms; ++i) load[i] = 0;
    }

    void sort_by_load() {
        const int n = p.num_sms;
        for (int i = 0; i < n; ++i) order[i] = i;
        for (int i = 1; i < n; ++i) {   // insertion sort, stable
            const int v = order[i];
            int j = i - 1;
            while (j >= 0 && load[order[j]] > load[v]) { order[j + 1] = order[j]; --j; }
            order[j + 1] = v;
        }
    }

    void add(int kind, int layer, int dep, int trig, int begin, int end, int sm, int slot, int64_t bytes) {
        Task &t = p.tasks[nt];
        t.kind = kind; t.layer = layer; t.dep = dep; t.trig = trig;
        t.begin = begin; t.end = end; t.sm = sm; t.slot = slot;
        if (p.bytes) p.bytes[nt] = bytes;
        load[sm] += bytes;
        ++nt;
    }

    // Pages [0, tiles * slabs) in contiguous ranges over the least-loaded SMs.
    int gemv_op(int op, int layer, int dep, int trig) {
        const RGemv g = rgemv(s, op);
        const int pages = g.tiles * g.slabs;
        const int T = pages < p.num_sms ? pages : p.num_sms;
        const int base = pages / T, extra = pages % T;
        sort_by_load();
        int pg = 0;
        for (int i = 0; i < T; ++i) {
            const int n = base + (i < extra ? 1 : 0);
            add(op, layer, dep, trig, pg, pg + n, order[i], i, (int64_t)n * kRPageBytes);
            pg += n;
        }
        return T;
    }

    // One task per (row, KV head, chunk), chunk-descending so that chunk 0's
    // task -- which merges the chunks of its (row, KV head) -- comes after
    // every other chunk it waits for on every queue.
    int attn_op(int layer, int dep, int trig) {
        const int items = attn_items(s);
        const int heads = kRows * s.nkv;
        const int per_chunk = (s.S + s.NC - 1) / s.NC;
        const int64_t est = (int64_t)4 * s.d * per_chunk;
        for (int i = 0; i < items; i += p.num_sms) {
            sort_by_load();
            const int n = items - i < p.num_sms ? items - i : p.num_sms;
            for (int k = 0; k < n; ++k) {
                const int ord = i + k;
                const int c = s.NC - 1 - ord / heads;
                const int item = (ord % heads) * s.NC + c;
                add(ROP_ATTN, layer, dep, trig, item, item + 1, order[k], ord, est);
            }
        }
        return items;
    }

    // The embedding rows, one task per 128 hidden columns.
    int embed_op(int dep, int trig) {
        const int tiles = s.H / kRTile;
        sort_by_load();
        for (int i = 0; i < tiles; ++i)
            add(ROP_EMBED, 0, dep, trig, i, i + 1, order[i % p.num_sms], i, (int64_t)kRows * kRTile * 2);
        return tiles;
    }
};

}  // namespace

PlanSizes rplan_sizes(const Shape &s, int num_sms) {
    const int per_layer = gemv_tasks(s, ROP_QKV, num_sms) + attn_items(s) + gemv_tasks(s, ROP_OPROJ, num_sms) +
                          gemv_tasks(s, ROP_GATEUP, num_sms) + gemv_tasks(s, ROP_DOWN, num_sms);
    PlanSizes z;
    z.num_tasks = s.H / kRTile + s.L * per_layer + gemv_tasks(s, ROP_LMHEAD, num_sms);
    z.num_events = rnum_events(s);
    z.num_ops = z.num_events;
    return z;
}

void rplan_build(const Shape &s, int num_sms, Plan &p) {
    p.s = s;
    p.num_sms = num_sms;
    const PlanSizes z = rplan_sizes(s, num_sms);
    p.num_events = z.num_events;
    p.num_ops = z.num_ops;
    RBuilder b(s, p);
    const int e_lm = rev_lm(s);
    // a step's embedding waits for the previous step's LM head (epoch - 1)
    p.thresholds[rev_embed()] = b.embed_op(e_lm, rev_embed());
    for (int l = 0; l < s.L; ++l) {
        const int in = l == 0 ? rev_embed() : rev_op(l - 1, ROP_DOWN);
        p.thresholds[rev_op(l, ROP_QKV)] = b.gemv_op(ROP_QKV, l, in, rev_op(l, ROP_QKV));
        p.thresholds[rev_op(l, ROP_ATTN)] = b.attn_op(l, rev_op(l, ROP_QKV), rev_op(l, ROP_ATTN));
        p.thresholds[rev_op(l, ROP_OPROJ)] = b.gemv_op(ROP_OPROJ, l, rev_op(l, ROP_ATTN), rev_op(l, ROP_OPROJ));
        p.thresholds[rev_op(l, ROP_GATEUP)] = b.gemv_op(ROP_GATEUP, l, rev_op(l, ROP_OPROJ), rev_op(l, ROP_GATEUP));
        p.thresholds[rev_op(l, ROP_DOWN)] = b.gemv_op(ROP_DOWN, l, rev_op(l, ROP_GATEUP), rev_op(l, ROP_DOWN));
    }
    p.thresholds[e_lm] = b.gemv_op(ROP_LMHEAD, s.L, rev_op(s.L - 1, ROP_DOWN), e_lm);
    p.num_lm_tasks = (int)p.thresholds[e_lm];
    p.num_tasks = b.nt;

    for (int i = 0; i <= num_sms; ++i) p.qoff[i] = 0;
    for (int i = 0; i < p.num_tasks; ++i) p.qoff[p.tasks[i].sm + 1]++;
    for (int i = 0; i < num_sms; ++i) p.qoff[i + 1] += p.qoff[i];
    int max_q = 0;
    for (int i = 0; i < num_sms; ++i) {
        const int n = p.qoff[i + 1] - p.qoff[i];
        if (n > max_q) max_q = n;
    }
    p.max_queue = max_q;
    for (int i = 0; i < num_sms; ++i) b.load[i] = p.qoff[i];
    for (int i = 0; i < p.num_tasks; ++i) p.queue[b.load[p.tasks[i].sm]++] = i;
}

}  // namespace mk
