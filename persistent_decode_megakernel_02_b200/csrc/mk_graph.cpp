// mk_graph.cpp -- host-side builder of the static task graph.
//
// The graph follows the MPK task/event model described on the page
// "显著提升小LLM的性能，所有kernel集成一个巨大kernel！" (Figure 2 / Figure 3 text):
// every op is split into tasks, each task runs on one SM, has one dependent
// event it waits for and one triggering event it bumps when done; an event
// fires when its counter reaches its threshold (the number of tasks that
// trigger it).  Tasks are placed in static per-SM queues (the Hazy page's
// per-SM "execution plan"), ops in model order, so every queue is
// dependency-ordered and the graph cannot deadlock.
//
// Placement balances weight bytes per SM across the whole step rather than
// per op: each op's tiles go to the SMs that have streamed the fewest bytes
// so far, so the per-SM loaders see equal totals.
//
// No heap allocation: the caller sizes the arrays with plan_sizes().
#include "mk.h"
#include "mk_internal.h"

namespace mk {

static constexpr int kMaxSms = 1024;

bool plan_attention(Shape &s, int num_sms, int flags, int attn_chunks) {
    const bool kv = (flags & MK_FLAG_ATTN_KV_ITEMS) != 0, qi = (flags & MK_FLAG_ATTN_Q_ITEMS) != 0;
    if (kv && qi) return false;
    // q heads an item could take: the largest divisor of G whose heads fit
    // the item's shared state
    int hg = 1;
    for (int h = s.G; h > 1; --h)
        if (s.G % h == 0 && h * s.d <= kAttnHeadDims) { hg = h; break; }
    int cap = (s.S + kAttnChunkPositions - 1) / kAttnChunkPositions;   // chunks a full cache needs
    if (cap < 1) cap = 1;
    int per_q = num_sms / (s.Bmax * s.nq);                             // chunks per q head the SMs give
    if (per_q < 1) per_q = 1;
    s.HA = (kv || (!qi && cap > per_q)) ? hg : 1;
    // the merge's shared staging holds the chunk partials (d + 2 floats
    // each) of every q head of an item
    auto fits = [&](long long nc, int ha) { return nc * ha * (s.d + 2) <= kStageFloats; };
    // chosen by default, KV-head items give way to q-head items where a
    // given chunk count's partials would not fit the merge's staging area
    if (!kv && s.HA > 1 && attn_chunks > 0 && !fits(attn_chunks, s.HA)) s.HA = 1;
    int nc = attn_chunks;
    if (nc <= 0) {
        nc = num_sms / (s.Bmax * (s.nq / s.HA));
        if (nc < 1) nc = 1;
        if (nc > cap) nc = cap;
        while (nc > 1 && !fits(nc, s.HA)) --nc;
    }
    s.NC = nc;
    return nc <= 4096 && fits(nc, s.HA);
}

// Tiles per scheduling unit of a GEMV op: tasks of ops whose pages pass
// through tensor memory must start on a 16-page-row boundary (the TMEM page
// order is laid out on that grid), so 8-row tiles of 2048 columns go in pairs.
static int gemv_unit(const Shape &s, int kind) {
    if (!tmem_page_op(s, kind)) return 1;
    const int page_rows_per_tile = tile_rows(s, kind, 0) * (op_k(s, kind) / kRowK);
    return page_rows_per_tile < 16 ? 16 / page_rows_per_tile : 1;
}

PlanSizes plan_sizes(const Shape &s, int num_sms) {
    OpTiles t = op_tiles(s);
    auto ntask = [&](int kind, int tiles) {
        const int u = gemv_unit(s, kind);
        const int units = (tiles + u - 1) / u;
        return units < num_sms ? units : num_sms;
    };
    PlanSizes z;
    int per_layer = ntask(OP_QKV, t.qkv) + t.attn_items + ntask(OP_OPROJ, t.oproj) +
                    ntask(OP_GATEUP, t.gateup) + ntask(OP_DOWN, t.down);
    z.num_tasks = s.L * per_layer + ntask(OP_LMHEAD, t.lmhead);
    z.num_events = 5 * s.L + 1;
    z.num_ops = 5 * s.L + 1;
    return z;
}

namespace {

struct Builder {
    const Shape &s;
    Plan &p;
    int64_t load[kMaxSms];
    int order[kMaxSms];
    int nt = 0;

    Builder(const Shape &s_, Plan &p_) : s(s_), p(p_) {
        for (int i = 0; i < p.num_sms; ++i) load[i] = 0;
    }

    // SMs sorted by bytes assigned so far (ties: lower index first).
    void sort_by_load() {
        int n = p.num_sms;
        for (int i = 0; i < n; ++i) order[i] = i;
        for (int i = 1; i < n; ++i) {  // insertion sort, stable
            int v = order[i];
            int j = i - 1;
            while (j >= 0 && load[order[j]] > load[v]) { order[j + 1] = order[j]; --j; }
            order[j + 1] = v;
        }
    }

    Task &add(int kind, int layer, int dep, int trig, int begin, int end, int sm, int slot,
              int64_t bytes) {
        Task &t = p.tasks[nt];
        t.kind = kind; t.layer = layer; t.dep = dep; t.trig = trig;
        t.begin = begin; t.end = end; t.sm = sm; t.slot = slot;
        if (p.bytes) p.bytes[nt] = bytes;
        load[sm] += bytes;
        ++nt;
        return t;
    }

    // Split the op's `ntiles` tiles over the least-loaded SMs, one
    // contiguous tile range per task, with equal unit counts (+-1) (a unit
    // is one tile, or two 8-row tiles when pages pass through tensor
    // memory).  Returns the number of tasks.
    int gemv_op(int kind, int layer, int dep, int trig, int ntiles) {
        const int K = op_k(s, kind);
        const int unit = gemv_unit(s, kind);
        const int nunits = (ntiles + unit - 1) / unit;
        int T = nunits < p.num_sms ? nunits : p.num_sms;
        int base = nunits / T, extra = nunits % T;
        sort_by_load();
        int tile = 0;
        for (int i = 0; i < T; ++i) {
            int n = (base + (i < extra ? 1 : 0)) * unit;
            if (tile + n > ntiles) n = ntiles - tile;
            long long rows = tile_row_offset(s, kind, tile + n) - tile_row_offset(s, kind, tile);
            if (kind == OP_LMHEAD) {
                long long valid = (long long)s.V - tile_row_offset(s, kind, tile);
                if (rows > valid) rows = valid;
            }
            add(kind, layer, dep, trig, tile, tile + n, order[i], i, rows * 2LL * K);
            tile += n;
        }
        return T;
    }

    // One task per attention item.  Items go to distinct SMs (the least
    // loaded ones) so an SM runs a second item of the same op only when
    // there are more items than SMs.
    // Work items (sequence, KV head, chunk) in descending chunk order: chunk
    // 0's task merges its KV head's partials and waits for the other chunks,
    // so on every queue it must come after any other chunk it could wait for
    // (the queues keep this order); chunks > 0 wait on nothing in the op.
    int attn_op(int layer, int dep, int trig) {
        OpTiles t = op_tiles(s);
        int per_chunk = (s.S + s.NC - 1) / s.NC;
        int64_t est = (int64_t)4 * s.d * per_chunk;   // K + V bf16 of one chunk at capacity
        const int heads = s.Bmax * (s.nq / s.HA);     // items per chunk index
        for (int i = 0; i < t.attn_items; i += p.num_sms) {
            sort_by_load();
            int n = t.attn_items - i < p.num_sms ? t.attn_items - i : p.num_sms;
            for (int k = 0; k < n; ++k) {
                const int ord = i + k;
                const int c = s.NC - 1 - ord / heads;
                const int item = (ord % heads) * s.NC + c;
                add(OP_ATTN, layer, dep, trig, item, item + 1, order[k], ord, est);
            }
        }
        return t.attn_items;
    }
};

}  // namespace

void plan_build(const Shape &s, int num_sms, Plan &p) {
    p.s = s;
    p.num_sms = num_sms;
    PlanSizes z = plan_sizes(s, num_sms);
    p.num_events = z.num_events;
    p.num_ops = z.num_ops;
    Builder b(s, p);
    OpTiles t = op_tiles(s);
    for (int l = 0; l < s.L; ++l) {
        int e_qkv = 5 * l, e_attn = e_qkv + 1, e_o = e_qkv + 2, e_gu = e_qkv + 3, e_down = e_qkv + 4;
        int dep_in = l == 0 ? -1 : e_qkv - 1;   // previous layer's down projection
        p.thresholds[e_qkv] = b.gemv_op(OP_QKV, l, dep_in, e_qkv, t.qkv);
        p.thresholds[e_attn] = b.attn_op(l, e_qkv, e_attn);
        p.thresholds[e_o] = b.gemv_op(OP_OPROJ, l, e_attn, e_o, t.oproj);
        p.thresholds[e_gu] = b.gemv_op(OP_GATEUP, l, e_o, e_gu, t.gateup);
        p.thresholds[e_down] = b.gemv_op(OP_DOWN, l, e_gu, e_down, t.down);
    }
    int e_lm = 5 * s.L;
    p.thresholds[e_lm] = b.gemv_op(OP_LMHEAD, s.L, e_lm - 1, e_lm, t.lmhead);
    p.num_lm_tasks = (int)p.thresholds[e_lm];
    p.num_tasks = b.nt;

    // group by SM, keeping op order inside each queue
    for (int i = 0; i <= num_sms; ++i) p.qoff[i] = 0;
    for (int i = 0; i < p.num_tasks; ++i) p.qoff[p.tasks[i].sm + 1]++;
    for (int i = 0; i < num_sms; ++i) p.qoff[i + 1] += p.qoff[i];
    int max_q = 0;
    for (int i = 0; i < num_sms; ++i) {
        int n = p.qoff[i + 1] - p.qoff[i];
        if (n > max_q) max_q = n;
    }
    p.max_queue = max_q;
    // stable fill: use the tail of qoff as a cursor by walking tasks in order
    // (cursor per SM kept in `b.load`, reused as scratch)
    for (int i = 0; i < num_sms; ++i) b.load[i] = p.qoff[i];
    for (int i = 0; i < p.num_tasks; ++i) {
        int sm = p.tasks[i].sm;
        p.queue[b.load[sm]++] = i;
    }
}

}  // namespace mk
