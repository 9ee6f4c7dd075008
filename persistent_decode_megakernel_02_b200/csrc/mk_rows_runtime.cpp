// mk_rows_runtime.cpp -- host side of the batched ("rows") step: shape
// checks, the task graph, the library copies of the weights in the page
// layout, scratch, and the launches behind mk_decode_step (a batch of up to
// 16 sequences) and mk_prefill (a prompt, 16 tokens per kernel step, in one
// launch) for contexts created with max_batch > 1 or MK_FLAG_ROWS.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <new>
#include <vector>

#include "../../include/mk.h"
#include "mk_rows.h"

namespace mk {
size_t rows_smem_bytes();
cudaError_t rows_prepare();
cudaError_t rows_launch(const RParams &p, int grid, cudaStream_t stream);
cudaError_t repack_rows(uint16_t *dst, const uint16_t *src, const uint16_t *src2, long long rows, int K, int tiles,
                        cudaStream_t stream);

struct RowsCtx {
    Shape s{};
    int num_sms = 0;
    int num_tasks = 0, num_events = 0, num_lm_tasks = 0, max_queue = 0;
    std::vector<Task> h_tasks;
    std::vector<int32_t> h_queue, h_qoff;
    std::vector<uint32_t> h_thr;
    std::vector<void *> allocs;
    std::vector<RLayerBuf> h_buf;
    RParams p{};
    ErrWord *d_err = nullptr;
    // what mk_reset clears: counters, tagged partials, split accumulators
    struct Span { void *ptr; size_t bytes; };
    std::vector<Span> zero_on_reset;
};

namespace {

template <class T>
cudaError_t ralloc(RowsCtx *c, T **out, size_t count, bool zero_on_reset = false) {
    void *ptr = nullptr;
    size_t bytes = count * sizeof(T);
    if (bytes == 0) bytes = 16;
    cudaError_t e = cudaMalloc(&ptr, bytes);
    if (e != cudaSuccess) return e;
    c->allocs.push_back(ptr);
    e = cudaMemset(ptr, 0, bytes);
    if (e != cudaSuccess) return e;
    if (zero_on_reset) c->zero_on_reset.push_back({ptr, bytes});
    *out = static_cast<T *>(ptr);
    return cudaSuccess;
}

int map_err(cudaError_t e) {
    if (e == cudaSuccess) return MK_OK;
    if (e == cudaErrorMemoryAllocation) return MK_ERR_OOM;
    return MK_ERR_CUDA;
}

}  // namespace

// Shapes the rows step tiles: 128-row weight tiles and 128-column slabs
// everywhere, whole heads per tile, the attention scratch (G * d <= 512).
bool rows_shape_ok(const Shape &s) {
    if (s.H % kRTile || s.QD % kRTile || s.KD % kRTile || s.F % kRTile) return false;
    if (s.G != 1 && s.G != 2 && s.G != 4) return false;
    if (s.G * s.d > 512) return false;
    if (s.Bmax < 1 || s.Bmax > kRows) return false;
    return true;
}

int rows_default_chunks(int S) { return (S + kRAttnChunk - 1) / kRAttnChunk; }

void rows_destroy(RowsCtx *c) {
    if (!c) return;
    for (void *p : c->allocs) cudaFree(p);
    delete c;
}

int rows_create(const mk_config *cfg, const mk_weights *w, const mk_kv *kv, const Shape &s, int num_sms,
                RowsCtx **out) {
    *out = nullptr;
    if (!rows_shape_ok(s)) return MK_ERR_INVALID;
    if ((size_t)0 == rows_smem_bytes()) return MK_ERR_INVALID;
    RowsCtx *c = new (std::nothrow) RowsCtx;
    if (!c) return MK_ERR_OOM;
    c->s = s;
    c->num_sms = num_sms;
    cudaError_t e = cudaSuccess;
#define RK_TRY(expr) do { e = (expr); if (e != cudaSuccess) { rows_destroy(c); return map_err(e); } } while (0)

    // ---- task graph (host), queue order on the device
    const PlanSizes z = rplan_sizes(s, num_sms);
    c->h_tasks.resize(z.num_tasks);
    c->h_queue.resize(z.num_tasks);
    c->h_qoff.resize(num_sms + 1);
    c->h_thr.resize(z.num_events);
    Plan plan;
    plan.tasks = c->h_tasks.data(); plan.queue = c->h_queue.data(); plan.qoff = c->h_qoff.data();
    plan.thresholds = c->h_thr.data(); plan.bytes = nullptr;
    rplan_build(s, num_sms, plan);
    c->num_tasks = plan.num_tasks;
    c->num_events = plan.num_events;
    c->num_lm_tasks = plan.num_lm_tasks;
    c->max_queue = plan.max_queue;

    RParams &p = c->p;
    p.s = s;
    Task *d_q; int32_t *d_qoff; uint32_t *d_thr, *d_ev, *d_ctrl;
    RK_TRY(ralloc(c, &d_q, c->num_tasks));
    RK_TRY(ralloc(c, &d_qoff, num_sms + 1));
    RK_TRY(ralloc(c, &d_thr, c->num_events));
    RK_TRY(ralloc(c, &d_ev, c->num_events, true));
    RK_TRY(ralloc(c, &d_ctrl, 8, true));
    RK_TRY(ralloc(c, &c->d_err, 1, true));
    {
        std::vector<Task> qt(c->num_tasks);
        for (int i = 0; i < c->num_tasks; ++i) {
            qt[i] = c->h_tasks[c->h_queue[i]];
            qt[i].sm = c->h_queue[i];
        }
        RK_TRY(cudaMemcpy(d_q, qt.data(), sizeof(Task) * c->num_tasks, cudaMemcpyHostToDevice));
    }
    RK_TRY(cudaMemcpy(d_qoff, c->h_qoff.data(), sizeof(int32_t) * (num_sms + 1), cudaMemcpyHostToDevice));
    RK_TRY(cudaMemcpy(d_thr, c->h_thr.data(), sizeof(uint32_t) * c->num_events, cudaMemcpyHostToDevice));

    // ---- RoPE table (cos/sin of pos * theta^(-2i/d), in double)
    const int half = s.d / 2;
    {
        std::vector<float> rope((size_t)s.S * half * 2);
        for (int pos = 0; pos < s.S; ++pos)
            for (int i = 0; i < half; ++i) {
                const double ang = (double)pos * std::pow((double)cfg->rope_theta, -2.0 * i / (double)s.d);
                rope[((size_t)pos * half + i) * 2 + 0] = (float)std::cos(ang);
                rope[((size_t)pos * half + i) * 2 + 1] = (float)std::sin(ang);
            }
        float2 *d_rope;
        RK_TRY(ralloc(c, &d_rope, (size_t)s.S * half));
        RK_TRY(cudaMemcpy(d_rope, rope.data(), sizeof(float) * rope.size(), cudaMemcpyHostToDevice));
        p.rope = d_rope;
    }

    // ---- weights in the page layout (library copies)
    std::vector<RLayerW> lw(s.L);
    {
        const size_t rb = 2 * (size_t)s.H;
        uint16_t *qkv_rm = nullptr;   // [wq; wk; wv] row-major staging
        RK_TRY(cudaMalloc(&qkv_rm, (size_t)(s.QD + 2 * s.KD) * rb));
        auto pages = [&](int op, uint16_t **dst) {
            const RGemv g = rgemv(s, op);
            return ralloc(c, dst, (size_t)g.tiles * g.slabs * (kRPageBytes / 2));
        };
        for (int l = 0; l < s.L && e == cudaSuccess; ++l) {
            uint16_t *q, *o, *gu, *dn;
            if (e == cudaSuccess) e = pages(ROP_QKV, &q);
            if (e == cudaSuccess) e = pages(ROP_OPROJ, &o);
            if (e == cudaSuccess) e = pages(ROP_GATEUP, &gu);
            if (e == cudaSuccess) e = pages(ROP_DOWN, &dn);
            char *dq = (char *)qkv_rm;
            if (e == cudaSuccess) e = cudaMemcpy(dq, w->wq[l], (size_t)s.QD * rb, cudaMemcpyDeviceToDevice);
            if (e == cudaSuccess)
                e = cudaMemcpy(dq + (size_t)s.QD * rb, w->wk[l], (size_t)s.KD * rb, cudaMemcpyDeviceToDevice);
            if (e == cudaSuccess)
                e = cudaMemcpy(dq + (size_t)(s.QD + s.KD) * rb, w->wv[l], (size_t)s.KD * rb, cudaMemcpyDeviceToDevice);
            if (e == cudaSuccess)
                e = repack_rows(q, qkv_rm, nullptr, s.QD + 2 * s.KD, s.H, rgemv(s, ROP_QKV).tiles, 0);
            if (e == cudaSuccess)
                e = repack_rows(o, (const uint16_t *)w->wo[l], nullptr, s.H, s.QD, rgemv(s, ROP_OPROJ).tiles, 0);
            if (e == cudaSuccess)
                e = repack_rows(gu, (const uint16_t *)w->wg[l], (const uint16_t *)w->wu[l], s.F, s.H,
                                rgemv(s, ROP_GATEUP).tiles, 0);
            if (e == cudaSuccess)
                e = repack_rows(dn, (const uint16_t *)w->wd[l], nullptr, s.H, s.F, rgemv(s, ROP_DOWN).tiles, 0);
            if (e == cudaSuccess) e = cudaDeviceSynchronize();   // the staging buffer is reused
            lw[l].qkv = q; lw[l].wo = o; lw[l].gu = gu; lw[l].wd = dn;
            lw[l].g_attn = (const uint16_t *)w->attn_norm[l];
            lw[l].g_mlp = (const uint16_t *)w->mlp_norm[l];
            lw[l].kc = (uint16_t *)kv->k[l];
            lw[l].vc = (uint16_t *)kv->v[l];
        }
        cudaFree(qkv_rm);
        if (e != cudaSuccess) { rows_destroy(c); return map_err(e); }
        uint16_t *lm;
        RK_TRY(pages(ROP_LMHEAD, &lm));
        RK_TRY(repack_rows(lm, (const uint16_t *)w->lm_head, nullptr, s.V, s.H, rgemv(s, ROP_LMHEAD).tiles, 0));
        RK_TRY(cudaDeviceSynchronize());
        p.lm = lm;
        RLayerW *d_lw;
        RK_TRY(ralloc(c, &d_lw, s.L));
        RK_TRY(cudaMemcpy(d_lw, lw.data(), sizeof(RLayerW) * s.L, cudaMemcpyHostToDevice));
        p.layers = d_lw;
    }

    // ---- scratch
    {
        const size_t xh = (size_t)(s.H / kRSlab) * (kRSlabBytes / 2);      // bf16 elements of an H-column input
        const size_t xqd = (size_t)(s.QD / kRSlab) * (kRSlabBytes / 2);
        const size_t xf = (size_t)(s.F / kRSlab) * (kRSlabBytes / 2);
        const size_t tiles_h = s.H / kRTile;
        c->h_buf.resize(s.L);
        for (int l = 0; l < s.L; ++l) {
            RLayerBuf &b = c->h_buf[l];
            RK_TRY(ralloc(c, &b.xq, xh));
            RK_TRY(ralloc(c, &b.xo, xqd));
            RK_TRY(ralloc(c, &b.xg, xh));
            RK_TRY(ralloc(c, &b.xd, xf));
            RK_TRY(ralloc(c, &b.xa, (size_t)kRows * s.H));
            RK_TRY(ralloc(c, &b.xb, (size_t)kRows * s.H));
            RK_TRY(ralloc(c, &b.ssq, tiles_h * kRows));
            RK_TRY(ralloc(c, &b.ssg, tiles_h * kRows));
            RK_TRY(ralloc(c, &b.q, (size_t)kRows * s.QD));
            RK_TRY(ralloc(c, &b.part, (size_t)kRows * s.nkv * s.NC * s.G * (s.d + 2), true));
            for (int op : {ROP_QKV, ROP_OPROJ, ROP_GATEUP, ROP_DOWN}) {
                const RGemv g = rgemv(s, op);
                RK_TRY(ralloc(c, &b.acc[rgemv_slot(op)], (size_t)g.tiles * kRTile * kRows, true));
                RK_TRY(ralloc(c, &b.cnt[rgemv_slot(op)], (size_t)g.tiles, true));
                RK_TRY(ralloc(c, &b.rdy[rgemv_slot(op)], (size_t)g.slabs, true));
            }
        }
        RLayerBuf *d_buf;
        RK_TRY(ralloc(c, &d_buf, s.L));
        RK_TRY(cudaMemcpy(d_buf, c->h_buf.data(), sizeof(RLayerBuf) * s.L, cudaMemcpyHostToDevice));
        p.buf = d_buf;
        RK_TRY(ralloc(c, &p.xlm, xh));
        RK_TRY(ralloc(c, &p.sslm, tiles_h * kRows));
        RK_TRY(ralloc(c, &p.rdy_lm, (size_t)(s.H / kRSlab), true));
        RK_TRY(ralloc(c, &p.x0, (size_t)kRows * s.H));
        const RGemv glm = rgemv(s, ROP_LMHEAD);
        RK_TRY(ralloc(c, &p.lm_acc, (size_t)glm.tiles * kRTile * kRows, true));
        RK_TRY(ralloc(c, &p.lm_tcnt, (size_t)glm.tiles, true));
        RK_TRY(ralloc(c, &p.amax_val, (size_t)kRows * c->num_lm_tasks));
        RK_TRY(ralloc(c, &p.amax_idx, (size_t)kRows * c->num_lm_tasks));
    }
    if (cfg->flags & MK_FLAG_TRACE) {
        std::vector<TraceRec> tr(c->num_tasks);
        for (int i = 0; i < c->num_tasks; ++i) {
            const Task &t = c->h_tasks[i];
            tr[i] = TraceRec{0, 0, 0, 0, 0, 0, t.sm, t.kind, t.layer, t.trig};
        }
        RK_TRY(ralloc(c, &p.trace, c->num_tasks));
        RK_TRY(ralloc(c, &p.sm_stats, (size_t)num_sms * kRStats, true));
        RK_TRY(cudaMemcpy(p.trace, tr.data(), sizeof(TraceRec) * c->num_tasks, cudaMemcpyHostToDevice));
    }
    RK_TRY(rows_prepare());
#undef RK_TRY

    p.qtasks = d_q; p.qoff = d_qoff; p.thresholds = d_thr; p.events = d_ev;
    p.lm_cnt = d_ctrl + 0; p.epoch = d_ctrl + 1; p.done_cnt = d_ctrl + 2; p.abort_flag = d_ctrl + 3;
    p.num_lm_tasks = c->num_lm_tasks;
    p.embed = (const uint16_t *)w->embed;
    p.g_final = (const uint16_t *)w->final_norm;
    p.err = c->d_err;
    p.timeout_ns = cfg->timeout_ns > 0 ? (unsigned long long)cfg->timeout_ns : 2000000000ull;
    *out = c;
    return MK_OK;
}

int rows_step(RowsCtx *c, const int32_t *tokens, const int32_t *positions, int batch, float *logits,
              int32_t *next_tok, cudaStream_t stream) {
    RParams p = c->p;
    p.tokens = tokens;
    p.positions = positions;
    p.n_total = batch;
    p.pf_slot = 0;
    p.pf_start = 0;
    p.n_steps = 1;
    p.lm_from = 0;
    p.out_row0 = 0;
    p.logits = logits;
    p.next_tok = next_tok;
    return rows_launch(p, c->num_sms, stream) == cudaSuccess ? MK_OK : MK_ERR_CUDA;
}

int rows_prefill(RowsCtx *c, const int32_t *tokens, int n, int slot, int start, float *logits, int32_t *next_tok,
                 cudaStream_t stream) {
    RParams p = c->p;
    p.tokens = tokens;
    p.positions = nullptr;
    p.n_total = n;
    p.pf_slot = slot;
    p.pf_start = start;
    p.n_steps = (n + kRows - 1) / kRows;
    p.lm_from = p.n_steps - 1;
    p.out_row0 = n - (p.n_steps - 1) * kRows - 1;   // the prompt's last token
    p.logits = logits;
    p.next_tok = next_tok;
    return rows_launch(p, c->num_sms, stream) == cudaSuccess ? MK_OK : MK_ERR_CUDA;
}

RParams rows_params(const RowsCtx *c) { return c->p; }

int rows_reset(RowsCtx *c) {
    for (const auto &z : c->zero_on_reset)
        if (cudaMemset(z.ptr, 0, z.bytes) != cudaSuccess) return MK_ERR_CUDA;
    if (cudaMemcpy(const_cast<uint32_t *>(c->p.thresholds), c->h_thr.data(), sizeof(uint32_t) * c->num_events,
                   cudaMemcpyHostToDevice) != cudaSuccess)
        return MK_ERR_CUDA;
    return MK_OK;
}

}  // namespace mk
