// mk_runtime.cpp -- implementation of the C ABI declared in include/mk.h:
// argument validation, task-graph construction (mk_graph.cpp), scratch
// allocation, and the one cooperative launch per decode step.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <new>
#include <vector>

#include "../../include/mk.h"
#include "mk_internal.h"
#include "mk_rows.h"

namespace mk {
size_t kernel_smem_bytes();
int kernel_launch_regs();
cudaError_t kernel_prepare();
cudaError_t kernel_occupancy(int *blocks_per_sm);
cudaError_t kernel_launch(const Params &p, int grid, cudaStream_t stream);
size_t tmem_pages_bytes(long long page_rows);
cudaError_t repack_tmem_pages(void *dst, const void *src, long long page_rows, cudaStream_t stream);
// the batched (rows) step: mk_rows_runtime.cpp
struct RowsCtx;
bool rows_shape_ok(const Shape &s);
int rows_default_chunks(int S);
int rows_create(const mk_config *cfg, const mk_weights *w, const mk_kv *kv, const Shape &s, int num_sms,
                RowsCtx **out);
int rows_step(RowsCtx *c, const int32_t *tokens, const int32_t *positions, int batch, float *logits,
              int32_t *next_tok, cudaStream_t stream);
int rows_prefill(RowsCtx *c, const int32_t *tokens, int n, int slot, int start, float *logits, int32_t *next_tok,
                 cudaStream_t stream);
int rows_reset(RowsCtx *c);
void rows_destroy(RowsCtx *c);
RParams rows_params(const RowsCtx *c);
size_t rows_smem_bytes();
}  // namespace mk

using namespace mk;

struct mk_ctx {
    int device = 0;
    mk_config cfg{};
    Shape s{};
    int num_sms = 0;
    int num_tasks = 0, num_events = 0, num_ops = 0, max_queue = 0, num_lm_tasks = 0;
    std::vector<Task> h_tasks;
    std::vector<int32_t> h_queue, h_qoff;
    std::vector<uint32_t> h_thresholds;
    // device allocations
    std::vector<void *> allocs;
    Params p{};            // template: step inputs filled per call
    ErrWord *d_err = nullptr;
    RowsCtx *rows = nullptr;             // the batched tensor-core step (max_batch > 1 or MK_FLAG_ROWS)
    RParams rp{};                        // its parameter template (host copy, for introspection)
    const uint16_t *lm_tmem = nullptr;   // library copy of the LM head in the TMEM page order
    long long steps = 0;
    bool failed = false;   // a device error was observed by mk_sync
};

namespace {

template <class T>
cudaError_t dalloc(mk_ctx *c, T **out, size_t count) {
    void *ptr = nullptr;
    size_t bytes = count * sizeof(T);
    if (bytes == 0) bytes = 16;
    cudaError_t e = cudaMalloc(&ptr, bytes);
    if (e != cudaSuccess) return e;
    c->allocs.push_back(ptr);
    *out = static_cast<T *>(ptr);
    return cudaSuccess;
}

bool aligned16(const void *p) { return p && ((uintptr_t)p & 15u) == 0; }

int shape_from_config(const mk_config *c, int num_sms, Shape &s) {
    if (!c) return MK_ERR_INVALID;
    if (c->layers < 1 || c->hidden < 8 || c->n_q_heads < 1 || c->n_kv_heads < 1 ||
        c->head_dim < 1 || c->ffn < 8 || c->vocab < 1 || c->max_seq < 1 || c->max_batch < 1)
        return MK_ERR_INVALID;
    if (c->max_batch > MK_MAX_BATCH) return MK_ERR_INVALID;
    const bool rows = c->max_batch > 1 || (c->flags & MK_FLAG_ROWS);
    if (c->n_q_heads % c->n_kv_heads != 0) return MK_ERR_INVALID;
    const int G = c->n_q_heads / c->n_kv_heads;
    if (G != 1 && G != 2 && G != 4 && G != 8) return MK_ERR_INVALID;
    if (c->head_dim != 64 && c->head_dim != 128) return MK_ERR_INVALID;
    static_assert(kMaxHidden == MK_MAX_HIDDEN && kMaxK == MK_MAX_K, "public bounds match the kernel's");
    if (c->hidden > kMaxHidden) return MK_ERR_INVALID;
    const long long QD = (long long)c->n_q_heads * c->head_dim;
    if (c->hidden % 8 || c->ffn % 8 || QD % 8) return MK_ERR_INVALID;
    if (c->hidden > kMaxK || c->ffn > kMaxK || QD > kMaxK) return MK_ERR_INVALID;
    if (!(c->rms_eps > 0.f) || !(c->rope_theta > 1.f)) return MK_ERR_INVALID;
    if (c->attn_chunks < 0 || c->timeout_ns < 0 || c->l2_lookahead_kb < 0) return MK_ERR_INVALID;
    if (c->poll_ns < 0 || c->poll_ns > 1000000) return MK_ERR_INVALID;
    if ((long long)c->max_seq * c->head_dim > (1LL << 40)) return MK_ERR_INVALID;
    if (num_sms < 1 || num_sms > 1024) return MK_ERR_INVALID;
    s.L = c->layers; s.H = c->hidden; s.nq = c->n_q_heads; s.nkv = c->n_kv_heads;
    s.d = c->head_dim; s.F = c->ffn; s.V = c->vocab; s.S = c->max_seq; s.Bmax = c->max_batch;
    s.G = G; s.QD = (int)QD; s.KD = c->n_kv_heads * c->head_dim;
    s.theta = c->rope_theta; s.eps = c->rms_eps;
    s.tmem = (c->flags & MK_FLAG_NO_TMEM_RING) ? 0 : 1;
    if (rows) {
        // the batched step: its own tiling, chunks of at least kRAttnChunk positions
        s.tmem = 0;
        s.HA = s.G;   // items per (row, KV head, chunk)
        s.NC = c->attn_chunks > 0 ? c->attn_chunks : rows_default_chunks(s.S);
        if (s.NC > 4096 || !rows_shape_ok(s)) return MK_ERR_INVALID;
        if (c->flags & MK_FLAG_EVENT_WAIT) return MK_ERR_INVALID;   // tasks always wait on events here
        return MK_OK;
    }
    if (!plan_attention(s, num_sms, c->flags, c->attn_chunks)) return MK_ERR_INVALID;
    return MK_OK;
}

int map_cuda(cudaError_t e) {
    if (e == cudaSuccess) return MK_OK;
    if (e == cudaErrorMemoryAllocation) return MK_ERR_OOM;
    return MK_ERR_CUDA;
}

void free_ctx(mk_ctx *c) {
    if (!c) return;
    for (void *p : c->allocs) cudaFree(p);
    rows_destroy(c->rows);
    delete c;
}

bool is_rows(const mk_config *c) { return c->max_batch > 1 || (c->flags & MK_FLAG_ROWS); }

}  // namespace

namespace mk {
// The devices the library runs on.  The binary holds sm_100a code only,
// which is arch-specific: it runs on compute capability 10.0 exactly, not on
// other Blackwell parts.  Both kernels are cooperative launches and take the
// dynamic shared memory they were built for.
int device_check(int major, int minor, int cooperative, size_t smem_optin, bool rows) {
    if (major != 10 || minor != 0) return MK_ERR_INVALID;
    if (!cooperative) return MK_ERR_INVALID;
    if (smem_optin < (rows ? rows_smem_bytes() : kernel_smem_bytes())) return MK_ERR_INVALID;
    return MK_OK;
}
}  // namespace mk

extern "C" {

int mk_device_supported(int major, int minor, int cooperative_launch, size_t smem_optin_bytes, int batched) {
    return device_check(major, minor, cooperative_launch, smem_optin_bytes, batched != 0);
}

const char *mk_status_string(int status) {
    switch (status) {
    case MK_OK: return "ok";
    case MK_ERR_INVALID: return "invalid argument";
    case MK_ERR_CUDA: return "CUDA error";
    case MK_ERR_TIMEOUT: return "device wait timed out";
    case MK_ERR_OOM: return "out of memory";
    case MK_ERR_STATE: return "context unusable after a device error (call mk_reset)";
    default: return "unknown status";
    }
}

int mk_plan(const mk_config *cfg, int num_sms, mk_info *info, int32_t *task_out,
            int32_t *queue_out, int32_t *qoff_out, uint32_t *thresholds_out, int64_t *bytes_out) {
    Shape s;
    int st = shape_from_config(cfg, num_sms, s);
    if (st != MK_OK) return st;
    const bool rows = is_rows(cfg);
    PlanSizes z = rows ? rplan_sizes(s, num_sms) : plan_sizes(s, num_sms);
    std::vector<Task> tasks(z.num_tasks);
    std::vector<int32_t> queue(z.num_tasks), qoff(num_sms + 1);
    std::vector<uint32_t> thr(z.num_events);
    std::vector<int64_t> bytes(z.num_tasks);
    Plan p;
    p.tasks = tasks.data(); p.queue = queue.data(); p.qoff = qoff.data();
    p.thresholds = thr.data(); p.bytes = bytes.data();
    if (rows) rplan_build(s, num_sms, p);
    else plan_build(s, num_sms, p);
    if (info) {
        std::memset(info, 0, sizeof *info);
        info->num_sms = num_sms;
        info->num_tasks = p.num_tasks;
        info->num_events = p.num_events;
        info->num_ops = p.num_ops;
        info->attn_chunks = s.NC;
        info->attn_heads = s.HA;
        info->max_queue = p.max_queue;
        info->page_bytes = rows ? kRPageBytes : kPageBytes;
        info->num_pages = rows ? kRStages : kNumPages;
    }
    for (int i = 0; i < p.num_tasks; ++i) {
        const Task &t = tasks[i];
        if (task_out) {
            int32_t *o = task_out + 8 * i;
            o[0] = t.kind; o[1] = t.layer; o[2] = t.dep; o[3] = t.trig;
            o[4] = t.begin; o[5] = t.end; o[6] = t.sm; o[7] = t.slot;
        }
        if (bytes_out) bytes_out[i] = bytes[i];
    }
    if (queue_out) std::memcpy(queue_out, queue.data(), sizeof(int32_t) * p.num_tasks);
    if (qoff_out) std::memcpy(qoff_out, qoff.data(), sizeof(int32_t) * (num_sms + 1));
    if (thresholds_out) std::memcpy(thresholds_out, thr.data(), sizeof(uint32_t) * p.num_events);
    return MK_OK;
}

int mk_create(const mk_config *cfg, const mk_weights *w, const mk_kv *kv, mk_ctx **out) {
    if (!out) return MK_ERR_INVALID;
    *out = nullptr;
    if (!cfg || !w || !kv) return MK_ERR_INVALID;
    const bool rows = is_rows(cfg);
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return MK_ERR_CUDA;
    cudaDeviceProp prop;
    if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) return MK_ERR_CUDA;
    int st = device_check(prop.major, prop.minor, prop.cooperativeLaunch, (size_t)prop.sharedMemPerBlockOptin, rows);
    if (st != MK_OK) return st;
    // The worker/control register split is only safe with the launch
    // allocation it was computed for; refuse to launch anything else.
    if (kernel_launch_regs() != kLaunchRegs) return MK_ERR_INVALID;
    Shape s;
    st = shape_from_config(cfg, prop.multiProcessorCount, s);
    if (st != MK_OK) return st;

    // pointer checks
    if (!aligned16(w->embed) || !aligned16(w->lm_head) || !aligned16(w->final_norm)) return MK_ERR_INVALID;
    if (!w->attn_norm || !w->mlp_norm || !w->wq || !w->wk || !w->wv || !w->wo || !w->wg ||
        !w->wu || !w->wd || !kv->k || !kv->v)
        return MK_ERR_INVALID;
    for (int l = 0; l < s.L; ++l) {
        const void *ps[] = {w->attn_norm[l], w->mlp_norm[l], w->wq[l], w->wk[l], w->wv[l],
                            w->wo[l], w->wg[l], w->wu[l], w->wd[l], kv->k[l], kv->v[l]};
        for (const void *q : ps)
            if (!aligned16(q)) return MK_ERR_INVALID;
    }

    mk_ctx *c = new (std::nothrow) mk_ctx;
    if (!c) return MK_ERR_OOM;
    c->device = dev;
    c->cfg = *cfg;
    c->s = s;
    c->num_sms = prop.multiProcessorCount;
    if (rows) {
        st = rows_create(cfg, w, kv, s, c->num_sms, &c->rows);
        if (st != MK_OK) { free_ctx(c); return st; }
        PlanSizes z = rplan_sizes(s, c->num_sms);
        c->h_tasks.resize(z.num_tasks);
        c->h_queue.resize(z.num_tasks);
        c->h_qoff.resize(c->num_sms + 1);
        c->h_thresholds.resize(z.num_events);
        Plan plan;
        plan.tasks = c->h_tasks.data(); plan.queue = c->h_queue.data(); plan.qoff = c->h_qoff.data();
        plan.thresholds = c->h_thresholds.data(); plan.bytes = nullptr;
        rplan_build(s, c->num_sms, plan);
        c->num_tasks = plan.num_tasks;
        c->num_events = plan.num_events;
        c->num_ops = plan.num_ops;
        c->max_queue = plan.max_queue;
        c->num_lm_tasks = plan.num_lm_tasks;
        c->rp = rows_params(c->rows);
        c->d_err = c->rp.err;
        c->p.events = c->rp.events;
        c->p.thresholds = c->rp.thresholds;
        *out = c;
        return MK_OK;
    }

    // ---- task graph (host)
    PlanSizes z = plan_sizes(s, c->num_sms);
    c->h_tasks.resize(z.num_tasks);
    c->h_queue.resize(z.num_tasks);
    c->h_qoff.resize(c->num_sms + 1);
    c->h_thresholds.resize(z.num_events);
    Plan plan;
    plan.tasks = c->h_tasks.data(); plan.queue = c->h_queue.data(); plan.qoff = c->h_qoff.data();
    plan.thresholds = c->h_thresholds.data(); plan.bytes = nullptr;
    plan_build(s, c->num_sms, plan);
    c->num_tasks = plan.num_tasks;
    c->num_events = plan.num_events;
    c->num_ops = plan.num_ops;
    c->max_queue = plan.max_queue;
    c->num_lm_tasks = plan.num_lm_tasks;

    // ---- RoPE table: cos/sin of pos * theta^(-2i/d), computed in double
    const int half = s.d / 2;
    std::vector<float> rope((size_t)s.S * half * 2);
    for (int pos = 0; pos < s.S; ++pos)
        for (int i = 0; i < half; ++i) {
            double inv = std::pow((double)cfg->rope_theta, -2.0 * i / (double)s.d);
            double ang = (double)pos * inv;
            rope[((size_t)pos * half + i) * 2 + 0] = (float)std::cos(ang);
            rope[((size_t)pos * half + i) * 2 + 1] = (float)std::sin(ang);
        }

    std::vector<LayerW> lw(s.L);
    for (int l = 0; l < s.L; ++l) {
        lw[l].wo = (const uint16_t *)w->wo[l];
        lw[l].wd = (const uint16_t *)w->wd[l];
        lw[l].g_attn = (const uint16_t *)w->attn_norm[l]; lw[l].g_mlp = (const uint16_t *)w->mlp_norm[l];
        lw[l].kc = (uint16_t *)kv->k[l]; lw[l].vc = (uint16_t *)kv->v[l];
    }

    // ---- device memory
    Params &p = c->p;
    p.s = s;
    cudaError_t e = cudaSuccess;
    Task *d_qtasks; int32_t *d_qoff; uint32_t *d_thr, *d_ev, *d_ctrl;
    LayerW *d_layers; float2 *d_rope;
    uint64_t *d_tag, *d_toktag; float *d_aval; int32_t *d_aidx;
    const TagLayout tl = tag_layout(s);
    const size_t B = s.Bmax;
#define MK_TRY(expr) do { e = (expr); if (e != cudaSuccess) { free_ctx(c); return map_cuda(e); } } while (0)
    MK_TRY(dalloc(c, &d_qtasks, c->num_tasks));
    MK_TRY(dalloc(c, &d_qoff, c->num_sms + 1));
    MK_TRY(dalloc(c, &d_thr, c->num_events));
    MK_TRY(dalloc(c, &d_ev, c->num_events));
    MK_TRY(dalloc(c, &d_ctrl, 8));             // lm_cnt, epoch, done_cnt, abort
    MK_TRY(dalloc(c, &c->d_err, 1));
    MK_TRY(dalloc(c, &d_layers, s.L));
    MK_TRY(dalloc(c, &d_rope, (size_t)s.S * half));
    MK_TRY(dalloc(c, &d_tag, tl.layer * s.L));
    MK_TRY(dalloc(c, &d_aval, B * c->num_lm_tasks));
    MK_TRY(dalloc(c, &d_aidx, B * c->num_lm_tasks));
    MK_TRY(dalloc(c, &d_toktag, 2 * B));
    TraceRec *d_trace = nullptr;
    unsigned long long *d_stats = nullptr;
    if (cfg->flags & MK_FLAG_TRACE) {
        MK_TRY(dalloc(c, &d_trace, c->num_tasks));
        MK_TRY(dalloc(c, &d_stats, (size_t)c->num_sms * kStatSlots));
        MK_TRY(cudaMemset(d_stats, 0, sizeof(unsigned long long) * c->num_sms * kStatSlots));
    }

    // ---- q/k/v into one buffer, gate/up into tile order (see LayerW / OpTiles)
    // ---- then, for ops whose pages pass through tensor memory, every
    //      matrix into the TMEM page order (tmem_page_src), library-owned
    {
        const size_t rb = 2 * (size_t)s.H;          // bytes of one row of K = H
        const size_t tile = 16 * rb;                 // one gate/up pair tile
        // row-major source (rows x K) -> TMEM page order; returns the copy
        auto to_tmem = [&](const void *src, long long rows, int K, const uint16_t **out) -> cudaError_t {
            const long long page_rows = rows * (K / kRowK);
            uint16_t *dst;
            cudaError_t err = dalloc(c, &dst, tmem_pages_bytes(page_rows) / 2);
            if (err == cudaSuccess) err = repack_tmem_pages(dst, src, page_rows, 0);
            if (err == cudaSuccess) *out = dst;
            return err;
        };
        void *tmp_qkv = nullptr, *tmp_gu = nullptr;   // row-major staging when repacking
        if (tmem_page_op(s, OP_QKV)) MK_TRY(cudaMalloc(&tmp_qkv, (size_t)(s.QD + 2 * s.KD) * rb));
        if (tmem_page_op(s, OP_GATEUP)) MK_TRY(cudaMalloc(&tmp_gu, (size_t)2 * s.F * rb));
        for (int l = 0; l < s.L && e == cudaSuccess; ++l) {
            uint16_t *qkv = (uint16_t *)tmp_qkv, *gu = (uint16_t *)tmp_gu;
            if (!qkv) e = dalloc(c, &qkv, (size_t)(s.QD + 2 * s.KD) * s.H);
            if (e == cudaSuccess && !gu) e = dalloc(c, &gu, (size_t)2 * s.F * s.H);
            char *dq = (char *)qkv;
            if (e == cudaSuccess) e = cudaMemcpy(dq, w->wq[l], (size_t)s.QD * rb, cudaMemcpyDeviceToDevice);
            if (e == cudaSuccess)
                e = cudaMemcpy(dq + (size_t)s.QD * rb, w->wk[l], (size_t)s.KD * rb, cudaMemcpyDeviceToDevice);
            if (e == cudaSuccess)
                e = cudaMemcpy(dq + (size_t)(s.QD + s.KD) * rb, w->wv[l], (size_t)s.KD * rb,
                               cudaMemcpyDeviceToDevice);
            if (e == cudaSuccess)
                e = cudaMemcpy2D(gu, tile, w->wg[l], 8 * rb, 8 * rb, s.F / 8, cudaMemcpyDeviceToDevice);
            if (e == cudaSuccess)
                e = cudaMemcpy2D((char *)gu + 8 * rb, tile, w->wu[l], 8 * rb, 8 * rb, s.F / 8,
                                 cudaMemcpyDeviceToDevice);
            lw[l].qkv = qkv;
            lw[l].gu = gu;
            if (e == cudaSuccess && tmem_page_op(s, OP_QKV)) e = to_tmem(qkv, s.QD + 2 * s.KD, s.H, &lw[l].qkv);
            if (e == cudaSuccess && tmem_page_op(s, OP_GATEUP)) e = to_tmem(gu, 2LL * s.F, s.H, &lw[l].gu);
            if (e == cudaSuccess && tmem_page_op(s, OP_OPROJ)) e = to_tmem(w->wo[l], s.H, s.QD, &lw[l].wo);
            if (e == cudaSuccess && tmem_page_op(s, OP_DOWN)) e = to_tmem(w->wd[l], s.H, s.F, &lw[l].wd);
            // the staging buffers are reused by the next layer
            if (e == cudaSuccess && (tmp_qkv || tmp_gu)) e = cudaDeviceSynchronize();
        }
        if (e == cudaSuccess && tmem_page_op(s, OP_LMHEAD)) e = to_tmem(w->lm_head, s.V, s.H, &c->lm_tmem);
        if (e == cudaSuccess) e = cudaDeviceSynchronize();
        if (tmp_qkv) cudaFree(tmp_qkv);
        if (tmp_gu) cudaFree(tmp_gu);
        if (e != cudaSuccess) { free_ctx(c); return map_cuda(e); }
    }
    MK_TRY(cudaDeviceSynchronize());

    {
        // the device reads the tasks in queue order, each record's `sm` field
        // replaced by the task id (one load per task, no indirection)
        std::vector<Task> qt(c->num_tasks);
        for (int i = 0; i < c->num_tasks; ++i) {
            qt[i] = c->h_tasks[c->h_queue[i]];
            qt[i].sm = c->h_queue[i];
        }
        MK_TRY(cudaMemcpy(d_qtasks, qt.data(), sizeof(Task) * c->num_tasks, cudaMemcpyHostToDevice));
    }
    MK_TRY(cudaMemcpy(d_qoff, c->h_qoff.data(), sizeof(int32_t) * (c->num_sms + 1), cudaMemcpyHostToDevice));
    MK_TRY(cudaMemcpy(d_thr, c->h_thresholds.data(), sizeof(uint32_t) * c->num_events, cudaMemcpyHostToDevice));
    MK_TRY(cudaMemcpy(d_layers, lw.data(), sizeof(LayerW) * s.L, cudaMemcpyHostToDevice));
    MK_TRY(cudaMemcpy(d_rope, rope.data(), sizeof(float) * rope.size(), cudaMemcpyHostToDevice));
    MK_TRY(cudaMemset(d_ev, 0, sizeof(uint32_t) * c->num_events));
    MK_TRY(cudaMemset(d_ctrl, 0, sizeof(uint32_t) * 8));
    MK_TRY(cudaMemset(c->d_err, 0, sizeof(ErrWord)));
    MK_TRY(cudaMemset(d_tag, 0, sizeof(uint64_t) * tl.layer * s.L));   // tag 0: never a step's
    MK_TRY(cudaMemset(d_toktag, 0, sizeof(uint64_t) * 2 * B));
    if (d_trace) {
        std::vector<TraceRec> tr(c->num_tasks);
        for (int i = 0; i < c->num_tasks; ++i) {
            const Task &t = c->h_tasks[i];
            tr[i] = TraceRec{0, 0, 0, 0, 0, 0, t.sm, t.kind, t.layer, t.trig};
        }
        MK_TRY(cudaMemcpy(d_trace, tr.data(), sizeof(TraceRec) * c->num_tasks, cudaMemcpyHostToDevice));
    }
    MK_TRY(kernel_prepare());
    int per_sm = 0;
    MK_TRY(kernel_occupancy(&per_sm));
    if (per_sm < 1) { free_ctx(c); return MK_ERR_INVALID; }
#undef MK_TRY

    p.qtasks = d_qtasks; p.qoff = d_qoff; p.thresholds = d_thr; p.events = d_ev;
    p.lm_cnt = d_ctrl + 0; p.epoch = d_ctrl + 1; p.done_cnt = d_ctrl + 2; p.abort_flag = d_ctrl + 3;
    p.num_lm_tasks = c->num_lm_tasks;
    p.layers = d_layers;
    p.embed = (const uint16_t *)w->embed;
    p.lm_head = c->lm_tmem ? c->lm_tmem : (const uint16_t *)w->lm_head;
    p.g_final = (const uint16_t *)w->final_norm;
    p.rope = d_rope;
    p.tag = d_tag; p.tl = tl;
    p.amax_val = d_aval; p.amax_idx = d_aidx;
    p.tok_tag = d_toktag;
    p.n_steps = 1;
    p.n_prompt = 1;
    p.eos = -1;
    p.tokens_out = nullptr;
    p.err = c->d_err;
    p.trace = d_trace;
    p.sm_stats = d_stats;
    p.timeout_ns = cfg->timeout_ns > 0 ? (unsigned long long)cfg->timeout_ns : 2000000000ull;
    p.l2_lookahead = (cfg->flags & MK_FLAG_NO_L2_PREFETCH) ? 0
                   : cfg->l2_lookahead_kb > 0 ? 1024LL * cfg->l2_lookahead_kb : kL2Lookahead;
    p.event_wait = (cfg->flags & MK_FLAG_EVENT_WAIT) ? 1 : 0;
    p.debug_withhold = -1;
    p.poll_ns = (unsigned int)cfg->poll_ns;
    *out = c;
    return MK_OK;
}

int mk_decode_step(mk_ctx *c, const int32_t *tokens, const int32_t *positions, int batch,
                   float *logits_out, int32_t *next_tok_out, mk_stream_t stream) {
    if (!c) return MK_ERR_INVALID;
    if (c->failed) return MK_ERR_STATE;
    if (batch < 1 || batch > c->s.Bmax) return MK_ERR_INVALID;
    if (!tokens || !positions || !next_tok_out) return MK_ERR_INVALID;
    if (((uintptr_t)tokens & 3u) || ((uintptr_t)positions & 3u) || ((uintptr_t)next_tok_out & 3u) ||
        ((uintptr_t)logits_out & 3u))
        return MK_ERR_INVALID;
    if (c->rows) {
        const int st = rows_step(c->rows, tokens, positions, batch, logits_out, next_tok_out, (cudaStream_t)stream);
        if (st == MK_OK) c->steps++;
        return st;
    }
    Params p = c->p;
    p.tokens = tokens;
    p.positions = positions;
    p.batch = batch;
    p.logits = logits_out;
    p.next_tok = next_tok_out;
    cudaError_t e = kernel_launch(p, c->num_sms, (cudaStream_t)stream);
    if (e != cudaSuccess) return MK_ERR_CUDA;
    c->steps++;
    return MK_OK;
}

int mk_generate(mk_ctx *c, const int32_t *tokens, int n_prompt, const int32_t *positions, int batch,
                int n_steps, int32_t eos, int32_t *tokens_out, int32_t *next_tok_out, mk_stream_t stream) {
    if (!c) return MK_ERR_INVALID;
    if (c->failed) return MK_ERR_STATE;
    if (c->rows) return MK_ERR_INVALID;   // one launch per generation: batch-1 contexts only
    if (batch < 1 || batch > c->s.Bmax || n_steps < 1 || n_steps > c->s.S) return MK_ERR_INVALID;
    if (n_prompt < 1 || n_prompt > n_steps) return MK_ERR_INVALID;
    if (!tokens || !positions || !tokens_out || !next_tok_out) return MK_ERR_INVALID;
    if (((uintptr_t)tokens & 3u) || ((uintptr_t)positions & 3u) || ((uintptr_t)tokens_out & 3u) ||
        ((uintptr_t)next_tok_out & 3u))
        return MK_ERR_INVALID;
    Params p = c->p;
    p.tokens = tokens;
    p.positions = positions;
    p.batch = batch;
    p.logits = nullptr;
    p.next_tok = next_tok_out;
    p.n_steps = n_steps;
    p.n_prompt = n_prompt;
    p.eos = eos < 0 ? -1 : eos;
    p.tokens_out = tokens_out;
    cudaError_t e = kernel_launch(p, c->num_sms, (cudaStream_t)stream);
    if (e != cudaSuccess) return MK_ERR_CUDA;
    c->steps += n_steps;
    return MK_OK;
}

int mk_prefill(mk_ctx *c, const int32_t *tokens, int n_tokens, int slot, int start_pos, float *logits_out,
               int32_t *next_tok_out, mk_stream_t stream) {
    if (!c) return MK_ERR_INVALID;
    if (c->failed) return MK_ERR_STATE;
    if (!c->rows) return MK_ERR_INVALID;
    if (!tokens || !next_tok_out || n_tokens < 1 || slot < 0 || slot >= c->s.Bmax || start_pos < 0 ||
        (long long)start_pos + n_tokens > c->s.S)
        return MK_ERR_INVALID;
    if (((uintptr_t)tokens & 3u) || ((uintptr_t)next_tok_out & 3u) || ((uintptr_t)logits_out & 3u))
        return MK_ERR_INVALID;
    const int st = rows_prefill(c->rows, tokens, n_tokens, slot, start_pos, logits_out, next_tok_out,
                                (cudaStream_t)stream);
    if (st == MK_OK) c->steps += (n_tokens + kRows - 1) / kRows;
    return st;
}

int mk_sync(mk_ctx *c, mk_stream_t stream) {
    if (!c) return MK_ERR_INVALID;
    if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return MK_ERR_CUDA;
    ErrWord ew;
    if (cudaMemcpy(&ew, c->d_err, sizeof ew, cudaMemcpyDeviceToHost) != cudaSuccess) return MK_ERR_CUDA;
    if (ew.code != 0) {
        c->failed = true;
        return (int)ew.code;
    }
    return MK_OK;
}

int mk_reset(mk_ctx *c) {
    if (!c) return MK_ERR_INVALID;
    if (cudaDeviceSynchronize() != cudaSuccess) return MK_ERR_CUDA;
    if (c->rows) {
        if (rows_reset(c->rows) != MK_OK || cudaDeviceSynchronize() != cudaSuccess) return MK_ERR_CUDA;
        c->steps = 0;
        c->failed = false;
        return MK_OK;
    }
    const Params &p = c->p;
    if (cudaMemset(p.events, 0, sizeof(uint32_t) * c->num_events) != cudaSuccess ||
        cudaMemset(p.lm_cnt, 0, sizeof(uint32_t) * 4) != cudaSuccess ||
        cudaMemset(c->d_err, 0, sizeof(ErrWord)) != cudaSuccess ||
        // the epoch restarts at 0: tags written before the reset must not
        // pass for the next steps'
        cudaMemset(p.tag, 0, sizeof(uint64_t) * p.tl.layer * c->s.L) != cudaSuccess ||
        cudaMemset(p.tok_tag, 0, sizeof(uint64_t) * 2 * c->s.Bmax) != cudaSuccess ||
        cudaMemcpy(const_cast<uint32_t *>(p.thresholds), c->h_thresholds.data(), sizeof(uint32_t) * c->num_events,
                   cudaMemcpyHostToDevice) != cudaSuccess)
        return MK_ERR_CUDA;
    if (cudaDeviceSynchronize() != cudaSuccess) return MK_ERR_CUDA;
    c->steps = 0;
    c->failed = false;
    c->p.debug_withhold = -1;
    return MK_OK;
}

int mk_destroy(mk_ctx *c) {
    if (!c) return MK_OK;
    cudaDeviceSynchronize();
    free_ctx(c);
    return MK_OK;
}

int mk_get_info(mk_ctx *c, mk_info *out) {
    if (!c || !out) return MK_ERR_INVALID;
    std::memset(out, 0, sizeof *out);
    out->num_sms = c->num_sms;
    out->num_tasks = c->num_tasks;
    out->num_events = c->num_events;
    out->num_ops = c->num_ops;
    out->attn_chunks = c->s.NC;
    out->attn_heads = c->s.HA;
    out->max_queue = c->max_queue;
    out->page_bytes = c->rows ? kRPageBytes : kPageBytes;
    out->num_pages = c->rows ? kRStages : kNumPages;
    out->steps_run = c->steps;
    ErrWord ew;
    if (cudaMemcpy(&ew, c->d_err, sizeof ew, cudaMemcpyDeviceToHost) != cudaSuccess) return MK_ERR_CUDA;
    out->err_code = ew.code;
    out->err_info = ew.where << 24 | (ew.info & 0xffffffu);
    out->err_task = ew.code ? ew.task : 0xffffffffu;
    return MK_OK;
}

int mk_get_event_counts(mk_ctx *c, uint32_t *counts_out, uint32_t *thresholds_out, int n) {
    if (!c || n < 0 || n > c->num_events) return MK_ERR_INVALID;
    if (counts_out &&
        cudaMemcpy(counts_out, c->p.events, sizeof(uint32_t) * n, cudaMemcpyDeviceToHost) != cudaSuccess)
        return MK_ERR_CUDA;
    if (thresholds_out &&
        cudaMemcpy(thresholds_out, c->p.thresholds, sizeof(uint32_t) * n, cudaMemcpyDeviceToHost) != cudaSuccess)
        return MK_ERR_CUDA;
    return MK_OK;
}

int mk_read_buffer(mk_ctx *c, int which, float *host_out, size_t count) {
    if (!c || !host_out) return MK_ERR_INVALID;
    const Shape &s = c->s;
    if (c->rows) {
        // the residual stream after the last layer, rows [kRows][hidden] fp32
        if (which != MK_BUF_HIDDEN || count > (size_t)kRows * s.H) return MK_ERR_INVALID;
        RLayerBuf last;
        if (cudaMemcpy(&last, c->rp.buf + (s.L - 1), sizeof last, cudaMemcpyDeviceToHost) != cudaSuccess ||
            (count && cudaMemcpy(host_out, last.xb, sizeof(float) * count, cudaMemcpyDeviceToHost) != cudaSuccess))
            return MK_ERR_CUDA;
        return MK_OK;
    }
    const TagLayout &tl = c->p.tl;
    const size_t last = (size_t)(s.L - 1) * tl.layer;
    size_t off = 0, n = 0;
    switch (which) {
    case MK_BUF_HIDDEN: off = tl.xb; n = (size_t)s.Bmax * s.H; break;
    case MK_BUF_Q: off = tl.q; n = (size_t)s.Bmax * s.QD; break;
    case MK_BUF_ATTN: off = tl.attn; n = (size_t)s.Bmax * s.QD; break;
    case MK_BUF_ACT: off = tl.act; n = (size_t)s.Bmax * s.F; break;
    default: return MK_ERR_INVALID;
    }
    if (count > n) return MK_ERR_INVALID;
    std::vector<uint64_t> words(count);
    if (count && cudaMemcpy(words.data(), c->p.tag + last + off, sizeof(uint64_t) * count,
                            cudaMemcpyDeviceToHost) != cudaSuccess)
        return MK_ERR_CUDA;
    for (size_t i = 0; i < count; ++i) {
        const uint32_t bits = (uint32_t)words[i];
        std::memcpy(host_out + i, &bits, sizeof bits);
    }
    return MK_OK;
}

int mk_get_trace(mk_ctx *c, mk_trace_rec *host_out, int n) {
    if (!c || !host_out || n < 0 || n > c->num_tasks) return MK_ERR_INVALID;
    if (c->rows) {
        if (!c->rp.trace) return MK_ERR_INVALID;
        if (cudaMemcpy(host_out, c->rp.trace, sizeof(TraceRec) * n, cudaMemcpyDeviceToHost) != cudaSuccess)
            return MK_ERR_CUDA;
        return MK_OK;
    }
    if (!c->p.trace) return MK_ERR_INVALID;
    static_assert(sizeof(mk_trace_rec) == sizeof(TraceRec), "trace record layout");
    if (cudaMemcpy(host_out, c->p.trace, sizeof(TraceRec) * n, cudaMemcpyDeviceToHost) != cudaSuccess)
        return MK_ERR_CUDA;
    return MK_OK;
}

int mk_get_sm_stats(mk_ctx *c, uint64_t *host_out, int n) {
    if (!c || !host_out || n < 0 || n > c->num_sms * kStatSlots) return MK_ERR_INVALID;
    if (c->rows) {
        if (!c->rp.sm_stats) return MK_ERR_INVALID;
        if (cudaMemcpy(host_out, c->rp.sm_stats, sizeof(uint64_t) * n, cudaMemcpyDeviceToHost) != cudaSuccess)
            return MK_ERR_CUDA;
        return MK_OK;
    }
    if (!c->p.sm_stats) return MK_ERR_INVALID;
    if (cudaMemcpy(host_out, c->p.sm_stats, sizeof(uint64_t) * n, cudaMemcpyDeviceToHost) != cudaSuccess)
        return MK_ERR_CUDA;
    return MK_OK;
}

int mk_get_graph(mk_ctx *c, int32_t *task_out, int32_t *queue_out, int32_t *qoff_out) {
    if (!c) return MK_ERR_INVALID;
    for (int i = 0; i < c->num_tasks && task_out; ++i) {
        const Task &t = c->h_tasks[i];
        int32_t *o = task_out + 8 * i;
        o[0] = t.kind; o[1] = t.layer; o[2] = t.dep; o[3] = t.trig;
        o[4] = t.begin; o[5] = t.end; o[6] = t.sm; o[7] = t.slot;
    }
    if (queue_out) std::memcpy(queue_out, c->h_queue.data(), sizeof(int32_t) * c->num_tasks);
    if (qoff_out) std::memcpy(qoff_out, c->h_qoff.data(), sizeof(int32_t) * (c->num_sms + 1));
    return MK_OK;
}

int mk_debug_set_threshold(mk_ctx *c, int event, uint32_t threshold) {
    if (!c || event < 0 || event >= c->num_events) return MK_ERR_INVALID;
    if (cudaDeviceSynchronize() != cudaSuccess) return MK_ERR_CUDA;
    if (cudaMemcpy(const_cast<uint32_t *>(c->p.thresholds) + event, &threshold, sizeof threshold, cudaMemcpyHostToDevice) != cudaSuccess)
        return MK_ERR_CUDA;
    return MK_OK;
}

int mk_debug_withhold_event(mk_ctx *c, int event) {
    if (!c || event < -1 || event >= c->num_events || c->rows) return MK_ERR_INVALID;
    c->p.debug_withhold = event;
    return MK_OK;
}

}  // extern "C"
