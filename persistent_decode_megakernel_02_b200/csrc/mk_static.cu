// mk_static.cu -- mk_decode_step_static: one decode step that allocates
// nothing.
//
// Some callers cannot allocate device memory at the point where they want
// to decode: code running inside a memory arena that owns all of the
// device's memory, allocation-free real-time serving loops, or hosts whose
// allocator must not be entered on the decode path.  This entry point takes
// everything per call (shape, weights in the kernel's packed layout, KV
// cache, inputs, outputs) and keeps all of its own scratch -- task tables,
// RoPE table, activations, attention partials, event counters, error word --
// in one file-scope device array of fixed size, MK_STATIC_SCRATCH_BYTES,
// that every GPU which loads the library holds until the process exits.
// It calls no cudaMalloc, cudaFree or allocating library routine; host
// staging of the tables uses static host storage.
//
// Every call shares that array and leaves the last call's contents in it;
// calls on the same device that overlap on the GPU (different streams, or
// several host threads) race on it.  Each device has its own copy of the
// array; the host-side staging is one static buffer guarded by a mutex, so
// host threads driving different devices do not mix their tables.  The first
// call on a device looks up the array's device address with
// cudaGetSymbolAddress (with that device current) and sets the kernel's
// shared-memory attribute; a call whose planned shape (the config's sizes
// and the attention items its flags and the SM count choose), weights or KV
// cache differ from the previous call's on that device uploads new tables
// and synchronises the stream.  Make such calls outside stream capture.  The
// uploaded tables carry a key the kernel checks against the key its launch
// was set up with: a launch set up for tables that have been replaced since
// (a replay of an earlier launch) runs nothing and reports MK_ERR_INVALID.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "../../include/mk.h"
#include "mk_internal.h"

namespace mk {
size_t kernel_smem_bytes();
int device_check(int major, int minor, int cooperative, size_t smem_optin, bool rows);
int kernel_launch_regs();
cudaError_t kernel_prepare();
cudaError_t kernel_launch(const Params &p, int grid, cudaStream_t stream);
}  // namespace mk

using namespace mk;

// The scratch of mk_decode_step_static.  In host code this name is only a
// stand-in for the device array: never pass it to a kernel, pass the address
// from cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char g_static_scratch[MK_STATIC_SCRATCH_BYTES];

namespace {

constexpr int kMaxDevices = 64;

struct DeviceSetup {
    bool ready = false;
    unsigned char *scratch = nullptr;   // device address of g_static_scratch
    int num_sms = 0;
};
DeviceSetup g_dev[kMaxDevices];

// Host staging of the tables (static storage; no allocation), shared by all
// devices and guarded by g_host_mutex for the whole host section of a call.
alignas(256) unsigned char g_host[MK_STATIC_SCRATCH_BYTES];
std::mutex g_host_mutex;

// What the tables currently in a device's scratch were built from: a hash of
// the shape (task graph, RoPE table) and a hash of the layer pointer table.
struct Signature {
    bool valid = false;
    uint64_t shape_key = 0;
    uint64_t layer_key = 0;
};
Signature g_sig[kMaxDevices];

uint64_t fnv1a(uint64_t h, const void *data, size_t n) {
    const unsigned char *b = static_cast<const unsigned char *>(data);
    for (size_t i = 0; i < n; ++i) { h ^= b[i]; h *= 1099511628211ull; }
    return h;
}

// Keyed on the planned shape, not on the config: everything that decides the
// task graph and the scratch layout (the attention items' heads and chunks
// depend on the flags and the SM count as well as on the sizes).
uint64_t shape_key(const Shape &s, int num_sms) {
    const long long f[] = {s.L, s.H, s.nq, s.nkv, s.d, s.F, s.V, s.S, s.Bmax, s.NC, s.HA, s.tmem, num_sms};
    uint64_t h = fnv1a(1469598103934665603ull, f, sizeof f);
    const float g[] = {s.theta, s.eps};
    return fnv1a(h, g, sizeof g);
}

struct Layout {
    size_t key,      // uint64: key of the tables below (checked by the kernel)
        tasks, queue, qtasks, qoff, thr, events, ctrl, err, tag, toktag, layers, rope;
    size_t aval, aidx, end;
};

size_t align_up(size_t v) { return (v + 255) & ~(size_t)255; }

bool shape_ok(const mk_config *c, int num_sms, Shape &s) {
    if (!c) return false;
    if (c->layers < 1 || c->hidden < 8 || c->n_q_heads < 1 || c->n_kv_heads < 1 ||
        c->head_dim < 1 || c->ffn < 8 || c->vocab < 1 || c->max_seq < 1 || c->max_batch < 1)
        return false;
    // the batch-1 step on CUDA cores only (the batched step is not offered here)
    if (c->max_batch > kMaxBatch || (c->flags & MK_FLAG_ROWS) || c->n_q_heads % c->n_kv_heads != 0) return false;
    const int G = c->n_q_heads / c->n_kv_heads;
    if (G != 1 && G != 2 && G != 4 && G != 8) return false;
    if (c->head_dim != 64 && c->head_dim != 128) return false;
    const long long QD = (long long)c->n_q_heads * c->head_dim;
    if (c->hidden % 8 || c->ffn % 8 || QD % 8) return false;
    if (c->hidden > kMaxHidden || c->ffn > kMaxK || QD > kMaxK) return false;
    if (!(c->rms_eps > 0.f) || !(c->rope_theta > 1.f)) return false;
    if (c->attn_chunks < 0 || c->timeout_ns < 0 || c->l2_lookahead_kb < 0) return false;
    if (c->poll_ns < 0 || c->poll_ns > 1000000) return false;
    if (c->flags & MK_FLAG_TRACE) return false;   // no trace buffer in the static scratch
    s.L = c->layers; s.H = c->hidden; s.nq = c->n_q_heads; s.nkv = c->n_kv_heads;
    s.d = c->head_dim; s.F = c->ffn; s.V = c->vocab; s.S = c->max_seq; s.Bmax = c->max_batch;
    s.G = G; s.QD = (int)QD; s.KD = c->n_kv_heads * c->head_dim;
    s.theta = c->rope_theta; s.eps = c->rms_eps;
    s.tmem = 0;   // weights come in the row-major packed layout: pages stay in shared memory
    return plan_attention(s, num_sms, c->flags, c->attn_chunks);
}

Layout layout_for(const Shape &s, const PlanSizes &z, int num_sms, int num_lm_tasks) {
    Layout l;
    size_t o = 0;
    auto take = [&](size_t bytes) { size_t at = o; o = align_up(o + bytes); return at; };
    const size_t B = s.Bmax;
    l.key = take(sizeof(uint64_t));
    l.tasks = take(sizeof(Task) * z.num_tasks);
    l.queue = take(sizeof(int32_t) * z.num_tasks);
    l.qtasks = take(sizeof(Task) * z.num_tasks);
    l.qoff = take(sizeof(int32_t) * (num_sms + 1));
    l.thr = take(sizeof(uint32_t) * z.num_events);
    l.events = take(sizeof(uint32_t) * z.num_events);
    l.ctrl = take(sizeof(uint32_t) * 8);
    l.err = take(sizeof(ErrWord));
    l.tag = take(sizeof(uint64_t) * tag_layout(s).layer * s.L);
    l.toktag = take(sizeof(uint64_t) * 2 * B);
    l.layers = take(sizeof(LayerW) * s.L);
    l.rope = take(sizeof(float2) * (size_t)s.S * (s.d / 2));
    l.aval = take(sizeof(float) * B * num_lm_tasks);
    l.aidx = take(sizeof(int32_t) * B * num_lm_tasks);
    l.end = o;
    return l;
}

bool aligned16(const void *p) { return p && ((uintptr_t)p & 15u) == 0; }

}  // namespace

extern "C" int mk_decode_step_static(const mk_config *cfg, const mk_packed_weights *w,
                                     const mk_kv *kv, const int32_t *tokens,
                                     const int32_t *positions, int batch, float *logits_out,
                                     int32_t *next_tok_out, int32_t *status_out,
                                     mk_stream_t stream) {
    if (!cfg || !w || !kv || !tokens || !positions || !next_tok_out) return MK_ERR_INVALID;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return MK_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return MK_ERR_INVALID;
    std::lock_guard<std::mutex> lock(g_host_mutex);
    DeviceSetup &ds = g_dev[dev];
    if (!ds.ready) {
        // once per device, with that device current
        void *ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_static_scratch) != cudaSuccess || !ptr) return MK_ERR_CUDA;
        cudaDeviceProp prop;
        if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) return MK_ERR_CUDA;
        const int st = device_check(prop.major, prop.minor, prop.cooperativeLaunch,
                                    (size_t)prop.sharedMemPerBlockOptin, false);
        if (st != MK_OK) return st;
        if (kernel_launch_regs() != kLaunchRegs) return MK_ERR_INVALID;
        if (kernel_prepare() != cudaSuccess) return MK_ERR_CUDA;
        ds.scratch = static_cast<unsigned char *>(ptr);
        ds.num_sms = prop.multiProcessorCount;
        ds.ready = true;
    }

    Shape s;
    if (!shape_ok(cfg, ds.num_sms, s)) return MK_ERR_INVALID;
    if (batch < 1 || batch > s.Bmax) return MK_ERR_INVALID;
    if (((uintptr_t)tokens & 3u) || ((uintptr_t)positions & 3u) || ((uintptr_t)next_tok_out & 3u) ||
        ((uintptr_t)logits_out & 3u) || ((uintptr_t)status_out & 3u))
        return MK_ERR_INVALID;
    if (!aligned16(w->embed) || !aligned16(w->lm_head) || !aligned16(w->final_norm)) return MK_ERR_INVALID;
    if (!w->attn_norm || !w->mlp_norm || !w->qkv || !w->wo || !w->gu || !w->wd || !kv->k || !kv->v)
        return MK_ERR_INVALID;
    for (int l = 0; l < s.L; ++l) {
        const void *ps[] = {w->attn_norm[l], w->mlp_norm[l], w->qkv[l], w->wo[l], w->gu[l],
                            w->wd[l], kv->k[l], kv->v[l]};
        for (const void *q : ps)
            if (!aligned16(q)) return MK_ERR_INVALID;
    }

    const PlanSizes z = plan_sizes(s, ds.num_sms);
    const int num_lm = (s.V + 7) / 8 < ds.num_sms ? (s.V + 7) / 8 : ds.num_sms;
    const Layout lay = layout_for(s, z, ds.num_sms, num_lm);
    if (lay.end > MK_STATIC_SCRATCH_BYTES) return MK_ERR_INVALID;   // shape too large for the fixed scratch

    unsigned char *d = ds.scratch;
    cudaStream_t st = (cudaStream_t)stream;
    Signature &sig = g_sig[dev];
    // the layer pointer table, built every call (small) and uploaded when it
    // differs from the one in the scratch
    LayerW *lw = reinterpret_cast<LayerW *>(g_host + lay.layers);
    for (int l = 0; l < s.L; ++l) {
        lw[l].qkv = (const uint16_t *)w->qkv[l];
        lw[l].gu = (const uint16_t *)w->gu[l];
        lw[l].wo = (const uint16_t *)w->wo[l];
        lw[l].wd = (const uint16_t *)w->wd[l];
        lw[l].g_attn = (const uint16_t *)w->attn_norm[l];
        lw[l].g_mlp = (const uint16_t *)w->mlp_norm[l];
        lw[l].kc = (uint16_t *)kv->k[l];
        lw[l].vc = (uint16_t *)kv->v[l];
    }
    const uint64_t skey = shape_key(s, ds.num_sms);
    const uint64_t lkey = fnv1a(skey, lw, sizeof(LayerW) * s.L);
    if (!sig.valid || sig.shape_key != skey) {
        // task graph and RoPE table for this shape, in static host storage
        sig.valid = false;
        Plan plan;
        plan.tasks = reinterpret_cast<Task *>(g_host + lay.tasks);
        plan.queue = reinterpret_cast<int32_t *>(g_host + lay.queue);
        plan.qoff = reinterpret_cast<int32_t *>(g_host + lay.qoff);
        plan.thresholds = reinterpret_cast<uint32_t *>(g_host + lay.thr);
        plan.bytes = nullptr;
        plan_build(s, ds.num_sms, plan);
        // the device reads the tasks in queue order, `sm` holding the task id
        Task *qt = reinterpret_cast<Task *>(g_host + lay.qtasks);
        for (int i = 0; i < plan.num_tasks; ++i) {
            qt[i] = plan.tasks[plan.queue[i]];
            qt[i].sm = plan.queue[i];
        }
        float2 *rope = reinterpret_cast<float2 *>(g_host + lay.rope);
        const int half = s.d / 2;
        for (int pos = 0; pos < s.S; ++pos)
            for (int i = 0; i < half; ++i) {
                const double ang = (double)pos * std::pow((double)cfg->rope_theta, -2.0 * i / (double)s.d);
                rope[(size_t)pos * half + i] = make_float2((float)std::cos(ang), (float)std::sin(ang));
            }
        if (cudaMemcpyAsync(d + lay.tasks, g_host + lay.tasks, lay.events - lay.tasks,
                            cudaMemcpyHostToDevice, st) != cudaSuccess ||
            cudaMemcpyAsync(d + lay.rope, g_host + lay.rope, lay.aval - lay.rope,
                            cudaMemcpyHostToDevice, st) != cudaSuccess ||
            cudaStreamSynchronize(st) != cudaSuccess)
            return MK_ERR_CUDA;
        sig.shape_key = skey;
        sig.layer_key = 0;
        sig.valid = true;
    }
    if (sig.layer_key != lkey) {
        // the layer table, then the key that names the whole table set
        uint64_t *hkey = reinterpret_cast<uint64_t *>(g_host + lay.key);
        *hkey = lkey;
        if (cudaMemcpyAsync(d + lay.layers, lw, sizeof(LayerW) * s.L, cudaMemcpyHostToDevice, st) != cudaSuccess ||
            cudaMemcpyAsync(d + lay.key, hkey, sizeof(uint64_t), cudaMemcpyHostToDevice, st) != cudaSuccess ||
            cudaStreamSynchronize(st) != cudaSuccess) {
            sig.valid = false;
            return MK_ERR_CUDA;
        }
        sig.layer_key = lkey;
    }
    // what must start at zero: event counters, the epoch / done /
    // abort words, the error word and the tagged activations (the epoch
    // restarts at 0 every call, so tags left by the previous call must not
    // pass for this one's; everything else is written before it is read
    // within the step)
    if (cudaMemsetAsync(d + lay.events, 0, lay.layers - lay.events, st) != cudaSuccess) return MK_ERR_CUDA;

    Params p{};
    p.s = s;
    p.qtasks = reinterpret_cast<const Task *>(d + lay.qtasks);
    p.qoff = reinterpret_cast<const int32_t *>(d + lay.qoff);
    p.thresholds = reinterpret_cast<const uint32_t *>(d + lay.thr);
    p.events = reinterpret_cast<uint32_t *>(d + lay.events);
    uint32_t *ctrl = reinterpret_cast<uint32_t *>(d + lay.ctrl);
    p.lm_cnt = ctrl + 0;
    p.epoch = ctrl + 1;
    p.done_cnt = ctrl + 2;
    p.abort_flag = ctrl + 3;
    p.num_lm_tasks = num_lm;
    p.layers = reinterpret_cast<const LayerW *>(d + lay.layers);
    p.embed = (const uint16_t *)w->embed;
    p.lm_head = (const uint16_t *)w->lm_head;
    p.g_final = (const uint16_t *)w->final_norm;
    p.rope = reinterpret_cast<const float2 *>(d + lay.rope);
    p.tokens = tokens;
    p.positions = positions;
    p.batch = batch;
    p.logits = logits_out;
    p.next_tok = next_tok_out;
    p.tag = reinterpret_cast<uint64_t *>(d + lay.tag);
    p.tok_tag = reinterpret_cast<uint64_t *>(d + lay.toktag);
    p.n_steps = 1;
    p.n_prompt = 1;
    p.eos = -1;
    p.tokens_out = nullptr;
    p.tl = tag_layout(s);
    p.amax_val = reinterpret_cast<float *>(d + lay.aval);
    p.amax_idx = reinterpret_cast<int32_t *>(d + lay.aidx);
    p.err = reinterpret_cast<ErrWord *>(d + lay.err);
    p.trace = nullptr;
    p.sm_stats = nullptr;
    p.timeout_ns = cfg->timeout_ns > 0 ? (unsigned long long)cfg->timeout_ns : 2000000000ull;
    p.l2_lookahead = (cfg->flags & MK_FLAG_NO_L2_PREFETCH) ? 0
                   : cfg->l2_lookahead_kb > 0 ? 1024LL * cfg->l2_lookahead_kb : kL2Lookahead;
    p.event_wait = (cfg->flags & MK_FLAG_EVENT_WAIT) ? 1 : 0;
    p.debug_withhold = -1;
    p.poll_ns = (unsigned int)cfg->poll_ns;
    p.table_key = reinterpret_cast<const uint64_t *>(d + lay.key);
    p.expect_key = lkey;
    if (kernel_launch(p, ds.num_sms, st) != cudaSuccess) return MK_ERR_CUDA;
    if (status_out &&
        cudaMemcpyAsync(status_out, d + lay.err, sizeof(int32_t), cudaMemcpyDeviceToDevice, st) != cudaSuccess)
        return MK_ERR_CUDA;
    return MK_OK;
}
