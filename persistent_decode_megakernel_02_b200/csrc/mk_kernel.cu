// mk_kernel.cu -- the persistent decode-step kernel for B200 (sm_100a).
//
// One CTA per SM, launched cooperatively so that every CTA is resident.
// Each CTA owns a static queue of tasks (built on the host, see
// mk_graph.cpp) and runs these roles in separate warps:
//
//  * loader warp (one thread): walks the queue ahead of the workers and,
//    for every page of every upcoming task, waits for a free page of the
//    shared-memory ring and issues 1-D bulk async copies (cp.async.bulk) of
//    the task's weight rows (or KV-cache prefix) into it, completing on the
//    page's mbarrier.  Weights do not depend on activations, so this runs
//    ahead of the task dependencies (the Hazy page's "paged shared memory,
//    next stage preloads its weights early").
//  * worker warps (8): run the task bodies on CUDA cores.  A task's input
//    activations are "tagged" words (value + step tag in one 64-bit store,
//    see TagLayout); the workers poll the words they read until every tag is
//    this step's, which is the task's dependency wait.
//  * signaler warp (one thread): bumps each finished task's triggering event
//    counter in global memory with a release add (MPK's event/threshold
//    model, "显著提升小LLM的性能..." page, Figure 3 text), off the workers'
//    path.
//  * scheduler warp (one thread, only with MK_FLAG_EVENT_WAIT): spins on each
//    queued task's dependent event counter until it reaches threshold *
//    epoch and only then lets the workers start the task -- the pages' own
//    gating, kept as an option; the tagged words make it redundant.
//
// Task bodies (the fused instruction list of the Hazy megakernel page and
// the per-layer *_layer calls of the MPK walkthrough, section 3.3.1):
//   QKV    RMSNorm -> q/k/v GEMV rows -> q and k to scratch, v appended to
//          the bf16 cache at the token's position
//   ATTN   RoPE of q and of the new k (the group's first q head appends the
//          rotated k to the cache) -> GQA decode attention of one q head over
//          one chunk of positions (split-K partial softmax); chunk 0's task
//          merges the partials when there are several chunks
//   OPROJ  O-projection GEMV rows + residual
//   GATEUP RMSNorm -> gate and up GEMV rows -> SiLU(gate) * up
//   DOWN   down-projection GEMV rows + residual
//   LMHEAD final RMSNorm -> LM-head GEMV rows -> per-task argmax; the last
//          task to finish reduces the partial argmaxes to the next token
//
// Every wait is bounded by timeout_ns (globaltimer); on expiry the CTA
// records MK_ERR_TIMEOUT in the error word, raises the abort flag that all
// other waits poll, lets its in-flight bulk copies land, and returns.
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <math.h>
#include <stddef.h>
#include <stdint.h>

#include "mk_internal.h"
#include "mk_ptx.cuh"

namespace mk {

// status codes (same values as the public header's enum)
constexpr uint32_t kErrInvalid = 1, kErrTimeout = 3;
enum Where : uint32_t { W_DEP = 1, W_READY = 2, W_FULL = 3, W_EMPTY = 4, W_WBAR = 5,
                        W_INPUT = 6, W_DRAIN = 7, W_TAG = 8 };

// The same value into every copy of a replicated tagged vector.
__device__ __forceinline__ void st_tag_rep(uint64_t *p, size_t stride, float v, uint32_t ep) {
#pragma unroll 1
    for (int r = 0; r < kReplicas; ++r) st_tag(p + r * stride, v, ep);
}

// ---------------------------------------------------------------------------
// shared memory
// ---------------------------------------------------------------------------
constexpr int kAttnCombine = kMaxHeadDim + 8;   // per-warp slot of the attention combine
static_assert(kWorkerWarps * kAttnCombine + 16 * 12 <= kStageFloats, "combine fits the staging area");
constexpr int kSigRing = 64;        // pending task completions the signaler can hold

// A task record as the loader publishes it to the workers: the task and the
// RMSNorm gain its input takes (null if none).
struct TaskRec {
    Task t;
    const uint16_t *gain;
};
constexpr int kTaskRing = 8;        // task records the loader may publish ahead

struct __align__(16) SmemCtl {
    // Every page that lands in a slot completes exactly one of two barriers:
    // full (a page the workers read from shared memory) or tland (a page the
    // stasher copies on into tensor memory), so that each consumer waits on
    // a barrier whose every phase is one of its own pages -- a consumer that
    // skips the other kind of page can never find its barrier two phases
    // behind (mbarrier parity waits cannot tell those apart).
    uint64_t full[kNumPages];
    uint64_t tland[kNumPages];
    uint64_t empty[kNumPages];
    uint64_t cpdone[kNumPages];   // a page copied on into tensor memory has been read
    uint64_t tfull[kTmemSlots];   // a TMEM slot holds a page
    uint64_t tempty[kTmemSlots];  // the workers are done with a TMEM slot
    uint32_t tmem_base;           // tensor-memory address of the allocation
    uint64_t wbar;              // worker barrier, one arrival per worker warp
    uint32_t ready_upto;        // tasks of this queue activated by the scheduler
    uint32_t abort;             // this CTA is bailing out
    uint32_t ep;                // epoch of this launch (steps completed + 1)
    uint32_t last_flag;         // broadcast of "this task arrived last"
    uint32_t loader_done;       // the loader has issued its last page
    uint32_t tq_pub;            // task records published by the loader
    uint32_t tq_reads;          // worker warps done reading a record (8 per task)
    int32_t tok[kMaxBatch];     // the workers' current step's tokens (first step: read once)
    int32_t pos[kMaxBatch];     // the first step's positions (step s runs at pos + s)
    int32_t wstep;              // the workers' current step
    uint32_t stop;              // generation ended early: every role leaves its loop
    TaskRec tq[kTaskRing];      // records of the next tasks of this queue
    uint32_t sig_post;          // task completions posted by the workers
    uint32_t sig_done;          // completions the signaler has published
    uint32_t sig_ev[kSigRing];  // event of each posted completion (ring)
    float red[2][kWorkerWarps][16];
    float scal[kWorkerWarps];
    float att_m[kWorkerWarps][1];   // LM-head argmax: per-warp best value
    float att_l[kWorkerWarps][1];   //   and its index (as float bits)
    // staging area: a row-per-warp GEMV task's input vector (read as
    // float4); an attention task's per-warp running outputs (kWorkerWarps x
    // kAttnCombine), later its merge inputs
    __align__(16) float stage[kStageFloats];
    unsigned long long wstat[16];   // trace-mode time accounting of worker thread 0
};
constexpr size_t kSmemBytes = (size_t)kNumPages * kPageBytes + sizeof(SmemCtl);
static_assert(offsetof(SmemCtl, stage) % 16 == 0, "float4 access to the staging area");
static_assert((kNumPages * kPageBytes) % 16 == 0, "SmemCtl placement");
static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");

// ---------------------------------------------------------------------------
// bounded waiting
// ---------------------------------------------------------------------------
struct Spin {
    unsigned long long t0 = 0;
    uint32_t n = 0;
};

// Record the first device error (later ones are dropped) and raise both
// abort flags.
__device__ void raise_error(const Params &p, SmemCtl *ctl, uint32_t code, uint32_t where,
                            uint32_t task, uint32_t info) {
    if (atomicCAS(&p.err->code, 0u, code) == 0u) {
        p.err->task = task;
        p.err->where = where;
        p.err->info = info;
    }
    *(volatile uint32_t *)&ctl->abort = 1;
    atomicExch(p.abort_flag, 1u);
    __threadfence();
}

// Returns false when the wait must be abandoned: this CTA or another one
// aborted, or the wait exceeded the time budget (then the error is raised).
__device__ __forceinline__ bool spin_ok(Spin &s, const Params &p, SmemCtl *ctl, uint32_t where,
                                        uint32_t task, uint32_t info) {
    if ((++s.n & 127u) != 0u) return true;
    if (*(volatile uint32_t *)&ctl->abort) return false;
    if (*(volatile uint32_t *)&ctl->stop) return false;
    if (ld_volatile_u32(p.abort_flag)) {
        *(volatile uint32_t *)&ctl->abort = 1;
        return false;
    }
    unsigned long long now = globaltimer();
    if (s.t0 == 0) {
        s.t0 = now;
        return true;
    }
    if (now - s.t0 > p.timeout_ns) {
        raise_error(p, ctl, kErrTimeout, where, task, info);
        return false;
    }
    return true;
}

__device__ __forceinline__ bool wait_mbar(uint64_t *bar, uint32_t parity, const Params &p,
                                          SmemCtl *ctl, uint32_t where, uint32_t task) {
    Spin s;
    while (!mbar_try_wait(bar, parity))
        if (!spin_ok(s, p, ctl, where, task, parity)) return false;
    return true;
}

// Warp-wide verdict of a bounded wait: lane 0 keeps the budget and raises the
// error, every lane gets the same answer, so the warp leaves a poll together.
__device__ __forceinline__ bool warp_spin_ok(Spin &s, const Params &p, SmemCtl *ctl, uint32_t task,
                                             uint32_t info) {
    int ok = 1;
    if ((threadIdx.x & 31) == 0) ok = spin_ok(s, p, ctl, W_TAG, task, info) ? 1 : 0;
    if (p.poll_ns) __nanosleep(p.poll_ns);
    return __shfl_sync(0xffffffffu, ok, 0) != 0;
}

// One tagged value, polled by a single thread (rare paths); on an abandoned
// wait the error is raised and the stale value returned.
__device__ __forceinline__ float wait_tag1(const Params &p, SmemCtl *ctl, const uint64_t *src, uint32_t ep,
                                        uint32_t task) {
    uint64_t v = ld_tag1(src);
    Spin s;
    while (!tag_ok(v, ep)) {
        if (!spin_ok(s, p, ctl, W_TAG, task, 1u)) break;
        v = ld_tag1(src);
    }
    return tag_val(v);
}

__device__ __forceinline__ uint64_t *tag_buf(const Params &p, int layer, size_t off) {
    return p.tag + (size_t)layer * p.tl.layer + off;
}
// The copy of the replicated vectors this SM reads.
__device__ __forceinline__ size_t my_copy(size_t stride) { return (size_t)(blockIdx.x % kReplicas) * stride; }

// ---------------------------------------------------------------------------
// task geometry shared by the loader and the workers
// ---------------------------------------------------------------------------
// Attention chunk of one work item (sequence b, q head h, chunk c).
struct AttnChunk {
    int b, h, kvh, c;
    bool active;      // sequence b takes part in this step
    int P;            // position of the new token
    int c0, c1;       // positions [c0, c1) of this chunk (c1 <= P + 1)
    int npre;         // cached positions loaded by pages: [c0, c0 + npre), all < P
    bool has_new;     // P is in [c0, c1)
    int nc;           // chunks with positions for this sequence (the others are empty)
};

__device__ __forceinline__ AttnChunk attn_chunk(const Params &p, const SmemCtl *ctl, int step, int item) {
    const Shape &s = p.s;
    AttnChunk a;
    const int groups = s.nq / s.HA;          // items per (sequence, chunk)
    a.b = item / (groups * s.NC);
    a.h = ((item / s.NC) % groups) * s.HA;   // the item's first q head
    a.kvh = a.h / s.G;
    a.c = item % s.NC;
    a.active = a.b < p.batch;
    a.P = 0; a.c0 = 0; a.c1 = 0; a.npre = 0; a.has_new = false; a.nc = 0;
    if (a.active) {
        a.P = ctl->pos[a.b] + step;
        int C = a.P + 1;
        // at most NC chunks, but no fewer than kAttnChunkPositions positions
        // per chunk: short contexts use one chunk (nothing to merge)
        const int nc = min(s.NC, (C + kAttnChunkPositions - 1) / kAttnChunkPositions);
        int Lc = (C + nc - 1) / nc;
        a.nc = nc;
        a.c0 = a.c * Lc;
        a.c1 = min(a.c0 + Lc, C);
        if (a.c0 >= C) { a.c0 = C; a.c1 = C; }
        int pend = min(a.c1, a.P);
        a.npre = max(0, pend - a.c0);
        a.has_new = a.c0 <= a.P && a.P < a.c1;
    }
    return a;
}

// Weights of every GEMV op are laid out so that tile t's 8 rows are
// contiguous at base + t * 8 * K (bf16 elements): the q/k/v and gate/up
// matrices are repacked into that order by mk_create, the O-projection,
// down-projection and LM head already are in it.  A task (tiles [begin,
// end)) is therefore one contiguous byte range, streamed page by page.
struct GemvStream {
    const char *src;      // next byte to load
    long long left;       // bytes of real rows still to load
    uint32_t page_bytes;  // rows_per_page * K * 2
    int npages;
};

__device__ __forceinline__ const uint16_t *gemv_base(const Params &p, int kind, int layer) {
    if (kind == OP_LMHEAD) return p.lm_head;
    const LayerW &L = p.layers[layer];
    switch (kind) {
    case OP_QKV: return L.qkv;
    case OP_OPROJ: return L.wo;
    case OP_GATEUP: return L.gu;
    default: return L.wd;
    }
}

__device__ __forceinline__ GemvStream gemv_stream(const Params &p, const Task &t) {
    const int K = op_k(p.s, t.kind);
    const int rpp = rows_per_page(K);
    const long long row_bytes = 2LL * K;
    const long long r0 = tile_row_offset(p.s, t.kind, t.begin);
    const long long r1 = tile_row_offset(p.s, t.kind, t.end);
    GemvStream g;
    g.src = reinterpret_cast<const char *>(gemv_base(p, t.kind, t.layer)) + r0 * row_bytes;
    long long rows = r1 - r0;
    if (t.kind == OP_LMHEAD) rows = min(rows, (long long)p.s.V - r0);
    g.left = rows * row_bytes;
    g.page_bytes = (uint32_t)(rpp * row_bytes);
    g.npages = (int)((r1 - r0 + rpp - 1) / rpp);   // a trailing 8-row tile gets a partial page
    return g;
}

// ---------------------------------------------------------------------------
// loader role (one thread)
// ---------------------------------------------------------------------------
struct Ring {
    uint32_t seq = 0;     // pages issued
    bool stats = false;
    unsigned long long t_empty = 0;
    // per slot: how its last occupant is released (by the workers through
    // `empty`, or -- a page moved on into tensor memory -- by the stasher's
    // copy completion through `cpdone`), and how often each barrier has
    // completed so far (its next wait's parity)
    uint32_t via_tmem = 0;   // bit s: slot s's last page went to TMEM
    uint32_t odd_empty = 0;  // bit s: pages of slot s released through `empty` so far, mod 2
    uint32_t odd_cp = 0;     // bit s: pages of slot s released through `cpdone` so far, mod 2
};

// Wait until the slot's previous page has been released, then arm the
// slot's landing barrier for `bytes` and return it in `bar` (the copies of
// the page complete on it).  `to_tmem`: this page will be copied on into
// tensor memory (landing on tland, released by the stasher) rather than read
// by the workers (landing on full, released by them).
__device__ __forceinline__ bool ring_acquire(const Params &p, SmemCtl *ctl, Ring &r, uint32_t bytes,
                                             uint32_t task, uint32_t &slot, bool to_tmem, uint64_t *&bar) {
    slot = r.seq % kNumPages;
    const unsigned long long t0 = r.stats ? globaltimer() : 0ull;
    bool ok = true;
    if (r.seq >= (uint32_t)kNumPages) {
        // the m-th release through a barrier completes its phase m - 1:
        // wait on parity (m - 1) & 1 = (m & 1) ^ 1
        if (r.via_tmem & (1u << slot))
            ok = wait_mbar(&ctl->cpdone[slot], ((r.odd_cp >> slot) & 1u) ^ 1u, p, ctl, W_EMPTY, task);
        else
            ok = wait_mbar(&ctl->empty[slot], ((r.odd_empty >> slot) & 1u) ^ 1u, p, ctl, W_EMPTY, task);
    }
    if (r.stats) r.t_empty += globaltimer() - t0;
    if (!ok) return false;
    if (to_tmem) { r.via_tmem |= 1u << slot; r.odd_cp ^= 1u << slot; }
    else { r.via_tmem &= ~(1u << slot); r.odd_empty ^= 1u << slot; }
    bar = to_tmem ? &ctl->tland[slot] : &ctl->full[slot];
    mbar_arrive_expect_tx(bar, bytes);
    ++r.seq;
    return true;
}

__device__ void loader_role(const Params &p, unsigned char *pages, SmemCtl *ctl) {
    const int q0 = p.qoff[blockIdx.x], q1 = p.qoff[blockIdx.x + 1];
    Ring ring;
    ring.stats = p.sm_stats != nullptr;
    const unsigned long long t_begin = ring.stats ? globaltimer() : 0ull;
    long long issued = 0;   // GEMV bytes copied into the ring so far
    bool ok = true;         // false when a wait was abandoned
    const uint64_t wpol = policy_evict_first();
    // L2 prefetch cursor: GEMV weight bytes of the queue, bulk-prefetched
    // into L2 up to l2_lookahead bytes beyond what the ring has taken, so
    // HBM keeps streaming while the ring is full (one instruction per 64 KB)
    const int qlen = q1 - q0;
    const long long pf_end = (long long)qlen * p.n_steps;   // queue positions over all steps
    long long pf_k = -1;
    const char *pf_src = nullptr;
    long long pf_left = 0, pf_done = 0;
    auto prefetch_to = [&](long long target) {
        while (pf_done < target) {
            if (pf_left <= 0) {
                do { ++pf_k; } while (pf_k < pf_end && p.qtasks[q0 + pf_k % qlen].kind == OP_ATTN);
                if (pf_k >= pf_end) { pf_done = 0x7fffffffffffffffLL; return; }
                const GemvStream g = gemv_stream(p, p.qtasks[q0 + pf_k % qlen]);
                pf_src = g.src;
                pf_left = g.left;
                continue;
            }
            const uint32_t n = (uint32_t)min(pf_left, (long long)kPageBytes);
            prefetch_l2(pf_src, n);
            pf_src += n;
            pf_left -= n;
            pf_done += n;
        }
    };
    for (int step = 0; step < p.n_steps && ok; ++step)
    for (int qi = q0; qi < q1 && ok; ++qi) {
        if (*(volatile uint32_t *)&ctl->stop) { ok = false; break; }   // generation ended
        const Task t = p.qtasks[qi];
        const int id = t.sm;
        {
            // publish the task's record to the workers (ring of kTaskRing:
            // wait until every warp has read the record this slot held)
            const int k = step * qlen + (qi - q0);
            Spin sr;
            while (k >= kTaskRing &&
                   *(volatile uint32_t *)&ctl->tq_reads < (uint32_t)kWorkerWarps * (uint32_t)(k - kTaskRing + 1))
                if (!spin_ok(sr, p, ctl, W_READY, (uint32_t)id, 4u)) { ok = false; break; }
            if (!ok) break;
            TaskRec &r = ctl->tq[k % kTaskRing];
            r.t = t;
            r.gain = t.kind == OP_QKV ? p.layers[t.layer].g_attn
                   : t.kind == OP_GATEUP ? p.layers[t.layer].g_mlp
                   : t.kind == OP_LMHEAD ? p.g_final : nullptr;
            st_release_cta_shared(&ctl->tq_pub, (uint32_t)(k + 1));
        }
        if (t.kind == OP_ATTN) {
            const AttnChunk a = attn_chunk(p, ctl, step, t.begin);
            const int npp = attn_pos_per_page(p.s.d);
            const LayerW &L = p.layers[t.layer];
            const size_t head_off = ((size_t)a.b * p.s.nkv + a.kvh) * p.s.S;
            for (int pos0 = a.c0; pos0 < a.c0 + a.npre; pos0 += npp) {
                const int n = min(npp, a.c0 + a.npre - pos0);
                const uint32_t bytes = (uint32_t)n * p.s.d * 2;
                uint32_t slot;
                uint64_t *bar;
                if (!ring_acquire(p, ctl, ring, 2 * bytes, (uint32_t)id, slot, false, bar)) { ok = false; break; }
                unsigned char *dst = pages + (size_t)slot * kPageBytes;
                const size_t off = (head_off + pos0) * p.s.d;
                bulk_g2s(dst, L.kc + off, bytes, bar);
                bulk_g2s(dst + (size_t)npp * p.s.d * 2, L.vc + off, bytes, bar);
            }
            continue;
        }
        GemvStream g = gemv_stream(p, t);
        const bool to_tmem = tmem_page_op(p.s, t.kind);
        for (int k = 0; k < g.npages; ++k) {
            const uint32_t bytes = (uint32_t)max(0LL, min((long long)g.page_bytes, g.left));
            if (p.l2_lookahead) prefetch_to(issued + bytes + p.l2_lookahead);
            uint32_t slot;
            uint64_t *bar;
            if (!ring_acquire(p, ctl, ring, bytes, (uint32_t)id, slot, to_tmem, bar)) { ok = false; break; }
            if (bytes) bulk_g2s_hint(pages + (size_t)slot * kPageBytes, g.src, bytes, bar, wpol);
            g.src += g.page_bytes;
            g.left -= bytes;
            issued += bytes;
        }
    }
    *(volatile uint32_t *)&ctl->loader_done = 1u;
    // Let every copy already issued land before this thread returns, so no
    // bulk copy can still be writing shared memory when the CTA exits: the
    // last page of each used slot has completed its landing barrier (the
    // m-th arming of a barrier completes its phase m - 1).
    const uint32_t used = ring.seq < (uint32_t)kNumPages ? ring.seq : (uint32_t)kNumPages;
    for (uint32_t sl = 0; sl < used; ++sl) {
        const bool t = (ring.via_tmem >> sl) & 1u;
        uint64_t *bar = t ? &ctl->tland[sl] : &ctl->full[sl];
        const uint32_t par = (((t ? ring.odd_cp : ring.odd_empty) >> sl) & 1u) ^ 1u;
        Spin s;
        while (!mbar_try_wait(bar, par)) {
            if ((++s.n & 127u) == 0u) {
                unsigned long long now = globaltimer();
                if (s.t0 == 0) s.t0 = now;
                else if (now - s.t0 > p.timeout_ns) break;
            }
        }
    }
    if (ring.stats) {
        unsigned long long *st = p.sm_stats + (size_t)blockIdx.x * kStatSlots;
        st[ST_LOADER_EMPTY] = ring.t_empty;
        st[ST_LOADER_PAGES] = ring.seq;
        st[ST_LOADER_TOTAL] = globaltimer() - t_begin;
    }
}

// ---------------------------------------------------------------------------
// scheduler role (one thread)
// ---------------------------------------------------------------------------
// Gates the queue on event counters (only when tasks wait on events): task
// qi becomes ready once its dependency's counter reaches threshold x epoch.
__device__ void scheduler_role(const Params &p, SmemCtl *ctl, uint32_t ep) {
    const int q0 = p.qoff[blockIdx.x], q1 = p.qoff[blockIdx.x + 1];
    unsigned long long t_dep = 0;
    const int qlen = q1 - q0;
    for (int step = 0; step < p.n_steps; ++step)
    for (int qi = q0; qi < q1; ++qi) {
        const int id = p.qtasks[qi].sm;
        const int dep = p.qtasks[qi].dep;
        if (dep >= 0) {
            const uint32_t target = p.thresholds[dep] * (ep + (uint32_t)step);
            Spin s;
            const unsigned long long t0 = p.sm_stats ? globaltimer() : 0ull;
            while ((int32_t)(ld_acquire_gpu(&p.events[dep]) - target) < 0)
                if (!spin_ok(s, p, ctl, W_DEP, (uint32_t)id, (uint32_t)dep)) return;
            if (p.sm_stats) t_dep += globaltimer() - t0;
        }
        if (p.trace) p.trace[id].t_ready = globaltimer();
        st_release_cta_shared(&ctl->ready_upto, (uint32_t)(step * qlen + qi - q0 + 1));
    }
    if (p.sm_stats) p.sm_stats[(size_t)blockIdx.x * kStatSlots + ST_SCHED_DEP] = t_dep;
}

// ---------------------------------------------------------------------------
// stasher role (one thread; only with Shape::tmem)
// ---------------------------------------------------------------------------
// Walks the same page sequence as the loader.  Every page of an op whose
// pages pass through tensor memory (tmem_page_op) is, once it has landed in
// its shared-memory slot, copied on into the next free TMEM slot with 16
// tcgen05.cp (one 4 KB block each, see tmem_page_src); one commit then
// signals the workers (tfull) and another frees the shared-memory slot for
// the loader (cpdone) as soon as the copies have read it.  Landed weights so
// leave the shared-memory ring at once, and the ring (3 pages in flight from
// HBM) plus tensor memory (4 landed pages) buffer 7 pages per SM.
__device__ void stasher_role(const Params &p, unsigned char *pages, SmemCtl *ctl) {
    const int q0 = p.qoff[blockIdx.x], q1 = p.qoff[blockIdx.x + 1];
    uint32_t k = 0;    // pages of the sequence (all kinds)
    uint32_t tk = 0;   // pages moved into tensor memory
    uint32_t odd = 0;  // bit s: pages of slot s moved so far, mod 2 (the parity of the next tland wait)
    const uint32_t tbase = ctl->tmem_base;
    bool ok = true;
    for (int step = 0; step < p.n_steps && ok; ++step)
    for (int qi = q0; qi < q1 && ok; ++qi) {
        const Task t = p.qtasks[qi];
        if (t.kind == OP_ATTN) {
            const AttnChunk a = attn_chunk(p, ctl, step, t.begin);
            const int npp = attn_pos_per_page(p.s.d);
            k += (uint32_t)((a.npre + npp - 1) / npp);
            continue;
        }
        const GemvStream g = gemv_stream(p, t);
        if (!tmem_page_op(p.s, t.kind)) { k += (uint32_t)g.npages; continue; }
        for (int pg = 0; pg < g.npages; ++pg, ++k) {
            const uint32_t slot = k % kNumPages;
            if (!wait_mbar(&ctl->tland[slot], (odd >> slot) & 1u, p, ctl, W_FULL, (uint32_t)t.sm)) { ok = false; break; }
            odd ^= 1u << slot;
            const uint32_t ts = tk % kTmemSlots;
            if (tk >= (uint32_t)kTmemSlots &&
                !wait_mbar(&ctl->tempty[ts], ((tk / kTmemSlots) - 1u) & 1u, p, ctl, W_EMPTY, (uint32_t)t.sm)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const unsigned char *src = pages + (size_t)slot * kPageBytes;
            const uint32_t dst = tbase + ts * kTmemSlotCols;
#pragma unroll 1
            for (int c = 0; c < 16; ++c) tmem_cp_128x256b(dst + 8 * c, smem_desc(src + 4096 * c, 2048, 128));
            tc_commit(&ctl->tfull[ts]);
            tc_commit(&ctl->cpdone[slot]);
            ++tk;
        }
    }
    // every copy issued must have completed before the CTA frees tensor
    // memory: the last commit arrives only after all earlier copies
    if (tk > 0) {
        const uint32_t ts = (tk - 1) % kTmemSlots, par = ((tk - 1) / kTmemSlots) & 1u;
        Spin sp;
        while (!mbar_try_wait(&ctl->tfull[ts], par)) {
            if ((++sp.n & 127u) == 0u) {
                const unsigned long long now = globaltimer();
                if (sp.t0 == 0) sp.t0 = now;
                else if (now - sp.t0 > p.timeout_ns) break;
            }
        }
    }
}

// Publishes task completions: workers post the finished task's event in a
// shared-memory ring (after the barrier that ends the task), this thread
// performs the gpu-scope release add, so no worker stalls on the release.
__device__ void signaler_role(const Params &p, SmemCtl *ctl) {
    const uint32_t total = (uint32_t)(p.qoff[blockIdx.x + 1] - p.qoff[blockIdx.x]) * (uint32_t)p.n_steps;
    uint32_t done = 0;
    while (done < total) {
        Spin s;
        uint32_t posted;
        while ((posted = ld_acquire_cta_shared(&ctl->sig_post)) == done)
            if (!spin_ok(s, p, ctl, W_READY, 0xfffffffeu, done)) return;
        for (; done < posted; ++done) red_release_gpu(&p.events[ctl->sig_ev[done % kSigRing]], 1u);
        *(volatile uint32_t *)&ctl->sig_done = done;
    }
}

// ---------------------------------------------------------------------------
// worker helpers
// ---------------------------------------------------------------------------
struct WState {
    uint32_t slot = 0;       // ring slot of the next page (of any kind)
    uint32_t odd = 0;        // bit s: pages read from slot s so far, mod 2 (the parity of the next full wait)
    uint32_t tslot = 0;      // tensor-memory slot of the next page that passes through it
    uint32_t tphase = 0;     // its tfull-barrier parity
    uint32_t wphase = 0;     // worker-barrier phase
    uint32_t need = 0;       // ready_upto value that activates the current task
    uint32_t ep = 0;         // this launch's epoch: the tag of this step's activations
    uint32_t ep_out = 0;     // tag the current task stores (ep, or stale under the test hook)
    const uint16_t *gain = nullptr;   // RMSNorm gain of the current task's input (null if none)
    int red_buf = 0;
    int task_id = 0;
    unsigned long long *stat = nullptr;   // per-phase accumulators in shared memory (trace mode, thread 0)
};
// Trace-mode time accounting of worker thread 0, accumulated in shared memory
// so it costs no registers across the task bodies.
enum WStat { WS_FULL = 0, WS_READY, WS_SYNC, WS_PRO, WS_DOT, WS_EPI, WS_END, WS_TASKS, WS_ATT, WS_FIRST, WS_TASKWAIT, WS_COLS, kWStats };
__device__ __forceinline__ unsigned long long phase_begin(const WState &w) {
    return w.stat ? globaltimer() : 0ull;
}
__device__ __forceinline__ void phase_end(const WState &w, unsigned long long t0, int which) {
    if (w.stat) w.stat[which] += globaltimer() - t0;
}
// Trace stamps of the current task (thread 0 only).
__device__ __forceinline__ void stamp_input(const Params &p, const WState &w) {
    if (p.trace && threadIdx.x == 0) p.trace[w.task_id].t_input = globaltimer();
}
__device__ __forceinline__ void stamp_done(const Params &p, const WState &w) {
    if (p.trace && threadIdx.x == 0) p.trace[w.task_id].t_done = globaltimer();
}

// All worker warps meet; bounded.
__device__ __forceinline__ bool worker_sync(const Params &p, SmemCtl *ctl, WState &w) {
    __syncwarp();
    const unsigned long long t0 = phase_begin(w);
    if ((threadIdx.x & 31) == 0) mbar_arrive(&ctl->wbar);
    bool ok = wait_mbar(&ctl->wbar, w.wphase, p, ctl, W_WBAR, (uint32_t)w.task_id);
    w.wphase ^= 1u;
    phase_end(w, t0, WS_SYNC);
    return ok;
}

// With MK_FLAG_EVENT_WAIT: wait until the scheduler has activated the
// current task (its dependent event fired); bounded.  Otherwise tasks start
// at once and wait on their tagged inputs.
__device__ __forceinline__ bool wait_ready(const Params &p, SmemCtl *ctl, WState &w) {
    if (!p.event_wait) return true;
    Spin s;
    const unsigned long long t0 = phase_begin(w);
    while (ld_acquire_cta_shared(&ctl->ready_upto) < w.need)
        if (!spin_ok(s, p, ctl, W_READY, (uint32_t)w.task_id, 0u)) return false;
    phase_end(w, t0, WS_READY);
    if (p.trace && threadIdx.x == 0) p.trace[w.task_id].t_start = globaltimer();
    return true;
}

// Trace stamps when tasks wait on their tagged inputs: the task counts as
// ready (and started) once every input word it needs carried this step's tag.
__device__ __forceinline__ void stamp_ready(const Params &p, const WState &w) {
    if (p.trace && !p.event_wait && threadIdx.x == 0) {
        const unsigned long long t = globaltimer();
        p.trace[w.task_id].t_ready = t;
        p.trace[w.task_id].t_start = t;
    }
}

__device__ __forceinline__ bool wait_page(const Params &p, SmemCtl *ctl, WState &w, uint32_t &slot) {
    slot = w.slot;
    const unsigned long long t0 = phase_begin(w);
    const bool ok = wait_mbar(&ctl->full[slot], (w.odd >> slot) & 1u, p, ctl, W_FULL, (uint32_t)w.task_id);
    phase_end(w, t0, WS_FULL);
    phase_end(w, t0, WS_TASKWAIT);
    return ok;
}

__device__ __forceinline__ void release_page(SmemCtl *ctl, WState &w, uint32_t slot) {
    __syncwarp();
    if ((threadIdx.x & 31) == 0) mbar_arrive(&ctl->empty[slot]);
    w.odd ^= 1u << slot;
    if (++w.slot == (uint32_t)kNumPages) w.slot = 0;
}

// A page that passes through tensor memory: wait until the stasher's copies
// into the next TMEM slot have completed.  The page also went through the
// next shared-memory slot (the stasher released that one), so the
// shared-memory position advances too.
__device__ __forceinline__ bool wait_tpage(const Params &p, SmemCtl *ctl, WState &w) {
    const unsigned long long t0 = phase_begin(w);
    const bool ok = wait_mbar(&ctl->tfull[w.tslot], w.tphase, p, ctl, W_FULL, (uint32_t)w.task_id);
    phase_end(w, t0, WS_FULL);
    phase_end(w, t0, WS_TASKWAIT);
    tc_fence_after();
    if (++w.slot == (uint32_t)kNumPages) w.slot = 0;
    return ok;
}
__device__ __forceinline__ void release_tpage(SmemCtl *ctl, WState &w) {
    tc_fence_before();
    __syncwarp();
    if ((threadIdx.x & 31) == 0) mbar_arrive(&ctl->tempty[w.tslot]);
    if (++w.tslot == (uint32_t)kTmemSlots) { w.tslot = 0; w.tphase ^= 1u; }
}

// Sum of one float over the 256 worker threads (bounded barrier inside).
__device__ __forceinline__ bool worker_block_sum(const Params &p, SmemCtl *ctl, WState &w, float v,
                                                 float &out) {
    v = warp_sum(v);
    const int warp = threadIdx.x >> 5;
    if ((threadIdx.x & 31) == 0) ctl->scal[warp] = v;
    if (!worker_sync(p, ctl, w)) return false;
    float t = 0.f;
#pragma unroll
    for (int i = 0; i < kWorkerWarps; ++i) t += ctl->scal[i];
    out = t;
    return true;
}

// Signal the task's triggering event after every worker's writes.
// Post the task's completion to the signaler (thread 0, after the barrier
// that ends the task: every worker's output stores happen before it; the
// release store to the ring makes them visible to the signaler, whose
// gpu-scope release add publishes them with the event).
__device__ __forceinline__ bool signal_event(const Params &p, SmemCtl *ctl, const Task &t) {
    const uint32_t n = ctl->sig_post;   // only thread 0 writes it
    Spin s;
    while (n - *(volatile uint32_t *)&ctl->sig_done >= (uint32_t)kSigRing)
        if (!spin_ok(s, p, ctl, W_READY, 0xfffffffdu, n)) return false;
    ctl->sig_ev[n % kSigRing] = (uint32_t)t.trig;
    st_release_cta_shared(&ctl->sig_post, n + 1u);
    return true;
}

// Copy a tagged vector of n values (n a multiple of 8, n <= 2 * 256 * NP)
// into ctl->stage, polling every word until it carries this step's tag.  The
// 256 worker threads take 16-byte pairs round-robin (coalesced), only stale
// pairs are reloaded.  ss returns the thread's partial sum of squares, added
// up in pair order once every pair is in (not in the order the pairs
// arrived), so the RMSNorm of a step does not depend on timing.  The
// caller's worker barrier publishes the stage to every warp.
// Stage layout: the first four values of every 8-value vector v at float4
// slot v, the last four at slot n/8 + v, so that a warp reading vectors
// lane + 32 j touches consecutive 16-byte slots (no bank conflicts).
template <int NP>
__device__ __forceinline__ bool stage_tagged(const Params &p, SmemCtl *ctl, const WState &w,
                                             const uint64_t *src, int n, float &ss) {
    constexpr int NB = NP < 8 ? NP : 8;   // loads in flight per thread
    const int tid = threadIdx.x;
    const int npairs = n >> 1, n8 = n >> 3;
    float2 *st = reinterpret_cast<float2 *>(ctl->stage);
    float acc = 0.f;
    uint32_t pend = 0;
    // pairs j = jb .. jb + NB - 1 of the thread: issue all loads, then store
    // the fresh ones (one round trip per batch); stale ones are polled after
    auto batch = [&](int jb, bool only_pending) {
        ulonglong2 q[NB];
#pragma unroll
        for (int k = 0; k < NB; ++k) {
            const int j = jb + k, i = tid + j * kWorkerThreads;
            const bool want = i < npairs && (!only_pending || (pend & (1u << j)));
            q[k] = want ? ld_tag2(src + 2 * i) : make_ulonglong2(0ull, 0ull);
            if (want) pend |= 1u << j;
        }
#pragma unroll
        for (int k = 0; k < NB; ++k) {
            const int j = jb + k, i = tid + j * kWorkerThreads;
            if ((pend & (1u << j)) && tag_ok(q[k].x, w.ep) && tag_ok(q[k].y, w.ep)) {
                const float2 v = make_float2(tag_val(q[k].x), tag_val(q[k].y));
                st[2 * (((i >> 1) & 1) * n8 + (i >> 2)) + (i & 1)] = v;
                pend &= ~(1u << j);
            }
        }
    };
#pragma unroll
    for (int jb = 0; jb < NP; jb += NB) batch(jb, false);
    Spin sp;
    while (__any_sync(0xffffffffu, pend != 0u)) {
        if (!warp_spin_ok(sp, p, ctl, (uint32_t)w.task_id, 0u)) return false;
#pragma unroll
        for (int jb = 0; jb < NP; jb += NB) batch(jb, true);
    }
    // this thread's own pairs, read back in order
#pragma unroll
    for (int j = 0; j < NP; ++j) {
        const int i = tid + j * kWorkerThreads;
        if (i < npairs) {
            const float2 v = st[2 * (((i >> 1) & 1) * n8 + (i >> 2)) + (i & 1)];
            acc = fmaf(v.x, v.x, fmaf(v.y, v.y, acc));
        }
    }
    ss = acc;
    return true;
}

// Poll nh q heads' partials of one KV head into ctl->stage, densely: head g
// takes `per` words (its chunks' o[d], m, l) at src + g * stride.  Pairs of
// words go round-robin over the 256 worker threads; a fresh pair is stored
// to shared memory at once, so only stale pairs are reloaded and no values
// stay in registers across the poll.
__device__ __forceinline__ bool stage_partials(const Params &p, SmemCtl *ctl, const WState &w,
                                               const uint64_t *src, int nh, int per, int stride) {
    constexpr int NP = kStageFloats / 2 / kWorkerThreads;   // pairs per thread at most
    const int tid = threadIdx.x;
    const int hp = per >> 1, npairs = nh * hp;
    float2 *st = reinterpret_cast<float2 *>(ctl->stage);
    uint32_t pend = 0;
    // all loads of a pass are issued before any result is looked at
    auto addr = [&](int j) {
        const int i = tid + j * kWorkerThreads;
        const int g = i / hp;
        return src + (size_t)g * stride + 2 * (i - g * hp);
    };
    ulonglong2 q[NP];
#pragma unroll
    for (int j = 0; j < NP; ++j) {
        const bool in = tid + j * kWorkerThreads < npairs;
        q[j] = in ? ld_tag2(addr(j)) : make_ulonglong2(0ull, 0ull);
        if (in) pend |= 1u << j;
    }
    Spin sp;
    while (true) {
#pragma unroll
        for (int j = 0; j < NP; ++j)
            if ((pend & (1u << j)) && tag_ok(q[j].x, w.ep) && tag_ok(q[j].y, w.ep)) {
                st[tid + j * kWorkerThreads] = make_float2(tag_val(q[j].x), tag_val(q[j].y));
                pend &= ~(1u << j);
            }
        if (!__any_sync(0xffffffffu, pend != 0u)) break;
        if (!warp_spin_ok(sp, p, ctl, (uint32_t)w.task_id, 5u)) return false;
#pragma unroll
        for (int j = 0; j < NP; ++j)
            if (pend & (1u << j)) q[j] = ld_tag2(addr(j));
    }
    return true;
}

// One tagged value per lane (lanes with `want`), polled by the whole warp;
// `v` is a first load the caller issued earlier.
__device__ __forceinline__ bool warp_tag1(const Params &p, SmemCtl *ctl, const WState &w,
                                          const uint64_t *src, bool want, uint64_t v, float &out) {
    bool pend = want && !tag_ok(v, w.ep);
    Spin s;
    while (__any_sync(0xffffffffu, pend)) {
        if (!warp_spin_ok(s, p, ctl, (uint32_t)w.task_id, 2u)) return false;
        if (pend) {
            v = ld_tag1(src);
            pend = !tag_ok(v, w.ep);
        }
    }
    out = tag_val(v);
    return true;
}

// ---------------------------------------------------------------------------
// GEMV task bodies
// ---------------------------------------------------------------------------
// Input vector of a GEMV op (a tagged buffer, or the bf16 embedding row for
// the first layer's QKV) and the RMSNorm gain applied to it, if any.
struct GemvInput {
    const uint64_t *src;
    const uint16_t *src_bf;
    const uint16_t *gain;
};

__device__ __forceinline__ GemvInput gemv_input(const Params &p, const SmemCtl *ctl, const WState &w,
                                                int kind, int layer, int b) {
    const Shape &s = p.s;
    const TagLayout &tl = p.tl;
    GemvInput in{nullptr, nullptr, w.gain};
    switch (kind) {
    case OP_QKV:
        if (layer == 0) in.src_bf = p.embed + (size_t)ctl->tok[b] * s.H;
        else in.src = tag_buf(p, layer - 1, tl.xb) + my_copy(tl.rep_h) + (size_t)b * s.H;
        break;
    case OP_GATEUP: in.src = tag_buf(p, layer, tl.xa) + my_copy(tl.rep_h) + (size_t)b * s.H; break;
    case OP_LMHEAD: in.src = tag_buf(p, s.L - 1, tl.xb) + my_copy(tl.rep_h) + (size_t)b * s.H; break;
    case OP_OPROJ: in.src = tag_buf(p, layer, tl.attn) + my_copy(tl.rep_qd) + (size_t)b * s.QD; break;
    default: in.src = tag_buf(p, layer, tl.act) + my_copy(tl.rep_f) + (size_t)b * s.F; break;
    }
    return in;
}

// Residual stream read by the O projection (layer > 0: the previous layer's
// down output) and the down projection (this layer's O output), and the
// buffer each writes.
__device__ __forceinline__ const uint64_t *resid_in(const Params &p, int kind, int layer, int b) {
    return (kind == OP_DOWN ? tag_buf(p, layer, p.tl.xa) : tag_buf(p, layer - 1, p.tl.xb)) +
           my_copy(p.tl.rep_h) + (size_t)b * p.s.H;
}
__device__ __forceinline__ uint64_t *resid_out(const Params &p, int kind, int layer, int b) {
    return tag_buf(p, layer, kind == OP_DOWN ? p.tl.xb : p.tl.xa) + (size_t)b * p.s.H;
}

__device__ __forceinline__ void scale_vec8(float *x, float sc, const uint16_t *gain, int v) {
    const uint4 g = __ldg(reinterpret_cast<const uint4 *>(gain) + v);
    x[0] *= sc * bf_lo(g.x); x[1] *= sc * bf_hi(g.x); x[2] *= sc * bf_lo(g.y); x[3] *= sc * bf_hi(g.y);
    x[4] *= sc * bf_lo(g.z); x[5] *= sc * bf_hi(g.z); x[6] *= sc * bf_lo(g.w); x[7] *= sc * bf_hi(g.w);
}

// Output row r of the fused q/k/v projection.  q and k rows go to their
// tagged buffers as computed (the attention tasks apply RoPE and append the
// rotated key to the cache); value rows are appended to the bf16 cache and,
// rounded the same way, to the tagged new-value buffer.
__device__ __forceinline__ void qkv_store_row(const Params &p, int layer, int r, float a, int b, int P,
                                              uint32_t ep) {
    const Shape &s = p.s;
    if (r < s.QD) {
        st_tag(tag_buf(p, layer, p.tl.q) + (size_t)b * s.QD + r, a, ep);
    } else if (r < s.QD + s.KD) {
        st_tag(tag_buf(p, layer, p.tl.kn) + (size_t)b * s.KD + (r - s.QD), a, ep);
    } else {
        const int vr = r - s.QD - s.KD;
        const int kvh = vr / s.d, dd = vr % s.d;
        const uint16_t vb = f2bf(a);
        p.layers[layer].vc[(((size_t)b * s.nkv + kvh) * s.S + P) * s.d + dd] = vb;
        st_tag(tag_buf(p, layer, p.tl.vn) + (size_t)b * s.KD + vr, bf2f(vb), ep);
    }
}

// Output of one finished row (or gate/up pair) of a unit epilogue, written
// by one lane (the O and down projections are handled by the caller, which
// owns the residual).
//   a: the row's dot product (the gate row of a pair tile);
//   c: the up row's, pair tiles only.
__device__ __forceinline__ void gemv_epilogue_row(const Params &p, int kind, int layer, int tile,
                                                  int r, float a, float c, int b, int P, uint32_t ep,
                                                  float &best_v, int &best_i) {
    const Shape &s = p.s;
    switch (kind) {
    case OP_QKV:
        qkv_store_row(p, layer, tile * 8 + r, a, b, P, ep);
        break;
    case OP_GATEUP:
        st_tag_rep(tag_buf(p, layer, p.tl.act) + (size_t)b * s.F + tile * 8 + r, p.tl.rep_f, a / (1.0f + expf(-a)) * c, ep);
        break;
    default: {  // OP_LMHEAD
        const int row = tile * 8 + r;
        if (row < s.V) {
            if (p.logits) p.logits[(size_t)b * s.V + row] = a;
            if (a > best_v || (a == best_v && row < best_i)) { best_v = a; best_i = row; }
        }
        break;
    }
    }
}

// Two partial sums per lane -> lanes 0..15 hold the warp total of `a`,
// lanes 16..31 the total of `c`.
__device__ __forceinline__ float dual_reduce(float a, float c, int lane) {
    const bool hi = lane & 16;
    float v = (hi ? c : a) + __shfl_xor_sync(0xffffffffu, hi ? a : c, 16);
    v += __shfl_xor_sync(0xffffffffu, v, 8);
    v += __shfl_xor_sync(0xffffffffu, v, 4);
    v += __shfl_xor_sync(0xffffffffu, v, 2);
    v += __shfl_xor_sync(0xffffffffu, v, 1);
    return v;
}

template <int NVL>
__device__ __forceinline__ float dot_row(const uint4 *row, const float (&xr)[NVL][8], int K8, int lane) {
    float2 acc = make_float2(0.f, 0.f);
#pragma unroll
    for (int j = 0; j < NVL; ++j) {
        const int v = lane + 32 * j;
        if (v < K8) acc = dot8x2(row[v], xr[j], acc);
    }
    return acc.x + acc.y;
}

// Two rows against the same input slice (two independent load/FMA streams,
// packed two-lane FMAs).
template <int NVL>
__device__ __forceinline__ void dot_rows2(const uint4 *ra, const uint4 *rc, const float (&xr)[NVL][8],
                                          int K8, int lane, float &acc_a, float &acc_c) {
    float2 a = make_float2(0.f, 0.f), c = make_float2(0.f, 0.f);
#pragma unroll
    for (int j = 0; j < NVL; ++j) {
        const int v = lane + 32 * j;
        if (v < K8) {
            const uint4 wa = ra[v];
            const uint4 wc = rc[v];
            a = dot8x2(wa, xr[j], a);
            c = dot8x2(wc, xr[j], c);
        }
    }
    acc_a = a.x + a.y;
    acc_c = c.x + c.y;
}

// The same two dot products for a page in tensor memory: row a's 8
// vectors (lane + 32j, j = 0..7) are the 32 columns at `ta`, row c's the 32
// columns at ta + 64; read in quarters of 8 columns so that only 16 row
// words are live at a time.
template <int NVL>
__device__ __forceinline__ void dot_tmem2(uint32_t ta, bool two, const float (&xr)[NVL][8], float &acc_a,
                                          float &acc_c) {
    static_assert(NVL == 8, "a TMEM page row is 2048 columns: 8 vectors per lane");
    float2 a = make_float2(0.f, 0.f), c = make_float2(0.f, 0.f);
    // the second row's columns are read even when the page has one row (a
    // trailing 8-row page): its result is then dropped.  All 64 columns of
    // both rows, then one wait (it covers every load before it)
    uint32_t ra[32], rc[32];
    tmem_ld32(ta, ra);
    tmem_ld32(ta + 64, rc);
    tmem_ld_wait();
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        a = dot8x2(make_uint4(ra[4 * j], ra[4 * j + 1], ra[4 * j + 2], ra[4 * j + 3]), xr[j], a);
        c = dot8x2(make_uint4(rc[4 * j], rc[4 * j + 1], rc[4 * j + 2], rc[4 * j + 3]), xr[j], c);
    }
    acc_a = a.x + a.y;
    acc_c = two ? c.x + c.y : 0.f;
}

// Epilogue of one unit (16 rows: a pair tile or two 8-row tiles; or one
// 8-row tile) whose row sums warp 0 holds: lane e (< rows) has row e's dot
// product `a`, and for pair tiles `c` is row e + 8's.  `resid` is lane L's
// residual of task row L (O / down projections).  Warp 0 calls it whole.
__device__ __forceinline__ void unit_epilogue(const Params &p, SmemCtl *ctl, const WState &w, const Task &t,
                                              int tile, bool pair, int rows, float a, float c, float resid,
                                              int tok, int P, float &best_v, int &best_i) {
    const Shape &s = p.s;
    const int kind = t.kind, layer = t.layer, b = 0;
    const int lane = threadIdx.x & 31, e = lane & 15;
    const int grp_row = 8 * (tile - t.begin) + e;   // row within the task
    const float rres = __shfl_sync(0xffffffffu, resid, grp_row & 31);
    if (pair) {
        if (lane < 8) gemv_epilogue_row(p, kind, layer, tile, lane, a, c, b, P, w.ep_out, best_v, best_i);
    } else if (lane < rows) {
        const int tl = tile + (e >> 3), r = e & 7;
        if (kind == OP_OPROJ || kind == OP_DOWN) {
            const int row = tl * 8 + r;
            const float base = grp_row < 32 ? rres
                             : (kind == OP_OPROJ && layer == 0)
                                   ? bf2f(p.embed[(size_t)tok * s.H + row])
                                   : wait_tag1(p, ctl, resid_in(p, kind, layer, b) + row, w.ep, (uint32_t)w.task_id);
            st_tag_rep(resid_out(p, kind, layer, b) + row, p.tl.rep_h, base + a, w.ep_out);
        } else {
            gemv_epilogue_row(p, kind, layer, tl, r, a, 0.f, b, P, w.ep_out, best_v, best_i);
        }
    }
}

// Convert a bf16 vector of n values (n a multiple of 8) into ctl->stage in
// the layout stage_tagged writes; ss returns the thread's sum of squares.
__device__ __forceinline__ void stage_embed(SmemCtl *ctl, const uint16_t *src, int n, float &ss) {
    float2 *st = reinterpret_cast<float2 *>(ctl->stage);
    const int n8 = n >> 3;
    float acc = 0.f;
    for (int i = threadIdx.x; i < (n >> 1); i += kWorkerThreads) {
        const uint32_t wd = __ldg(reinterpret_cast<const uint32_t *>(src) + i);
        const float2 v = make_float2(bf_lo(wd), bf_hi(wd));
        st[2 * (((i >> 1) & 1) * n8 + (i >> 2)) + (i & 1)] = v;
        acc = fmaf(v.x, v.x, fmaf(v.y, v.y, acc));
    }
    ss = acc;
}

// One warp per row of 2048 (or fewer) columns.  Each lane keeps NVL
// 8-element vectors of its input (vectors lane, lane+32, ...).  A 64 KB page
// holds 16 such rows and warp w takes rows w and 8 + w of every page.
//  * K <= 2048: a page is a unit of 16 matrix rows (a pair tile -- the 8
//    first-half q/k rows and their RoPE partners, or 8 gate rows and the
//    matching up rows -- or two consecutive 8-row tiles); every warp holds
//    the whole input and finishes its rows itself (no cross-warp reduction).
//  * K = 2048 * nseg (nseg = 2 or 4): each matrix row is nseg 2048-column
//    segments, so a page holds 16 / nseg matrix rows and its row w is
//    segment w % nseg of a row; warp w keeps only that segment of the input.
//    The segment sums of a unit go to shared memory and warp 0 adds them up
//    once the unit's nseg pages are done.
// The input vector is staged once per task in shared memory by all worker
// threads (tagged loads, waiting for this step's tags); everything that does
// not depend on it (gains, RoPE cos/sin) is loaded before.
template <int NVL>
__device__ bool gemv_rows(const Params &p, const Task &t, unsigned char *pages, SmemCtl *ctl,
                          WState &w) {
    const Shape &s = p.s;
    const int kind = t.kind, layer = t.layer;
    const int K = op_k(s, kind);
    const int nseg = K > kRowK ? K / kRowK : 1;
    const int K8 = nseg > 1 ? kRowK / 8 : K >> 3;     // vectors per page row
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int seg = warp % nseg;
    const int b = 0;
    const size_t row_bytes = (size_t)K8 * 16;          // one page row
    const int P = ctl->pos[b] + ctl->wstep;
    const int tok = ctl->tok[b];
    // pair tiles (8 gate + the 8 matching up rows): every GATEUP tile
    const int npair = kind == OP_GATEUP ? 0x7fffffff : 0;
    const bool resid_op = kind == OP_OPROJ || kind == OP_DOWN;
    const int task_rows = 8 * (t.end - t.begin);
    const bool tmem = tmem_page_op(s, kind);   // pages come through tensor memory

    // ---- before the dependency
    const uint16_t *gain = w.gain;
    float xr[NVL][8];
    uint4 gv[NVL];   // the RMSNorm gain slice, loaded before the dependency
    const bool embed_in = kind == OP_QKV && layer == 0;
    const bool embed_regs = embed_in && nseg == 1;      // warps read the embedding row themselves
#pragma unroll
    for (int j = 0; j < NVL; ++j) {
        const int v = lane + 32 * j;
        const int vg = seg * K8 + v;                    // vector index in the whole input
        gv[j] = (gain && v < K8) ? __ldg(reinterpret_cast<const uint4 *>(gain) + vg) : make_uint4(0, 0, 0, 0);
        if (embed_regs && v < K8) {
            const uint4 e = __ldg(reinterpret_cast<const uint4 *>(p.embed + (size_t)tok * s.H) + v);
            xr[j][0] = bf_lo(e.x); xr[j][1] = bf_hi(e.x); xr[j][2] = bf_lo(e.y); xr[j][3] = bf_hi(e.y);
            xr[j][4] = bf_lo(e.z); xr[j][5] = bf_hi(e.z); xr[j][6] = bf_lo(e.w); xr[j][7] = bf_hi(e.w);
        }
    }
    // per-tile values.  Whole rows per warp: lane L holds those of tile
    // begin + L, row `warp`.  Segments: warp 0's lane L holds the residual of
    // task row L.
    float pre0 = 0.f;
    const int my_tile = t.begin + lane;
    if (kind == OP_OPROJ && layer == 0) {
        if (nseg == 1 && my_tile < t.end) pre0 = bf2f(p.embed[(size_t)tok * s.H + my_tile * 8 + warp]);
        if (nseg > 1 && warp == 0 && lane < task_rows) pre0 = bf2f(p.embed[(size_t)tok * s.H + 8 * t.begin + lane]);
    }

    // ---- the dependency (tagged inputs), then the activation
    if (!wait_ready(p, ctl, w)) return false;
    unsigned long long tp = phase_begin(w);
    if (embed_regs) {
        // the embedding row needs no dependency: each warp holds it already
        stamp_ready(p, w);
        if (gain) {
            float ss = 0.f;
#pragma unroll
            for (int j = 0; j < NVL; ++j)
                if (lane + 32 * j < K8) {
#pragma unroll
                    for (int e = 0; e < 8; ++e) ss = fmaf(xr[j][e], xr[j][e], ss);
                }
            const float sc = 1.0f / sqrtf(warp_sum(ss) / (float)s.H + s.eps);
#pragma unroll
            for (int j = 0; j < NVL; ++j) {
                const uint4 g = gv[j];
                xr[j][0] *= sc * bf_lo(g.x); xr[j][1] *= sc * bf_hi(g.x);
                xr[j][2] *= sc * bf_lo(g.y); xr[j][3] *= sc * bf_hi(g.y);
                xr[j][4] *= sc * bf_lo(g.z); xr[j][5] *= sc * bf_hi(g.z);
                xr[j][6] *= sc * bf_lo(g.w); xr[j][7] *= sc * bf_hi(g.w);
            }
        }
    } else {
        // the activation: the worker threads copy the input vector into
        // ctl->stage together (tagged: waiting for this step's tags), meet,
        // and then every warp takes its part from there
        const GemvInput in = gemv_input(p, ctl, w, kind, layer, b);
        // the residual word goes out first, so its round trip overlaps the
        // input's: whole rows: lane L's of tile begin + L, row `warp`;
        // segments: warp 0 lane L's of task row L
        const bool resid_wait = resid_op && !(kind == OP_OPROJ && layer == 0) && (nseg == 1 || warp == 0);
        const uint64_t *rsrc = resid_wait ? resid_in(p, kind, layer, b) + (nseg == 1 ? my_tile * 8 + warp : 8 * t.begin + lane)
                                          : nullptr;
        const bool rwant = resid_wait && (nseg == 1 ? my_tile < t.end : lane < task_rows);
        const uint64_t rfirst = rwant ? ld_tag1(rsrc) : 0ull;
        float ss = 0.f;
        if (in.src_bf) stage_embed(ctl, in.src_bf, K, ss);
        else if (!(K <= kRowK ? stage_tagged<kRowK / 512>(p, ctl, w, in.src, K, ss) : stage_tagged<kStageFloats / 512>(p, ctl, w, in.src, K, ss))) return false;
        if (resid_wait && !warp_tag1(p, ctl, w, rsrc, rwant, rfirst, pre0)) return false;
        ss = warp_sum(ss);
        if (lane == 0) ctl->scal[warp] = ss;
        if (!worker_sync(p, ctl, w)) return false;
        stamp_ready(p, w);
        const float4 *src = reinterpret_cast<const float4 *>(ctl->stage);
        const int n8 = K >> 3;
#pragma unroll
        for (int j = 0; j < NVL; ++j) {
            const int v = lane + 32 * j;
            if (v < K8) {
                const float4 a0 = src[seg * K8 + v];
                const float4 a1 = src[n8 + seg * K8 + v];
                xr[j][0] = a0.x; xr[j][1] = a0.y; xr[j][2] = a0.z; xr[j][3] = a0.w;
                xr[j][4] = a1.x; xr[j][5] = a1.y; xr[j][6] = a1.z; xr[j][7] = a1.w;
            } else {
#pragma unroll
                for (int e = 0; e < 8; ++e) xr[j][e] = 0.f;
            }
        }
        if (gain) {
            float tot = 0.f;
#pragma unroll
            for (int i = 0; i < kWorkerWarps; ++i) tot += ctl->scal[i];
            const float sc = 1.0f / sqrtf(tot / (float)s.H + s.eps);
#pragma unroll
            for (int j = 0; j < NVL; ++j) {
                const uint4 g = gv[j];
                xr[j][0] *= sc * bf_lo(g.x); xr[j][1] *= sc * bf_hi(g.x);
                xr[j][2] *= sc * bf_lo(g.y); xr[j][3] *= sc * bf_hi(g.y);
                xr[j][4] *= sc * bf_lo(g.z); xr[j][5] *= sc * bf_hi(g.z);
                xr[j][6] *= sc * bf_lo(g.w); xr[j][7] *= sc * bf_hi(g.w);
            }
        }
    }
    phase_end(w, tp, WS_PRO);
    stamp_input(p, w);

    float best_v = -INFINITY;
    int best_i = 0x7fffffff;
    int tile = t.begin;
    int pu = 0;   // page of the current unit (segments)
    while (tile < t.end) {
        const bool pair = tile < npair;
        const bool two = pair || tile + 1 < t.end;
        float acc_a = 0.f, acc_c = 0.f;
        // rows warp and 8 + warp of the page
        if constexpr (NVL == 8) {
            if (tmem) {
                // the page sits in tensor memory: row warp at column 32 *
                // (warp / 4) of the slot, row 8 + warp 64 columns further,
                // both in this warp's lane quarter
                if (!wait_tpage(p, ctl, w)) return false;
                tp = phase_begin(w);
                const uint32_t ta = ctl->tmem_base + ((uint32_t)(32 * (warp & 3)) << 16) +
                                    w.tslot * (uint32_t)kTmemSlotCols + 32u * (uint32_t)(warp >> 2);
                dot_tmem2<NVL>(ta, two || nseg > 1, xr, acc_a, acc_c);
                release_tpage(ctl, w);
            }
        }
        if (!tmem) {
            uint32_t slot;
            if (!wait_page(p, ctl, w, slot)) return false;
            tp = phase_begin(w);
            const unsigned char *pg = pages + (size_t)slot * kPageBytes;
            const uint4 *row_a = reinterpret_cast<const uint4 *>(pg + warp * row_bytes);
            if (two || nseg > 1) {
                dot_rows2<NVL>(row_a, reinterpret_cast<const uint4 *>(pg + (8 + warp) * row_bytes), xr, K8,
                               lane, acc_a, acc_c);
            } else {
                acc_a = dot_row<NVL>(row_a, xr, K8, lane);
            }
            release_page(ctl, w, slot);
        }
        phase_end(w, tp, WS_DOT);
        tp = phase_begin(w);
        const float v = dual_reduce(acc_a, acc_c, lane);
        if (nseg > 1) {
            // segment sums in page-row order: matrix row r, segment q at r * nseg + q
            float *red = &ctl->red[w.red_buf][0][0];
            if (lane == 0) red[pu * 16 + warp] = v;
            if (lane == 16) red[pu * 16 + 8 + warp] = v;
            const int rows = two ? 16 : 8;
            if (++pu == rows * nseg / 16) {
                pu = 0;
                if (!worker_sync(p, ctl, w)) return false;
                if (warp == 0) {
                    const int e = lane & 15;
                    float a = 0.f, c = 0.f;
                    for (int q = 0; q < nseg; ++q) {
                        a += red[e * nseg + q];
                        c += red[((e + 8) & 15) * nseg + q];
                    }
                    unit_epilogue(p, ctl, w, t, tile, pair, rows, a, c, pre0, tok, P, best_v, best_i);
                }
                w.red_buf ^= 1;
                tile += pair ? 1 : (two ? 2 : 1);
            }
            phase_end(w, tp, WS_EPI);
            continue;
        }
        // tile handled by this lane: lanes 0..15 the first page's, 16..31 the second's
        const int my = (lane < 16 || pair) ? tile : tile + 1;
        const int off = my - t.begin;
        const float q0 = __shfl_sync(0xffffffffu, pre0, off & 31);
        if (pair) {   // gate/up: SiLU(gate) * up
            const float c = __shfl_sync(0xffffffffu, v, 16);
            if (lane == 0)
                st_tag_rep(tag_buf(p, layer, p.tl.act) + (size_t)b * s.F + tile * 8 + warp, p.tl.rep_f,
                           v / (1.0f + expf(-v)) * c, w.ep_out);
            tile += 1;
        } else {
            if ((lane == 0) || (lane == 16 && two)) {
                const int row = my * 8 + warp;
                switch (kind) {
                case OP_QKV:
                    qkv_store_row(p, layer, row, v, b, P, w.ep_out);
                    break;
                case OP_OPROJ:
                case OP_DOWN: {
                    float resid = q0;
                    if (off >= 32)
                        resid = (kind == OP_OPROJ && layer == 0)
                                    ? bf2f(p.embed[(size_t)tok * s.H + row])
                                    : wait_tag1(p, ctl, resid_in(p, kind, layer, b) + row, w.ep, (uint32_t)w.task_id);
                    st_tag_rep(resid_out(p, kind, layer, b) + row, p.tl.rep_h, resid + v, w.ep_out);
                    break;
                }
                default:   // OP_LMHEAD
                    if (row < s.V) {
                        if (p.logits) p.logits[(size_t)b * s.V + row] = v;
                        if (v > best_v || (v == best_v && row < best_i)) { best_v = v; best_i = row; }
                    }
                    break;
                }
            }
            tile += two ? 2 : 1;
        }
        phase_end(w, tp, WS_EPI);
    }
    stamp_done(p, w);
    if (kind == OP_LMHEAD) {
        // segments: warp 0 holds the candidates (lanes 0..15); whole rows:
        // lanes 0 and 16 of every warp
        if (nseg == 1) {
            const float ov = __shfl_sync(0xffffffffu, best_v, 16);
            const int oi = __shfl_sync(0xffffffffu, best_i, 16);
            if (ov > best_v || (ov == best_v && oi < best_i)) { best_v = ov; best_i = oi; }
        } else {
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                const float ov = __shfl_xor_sync(0xffffffffu, best_v, o);
                const int oi = __shfl_xor_sync(0xffffffffu, best_i, o);
                if (ov > best_v || (ov == best_v && oi < best_i)) { best_v = ov; best_i = oi; }
            }
        }
        if (lane == 0) { ctl->att_m[warp][0] = best_v; ctl->att_l[warp][0] = __int_as_float(best_i); }
        if (!worker_sync(p, ctl, w)) return false;
        if (threadIdx.x == 0) {
            for (int k = 1; k < kWorkerWarps; ++k) {
                const float v = ctl->att_m[k][0];
                const int i = __float_as_int(ctl->att_l[k][0]);
                if (v > best_v || (v == best_v && i < best_i)) { best_v = v; best_i = i; }
            }
            p.amax_val[(size_t)b * p.num_lm_tasks + t.slot] = best_v;
            p.amax_idx[(size_t)b * p.num_lm_tasks + t.slot] = best_i;
        }
    }
    return true;
}

// Column split, for K other than 2048 * {1, 2, 4} (e.g. 14336): thread t
// owns 16-byte vectors t, t+256, ... of every row; rows go two at a time,
// each pair reduced across the warp and parked in shared memory, one
// cross-warp sum per 16-row unit, and warp 0 runs the unit's epilogue.
template <int NV>
__device__ bool gemv_cols(const Params &p, const Task &t, unsigned char *pages, SmemCtl *ctl,
                          WState &w) {
    const Shape &s = p.s;
    const int kind = t.kind, layer = t.layer;
    const int K = op_k(s, kind);
    const int K8 = K >> 3;
    const int rpp = rows_per_page(K);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int b = 0;
    const int npair = kind == OP_GATEUP ? 0x7fffffff : 0;   // gate/up pair tiles
    const int P = ctl->pos[b] + ctl->wstep;
    const int tok = ctl->tok[b];
    // residual of row 8 * begin + lane (warp 0), for the O / down projections
    const bool resid_op = kind == OP_OPROJ || kind == OP_DOWN;
    const int task_rows = 8 * (t.end - t.begin);
    float resid = 0.f;
    if (kind == OP_OPROJ && layer == 0 && warp == 0 && lane < task_rows)
        resid = bf2f(p.embed[(size_t)tok * s.H + 8 * t.begin + lane]);
    if (!wait_ready(p, ctl, w)) return false;
    unsigned long long tp = phase_begin(w);
    const GemvInput in = gemv_input(p, ctl, w, kind, layer, b);
    // thread tid takes 16-byte vectors tid, tid + 256, ... of the input: from
    // the embedding row, or as 4 tagged pairs each, stale pairs reloaded
    // until every tag is this step's
    float xr[NV][8];
    uint32_t pend = 0;
#pragma unroll
    for (int j = 0; j < NV; ++j) {
        const int v = tid + j * kWorkerThreads;
#pragma unroll
        for (int e = 0; e < 8; ++e) xr[j][e] = 0.f;
        if (v < K8) {
            if (in.src_bf) {
                const uint4 e = __ldg(reinterpret_cast<const uint4 *>(in.src_bf) + v);
                xr[j][0] = bf_lo(e.x); xr[j][1] = bf_hi(e.x); xr[j][2] = bf_lo(e.y); xr[j][3] = bf_hi(e.y);
                xr[j][4] = bf_lo(e.z); xr[j][5] = bf_hi(e.z); xr[j][6] = bf_lo(e.w); xr[j][7] = bf_hi(e.w);
            } else {
#pragma unroll
                for (int h = 0; h < 4; ++h) {
                    const ulonglong2 q = ld_tag2(in.src + 8 * v + 2 * h);
                    xr[j][2 * h] = tag_val(q.x);
                    xr[j][2 * h + 1] = tag_val(q.y);
                    if (!tag_ok(q.x, w.ep) || !tag_ok(q.y, w.ep)) pend |= 1u << (4 * j + h);
                }
            }
        }
    }
    if (__any_sync(0xffffffffu, pend != 0u)) {
        Spin sp;
        if constexpr (NV <= 2) {
            // few vectors: reload stale pairs with their values
            while (__any_sync(0xffffffffu, pend != 0u)) {
                if (!warp_spin_ok(sp, p, ctl, (uint32_t)w.task_id, 3u)) return false;
#pragma unroll
                for (int j = 0; j < NV; ++j)
#pragma unroll
                    for (int h = 0; h < 4; ++h)
                        if (pend & (1u << (4 * j + h))) {
                            const ulonglong2 q = ld_tag2(in.src + 8 * (tid + j * kWorkerThreads) + 2 * h);
                            xr[j][2 * h] = tag_val(q.x);
                            xr[j][2 * h + 1] = tag_val(q.y);
                            if (tag_ok(q.x, w.ep) && tag_ok(q.y, w.ep)) pend &= ~(1u << (4 * j + h));
                        }
            }
        } else {
            // many vectors: poll only the tag halves of the stale pairs (one
            // register each), then load the values once more -- a word whose
            // tag was seen reads back this step's value
            while (__any_sync(0xffffffffu, pend != 0u)) {
                if (!warp_spin_ok(sp, p, ctl, (uint32_t)w.task_id, 3u)) return false;
#pragma unroll
                for (int j = 0; j < NV; ++j)
#pragma unroll
                    for (int h = 0; h < 4; ++h)
                        if (pend & (1u << (4 * j + h))) {
                            const uint64_t *q = in.src + 8 * (tid + j * kWorkerThreads) + 2 * h;
                            if (ld_tag_hi(q) == w.ep && ld_tag_hi(q + 1) == w.ep) pend &= ~(1u << (4 * j + h));
                        }
            }
#pragma unroll
            for (int j = 0; j < NV; ++j) {
                const int v = tid + j * kWorkerThreads;
                if (v < K8)
#pragma unroll
                    for (int h = 0; h < 4; ++h) {
                        const ulonglong2 q = ld_tag2(in.src + 8 * v + 2 * h);
                        xr[j][2 * h] = tag_val(q.x);
                        xr[j][2 * h + 1] = tag_val(q.y);
                    }
            }
        }
    }
    if (resid_op && !(kind == OP_OPROJ && layer == 0) && warp == 0) {
        const uint64_t *rsrc = resid_in(p, kind, layer, b) + 8 * t.begin + lane;
        if (!warp_tag1(p, ctl, w, rsrc, lane < task_rows, lane < task_rows ? ld_tag1(rsrc) : 0ull, resid))
            return false;
    }
    float ss = 0.f;
#pragma unroll
    for (int j = 0; j < NV; ++j)
#pragma unroll
        for (int e = 0; e < 8; ++e) ss = fmaf(xr[j][e], xr[j][e], ss);
    if (in.gain) {
        float tot;
        if (!worker_block_sum(p, ctl, w, ss, tot)) return false;
        stamp_ready(p, w);
        const float sc = 1.0f / sqrtf(tot / (float)s.H + s.eps);
#pragma unroll
        for (int j = 0; j < NV; ++j) {
            const int v = tid + j * kWorkerThreads;
            if (v < K8) scale_vec8(xr[j], sc, in.gain, v);
        }
    } else {
        // trace mode: the stamp marks the moment every thread has its input
        if (p.trace && !p.event_wait && !worker_sync(p, ctl, w)) return false;
        stamp_ready(p, w);
    }
    phase_end(w, tp, WS_PRO);
    stamp_input(p, w);
    bool first_page = true;
    float best_v = -INFINITY;
    int best_i = 0x7fffffff;
    const size_t row_bytes = (size_t)K * 2;
    // groups of 16 rows: one pair tile, or two consecutive 8-row tiles.  Rows
    // go two at a time in page order (rows 2k and 2k + 1), each pair reduced
    // across the warp right away and its warp partials parked in shared
    // memory, so the loop stays rolled: compact code that stays in the
    // instruction cache instead of 16 unrolled rows.
    int tile = t.begin;
    uint32_t slot = 0;
    const unsigned char *page = pages;
    while (tile < t.end) {
        const bool pair = tile < npair;
        const int rows = pair ? 16 : (tile + 1 < t.end ? 16 : 8);
        float *red = ctl->red[w.red_buf][warp];
#pragma unroll 1
        for (int k = 0; k < rows; k += 2) {
            float acc2[2];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int rr = k + h;
                if ((rr & (rpp - 1)) == 0) {
                    if (!wait_page(p, ctl, w, slot)) return false;
                    page = pages + (size_t)slot * kPageBytes;
                    tp = phase_begin(w);
                }
                const uint4 *row = reinterpret_cast<const uint4 *>(page + (size_t)(rr & (rpp - 1)) * row_bytes);
                float acc = 0.f;
#pragma unroll
                for (int j = 0; j < NV; ++j) {
                    const int v = tid + j * kWorkerThreads;
                    if (v < K8) acc += dot8(row[v], xr[j]);
                }
                acc2[h] = acc;
                if (((rr + 1) & (rpp - 1)) == 0 || rr + 1 == rows) {
                    release_page(ctl, w, slot);
                    phase_end(w, tp, first_page ? WS_FIRST : WS_COLS);
                    first_page = false;
                }
            }
            const float v = dual_reduce(acc2[0], acc2[1], lane);
            if (lane == 0) red[k] = v;
            if (lane == 16) red[k + 1] = v;
        }
        tp = phase_begin(w);
        if (!worker_sync(p, ctl, w)) return false;
        if (warp == 0) {
            const int e = lane & 15;                      // row within the group
            float a = 0.f, c = 0.f;
#pragma unroll
            for (int i = 0; i < kWorkerWarps; ++i) {
                a += ctl->red[w.red_buf][i][e];
                c += ctl->red[w.red_buf][i][(e + 8) & 15];
            }
            unit_epilogue(p, ctl, w, t, tile, pair, rows, a, c, resid, tok, P, best_v, best_i);
        }
        w.red_buf ^= 1;
        tile += pair ? 1 : (rows == 16 ? 2 : 1);
        phase_end(w, tp, WS_EPI);
    }
    stamp_done(p, w);
    if (kind == OP_LMHEAD && warp == 0) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, best_v, o);
            const int oi = __shfl_xor_sync(0xffffffffu, best_i, o);
            if (ov > best_v || (ov == best_v && oi < best_i)) { best_v = ov; best_i = oi; }
        }
        if (lane == 0) {
            p.amax_val[(size_t)b * p.num_lm_tasks + t.slot] = best_v;
            p.amax_idx[(size_t)b * p.num_lm_tasks + t.slot] = best_i;
        }
    }
    return true;
}

// ---------------------------------------------------------------------------
// attention task body: one chunk of positions of one q head
// ---------------------------------------------------------------------------
// Prefix K/V rows of the chunk arrive through the ring (a page holds the K
// block then the V block of up to 256 / 128 positions).  Each warp takes
// blocks of 32 positions: lanes compute the 32 scores at once (lane j reads
// K row j in a rotated chunk order, so the 8 lanes of a shared-memory phase
// hit different banks; q sits in shared memory padded the same way), the
// warp updates its online-softmax state (max, sum) with two reductions,
// and accumulates P·V with lanes over head dims.  The new position's k/v
// come from tagged words (warp 0).  The warps' states are combined through
// shared memory; a single-chunk task writes the q head's output directly,
// otherwise the chunk's (o, m, l) partial goes out tagged and chunk 0's task
// merges the partials of its q head.
template <int D>   // head_dim: 64 or 128
__device__ bool attn_task(const Params &p, const Task &t, unsigned char *pages, SmemCtl *ctl,
                          WState &w) {
    const Shape &s = p.s;
    constexpr int DPL = D / 32;   // head dims per lane in P·V
    constexpr int NCH = D / 8;    // 16-byte chunks of a K row
    constexpr int KP = DPL / 2;   // tagged pairs of the new k (and v) per lane
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const AttnChunk a = attn_chunk(p, ctl, ctl->wstep, t.begin);
    const int npp = attn_pos_per_page(D);
    if (!wait_ready(p, ctl, w)) return false;
    unsigned long long tp = phase_begin(w);
    const int npages = (a.npre + npp - 1) / npp;
    float *qs = ctl->stage + kWorkerWarps * kAttnCombine;   // q: chunk c (8 values) at qs + 12 c

    // ---- q (thread i < D/2 takes elements i and i + D/2, the pair RoPE
    // rotates together) and the new k / v (warp 0), tagged, polled until
    // fresh; RoPE at the token's position is applied here
    const bool new_warp = a.has_new && warp == 0;
    float kn[DPL], vn[DPL];
#pragma unroll
    for (int i = 0; i < DPL; ++i) { kn[i] = 0.f; vn[i] = 0.f; }
    if (a.active) {
        const uint64_t *qsrc = tag_buf(p, t.layer, p.tl.q) + (size_t)a.b * s.QD + (size_t)a.h * D;
        const uint64_t *ksrc = tag_buf(p, t.layer, p.tl.kn) + (size_t)a.b * s.KD + (size_t)a.kvh * D + lane * DPL;
        const uint64_t *vsrc = tag_buf(p, t.layer, p.tl.vn) + (size_t)a.b * s.KD + (size_t)a.kvh * D + lane * DPL;
        float q_lo = 0.f, q_hi = 0.f;
        uint32_t pend = 0;
        // bits 0, 1: this thread's q elements i, i + D/2; bits 2 .. 1+KP: new
        // k pairs; then new v pairs
        auto load = [&](int bit) {
            bool ok;
            if (bit < 2) {
                const uint64_t v = ld_tag1(qsrc + tid + (bit ? D / 2 : 0));
                if (bit) q_hi = tag_val(v); else q_lo = tag_val(v);
                ok = tag_ok(v, w.ep);
            } else {
                const bool isk = bit < 2 + KP;
                const int h = isk ? bit - 2 : bit - 2 - KP;
                const ulonglong2 v = ld_tag2((isk ? ksrc : vsrc) + 2 * h);
                float *dst = isk ? kn : vn;
                dst[2 * h] = tag_val(v.x);
                dst[2 * h + 1] = tag_val(v.y);
                ok = tag_ok(v.x, w.ep) && tag_ok(v.y, w.ep);
            }
            if (ok) pend &= ~(1u << bit);
            else pend |= 1u << bit;
        };
#pragma unroll
        for (int bit = 0; bit < 2 + 2 * KP; ++bit)
            if ((bit < 2 && tid < D / 2) || (bit >= 2 && new_warp)) load(bit);
        Spin sp;
        while (__any_sync(0xffffffffu, pend != 0u)) {
            if (!warp_spin_ok(sp, p, ctl, (uint32_t)w.task_id, 4u)) return false;
#pragma unroll
            for (int bit = 0; bit < 2 + 2 * KP; ++bit)
                if (pend & (1u << bit)) load(bit);
        }
        if (tid < D / 2) {
            const float2 cs = p.rope[(size_t)a.P * (D / 2) + tid];
            const float scale = 1.0f / sqrtf((float)D);
            const int e = tid, f = tid + D / 2;
            qs[12 * (e >> 3) + (e & 7)] = (q_lo * cs.x - q_hi * cs.y) * scale;
            qs[12 * (f >> 3) + (f & 7)] = (q_hi * cs.x + q_lo * cs.y) * scale;
        }
        if (new_warp) {
            // rotate the new key (lane L holds elements L*DPL..; the partner of
            // an element sits D/2 further, i.e. in lane L ^ 16), round it to
            // bf16 as the cache stores it; the group's first q head appends it
            uint16_t kb[DPL];
#pragma unroll
            for (int j = 0; j < DPL; ++j) {
                const float other = __shfl_xor_sync(0xffffffffu, kn[j], 16);
                const int e = lane * DPL + j;
                const int i = e % (D / 2);
                const float2 cs = p.rope[(size_t)a.P * (D / 2) + i];
                const float r = lane < 16 ? kn[j] * cs.x - other * cs.y : kn[j] * cs.x + other * cs.y;
                kb[j] = f2bf(r);
            }
#pragma unroll
            for (int j = 0; j < DPL; ++j) kn[j] = bf2f(kb[j]);
            if (a.h % s.G == 0) {
                uint16_t *kc = p.layers[t.layer].kc + (((size_t)a.b * s.nkv + a.kvh) * s.S + a.P) * D + lane * DPL;
#pragma unroll
                for (int j = 0; j < DPL; ++j) kc[j] = kb[j];
            }
        }
    }
    if (!worker_sync(p, ctl, w)) return false;   // q visible to every warp
    stamp_ready(p, w);
    phase_end(w, tp, WS_PRO);
    stamp_input(p, w);

    // l: this lane's share of the softmax sum (m is warp-uniform, so the
    // shares add up after the loop)
    float m = -INFINITY, l = 0.f, o[DPL];
#pragma unroll
    for (int i = 0; i < DPL; ++i) o[i] = 0.f;
    for (int pg = 0; pg < npages; ++pg) {
        uint32_t slot;
        if (!wait_page(p, ctl, w, slot)) return false;
        tp = phase_begin(w);
        const uint16_t *Kp = reinterpret_cast<const uint16_t *>(pages + (size_t)slot * kPageBytes);
        const uint16_t *Vp = Kp + (size_t)npp * D;
        const int n = min(npp, a.npre - pg * npp);
        for (int j0 = warp * 32; j0 < n; j0 += kWorkerWarps * 32) {
            const int j = j0 + lane;
            float sc = -INFINITY;
            if (j < n) {
                const uint4 *krow = reinterpret_cast<const uint4 *>(Kp + (size_t)j * D);
                float2 a0 = make_float2(0.f, 0.f), a1 = make_float2(0.f, 0.f);
#pragma unroll
                for (int c = 0; c < NCH; ++c) {
                    const int cc = (c + lane) & (NCH - 1);
                    const uint4 kw = krow[cc];
                    const float4 q0 = *reinterpret_cast<const float4 *>(qs + 12 * cc);
                    const float4 q1 = *reinterpret_cast<const float4 *>(qs + 12 * cc + 4);
                    a0 = ffma2(make_float2(bf_lo(kw.x), bf_hi(kw.x)), make_float2(q0.x, q0.y), a0);
                    a1 = ffma2(make_float2(bf_lo(kw.y), bf_hi(kw.y)), make_float2(q0.z, q0.w), a1);
                    a0 = ffma2(make_float2(bf_lo(kw.z), bf_hi(kw.z)), make_float2(q1.x, q1.y), a0);
                    a1 = ffma2(make_float2(bf_lo(kw.w), bf_hi(kw.w)), make_float2(q1.z, q1.w), a1);
                }
                sc = (a0.x + a0.y) + (a1.x + a1.y);
            }
            const float mn = fmaxf(m, warp_max(sc));    // finite: lane 0's position is valid
            const float corr = expf(m - mn);
            const float pe = j < n ? expf(sc - mn) : 0.f;
            l = fmaf(l, corr, pe);
            m = mn;
            const uint16_t *vb = Vp + (size_t)j0 * D + lane * DPL;
            // P·V over the block's positions, two independent sums
            float ta[DPL], tb[DPL];
#pragma unroll
            for (int i = 0; i < DPL; ++i) { ta[i] = 0.f; tb[i] = 0.f; }
            auto pv = [&](int k, float *t) {
                const float pk = __shfl_sync(0xffffffffu, pe, k);
                if constexpr (DPL == 2) {
                    const uint32_t vw = *reinterpret_cast<const uint32_t *>(vb + (size_t)k * D);
                    t[0] = fmaf(pk, bf_lo(vw), t[0]);
                    t[1] = fmaf(pk, bf_hi(vw), t[1]);
                } else {
                    const uint2 vw = *reinterpret_cast<const uint2 *>(vb + (size_t)k * D);
                    t[0] = fmaf(pk, bf_lo(vw.x), t[0]);
                    t[1] = fmaf(pk, bf_hi(vw.x), t[1]);
                    t[2] = fmaf(pk, bf_lo(vw.y), t[2]);
                    t[3] = fmaf(pk, bf_hi(vw.y), t[3]);
                }
            };
            if (j0 + 32 <= n) {
#pragma unroll
                for (int k = 0; k < 32; k += 2) { pv(k, ta); pv(k + 1, tb); }
            } else {
                const int cnt = n - j0;
                for (int k = 0; k < cnt; ++k) pv(k, ta);
            }
#pragma unroll
            for (int i = 0; i < DPL; ++i) o[i] = fmaf(o[i], corr, ta[i] + tb[i]);
        }
        release_page(ctl, w, slot);
        phase_end(w, tp, WS_DOT);
    }
    l = warp_sum(l);
    tp = phase_begin(w);
    if (new_warp) {
        float sc = 0.f;
#pragma unroll
        for (int i = 0; i < DPL; ++i) {
            const int e = lane * DPL + i;
            sc = fmaf(qs[12 * (e >> 3) + (e & 7)], kn[i], sc);
        }
        sc = warp_sum(sc);
        const float mn = fmaxf(m, sc);
        const float corr = expf(m - mn);
        const float pe = expf(sc - mn);
        l = l * corr + pe;
#pragma unroll
        for (int i = 0; i < DPL; ++i) o[i] = fmaf(o[i], corr, pe * vn[i]);
        m = mn;
    }

    // ---- combine the warps' states
    float *cw = ctl->stage + warp * kAttnCombine;
#pragma unroll
    for (int i = 0; i < DPL; ++i) cw[lane * DPL + i] = o[i];
    if (lane == 0) { cw[D] = m; cw[D + 1] = l; }
    if (!worker_sync(p, ctl, w)) return false;
    uint64_t *part = tag_buf(p, t.layer, p.tl.part) + ((size_t)a.b * s.nq + a.h) * s.NC * (D + 2);
    // chunks at or past nc hold no positions and write nothing
    if (a.active && a.c < a.nc && tid < D) {
        float M = -INFINITY;
#pragma unroll
        for (int k = 0; k < kWorkerWarps; ++k) M = fmaxf(M, ctl->stage[k * kAttnCombine + D]);
        float O = 0.f, L = 0.f;
        if (M != -INFINITY) {
#pragma unroll
            for (int k = 0; k < kWorkerWarps; ++k) {
                const float *ck = ctl->stage + k * kAttnCombine;
                const float f = expf(ck[D] - M);
                O = fmaf(f, ck[tid], O);
                L = fmaf(f, ck[D + 1], L);
            }
        }
        if (a.nc == 1) {
            st_tag_rep(tag_buf(p, t.layer, p.tl.attn) + (size_t)a.b * s.QD + (size_t)a.h * D + tid,
                       p.tl.rep_qd, O / L, w.ep_out);
        } else {
            uint64_t *dst = part + (size_t)a.c * (D + 2);
            st_tag(dst + tid, O, w.ep_out);
            if (tid == 0) {
                st_tag(dst + D, M, w.ep_out);
                st_tag(dst + D + 1, L, w.ep_out);
            }
        }
    }
    stamp_done(p, w);
    if (a.active && a.nc > 1 && a.c == 0) {
        // chunk 0's task merges its q head's partials: polls them into shared
        // memory (tagged, so it waits for exactly the chunks it reads), then
        // combines them there
        const int nc = a.nc;
        if (!worker_sync(p, ctl, w)) return false;   // the combine above is done with the stage
        if (!stage_partials(p, ctl, w, part, 1, nc * (D + 2), s.NC * (D + 2))) return false;
        if (!worker_sync(p, ctl, w)) return false;
        if (tid < D) {
            const float *sg = ctl->stage;
            float M = -INFINITY;
            for (int c = 0; c < nc; ++c) M = fmaxf(M, sg[c * (D + 2) + D]);
            float num = 0.f, den = 0.f;
            for (int c = 0; c < nc; ++c) {
                const float mc = sg[c * (D + 2) + D];
                if (mc == -INFINITY) continue;
                const float f = expf(mc - M);
                num = fmaf(f, sg[c * (D + 2) + tid], num);
                den = fmaf(f, sg[c * (D + 2) + D + 1], den);
            }
            st_tag_rep(tag_buf(p, t.layer, p.tl.attn) + (size_t)a.b * s.QD + (size_t)a.h * D + tid,
                       p.tl.rep_qd, num / den, w.ep_out);
        }
    }
    if (!worker_sync(p, ctl, w)) return false;
    if (tid == 0) signal_event(p, ctl, t);
    phase_end(w, tp, WS_ATT);
    return true;
}

// Attention item of HA q heads sharing one KV head (MK_FLAG_ATTN_KV_ITEMS,
// the default for long caches): the same chunk, pages and merge as
// attn_task, but every K row a lane reads is scored against all HA queries
// and every V row a lane reads feeds all HA outputs, so the item reads its
// KV head's positions once for the group.  The block loop keeps the
// queries in registers: a lane is a (position, dim group) pair and holds its
// group's slice of all HA queries (64 floats), so scoring reads only K rows
// from shared memory (in a rotated chunk order free of bank conflicts,
// attn_kv_rot) and the dim groups of a position add up with shuffles.  The
// warp takes the per-head maximum in one instruction, the softmax weights go
// to a per-warp slot of shared memory, and P·V broadcasts them from there
// (one vector load per position for all heads) with lanes over head dims.
// Softmax sums are kept per lane and added up once after the pages.
template <int D, int HA>   // head_dim 64 or 128; q heads per item, HA * D <= kAttnHeadDims
__device__ bool attn_kv_task(const Params &p, const Task &t, unsigned char *pages, SmemCtl *ctl,
                             WState &w) {
    const Shape &s = p.s;
    constexpr int DPL = D / 32;                  // head dims per lane in P·V
    constexpr int NCH = D / 8;                   // 16-byte chunks of a K row
    constexpr int KP = DPL / 2;                  // tagged pairs of the new k (and v) per lane
    constexpr int QST = 12 * NCH;                // floats of one head's padded query
    constexpr int QN = HA * D / 2;               // rotation pairs of the item's queries
    constexpr int QR = (QN + kWorkerThreads - 1) / kWorkerThreads;
    constexpr int CMB = HA * (D + 2);            // per-warp combine slot: o of each head, then (m, l) pairs
    constexpr int NB = 2 * QR + 2 * KP;          // pending bits of the input poll
    static_assert(HA * D <= kAttnHeadDims, "item heads fit");
    static_assert(kWorkerWarps * CMB + HA * QST + kWorkerWarps * 32 * HA <= kStageFloats, "stage");
    static_assert(NB <= 32, "poll bits");
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const AttnChunk a = attn_chunk(p, ctl, ctl->wstep, t.begin);
    const int npp = attn_pos_per_page(D);
    if (!wait_ready(p, ctl, w)) return false;
    unsigned long long tp = phase_begin(w);
    const int npages = (a.npre + npp - 1) / npp;
    float *qs = ctl->stage + kWorkerWarps * CMB;          // head hh, chunk c at qs + hh * QST + 12 c
    float *pb = qs + HA * QST + warp * 32 * HA;           // this warp's weights [32 positions][HA]

    // ---- the queries (thread i < QN takes element pair (e, e + D/2) of
    // head i / (D/2), the pair RoPE rotates together) and the new k / v
    // (warp 0), tagged, polled until fresh
    const bool new_warp = a.has_new && warp == 0;
    float kn[DPL], vn[DPL];
#pragma unroll
    for (int i = 0; i < DPL; ++i) { kn[i] = 0.f; vn[i] = 0.f; }
    if (a.active) {
        const uint64_t *qsrc = tag_buf(p, t.layer, p.tl.q) + (size_t)a.b * s.QD + (size_t)a.h * D;
        const uint64_t *ksrc = tag_buf(p, t.layer, p.tl.kn) + (size_t)a.b * s.KD + (size_t)a.kvh * D + lane * DPL;
        const uint64_t *vsrc = tag_buf(p, t.layer, p.tl.vn) + (size_t)a.b * s.KD + (size_t)a.kvh * D + lane * DPL;
        float qv[2 * QR];
#pragma unroll
        for (int i = 0; i < 2 * QR; ++i) qv[i] = 0.f;
        uint32_t pend = 0;
        auto load = [&](int bit) {
            bool ok;
            if (bit < 2 * QR) {
                const int i = tid + (bit >> 1) * kWorkerThreads;
                const int hh = i / (D / 2), e = i % (D / 2);
                const uint64_t v = ld_tag1(qsrc + hh * D + e + ((bit & 1) ? D / 2 : 0));
                qv[bit] = tag_val(v);
                ok = tag_ok(v, w.ep);
            } else {
                const int bb = bit - 2 * QR;
                const bool isk = bb < KP;
                const int h = isk ? bb : bb - KP;
                const ulonglong2 v = ld_tag2((isk ? ksrc : vsrc) + 2 * h);
                float *dst = isk ? kn : vn;
                dst[2 * h] = tag_val(v.x);
                dst[2 * h + 1] = tag_val(v.y);
                ok = tag_ok(v.x, w.ep) && tag_ok(v.y, w.ep);
            }
            if (ok) pend &= ~(1u << bit);
            else pend |= 1u << bit;
        };
#pragma unroll
        for (int bit = 0; bit < NB; ++bit)
            if (bit < 2 * QR ? tid + (bit >> 1) * kWorkerThreads < QN : new_warp) load(bit);
        Spin sp;
        while (__any_sync(0xffffffffu, pend != 0u)) {
            if (!warp_spin_ok(sp, p, ctl, (uint32_t)w.task_id, 4u)) return false;
#pragma unroll
            for (int bit = 0; bit < NB; ++bit)
                if (pend & (1u << bit)) load(bit);
        }
        const float scale = 1.0f / sqrtf((float)D);
#pragma unroll
        for (int r = 0; r < QR; ++r) {
            const int i = tid + r * kWorkerThreads;
            if (i < QN) {
                const int hh = i / (D / 2), e = i % (D / 2), f = e + D / 2;
                const float2 cs = p.rope[(size_t)a.P * (D / 2) + e];
                float *qh = qs + hh * QST;
                qh[12 * (e >> 3) + (e & 7)] = (qv[2 * r] * cs.x - qv[2 * r + 1] * cs.y) * scale;
                qh[12 * (f >> 3) + (f & 7)] = (qv[2 * r + 1] * cs.x + qv[2 * r] * cs.y) * scale;
            }
        }
        if (new_warp) {
            // rotate the new key (the partner of an element sits D/2 further,
            // in lane L ^ 16), round it to bf16 as the cache stores it; the
            // item holding the group's first q head appends it
            uint16_t kb[DPL];
#pragma unroll
            for (int j = 0; j < DPL; ++j) {
                const float other = __shfl_xor_sync(0xffffffffu, kn[j], 16);
                const int e = lane * DPL + j;
                const int i = e % (D / 2);
                const float2 cs = p.rope[(size_t)a.P * (D / 2) + i];
                const float r = lane < 16 ? kn[j] * cs.x - other * cs.y : kn[j] * cs.x + other * cs.y;
                kb[j] = f2bf(r);
            }
#pragma unroll
            for (int j = 0; j < DPL; ++j) kn[j] = bf2f(kb[j]);
            if (a.h % s.G == 0) {
                uint16_t *kc = p.layers[t.layer].kc + (((size_t)a.b * s.nkv + a.kvh) * s.S + a.P) * D + lane * DPL;
#pragma unroll
                for (int j = 0; j < DPL; ++j) kc[j] = kb[j];
            }
        }
    }
    if (!worker_sync(p, ctl, w)) return false;   // queries visible to every warp
    stamp_ready(p, w);
    phase_end(w, tp, WS_PRO);
    stamp_input(p, w);

    // ---- the block loop, queries in registers: lane (pp, g) scores
    // position pp of each pass against its NS chunks of every head (the
    // item's HA x 64-dim slice); the NG lanes of a position add up
    constexpr int NG = HA * D / 64;            // lanes per position (dim groups)
    constexpr int NS = 8 / HA;                 // 16-byte chunks per lane
    constexpr int PPI = 32 / NG;               // positions per pass
    constexpr int IT = NG;                     // passes per 32-position block
    static_assert(NG * NS == NCH && NG <= 8, "dim groups");
    constexpr int LPH = NG / HA;               // lanes per (position, head) after the reduce-scatter
    const int g = lane % NG, pp = lane / NG, hg = g / LPH;
    const int rot = attn_kv_rot(pp, g, NG, NS, D);
    float2 qr[NS][HA][4];
#pragma unroll
    for (int k = 0; k < NS; ++k) {
        const int cc = g * NS + (k + rot) % NS;
#pragma unroll
        for (int hh = 0; hh < HA; ++hh) {
            const float4 q0 = *reinterpret_cast<const float4 *>(qs + hh * QST + 12 * cc);
            const float4 q1 = *reinterpret_cast<const float4 *>(qs + hh * QST + 12 * cc + 4);
            qr[k][hh][0] = make_float2(q0.x, q0.y);
            qr[k][hh][1] = make_float2(q0.z, q0.w);
            qr[k][hh][2] = make_float2(q1.x, q1.y);
            qr[k][hh][3] = make_float2(q1.z, q1.w);
        }
    }
    float m[HA], o[HA][DPL];
    float lw = 0.f;   // lanes g % LPH == 0: this lane's share of head hg's softmax sum
#pragma unroll
    for (int hh = 0; hh < HA; ++hh) {
        m[hh] = -INFINITY;
#pragma unroll
        for (int i = 0; i < DPL; ++i) o[hh][i] = 0.f;
    }
    for (int pg = 0; pg < npages; ++pg) {
        uint32_t slot;
        if (!wait_page(p, ctl, w, slot)) return false;
        tp = phase_begin(w);
        const uint16_t *Kp = reinterpret_cast<const uint16_t *>(pages + (size_t)slot * kPageBytes);
        const uint16_t *Vp = Kp + (size_t)npp * D;
        const int n = min(npp, a.npre - pg * npp);
        for (int j0 = warp * 32; j0 < n; j0 += kWorkerWarps * 32) {
            // per pass, the NG lanes of a position reduce-scatter their
            // partial dots: lane g ends with head g / LPH's full score
            float xs[IT];
#pragma unroll
            for (int it = 0; it < IT; ++it) {
                const int j = j0 + it * PPI + pp;
                float2 acc[HA];
#pragma unroll
                for (int hh = 0; hh < HA; ++hh) acc[hh] = make_float2(0.f, 0.f);
                if (j < n) {
                    const uint4 *krow = reinterpret_cast<const uint4 *>(Kp + (size_t)j * D);
#pragma unroll
                    for (int k = 0; k < NS; ++k) {
                        const uint4 kw = krow[g * NS + (k + rot) % NS];
                        const float2 k01 = make_float2(bf_lo(kw.x), bf_hi(kw.x));
                        const float2 k23 = make_float2(bf_lo(kw.y), bf_hi(kw.y));
                        const float2 k45 = make_float2(bf_lo(kw.z), bf_hi(kw.z));
                        const float2 k67 = make_float2(bf_lo(kw.w), bf_hi(kw.w));
#pragma unroll
                        for (int hh = 0; hh < HA; ++hh) {
                            acc[hh] = ffma2(k01, qr[k][hh][0], acc[hh]);
                            acc[hh] = ffma2(k23, qr[k][hh][1], acc[hh]);
                            acc[hh] = ffma2(k45, qr[k][hh][2], acc[hh]);
                            acc[hh] = ffma2(k67, qr[k][hh][3], acc[hh]);
                        }
                    }
                }
                float v[HA];
#pragma unroll
                for (int hh = 0; hh < HA; ++hh) v[hh] = acc[hh].x + acc[hh].y;
                reduce_scatter<HA, NG / 2>(v, g);
                xs[it] = j < n ? v[0] : -INFINITY;
            }
            // head hg's block maximum: over the lane's passes, then over the
            // lanes holding the same head (other positions, twin groups)
            float mx = xs[0];
#pragma unroll
            for (int it = 1; it < IT; ++it) mx = fmaxf(mx, xs[it]);
#pragma unroll
            for (int off = 1; off < LPH; off <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
#pragma unroll
            for (int off = NG; off < 32; off <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
            float corr[HA];
            float mg = 0.f, cg = 0.f;   // head hg's new maximum and rescale
#pragma unroll
            for (int hh = 0; hh < HA; ++hh) {
                const float mn = fmaxf(m[hh], __shfl_sync(0xffffffffu, mx, hh * LPH));   // finite: position j0 is valid
                corr[hh] = expf(m[hh] - mn);
                m[hh] = mn;
                if (hg == hh) { mg = mn; cg = corr[hh]; }
            }
            // one lane per (position, head): the weights go to the warp's
            // slot for P·V, the sum stays in the lane
            if (g % LPH == 0) {
                float ls = 0.f;
#pragma unroll
                for (int it = 0; it < IT; ++it) {
                    const float pe = expf(xs[it] - mg);   // 0 for positions past n (x = -inf)
                    ls += pe;
                    pb[(it * PPI + pp) * HA + hg] = pe;
                }
                lw = fmaf(lw, cg, ls);
            }
            __syncwarp();
            const uint16_t *vb = Vp + (size_t)j0 * D + lane * DPL;
            float tv[HA][DPL];
#pragma unroll
            for (int hh = 0; hh < HA; ++hh)
#pragma unroll
                for (int i = 0; i < DPL; ++i) tv[hh][i] = 0.f;
            auto pv = [&](int k) {
                float pk[HA];
                if constexpr (HA % 4 == 0) {
#pragma unroll
                    for (int hh = 0; hh < HA; hh += 4) {
                        const float4 q = *reinterpret_cast<const float4 *>(pb + k * HA + hh);
                        pk[hh] = q.x; pk[hh + 1] = q.y; pk[hh + 2] = q.z; pk[hh + 3] = q.w;
                    }
                } else {
                    const float2 q = *reinterpret_cast<const float2 *>(pb + k * HA);
                    pk[0] = q.x; pk[1] = q.y;
                }
                float v[DPL];
                if constexpr (DPL == 2) {
                    const uint32_t vw = *reinterpret_cast<const uint32_t *>(vb + (size_t)k * D);
                    v[0] = bf_lo(vw); v[1] = bf_hi(vw);
                } else {
                    const uint2 vw = *reinterpret_cast<const uint2 *>(vb + (size_t)k * D);
                    v[0] = bf_lo(vw.x); v[1] = bf_hi(vw.x); v[2] = bf_lo(vw.y); v[3] = bf_hi(vw.y);
                }
#pragma unroll
                for (int hh = 0; hh < HA; ++hh)
#pragma unroll
                    for (int i = 0; i < DPL; ++i) tv[hh][i] = fmaf(pk[hh], v[i], tv[hh][i]);
            };
            if (j0 + 32 <= n) {
#pragma unroll
                for (int k = 0; k < 32; ++k) pv(k);
            } else {
                const int cnt = n - j0;
                for (int k = 0; k < cnt; ++k) pv(k);
            }
#pragma unroll
            for (int hh = 0; hh < HA; ++hh)
#pragma unroll
                for (int i = 0; i < DPL; ++i) o[hh][i] = fmaf(o[hh][i], corr[hh], tv[hh][i]);
            __syncwarp();   // the weights slot is rewritten by the next block
        }
        release_page(ctl, w, slot);
        phase_end(w, tp, WS_DOT);
    }
    // head h's softmax sum: the lanes of head h add up (lane h * LPH holds it)
#pragma unroll
    for (int off = NG; off < 32; off <<= 1) lw += __shfl_xor_sync(0xffffffffu, lw, off);
    float l[HA];
#pragma unroll
    for (int hh = 0; hh < HA; ++hh) l[hh] = __shfl_sync(0xffffffffu, lw, hh * LPH);
    tp = phase_begin(w);
    if (new_warp) {
#pragma unroll
        for (int hh = 0; hh < HA; ++hh) {
            float sc = 0.f;
#pragma unroll
            for (int i = 0; i < DPL; ++i) {
                const int e = lane * DPL + i;
                sc = fmaf(qs[hh * QST + 12 * (e >> 3) + (e & 7)], kn[i], sc);
            }
            sc = warp_sum(sc);
            const float mn = fmaxf(m[hh], sc);
            const float corr = expf(m[hh] - mn);
            const float pe = expf(sc - mn);
            l[hh] = l[hh] * corr + pe;
#pragma unroll
            for (int i = 0; i < DPL; ++i) o[hh][i] = fmaf(o[hh][i], corr, pe * vn[i]);
            m[hh] = mn;
        }
    }

    // ---- combine the warps' states
    float *cw = ctl->stage + warp * CMB;
#pragma unroll
    for (int hh = 0; hh < HA; ++hh) {
#pragma unroll
        for (int i = 0; i < DPL; ++i) cw[hh * D + lane * DPL + i] = o[hh][i];
        if (lane == 0) { cw[HA * D + 2 * hh] = m[hh]; cw[HA * D + 2 * hh + 1] = l[hh]; }
    }
    if (!worker_sync(p, ctl, w)) return false;
    // the partials of q head h: [NC][D + 2] at part + (b * nq + h) * NC * (D + 2)
    uint64_t *part = tag_buf(p, t.layer, p.tl.part) + ((size_t)a.b * s.nq + a.h) * s.NC * (D + 2);
    uint64_t *attn = tag_buf(p, t.layer, p.tl.attn) + (size_t)a.b * s.QD + (size_t)a.h * D;
    if (a.active && a.c < a.nc) {
        for (int i = tid; i < HA * D; i += kWorkerThreads) {
            const int hh = i / D, e = i % D;
            float M = -INFINITY;
#pragma unroll
            for (int k = 0; k < kWorkerWarps; ++k) M = fmaxf(M, ctl->stage[k * CMB + HA * D + 2 * hh]);
            float O = 0.f, L = 0.f;
            if (M != -INFINITY) {
#pragma unroll
                for (int k = 0; k < kWorkerWarps; ++k) {
                    const float *ck = ctl->stage + k * CMB;
                    const float f = expf(ck[HA * D + 2 * hh] - M);
                    O = fmaf(f, ck[hh * D + e], O);
                    L = fmaf(f, ck[HA * D + 2 * hh + 1], L);
                }
            }
            if (a.nc == 1) {
                st_tag_rep(attn + i, p.tl.rep_qd, O / L, w.ep_out);
            } else {
                uint64_t *dst = part + ((size_t)hh * s.NC + a.c) * (D + 2);
                st_tag(dst + e, O, w.ep_out);
                if (e == 0) {
                    st_tag(dst + D, M, w.ep_out);
                    st_tag(dst + D + 1, L, w.ep_out);
                }
            }
        }
    }
    stamp_done(p, w);
    if (a.active && a.nc > 1 && a.c == 0) {
        // chunk 0's item merges the partials of its q heads: polls them into
        // shared memory ([head][chunk][D + 2]; tagged, so it waits for
        // exactly the chunks it reads), then combines them there
        const int nc = a.nc;
        if (!worker_sync(p, ctl, w)) return false;   // the combine above is done with the stage
        if (!stage_partials(p, ctl, w, part, HA, nc * (D + 2), s.NC * (D + 2))) return false;
        if (!worker_sync(p, ctl, w)) return false;
        for (int i = tid; i < HA * D; i += kWorkerThreads) {
            const int hh = i / D, e = i % D;
            const float *sg = ctl->stage + (size_t)hh * nc * (D + 2);
            float M = -INFINITY;
            for (int c = 0; c < nc; ++c) M = fmaxf(M, sg[c * (D + 2) + D]);
            float num = 0.f, den = 0.f;
            for (int c = 0; c < nc; ++c) {
                const float mc = sg[c * (D + 2) + D];
                if (mc == -INFINITY) continue;
                const float f = expf(mc - M);
                num = fmaf(f, sg[c * (D + 2) + e], num);
                den = fmaf(f, sg[c * (D + 2) + D + 1], den);
            }
            st_tag_rep(attn + i, p.tl.rep_qd, num / den, w.ep_out);
        }
    }
    if (!worker_sync(p, ctl, w)) return false;
    if (tid == 0) signal_event(p, ctl, t);
    phase_end(w, tp, WS_ATT);
    return true;
}

// ---------------------------------------------------------------------------
// worker role
// ---------------------------------------------------------------------------
// KVI: the kernel instantiation with KV-head attention items (Shape::HA >
// 1); the other one holds only the q-head body, so the code of the
// short-context kernel does not grow with the long-context one's.
template <bool KVI>
__device__ bool run_task(const Params &p, const Task &t, unsigned char *pages, SmemCtl *ctl,
                         WState &w) {
    if (t.kind == OP_ATTN) {   // head_dim 64 or 128, HA * head_dim <= 512 (checked by mk_create)
        if constexpr (KVI) {
            const int ha = p.s.HA;
            if (p.s.d == 64)
                return ha == 2 ? attn_kv_task<64, 2>(p, t, pages, ctl, w)
                     : ha == 4 ? attn_kv_task<64, 4>(p, t, pages, ctl, w)
                               : attn_kv_task<64, 8>(p, t, pages, ctl, w);
            return ha == 2 ? attn_kv_task<128, 2>(p, t, pages, ctl, w) : attn_kv_task<128, 4>(p, t, pages, ctl, w);
        } else {
            return p.s.d == 64 ? attn_task<64>(p, t, pages, ctl, w) : attn_task<128>(p, t, pages, ctl, w);
        }
    }
    // Few instantiations on purpose: every body is inlined into the one
    // kernel, and more variants raise the register pressure of the whole and
    // spread the hot loop over more instruction-cache lines.
    if (rows_gemv(op_k(p.s, t.kind))) return gemv_rows<kRowK / 256>(p, t, pages, ctl, w);
    return gemv_cols<kMaxK / 2048>(p, t, pages, ctl, w);
}

// The last LM-head task of a step (warp 0 of its CTA): reduce the tasks'
// partial argmaxes to each sequence's next token; when generating, record
// it and publish the next step's input token (and whether the sequence is
// done) as tagged words.  Kept out of line: it runs once per step.
__device__ __noinline__ bool lm_reduce(const Params &p, SmemCtl *ctl, int step, uint32_t ep, int task_id) {
    const int tid = threadIdx.x;
    __threadfence();
    int nxt[kMaxBatch] = {};
    bool all_done = true;
    for (int b = 0; b < p.batch; ++b) {
        float bv = -INFINITY;
        int bi = 0x7fffffff;
        for (int k = tid; k < p.num_lm_tasks; k += 32) {
            const float v = __ldcg(p.amax_val + (size_t)b * p.num_lm_tasks + k);
            const int i = __ldcg(p.amax_idx + (size_t)b * p.num_lm_tasks + k);
            if (v > bv || (v == bv && i < bi)) { bv = v; bi = i; }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
            const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
            if (ov > bv || (ov == bv && oi < bi)) { bv = ov; bi = oi; }
        }
        if (tid == 0) {
            p.next_tok[b] = bi;
            nxt[b] = bi;
            if (p.tokens_out) {
                // while the prompt is fed the next token is the prompt's; after
                // it, the argmax.  A sequence that produced eos keeps reporting
                // eos (eos counts only once generation has begun)
                const bool prompting = step + 1 < p.n_prompt;
                const bool done_before =
                    step > 0 && __float_as_int(wait_tag1(p, ctl, p.tok_tag + 2 * b + 1, ep,
                                                         (uint32_t)task_id)) != 0;
                const bool done = done_before || (!prompting && p.eos >= 0 && bi == p.eos);
                p.tokens_out[(size_t)step * p.batch + b] = done_before ? p.eos : bi;
                all_done = all_done && done;
                if (prompting) nxt[b] = p.tokens[(size_t)(step + 1) * p.batch + b];
                if (step + 1 < p.n_steps)
                    st_tag(p.tok_tag + 2 * b + 1, __int_as_float(done ? 1 : 0), ep + 1u);
            }
        }
    }
    if (tid == 0 && p.tokens_out && step + 1 < p.n_steps)
        for (int b = 0; b < p.batch; ++b)
            st_tag(p.tok_tag + 2 * b, __int_as_float(all_done ? -1 : nxt[b]), ep + 1u);
    return true;
}

template <bool KVI>
__device__ void worker_role(const Params &p, unsigned char *pages, SmemCtl *ctl) {
    const int q0 = p.qoff[blockIdx.x], q1 = p.qoff[blockIdx.x + 1];
    const int qlen = q1 - q0;
    const int tid = threadIdx.x;
    WState w;
    if (p.sm_stats && tid == 0) {
        w.stat = ctl->wstat;
        for (int i = 0; i < kWStats; ++i) ctl->wstat[i] = 0;
    }
    const unsigned long long t_begin = phase_begin(w);
    for (int step = 0; step < p.n_steps; ++step) {
        w.ep = ctl->ep + (uint32_t)step;
        if (step > 0) {
            // this step's tokens: the previous step's argmax, published as
            // tagged words by the task that reduced it (-1: generation over);
            // warp 0 takes them into shared memory, the barrier publishes them
            if (tid < 32) {
                for (int b = 0; b < p.batch; ++b) {
                    float v;
                    if (!warp_tag1(p, ctl, w, p.tok_tag + 2 * b, true, ld_tag1(p.tok_tag + 2 * b), v)) return;
                    if (tid == 0) {
                        ctl->tok[b] = __float_as_int(v);
                        if (__float_as_int(v) < 0) *(volatile uint32_t *)&ctl->stop = 1u;
                    }
                }
                if (tid == 0) ctl->wstep = step;
            }
            if (!worker_sync(p, ctl, w)) return;
            if (*(volatile uint32_t *)&ctl->stop) break;
        }
    for (int qi = q0; qi < q1; ++qi) {
        // the task's record, published by the loader (normally well ahead)
        const int k = step * qlen + (qi - q0);
        {
            Spin sr;
            while (ld_acquire_cta_shared(&ctl->tq_pub) <= (uint32_t)k)
                if (!spin_ok(sr, p, ctl, W_READY, 0xfffffffcu, (uint32_t)k)) return;
        }
        const TaskRec &rec = ctl->tq[k % kTaskRing];
        const Task t = rec.t;
        w.gain = rec.gain;
        __syncwarp();
        if ((threadIdx.x & 31) == 0) atomicAdd(&ctl->tq_reads, 1u);
        const int id = t.sm;
        w.task_id = id;
        w.ep_out = t.trig == p.debug_withhold ? w.ep - 1u : w.ep;
        w.need = (uint32_t)(k + 1);   // the task body waits for it (counter-gated mode)
        if (!run_task<KVI>(p, t, pages, ctl, w)) return;
        const unsigned long long te = phase_begin(w);
        if (t.kind != OP_ATTN) {
            // every output of the task is written (tile epilogues by threads < 8)
            if (!worker_sync(p, ctl, w)) return;
            if (t.kind == OP_LMHEAD) {
                if (tid == 0) {
                    // after the barrier: a release that covers every thread's partials
                    const uint32_t old = atom_add_acqrel_gpu(p.lm_cnt, 1u);
                    const uint32_t last = (old + 1u == (uint32_t)p.num_lm_tasks * w.ep) ? 1u : 0u;
                    ctl->last_flag = last;
                }
                if (!worker_sync(p, ctl, w)) return;
                if (ctl->last_flag && tid < 32 && !lm_reduce(p, ctl, step, w.ep, w.task_id)) return;
            }
            if (tid == 0) signal_event(p, ctl, t);
        }
        if (p.trace && tid == 0) {
            p.trace[id].t_end = globaltimer();
            if (w.stat) {
                p.trace[id].t_wait = w.stat[WS_TASKWAIT];
                w.stat[WS_TASKWAIT] = 0;
            }
        }
        phase_end(w, te, WS_END);
        if (w.stat) w.stat[WS_TASKS] += 1;
    }
    }
    if (w.stat) {
        unsigned long long *st = p.sm_stats + (size_t)blockIdx.x * kStatSlots;
        st[ST_WORKER_FULL] = w.stat[WS_FULL];
        st[ST_WORKER_READY] = w.stat[WS_READY];
        st[ST_WORKER_SYNC] = w.stat[WS_SYNC];
        st[ST_WORKER_PROLOGUE] = w.stat[WS_PRO];
        st[ST_WORKER_DOT] = w.stat[WS_DOT];
        st[ST_WORKER_EPI] = w.stat[WS_EPI];
        st[ST_WORKER_END] = w.stat[WS_END];
        st[ST_WORKER_TASKS] = w.stat[WS_TASKS];
        st[ST_WORKER_ATTN_TAIL] = w.stat[WS_ATT];
        st[14] = w.stat[WS_FIRST];
        st[15] = w.stat[WS_COLS];
        st[ST_WORKER_TOTAL] = globaltimer() - t_begin;
    }
}

// ---------------------------------------------------------------------------
// the kernel
// ---------------------------------------------------------------------------
template <bool KVI>
__global__ void __launch_bounds__(kThreads, 1) mk_step_kernel(const __grid_constant__ Params p) {
    extern __shared__ __align__(128) unsigned char smem[];
    unsigned char *pages = smem;
    SmemCtl *ctl = reinterpret_cast<SmemCtl *>(smem + (size_t)kNumPages * kPageBytes);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    if (tid == 0) {
        for (int i = 0; i < kNumPages; ++i) {
            mbar_init(&ctl->full[i], 1);
            mbar_init(&ctl->tland[i], 1);
            mbar_init(&ctl->empty[i], kWorkerWarps);
            mbar_init(&ctl->cpdone[i], 1);
        }
        for (int i = 0; i < kTmemSlots; ++i) {
            mbar_init(&ctl->tfull[i], 1);
            mbar_init(&ctl->tempty[i], kWorkerWarps);
        }
        mbar_init(&ctl->wbar, kWorkerWarps);
        ctl->sig_post = 0;
        ctl->sig_done = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        ctl->ready_upto = 0;
        ctl->last_flag = 0;
        ctl->loader_done = 0;
        ctl->ep = ld_volatile_u32(p.epoch) + 1u;
        uint32_t stop = ld_volatile_u32(p.abort_flag) ? 1u : 0u;
        if (!stop && p.table_key && *(const volatile uint64_t *)p.table_key != p.expect_key) {
            // the shared tables were rebuilt for another shape or other
            // weights since this launch was set up: run nothing
            if (atomicCAS(&p.err->code, 0u, kErrInvalid) == 0u) {
                p.err->task = 0xffffffffu;
                p.err->where = W_INPUT;
                p.err->info = 0xfffffffeu;
            }
            stop = 1u;
        }
        ctl->tq_pub = 0;
        ctl->tq_reads = 0;
        ctl->stop = 0;
        ctl->wstep = 0;
        for (int b = 0; b < kMaxBatch; ++b) { ctl->tok[b] = 0; ctl->pos[b] = 0; }
        for (int b = 0; b < p.batch && !stop; ++b) {
            const int tok = p.tokens[b], pos = p.positions[b];
            ctl->tok[b] = tok;
            ctl->pos[b] = pos;
            bool bad = tok < 0 || tok >= p.s.V || pos < 0 || pos > p.s.S - p.n_steps;
            for (int i = 1; i < p.n_prompt && !bad; ++i) {
                const int ti = p.tokens[(size_t)i * p.batch + b];
                bad = ti < 0 || ti >= p.s.V;
            }
            if (bad) {
                if (atomicCAS(&p.err->code, 0u, kErrInvalid) == 0u) {
                    p.err->task = 0xffffffffu;
                    p.err->where = W_INPUT;
                    p.err->info = (uint32_t)b;
                }
                stop = 1u;
            }
        }
        ctl->abort = stop;
    }
    __syncthreads();
    if (ctl->abort) return;   // nothing was started
    // Tensor memory for the weight ring: the whole allocation of the SM
    // (one persistent CTA per SM, so nothing else on it holds any).  It is
    // freed at the end of the kernel, after every role has returned -- the
    // stasher only returns once its last copies have completed.
    const bool use_tmem = p.s.tmem != 0;
    if (use_tmem) {
        if (warp == kStashWarp) tmem_alloc(&ctl->tmem_base, kTmemCols);
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
    }
    if (tid == 0) {
        // the last CTA to read the epoch publishes the launch's last step's
        // epoch for the next launch (steps take epochs ep .. ep + n_steps - 1)
        const uint32_t n = (uint32_t)p.n_steps;
        const uint32_t ep_last = ctl->ep + n - 1u;
        const uint32_t old = atomicAdd(p.done_cnt, n);
        if (old + n == gridDim.x * ep_last) atomicExch(p.epoch, ep_last);
    }
    if (warp < kWorkerWarps) {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kWorkerRegs));
        worker_role<KVI>(p, pages, ctl);
    } else {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kControlRegs));
        if (warp == kLoaderWarp) {
            if (lane == 0) loader_role(p, pages, ctl);
        } else if (warp == kSchedWarp) {
            if (lane == 0 && p.event_wait) scheduler_role(p, ctl, ctl->ep);
        } else if (warp == kStashWarp) {
            if (lane == 0 && use_tmem) stasher_role(p, pages, ctl);
        } else {
            if (lane == 0) signaler_role(p, ctl);
        }
    }
    if (use_tmem) {
        tc_fence_before();
        __syncthreads();
        if (warp == kStashWarp) {
            tc_fence_after();
            tmem_dealloc(ctl->tmem_base, kTmemCols);
        }
    }
}

// ---------------------------------------------------------------------------
// host-side launch helpers (called from mk_runtime.cpp)
// ---------------------------------------------------------------------------
size_t kernel_smem_bytes() { return kSmemBytes; }

// Registers per thread the kernel was compiled to launch with; the register
// split (setmaxnreg) is only valid when this equals kLaunchRegs.
int kernel_launch_regs() {
    cudaFuncAttributes a, b;
    if (cudaFuncGetAttributes(&a, mk_step_kernel<false>) != cudaSuccess) return -1;
    if (cudaFuncGetAttributes(&b, mk_step_kernel<true>) != cudaSuccess) return -1;
    return a.numRegs == b.numRegs ? a.numRegs : -1;
}

cudaError_t kernel_prepare() {
    cudaError_t e = cudaFuncSetAttribute(mk_step_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kSmemBytes);
    if (e != cudaSuccess) return e;
    return cudaFuncSetAttribute(mk_step_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)kSmemBytes);
}

cudaError_t kernel_occupancy(int *blocks_per_sm) {
    int a = 0, b = 0;
    cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&a, mk_step_kernel<false>, kThreads, kSmemBytes);
    if (e == cudaSuccess)
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, mk_step_kernel<true>, kThreads, kSmemBytes);
    *blocks_per_sm = a < b ? a : b;
    return e;
}

// Weights of a GEMV op into the TMEM page order (see tmem_page_src): `src`
// is the row-major matrix viewed as `page_rows` rows of 2048 bf16, `dst`
// receives ceil(page_rows / 16) whole 64 KB pages (rows past the end of a
// trailing partial page are zero).  Set-up only (mk_create).
__global__ void repack_tmem_pages_kernel(uint4 *dst, const uint4 *src, long long page_rows, long long total) {
    for (long long u = (long long)blockIdx.x * blockDim.x + threadIdx.x; u < total;
         u += (long long)gridDim.x * blockDim.x) {
        int row, vec;
        tmem_page_src((int)(u & 4095), row, vec);
        const long long pr = (u >> 12) * 16 + row;
        dst[u] = pr < page_rows ? src[pr * 256 + vec] : make_uint4(0u, 0u, 0u, 0u);
    }
}

size_t tmem_pages_bytes(long long page_rows) { return (size_t)((page_rows + 15) / 16) * kPageBytes; }

cudaError_t repack_tmem_pages(void *dst, const void *src, long long page_rows, cudaStream_t stream) {
    const long long total = (long long)(tmem_pages_bytes(page_rows) / 16);
    const long long blocks = (total + 255) / 256;
    repack_tmem_pages_kernel<<<(unsigned)(blocks < 8192 ? blocks : 8192), 256, 0, stream>>>(
        static_cast<uint4 *>(dst), static_cast<const uint4 *>(src), page_rows, total);
    return cudaGetLastError();
}

cudaError_t kernel_launch(const Params &p, int grid, cudaStream_t stream) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = kSmemBytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return p.s.HA > 1 ? cudaLaunchKernelEx(&cfg, mk_step_kernel<true>, p)
                      : cudaLaunchKernelEx(&cfg, mk_step_kernel<false>, p);
}

}  // namespace mk
