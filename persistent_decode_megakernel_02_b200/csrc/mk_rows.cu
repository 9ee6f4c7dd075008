// mk_rows.cu -- the batched ("rows") decode step on tcgen05 tensor cores.
//
// One persistent CTA per SM runs a static queue of tasks (mk_rows_graph.cpp)
// for every kernel step of the launch.  A kernel step processes up to kRows
// rows -- tokens of independent sequences (a batch), or consecutive tokens of
// one sequence (a prompt) -- so every matrix op is a contraction of the
// weights with kRows input vectors, which this kernel runs on the tensor
// cores: the Hazy megakernel page (sfrk.com.cn/ruanjian/202506/86466, the
// paragraph on the asynchronous-barrier measurements) notes that Blackwell
// favours tensor cores, and the MPK news summary (qian.cx, closing roadmap
// paragraph) names mixed batching as the next step.
//
// Roles of a CTA (12 warps):
//  * loader (warp 8, one thread): streams the weight pages of the SM's GEMV
//    tasks (128 x 128 bf16 in the tcgen05 canonical layout, 32 KB each) and
//    the cached K/V positions of its attention items into a ring of
//    kRStages shared-memory pages, ahead of every dependency.
//  * scheduler (warp 9, one thread): gates the embedding and attention
//    tasks on their dependency's event counter (counter >= threshold x
//    epoch, MPK's event model, the "显著提升小LLM的性能..." page, Figure 3
//    text), publishes every task to the compute warps, and for a GEMV task
//    streams the activation slab that goes with every weight page (the bf16
//    high and low halves of the kRows input vectors, 128 columns, 8 KB) into
//    a second ring -- each slab as soon as its own writers have released it
//    (a counter per input slab: the producing op's tile, or the attention
//    items of its heads), so an op's first pages overlap the tail of the op
//    before it instead of waiting for all of it.
//  * MMA issuer (warp 10, one thread; the warp owns the tensor memory):
//    per page, 8 tcgen05.mma (M = 128, N = 2 kRows, K = 16) into an fp32
//    accumulator in tensor memory; a commit frees the page and the slab, and
//    another hands a finished tile segment to the epilogue.  Two
//    accumulators alternate so the epilogue of one segment overlaps the
//    contraction of the next.
//  * compute warps (0-7): the epilogues (warps 0-3, one TMEM lane -- one
//    weight row -- per thread: RMSNorm scale, RoPE and the KV append, the
//    residual adds, SiLU(gate) * up, the LM head's logits and argmax), the
//    attention items (all 8 warps) and the embedding.
//  * signaler (warp 11, one thread): bumps the event counter of every
//    finished task (release), off the compute warps' path.
// A tile whose pages were split over several SMs is summed in global memory
// (vector atomic adds); the SM that adds its last page finishes it.
//
// Every wait is bounded by timeout_ns: on expiry the CTA records
// MK_ERR_TIMEOUT, raises the abort flag every wait polls, lets its copies
// and contractions complete, frees its tensor memory and returns.
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <math.h>
#include <stddef.h>
#include <stdint.h>

#include "mk_rows.h"
#include "mk_ptx.cuh"

namespace mk {
namespace rows {

constexpr uint32_t kErrInvalid = 1, kErrTimeout = 3;
enum Where : uint32_t { W_DEP = 1, W_READY = 2, W_FULL = 3, W_EMPTY = 4, W_BAR = 5, W_INPUT = 6,
                        W_ACC = 7, W_TAG = 8 };

constexpr int kComputeWarps = 8;
constexpr int kEpiWarps = 4;          // one TMEM lane quarter each
constexpr int kLoaderWarp = 8, kSchedWarp = 9, kMmaWarp = 10, kSigWarp = 11;
constexpr int kThreads = 12 * 32;
constexpr int kSigRing = 64;
constexpr int kMaxGD = 512;           // G * head_dim the attention scratch holds
constexpr int kAttnSlot = kMaxGD + 16;

struct __align__(16) Ctl {
    // weight / KV page ring: a page lands on full_m (pages the MMA reads) or
    // full_c (pages the compute warps read) and is released through empty_m
    // (the MMA's commit) or empty_c (the compute warps) -- one barrier per
    // consumer, so no consumer can find its barrier two phases behind
    uint64_t full_m[kRStages], full_c[kRStages], empty_m[kRStages], empty_c[kRStages];
    uint64_t bfull[kRStages], bempty[kRStages];   // activation slab ring (MMA only)
    uint64_t accfull[2], accempty[2];             // TMEM accumulators
    uint64_t cbar, ebar;                          // compute-warp and epilogue-warp barriers
    uint32_t tmem_base;
    uint32_t abort, stop;
    uint32_t ep;                                  // epoch of the launch's first step
    uint32_t ready_upto;                          // tasks the scheduler has released
    uint32_t sig_post, sig_done, sig_ev[kSigRing];
    uint32_t last_flag;
    float rs[kRows];                              // 1/rms of every row's op input
    float bestv[kRows];                           // LM task: best logit per row so far
    int32_t besti[kRows];
    // cross-warp sums and argmaxes of a tile's epilogue, double-buffered: a
    // warp may start the next tile's before warp 0 has read this one's
    float redv[2][kComputeWarps][kRows];
    int32_t redi[2][kComputeWarps][kRows];
    // epilogue exchange (RoPE partner rows, gate/up pairs) and attention
    // scratch share one area: a CTA runs one task at a time
    union __align__(16) {
        float xbuf[kRTile][kRows + 1];
        struct {
            float q[kMaxGD];                      // G query heads, head-major
            float st[kComputeWarps][kAttnSlot];   // per-warp G x (d output, m, l)
            float4 pw[kComputeWarps][32];         // per warp: a block's softmax weights, 4 heads per position
        } at;
    };
};
constexpr size_t kRingBytes = (size_t)kRStages * (kRPageBytes + kRSlabBytes);
constexpr size_t kSmem = kRingBytes + sizeof(Ctl);
static_assert(kSmem <= 227 * 1024, "shared memory budget");

// ---------------------------------------------------------------------------
// bounded waiting
// ---------------------------------------------------------------------------
struct Spin {
    unsigned long long t0 = 0;
    uint32_t n = 0;
};

__device__ void raise_error(const RParams &p, Ctl *c, uint32_t code, uint32_t where, uint32_t task,
                            uint32_t info) {
    if (atomicCAS(&p.err->code, 0u, code) == 0u) {
        p.err->task = task;
        p.err->where = where;
        p.err->info = info;
    }
    *(volatile uint32_t *)&c->abort = 1;
    atomicExch(p.abort_flag, 1u);
    __threadfence();
}

__device__ __forceinline__ bool spin_ok(Spin &s, const RParams &p, Ctl *c, uint32_t where, uint32_t task,
                                        uint32_t info) {
    if ((++s.n & 127u) != 0u) return true;
    if (*(volatile uint32_t *)&c->abort) return false;
    if (ld_volatile_u32(p.abort_flag)) {
        *(volatile uint32_t *)&c->abort = 1;
        return false;
    }
    const unsigned long long now = globaltimer();
    if (s.t0 == 0) {
        s.t0 = now;
        return true;
    }
    if (now - s.t0 > p.timeout_ns) {
        raise_error(p, c, kErrTimeout, where, task, info);
        return false;
    }
    return true;
}

__device__ __forceinline__ bool wait_bar(uint64_t *bar, uint32_t parity, const RParams &p, Ctl *c,
                                         uint32_t where, uint32_t task) {
    Spin s;
    while (!mbar_try_wait(bar, parity))
        if (!spin_ok(s, p, c, where, task, parity)) return false;
    return true;
}

// wait_bar that adds the time waited to *acc (trace mode; acc null: plain).
__device__ __forceinline__ bool wait_bar_t(uint64_t *bar, uint32_t parity, const RParams &p, Ctl *c,
                                           uint32_t where, uint32_t task, unsigned long long *acc) {
    if (!acc) return wait_bar(bar, parity, p, c, where, task);
    const unsigned long long t0 = globaltimer();
    const bool ok = wait_bar(bar, parity, p, c, where, task);
    *acc += globaltimer() - t0;
    return ok;
}
__device__ __forceinline__ unsigned long long *stat_slot(const RParams &p, int which) {
    return p.sm_stats ? p.sm_stats + (size_t)blockIdx.x * kRStats + which : nullptr;
}

// A barrier among `warps` warps (an mbarrier with that many arrivals, one
// per warp): bounded, unlike bar.sync, so a warp that gave up on a wait
// cannot leave the others blocked.
__device__ __forceinline__ bool group_sync(uint64_t *bar, uint32_t &phase, const RParams &p, Ctl *c,
                                           uint32_t task) {
    __syncwarp();
    if ((threadIdx.x & 31) == 0) mbar_arrive(bar);
    const bool ok = wait_bar_t(bar, phase, p, c, W_BAR, task, threadIdx.x == 0 ? stat_slot(p, RS_CMP_SYNC) : nullptr);
    phase ^= 1u;
    return ok;
}

// ---------------------------------------------------------------------------
// task geometry, identical in every role
// ---------------------------------------------------------------------------
__device__ __forceinline__ bool is_gemv(int kind) {
    return kind == ROP_QKV || kind == ROP_OPROJ || kind == ROP_GATEUP || kind == ROP_DOWN || kind == ROP_LMHEAD;
}
// The LM head runs in the steps that produce outputs only (a prompt's last).
__device__ __forceinline__ bool task_on(const RParams &p, const Task &t, int step) {
    return t.kind != ROP_LMHEAD || step >= p.lm_from;
}

struct Item {       // one attention item: row r, KV head h, chunk c
    int r, h, c;
    bool active;
    int P, slot;
    int c0, c1;     // positions [c0, c1) of the chunk
    int nring;      // positions [c0, c0 + nring) come through the page ring (written before the launch)
    int nc;         // chunks holding positions for this row
};

__device__ __forceinline__ Item attn_item(const RParams &p, int step, int item) {
    const Shape &s = p.s;
    Item a;
    a.r = item / (s.nkv * s.NC);
    a.h = (item / s.NC) % s.nkv;
    a.c = item % s.NC;
    a.active = a.r < rrows_in_step(p, step);
    a.P = 0; a.slot = 0; a.c0 = 0; a.c1 = 0; a.nring = 0; a.nc = 0;
    if (a.active) {
        const RRow rw = rrow(p, step, a.r);
        a.P = rw.pos;
        a.slot = rw.slot;
        const int C = a.P + 1;
        const int nc = min(s.NC, (C + kRAttnChunk - 1) / kRAttnChunk);
        const int Lc = (C + nc - 1) / nc;
        a.nc = nc;
        a.c0 = a.c * Lc;
        a.c1 = min(a.c0 + Lc, C);
        if (a.c0 >= C) { a.c0 = C; a.c1 = C; }
        a.nring = max(0, min(a.c1, rw.pre) - a.c0);
    }
    return a;
}

__device__ __forceinline__ int attn_pages(const RParams &p, const Item &a) {
    const int npp = rattn_pos_per_page(p.s.d);
    return (a.nring + npp - 1) / npp;
}

__device__ __forceinline__ const uint16_t *gemv_weights(const RParams &p, const Task &t) {
    if (t.kind == ROP_LMHEAD) return p.lm;
    const RLayerW &L = p.layers[t.layer];
    return t.kind == ROP_QKV ? L.qkv : t.kind == ROP_OPROJ ? L.wo : t.kind == ROP_GATEUP ? L.gu : L.wd;
}
__device__ __forceinline__ const uint16_t *gemv_input(const RParams &p, const Task &t) {
    if (t.kind == ROP_LMHEAD) return p.xlm;
    const RLayerBuf &B = p.buf[t.layer];
    return t.kind == ROP_QKV ? B.xq : t.kind == ROP_OPROJ ? B.xo : t.kind == ROP_GATEUP ? B.xg : B.xd;
}

// ---------------------------------------------------------------------------
// loader: weight pages and cached K/V into the page ring
// ---------------------------------------------------------------------------
struct Ring {
    uint32_t seq = 0;
    uint32_t via_m = 0;     // bit s: slot s's last page is the MMA's
    uint32_t odd_m = 0;     // bit s: MMA pages placed in slot s so far, mod 2
    uint32_t odd_c = 0;     // bit s: compute pages placed in slot s so far, mod 2
};

__device__ __forceinline__ bool ring_acquire(const RParams &p, Ctl *c, Ring &r, uint32_t bytes, bool for_mma,
                                             uint32_t task, uint32_t &slot, uint64_t *&bar) {
    slot = r.seq % kRStages;
    if (r.seq >= (uint32_t)kRStages) {
        const bool prev_m = (r.via_m >> slot) & 1u;
        const uint32_t par = (((prev_m ? r.odd_m : r.odd_c) >> slot) & 1u) ^ 1u;
        if (!wait_bar_t(prev_m ? &c->empty_m[slot] : &c->empty_c[slot], par, p, c, W_EMPTY, task,
                        stat_slot(p, RS_LOAD_SLOT)))
            return false;
    }
    if (for_mma) { r.via_m |= 1u << slot; r.odd_m ^= 1u << slot; }
    else { r.via_m &= ~(1u << slot); r.odd_c ^= 1u << slot; }
    bar = for_mma ? &c->full_m[slot] : &c->full_c[slot];
    mbar_arrive_expect_tx(bar, bytes);
    ++r.seq;
    return true;
}

__device__ void loader_role(const RParams &p, unsigned char *ring, Ctl *c) {
    const int q0 = p.qoff[blockIdx.x], q1 = p.qoff[blockIdx.x + 1];
    const unsigned long long t_begin = p.sm_stats ? globaltimer() : 0ull;
    const uint64_t pol = policy_evict_first();
    const int npp = rattn_pos_per_page(p.s.d);
    Ring rg;
    bool ok = true;
    for (int step = 0; step < p.n_steps && ok; ++step)
    for (int qi = q0; qi < q1 && ok; ++qi) {
        const Task t = p.qtasks[qi];
        if (is_gemv(t.kind)) {
            if (!task_on(p, t, step)) continue;
            const char *w = reinterpret_cast<const char *>(gemv_weights(p, t));
            for (int pg = t.begin; pg < t.end; ++pg) {
                uint32_t slot;
                uint64_t *bar;
                if (!ring_acquire(p, c, rg, kRPageBytes, true, (uint32_t)t.sm, slot, bar)) { ok = false; break; }
                bulk_g2s_hint(ring + (size_t)slot * kRPageBytes, w + (size_t)pg * kRPageBytes, kRPageBytes, bar, pol);
            }
        } else if (t.kind == ROP_ATTN) {
            const Item a = attn_item(p, step, t.begin);
            const RLayerW &L = p.layers[t.layer];
            const size_t head = ((size_t)a.slot * p.s.nkv + a.h) * p.s.S;
            for (int p0 = a.c0; p0 < a.c0 + a.nring; p0 += npp) {
                const int n = min(npp, a.c0 + a.nring - p0);
                const uint32_t bytes = (uint32_t)n * p.s.d * 2;
                uint32_t slot;
                uint64_t *bar;
                if (!ring_acquire(p, c, rg, 2 * bytes, false, (uint32_t)t.sm, slot, bar)) { ok = false; break; }
                unsigned char *dst = ring + (size_t)slot * kRPageBytes;
                const size_t off = (head + p0) * p.s.d;
                bulk_g2s(dst, L.kc + off, bytes, bar);
                bulk_g2s(dst + (size_t)npp * p.s.d * 2, L.vc + off, bytes, bar);
            }
        }
    }
    if (p.sm_stats) *stat_slot(p, RS_LOAD_TOTAL) = globaltimer() - t_begin;
    // let every copy issued land before the CTA can exit
    const uint32_t used = rg.seq < (uint32_t)kRStages ? rg.seq : (uint32_t)kRStages;
    for (uint32_t sl = 0; sl < used; ++sl) {
        const bool m = (rg.via_m >> sl) & 1u;
        uint64_t *bar = m ? &c->full_m[sl] : &c->full_c[sl];
        const uint32_t par = (((m ? rg.odd_m : rg.odd_c) >> sl) & 1u) ^ 1u;
        Spin s;
        while (!mbar_try_wait(bar, par)) {
            if ((++s.n & 127u) == 0u) {
                const unsigned long long now = globaltimer();
                if (s.t0 == 0) s.t0 = now;
                else if (now - s.t0 > p.timeout_ns) break;
            }
        }
    }
}

// ---------------------------------------------------------------------------
// scheduler: event gating, activation slabs
// ---------------------------------------------------------------------------
__device__ void sched_role(const RParams &p, unsigned char *slabs, Ctl *c) {
    const int q0 = p.qoff[blockIdx.x], q1 = p.qoff[blockIdx.x + 1];
    const int qlen = q1 - q0;
    uint32_t bseq = 0;
    for (int step = 0; step < p.n_steps; ++step) {
        const uint32_t ep = c->ep + (uint32_t)step;
        for (int qi = q0; qi < q1; ++qi) {
            const Task t = p.qtasks[qi];
            const bool gemv = is_gemv(t.kind);
            if (!gemv) {
                // embedding (the first op of a step waits for the previous
                // step's last) and attention: the whole dependency op
                const uint32_t target = p.thresholds[t.dep] * (t.kind == ROP_EMBED ? ep - 1u : ep);
                Spin s;
                const unsigned long long td = p.sm_stats ? globaltimer() : 0ull;
                while ((int32_t)(ld_acquire_gpu(&p.events[t.dep]) - target) < 0)
                    if (!spin_ok(s, p, c, W_DEP, (uint32_t)t.sm, (uint32_t)t.dep)) return;
                if (p.sm_stats) *stat_slot(p, RS_SCHED_DEP) += globaltimer() - td;
                // what the producers wrote is read by the compute warps
                asm volatile("fence.proxy.async.global;" ::: "memory");
            }
            // a GEMV task's compute warps only read what its accumulators
            // depend on (through the slabs below) and what the producers of
            // those slabs' inputs wrote before them, so they start at once
            if (p.trace) p.trace[t.sm].t_ready = globaltimer();
            st_release_cta_shared(&c->ready_upto, (uint32_t)(step * qlen + (qi - q0) + 1));
            if (!gemv || !task_on(p, t, step)) continue;
            const RGemv g = rgemv(p.s, t.kind);
            const char *x = reinterpret_cast<const char *>(gemv_input(p, t));
            const uint32_t *rdy = t.kind == ROP_LMHEAD ? p.rdy_lm : p.buf[t.layer].rdy[rgemv_slot(t.kind)];
            const uint32_t need = rslab_writers(p.s, t.kind) * ep;
            for (int pg = t.begin; pg < t.end; ++pg, ++bseq) {
                const uint32_t slot = bseq % kRStages;
                if (bseq >= (uint32_t)kRStages &&
                    !wait_bar_t(&c->bempty[slot], ((bseq / kRStages) - 1u) & 1u, p, c, W_EMPTY, (uint32_t)t.sm,
                                stat_slot(p, RS_SCHED_SLAB)))
                    return;
                {
                    // the page's input slab is written (all its writers released)
                    Spin s;
                    const unsigned long long td = p.sm_stats ? globaltimer() : 0ull;
                    while ((int32_t)(ld_acquire_gpu(&rdy[pg % g.slabs]) - need) < 0)
                        if (!spin_ok(s, p, c, W_DEP, (uint32_t)t.sm, (uint32_t)(pg % g.slabs))) return;
                    if (p.sm_stats) *stat_slot(p, RS_SCHED_DEP) += globaltimer() - td;
                    asm volatile("fence.proxy.async.global;" ::: "memory");
                }
                mbar_arrive_expect_tx(&c->bfull[slot], kRSlabBytes);
                bulk_g2s(slabs + (size_t)slot * kRSlabBytes, x + (size_t)(pg % g.slabs) * kRSlabBytes, kRSlabBytes,
                         &c->bfull[slot]);
            }
        }
    }
    // the slab copies land before the CTA can exit: the MMA issuer waits
    // for every one of them, and the kernel ends after it
}

// ---------------------------------------------------------------------------
// MMA issuer
// ---------------------------------------------------------------------------
// Instruction descriptor of tcgen05.mma kind::f16: fp32 accumulator, bf16 A
// and B, both K-major, N = kRowsN, M = 128.
constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(kRowsN >> 3) << 17) | (8u << 24);

__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(kIdesc), "r"(accumulate)
        : "memory");
}

// Segments of a GEMV task: maximal runs of its pages within one tile.
__device__ __forceinline__ int seg_end(int pg, int end, int slabs) {
    const int tile_end = (pg / slabs + 1) * slabs;
    return tile_end < end ? tile_end : end;
}

__device__ void mma_role(const RParams &p, unsigned char *ring, unsigned char *slabs, Ctl *c) {
    const int q0 = p.qoff[blockIdx.x], q1 = p.qoff[blockIdx.x + 1];
    const unsigned long long t_begin = p.sm_stats ? globaltimer() : 0ull;
    uint32_t aseq = 0, odd_m = 0, bseq = 0, segs = 0;
    bool ok = true;
    for (int step = 0; step < p.n_steps && ok; ++step)
    for (int qi = q0; qi < q1 && ok; ++qi) {
        const Task t = p.qtasks[qi];
        if (t.kind == ROP_ATTN) {
            aseq += (uint32_t)attn_pages(p, attn_item(p, step, t.begin));
            continue;
        }
        if (!is_gemv(t.kind) || !task_on(p, t, step)) continue;
        if (p.trace) p.trace[t.sm].t_wait = globaltimer();
        const RGemv g = rgemv(p.s, t.kind);
        for (int pg = t.begin; pg < t.end && ok;) {
            const int pe = seg_end(pg, t.end, g.slabs);
            const uint32_t acc = segs & 1u;
            if (segs >= 2u && !wait_bar_t(&c->accempty[acc], ((segs >> 1) - 1u) & 1u, p, c, W_ACC, (uint32_t)t.sm,
                                          stat_slot(p, RS_MMA_ACC))) {
                ok = false;
                break;
            }
            tc_fence_after();
            const uint32_t dt = c->tmem_base + acc * kRAccCols;
            for (int q = pg; q < pe; ++q) {
                const uint32_t as = aseq % kRStages, bs = bseq % kRStages;
                if (!wait_bar_t(&c->full_m[as], (odd_m >> as) & 1u, p, c, W_FULL, (uint32_t)t.sm,
                                stat_slot(p, RS_MMA_PAGE)) ||
                    !wait_bar_t(&c->bfull[bs], (bseq / kRStages) & 1u, p, c, W_FULL, (uint32_t)t.sm,
                                stat_slot(p, RS_MMA_SLAB))) {
                    ok = false;
                    break;
                }
                odd_m ^= 1u << as;
                ++aseq;
                ++bseq;
                tc_fence_after();
                const unsigned char *A = ring + (size_t)as * kRPageBytes;
                const unsigned char *B = slabs + (size_t)bs * kRSlabBytes;
#pragma unroll
                for (int kk = 0; kk < kRSlab / 16; ++kk)
                    mma_bf16(dt, smem_desc(A + kk * 4096, 2048, 128), smem_desc(B + kk * 1024, 512, 128),
                             (q > pg || kk > 0) ? 1u : 0u);
                tc_commit(&c->empty_m[as]);
                tc_commit(&c->bempty[bs]);
            }
            if (!ok) break;
            tc_commit(&c->accfull[acc]);
            ++segs;
            pg = pe;
        }
    }
    if (p.sm_stats) *stat_slot(p, RS_MMA_TOTAL) = globaltimer() - t_begin;
    // every contraction issued has completed before tensor memory is freed:
    // the last commit arrives only after all earlier tcgen05 operations
    if (segs > 0) {
        const uint32_t acc = (segs - 1) & 1u, par = ((segs - 1) >> 1) & 1u;
        Spin s;
        while (!mbar_try_wait(&c->accfull[acc], par)) {
            if ((++s.n & 127u) == 0u) {
                const unsigned long long now = globaltimer();
                if (s.t0 == 0) s.t0 = now;
                else if (now - s.t0 > p.timeout_ns) break;
            }
        }
    }
}

// ---------------------------------------------------------------------------
// signaler
// ---------------------------------------------------------------------------
__device__ void signaler_role(const RParams &p, Ctl *c) {
    const uint32_t total = (uint32_t)(p.qoff[blockIdx.x + 1] - p.qoff[blockIdx.x]) * (uint32_t)p.n_steps;
    uint32_t done = 0;
    while (done < total) {
        Spin s;
        uint32_t posted;
        while ((posted = ld_acquire_cta_shared(&c->sig_post)) == done)
            if (!spin_ok(s, p, c, W_READY, 0xfffffffeu, done)) return;
        for (; done < posted; ++done) red_release_gpu(&p.events[c->sig_ev[done % kSigRing]], 1u);
        *(volatile uint32_t *)&c->sig_done = done;
    }
}

__device__ __forceinline__ bool post_done(const RParams &p, Ctl *c, const Task &t) {
    const uint32_t n = c->sig_post;
    Spin s;
    while (n - *(volatile uint32_t *)&c->sig_done >= (uint32_t)kSigRing)
        if (!spin_ok(s, p, c, W_READY, 0xfffffffdu, n)) return false;
    c->sig_ev[n % kSigRing] = (uint32_t)t.trig;
    st_release_cta_shared(&c->sig_post, n + 1u);
    return true;
}

// ---------------------------------------------------------------------------
// compute warps
// ---------------------------------------------------------------------------
struct CState {
    uint32_t aseq = 0, odd_c = 0;   // page ring position, parity of the next full_c wait per slot
    uint32_t segs = 0;              // accumulator segments consumed
    uint32_t cph = 0, eph = 0;      // compute / epilogue barrier phases
    uint32_t rb = 0;                // reduction buffer of the next tile epilogue
    uint32_t ep = 0;                // the step's epoch
    int step = 0;
    int task_id = 0;
};

__device__ __forceinline__ float ldcg(const float *p) { return __ldcg(p); }

__device__ __forceinline__ void st_split(uint16_t *x, int r, int k, float v) {
    const __nv_bfloat16 hi = __float2bfloat16_rn(v);
    const __nv_bfloat16 lo = __float2bfloat16_rn(v - __bfloat162float(hi));
    x[rx_elem(r, k)] = __bfloat16_as_ushort(hi);
    x[rx_elem(kRows + r, k)] = __bfloat16_as_ushort(lo);
}

// Sum over the 128 epilogue threads of v[r] for every row r; thread r < kRows
// of warp 0 ends up with row r's total in `out` (others: undefined).
__device__ __forceinline__ bool epi_rowsum(const RParams &p, Ctl *c, CState &cs, const float (&v)[kRows],
                                           float &out) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rb = cs.rb;
    cs.rb ^= 1u;
#pragma unroll
    for (int r = 0; r < kRows; ++r) {
        float x = v[r];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
        if (lane == 0) c->redv[rb][warp][r] = x;
    }
    if (!group_sync(&c->ebar, cs.eph, p, c, (uint32_t)cs.task_id)) return false;
    out = 0.f;
    if (threadIdx.x < kRows)
        for (int w = 0; w < kEpiWarps; ++w) out += c->redv[rb][w][threadIdx.x];
    return true;
}

// 1/rms of every row of the op's input, from the producing op's per-tile
// sums of squares [H / 128][kRows], into c->rs (epilogue threads).
__device__ __forceinline__ bool load_rs(const RParams &p, Ctl *c, CState &cs, const float *ss) {
    if (threadIdx.x < kRows) {
        float t = 0.f;
        for (int i = 0; i < p.s.H / kRTile; ++i) t += ldcg(ss + (size_t)i * kRows + threadIdx.x);
        c->rs[threadIdx.x] = 1.0f / sqrtf(t / (float)p.s.H + p.s.eps);
    }
    return group_sync(&c->ebar, cs.eph, p, c, (uint32_t)cs.task_id);
}

// A new residual-stream column R (= hidden index) for every row: stored in
// fp32, as the next op's bf16 high/low input with its RMSNorm gain folded in,
// and summed into the per-tile sums of squares of the next RMSNorm.
__device__ __forceinline__ bool resid_out(const RParams &p, Ctl *c, CState &cs, int tile, int m,
                                          const float (&x)[kRows], int nrows, float *x_out, uint16_t *x_next,
                                          const uint16_t *gain, float *ss_out, uint32_t *rdy_next) {
    const int R = tile * kRTile + m;
    const float g = __bfloat162float(__ushort_as_bfloat16(gain[R]));
    float sq[kRows];
#pragma unroll
    for (int r = 0; r < kRows; ++r) {
        const bool on = r < nrows;
        if (on) x_out[(size_t)r * p.s.H + R] = x[r];
        st_split(x_next, r, R, on ? x[r] * g : 0.f);
        sq[r] = on ? x[r] * x[r] : 0.f;
    }
    // the slab is read by bulk copies (the async proxy) on other SMs
    asm volatile("fence.proxy.async.global;" ::: "memory");
    float tot;
    if (!epi_rowsum(p, c, cs, sq, tot)) return false;
    if (threadIdx.x < kRows) ss_out[(size_t)tile * kRows + threadIdx.x] = tot;
    // slab `tile` of the next op's input is written (every thread's part
    // before the barrier in epi_rowsum, the row sums before the warp sync):
    // one release lets that op's pages on it start
    __syncwarp();
    if (threadIdx.x == 0) red_release_gpu(rdy_next + tile, 1u);
    return true;
}

__device__ __forceinline__ float silu(float g) { return g / (1.0f + expf(-g)); }

// The epilogue of a finished tile: y[r] = the tile's row m (this thread's)
// of the contraction with row r's input.
__device__ bool tile_epilogue(const RParams &p, Ctl *c, CState &cs, const Task &t, int tile, float (&y)[kRows]) {
    const Shape &s = p.s;
    const int m = threadIdx.x;
    const int nrows = rrows_in_step(p, cs.step);
    switch (t.kind) {
    case ROP_QKV: {
        const RLayerBuf &B = p.buf[t.layer];
        if (!load_rs(p, c, cs, B.ssq)) return false;
#pragma unroll
        for (int r = 0; r < kRows; ++r) { y[r] *= c->rs[r]; c->xbuf[m][r] = y[r]; }
        if (!group_sync(&c->ebar, cs.eph, p, c, (uint32_t)cs.task_id)) return false;
        const int R = tile * kRTile + m;
        const int d = s.d, half = d / 2;
        const int i = R % d;                   // tiles hold whole heads
        const int partner = m ^ half;
        const RLayerW &L = p.layers[t.layer];
        for (int r = 0; r < nrows; ++r) {
            const RRow rw = rrow(p, cs.step, r);
            const float o = c->xbuf[partner][r];
            if (R < s.QD + s.KD) {
                const float2 cs2 = p.rope[(size_t)rw.pos * half + (i % half)];
                const float rot = i < half ? y[r] * cs2.x - o * cs2.y : y[r] * cs2.x + o * cs2.y;
                if (R < s.QD) {
                    B.q[(size_t)r * s.QD + R] = rot * (1.0f / sqrtf((float)d));
                } else {
                    const int kvh = (R - s.QD) / d;
                    L.kc[(((size_t)rw.slot * s.nkv + kvh) * s.S + rw.pos) * d + i] =
                        __bfloat16_as_ushort(__float2bfloat16_rn(rot));
                }
            } else {
                const int kvh = (R - s.QD - s.KD) / d;
                L.vc[(((size_t)rw.slot * s.nkv + kvh) * s.S + rw.pos) * d + i] =
                    __bfloat16_as_ushort(__float2bfloat16_rn(y[r]));
            }
        }
        return true;
    }
    case ROP_OPROJ: {
        const RLayerBuf &B = p.buf[t.layer];
        const float *xin = t.layer == 0 ? p.x0 : p.buf[t.layer - 1].xb;
        const int R = tile * kRTile + m;
        float x[kRows];
#pragma unroll
        for (int r = 0; r < kRows; ++r) x[r] = r < nrows ? ldcg(xin + (size_t)r * s.H + R) + y[r] : 0.f;
        return resid_out(p, c, cs, tile, m, x, nrows, B.xa, B.xg, p.layers[t.layer].g_mlp, B.ssg,
                         B.rdy[rgemv_slot(ROP_GATEUP)]);
    }
    case ROP_GATEUP: {
        const RLayerBuf &B = p.buf[t.layer];
        if (!load_rs(p, c, cs, B.ssg)) return false;
#pragma unroll
        for (int r = 0; r < kRows; ++r) { y[r] *= c->rs[r]; c->xbuf[m][r] = y[r]; }
        if (!group_sync(&c->ebar, cs.eph, p, c, (uint32_t)cs.task_id)) return false;
        if (m < kRTile / 2) {
            const int j = tile * (kRTile / 2) + m;   // FFN index: gate row m, up row m + 64
#pragma unroll
            for (int r = 0; r < kRows; ++r)
                st_split(B.xd, r, j, r < nrows ? silu(y[r]) * c->xbuf[m + kRTile / 2][r] : 0.f);
            // half of slab tile / 2 of the down projection's input: each
            // writer warp releases its 32 columns (4 releases a slab)
            asm volatile("fence.proxy.async.global;" ::: "memory");
            __syncwarp();
            if ((m & 31) == 0) red_release_gpu(B.rdy[rgemv_slot(ROP_DOWN)] + tile / 2, 1u);
        }
        return true;
    }
    case ROP_DOWN: {
        const RLayerBuf &B = p.buf[t.layer];
        const bool last = t.layer + 1 == s.L;
        const int R = tile * kRTile + m;
        float x[kRows];
#pragma unroll
        for (int r = 0; r < kRows; ++r) x[r] = r < nrows ? ldcg(B.xa + (size_t)r * s.H + R) + y[r] : 0.f;
        return resid_out(p, c, cs, tile, m, x, nrows, B.xb, last ? p.xlm : p.buf[t.layer + 1].xq,
                         last ? p.g_final : p.layers[t.layer + 1].g_attn, last ? p.sslm : p.buf[t.layer + 1].ssq,
                         last ? p.rdy_lm : p.buf[t.layer + 1].rdy[rgemv_slot(ROP_QKV)]);
    }
    default: {   // ROP_LMHEAD
        if (!load_rs(p, c, cs, p.sslm)) return false;
        const int R = tile * kRTile + m;
        const bool valid = R < s.V;
        const bool out = p.logits && cs.step + 1 == p.n_steps;
        const int r0 = p.out_row0;
        const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
        const uint32_t rb = cs.rb;
        cs.rb ^= 1u;
#pragma unroll
        for (int r = 0; r < kRows; ++r) {
            float v = valid ? y[r] * c->rs[r] : -INFINITY;
            if (out && valid && r < nrows && r >= r0) p.logits[(size_t)(r - r0) * s.V + R] = v;
            int idx = valid ? R : 0x7fffffff;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                const float ov = __shfl_xor_sync(0xffffffffu, v, o);
                const int oi = __shfl_xor_sync(0xffffffffu, idx, o);
                if (ov > v || (ov == v && oi < idx)) { v = ov; idx = oi; }
            }
            if (lane == 0) { c->redv[rb][warp][r] = v; c->redi[rb][warp][r] = idx; }
        }
        if (!group_sync(&c->ebar, cs.eph, p, c, (uint32_t)cs.task_id)) return false;
        if (threadIdx.x < kRows) {
            const int r = threadIdx.x;
            float v = c->bestv[r];
            int idx = c->besti[r];
            for (int w = 0; w < kEpiWarps; ++w) {
                const float ov = c->redv[rb][w][r];
                const int oi = c->redi[rb][w][r];
                if (ov > v || (ov == v && oi < idx)) { v = ov; idx = oi; }
            }
            c->bestv[r] = v;
            c->besti[r] = idx;
        }
        return true;
    }
    }
}

__device__ __forceinline__ float *split_acc(const RParams &p, const Task &t) {
    return t.kind == ROP_LMHEAD ? p.lm_acc : p.buf[t.layer].acc[rgemv_slot(t.kind)];
}
__device__ __forceinline__ uint32_t *split_cnt(const RParams &p, const Task &t) {
    return t.kind == ROP_LMHEAD ? p.lm_tcnt : p.buf[t.layer].cnt[rgemv_slot(t.kind)];
}

// A GEMV task on the epilogue warps (0-3): every segment's accumulator, then
// the tile's epilogue -- directly for a whole tile, else after adding the
// partial into the tile's global sum, by the SM that adds the last page.
__device__ bool gemv_task(const RParams &p, Ctl *c, CState &cs, const Task &t) {
    const RGemv g = rgemv(p.s, t.kind);
    const int m = threadIdx.x, warp = m >> 5;
    if (t.kind == ROP_LMHEAD && m < kRows) { c->bestv[m] = -INFINITY; c->besti[m] = 0x7fffffff; }
    for (int pg = t.begin; pg < t.end;) {
        const int pe = seg_end(pg, t.end, g.slabs);
        const int tile = pg / g.slabs;
        const uint32_t acc = cs.segs & 1u;
        if (!wait_bar_t(&c->accfull[acc], (cs.segs >> 1) & 1u, p, c, W_ACC, (uint32_t)cs.task_id,
                        m == 0 ? stat_slot(p, RS_CMP_ACC) : nullptr))
            return false;
        tc_fence_after();
        if (p.trace && m == 0 && pg == t.begin) p.trace[t.sm].t_input = globaltimer();
        uint32_t d[32];
        tmem_ld32(c->tmem_base + ((uint32_t)(32 * warp) << 16) + acc * kRAccCols, d);
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if ((threadIdx.x & 31) == 0) mbar_arrive(&c->accempty[acc]);
        ++cs.segs;
        float y[kRows];
#pragma unroll
        for (int r = 0; r < kRows; ++r) y[r] = __uint_as_float(d[r]) + __uint_as_float(d[kRows + r]);
        const int npg = pe - pg;
        bool finish = npg == g.slabs;
        if (!finish) {
            // add this segment's partial; the SM adding the tile's last page finishes it
            float *a = split_acc(p, t) + ((size_t)tile * kRTile + m) * kRows;
#pragma unroll
            for (int r = 0; r < kRows; r += 4)
                asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(a + r), "f"(y[r]), "f"(y[r + 1]),
                             "f"(y[r + 2]), "f"(y[r + 3])
                             : "memory");
            // the barrier puts every thread's adds before thread m == 0's
            // release; the finisher's acquire puts all of them before its reads
            if (!group_sync(&c->ebar, cs.eph, p, c, (uint32_t)cs.task_id)) return false;
            if (m == 0) {
                // a tile receives exactly `slabs` pages per step, and two
                // steps' adds to one tile never interleave (the next step's
                // op waits for this one through the dependency chain)
                const uint32_t old = atom_add_acqrel_gpu(split_cnt(p, t) + tile, (uint32_t)npg);
                c->last_flag = ((old + (uint32_t)npg) % (uint32_t)g.slabs == 0u) ? 1u : 0u;
            }
            if (!group_sync(&c->ebar, cs.eph, p, c, (uint32_t)cs.task_id)) return false;
            finish = c->last_flag != 0u;
            if (finish) {
#pragma unroll
                for (int r = 0; r < kRows; r += 4) {
                    const float4 v = __ldcg(reinterpret_cast<const float4 *>(a + r));
                    y[r] = v.x; y[r + 1] = v.y; y[r + 2] = v.z; y[r + 3] = v.w;
                    *reinterpret_cast<float4 *>(a + r) = make_float4(0.f, 0.f, 0.f, 0.f);
                }
            }
        }
        if (finish && !tile_epilogue(p, c, cs, t, tile, y)) return false;
        pg = pe;
    }
    return true;
}

// Embedding rows for 128 hidden columns (epilogue warps): the layer-0
// residual stream and its QKV input.
__device__ bool embed_task(const RParams &p, Ctl *c, CState &cs, const Task &t) {
    const int tile = t.begin, m = threadIdx.x;
    const int nrows = rrows_in_step(p, cs.step);
    float x[kRows];
#pragma unroll
    for (int r = 0; r < kRows; ++r)
        x[r] = r < nrows ? __bfloat162float(__ushort_as_bfloat16(
                               p.embed[(size_t)rrow(p, cs.step, r).tok * p.s.H + tile * kRTile + m]))
                         : 0.f;
    const RLayerBuf &B = p.buf[0];
    return resid_out(p, c, cs, tile, m, x, nrows, p.x0, B.xq, p.layers[0].g_attn, B.ssq,
                     B.rdy[rgemv_slot(ROP_QKV)]);
}

// One block of up to 32 positions of an attention item (G query heads of
// one KV head), queries in registers: lane (pp, g) of the warp is position
// pp of each pass and dim group g (NG = G * D / 64 groups of NS = 8 / G
// 16-byte chunks; its query slices `qr` were loaded once per item), reading
// K chunks in the rotated order of attn_kv_rot (no bank conflicts when K
// sits in the ring); the NG lanes of a position reduce-scatter their partial
// dots so each ends with one head's score.  The softmax weights go to the
// warp's slot (4 heads per position), P·V reads them back with lanes over
// head dims.  `lw`: this lane's share of head hg's softmax sum (lanes with
// g % (NG / G) == 0).  K and V rows come from a landed page of the ring or,
// with GLOBAL, for positions written during this launch, from global memory
// through L2 (ld.global.cg: other SMs wrote them in this launch, so no
// stale L1 line may be used).
template <int D, int G, bool GLOBAL>
__device__ __forceinline__ void attn_block(Ctl *c, const uint16_t *K, const uint16_t *V, int n,
                                           const float2 (&qr)[8 / G][G][4], int g, int pp, int rot,
                                           float (&mx)[G], float &lw, float (&o)[G][D / 32]) {
    constexpr int NG = G * D / 64, NS = 8 / G, PPI = 32 / NG, IT = NG, LPH = NG / G, DPL = D / 32;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int hg = g / LPH;
    float xs[IT];
#pragma unroll
    for (int it = 0; it < IT; ++it) {
        const int j = it * PPI + pp;
        float2 acc[G];
#pragma unroll
        for (int h = 0; h < G; ++h) acc[h] = make_float2(0.f, 0.f);
        if (j < n) {
            const uint4 *krow = reinterpret_cast<const uint4 *>(K + (size_t)j * D);
#pragma unroll
            for (int k = 0; k < NS; ++k) {
                const int cc = g * NS + (k + rot) % NS;
                uint4 kw;
                if constexpr (GLOBAL) kw = __ldcg(krow + cc);
                else kw = krow[cc];
                const float2 k01 = make_float2(bf_lo(kw.x), bf_hi(kw.x));
                const float2 k23 = make_float2(bf_lo(kw.y), bf_hi(kw.y));
                const float2 k45 = make_float2(bf_lo(kw.z), bf_hi(kw.z));
                const float2 k67 = make_float2(bf_lo(kw.w), bf_hi(kw.w));
#pragma unroll
                for (int h = 0; h < G; ++h) {
                    acc[h] = ffma2(k01, qr[k][h][0], acc[h]);
                    acc[h] = ffma2(k23, qr[k][h][1], acc[h]);
                    acc[h] = ffma2(k45, qr[k][h][2], acc[h]);
                    acc[h] = ffma2(k67, qr[k][h][3], acc[h]);
                }
            }
        }
        float v[G];
#pragma unroll
        for (int h = 0; h < G; ++h) v[h] = acc[h].x + acc[h].y;
        reduce_scatter<G, NG / 2>(v, g);
        xs[it] = j < n ? v[0] : -INFINITY;
    }
    // head hg's block maximum: the lane's passes, then the lanes holding the
    // same head (twin dim groups, other positions)
    float m = xs[0];
#pragma unroll
    for (int it = 1; it < IT; ++it) m = fmaxf(m, xs[it]);
#pragma unroll
    for (int off = 1; off < LPH; off <<= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
#pragma unroll
    for (int off = NG; off < 32; off <<= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    float corr[G];
    float mg = 0.f, cg = 0.f;
#pragma unroll
    for (int h = 0; h < G; ++h) {
        const float mn = fmaxf(mx[h], __shfl_sync(0xffffffffu, m, h * LPH));   // finite: position 0 is valid
        corr[h] = expf(mx[h] - mn);
        mx[h] = mn;
        if (hg == h) { mg = mn; cg = corr[h]; }
    }
    float *pwf = reinterpret_cast<float *>(c->at.pw[warp]);   // [32 positions][4 heads]
    if (g % LPH == 0) {
        float ls = 0.f;
#pragma unroll
        for (int it = 0; it < IT; ++it) {
            const float pe = expf(xs[it] - mg);   // 0 past n (xs = -inf)
            ls += pe;
            pwf[(it * PPI + pp) * 4 + hg] = pe;
        }
        lw = fmaf(lw, cg, ls);
    }
    __syncwarp();
    const float4 *pw = c->at.pw[warp];
    float tv[G][DPL];
#pragma unroll
    for (int h = 0; h < G; ++h)
#pragma unroll
        for (int i = 0; i < DPL; ++i) tv[h][i] = 0.f;
    auto pvk = [&](int k) {
        const uint16_t *vr = V + (size_t)k * D + lane * DPL;
        float v[DPL];
        if constexpr (DPL == 2) {
            uint32_t w;
            if constexpr (GLOBAL) w = __ldcg(reinterpret_cast<const unsigned int *>(vr));
            else w = *reinterpret_cast<const uint32_t *>(vr);
            v[0] = bf_lo(w); v[1] = bf_hi(w);
        } else {
            uint2 w;
            if constexpr (GLOBAL) w = __ldcg(reinterpret_cast<const uint2 *>(vr));
            else w = *reinterpret_cast<const uint2 *>(vr);
            v[0] = bf_lo(w.x); v[1] = bf_hi(w.x); v[2] = bf_lo(w.y); v[3] = bf_hi(w.y);
        }
        const float4 pk4 = pw[k];
        const float pk[4] = {pk4.x, pk4.y, pk4.z, pk4.w};
#pragma unroll
        for (int h = 0; h < G; ++h) {
#pragma unroll
            for (int i = 0; i < DPL; ++i) tv[h][i] = fmaf(pk[h], v[i], tv[h][i]);
        }
    };
    if (n == 32) {
#pragma unroll
        for (int k = 0; k < 32; ++k) pvk(k);   // loads independent of the sums: all in flight
    } else {
        for (int k = 0; k < n; ++k) pvk(k);
    }
#pragma unroll
    for (int h = 0; h < G; ++h)
#pragma unroll
        for (int i = 0; i < DPL; ++i) o[h][i] = fmaf(o[h][i], corr[h], tv[h][i]);
    __syncwarp();   // the next block's weights overwrite pw
}

// One attention item (row r, KV head h, chunk c) on the 8 compute warps:
// the G query heads that share KV head h, over the chunk's positions --
// those written before the launch from the page ring, the rest (this
// launch's rows of the same sequence) from the cache.  One chunk: the heads'
// outputs go straight to the O projection's input; several: a tagged
// partial (o, m, l) per head, merged by chunk 0's item.
template <int D, int G>
__device__ bool attn_task(const RParams &p, unsigned char *ring, Ctl *c, CState &cs, const Task &t) {
    constexpr int DPL = D / 32;
    const Shape &s = p.s;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const Item a = attn_item(p, cs.step, t.begin);
    const int npp = rattn_pos_per_page(D);
    const int npages = attn_pages(p, a);
    const RLayerBuf &B = p.buf[t.layer];
    const RLayerW &L = p.layers[t.layer];
    if (a.active)
        for (int i = tid; i < G * D; i += kComputeWarps * 32)
            c->at.q[i] = ldcg(B.q + (size_t)a.r * s.QD + (size_t)a.h * G * D + i);
    if (!group_sync(&c->cbar, cs.cph, p, c, (uint32_t)cs.task_id)) return false;
    if (p.trace && tid == 0) p.trace[t.sm].t_input = globaltimer();
    // the lane's query slices (see attn_block), loaded once
    constexpr int NG = G * D / 64, NS = 8 / G, LPH = NG / G;
    const int gq = lane % NG, pq = lane / NG;
    const int rot = attn_kv_rot(pq, gq, NG, NS, D);
    float2 qr[NS][G][4];
#pragma unroll
    for (int k = 0; k < NS; ++k) {
        const int cc = gq * NS + (k + rot) % NS;
#pragma unroll
        for (int h = 0; h < G; ++h) {
            const float4 q0 = *reinterpret_cast<const float4 *>(c->at.q + h * D + 8 * cc);
            const float4 q1 = *reinterpret_cast<const float4 *>(c->at.q + h * D + 8 * cc + 4);
            qr[k][h][0] = make_float2(q0.x, q0.y);
            qr[k][h][1] = make_float2(q0.z, q0.w);
            qr[k][h][2] = make_float2(q1.x, q1.y);
            qr[k][h][3] = make_float2(q1.z, q1.w);
        }
    }
    float mx[G], o[G][DPL];
    float lw = 0.f;
#pragma unroll
    for (int g = 0; g < G; ++g) {
        mx[g] = -INFINITY;
#pragma unroll
        for (int i = 0; i < DPL; ++i) o[g][i] = 0.f;
    }
    // the two halves of the warps take alternate pages (4 warps x 32
    // positions = one page at head_dim 64); every warp still waits for every
    // page in order, so its view of each slot's barrier phases stays exact
    for (int pg = 0; pg < npages; ++pg) {
        const uint32_t slot = cs.aseq % kRStages;
        if (!wait_bar_t(&c->full_c[slot], (cs.odd_c >> slot) & 1u, p, c, W_FULL, (uint32_t)cs.task_id,
                        tid == 0 ? stat_slot(p, RS_CMP_KV) : nullptr))
            return false;
        const uint16_t *Kp = reinterpret_cast<const uint16_t *>(ring + (size_t)slot * kRPageBytes);
        const uint16_t *Vp = Kp + (size_t)npp * D;
        const int n = min(npp, a.nring - pg * npp);
        if ((pg & 1) == (warp >> 2))
            for (int j0 = (warp & 3) * 32; j0 < n; j0 += 4 * 32)
                attn_block<D, G, false>(c, Kp + (size_t)j0 * D, Vp + (size_t)j0 * D, min(32, n - j0), qr, gq, pq,
                                        rot, mx, lw, o);
        __syncwarp();
        if (lane == 0) mbar_arrive(&c->empty_c[slot]);
        cs.odd_c ^= 1u << slot;
        ++cs.aseq;
    }
    if (a.active) {
        // positions written during this launch: straight from the cache
        const size_t head = ((size_t)a.slot * s.nkv + a.h) * s.S;
        for (int j0 = a.c0 + a.nring + warp * 32; j0 < a.c1; j0 += kComputeWarps * 32)
            attn_block<D, G, true>(c, L.kc + (head + j0) * D, L.vc + (head + j0) * D, min(32, a.c1 - j0), qr, gq,
                                   pq, rot, mx, lw, o);
    }
    // head h's softmax sum: the lanes of head h add up (lane h * LPH holds it)
#pragma unroll
    for (int off = NG; off < 32; off <<= 1) lw += __shfl_xor_sync(0xffffffffu, lw, off);
    float l[G];
#pragma unroll
    for (int g = 0; g < G; ++g) l[g] = __shfl_sync(0xffffffffu, lw, g * LPH);
    // combine the warps' states: slot of warp w = G x (o[D], m, l)
    float *st = c->at.st[warp];
#pragma unroll
    for (int g = 0; g < G; ++g) {
#pragma unroll
        for (int i = 0; i < DPL; ++i) st[g * (D + 2) + lane * DPL + i] = o[g][i];
        if (lane == 0) { st[g * (D + 2) + D] = mx[g]; st[g * (D + 2) + D + 1] = l[g]; }
    }
    if (!group_sync(&c->cbar, cs.cph, p, c, (uint32_t)cs.task_id)) return false;
    uint64_t *part = B.part + (((size_t)a.r * s.nkv + a.h) * s.NC) * (G * (D + 2));
    if (a.active && a.c < a.nc) {
        for (int e = tid; e < G * D; e += kComputeWarps * 32) {
            const int g = e / D, i = e % D;
            float M = -INFINITY;
            for (int w = 0; w < kComputeWarps; ++w) M = fmaxf(M, c->at.st[w][g * (D + 2) + D]);
            float O = 0.f, Ls = 0.f;
            if (M != -INFINITY)
                for (int w = 0; w < kComputeWarps; ++w) {
                    const float f = expf(c->at.st[w][g * (D + 2) + D] - M);
                    O = fmaf(f, c->at.st[w][g * (D + 2) + i], O);
                    Ls = fmaf(f, c->at.st[w][g * (D + 2) + D + 1], Ls);
                }
            if (a.nc == 1) {
                st_split(B.xo, a.r, (a.h * G + g) * D + i, O / Ls);
            } else {
                uint64_t *dst = part + (size_t)a.c * (G * (D + 2)) + g * (D + 2);
                st_tag(dst + i, O, cs.ep);
                if (i == 0) { st_tag(dst + D, M, cs.ep); st_tag(dst + D + 1, Ls, cs.ep); }
            }
        }
    }
    if (a.active && a.nc > 1 && a.c == 0) {
        // chunk 0 merges the chunks' partials (every other chunk's item is
        // ahead of this one on its SM's queue, so the wait always ends)
        for (int e = tid; e < G * D; e += kComputeWarps * 32) {
            const int g = e / D, i = e % D;
            float M = -INFINITY, num = 0.f, den = 0.f;
            for (int k = 0; k < a.nc; ++k) {
                const uint64_t *src = part + (size_t)k * (G * (D + 2)) + g * (D + 2);
                Spin sp;
                uint64_t wm = ld_tag1(src + D), wl = ld_tag1(src + D + 1), wo = ld_tag1(src + i);
                while (!tag_ok(wm, cs.ep) || !tag_ok(wl, cs.ep) || !tag_ok(wo, cs.ep)) {
                    if (!spin_ok(sp, p, c, W_TAG, (uint32_t)cs.task_id, (uint32_t)k)) return false;
                    wm = ld_tag1(src + D); wl = ld_tag1(src + D + 1); wo = ld_tag1(src + i);
                }
                const float mk = tag_val(wm);
                if (mk == -INFINITY) continue;
                const float Mn = fmaxf(M, mk);
                const float f0 = expf(M - Mn), f1 = expf(mk - Mn);
                num = num * f0 + f1 * tag_val(wo);
                den = den * f0 + f1 * tag_val(wl);
                M = Mn;
            }
            st_split(B.xo, a.r, (a.h * G + g) * D + i, num / den);
        }
    }
    return true;
}

template <int D>
__device__ __forceinline__ bool attn_dispatch(const RParams &p, unsigned char *ring, Ctl *c, CState &cs,
                                              const Task &t) {
    switch (p.s.G) {
    case 1: return attn_task<D, 1>(p, ring, c, cs, t);
    case 2: return attn_task<D, 2>(p, ring, c, cs, t);
    default: return attn_task<D, 4>(p, ring, c, cs, t);
    }
}

// The last LM-head task of the last step reduces the tasks' partial
// argmaxes to every row's next token (warp 0).
__device__ void lm_reduce(const RParams &p, int nrows) {
    const int lane = threadIdx.x & 31;
    __threadfence();
    for (int r = p.out_row0; r < nrows; ++r) {
        float bv = -INFINITY;
        int bi = 0x7fffffff;
        for (int k = lane; k < p.num_lm_tasks; k += 32) {
            const float v = __ldcg(p.amax_val + (size_t)r * p.num_lm_tasks + k);
            const int i = __ldcg(p.amax_idx + (size_t)r * p.num_lm_tasks + k);
            if (v > bv || (v == bv && i < bi)) { bv = v; bi = i; }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
            const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
            if (ov > bv || (ov == bv && oi < bi)) { bv = ov; bi = oi; }
        }
        if (lane == 0) p.next_tok[r - p.out_row0] = bi;
    }
}

__device__ void compute_role(const RParams &p, unsigned char *ring, Ctl *c) {
    const int q0 = p.qoff[blockIdx.x], q1 = p.qoff[blockIdx.x + 1];
    const int qlen = q1 - q0;
    const int tid = threadIdx.x, warp = tid >> 5;
    const unsigned long long t_begin = p.sm_stats ? globaltimer() : 0ull;
    CState cs;
    for (int step = 0; step < p.n_steps; ++step) {
        cs.step = step;
        cs.ep = c->ep + (uint32_t)step;
        for (int qi = q0; qi < q1; ++qi) {
            const Task t = p.qtasks[qi];
            cs.task_id = t.sm;
            {
                // released by the scheduler once the dependency has fired
                const uint32_t k = (uint32_t)(step * qlen + (qi - q0));
                Spin s;
                const unsigned long long tr = (p.sm_stats && tid == 0) ? globaltimer() : 0ull;
                while (ld_acquire_cta_shared(&c->ready_upto) <= k)
                    if (!spin_ok(s, p, c, W_READY, (uint32_t)t.sm, 0u)) return;
                if (p.sm_stats && tid == 0) *stat_slot(p, RS_CMP_READY) += globaltimer() - tr;
            }
            const unsigned long long tb = (p.sm_stats && tid == 0) ? globaltimer() : 0ull;
            const unsigned long long acc0 = (p.sm_stats && tid == 0) ? *stat_slot(p, RS_CMP_ACC) : 0ull;
            if (p.trace && tid == 0) p.trace[t.sm].t_start = globaltimer();
            bool ok = true;
            if (t.kind == ROP_ATTN) {
                ok = p.s.d == 64 ? attn_dispatch<64>(p, ring, c, cs, t) : attn_dispatch<128>(p, ring, c, cs, t);
            } else if (warp < kEpiWarps) {
                if (t.kind == ROP_EMBED) ok = embed_task(p, c, cs, t);
                else if (task_on(p, t, step)) ok = gemv_task(p, c, cs, t);
            } else if (is_gemv(t.kind) && task_on(p, t, step)) {
                // warps 4-7 keep the accumulator count in step
                const RGemv g = rgemv(p.s, t.kind);
                for (int pg = t.begin; pg < t.end; pg = seg_end(pg, t.end, g.slabs)) ++cs.segs;
            }
            if (!ok) return;
            if (p.sm_stats && tid == 0) {
                const unsigned long long dt = globaltimer() - tb;
                if (t.kind == ROP_ATTN) *stat_slot(p, RS_CMP_ATTN) += dt;
                else *stat_slot(p, RS_CMP_EPI) += dt - (*stat_slot(p, RS_CMP_ACC) - acc0);
            }
            if (is_gemv(t.kind) && task_on(p, t, step)) cs.aseq += (uint32_t)(t.end - t.begin);
            // every write of the task is done (and ordered before the bulk
            // copies that read it on other SMs) before its completion posts
            asm volatile("fence.proxy.async.global;" ::: "memory");
            if (p.trace && tid == 0) p.trace[t.sm].t_done = globaltimer();
            if (!group_sync(&c->cbar, cs.cph, p, c, (uint32_t)t.sm)) return;
            if (t.kind == ROP_ATTN && tid == 0) {
                // chunk 0's item of (row, KV head) has written the heads'
                // outputs (directly or merged; nothing for an inactive row):
                // it releases the O-projection input slabs they fall in
                const Item a = attn_item(p, step, t.begin);
                if (a.c == 0) {
                    const int gd = p.s.G * p.s.d;
                    uint32_t *rdy = p.buf[t.layer].rdy[rgemv_slot(ROP_OPROJ)];
                    for (int sl = a.h * gd / kRSlab; sl <= (a.h * gd + gd - 1) / kRSlab; ++sl) red_release_gpu(rdy + sl, 1u);
                }
            }
            if (t.kind == ROP_LMHEAD && task_on(p, t, step)) {
                // the task's argmax partials, then (their writers met at the
                // barrier) its count: the task that completes a step's count
                // reduces every task's partials
                const int nrows = rrows_in_step(p, step);
                if (tid < nrows) {
                    p.amax_val[(size_t)tid * p.num_lm_tasks + t.slot] = c->bestv[tid];
                    p.amax_idx[(size_t)tid * p.num_lm_tasks + t.slot] = c->besti[tid];
                }
                if (!group_sync(&c->cbar, cs.cph, p, c, (uint32_t)t.sm)) return;
                if (tid == 0) {
                    // after the barrier: a release that covers every thread's partials
                    // the LM tasks of one step finish before any of the next
                    // step's start, so the count's multiples mark each step's last
                    const uint32_t old = atom_add_acqrel_gpu(p.lm_cnt, 1u);
                    c->last_flag = ((old + 1u) % (uint32_t)p.num_lm_tasks == 0u) ? 1u : 0u;
                }
                if (!group_sync(&c->cbar, cs.cph, p, c, (uint32_t)t.sm)) return;
                if (c->last_flag && step + 1 == p.n_steps && warp == 0) lm_reduce(p, nrows);
            }
            if (tid == 0 && !post_done(p, c, t)) return;
            if (p.trace && tid == 0) p.trace[t.sm].t_end = globaltimer();
        }
    }
    if (p.sm_stats && tid == 0) *stat_slot(p, RS_CMP_TOTAL) = globaltimer() - t_begin;
}

// ---------------------------------------------------------------------------
// the kernel
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kThreads, 1) mk_rows_kernel(const __grid_constant__ RParams p) {
    extern __shared__ __align__(1024) unsigned char smem[];
    unsigned char *ring = smem;
    unsigned char *slabs = smem + (size_t)kRStages * kRPageBytes;
    Ctl *c = reinterpret_cast<Ctl *>(smem + kRingBytes);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid == 0) {
        for (int i = 0; i < kRStages; ++i) {
            mbar_init(&c->full_m[i], 1);
            mbar_init(&c->full_c[i], 1);
            mbar_init(&c->empty_m[i], 1);
            mbar_init(&c->empty_c[i], kComputeWarps);
            mbar_init(&c->bfull[i], 1);
            mbar_init(&c->bempty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&c->accfull[i], 1);
            mbar_init(&c->accempty[i], kEpiWarps);
        }
        mbar_init(&c->cbar, kComputeWarps);
        mbar_init(&c->ebar, kEpiWarps);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        c->ready_upto = 0;
        c->sig_post = 0;
        c->sig_done = 0;
        c->last_flag = 0;
        c->stop = 0;
        c->ep = ld_volatile_u32(p.epoch) + 1u;
        uint32_t stop = ld_volatile_u32(p.abort_flag) ? 1u : 0u;
        for (int st = 0; st < p.n_steps && !stop; ++st)
            for (int r = 0; r < rrows_in_step(p, st) && !stop; ++r) {
                const RRow rw = rrow(p, st, r);
                if (rw.tok < 0 || rw.tok >= p.s.V || rw.pos < 0 || rw.pos >= p.s.S || rw.slot < 0 ||
                    rw.slot >= p.s.Bmax || rw.pre < 0 || rw.pre > rw.pos) {
                    if (atomicCAS(&p.err->code, 0u, kErrInvalid) == 0u) {
                        p.err->task = 0xffffffffu;
                        p.err->where = W_INPUT;
                        p.err->info = (uint32_t)(st * kRows + r);
                    }
                    stop = 1u;
                }
            }
        c->abort = stop;
    }
    __syncthreads();
    if (c->abort) return;
    if (warp == kMmaWarp) tmem_alloc(&c->tmem_base, kRTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (tid == 0) {
        const uint32_t n = (uint32_t)p.n_steps;
        const uint32_t ep_last = c->ep + n - 1u;
        const uint32_t old = atomicAdd(p.done_cnt, n);
        if (old + n == gridDim.x * ep_last) atomicExch(p.epoch, ep_last);
    }
    if (warp < kComputeWarps) {
        compute_role(p, ring, c);
    } else if (lane == 0) {
        if (warp == kLoaderWarp) loader_role(p, ring, c);
        else if (warp == kSchedWarp) sched_role(p, slabs, c);
        else if (warp == kMmaWarp) mma_role(p, ring, slabs, c);
        else if (warp == kSigWarp) signaler_role(p, c);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(c->tmem_base, kRTmemCols);
    }
}

}  // namespace rows

// ---------------------------------------------------------------------------
// host-side helpers (mk_runtime.cpp)
// ---------------------------------------------------------------------------
size_t rows_smem_bytes() { return rows::kSmem; }

cudaError_t rows_prepare() {
    return cudaFuncSetAttribute(rows::mk_rows_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)rows::kSmem);
}

cudaError_t rows_launch(const RParams &p, int grid, cudaStream_t stream) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(rows::kThreads);
    cfg.dynamicSmemBytes = rows::kSmem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, rows::mk_rows_kernel, p);
}

// Weights of one GEMV op into the page layout (rpage_elem): `src` is the
// row-major matrix [rows][K] (rows >= tiles * 128 - padding, zero beyond
// `rows`); for the gate/up op, `src2` is the up matrix and tile i holds gate
// rows 64i.. and up rows 64i.. (src = gate).  dst: tiles * (K / 128) pages.
__global__ void repack_rows_kernel(uint16_t *dst, const uint16_t *src, const uint16_t *src2, long long rows, int K,
                                   int tiles) {
    const int slabs = K / kRSlab;
    const long long total = (long long)tiles * slabs * kRTile * kRSlab;
    for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < total;
         e += (long long)gridDim.x * blockDim.x) {
        const long long page = e / (kRTile * kRSlab);
        const int within = (int)(e % (kRTile * kRSlab));
        const int m = within / kRSlab, k = within % kRSlab;
        const int tile = (int)(page / slabs), slab = (int)(page % slabs);
        long long row;
        const uint16_t *s = src;
        if (src2) {   // gate/up pairs
            row = (long long)tile * (kRTile / 2) + (m % (kRTile / 2));
            if (m >= kRTile / 2) s = src2;
        } else {
            row = (long long)tile * kRTile + m;
        }
        const uint16_t v = row < rows ? s[row * K + (long long)slab * kRSlab + k] : (uint16_t)0;
        dst[page * (kRTile * kRSlab) + (long long)rpage_elem(m, k)] = v;
    }
}

cudaError_t repack_rows(uint16_t *dst, const uint16_t *src, const uint16_t *src2, long long rows, int K, int tiles,
                        cudaStream_t stream) {
    const long long total = (long long)tiles * (K / kRSlab) * kRTile * kRSlab;
    const long long blocks = (total + 255) / 256;
    repack_rows_kernel<<<(unsigned)(blocks < 16384 ? blocks : 16384), 256, 0, stream>>>(dst, src, src2, rows, K,
                                                                                        tiles);
    return cudaGetLastError();
}

}  // namespace mk
