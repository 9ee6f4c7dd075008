// Host-side check of the batched kernel's per-slab readiness targets
// (mk_rows.h, rslab_writers): for every GEMV op of several shapes, count the
// releases each input slab receives in one step from the producers as the
// kernel makes them --
//   QKV, gate/up, LM head input: the residual tile i of the producing op
//     (down / O-projection / embedding, 128 rows) releases slab i once;
//   down input: gate/up tile t (64 FFN outputs) releases slab t / 2 once
//     per writer warp (64 / 32 = 2 warps);
//   O-projection input: the chunk-0 item of every (row, KV head) releases
//     each slab its G heads x head_dim columns touch, once
// -- and compare with rslab_writers.  Prints "ok" or the first mismatch.
#include <cstdio>
#include <vector>
#include "../persistent_decode_megakernel_02_b200/csrc/mk_rows.h"

using namespace mk;

static int check(const char *name, int H, int nq, int nkv, int d, int F) {
    Shape s{};
    s.H = H; s.nq = nq; s.nkv = nkv; s.d = d; s.F = F;
    s.G = nq / nkv; s.QD = nq * d; s.KD = nkv * d;
    // residual-tile producers: one release per 128-row tile = per slab
    for (int op : {ROP_QKV, ROP_GATEUP, ROP_LMHEAD}) {
        std::vector<int> n(H / kRSlab, 0);
        for (int tile = 0; tile < H / kRTile; ++tile) n[tile] += 1;
        for (int v : n)
            if ((unsigned)v != rslab_writers(s, op)) { printf("%s op %d: %d releases, target %u\n", name, op, v, rslab_writers(s, op)); return 1; }
    }
    {   // gate/up tiles of 64 outputs, 2 writer warps each
        std::vector<int> n(F / kRSlab, 0);
        for (int t = 0; t < 2 * F / kRTile; ++t)
            for (int w = 0; w < (kRTile / 2) / 32; ++w) n[(t * (kRTile / 2)) / kRSlab] += 1;
        for (int v : n)
            if ((unsigned)v != rslab_writers(s, ROP_DOWN)) { printf("%s down: %d releases, target %u\n", name, v, rslab_writers(s, ROP_DOWN)); return 1; }
    }
    {   // attention: every (row, KV head) once, over the slabs its columns touch
        std::vector<int> n(s.QD / kRSlab, 0);
        for (int r = 0; r < kRows; ++r)
            for (int h = 0; h < nkv; ++h) {
                std::vector<bool> touched(s.QD / kRSlab, false);
                for (int col = h * s.G * d; col < (h + 1) * s.G * d; ++col) touched[col / kRSlab] = true;
                for (size_t sl = 0; sl < touched.size(); ++sl) n[sl] += touched[sl] ? 1 : 0;
            }
        for (int v : n)
            if ((unsigned)v != rslab_writers(s, ROP_OPROJ)) { printf("%s O-projection: %d releases, target %u\n", name, v, rslab_writers(s, ROP_OPROJ)); return 1; }
    }
    return 0;
}

int main() {
    if (check("tiny", 256, 4, 2, 64, 768)) return 1;         // G d = 128
    if (check("g1-d64", 256, 4, 4, 64, 768)) return 1;       // G d = 64: two groups per slab
    if (check("1b", 2048, 32, 8, 64, 8192)) return 1;        // G d = 256
    if (check("8b", 4096, 32, 8, 128, 14336)) return 1;      // G d = 512
    if (check("d128-g1", 512, 4, 4, 128, 768)) return 1;     // G d = 128
    printf("ok\n");
    return 0;
}
