// Host-side check of the TMEM page order (mk_internal.h, tmem_page_src)
// against the lane/column mapping of tcgen05.cp.128x256b with a no-swizzle
// shared-memory descriptor (leading byte offset 2048, stride byte offset
// 128): TMEM lane r, columns 8c..8c+3 receive the 16 bytes at
// 4096c + (r / 8) * 128 + (r % 8) * 16 of the page, columns 8c+4..8c+7 the
// 16 bytes 2048 further.  Also the chunk rotation of the KV-head attention
// loop (attn_kv_rot): conflict-free shared-memory reads.  Prints "ok" or the
// first violation.
#include <cstdio>
#include "../persistent_decode_megakernel_02_b200/csrc/mk_internal.h"

using namespace mk;

int main() {
    // 1. a permutation of the 4096 vectors of a page
    static int seen[16][256];
    int src_row[4096], src_vec[4096];
    for (int u = 0; u < 4096; ++u) {
        int row, vec;
        tmem_page_src(u, row, vec);
        if (row < 0 || row >= 16 || vec < 0 || vec >= 256) { printf("out of range at %d\n", u); return 1; }
        if (seen[row][vec]++) { printf("vector (%d, %d) twice\n", row, vec); return 1; }
        src_row[u] = row; src_vec[u] = vec;
        // 2. page rows 0..7 sit in the first 32 KB (a trailing 8-row page)
        if ((row < 8) != (u < 2048)) { printf("row %d at vector %d crosses the half\n", row, u); return 1; }
    }
    // 3. through the copy: warp w (lane quarter w % 4) reads page rows w and
    //    8 + w as 32 columns each at 32 * (w / 4) and 64 + 32 * (w / 4); lane
    //    L must find vector L + 32 m of the row in words 4m..4m+3
    for (int w = 0; w < 8; ++w)
        for (int L = 0; L < 32; ++L) {
            const int lane = 32 * (w % 4) + L;
            for (int which = 0; which < 2; ++which) {
                const int row = which ? 8 + w : w;
                const int col0 = 64 * which + 32 * (w / 4);
                for (int m = 0; m < 8; ++m) {
                    const int col = col0 + 4 * m;            // first column of the vector
                    const int c = col / 8, q = (col % 8) / 4;
                    const int byte = 4096 * c + 2048 * q + (lane / 8) * 128 + (lane % 8) * 16;
                    const int u = byte / 16;
                    if (src_row[u] != row || src_vec[u] != L + 32 * m) {
                        printf("warp %d lane %d row %d vector %d: found (%d, %d)\n", w, L, row, L + 32 * m,
                               src_row[u], src_vec[u]);
                        return 1;
                    }
                }
            }
        }
    // 4. the KV-head attention loop's chunk rotation: for every head_dim,
    //    heads per item, pass s and quarter-warp, the 8 lanes read 8
    //    distinct bank groups (chunk index mod 8), and each lane's NS
    //    passes read its NS chunks once each
    const int cases[7][2] = {{64, 1}, {64, 2}, {64, 4}, {64, 8}, {128, 1}, {128, 2}, {128, 4}};
    for (const auto &cs : cases) {
        const int d = cs[0], ha = cs[1], ng = ha * d / 64, ns = 8 / ha;
        if (ng * ns != d / 8) { printf("groups x chunks != row chunks (d %d, ha %d)\n", d, ha); return 1; }
        for (int lane = 0; lane < 32; ++lane) {
            const int g = lane % ng, p = lane / ng;
            int hit = 0;
            for (int s = 0; s < ns; ++s) hit |= 1 << ((s + attn_kv_rot(p, g, ng, ns, d)) % ns);
            if (hit != (1 << ns) - 1) { printf("lane %d misses a chunk (d %d, ha %d)\n", lane, d, ha); return 1; }
        }
        for (int s = 0; s < ns; ++s)
            for (int q = 0; q < 4; ++q) {
                int banks = 0;
                for (int lane = 8 * q; lane < 8 * q + 8; ++lane) {
                    const int g = lane % ng, p = lane / ng;
                    const int c = g * ns + (s + attn_kv_rot(p, g, ng, ns, d)) % ns;
                    banks |= 1 << (c % 8);
                }
                if (banks != 0xff) { printf("bank conflict: d %d ha %d pass %d quarter %d\n", d, ha, s, q); return 1; }
            }
    }
    printf("ok\n");
    return 0;
}
