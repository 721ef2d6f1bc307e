// Host driver for test_hilbert_table.py: Hilbert keys of grid points by the
// device library's state-machine tables (hilbert_table.cuh), on the CPU.
// stdin: bits, count, then count x (x, y, z) as uint32; stdout: count keys.
#include <cstdint>
#include <cstdio>
#include <vector>

#include "../space_filling_curve_b200/csrc/hilbert_table.cuh"

static uint32_t spread(uint32_t v, int bits) {
    uint32_t r = 0;
    for (int k = 0; k < bits; ++k) r |= ((v >> k) & 1u) << (3 * k);
    return r;
}

int main() {
    const tess::HilbertTables& T = tess::kHilbertTables;
    uint32_t hdr[2];
    if (fread(hdr, 4, 2, stdin) != 2) return 2;
    const int bits = (int)hdr[0];
    std::vector<uint32_t> q(3 * (size_t)hdr[1]), out(hdr[1]);
    if (fread(q.data(), 4, q.size(), stdin) != q.size()) return 2;
    for (size_t i = 0; i < out.size(); ++i) {
        const uint32_t m = (spread(q[3 * i], bits) << 2) | (spread(q[3 * i + 1], bits) << 1) | spread(q[3 * i + 2], bits);
        uint32_t st = 0, key = 0;
        int l = bits;
        if (l & 1) {
            const uint32_t e = T.one[(m >> (3 * (l - 1))) & 7u];
            key = e & 7u;
            st = e >> 6;
            --l;
        }
        for (; l > 0; l -= 2) {
            const uint32_t e = T.two[st * 64 + ((m >> (3 * (l - 2))) & 63u)];
            key = (key << 6) | (e & 63u);
            st = e >> 6;
        }
        out[i] = key;
    }
    fprintf(stderr, "states %d\n", T.nstates);
    fwrite(out.data(), 4, out.size(), stdout);
    return 0;
}
