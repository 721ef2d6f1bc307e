// Host driver for test_scan_plan.py: the chunk plan of the library's offset
// scan (csrc/scan.cuh) for many array lengths and SM counts, checked against
// the conditions its kernel relies on.  Prints "ok" or the first violation.
#include <cstdio>

#include "../space_filling_curve_b200/csrc/scan.cuh"

int main() {
    const long long ms[] = {0, 1, 3, 4, 5, 2047, 2048, 2049, 4096, 65535, 262144, 1 << 20, 8376438, 10048049,
                            (1LL << 31) - 1};
    const int smss[] = {1, 2, 8, 132, 148, 160, 1000};
    for (long long m : ms) {
        for (int sms : smss) {
            const tess::ScanPlan P = tess::scan_plan(m, sms);
            const long long words = tess::scan_state_len(m);
            const char* bad = nullptr;
            if (P.chunk < 4 || P.chunk % 4) bad = "chunk not a positive multiple of 4 (int4 accesses)";
            else if (P.nchunks < 1) bad = "no block";
            else if ((long long)P.nchunks * P.chunk < m) bad = "chunks do not cover the array";
            else if (m > 0 && (long long)(P.nchunks - 1) * P.chunk >= m) bad = "an empty chunk";
            else if (P.nchunks + 1 > words) bad = "look-back words short of chunks + counter";
            else if (P.nchunks > tess::SCAN_MAX_CHUNKS) bad = "more chunks than the cap";
            else if (P.nchunks > 4 * sms && P.nchunks > 1) bad = "more chunks than 4 blocks per SM";
            if (bad) {
                printf("m=%lld sms=%d chunk=%lld nchunks=%d words=%lld: %s\n", m, sms, P.chunk, P.nchunks, words, bad);
                return 1;
            }
        }
    }
    printf("ok\n");
    return 0;
}
