// Host-only check of the persistent kernel's work-unit schedule: for one
// geometry given on the command line it decodes every unit index and checks
// that each (batch*head, patch, query-tile pair) of the patch range occurs
// (a group of tiles_per_unit query tiles) exactly once, that unit costs never increase along the order when an
// order was built (at most kMaxPatchOrder patches), and prints the number of
// ordered patches, the number of cost classes and the batch*head values the
// first `wave` units touch. Built and run by test_unit_schedule.py, which
// also runs its "cover" mode (the overlapping-window coverage rule).
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <set>
#include <vector>

#include "../patch_res_diffusion_b200/csrc/npa_geometry.cuh"

// "cover L P m": checks md_cover_range against a scan of every window along
// an axis of length L, for every coordinate.
static int check_cover(int L, int P, int m) {
    const int n = (L + P - 1) / P;
    for (int x = 0; x < L; ++x) {
        int lo, hi, blo = -1, bhi = -1;
        npa::md_cover_range(n, P, m, x, &lo, &hi);
        for (int i = 0; i < n; ++i) {
            const int w0 = i * P - m < 0 ? 0 : i * P - m, w1 = (i + 1) * P + m < L ? (i + 1) * P + m : L;
            if (x >= w0 && x < w1) {
                if (blo < 0) blo = i;
                if (bhi >= 0 && bhi != i - 1) {
                    std::printf("FAIL windows containing %d are not contiguous\n", x);
                    return 1;
                }
                bhi = i;
            }
        }
        if (lo != blo || hi != bhi) {
            std::printf("FAIL x %d: range [%d, %d], scan [%d, %d]\n", x, lo, hi, blo, bhi);
            return 1;
        }
    }
    std::printf("ok cover\n");
    return 0;
}

int main(int argc, char **argv) {
    if (argc == 5 && std::strcmp(argv[1], "cover") == 0)
        return check_cover(std::atoi(argv[2]), std::atoi(argv[3]), std::atoi(argv[4]));
    if (argc != 15 && argc != 16) {
        std::fprintf(stderr,
                     "usage: BH H W Ph Pw mh mw kb kc_log2 tiles_per_unit n_qblocks patch_begin patch_count wave "
                     "[head_major]\n");
        return 2;
    }
    int a[14];
    for (int i = 0; i < 14; ++i) a[i] = std::atoi(argv[i + 1]);
    npa::FwdParams p;
    std::memset(&p, 0, sizeof(p));
    p.BH = a[0];
    p.H = a[1];
    p.W = a[2];
    p.Ph = a[3];
    p.Pw = a[4];
    p.mh = a[5];
    p.mw = a[6];
    p.kb = a[7];
    p.kc_log2 = a[8];
    p.kr = p.kb >> p.kc_log2;
    p.tiles_per_unit = a[9];
    p.n_qblocks = a[10];
    p.nPh = (p.H + p.Ph - 1) / p.Ph;
    p.nPw = (p.W + p.Pw - 1) / p.Pw;
    p.patch_begin = a[11];
    p.patch_count = a[12] < 0 ? p.nPh * p.nPw - p.patch_begin : a[12];
    const int wave = a[13];
    p.n_units = p.BH * p.patch_count * p.n_qblocks;
    npa::order_patches(p);
    const int n_patches = p.nPh * p.nPw;
    std::vector<int> seen((size_t)p.BH * n_patches * p.n_qblocks, 0);
    int prev_cost = 1 << 30;
    std::set<int> wave_bh;
    for (int u = 0; u < p.n_units; ++u) {
        const npa::Work w = npa::decode_work(p, u);
        const int patch = (w.pr0 / p.Ph) * p.nPw + w.pc0 / p.Pw;
        const int qb = w.tile0 / p.tiles_per_unit;
        if (w.tile0 % p.tiles_per_unit != 0 || w.bh < 0 || w.bh >= p.BH || patch < p.patch_begin || patch >= p.patch_begin + p.patch_count ||
            qb < 0 || qb >= p.n_qblocks) {
            std::printf("FAIL unit %d decodes outside the range (bh %d patch %d pair %d)\n", u, w.bh, patch, qb);
            return 1;
        }
        const int cost = npa::patch_cost(p, patch);
        if (p.n_perm > 0 && cost > prev_cost) {
            std::printf("FAIL unit %d cost %d after %d\n", u, cost, prev_cost);
            return 1;
        }
        prev_cost = cost;
        if (++seen[((size_t)w.bh * n_patches + patch) * p.n_qblocks + qb] != 1) {
            std::printf("FAIL unit %d repeats (bh %d patch %d pair %d)\n", u, w.bh, patch, qb);
            return 1;
        }
        if (u < wave) wave_bh.insert(w.bh);
    }
    // the per-CTA lists (wave = CTA count): every unit exactly once; the
    // predicted finish time of the busiest CTA over the mean (and its list
    // scheduling bound: the mean plus the costliest unit); the heads the first
    // unit of every CTA touches
    const int grid = p.n_units < wave ? p.n_units : wave;
    npa::build_schedule(p, grid, argc == 16 && std::atoi(argv[15]) != 0);
    double balance = 0.0, bound = 0.0;
    std::set<int> first_bh;
    if (p.n_sched) {
        if (p.n_sched != p.n_units || p.cta_first[grid] != p.n_units) {
            std::printf("FAIL schedule holds %d of %d units\n", (int)p.cta_first[grid], p.n_units);
            return 1;
        }
        std::vector<int> hit(p.n_units, 0);
        long long total = 0, worst = 0, biggest = 0;
        for (int c = 0; c < grid; ++c) {
            long long t = 0;
            for (int k = p.cta_first[c]; k < p.cta_first[c + 1]; ++k) {
                const int u = p.sched[k];
                if (u >= p.n_units || ++hit[u] != 1) {
                    std::printf("FAIL schedule repeats or exceeds unit %d\n", u);
                    return 1;
                }
                int bh;
                const long long cost = npa::unit_cost(p, npa::unit_patch(p, u, &bh));
                t += cost;
                if (cost > biggest) biggest = cost;
                if (k == p.cta_first[c]) first_bh.insert(bh);
            }
            total += t;
            if (t > worst) worst = t;
        }
        balance = (double)worst * grid / (double)total;
        bound = 1.0 + (double)biggest * grid / (double)total;  // list scheduling: mean + one unit
    }
    std::printf("ok units %d ordered %d classes %d wave_heads %d sched %d balance %.4f first_heads %d bound %.4f\n",
                p.n_units, p.n_perm, p.n_cls, (int)wave_bh.size(), p.n_sched, balance, (int)first_bh.size(), bound);
    return 0;
}
