// Host-only check of the block-scaled GEMM's work schedule (build_schedule in tl_nvfp4_api.cu):
// every k-tile of every n-tile is covered exactly once, split n-tiles carry consistent ranks,
// part counts, consecutive partial slots and k order, the workspace limits hold, the work per
// CTA (in 256-row units times k-tiles) is balanced, and the k ranges of every weight row are the
// same with 128-row and with 256-row n-tiles (so outputs do not depend on the launch); and the
// chunks a host-buffer run cuts the stack into. Built and run by tests/test_schedule.py; no GPU
// is touched.
#include "../nvfp4_weight_gemm_b200/csrc/tl_nvfp4_api.cu"

#include <algorithm>
#include <cstdio>
#include <map>
#include <set>
#include <utility>
#include <vector>

static int check(const std::vector<std::pair<int, int>>& shapes, int grid, double min_eff, bool verbose,
                 int rows = 128) {
    std::vector<tl_nvfp4_matrix> mats;
    for (auto& sh : shapes) {
        tl_nvfp4_matrix m{};
        m.N = sh.first;
        m.K = sh.second;
        mats.push_back(m);
    }
    BsSchedule sc;
    build_schedule(mats.data(), (int)mats.size(), grid, &sc, rows);
    int bad = 0;
    if ((int)sc.begin.size() != grid + 1 || sc.begin[0] != 0 || sc.begin[grid] != (int)sc.segs.size()) {
        printf("per-CTA offsets malformed\n");
        return 1;
    }
    std::map<std::pair<int, int>, std::vector<std::pair<int, int>>> cov;
    std::map<int, std::vector<tl::BsSeg>> splits;
    std::vector<long long> load(grid, 0);
    const int halves = 256 / rows;
    for (int c = 0; c < grid; ++c) {
        for (int i = sc.begin[c]; i < sc.begin[c + 1]; ++i) {
            const tl::BsSeg& g = sc.segs[i];
            cov[{g.mat, g.ntile}].push_back({g.k0, g.k1});
            if (g.ntile % halves == 0) load[c] += g.k1 - g.k0;   // work in 256-row units
            if (g.k1 <= g.k0) { ++bad; printf("empty segment\n"); }
            if (g.split >= 0) splits[g.split].push_back(g);
            else if (g.k0 != 0 || g.k1 != mats[g.mat].K / 256) { ++bad; printf("whole segment is not whole\n"); }
        }
    }
    long long total = 0;
    for (size_t i = 0; i < mats.size(); ++i) {
        const int nt = (mats[i].N + rows - 1) / rows, kt = mats[i].K / 256;
        total += (long long)((mats[i].N + 255) / 256) * kt;
        for (int j = 0; j < nt; ++j) {
            auto v = cov[{(int)i, j}];
            std::sort(v.begin(), v.end());
            int k = 0;
            for (auto& r : v) {
                if (r.first != k) ++bad;
                k = r.second;
            }
            if (k != kt) { ++bad; printf("coverage: matrix %zu n-tile %d\n", i, j); }
        }
    }
    std::set<int> slots;
    for (auto& kv : splits) {
        auto& v = kv.second;
        std::sort(v.begin(), v.end(), [](const tl::BsSeg& a, const tl::BsSeg& b) { return a.rank < b.rank; });
        for (size_t r = 0; r < v.size(); ++r) {
            if (v[r].rank != r || v[r].parts != v.size() || v[r].slot - v[r].rank != v[0].slot) {
                ++bad;
                printf("split bookkeeping\n");
            }
            if (r && v[r].k0 != v[r - 1].k1) { ++bad; printf("split parts out of k order\n"); }
            if (!slots.insert(v[r].slot).second) { ++bad; printf("partial slot used twice\n"); }
        }
    }
    if (sc.slots > 4 * grid || sc.splits > 2 * grid) { ++bad; printf("workspace limits exceeded\n"); }
    const long long mx = *std::max_element(load.begin(), load.end());
    const double eff = (double)total / grid / (double)mx;
    const long long ideal = (total + grid - 1) / grid;
    if (mx > ideal) { ++bad; printf("a CTA has %lld k-tiles, more than ceil(total / grid) = %lld\n", mx, ideal); }
    if (eff < min_eff) { ++bad; printf("balance %.4f below %.4f\n", eff, min_eff); }
    if (verbose || bad)
        printf("%d-row n-tiles, %zu matrices, grid %d: %lld k-tiles, largest CTA share %lld (balance %.4f), %zu segments, "
               "%d splits, %d slots, bad %d\n",
               rows, mats.size(), grid, total, mx, eff, sc.segs.size(), sc.splits, sc.slots, bad);
    return bad;
}

// The k ranges of every n-tile, sorted: for (matrix, n-tile) the list of (k0, k1).
static std::map<std::pair<int, int>, std::vector<std::pair<int, int>>> cuts(
        const std::vector<std::pair<int, int>>& shapes, int grid, int rows) {
    std::vector<tl_nvfp4_matrix> mats;
    for (auto& sh : shapes) {
        tl_nvfp4_matrix m{};
        m.N = sh.first;
        m.K = sh.second;
        mats.push_back(m);
    }
    BsSchedule sc;
    build_schedule(mats.data(), (int)mats.size(), grid, &sc, rows);
    std::map<std::pair<int, int>, std::vector<std::pair<int, int>>> out;
    for (const tl::BsSeg& g : sc.segs) out[{g.mat, g.ntile}].push_back({g.k0, g.k1});
    for (auto& kv : out) std::sort(kv.second.begin(), kv.second.end());
    return out;
}

// Every weight row gets the same k ranges with 128-row and with 256-row n-tiles.
static int same_cuts(const std::vector<std::pair<int, int>>& shapes, int grid) {
    auto a = cuts(shapes, grid, 128), b = cuts(shapes, grid, 256);
    int bad = 0;
    for (auto& kv : a) {
        auto it = b.find({kv.first.first, kv.first.second / 2});
        if (it == b.end() || it->second != kv.second) ++bad;
    }
    if (bad) printf("k ranges differ between 128- and 256-row n-tiles (%d n-tiles)\n", bad);
    return bad;
}

// Chunks of a host-buffer run: boundaries strictly increasing from 0 to n, at most
// min(8, n) chunks; the 64-layer stack splits at every eighth of its layers.
static int check_chunks(const std::vector<std::pair<int, int>>& shapes, const std::vector<int>* expect) {
    std::vector<tl_nvfp4_matrix> mats;
    for (auto& sh : shapes) {
        tl_nvfp4_matrix m{};
        m.N = sh.first;
        m.K = sh.second;
        mats.push_back(m);
    }
    const int n = (int)mats.size();
    const std::vector<int> cut = host_chunk_cuts(mats.data(), n, kHostChunks);
    int bad = 0;
    if (cut.empty() || cut.front() != 0 || cut.back() != n) ++bad;
    for (size_t i = 1; i < cut.size(); ++i)
        if (cut[i] <= cut[i - 1]) ++bad;
    if ((int)cut.size() - 1 > std::min(kHostChunks, n)) ++bad;
    if (expect && cut != *expect) ++bad;
    if (bad) printf("host-buffer chunks malformed for %d matrices\n", n);
    return bad;
}

int main() {
    int bad = 0;
    std::vector<std::pair<int, int>> stack;
    for (int l = 0; l < 64; ++l) {
        stack.push_back({7168, 5120});
        stack.push_back({5120, 5120});
        stack.push_back({34816, 5120});
        stack.push_back({5120, 17408});
    }
    // n-tiles of 128 weight rows, and of 256 (two weight tiles per stage)
    for (int rows = 128; rows <= 256; rows *= 2) {
        bad += check(stack, 148, 0.999, true, rows);           // the 64-layer stack
        bad += check({{5120, 5120}}, 148, 0.0, true, rows);      // single matrices: one k-tile short at most
        bad += check({{34816, 5120}}, 148, 0.0, true, rows);
        bad += check({{5120, 17408}}, 148, 0.0, true, rows);
        bad += check({{677, 2304}}, 27, 0.0, true, rows);
        bad += check({{256, 512}}, 2, 0.0, true, rows);
        srand(7);
        for (int it = 0; it < 300; ++it) {
            std::vector<std::pair<int, int>> sh;
            const int n = 1 + rand() % 40;
            for (int i = 0; i < n; ++i) sh.push_back({1 + rand() % 20000, 256 * (1 + rand() % 80)});
            long long tiles = 0;
            for (auto& s2 : sh) tiles += (long long)((s2.first + 255) / 256) * (s2.second / 256);
            const int grid = (int)std::min<long long>(tiles, 1 + rand() % 160);
            bad += check(sh, grid, 0.0, false, rows);
        }
    }
    {
        std::vector<std::pair<int, int>> stack;
        for (int l = 0; l < 64; ++l) {
            stack.push_back({7168, 5120});
            stack.push_back({5120, 5120});
            stack.push_back({34816, 5120});
            stack.push_back({5120, 17408});
        }
        bad += same_cuts(stack, 148);
        bad += same_cuts({{677, 2304}}, 27);
        srand(11);
        for (int it = 0; it < 200; ++it) {
            std::vector<std::pair<int, int>> sh;
            const int n = 1 + rand() % 40;
            for (int i = 0; i < n; ++i) sh.push_back({1 + rand() % 20000, 256 * (1 + rand() % 80)});
            long long units = 0;
            for (auto& s2 : sh) units += (long long)((s2.first + 255) / 256) * (s2.second / 256);
            bad += same_cuts(sh, (int)std::min<long long>(units, 1 + rand() % 160));
        }
    }
    {
        std::vector<std::pair<int, int>> stack;
        for (int l = 0; l < 64; ++l) {
            stack.push_back({7168, 5120});
            stack.push_back({5120, 5120});
            stack.push_back({34816, 5120});
            stack.push_back({5120, 17408});
        }
        std::vector<int> every8{0, 32, 64, 96, 128, 160, 192, 224, 256};
        bad += check_chunks(stack, &every8);
        bad += check_chunks({{677, 2304}}, nullptr);
        bad += check_chunks({{256, 512}, {100000, 25600}, {128, 256}}, nullptr);
        srand(13);
        for (int it = 0; it < 300; ++it) {
            std::vector<std::pair<int, int>> sh;
            const int n = 1 + rand() % 300;
            for (int i = 0; i < n; ++i) sh.push_back({1 + rand() % 40000, 256 * (1 + rand() % 100)});
            bad += check_chunks(sh, nullptr);
        }
    }
    printf("bad=%d\n", bad);
    return bad != 0;
}
