// CPU check of the per-row selection logic of the fused score + top-k kernel
// (learned_block_sparse_pool_b200/csrc/select_rows.cuh), compiled for the host.
//
// For seeded rows of many kinds (Gaussian, skewed with a boosted block,
// integer-valued with heavy ties, constant, sorted, short) and budgets from 1
// to n, the rows go through the same passes the kernel runs -- strided
// sample, two counting passes under the fp16 map (on perturbed scores, as
// the kernel's reduced-precision products see them), collection of the band
// with an exact count of the scores above it, resolve, emit in index order -- and the kept list must equal a
// brute-force top-k
// (score descending, lowest index first on ties, emitted ascending).  Rows
// the logic marks as failed are finished by brute force, as the kernel's
// fallback does, and counted.  Prints "rows R failed F" and exits 0 when
// every row matches.
#include <math.h>
#include <stdio.h>
#include <stdlib.h>

#include <algorithm>
#include <random>
#include <vector>

#include "select_rows.cuh"

using namespace veda::rowsel;

static std::vector<int> brute(const std::vector<float>& s, int k)
{
    std::vector<int> o(s.size());
    for (size_t j = 0; j < s.size(); ++j) o[j] = (int)j;
    std::stable_sort(o.begin(), o.end(), [&](int a, int b) {
        // -0 == +0; NaN ranks lowest
        const bool na = s[a] != s[a], nb = s[b] != s[b];
        if (na || nb) return !na && nb;
        return s[a] > s[b];
    });
    o.resize(k);
    std::sort(o.begin(), o.end());
    return o;
}

// The kernel's passes on one row; returns false when the row falls back.
// Count pass A sees perturbed scores (as the kernel's reduced-precision
// tensor-core products do: relative errors up to eA); pass B, collection and
// emission see the exact ones (the kernel computes them identically).
static bool select_row(const std::vector<float>& s, int k, std::vector<int>& out, std::mt19937_64& rng,
                       float eA = 4e-3f, float eB = 0.0f)
{
    const int nk = (int)s.size();
    out.clear();
    if (k == nk) {
        for (int j = 0; j < nk; ++j) out.push_back(j);
        return true;
    }
    std::uniform_real_distribution<float> U(-1.f, 1.f);
    Row R;
    float v[kSample];
    for (int m = 0; m < kSample; ++m) v[m] = s[sample_pos(m, nk)];
    sort_desc<kSample>(v);
    plan_from_sorted(R, v, nk, k);
    for (int pass = 0; pass < 2; ++pass) {
        if (pass == 1) {
            plan_in_band(R, k);
            restart_ladder(R, nk);
        }
        const float e = pass == 0 ? eA : eB;
        int c[kM] = {};
        float gmax = -INFINITY, gmin = INFINITY;
        for (int j = 0; j < nk; ++j) {
            const float sj = s[j] * (1.0f + e * U(rng));
            const float gs = R.g(sj);
            for (int i = 0; i < kM; ++i) c[i] += gs >= R.t[i];
            gmax = fmaxf(gmax, gs);
            gmin = fminf(gmin, gs);
        }
        if (pass == 0) {
            R.gmax = gmax;
            R.gmin = gmin;
        }
        finish_count(R, c, k);
    }
    // collect (exact scores): the band and an exact count of the scores above it
    float band[kCap];
    for (int i = 0; i < kCap; ++i) band[i] = -INFINITY;
    int m = 0, above = 0;
    bool nan = false;
    for (int j = 0; j < nk; ++j) {
        nan |= s[j] != s[j];
        const float gs = R.g(s[j]);
        above += above_band(R, gs);
        if (in_band(R, gs)) {
            if (m < kCap) band[m] = s[j];
            ++m;
        }
    }
    sort_desc<kCap>(band);
    resolve_sorted(R, band, m, above, k, nan);
    if (R.fail) return false;
    int eq = 0;
    for (int j = 0; j < nk; ++j) {
        const bool sel = s[j] > R.tau || (s[j] == R.tau && eq < R.need);
        eq += s[j] == R.tau;
        if (sel) out.push_back(j);
    }
    return (int)out.size() == k;
}

int main()
{
    std::mt19937_64 rng(12345);
    std::normal_distribution<float> N01(0.f, 1.f);
    long rows = 0, failed = 0, bad = 0;
    const int sizes[] = {1, 2, 7, 64, 127, 128, 129, 200, 255, 256, 257, 500, 977, 1922, 2741, 4096};
    for (int n : sizes) {
        for (int kind = 0; kind < 7; ++kind) {
            for (int rep = 0; rep < 6; ++rep) {
                std::vector<float> s(n);
                for (int j = 0; j < n; ++j) {
                    float x = N01(rng);
                    switch (kind) {
                    case 0: break;                                              // Gaussian
                    case 1: x = 50.f + 0.001f * x; break;                       // large offset, tiny spread
                    case 2: x = (float)(int)(3.f * x); break;                   // integers: heavy ties
                    case 3: x = 1.f; break;                                     // constant row
                    case 4: x = (float)j * 0.01f + 0.001f * x; break;           // sorted with noise
                    case 5: if ((j / 7) % 20 == 3) x += 3.f; break;             // boosted blocks
                    case 6: x = x * x * x; break;                               // heavy tails
                    }
                    s[j] = x;
                }
                if (n > 3 && kind == 0 && rep == 5) s[n / 2] = -0.0f, s[n / 3] = 0.0f;
                const int ks[] = {1, 2, n / 20, n / 10, n / 2, n - 1, n, 16, 32, 64, 98, 138, 193, 549};
                for (int k : ks) {
                    if (k < 1 || k > n) continue;
                    std::vector<int> got;
                    ++rows;
                    if (!select_row(s, k, got, rng)) {
                        ++failed;
                        continue;       // the kernel finishes such a row on its materialised scores
                    }
                    if (got != brute(s, k)) {
                        if (++bad <= 5) fprintf(stderr, "mismatch: n %d kind %d rep %d k %d\n", n, kind, rep, k);
                    }
                }
            }
        }
    }
    // continuous rows must essentially never fall back
    long cont_rows = 0, cont_failed = 0;
    for (int t = 0; t < 2000; ++t) {
        const int n = 977 + (t % 3) * 882;   // 977, 1859, 2741
        const int k = (t % 2) ? (n + 9) / 10 : (n + 19) / 20;
        std::vector<float> s(n);
        for (auto& x : s) x = N01(rng);
        std::vector<int> got;
        ++cont_rows;
        if (!select_row(s, k, got, rng)) {
            ++cont_failed;
            continue;
        }
        if (got != brute(s, k)) ++bad;
    }
    printf("rows %ld failed %ld mismatched %ld continuous_rows %ld continuous_failed %ld\n", rows, failed, bad,
           cont_rows, cont_failed);
    return (bad == 0 && cont_failed * 50 <= cont_rows) ? 0 : 1;
}
