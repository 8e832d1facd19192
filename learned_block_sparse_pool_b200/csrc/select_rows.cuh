// Per-row logic of the fused score + top-k selection (tile_select_kernel):
// exact fixed-budget top-k of one row of tile scores that is seen only in
// chunks, several times over (the scores are recomputed on the tensor cores
// for every pass instead of being stored).
//
// For one (b, h, query tile) row of nk scores and a budget k it finds the
// k-th largest score tau and how many scores equal to tau are kept, so that
// a last pass in index order can emit the kept tiles ascending, ties to the
// lowest index (tao.media, "Affine launches MiniMax-H3 video studio...",
// section "How the SN120 Competition Works": fixed block budgets per query
// tile and head).  The passes:
//   sample  64 scores spread evenly over the row, sorted, give thresholds
//           around the expected rank of the k-th score and a monotone map g
//           (an affine map rounded to fp16) under which scores are counted;
//   count A how many scores reach each of 8 thresholds: the k-th score lies
//           between two neighbouring ones (the band); the row's largest and
//           smallest g are noted too;
//   count B 8 thresholds across that band (and a little past its ends),
//           denser where the k-th score is expected, narrow it again from
//           their counts alone;
//   collect the band's exact scores (at most kCap) are kept on chip and the
//           scores above the band are counted exactly;
//   resolve tau = the (k - above)-th largest band score;
//   emit    every score > tau, and the first `need` scores == tau.
// Count pass A only guides pass B, so it may see approximate scores; pass B
// re-derives the band from its own counts (restart_ladder), and the count of
// scores above the band is taken again while collecting.  Any monotone g gives the same result (it only decides which
// scores are looked at exactly), so the fp16 rounding cannot change the kept
// set.  A row whose band does not fit, whose exact counts put the k-th score
// outside the band, or that holds a NaN, is marked failed and finished by
// the exact warp-per-row top-k on its materialised scores.
//
// This header compiles for the device (nvcc) and for the host (a plain C++
// compiler), so the logic is tested on the CPU against a brute-force top-k.
#pragma once

#include <math.h>
#include <stdint.h>

#if defined(__CUDACC__)
#include <cuda_fp16.h>
#define VEDA_HD __host__ __device__ __forceinline__
#else
#define VEDA_HD inline
#endif

namespace veda {
namespace rowsel {

constexpr int kSample = 64;    // scores in the sample chunk
constexpr int kM = 8;          // thresholds per counting pass
constexpr int kCap = 64;       // band scores kept per row

// Round a float to the nearest fp16 value (ties to even), returned as float;
// overflow gives +-inf.  The device uses the hardware conversion; the host
// version rounds the same way in software.
VEDA_HD float f16_round(float x)
{
#if defined(__CUDA_ARCH__)
    return __half2float(__float2half_rn(x));
#else
    if (x != x) return x;
    const float a = fabsf(x);
    if (a >= 65520.0f) return x > 0 ? INFINITY : -INFINITY;
    float q;                                       // the fp16 quantum at |x|
    if (a < 6.103515625e-05f) {
        q = 5.9604644775390625e-08f;               // 2^-24: subnormal spacing
    } else {
        int e;
        frexpf(a, &e);                             // a in [2^(e-1), 2^e)
        q = ldexpf(1.0f, e - 11);                  // 11 significant bits
    }
    const float r = nearbyintf(a / q) * q;         // a / q is exact (power-of-two scale)
    return x < 0 ? -r : r;
#endif
}

struct Map {
    float scale, bias;                 // g(s) = f16_round(fma(s, scale, bias)), scale > 0
    VEDA_HD float operator()(float s) const { return f16_round(fmaf(s, scale, bias)); }
};

// Key tile of sample m (0 <= m < kSample) of a row of nk tiles: evenly
// spread over the row at the fractional stride nk / kSample (a whole-tile
// stride of about one frame's worth of tiles would sample the same place of
// every frame).
VEDA_HD int sample_pos(int m, int nk)
{
    return (int)(((int64_t)m * nk) / kSample);
}

// Bitonic sort of N values (N a power of two), descending.  Every index is a
// compile-time constant once unrolled, so the array stays in registers.
template <int N>
VEDA_HD void sort_desc(float (&v)[N])
{
#pragma unroll
    for (int k = 2; k <= N; k <<= 1) {
#pragma unroll
        for (int j = k >> 1; j > 0; j >>= 1) {
#pragma unroll
            for (int i = 0; i < N; ++i) {
                const int l = i ^ j;
                if (l > i) {
                    const float a = v[i], b = v[l];
                    const float hi = fmaxf(a, b), lo = fminf(a, b);
                    const bool desc = (i & k) == 0;
                    v[i] = desc ? hi : lo;
                    v[l] = desc ? lo : hi;
                }
            }
        }
    }
}

// Value at position `r` (0-based) of a register array, by a full scan (so
// the array is never indexed dynamically).
template <int N>
VEDA_HD float pick(const float (&v)[N], int r)
{
    float x = v[0];
#pragma unroll
    for (int i = 1; i < N; ++i) x = (i == r) ? v[i] : x;
    return x;
}

VEDA_HD int iround(float x) { return (int)floorf(x + 0.5f); }
VEDA_HD int clampi(int x, int a, int b) { return x < a ? a : (x > b ? b : x); }

struct Row {
    Map g;
    float t[kM];        // thresholds of the current counting pass, in g units, non-increasing
    float hi, lo;       // current band [lo, hi) in g units
    bool open_top;      // the band has no upper bound (hi = +inf, +inf included)
    int above;          // #(g(s) >= hi), or 0 when open_top
    int band;           // #(lo <= g(s) < hi)
    float gmax, gmin;   // largest and smallest g(s) of the row (count pass A)
    float tau;          // the k-th largest score
    int need;           // scores == tau that are kept
    bool fail;
};

// Sample pass: v = the sampled scores sorted descending, nk the row length,
// k the budget (1 <= k < nk).  Sets the map g and the thresholds of count
// pass A at sample ranks spanning the expected rank of the k-th score +- 3
// binomial standard deviations (and 2 ranks).
VEDA_HD void plan_from_sorted(Row& R, const float (&v)[kSample], int nk, int k)
{
    const float q = (float)k / (float)nk;
    const float rank = q * kSample - 1.0f;                     // expected sample rank of the k-th score
    const float sd = sqrtf(kSample * q * (1.0f - q));
    const float r_lo = rank - 3.0f * sd - 2.0f, r_hi = rank + 3.0f * sd + 2.0f;
    int rk[kM];
#pragma unroll
    for (int i = 0; i < kM; ++i)
        rk[i] = clampi(iround(r_lo + (r_hi - r_lo) * (float)i / (float)(kM - 1)), 0, kSample - 1);
    const float c = pick<kSample>(v, clampi(iround(rank), 0, kSample - 1));
    const float top = pick<kSample>(v, rk[0]), bot = pick<kSample>(v, rk[kM - 1]);
    const float span = top - bot, range = v[0] - v[kSample - 1];
    // the bracket spans 2048 fp16 units, unless that would push the sample's
    // whole range (times 4) past fp16's reach: the row's extremes must stay
    // finite for count pass B
    float scale = (span > 0.0f && isfinite(span)) ? 2048.0f / span : 1.0f;
    if (range > 0.0f && isfinite(range)) scale = fminf(scale, 8192.0f / range);
    R.g.scale = scale;
    // + 0.0f: a bias of -0 would map the scores -0 and +0 to different g
    R.g.bias = (isfinite(c) ? -c * R.g.scale : 0.0f) + 0.0f;
#pragma unroll
    for (int i = 0; i < kM; ++i) R.t[i] = R.g(pick<kSample>(v, rk[i]));
    R.gmax = R.g(v[0]);          // until count pass A has seen the whole row
    R.gmin = R.g(v[kSample - 1]);
    R.hi = INFINITY;
    R.lo = -INFINITY;
    R.open_top = true;
    R.above = 0;
    R.band = nk;
    R.fail = false;
}

// End of a counting pass: c[i] = #(g(s) >= t[i]).  The ladder is the current
// band's top (count `above`), the thresholds, and its bottom (count
// above + band); the new band lies between the first rung whose count
// reaches k and the rung above it.
VEDA_HD void finish_count(Row& R, const int (&c)[kM], int k)
{
    float L_hi = R.hi;
    bool open = R.open_top;
    int C_hi = R.above;
    bool found = false;
#pragma unroll
    for (int i = 0; i < kM; ++i) {
        if (!found && c[i] >= k) {
            R.lo = R.t[i];
            R.band = c[i] - C_hi;
            R.hi = L_hi;
            R.open_top = open;
            R.above = C_hi;
            found = true;
        }
        if (!found) {
            L_hi = R.t[i];
            C_hi = c[i];
            open = false;
        }
    }
    if (!found) {   // below the last threshold: [old lo, t[kM-1])
        R.band = R.above + R.band - C_hi;
        R.hi = L_hi;
        R.open_top = open;
        R.above = C_hi;
    }
}

// Thresholds of count pass B around the band [lo, hi) of pass A (an
// unbounded side is replaced by the row's extreme seen in pass A): centred on
// where the k-th score would lie if the band's scores were spread evenly (the
// (k - above)-th of `band` from the top), at offsets of 4 % to 55 % of the
// band's width on either side (finer where the k-th score is expected), and
// reaching past both ends, so that pass A's counts (which may come from
// approximate scores) are not needed to place the k-th score.
// The band is then re-derived from pass B's counts alone (restart_ladder).
VEDA_HD void plan_in_band(Row& R, int k)
{
    const float hi = R.open_top ? fmaxf(R.gmax, R.lo) : R.hi;
    const float lo = isinf(R.lo) ? fminf(R.gmin, hi) : R.lo;
    const float w = hi - lo;
    const float f = ((float)(k - R.above) - 0.5f) / (float)(R.band > 0 ? R.band : 1);
    const float xc = hi - f * w;
    const float off[kM] = {0.55f, 0.3f, 0.12f, 0.04f, -0.04f, -0.12f, -0.3f, -0.55f};
    // past the ends: 5 % of the width, and at least 16 g units (about 1 % of
    // the sampled bracket), which covers the error of pass A's approximate
    // scores when the band is very narrow (a budget of one or two tiles)
    const float mg = 0.05f * w + 16.0f;
#pragma unroll
    for (int i = 0; i < kM; ++i) R.t[i] = f16_round(fminf(fmaxf(xc + off[i] * w, lo - mg), hi + mg));
#pragma unroll
    for (int i = 1; i < kM; ++i) R.t[i] = fminf(R.t[i], R.t[i - 1]);   // non-increasing after rounding
}

// Forget the band before a counting pass whose counts alone place the k-th
// score (the ladder is then +inf, the thresholds, -inf).
VEDA_HD void restart_ladder(Row& R, int nk)
{
    R.hi = INFINITY;
    R.lo = -INFINITY;
    R.open_top = true;
    R.above = 0;
    R.band = nk;
}

VEDA_HD bool in_band(const Row& R, float gs)
{
    return gs >= R.lo && (R.open_top || gs < R.hi);
}

VEDA_HD bool above_band(const Row& R, float gs)
{
    return !R.open_top && gs >= R.hi;
}

// Resolve: v = the m collected band scores (m <= kCap) padded with -inf and
// sorted descending; above = the exact count of scores over the band.  Sets
// tau and need, or marks the row failed when the band was not collected
// whole, does not hold the k-th score, or holds a NaN.
VEDA_HD void resolve_sorted(Row& R, const float (&v)[kCap], int m, int above, int k, bool saw_nan)
{
    const int r = k - above;
    if (R.fail || saw_nan || m > kCap || r < 1 || r > m) {
        R.fail = true;
        return;
    }
    R.tau = pick<kCap>(v, r - 1);
    int gt = 0;
#pragma unroll
    for (int i = 0; i < kCap; ++i) gt += (i < m && v[i] > R.tau) ? 1 : 0;
    R.need = r - gt;
}

}  // namespace rowsel
}  // namespace veda
