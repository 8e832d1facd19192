// Fixed-budget top-k per score row (one warp per row).
//
// For every (b, h, query tile) row of fp32 tile scores, keep the k key tiles
// of highest score; equal scores go to the lowest tile index; emit the kept
// indices in ascending order.  Budgets are fixed counts per (query tile,
// head) (tao.media, "Affine launches MiniMax-H3 video studio...", section
// "How the SN120 Competition Works"; veyrul.com, "Veda R2VA for MiniMax-H3",
// second paragraph: 32 reference + 32 video tiles chosen independently).
//
// Algorithm (exact; no sorting), one warp per row, on order-preserving
// 32-bit keys of the scores:
//   1. Bracket: 256 keys sampled at a fixed stride are binned linearly in key
//      space (one shared-memory histogram); the lower edge `lo` of the bin
//      holding the sample rank of the k-th largest key plus a 3-sigma margin
//      is a bound that, with high probability, at least k keys reach.
//   2. One streaming pass over the row (float4 loads, issued together with
//      the sample's) keeps every key >= lo, with its index, in a candidate
//      list in shared memory, in index order.
//   3. If at least k keys were kept (and the list did not overflow), the
//      top-k set and every key tied with its smallest member are among them.
//      The candidates are binned linearly between their smallest and largest
//      key; the bin b holding the k-th largest key is found from the
//      histogram, and the (at most 32) keys of bin b are ranked exactly
//      against each other, which gives the k-th largest key tau and how
//      many keys equal to tau are taken.  (A bin of more than 32 keys --
//      heavy ties -- falls back to an 8-bit radix select over the
//      candidates.)  One ballot pass over the candidates then emits the kept
//      indices in ascending order, ties to the lowest index.  If the bracket
//      missed, a radix select runs over the whole row, re-read from global
//      memory, followed by an emit pass over the row.
// The sample only decides how much work is done, never which tiles are kept.
// -0.0 and +0.0 are one key (a tie); NaN ranks below every number.
#include <algorithm>
#include <cmath>

#include "veda_internal.cuh"

namespace veda {
namespace {

constexpr int kWarps = 8;
constexpr int NB = 256;

__device__ __forceinline__ uint32_t order_key(float f)
{
    uint32_t u = __float_as_uint(f);
    if ((u & 0x7fffffffu) > 0x7f800000u) return 0u;    // NaN: lowest
    if (u == 0x80000000u) u = 0u;                       // -0 == +0
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Smallest digit value (from the top) at which the suffix count reaches
// `rem`: returns the digit and writes the count of strictly larger digits.
__device__ __forceinline__ int find_digit_from_top(const uint32_t* hist, int rem, int lane, int* above_out)
{
    uint32_t mine[NB / 32];
    uint32_t lane_sum = 0;
#pragma unroll
    for (int q = 0; q < NB / 32; ++q) {
        mine[q] = hist[lane * (NB / 32) + q];
        lane_sum += mine[q];
    }
    // inclusive suffix sum over lanes (lanes holding higher digits first)
    uint32_t suf = lane_sum;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const uint32_t o = __shfl_down_sync(0xffffffffu, suf, off);
        if (lane + off < 32) suf += o;
    }
    const uint32_t above_lane = suf - lane_sum;   // count in lanes > this lane
    const bool here = above_lane < (uint32_t)rem && suf >= (uint32_t)rem;
    int digit = -1, above = 0;
    if (here) {
        uint32_t cum = above_lane;
#pragma unroll
        for (int q = NB / 32 - 1; q >= 0; --q) {
            if (digit < 0 && cum + mine[q] >= (uint32_t)rem) {
                digit = lane * (NB / 32) + q;
                above = (int)cum;
            }
            cum += mine[q];
        }
    }
    const uint32_t who = __ballot_sync(0xffffffffu, here);
    const int src = who ? __ffs(who) - 1 : 0;   // a lane always matches when the counts cover rem
    digit = __shfl_sync(0xffffffffu, digit, src);
    above = __shfl_sync(0xffffffffu, above, src);
    *above_out = above;
    return digit < 0 ? 0 : digit;
}

__device__ __forceinline__ void clear_hist(uint32_t* hist, int lane)
{
#pragma unroll
    for (int q = 0; q < NB / 32; ++q) hist[lane + 32 * q] = 0u;
    __syncwarp();
}

constexpr int kSample = 256;
constexpr int kCapMax = 2048;
constexpr int kChunk = 512;     // keys per streaming step of a warp (float4 per lane x 128)   // candidate-list capacity bound (shared memory)

// Radix select over `cnt` keys provided by get(c) (c in [0, cnt)), all in
// [kmin, kmax]: returns the key tau of rank `rank` (0 = largest) and, through
// *need, how many keys equal to tau rank at or above `rank` (taking every key
// > tau plus the first *need keys == tau gives exactly rank + 1 keys).  The
// leading bytes that kmin and kmax share are skipped.
template <typename Get>
__device__ __forceinline__ uint32_t radix_rank(Get get, int cnt, int rank, uint32_t kmin, uint32_t kmax,
                                               uint32_t* hist, int lane, int* need)
{
    const uint32_t diff = kmin ^ kmax;
    int rem = rank + 1;
    if (diff == 0u) {                       // every key equal
        *need = rem;
        return kmax;
    }
    const int top = (31 - __clz(diff)) & ~7;   // shift of the highest differing byte
    uint32_t pmask = top == 24 ? 0u : ~0u << (top + 8);
    uint32_t prefix = kmax & pmask;
#pragma unroll 1
    for (int shift = top; shift >= 0; shift -= 8) {
        clear_hist(hist, lane);
        for (int c = lane; c < cnt; c += 32) {
            const uint32_t kk = get(c);
            if ((kk & pmask) == prefix) atomicAdd(&hist[(kk >> shift) & 255u], 1u);
        }
        __syncwarp();
        int ab = 0;
        const int dg = find_digit_from_top(hist, rem, lane, &ab);
        rem -= ab;
        prefix |= (uint32_t)dg << shift;
        pmask |= 255u << shift;
    }
    *need = rem;
    return prefix;
}

__device__ __forceinline__ uint32_t warp_min(uint32_t x) { return __reduce_min_sync(0xffffffffu, x); }
__device__ __forceinline__ uint32_t warp_max(uint32_t x) { return __reduce_max_sync(0xffffffffu, x); }

// Inverse of order_key for keys of numbers.
__device__ __forceinline__ float key_value(uint32_t k)
{
    return __uint_as_float((k & 0x80000000u) ? (k ^ 0x80000000u) : ~k);
}

// Linear bins in value between two finite values lo < hi: bin(v) =
// min(255, floor((v - lo) * 256 / (hi - lo))), non-decreasing in v (each step
// rounds monotonically).  `ok` is false when the range is not finite.
struct Bins {
    float lo, scale;
    bool ok;
    __device__ __forceinline__ Bins(uint32_t kmin, uint32_t kmax)
    {
        lo = key_value(kmin);
        const float hi = key_value(kmax);
        scale = 256.f / (hi - lo);
        ok = kmin != 0u && isfinite(lo) && isfinite(hi) && isfinite(scale) && scale > 0.f;
    }
    __device__ __forceinline__ uint32_t operator()(uint32_t k) const
    {
        return min(255u, (uint32_t)((key_value(k) - lo) * scale));
    }
};

// The k-th largest of `cnt` candidate keys (cnt >= k), all in [kmin, kmax],
// kmin < kmax: one histogram over linear value bins locates the bin holding
// it, and the bin's keys are ranked exactly against each other.  Returns
// false when the range is not finite or that bin holds more than 32 keys.  On success *tau is
// the k-th largest key and *need the number of keys equal to tau among the
// k largest (taking every key > tau and the first *need keys == tau in
// candidate order gives exactly k keys).
__device__ __forceinline__ bool bin_select(const uint32_t* ckey, int cnt, int k, uint32_t kmin, uint32_t kmax,
                                           uint32_t* hist, int lane, uint32_t* tau, int* need)
{
    const Bins bin(kmin, kmax);
    if (!bin.ok) return false;
    clear_hist(hist, lane);
    for (int c = lane; c < cnt; c += 32) atomicAdd(&hist[bin(ckey[c])], 1u);
    __syncwarp();
    int above = 0;
    const uint32_t b = (uint32_t)find_digit_from_top(hist, k, lane, &above);
    const int nb = (int)hist[b];
    __syncwarp();                                   // every lane has read the histogram
    if (nb > 32) return false;
    // gather bin b's keys (candidate order) into hist[0 .. nb)
    const uint32_t lt_mask = (1u << lane) - 1u;
    int pos = 0;
    for (int cb = 0; cb < cnt && pos < nb; cb += 32) {
        const int c = cb + lane;
        const uint32_t kk = c < cnt ? ckey[c] : 0u;
        const bool in = c < cnt && bin(kk) == b;
        const uint32_t bal = __ballot_sync(0xffffffffu, in);
        if (in) hist[pos + __popc(bal & lt_mask)] = kk;
        pos += __popc(bal);
    }
    __syncwarp();
    const int nb_need = k - above;                  // keys still to take from bin b (>= 1)
    const uint32_t mine = lane < nb ? hist[lane] : 0u;
    int gt = 0, ge = 0;
    for (int t = 0; t < nb; ++t) {
        const uint32_t x = hist[t];
        gt += x > mine;
        ge += x >= mine;
    }
    const uint32_t hit = __ballot_sync(0xffffffffu, lane < nb && gt < nb_need && nb_need <= ge);
    const int src = __ffs(hit) - 1;                 // some key of the bin has this rank
    *tau = __shfl_sync(0xffffffffu, mine, src);
    *need = nb_need - __shfl_sync(0xffffffffu, gt, src);
    __syncwarp();
    return true;
}

// Lower bracket rank in a sample of kSample keys for budget k of n: the
// expected sample rank of the k-th largest key plus three standard deviations
// (binomial) and a small constant.
__host__ __device__ __forceinline__ int bracket_rank(int n, int k)
{
    const double q = (double)k / (double)n;
    const double mean = q * kSample;
    const double sd = sqrt(kSample * q * (1.0 - q));
    const int r = (int)(mean + 3.0 * sd + 3.0);
    return r < kSample - 1 ? r : kSample - 1;
}

// One warp per row.  Per-warp shared memory: histogram | candidate keys
// (cap + 1) | candidate indices (cap + 1); entry cap is a spare slot that
// absorbs the stores of entries not kept.
__global__ void __launch_bounds__(32 * kWarps, 4) topk_kernel(const TopkParams P, int cap, int r_lo)
{
    extern __shared__ uint32_t smem[];
    const int lane = threadIdx.x & 31;
    const int w = threadIdx.x >> 5;
    const int n = P.n, k = P.k;
    uint32_t* hist = smem + (size_t)w * (NB + 2 * (cap + 1));
    uint32_t* ckey = hist + NB;
    int32_t* cidx = reinterpret_cast<int32_t*>(ckey + cap + 1);
    const uint32_t lt_mask = (1u << lane) - 1u;
    const bool sampled = n > kSample && r_lo < kSample - 1;

    const int64_t n_rows = P.row_list ? (int64_t)*P.row_count : P.rows;
    for (int64_t rr = (int64_t)blockIdx.x * kWarps + w; rr < n_rows; rr += (int64_t)gridDim.x * kWarps) {
        const int64_t row = P.row_list ? (int64_t)P.row_list[rr] : rr;
        const float* src = P.scores + row * P.ld;
        int32_t* dst = P.idx + row * (int64_t)k;

        if (k == n) {                       // every tile kept
            for (int e = lane; e < n; e += 32) dst[e] = e;
            continue;
        }

        // ---- 1. loads of the first kChunk keys and of the strided sample ----
        // lane L holds keys 128u + 4L .. 128u + 4L + 3 of each kChunk-key chunk
        float4 v[kChunk / 128];
        auto load_chunk = [&](int base) {
#pragma unroll
            for (int u = 0; u < kChunk / 128; ++u) {
                const int e = base + 128 * u + 4 * lane;
                v[u] = e < n ? __ldcs(reinterpret_cast<const float4*>(src + e))
                             : make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
            }
        };
        load_chunk(0);
        uint32_t lo = 0u;                   // 0: keep everything
        if (sampled) {
            uint32_t sk[kSample / 32];
#pragma unroll
            for (int m = 0; m < kSample / 32; ++m) sk[m] = order_key(__ldg(src + ((lane + 32 * m) * n) / kSample));
            uint32_t smin = sk[0], smax = sk[0];
#pragma unroll
            for (int m = 1; m < kSample / 32; ++m) {
                smin = min(smin, sk[m]);
                smax = max(smax, sk[m]);
            }
            smin = warp_min(smin);
            smax = warp_max(smax);
            const Bins bin(smin, smax);
            if (smin == smax) {
                lo = smin;
            } else if (bin.ok) {
                clear_hist(hist, lane);
                uint32_t sbin[kSample / 32];
#pragma unroll
                for (int m = 0; m < kSample / 32; ++m) {
                    sbin[m] = bin(sk[m]);
                    atomicAdd(&hist[sbin[m]], 1u);
                }
                __syncwarp();
                int dummy = 0;
                const uint32_t b = (uint32_t)find_digit_from_top(hist, r_lo + 1, lane, &dummy);
                // the smallest sample in bins >= b: at least r_lo + 1 samples reach it
                uint32_t m_lo = 0xffffffffu;
#pragma unroll
                for (int m = 0; m < kSample / 32; ++m)
                    if (sbin[m] >= b) m_lo = min(m_lo, sk[m]);
                lo = warp_min(m_lo);
            }
        }

        // ---- 2. streaming pass: scores >= value(lo), with indices, in index order ----
        // For lo > 0 (the key of a number) the test key >= lo is the float test
        // v >= value(lo): NaN fails both, and -0 / +0 compare equal in both.
        // The scores are kept as they are; their keys are formed afterwards,
        // for the kept ones only.
        const bool keep_all = lo == 0u;
        const float lo_f = keep_all ? 0.f : key_value(lo);
        int nc = 0;
        for (int base = 0; base < n; base += kChunk) {
            if (base > 0) load_chunk(base);
            const bool full = base + kChunk <= n;               // no row end in this chunk
#pragma unroll
            for (int u = 0; u < kChunk / 128; ++u) {
                const int e = base + 128 * u + 4 * lane;
                const float f[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
                bool in[4];
                int cnt = 0;
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    // past the end (the row's padding) never counts
                    in[c] = (full || e + c < n) && (keep_all || f[c] >= lo_f);
                    cnt += in[c];
                }
                const uint32_t b0 = __ballot_sync(0xffffffffu, cnt & 1);
                const uint32_t b1 = __ballot_sync(0xffffffffu, cnt & 2);
                const uint32_t b2 = __ballot_sync(0xffffffffu, cnt & 4);
                int pos = nc + __popc(b0 & lt_mask) + 2 * __popc(b1 & lt_mask) + 4 * __popc(b2 & lt_mask);
                // branch-free: entries that are not kept, or past the list's
                // capacity, go to the spare slot `cap`
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const int slot = in[c] ? min(pos, cap) : cap;
                    ckey[slot] = __float_as_uint(f[c]);
                    cidx[slot] = e + c;
                    pos += in[c];
                }
                nc += __popc(b0) + 2 * __popc(b1) + 4 * __popc(b2);
            }
        }
        __syncwarp();
        // keys of the kept scores, and their range
        uint32_t cmax = 0u, cmin = 0xffffffffu;
        if (nc <= cap) {
            for (int c = lane; c < nc; c += 32) {
                const uint32_t kk = order_key(__uint_as_float(ckey[c]));
                ckey[c] = kk;
                cmax = max(cmax, kk);
                cmin = min(cmin, kk);
            }
            __syncwarp();
        }

        // ---- 3. exact selection ----
        if (nc >= k && nc <= cap) {
            const uint32_t kmin = warp_min(cmin), kmax = warp_max(cmax);
            int need = k;
            uint32_t tau = kmax;            // all candidates equal: the first k
            if (kmin != kmax && !bin_select(ckey, nc, k, kmin, kmax, hist, lane, &tau, &need))
                tau = radix_rank([&](int c) { return ckey[c]; }, nc, k - 1, kmin, kmax, hist, lane, &need);
            int out = 0, eq_seen = 0;
            for (int cb = 0; cb < nc && out < k; cb += 32) {
                const int c = cb + lane;
                const bool valid = c < nc;
                const uint32_t kk = valid ? ckey[c] : 0u;
                const bool gt = valid && kk > tau;
                const bool eq = valid && kk == tau;
                const uint32_t eqb = __ballot_sync(0xffffffffu, eq);
                const bool sel = gt || (eq && eq_seen + __popc(eqb & lt_mask) < need);
                const uint32_t selb = __ballot_sync(0xffffffffu, sel);
                const int slot = out + __popc(selb & lt_mask);
                if (sel && slot < k) dst[slot] = cidx[c];
                out += __popc(selb);
                eq_seen += __popc(eqb);
            }
        } else {                            // bracket missed: select over the whole row
            uint32_t rmin = 0xffffffffu, rmax = 0u;
            for (int e = lane; e < n; e += 32) {
                const uint32_t kk = order_key(__ldcg(src + e));
                rmin = min(rmin, kk);
                rmax = max(rmax, kk);
            }
            int need = 0;
            const uint32_t tau = radix_rank([&](int c) { return order_key(__ldcg(src + c)); }, n, k - 1,
                                            warp_min(rmin), warp_max(rmax), hist, lane, &need);
            int out = 0, eq_seen = 0;
            for (int base = 0; base < n && out < k; base += 32) {
                const int e = base + lane;
                const bool valid = e < n;
                const uint32_t kk = valid ? order_key(__ldcg(src + e)) : 0u;
                const bool gt = valid && kk > tau;
                const bool eq = valid && kk == tau;
                const uint32_t eqb = __ballot_sync(0xffffffffu, eq);
                const bool sel = gt || (eq && eq_seen + __popc(eqb & lt_mask) < need);
                const uint32_t selb = __ballot_sync(0xffffffffu, sel);
                const int slot = out + __popc(selb & lt_mask);
                if (sel && slot < k) dst[slot] = e;
                out += __popc(selb);
                eq_seen += __popc(eqb);
            }
        }
        __syncwarp();
    }
}

// Candidate-list capacity for a row length and budget: about twice the
// expected number of keys at or above the bracket, at least k + 64, at most
// the row length and kCapMax.
int topk_capacity(int n, int k)
{
    if (n <= kSample) return n;
    const int expect = (int)ceil((double)n * (bracket_rank(n, k) + 1) / kSample);
    return std::min(std::min(n, kCapMax), std::max(k + 64, 2 * expect + 32));
}

size_t topk_smem_bytes(int n, int k)
{
    const int cap = topk_capacity(n, k);
    return sizeof(uint32_t) * (size_t)kWarps * (NB + 2 * ((size_t)cap + 1));
}

}  // namespace

int topk_max_tiles() { return 32 * 128; }

cudaError_t launch_topk(const TopkParams& p, cudaStream_t s)
{
    if (p.rows == 0) return cudaSuccess;
    if (p.n > topk_max_tiles()) return cudaErrorInvalidValue;
    // rows are read as float4: 16-byte aligned, stride a multiple of 4
    if ((reinterpret_cast<uintptr_t>(p.scores) & 15u) != 0 || (p.ld & 3) != 0 || p.ld < p.n)
        return cudaErrorInvalidValue;
    const int cap = topk_capacity(p.n, p.k);
    const size_t smem = topk_smem_bytes(p.n, p.k);
    cudaError_t e = cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, topk_kernel, 32 * kWarps, smem);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) per_sm = 1;
    int64_t grid = (int64_t)num_sms() * per_sm;
    const int64_t need = (p.rows + kWarps - 1) / kWarps;   // a row list is never longer than `rows`
    if (grid > need) grid = need;
    if (p.row_list && !p.row_count) return cudaErrorInvalidValue;
    const int r_lo = p.n > kSample ? bracket_rank(p.n, p.k) : kSample - 1;
    topk_kernel<<<(unsigned)grid, 32 * kWarps, smem, s>>>(p, cap, r_lo);
    return cudaGetLastError();
}

}  // namespace veda
