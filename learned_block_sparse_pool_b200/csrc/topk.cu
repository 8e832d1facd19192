// Fixed-budget top-k per score row (one warp per row).
//
// For every (b, h, query tile) row of fp32 tile scores, keep the k key tiles
// of highest score; equal scores go to the lowest tile index; emit the kept
// indices in ascending order.  Budgets are fixed counts per (query tile,
// head) (tao.media, "Affine launches MiniMax-H3 video studio...", section
// "How the SN120 Competition Works"; veyrul.com, "Veda R2VA for MiniMax-H3",
// second paragraph: 32 reference + 32 video tiles chosen independently).
//
// Algorithm (exact; no sorting), one warp per row:
//   1. Bracket: 256 keys sampled at a fixed stride give a lower bound `lo`
//      that, with a 3-sigma margin, at least k keys of the row reach.
//   2. One streaming pass over the row (coalesced loads, many in flight)
//      keeps every key >= lo, with its index, in a small candidate list in
//      shared memory, in index order.
//   3. If at least k keys were kept (and the list did not overflow), the
//      top-k set and every key tied with its smallest member are among them:
//      an 8-bit radix select over the candidates' order-preserving keys finds
//      the k-th largest key tau and how many keys equal to tau are still
//      needed, and one ballot pass over the candidates emits the kept indices
//      in ascending order (ties to the lowest index).  Otherwise (a skewed or
//      tied row) the same radix select runs over the whole row, re-read from
//      global memory, followed by an emit pass over the row.
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
constexpr int kCapMax = 2048;   // candidate-list capacity bound (shared memory)

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
// (cap) | candidate indices (cap); the sample (kSample keys) is held in the
// candidate region before the candidates are written.
__global__ void __launch_bounds__(32 * kWarps) topk_kernel(const TopkParams P, int cap, int r_lo)
{
    extern __shared__ uint32_t smem[];
    const int lane = threadIdx.x & 31;
    const int w = threadIdx.x >> 5;
    const int n = P.n, k = P.k;
    const int region = cap * 2 > kSample ? cap * 2 : kSample;
    uint32_t* hist = smem + (size_t)w * (NB + region);
    uint32_t* ckey = hist + NB;
    uint32_t* samp = ckey;
    int32_t* cidx = reinterpret_cast<int32_t*>(ckey + cap);
    const uint32_t lt_mask = (1u << lane) - 1u;
    const bool sampled = n > kSample && r_lo < kSample - 1;

    for (int64_t row = (int64_t)blockIdx.x * kWarps + w; row < P.rows;
         row += (int64_t)gridDim.x * kWarps) {
        const float* src = P.scores + row * P.ld;
        int32_t* dst = P.idx + row * (int64_t)k;

        if (k == n) {                       // every tile kept
            for (int e = lane; e < n; e += 32) dst[e] = e;
            continue;
        }

        // ---- 1. bracket from a strided sample ----
        uint32_t lo = 0u;                   // 0: keep everything
        if (sampled) {
            uint32_t smin = 0xffffffffu, smax = 0u;
#pragma unroll
            for (int m = 0; m < kSample / 32; ++m) {
                const int sidx = (int)(((int64_t)(lane + 32 * m) * n) / kSample);
                const uint32_t kk = order_key(__ldg(src + sidx));
                samp[lane + 32 * m] = kk;
                smin = min(smin, kk);
                smax = max(smax, kk);
            }
            smin = warp_min(smin);
            smax = warp_max(smax);
            __syncwarp();
            int dummy = 0;
            lo = radix_rank([&](int c) { return samp[c]; }, kSample, r_lo, smin, smax, hist, lane, &dummy);
        }

        // ---- 2. streaming pass: keys >= lo, with indices, in index order ----
        // chunks of 1024 keys: lane L holds keys 128u + 4L .. 128u + 4L + 3
        int nc = 0;
        uint32_t cmax = 0u, cmin = 0xffffffffu;
        for (int base = 0; base < n; base += 1024) {
            float4 v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int e = base + 128 * u + 4 * lane;
                v[u] = e < n ? __ldcs(reinterpret_cast<const float4*>(src + e))
                             : make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int e = base + 128 * u + 4 * lane;
                const float f[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
                uint32_t kk[4];
                int cnt = 0;
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    kk[c] = order_key(f[c]);
                    // past the end (the row's padding) never counts
                    if (e + c < n && kk[c] >= lo) ++cnt;
                }
                const uint32_t b0 = __ballot_sync(0xffffffffu, cnt & 1);
                const uint32_t b1 = __ballot_sync(0xffffffffu, cnt & 2);
                const uint32_t b2 = __ballot_sync(0xffffffffu, cnt & 4);
                int pos = nc + __popc(b0 & lt_mask) + 2 * __popc(b1 & lt_mask) + 4 * __popc(b2 & lt_mask);
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    if (e + c < n && kk[c] >= lo) {
                        if (pos < cap) {
                            ckey[pos] = kk[c];
                            cidx[pos] = e + c;
                        }
                        ++pos;
                        cmax = max(cmax, kk[c]);
                        cmin = min(cmin, kk[c]);
                    }
                }
                nc += __popc(b0) + 2 * __popc(b1) + 4 * __popc(b2);
            }
        }
        __syncwarp();

        // ---- 3. exact selection ----
        if (nc >= k && nc <= cap) {
            int need = 0;
            const uint32_t tau = radix_rank([&](int c) { return ckey[c]; }, nc, k - 1, warp_min(cmin),
                                            warp_max(cmax), hist, lane, &need);
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
    const int region = std::max(2 * cap, kSample);
    return sizeof(uint32_t) * (size_t)kWarps * (NB + (size_t)region);
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
    const int64_t need = (p.rows + kWarps - 1) / kWarps;
    if (grid > need) grid = need;
        const int r_lo = p.n > kSample ? bracket_rank(p.n, p.k) : kSample - 1;
    topk_kernel<<<(unsigned)grid, 32 * kWarps, smem, s>>>(p, cap, r_lo);
    return cudaGetLastError();
}

}  // namespace veda
