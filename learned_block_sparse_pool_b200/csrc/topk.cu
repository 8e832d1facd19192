// Fixed-budget top-k per score row (one warp per row).
//
// For every (b, h, query tile) row of fp32 tile scores, keep the k key tiles
// of highest score; equal scores go to the lowest tile index; emit the kept
// indices in ascending order.  Budgets are fixed counts per (query tile,
// head) (tao.media, "Affine launches MiniMax-H3 video studio...", section
// "How the SN120 Competition Works"; veyrul.com, "Veda R2VA for MiniMax-H3",
// second paragraph: 32 reference + 32 video tiles chosen independently).
//
// Algorithm (exact; no sorting):
//   1. The warp loads its row once (coalesced 4-byte lanes, all loads in
//      flight) into registers, with the row's min and max.
//   2. A 256-bucket histogram over a monotone linear map of [min, max]
//      locates the bucket b* holding the k-th largest score.  Buckets are
//      monotone in the value, so every element of a higher bucket is
//      strictly larger than every element of b*, and equal values share a
//      bucket.
//   3. The few elements of b* are compacted to shared memory and an 8-bit
//      radix select over their order-preserving 32-bit keys finds the exact
//      k-th largest key tau and how many elements equal to tau are still
//      needed.  (If b* holds too many elements -- near-constant rows -- the
//      radix select runs over the whole row instead.)
//   4. One pass in index order emits key > tau, plus the first `need` keys
//      equal to tau: warp ballots give each lane its output slot, so the
//      list is written ascending and coalesced.
// -0.0 and +0.0 are one key (a tie); NaN ranks below every number.
#include <float.h>

#include "veda_internal.cuh"

namespace veda {
namespace {

constexpr int kWarps = 8;
constexpr int NB = 256;
constexpr int kCandMax = 512;

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

template <int PL>   // elements per lane held in registers (n <= 32 * PL)
__global__ void __launch_bounds__(32 * kWarps) topk_kernel(const TopkParams P)
{
    __shared__ uint32_t hist_s[kWarps][NB];
    __shared__ uint32_t cand_s[kWarps][kCandMax];
    const int lane = threadIdx.x & 31;
    const int w = threadIdx.x >> 5;
    uint32_t* hist = hist_s[w];
    uint32_t* cand = cand_s[w];
    const uint32_t lt_mask = (1u << lane) - 1u;
    const int n = P.n;

    for (int64_t row = (int64_t)blockIdx.x * kWarps + w; row < P.rows;
         row += (int64_t)gridDim.x * kWarps) {
        const float* src = P.scores + row * P.ld;
        float v[PL];
#pragma unroll
        for (int m = 0; m < PL; ++m) {
            const int e = lane + 32 * m;
            v[m] = (e < n) ? __ldcs(src + e) : 0.f;
        }
        float lo = FLT_MAX, hi = -FLT_MAX;
#pragma unroll
        for (int m = 0; m < PL; ++m) {
            const int e = lane + 32 * m;
            if (e < n && v[m] == v[m]) {
                lo = fminf(lo, v[m]);
                hi = fmaxf(hi, v[m]);
            }
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, off));
            hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, off));
        }
        float sc = 0.f;
        if (hi > lo) {
            const float range = hi - lo;
            if (range < FLT_MAX) sc = ((float)NB * 0.999999f) / range;
        }

        // ---- 2. bucket histogram ----
        clear_hist(hist, lane);
#pragma unroll
        for (int m = 0; m < PL; ++m) {
            const int e = lane + 32 * m;
            if (e < n) {
                const float f = (v[m] == v[m]) ? v[m] : lo;
                const int bk = min(NB - 1, max(0, (int)((f - lo) * sc)));
                atomicAdd(&hist[bk], 1u);
            }
        }
        __syncwarp();
        int above = 0;
        const int bstar = find_digit_from_top(hist, P.k, lane, &above);
        int rem = P.k - above;          // kept elements still to take from bucket b*

        // ---- 3. candidates of b*, exact k-th key by radix select ----
        int nc = 0;
#pragma unroll
        for (int m = 0; m < PL; ++m) {
            const int e = lane + 32 * m;
            bool in = false;
            if (e < n) {
                const float f = (v[m] == v[m]) ? v[m] : lo;
                in = min(NB - 1, max(0, (int)((f - lo) * sc))) == bstar;
            }
            const uint32_t bal = __ballot_sync(0xffffffffu, in);
            const int pos = nc + __popc(bal & lt_mask);
            if (in && pos < kCandMax) cand[pos] = order_key(v[m]);
            nc += __popc(bal);
        }
        __syncwarp();
        const bool small = nc <= kCandMax;
        uint32_t prefix = 0u, pmask = 0u;
        if (!small) rem = P.k;          // fall back: radix select over the whole row
#pragma unroll 1
        for (int shift = 24; shift >= 0; shift -= 8) {
            clear_hist(hist, lane);
            if (small) {
                for (int c = lane; c < nc; c += 32) {
                    const uint32_t key = cand[c];
                    if ((key & pmask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
                }
            } else {
#pragma unroll
                for (int m = 0; m < PL; ++m) {
                    const int e = lane + 32 * m;
                    const uint32_t key = order_key(v[m]);
                    if (e < n && (key & pmask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
                }
            }
            __syncwarp();
            int ab = 0;
            const int dgt = find_digit_from_top(hist, rem, lane, &ab);
            rem -= ab;
            prefix |= (uint32_t)dgt << shift;
            pmask |= 255u << shift;
        }
        const uint32_t tau = prefix;
        const int need = rem;           // keys equal to tau to keep, lowest index first

        // ---- 4. emit in index order ----
        int32_t* dst = P.idx + row * (int64_t)P.k;
        int out = 0, eq_seen = 0;
#pragma unroll
        for (int m = 0; m < PL; ++m) {
            const int e = lane + 32 * m;
            const uint32_t key = order_key(v[m]);
            const bool valid = e < n;
            const bool gt = valid && key > tau;
            const bool eq = valid && key == tau;
            const uint32_t eqb = __ballot_sync(0xffffffffu, eq);
            const bool sel = gt || (eq && eq_seen + __popc(eqb & lt_mask) < need);
            const uint32_t selb = __ballot_sync(0xffffffffu, sel);
            const int slot = out + __popc(selb & lt_mask);
            if (sel && slot < P.k) dst[slot] = e;
            out += __popc(selb);
            eq_seen += __popc(eqb);
        }
        __syncwarp();
    }
}

template <int PL>
cudaError_t launch_pl(const TopkParams& p, cudaStream_t s)
{
    int per_sm = 0;
    cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, topk_kernel<PL>, 32 * kWarps, 0);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) per_sm = 1;
    int64_t grid = (int64_t)num_sms() * per_sm;
    const int64_t need = (p.rows + kWarps - 1) / kWarps;
    if (grid > need) grid = need;
    topk_kernel<PL><<<(unsigned)grid, 32 * kWarps, 0, s>>>(p);
    return cudaGetLastError();
}

}  // namespace

int topk_max_tiles() { return 32 * 128; }

cudaError_t launch_topk(const TopkParams& p, cudaStream_t s)
{
    if (p.rows == 0) return cudaSuccess;
    if (p.n <= 32 * 4) return launch_pl<4>(p, s);
    if (p.n <= 32 * 16) return launch_pl<16>(p, s);
    if (p.n <= 32 * 32) return launch_pl<32>(p, s);
    if (p.n <= 32 * 64) return launch_pl<64>(p, s);
    if (p.n <= 32 * 96) return launch_pl<96>(p, s);
    if (p.n <= 32 * 128) return launch_pl<128>(p, s);
    return cudaErrorInvalidValue;
}

}  // namespace veda
