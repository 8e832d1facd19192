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
//      flight) into registers as order-preserving 32-bit keys, and reduces
//      the row's smallest and largest key.
//   2. Radix select on the key bits below the row's common prefix (the bits
//      where the smallest and largest key agree are shared by every key), 8
//      bits at a time, most significant first: a 256-bin shared-memory
//      histogram locates the digit holding the k-th largest key.  After the
//      first digit the (few) keys still matching the prefix are compacted to
//      shared memory and the remaining digits are resolved over them only.
//      The result is the exact k-th largest key tau and how many keys equal
//      to tau are still needed.
//   3. One pass in index order emits key > tau, plus the first `need` keys
//      equal to tau: warp ballots give each lane its output slot, so the
//      list is written ascending and coalesced.

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

// One warp per row; the row's keys live in this warp's slice of dynamic
// shared memory (lane-strided: key e at keys[e]).
__global__ void __launch_bounds__(32 * kWarps) topk_kernel(const TopkParams P)
{
    extern __shared__ uint32_t smem[];
    const int lane = threadIdx.x & 31;
    const int w = threadIdx.x >> 5;
    const int n = P.n;
    const int nkeys = (n + 31) & ~31;
    uint32_t* hist = smem + (size_t)w * (NB + kCandMax + nkeys);
    uint32_t* cand = hist + NB;
    uint32_t* keys = cand + kCandMax;
    const uint32_t lt_mask = (1u << lane) - 1u;

    for (int64_t row = (int64_t)blockIdx.x * kWarps + w; row < P.rows;
         row += (int64_t)gridDim.x * kWarps) {
        const float* src = P.scores + row * P.ld;
        // ---- load: keys to shared memory, smallest and largest key ----
        uint32_t kmin = 0xffffffffu, kmax = 0u;
#pragma unroll 8
        for (int e = lane; e < n; e += 32) {
            const uint32_t kk = order_key(__ldcs(src + e));
            keys[e] = kk;
            kmin = min(kmin, kk);
            kmax = max(kmax, kk);
        }
        kmin = __reduce_min_sync(0xffffffffu, kmin);
        kmax = __reduce_max_sync(0xffffffffu, kmax);
        __syncwarp();

        uint32_t tau;
        int need;
        if (kmin == kmax) {            // every key equal: the first k indices
            tau = kmin;
            need = P.k;
        } else {
            const int top = 31 - __clz(kmin ^ kmax);             // highest bit where keys differ
            uint32_t pmask = top == 31 ? 0u : ~((1u << (top + 1)) - 1u);
            uint32_t prefix = kmin & pmask;                       // shared by every key
            int rem = P.k;
            int shift = top >= 7 ? top - 7 : 0;
            // ---- first digit over the whole row ----
            clear_hist(hist, lane);
#pragma unroll 4
            for (int e = lane; e < n; e += 32) atomicAdd(&hist[(keys[e] >> shift) & 255u], 1u);
            __syncwarp();
            {
                int ab = 0;
                const int dg = find_digit_from_top(hist, rem, lane, &ab);
                rem -= ab;
                pmask |= 255u << shift;
                prefix = (prefix & ~(255u << shift)) | ((uint32_t)dg << shift);
            }
            // ---- compact the keys that still match ----
            int nc = 0;
            for (int base = 0; base < n; base += 32) {
                const int e = base + lane;
                const uint32_t kk = e < n ? keys[e] : 0u;
                const bool in = (e < n) && (kk & pmask) == prefix;
                const uint32_t bal = __ballot_sync(0xffffffffu, in);
                const int pos = nc + __popc(bal & lt_mask);
                if (in && pos < kCandMax) cand[pos] = kk;
                nc += __popc(bal);
            }
            __syncwarp();
            const bool small = nc <= kCandMax;
            const uint32_t* pool = small ? cand : keys;
            const int npool = small ? nc : n;
            // ---- remaining digits, over the candidates (or the row) ----
#pragma unroll 1
            while (shift > 0) {
                const int nshift = shift >= 8 ? shift - 8 : 0;
                const uint32_t dmask = (1u << (shift - nshift)) - 1u;
                clear_hist(hist, lane);
                for (int c = lane; c < npool; c += 32) {
                    const uint32_t kk = pool[c];
                    if ((kk & pmask) == prefix) atomicAdd(&hist[(kk >> nshift) & dmask], 1u);
                }
                __syncwarp();
                int ab = 0;
                const int dg = find_digit_from_top(hist, rem, lane, &ab);
                rem -= ab;
                pmask |= dmask << nshift;
                prefix |= (uint32_t)dg << nshift;
                shift = nshift;
            }
            tau = prefix;
            need = rem;
        }

        // ---- emit in index order: key > tau, then the first `need` keys == tau ----
        int32_t* dst = P.idx + row * (int64_t)P.k;
        int out = 0, eq_seen = 0;
        for (int base = 0; base < n && out < P.k; base += 32) {
            const int e = base + lane;
            const uint32_t kk = e < n ? keys[e] : 0u;
            const bool valid = e < n;
            const bool gt = valid && kk > tau;
            const bool eq = valid && kk == tau;
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

size_t topk_smem_bytes(int n) { return sizeof(uint32_t) * (size_t)kWarps * (NB + kCandMax + ((n + 31) & ~31)); }

}  // namespace

int topk_max_tiles() { return 32 * 128; }

cudaError_t launch_topk(const TopkParams& p, cudaStream_t s)
{
    if (p.rows == 0) return cudaSuccess;
    if (p.n > topk_max_tiles()) return cudaErrorInvalidValue;
    const size_t smem = topk_smem_bytes(p.n);
    cudaError_t e = cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, topk_kernel, 32 * kWarps, smem);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) per_sm = 1;
    int64_t grid = (int64_t)num_sms() * per_sm;
    const int64_t need = (p.rows + kWarps - 1) / kWarps;
    if (grid > need) grid = need;
    topk_kernel<<<(unsigned)grid, 32 * kWarps, smem, s>>>(p);
    return cudaGetLastError();
}

}  // namespace veda
