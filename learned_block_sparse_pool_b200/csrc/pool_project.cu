// Tile pooling + selector projection (one HBM pass over Q and K).
//
// Computes, for every (b, h, tile i) of each job (Q with W_q; video K and
// reference K with W_k):
//     pooled = mean of the tokens of tile i that exist (a short last tile is
//              averaged over its own tokens),
//     xhat   = pooled (row vector, fp32) times W[h] ([d, r]),
// which is the selector input: the trained query / key projections applied
// to tile-pooled Q and K (tao.media, "Affine launches MiniMax-H3 video
// studio...", sections "Training the Selector, Not the Generator" and "How
// the SN120 Competition Works").
//
// Design (HBM-bound): a persistent grid, a multiple of the SM count, walks
// the (job, b, h, tile) items in order; each CTA owns one contiguous run of
// items, so it loads W[h] into shared memory once per head it meets.  Within
// a tile, each thread owns one 16-byte column chunk of the row and a set of
// tokens: every warp load is a 128-bit, fully coalesced access, and a tile's
// loads are issued before the previous tile is summed.  Up to four
// consecutive tiles of a head are pooled per round and reduced and projected
// together, so the per-tile barrier and projection overhead stays small.
#include <cuda_bf16.h>

#include "veda_internal.cuh"

namespace veda {
namespace {

constexpr int kThreads = 256;
constexpr int kMaxTile = 128;
constexpr int kPlaneWidth = 64;   // columns of a bf16 plane row (r <= 64, zero padded)

__device__ __forceinline__ void unpack(const uint4& raw, float* f, const float*)
{
    f[0] = __uint_as_float(raw.x);
    f[1] = __uint_as_float(raw.y);
    f[2] = __uint_as_float(raw.z);
    f[3] = __uint_as_float(raw.w);
}

__device__ __forceinline__ void unpack(const uint4& raw, float* f, const __nv_bfloat16*)
{
    const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = __uint_as_float(w[i] << 16);
        f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
}

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

__device__ __forceinline__ uint4 load_stream(const void* p)
{
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

constexpr int kGroup = 4;   // tiles of one head pooled per round
constexpr int kWarps = kThreads / 32;

// CTAs per SM the kernel is compiled for: with bf16 rows (8 loads of 16 bytes
// per thread per tile) it fits 80 registers, so three CTAs per SM keep 1.5x
// the bytes in flight of two (a 64-register cap for four spills).
template <typename Tin>
constexpr int min_blocks() { return sizeof(Tin) == 2 ? 3 : 1; }

// Writes one projected value s = xhat[b, h, tile ti][c] of job J: the fp32
// output (c < r) and, where the job asks for them, its three bf16 planes
// (columns r..63 of a plane row are written as zeros) and the sampled tiles'
// planes.
__device__ __forceinline__ void store_projection(const PoolParams& P, const PoolJob& J, int bb, int hh, int ti,
                                                 int c, float s)
{
    const int64_t orow = (int64_t)(bb * P.H + hh) * J.n_tiles + ti;
    if (c < P.r) J.out[orow * P.r + c] = s;
    if (J.planes) {
        // three bf16 terms summing to s: each difference is exact in fp32
        const __nv_bfloat16 p0 = __float2bfloat16_rn(s);
        const float r1 = s - __bfloat162float(p0);
        const __nv_bfloat16 p1 = __float2bfloat16_rn(r1);
        const __nv_bfloat16 p2 = __float2bfloat16_rn(r1 - __bfloat162float(p1));
        uint16_t* dst = J.planes + orow * kPlaneWidth + c;
        dst[0] = __bfloat16_as_ushort(p0);
        dst[J.plane_stride] = __bfloat16_as_ushort(p1);
        dst[2 * J.plane_stride] = __bfloat16_as_ushort(p2);
        if (J.sample_planes) {
            // sample rows m with floor(m n / 64) == this tile: 64 i <= m n < 64 (i + 1)
            const int64_t n = J.n_tiles;
            const int64_t m_lo = (64 * (int64_t)ti + n - 1) / n, m_hi = min((int64_t)63, (64 * ((int64_t)ti + 1) + n - 1) / n - 1);
            for (int64_t m = m_lo; m <= m_hi; ++m) {
                uint16_t* sd = J.sample_planes + ((int64_t)(bb * P.H + hh) * 64 + m) * kPlaneWidth + c;
                sd[0] = __bfloat16_as_ushort(p0);
                sd[J.sample_plane_stride] = __bfloat16_as_ushort(p1);
                sd[2 * J.sample_plane_stride] = __bfloat16_as_ushort(p2);
            }
        }
    }
}

// Batch index of a round of ng tiles of job J that ends before item `it`.
__device__ __forceinline__ int round_batch(const PoolParams& P, const PoolJob& J, int64_t it, int ng)
{
    return (int)(((it - ng - J.first_item) / J.n_tiles) / P.H);
}

// Projection of one round's pooled vectors (ng consecutive tiles i0.. of head
// hh, the round ending before item `it`): one output (g, c) per thread.
template <int D>
__device__ __forceinline__ void project_round(const PoolParams& P, const PoolJob& J, int hh, int64_t it, int ng,
                                              int i0, const float* w_s, const float* pooled, int tid, int nthreads)
{
    const int r = P.r;
    const int bb = round_batch(P, J, it, ng);
    const int rc = J.planes ? kPlaneWidth : r;   // columns written per tile
    for (int x = tid; x < ng * rc; x += nthreads) {
        const int g = x / rc, c = x % rc;
        float s = 0.f;
        if (c < r) {
            const float* pv = pooled + g * D;
#pragma unroll 8
            for (int e = 0; e < D; ++e) s = fmaf(pv[e], w_s[e * r + c], s);
        }
        store_projection(P, J, bb, hh, i0 + g, c, s);
    }
}

template <typename Tin, int D>
__global__ void __launch_bounds__(kThreads, min_blocks<Tin>()) pool_project_kernel(const PoolParams P)
{
    constexpr int EPC = 16 / sizeof(Tin);      // elements per 16-byte chunk
    constexpr int CPR = D / EPC;               // chunks per token row (divides 32)
    constexpr int RP = kThreads / CPR;         // token rows loaded in parallel
    constexpr int LOADS = kMaxTile / RP;       // loads per thread per tile (max)
    static_assert(32 % CPR == 0, "a warp holds whole token rows");

    extern __shared__ float smem[];
    const int r = P.r;
    float* w_s = smem;                         // [D][r]
    float* part = w_s + D * r;                 // [kGroup][kWarps][D]: one partial sum per warp
    float* pooled = part + kGroup * kWarps * D;   // [kGroup][D]

    const int tid = threadIdx.x;
    const int chunk = tid % CPR;
    const int row0 = tid / CPR;
    const int warp = tid / 32, lane = tid % 32;

    const int64_t it0 = (int64_t)blockIdx.x * P.total_items / gridDim.x;
    const int64_t it1 = (int64_t)(blockIdx.x + 1) * P.total_items / gridDim.x;
    if (it0 >= it1) return;
    // decode the first item of this CTA's run once; later items are stepped to
    int j = 0;
    while (j + 1 < P.n_jobs && it0 >= P.job[j + 1].first_item) ++j;
    int i, h, b;
    {
        const int64_t local = it0 - P.job[j].first_item;
        i = (int)(local % P.job[j].n_tiles);
        const int64_t bh = local / P.job[j].n_tiles;
        h = (int)(bh % P.H);
        b = (int)(bh / P.H);
    }
    int cur_job = -1, cur_h = -1;

    // one thread's 16-byte loads of its column chunk for one tile
    uint4 raw[LOADS];
    auto issue = [&](const PoolJob& J, int bb, int hh, int ii) {
        const int t0 = ii * P.T;
        const int cnt = (int)min((int64_t)P.T, J.n_tokens - (int64_t)t0);
        const char* base = reinterpret_cast<const char*>(J.x) +
                           ((int64_t)bb * J.sb + (int64_t)hh * J.sh + (int64_t)(t0 + row0) * J.st + chunk * EPC) *
                               (int64_t)sizeof(Tin);
        const int64_t step = (int64_t)RP * J.st * (int64_t)sizeof(Tin);
#pragma unroll
        for (int u = 0; u < LOADS; ++u)
            raw[u] = (row0 + u * RP < cnt) ? load_stream(base + u * step) : make_uint4(0u, 0u, 0u, 0u);
    };

    int64_t it = it0;
    issue(P.job[j], b, h, i);
    while (it < it1) {
        const PoolJob& J = P.job[j];
        if (j != cur_job || h != cur_h) {
            __syncthreads();   // the previous round's projection no longer reads w_s
            const Tin* W = static_cast<const Tin*>(J.w) + (int64_t)h * D * r;
            for (int e = tid; e < D * r; e += kThreads) w_s[e] = to_f32(W[e]);
            cur_job = j;
            cur_h = h;
        }
        // a round: up to kGroup consecutive tiles of this (job, b, h)
        const int i0 = i;
        const int ng = (int)min((int64_t)kGroup, min((int64_t)(J.n_tiles - i0), it1 - it));
        for (int g = 0; g < ng; ++g) {
            float acc[EPC];
#pragma unroll
            for (int e = 0; e < EPC; ++e) acc[e] = 0.f;
#pragma unroll
            for (int u = 0; u < LOADS; ++u) {
                float f[EPC];
                unpack(raw[u], f, (const Tin*)nullptr);
#pragma unroll
                for (int e = 0; e < EPC; ++e) acc[e] += f[e];
            }
            // next tile's loads go out before this one's partial sums are stored
            int ni = i + 1, nh = h, nb = b, nj = j;
            if (ni == J.n_tiles) {
                ni = 0;
                if (++nh == P.H) {
                    nh = 0;
                    if (++nb == P.B) {
                        nb = 0;
                        ++nj;
                    }
                }
            }
            if (it + 1 < it1) issue(P.job[nj], nb, nh, ni);
            // the lanes of a warp that hold the same column chunk (CPR apart) add up their rows
#pragma unroll
            for (int off = CPR; off < 32; off <<= 1)
#pragma unroll
                for (int e = 0; e < EPC; ++e) acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], off);
            if (lane < CPR) {
                float* dst = part + (g * kWarps + warp) * D + chunk * EPC;
#pragma unroll
                for (int e = 0; e < EPC; ++e) dst[e] = acc[e];
            }
            i = ni; h = nh; b = nb; j = nj;
            ++it;
        }
        __syncthreads();
        // pooled means of the round's tiles
        for (int x = tid; x < ng * D; x += kThreads) {
            const int g = x / D, e = x % D;
            const int t0 = (i0 + g) * P.T;
            const int cnt = (int)min((int64_t)P.T, J.n_tokens - (int64_t)t0);
            float s = 0.f;
#pragma unroll
            for (int q = 0; q < kWarps; ++q) s += part[(g * kWarps + q) * D + e];
            pooled[g * D + e] = s / (float)cnt;
        }
        __syncthreads();
        project_round<D>(P, J, cur_h, it, ng, i0, w_s, pooled, tid, kThreads);
    }
}

template <typename Tin, int D>
cudaError_t launch_typed(const PoolParams& p, cudaStream_t s)
{
    const size_t smem = sizeof(float) * ((size_t)D * p.r + (size_t)kGroup * kWarps * D + (size_t)kGroup * D);
    auto kern = pool_project_kernel<Tin, D>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kThreads, smem);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) per_sm = 1;
    int64_t grid = (int64_t)num_sms() * per_sm;
    if (grid > p.total_items) grid = p.total_items;
    kern<<<(unsigned)grid, kThreads, smem, s>>>(p);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_pool_project(const PoolParams& p, cudaStream_t s)
{
    if (p.total_items == 0) return cudaSuccess;
    if (p.dtype == VEDA_BF16) {
        return p.d == 128 ? launch_typed<__nv_bfloat16, 128>(p, s) : launch_typed<__nv_bfloat16, 64>(p, s);
    }
    return p.d == 128 ? launch_typed<float, 128>(p, s) : launch_typed<float, 64>(p, s);
}

}  // namespace veda
