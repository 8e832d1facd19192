// Fused tile scoring + fixed-budget top-k on the 5th-generation tensor cores.
//
// The selector scores every key tile for each (query tile, head) and keeps
// the top `budget` (tao.media, "Affine launches MiniMax-H3 video studio...",
// sections "Training the Selector, Not the Generator" and "How the SN120
// Competition Works"; reference and video tiles are selected independently:
// veyrul.com, "Veda R2VA for MiniMax-H3", second paragraph).  It runs in one
// of two modes:
//   scores only (the default selection path): the tensor-core scores of each
//     chunk are staged through shared memory (a per-warp transpose) and
//     written to the workspace's score matrix in coalesced rows; the
//     warp-per-row top-k then selects from them;
//   on chip: both steps without ever writing the score matrix to memory, as
//     follows.
//
//   scores  s[i][j] = qhat_i . khat_j on the tensor cores.  The pool +
//           project kernel writes each projection as three bf16 planes
//           x = x0 + x1 + x2 (x0 = bf16(x), x1 = bf16(x - x0), x2 = bf16(x -
//           x0 - x1)); the six plane products with i + j <= 2 (smallest
//           first) give the dot product to fp32 accuracy with fp32
//           accumulation in TMEM.  The sample and the first counting pass,
//           which only guide the others, use the three leading products.  One
//           MMA group = 128 query tiles x 64 key tiles (a chunk); the query
//           planes are the MMA's A operand, held in TMEM for the whole unit,
//           the key planes come from shared memory.
//   top-k   one thread per query tile (= TMEM lane) runs the exact selection
//           of select_rows.cuh over the chunks of its row, which are
//           recomputed for every pass: a sample of 64 tiles, two counting
//           passes in registers (fp16x2 compares), a collection of the band
//           around the k-th score, and an emit pass in index order
//           (ascending list, ties to the lowest index).
//
// Two CTAs per SM, each persistent over units = (job, b h, block of 128 query
// tiles), head-major so that concurrent CTAs share k-hat in L2:
//   warp 5      TMA producer: one 24 KB stage of three k-hat planes per chunk
//               (two-stage ring).
//   warp 4      TMEM allocation and the MMAs: 6 products x 4 K-steps per
//               chunk into one of two 64-column TMEM score buffers.
//   warps 0-3   selection: each thread writes its row's q-hat planes into TMEM
//               at the start of a unit, then per chunk loads its row of a
//               score buffer (tcgen05.ld), frees the buffer and runs its pass.
// Rows whose band does not fit (or that hold a NaN) are finished by the
// exact warp-per-row top-k: their scores are written to the workspace's
// score matrix in the emit pass and their ids listed for launch_topk.
// Every mbarrier wait is bounded, as in the attention kernel.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <string.h>

#include "select_rows.cuh"
#include "tc_ptx.cuh"
#include "veda_internal.cuh"

namespace veda {
namespace {

using namespace tc;
namespace rs = rowsel;

constexpr int kRows = 128;                      // query tiles per unit (MMA M, TMEM lanes)
constexpr int kCols = 64;                       // key tiles per chunk (MMA N)
constexpr int kPlaneBytes = kCols * 128;        // 64 key rows x 64 bf16
constexpr int kStageBytes = 3 * kPlaneBytes;    // three planes
constexpr int kNS = 2;                          // k-hat stages
constexpr int kNB = 2;                          // TMEM score buffers
constexpr int kThreads = 192;
constexpr int kMmaWarp = 4, kProducerWarp = 5;
constexpr uint32_t kTmemCols = 256;             // per CTA (two CTAs per SM)
constexpr uint32_t kColA = 0;                   // q-hat planes: 3 x 32 columns (bf16 pairs)
constexpr uint32_t kColS = 128;                 // score buffers: kNB x 64 columns
static_assert(rs::kSample == kCols && rs::kCap == kCols, "the sample and band sorts share one 64-value network");

// Passes of a unit: the sample chunk, then nc chunks per pass.
enum { kSamplePass = 0, kCountA = 1, kCountB = 2, kCollect = 3, kEmit = 4, kStore = 5 };

struct JobDev {
    int32_t nk, k, nc, mode;   // mode 0: every tile kept; 2: selected on chip; 3: scores written out
    int32_t* idx;
    float* sc;
    int64_t ld;
    int32_t* fb;
    int64_t first_unit;
};

struct TcSelParams {
    const uint16_t* q_planes;   // [3][BH][nq][64]
    CUtensorMap kmap[2];        // key planes
    CUtensorMap smap[2];        // planes of the sampled key tiles
    JobDev job[2];
    int32_t n_jobs;
    int32_t BH, nq, n_blk;
    int64_t units;
    uint32_t* status;
    long long wait_limit;
};

struct __align__(1024) Smem {
    uint8_t kv[kNS][kStageBytes];
    union {
        // band scores, entry e of row t at list[e][t]; entry kCap absorbs the
        // stores of scores outside the band (branch-free collection)
        float list[rs::kCap + 1][kRows];
        // scores-only pass: each warp's 32 rows of a chunk, transposed so the
        // warp writes whole row segments (rows padded to 68 floats)
        float stage[4][32][kCols + 4];
    };
    uint64_t a_full, a_free, kv_full[kNS], kv_empty[kNS], s_full[kNB], s_empty[kNB], drain;
    uint32_t tmem_base;
    volatile int abort_flag;
};

// Chunks of one unit: the sample and four passes, or one pass writing scores.
__device__ __forceinline__ int chunks_of(const JobDev& J) { return J.mode == 3 ? J.nc : 1 + 4 * J.nc; }

__device__ __forceinline__ void decode(const JobDev& J, int ci, int& pass, int& c)
{
    if (J.mode == 3) {
        pass = kStore;
        c = ci;
    } else if (ci == 0) {
        pass = kSamplePass;
        c = 0;
    } else {
        pass = 1 + (ci - 1) / J.nc;
        c = (ci - 1) % J.nc;
    }
}

__device__ __forceinline__ void unit_of(const TcSelParams& P, int64_t u, int& jb, int& bh, int& blk)
{
    jb = (P.n_jobs > 1 && u >= P.job[1].first_unit) ? 1 : 0;
    const int64_t l = u - P.job[jb].first_unit;
    bh = (int)(l / P.n_blk);
    blk = (int)(l % P.n_blk);
}

// ---- paired fp32 helpers --------------------------------------------------
__device__ __forceinline__ uint64_t f2_pack(float lo, float hi)
{
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t v, float& lo, float& hi)
{
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c)
{
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}

// ---- fp16x2 helpers for the counting passes (g values are fp16) ----------
__device__ __forceinline__ uint32_t h2_from(float lo, float hi)
{
    uint32_t d;
    asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
    return d;
}
__device__ __forceinline__ uint32_t h2_ge(uint32_t a, uint32_t b)
{
    uint32_t d;
    asm("set.ge.f16x2.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}
__device__ __forceinline__ uint32_t h2_lt(uint32_t a, uint32_t b)
{
    uint32_t d;
    asm("set.lt.f16x2.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}
__device__ __forceinline__ uint32_t h2_add(uint32_t a, uint32_t b)
{
    uint32_t d;
    asm("add.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}
__device__ __forceinline__ uint32_t h2_max(uint32_t a, uint32_t b)
{
    uint32_t d;
    asm("max.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}
__device__ __forceinline__ uint32_t h2_min(uint32_t a, uint32_t b)
{
    uint32_t d;
    asm("min.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}
__device__ __forceinline__ uint32_t h2_splat(float x)   // x is an fp16 value
{
    const uint32_t h = __half_as_ushort(__float2half_rn(x));
    return h | (h << 16);
}
__device__ __forceinline__ float h_lo(uint32_t v) { return __half2float(__ushort_as_half((unsigned short)(v & 0xffffu))); }
__device__ __forceinline__ float h_hi(uint32_t v) { return __half2float(__ushort_as_half((unsigned short)(v >> 16))); }

constexpr uint32_t kOne2 = 0x3C003C00u;   // fp16x2 (1.0, 1.0)
constexpr uint32_t kNaN2 = 0x7E007E00u;   // fp16x2 (NaN, NaN): no comparison holds

// g of a pair of scores, as fp16x2 (lower half: the first score): the same
// fma and round-to-nearest conversion as rowsel::Map, element by element.
__device__ __forceinline__ uint32_t g_pair(float a, float b, uint64_t scale2, uint64_t bias2)
{
    float y0, y1;
    f2_unpack(f2_fma(f2_pack(a, b), scale2, bias2), y0, y1);
    return h2_from(y0, y1);
}

__global__ void __launch_bounds__(kThreads, 2) tile_select_kernel(const __grid_constant__ TcSelParams P)
{
    extern __shared__ uint8_t smem_raw[];
    Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        mbar_init(&sm.a_full, kRows);
        mbar_init(&sm.a_free, 1);
        for (int i = 0; i < kNS; ++i) {
            mbar_init(&sm.kv_full[i], 1);
            mbar_init(&sm.kv_empty[i], 1);
        }
        for (int i = 0; i < kNB; ++i) {
            mbar_init(&sm.s_full[i], 1);
            mbar_init(&sm.s_empty[i], kRows);
        }
        mbar_init(&sm.drain, 1);
        sm.abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    if (warp == kMmaWarp) tmem_alloc(&sm.tmem_base, kTmemCols);
    fence_before();
    __syncthreads();
    fence_after();
    const uint32_t tmem = sm.tmem_base;

    if (warp == kProducerWarp) {
        // ----------------------------------------------------- TMA producer ---
        if (lane == 0) {
            uint32_t f = 0;
            bool ok = true;
            for (int64_t u = blockIdx.x; u < P.units && ok; u += gridDim.x) {
                int jb, bh, blk;
                unit_of(P, u, jb, bh, blk);
                const JobDev& J = P.job[jb];
                if (J.mode == 0) continue;
                const int nci = chunks_of(J);
                for (int ci = 0; ci < nci && ok; ++ci) {
                    int pass, c;
                    decode(J, ci, pass, c);
                    const uint32_t st = f % kNS;
                    if (f >= kNS &&
                        !(ok = wait_phase(&sm.abort_flag, &sm.kv_empty[st], ((f / kNS) - 1) & 1, P.status, P.wait_limit)))
                        break;
                    mbar_expect_tx(&sm.kv_full[st], kStageBytes);
                    for (int p = 0; p < 3; ++p) {
                        if (pass == kSamplePass)
                            tma_load_3d(sm.kv[st] + p * kPlaneBytes, &P.smap[jb], &sm.kv_full[st], 0, 0, p * P.BH + bh);
                        else
                            tma_load_3d(sm.kv[st] + p * kPlaneBytes, &P.kmap[jb], &sm.kv_full[st], 0, c * kCols,
                                        p * P.BH + bh);
                    }
                    ++f;
                }
            }
            // drain: every issued load lands before the CTA can exit
            for (uint32_t k = (f > kNS ? f - kNS : 0); k < f; ++k)
                if (!drain_phase(&sm.kv_full[k % kNS], (k / kNS) & 1, P.status)) break;
        }
    } else if (warp == kMmaWarp) {
        // ------------------------------------------------------ MMA issuer ---
        constexpr uint32_t idS = idesc_bf16(false, kCols);
        uint32_t ua = 0, f = 0, nbuf = 0;
        bool ok = true;
        for (int64_t u = blockIdx.x; u < P.units && ok; u += gridDim.x) {
            int jb, bh, blk;
            unit_of(P, u, jb, bh, blk);
            const JobDev& J = P.job[jb];
            if (J.mode == 0) continue;
            // the unit's q-hat planes are in TMEM
            if (!(ok = warp_wait(&sm.abort_flag, &sm.a_full, ua & 1, P.status, P.wait_limit))) break;
            const int nci = chunks_of(J);
            for (int ci = 0; ci < nci && ok; ++ci) {
                int pass, c;
                decode(J, ci, pass, c);
                const uint32_t st = f % kNS, b = nbuf % kNB;
                if (!(ok = warp_wait(&sm.abort_flag, &sm.kv_full[st], (f / kNS) & 1, P.status, P.wait_limit))) break;
                if (nbuf >= kNB &&
                    !(ok = warp_wait(&sm.abort_flag, &sm.s_empty[b], ((nbuf / kNB) - 1) & 1, P.status, P.wait_limit)))
                    break;
                fence_after();
                const uint32_t kaddr = smem_u32(sm.kv[st]);
                const uint32_t d = tmem + kColS + b * kCols;
                // plane products (q plane in TMEM, k plane in shared memory),
                // smallest terms first; the sample and count pass A, which
                // only guide the later passes, omit the three smallest.  Count
                // pass B, collect and emit see the same (full) scores, bit for
                // bit, so the band pass B counts is exactly the band collected.
                constexpr int pa[6] = {2, 1, 0, 1, 0, 0};
                constexpr int pb[6] = {0, 1, 2, 0, 1, 0};
                const int t0 = (pass == kSamplePass || pass == kCountA) ? 3 : 0;
#pragma unroll 1
                for (int t = t0; t < 6; ++t)
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        umma_ts(d, tmem + kColA + pa[t] * 32 + kk * 8,
                                smem_desc(kaddr + pb[t] * kPlaneBytes + kk * 32, 16, 1024), idS,
                                (t > t0 || kk > 0) ? 1u : 0u);
                umma_commit(&sm.s_full[b]);
                umma_commit(&sm.kv_empty[st]);
                if (ci == nci - 1) umma_commit(&sm.a_free);   // last read of this unit's q-hat planes
                ++f;
                ++nbuf;
            }
            ++ua;
        }
        // drain: all issued MMAs complete before TMEM is released
        umma_commit(&sm.drain);
        drain_phase(&sm.drain, 0, P.status);
    } else {
        // ------------------------------------------------------- selection ---
        const int tid = threadIdx.x;               // row of the unit = TMEM lane
        const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
        uint32_t nbuf = 0, ua = 0;
        bool ok = true;
        for (int64_t u = blockIdx.x; u < P.units && ok; u += gridDim.x) {
            int jb, bh, blk;
            unit_of(P, u, jb, bh, blk);
            const JobDev& J = P.job[jb];
            const int row = blk * kRows + tid;
            const bool vrow = row < P.nq;
            const int64_t grow = (int64_t)bh * P.nq + row;
            int32_t* out = J.idx + grow * J.k;
            if (J.mode == 0) {                     // every tile kept
                if (vrow)
                    for (int j = 0; j < J.nk; ++j) out[j] = j;
                continue;
            }
            // this row's q-hat planes into TMEM (the A operand), once the
            // previous unit's MMAs have read theirs
            if (ua >= 1 && !(ok = warp_wait(&sm.abort_flag, &sm.a_free, (ua - 1) & 1, P.status, P.wait_limit))) break;
            fence_after();
#pragma unroll 1
            for (int p = 0; p < 3; ++p) {
                uint32_t a[32];
                const uint4* src = reinterpret_cast<const uint4*>(P.q_planes + (((int64_t)p * P.BH + bh) * P.nq + row) * 64);
#pragma unroll
                for (int c4 = 0; c4 < 8; ++c4) {
                    const uint4 x = vrow ? __ldg(src + c4) : make_uint4(0u, 0u, 0u, 0u);
                    a[4 * c4] = x.x;
                    a[4 * c4 + 1] = x.y;
                    a[4 * c4 + 2] = x.z;
                    a[4 * c4 + 3] = x.w;
                }
                VEDA_TMEM_ST32(tmem + lane_off + kColA + 32 * p, a);
            }
            tmem_wait_st();
            fence_before();
            mbar_arrive(&sm.a_full);

            rs::Row R{};
            uint64_t scale2 = 0, bias2 = 0;
            uint32_t t2[rs::kM], acc[rs::kM];
            uint32_t hmax = 0xFC00FC00u, hmin = 0x7C007C00u;   // (-inf, -inf), (+inf, +inf)
            uint32_t lo2 = 0, hi2 = 0, abv2 = 0;
            int m = 0, pos = 0, eq = 0;
            bool nan = false;
            auto set_thresholds = [&]() {
#pragma unroll
                for (int i = 0; i < rs::kM; ++i) {
                    t2[i] = h2_splat(R.t[i]);
                    acc[i] = 0u;
                }
            };
            const int nci = chunks_of(J);
            for (int ci = 0; ci < nci; ++ci) {
                int pass, c;
                decode(J, ci, pass, c);
                const uint32_t b = nbuf % kNB;
                if (!(ok = warp_wait(&sm.abort_flag, &sm.s_full[b], (nbuf / kNB) & 1, P.status, P.wait_limit))) break;
                fence_after();
                uint32_t sv[kCols];
                const uint32_t ta = tmem + lane_off + kColS + b * kCols;
                VEDA_TMEM_LD32(ta + 0, (sv + 0));
                VEDA_TMEM_LD32(ta + 32, (sv + 32));
                tmem_wait_ld();
                fence_before();
                mbar_arrive(&sm.s_empty[b]);       // the scores are in registers: the buffer is free
                ++nbuf;
                const int j0 = c * kCols;
                const int nvalid = (pass == kSamplePass) ? kCols : min(kCols, J.nk - j0);
                const bool last = (pass != kSamplePass) && (c == J.nc - 1);
                bool sort_now = pass == kSamplePass;   // the sample, or the collected band

                if (pass == kStore) {
                    // the chunk's exact scores: each thread puts its row in the
                    // warp's staging area, then the warp writes two rows (256
                    // contiguous bytes each) per 16-byte store instruction
                    float(*stg)[kCols + 4] = sm.stage[warp];
#pragma unroll
                    for (int e = 0; e < kCols; e += 4)
                        *reinterpret_cast<uint4*>(&stg[lane][e]) = make_uint4(sv[e], sv[e + 1], sv[e + 2], sv[e + 3]);
                    __syncwarp();
                    const int c4 = (lane & 15) * 4;
#pragma unroll 4
                    for (int it = 0; it < 16; ++it) {
                        const int r = 2 * it + (lane >> 4);
                        const int grow_r = blk * kRows + warp * 32 + r;
                        if (grow_r < P.nq) {
                            float* dst = J.sc + ((int64_t)bh * P.nq + grow_r) * J.ld + j0 + c4;
                            const float4 x = *reinterpret_cast<const float4*>(&stg[r][c4]);
                            if (c4 + 4 <= nvalid) {
                                *reinterpret_cast<float4*>(dst) = x;
                            } else {
                                if (c4 < nvalid) dst[0] = x.x;
                                if (c4 + 1 < nvalid) dst[1] = x.y;
                                if (c4 + 2 < nvalid) dst[2] = x.z;
                            }
                        }
                    }
                    __syncwarp();                  // the staging area is reused by the next chunk
                } else if (pass == kCountA || pass == kCountB) {
#pragma unroll
                    for (int e = 0; e < kCols; e += 2) {
                        uint32_t h = g_pair(__uint_as_float(sv[e]), __uint_as_float(sv[e + 1]), scale2, bias2);
                        // past the row's end: NaN, which no comparison counts
                        if (e >= nvalid) h = kNaN2;
                        else if (e + 1 >= nvalid) h = (h & 0xffffu) | (kNaN2 & 0xffff0000u);
#pragma unroll
                        for (int i = 0; i < rs::kM; ++i) acc[i] = h2_add(acc[i], h2_ge(h, t2[i]));
                        hmax = h2_max(hmax, h);
                        hmin = h2_min(hmin, h);
                    }
                    if (last) {
                        int cnt[rs::kM];
#pragma unroll
                        for (int i = 0; i < rs::kM; ++i) cnt[i] = (int)(h_lo(acc[i]) + h_hi(acc[i]));
                        if (vrow) {
                            if (pass == kCountA) {
                                R.gmax = fmaxf(h_lo(hmax), h_hi(hmax));
                                R.gmin = fminf(h_lo(hmin), h_hi(hmin));
                            }
                            rs::finish_count(R, cnt, J.k);
                            if (pass == kCountA) {
                                rs::plan_in_band(R, J.k);
                                rs::restart_ladder(R, J.nk);
                            }
                        }
                        set_thresholds();
                        lo2 = h2_splat(R.lo);
                        hi2 = R.open_top ? 0u : h2_splat(R.hi);
                    }
                } else if (pass == kCollect) {
                    const uint32_t tid_col = smem_u32(&sm.list[0][tid]);
#pragma unroll
                    for (int e = 0; e < kCols; e += 2) {
                        const float a0 = __uint_as_float(sv[e]), a1 = __uint_as_float(sv[e + 1]);
                        const bool v0 = e < nvalid, v1 = e + 1 < nvalid;
                        nan |= (v0 && a0 != a0) || (v1 && a1 != a1);
                        const uint32_t h = g_pair(a0, a1, scale2, bias2);
                        const uint32_t in = h2_ge(h, lo2) & (R.open_top ? kOne2 : h2_lt(h, hi2));
                        uint32_t up = R.open_top ? 0u : h2_ge(h, hi2);
                        if (!v1) up &= 0xffffu;
                        if (v0) abv2 = h2_add(abv2, up);
                        const bool in0 = v0 && (in & 0xffffu), in1 = v1 && (in >> 16);
                        // branch-free: scores outside the band land in the spare entry
                        const int s0 = in0 ? min(m, rs::kCap) : rs::kCap;
                        m += in0 ? 1 : 0;
                        const int s1 = in1 ? min(m, rs::kCap) : rs::kCap;
                        m += in1 ? 1 : 0;
                        asm volatile("st.shared.b32 [%0], %1;" ::"r"(tid_col + (uint32_t)s0 * (kRows * 4)), "r"(sv[e]) : "memory");
                        asm volatile("st.shared.b32 [%0], %1;" ::"r"(tid_col + (uint32_t)s1 * (kRows * 4)), "r"(sv[e + 1]) : "memory");
                    }
                    if (last) {
                        // the band's scores, padded with -inf, into the sort below
#pragma unroll
                        for (int i = 0; i < rs::kCap; ++i)
                            sv[i] = i < m ? __float_as_uint(sm.list[i][tid]) : __float_as_uint(-INFINITY);
                        sort_now = true;
                    }
                } else if (pass == kEmit) {
                    if (vrow) {
                        if (R.fail) {
                            float* dst = J.sc + grow * J.ld + j0;
#pragma unroll
                            for (int e = 0; e < kCols; ++e)
                                if (e < nvalid) dst[e] = __uint_as_float(sv[e]);
                        } else {
                            // selected columns of this chunk as a bit mask, then one store per kept tile
                            uint32_t mk[2] = {0u, 0u};
#pragma unroll
                            for (int e = 0; e < kCols; ++e) {
                                const float x = __uint_as_float(sv[e]);
                                const bool v = e < nvalid;
                                const bool is_eq = v && x == R.tau;
                                const bool sel = v && (x > R.tau || (is_eq && eq < R.need));
                                eq += is_eq ? 1 : 0;
                                mk[e >> 5] |= (sel ? 1u : 0u) << (e & 31);
                            }
#pragma unroll
                            for (int h = 0; h < 2; ++h) {
                                uint32_t bits = mk[h];
                                while (bits) {
                                    const int e = __ffs(bits) - 1;
                                    bits &= bits - 1u;
                                    if (pos < J.k) out[pos] = j0 + 32 * h + e;
                                    ++pos;
                                }
                            }
                        }
                    }
                }

                if (sort_now) {                    // one sorting network for both uses
                    float v[kCols];
#pragma unroll
                    for (int e = 0; e < kCols; ++e) v[e] = __uint_as_float(sv[e]);
                    rs::sort_desc<kCols>(v);
                    if (pass == kSamplePass) {
                        if (vrow) rs::plan_from_sorted(R, v, J.nk, J.k);
                        scale2 = f2_pack(R.g.scale, R.g.scale);
                        bias2 = f2_pack(R.g.bias, R.g.bias);
                        set_thresholds();
                    } else if (vrow) {
                        const int above = (int)(h_lo(abv2) + h_hi(abv2));
                        rs::resolve_sorted(R, v, m, above, J.k, nan);
                        if (R.fail) {
                            const int slot = atomicAdd(J.fb, 1);
                            J.fb[1 + slot] = (int32_t)grow;
                        }
                    }
                }
            }
            ++ua;
        }
    }

    // ------------------------------------------------------------ teardown ---
    fence_before();
    __syncthreads();
    fence_after();
    if (warp == kMmaWarp) tmem_dealloc(tmem, kTmemCols);
}

// Tensor map over bf16 planes [3 BH][rows][64] (row stride `row_step` rows,
// 128 bytes each), box = 64 columns x kCols rows of one plane and head.
bool make_plane_map(PFN_cuTensorMapEncodeTiled_v12000 enc, CUtensorMap* m, const void* base, int64_t rows,
                    int64_t row_step, int64_t rows_per_head, int64_t n_heads3)
{
    cuuint64_t gdim[3] = {64, (cuuint64_t)rows, (cuuint64_t)n_heads3};
    cuuint64_t gstride[2] = {(cuuint64_t)(row_step * 128), (cuuint64_t)(rows_per_head * 128)};
    cuuint32_t box[3] = {64, (cuuint32_t)kCols, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    const CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), gdim, gstride, box, estr,
                           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

}  // namespace

bool select_tc_supported(int r, int n_tiles_max)
{
    if (r > 64 || n_tiles_max > topk_max_tiles()) return false;
    int dev = 0, major = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return false;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return false;
    return major == 10;
}

cudaError_t launch_select_tc(const SelectParams& a, cudaStream_t s)
{
    if (a.BH == 0 || a.nq == 0) return cudaSuccess;
    auto enc = encode_fn();
    if (!enc) return cudaErrorNotSupported;
    TcSelParams P;
    memset(&P, 0, sizeof P);
    const int64_t BH3 = 3 * (int64_t)a.BH;
    if ((reinterpret_cast<uintptr_t>(a.q_planes) & 15u) != 0) return cudaErrorInvalidValue;
    P.q_planes = a.q_planes;
    P.n_jobs = a.n_jobs;
    P.BH = a.BH;
    P.nq = a.nq;
    P.n_blk = (a.nq + kRows - 1) / kRows;
    int64_t units = 0;
    for (int jb = 0; jb < a.n_jobs; ++jb) {
        const SelectJob& S = a.job[jb];
        JobDev& J = P.job[jb];
        J.nk = S.nk;
        J.k = S.k;
        J.nc = (S.nk + kCols - 1) / kCols;
        J.mode = a.scores_only ? 3 : (S.k == S.nk ? 0 : 2);
        if (J.mode == 2 && !S.k_sample) return cudaErrorInvalidValue;
        J.idx = S.idx;
        J.sc = S.sc;
        J.ld = S.ld;
        J.fb = S.fb;
        J.first_unit = units;
        units += (int64_t)a.BH * P.n_blk;
        if (!make_plane_map(enc, &P.kmap[jb], S.k_planes, S.nk, 1, S.nk, BH3)) return cudaErrorInvalidValue;
        if (J.mode == 3 && ((J.ld & 3) != 0 || (reinterpret_cast<uintptr_t>(S.sc) & 15u) != 0))
            return cudaErrorInvalidValue;
        if (J.mode == 2) {
            // the planes of the 64 sampled key tiles of each head (one box)
            if (!make_plane_map(enc, &P.smap[jb], S.k_sample, kCols, 1, kCols, BH3)) return cudaErrorInvalidValue;
        } else {
            P.smap[jb] = P.kmap[jb];
        }
        // no row left to the exact top-k yet (the list stays empty unless the
        // rows are selected on chip)
        cudaError_t e = cudaMemsetAsync(S.fb, 0, sizeof(int32_t), s);
        if (e != cudaSuccess) return e;
    }
    P.units = units;
    P.status = a.status;
    P.wait_limit = a.short_waits ? 64 : kWaitLimit;

    const size_t smem = sizeof(Smem) + 1024;
    cudaError_t e = cudaFuncSetAttribute(tile_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, tile_select_kernel, kThreads, smem);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) per_sm = 1;
    if (per_sm > 2) per_sm = 2;                  // TMEM: 256 columns per CTA
    int64_t grid = (int64_t)num_sms() * per_sm;
    if (grid > units) grid = units;
    tile_select_kernel<<<(unsigned)grid, kThreads, smem, s>>>(P);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;

    // rows the kernel could not finish: exact warp-per-row top-k on their scores
    for (int jb = 0; jb < a.n_jobs; ++jb) {
        if (P.job[jb].mode != 2) continue;
        const SelectJob& S = a.job[jb];
        TopkParams T{};
        T.scores = S.sc;
        T.ld = S.ld;
        T.rows = (int64_t)a.BH * a.nq;
        T.n = S.nk;
        T.k = S.k;
        T.idx = S.idx;
        T.status = a.status;
        T.row_list = S.fb + 1;
        T.row_count = S.fb;
        if ((e = launch_topk(T, s)) != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace veda
