// Block-sparse attention on the 5th-generation tensor cores: tcgen05 MMAs
// with accumulators in TMEM, K/V tiles gathered by index with TMA, bf16,
// head dim 128, tile 128.
//
// What it computes: each video query attends to every token of its query
// tile's kept video tiles, kept reference tiles, and every dense (text / VLM
// / audio) token, with one softmax over that set (tao.media, "Affine launches
// MiniMax-H3 video studio...", section "Training the Selector, Not the
// Generator": a predictor selects blocks for a sparse execution kernel;
// veyrul.com, "Veda R2VA for MiniMax-H3", second paragraph: reference and
// video tiles are selected, text / VLM / audio attention stays dense).
//
// Design (one CTA per SM, persistent, units in head-major order so the CTAs
// in flight share one head's K/V in L2):
//   warp 8      TMA producer: the Q tile and a 5-stage ring of 32 KB K/V
//               tiles, loaded in exactly the order the MMA warp consumes
//               them: K0, K1, V0, K2, V1, ..., V(n-1).  Each tile is two
//               128-row x 128-byte boxes with the 128-byte swizzle.  K/V
//               loads carry an L2 evict-last policy (the other query tiles
//               of the head read them again), Q loads and the O stores an
//               evict-first one.
//   warp 9      allocates TMEM and issues the MMAs (the warp runs the loop,
//               one elected lane issues).  Kept tile j goes to softmax group
//               g = j & 1: S(j) = Q K(j)^T into S buffer g, then
//               O(g) += P(j) V(j) with P read from TMEM, and S(j+2) is issued
//               right behind P(j) V(j) into the same buffer (the tensor pipe
//               runs one thread's MMAs in issue order).
//   warps 0-7   two softmax groups of four warps; warp % 4 is the TMEM lane
//               quarter (thread = query row).  Each group takes every other
//               kept tile, so the two groups run half a tile apart and one
//               group's TMEM traffic overlaps the other's exponentials.  Per
//               tile: load S, mask keys past a segment's end, running max in
//               base-2 units with a lazy rescale of the group's O (only when
//               the max grows by more than 2^8; the final division makes the
//               stale max exact), P as packed bf16 over the S buffer.  The
//               epilogue merges the two groups' (max, sum, O) and stores the
//               rows (group g writes channels [64g, 64g + 64)).
// Every mbarrier wait is bounded: on expiry the waiting thread records
// VEDA_ERR_TIMEOUT in the status word and raises a CTA-wide abort flag; all
// roles then leave their loops, outstanding TMA loads and MMAs are drained
// (again with a bound) and TMEM is released before the CTA exits.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include "tc_ptx.cuh"
#include "veda_internal.cuh"

namespace veda {
namespace {

constexpr int D = 128;
constexpr int TT = 128;                   // tile rows (queries / keys)
constexpr int NS = 5;                     // K/V ring stages
constexpr int kTileBytes = TT * D * 2;    // 32 KB
constexpr int kBoxBytes = kTileBytes / 2; // 128 rows x 128 bytes
constexpr int kThreads = 320;             // 10 warps: 8 softmax (two groups of 4), producer, MMA
// TMEM columns: S of group g at 128*g (its P, packed bf16, aliases the first
// 64 columns), O accumulator of group g at 256 + 128*g.
__host__ __device__ constexpr uint32_t col_s(uint32_t g) { return 128u * g; }
__host__ __device__ constexpr uint32_t col_o(uint32_t g) { return 256u + 128u * g; }
constexpr float kRescaleThreshold = 8.0f;     // log2 units: rescale O when the max grows > 2^8

struct TcParams {
    CUtensorMap tm[7];          // Q, Kv, Vv, Kr, Vr, Kd, Vd
    int8_t pos_h[7], pos_n[7], pos_b[7];
    int64_t n_tok[3];           // video, ref, dense tokens
    int64_t n_qtok;             // query tokens (rows of Q and of the output)
    int32_t n_tiles[3];
    const int32_t* idx_v;
    const int32_t* idx_r;
    int32_t k_v, k_r, n_d;
    int32_t B, H, nq;
    int64_t units;
    __nv_bfloat16* out;
    float* lse;
    float scale_log2;
    uint32_t* status;
    long long wait_limit;       // clocks a pipeline wait may take before the CTA aborts
    int32_t n_split;            // >1: each (b, h, query tile) is split into n_split key ranges
    float* part_o;              // [n_split][B H][n_qtok][D] unnormalised O of each range
    float* part_ml;             // [n_split][B H][n_qtok][2] (max in base-2 units, sum) of each range
};

// A work unit: (b, h, query tile i) and, when the kept list is split, the
// range [j0, j0 + nl) of it that this unit covers.
struct UnitRef {
    int64_t row;                // (b H + h) nq + i: the kept-list row
    int i, h, b, s, j0, nl;
};

template <bool kSplit>
__device__ __forceinline__ UnitRef unit_ref(const TcParams& P, int64_t u, int n_list)
{
    UnitRef r;
    r.row = kSplit ? u / P.n_split : u;
    r.s = kSplit ? (int)(u % P.n_split) : 0;
    r.i = (int)(r.row % P.nq);
    const int64_t bh = r.row / P.nq;
    r.h = (int)(bh % P.H);
    r.b = (int)(bh / P.H);
    r.j0 = kSplit ? (int)((int64_t)r.s * n_list / P.n_split) : 0;
    r.nl = kSplit ? (int)((int64_t)(r.s + 1) * n_list / P.n_split) - r.j0 : n_list;
    return r;
}

struct __align__(1024) Smem {
    uint8_t q[kTileBytes];
    uint8_t kv[NS][kTileBytes];
    uint64_t q_full, q_empty, kv_full[NS], kv_empty[NS];
    uint64_t s_full[2];         // S of softmax group g ready in TMEM buffer g
    uint64_t p_full[2];         // P of group g written (aliasing S buffer g)
    uint64_t pv_done[2];        // P V of group g completed
    uint64_t o_free;            // both O accumulators read by the epilogue
    uint64_t xchg[4];           // per lane quarter: the two groups' (max, sum) exchanged
    uint64_t drain;
    float red_m[2][2][128];     // [unit parity][group][row] running max (base-2 units)
    float red_l[2][2][128];     // [unit parity][group][row] running sum
    uint32_t tmem_base;
    volatile int abort_flag;
};

// ---------------------------------------------------------------- PTX ---
using tc::drain_phase;
using tc::fence_after;
using tc::fence_before;
using tc::idesc_bf16;
using tc::kWaitLimit;
using tc::mbar_arrive;
using tc::mbar_expect_tx;
using tc::mbar_init;
using tc::smem_desc;
using tc::smem_u32;
using tc::tmem_wait_ld;
using tc::tmem_wait_st;
using tc::umma_commit;
using tc::umma_ss;
using tc::umma_ts;

__device__ __forceinline__ bool wait_phase(Smem& sm, uint64_t* b, uint32_t parity, uint32_t* status, long long limit)
{
    return tc::wait_phase(&sm.abort_flag, b, parity, status, limit);
}

__device__ __forceinline__ bool warp_wait(Smem& sm, uint64_t* b, uint32_t parity, uint32_t* status, long long limit)
{
    return tc::warp_wait(&sm.abort_flag, b, parity, status, limit);
}

__device__ __forceinline__ void tma_load(void* dst, const CUtensorMap* map, uint64_t* bar, int c0, int c1, int c2,
                                         int c3, uint64_t policy)
{
    tc::tma_load_4d_hint(dst, map, bar, c0, c1, c2, c3, policy);
}

#define TMEM_LD32(taddr, r) VEDA_TMEM_LD32(taddr, r)

#define TMEM_ST32(taddr, r)                                                                                      \
    asm volatile(                                                                                                \
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16," \
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),                        \
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),       \
        "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]),          \
        "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]),         \
        "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])                     \
        : "memory")

#define TMEM_ST16(taddr, r)                                                                                      \
    asm volatile(                                                                                                \
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" \
        ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),   \
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])            \
        : "memory")


__device__ __forceinline__ float fast_exp2(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ float max3f(float a, float b, float c)
{
    float m;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(m) : "f"(a), "f"(b), "f"(c));
    return m;
}

// Packed pairs of fp32 (two lanes of one 64-bit register) for the f32x2 ops.
__device__ __forceinline__ uint64_t pk2(uint32_t lo, uint32_t hi)
{
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "r"(lo), "r"(hi));
    return r;
}

__device__ __forceinline__ void upk2(uint64_t v, float& lo, float& hi)
{
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}

__device__ __forceinline__ uint64_t ffma2(uint64_t a, uint64_t b, uint64_t c)
{
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}

__device__ __forceinline__ uint64_t fadd2(uint64_t a, uint64_t b)
{
    uint64_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

// ------------------------------------------------------------ tile list ---
struct TileRef {
    int seg;     // 0 video, 1 reference, 2 dense
    int tile;
    int valid;   // keys of this tile that exist (0: index out of range)
};

__device__ __forceinline__ TileRef resolve(const TcParams& P, int64_t row, int j)
{
    TileRef r;
    if (j < P.k_v) {
        r.seg = 0;
        r.tile = P.idx_v ? __ldg(P.idx_v + row * P.k_v + j) : j;   // null: every tile
    } else if (j < P.k_v + P.k_r) {
        r.seg = 1;
        r.tile = P.idx_r ? __ldg(P.idx_r + row * P.k_r + (j - P.k_v)) : j - P.k_v;
    } else {
        r.seg = 2;
        r.tile = j - P.k_v - P.k_r;
    }
    const bool ok = r.tile >= 0 && r.tile < P.n_tiles[r.seg];
    r.valid = ok ? (int)min((int64_t)TT, P.n_tok[r.seg] - (int64_t)r.tile * TT) : 0;
    return r;
}

__device__ __forceinline__ void load_box_pair(const TcParams& P, int m, uint8_t* dst, uint64_t* bar, int h, int tok,
                                              int b)
{
    const int ph = P.pos_h[m], pn = P.pos_n[m];
    const int c1 = ph == 1 ? h : (pn == 1 ? tok : b);
    const int c2 = ph == 2 ? h : (pn == 2 ? tok : b);
    const int c3 = ph == 3 ? h : (pn == 3 ? tok : b);
    // Q is read by one unit only; a K/V tile is read again by the other query
    // tiles of its head in flight (head-major unit order), so it stays in L2
    // ahead of the streaming Q loads and O stores
    const uint64_t policy = m == 0 ? tc::l2_policy_evict_first() : tc::l2_policy_evict_last();
    tma_load(dst, &P.tm[m], bar, 0, c1, c2, c3, policy);
    tma_load(dst + kBoxBytes, &P.tm[m], bar, 64, c1, c2, c3, policy);
}

// --------------------------------------------------------------- kernel ---
template <bool kSplit>
__global__ void __launch_bounds__(kThreads, 1) attn_tc_kernel(const __grid_constant__ TcParams P)
{
    extern __shared__ uint8_t smem_raw[];
    Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int n_list = P.k_v + P.k_r + P.n_d;
    constexpr int kProducerWarp = 8, kMmaWarp = 9;

    if (threadIdx.x == 0) {
        mbar_init(&sm.q_full, 1);
        mbar_init(&sm.q_empty, 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&sm.s_full[i], 1);
            mbar_init(&sm.p_full[i], 128);
            mbar_init(&sm.pv_done[i], 1);
        }
        for (int i = 0; i < NS; ++i) {
            mbar_init(&sm.kv_full[i], 1);
            mbar_init(&sm.kv_empty[i], 1);
        }
        mbar_init(&sm.o_free, 256);
        for (int q = 0; q < 4; ++q) mbar_init(&sm.xchg[q], 64);
        mbar_init(&sm.drain, 1);
        sm.abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    if (warp == kMmaWarp) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&sm.tmem_base)),
                     "r"(512)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    fence_before();
    __syncthreads();
    fence_after();
    const uint32_t tmem = sm.tmem_base;

    if (warp == kProducerWarp && lane == 0) {
        // ------------------------------------------------ TMA producer ---
        uint32_t uq = 0, f = 0;
        bool ok = true;
        for (int64_t u = blockIdx.x; u < P.units && ok; u += gridDim.x) {
            const UnitRef ur = unit_ref<kSplit>(P, u, n_list);
            const int i = ur.i, h = ur.h, b = ur.b;
            const int nl = kSplit ? ur.nl : n_list, j0 = kSplit ? ur.j0 : 0;
            const int64_t urow = kSplit ? ur.row : u;
            // the previous unit's last S has read the Q buffer
            if (uq >= 1 && !(ok = wait_phase(sm, &sm.q_empty, (uq - 1) & 1, P.status, P.wait_limit))) break;
            mbar_expect_tx(&sm.q_full, kTileBytes);
            load_box_pair(P, 0, sm.q, &sm.q_full, h, i * TT, b);
            ++uq;
            auto load_kv = [&](int j, int which) -> bool {
                const TileRef r = resolve(P, urow, j0 + j);
                const uint32_t st = f % NS;
                if (f >= NS && !wait_phase(sm, &sm.kv_empty[st], ((f / NS) - 1) & 1, P.status, P.wait_limit)) return false;
                mbar_expect_tx(&sm.kv_full[st], kTileBytes);
                const int tok = r.valid > 0 ? r.tile * TT : (int)P.n_tok[r.seg];
                load_box_pair(P, 1 + 2 * r.seg + which, sm.kv[st], &sm.kv_full[st], h, tok, b);
                ++f;
                return true;
            };
            // the MMA warp's consumption order: K0, K1, V0, K2, V1, ..., V(n-1)
            if (!(ok = load_kv(0, 0))) break;
            for (int j = 0; j < nl && ok; ++j) {
                if (j + 1 < nl) ok = load_kv(j + 1, 0);
                if (ok) ok = load_kv(j, 1);
            }
        }
        // drain: every issued load must land before the CTA can exit
        for (uint32_t k = (f > NS ? f - NS : 0); k < f; ++k)
            if (!drain_phase(&sm.kv_full[k % NS], (k / NS) & 1, P.status)) break;
        if (uq > 0) drain_phase(&sm.q_full, (uq - 1) & 1, P.status);
    } else if (warp == kMmaWarp) {
        // ------------------------------------------------- MMA issuer ---
        // The whole warp runs this loop (warp-uniform waits and operands); one
        // elected lane issues each MMA and commit.  Kept tile j goes to softmax
        // group g = j & 1.  S(j+2) reuses group g's TMEM buffer, which holds
        // P(j): it is issued right after P(j) V(j), and the tensor pipe runs one
        // thread's MMAs in issue order.
        constexpr uint32_t idS = idesc_bf16(false), idPV = idesc_bf16(true);
        uint32_t uq = 0, pc0 = 0, pc1 = 0, units_done = 0;
        uint32_t kst = 0, kph = 0;      // K/V ring: stage of the next tile consumed, and its fill phase
        auto ring_next = [&]() {
            if (++kst == NS) { kst = 0; kph ^= 1u; }
        };
        bool ok = true;
        for (int64_t u = blockIdx.x; u < P.units && ok; u += gridDim.x) {
            const int nl = kSplit ? unit_ref<kSplit>(P, u, n_list).nl : n_list;
            if (!(ok = warp_wait(sm, &sm.q_full, uq & 1, P.status, P.wait_limit))) break;
            ++uq;
            fence_after();
            const uint32_t qaddr = smem_u32(sm.q);
            auto issue_s = [&](int j) -> bool {
                const uint32_t st = kst, g = j & 1;
                if (!warp_wait(sm, &sm.kv_full[st], kph, P.status, P.wait_limit)) return false;
                fence_after();
                const uint32_t kaddr = smem_u32(sm.kv[st]);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * kBoxBytes + (kk & 3) * 32;
                    umma_ss(tmem + col_s(g), smem_desc(qaddr + off, 16, 1024), smem_desc(kaddr + off, 16, 1024), idS,
                            kk > 0);
                }
                umma_commit(&sm.s_full[g]);
                umma_commit(&sm.kv_empty[st]);
                if (j == nl - 1) umma_commit(&sm.q_empty);   // last read of this Q tile
                ring_next();
                return true;
            };
            if (!(ok = issue_s(0))) break;
            if (nl > 1 && !(ok = issue_s(1))) break;
            for (int j = 0; j < nl && ok; ++j) {
                const uint32_t g = j & 1, st = kst;
                if (!(ok = warp_wait(sm, &sm.kv_full[st], kph, P.status, P.wait_limit))) break;
                if (!(ok = warp_wait(sm, &sm.p_full[g], (g ? pc1 : pc0) & 1, P.status, P.wait_limit))) break;
                if (j == 0 && units_done > 0 &&
                    !(ok = warp_wait(sm, &sm.o_free, (units_done - 1) & 1, P.status, P.wait_limit)))
                    break;
                fence_after();
                const uint32_t vaddr = smem_u32(sm.kv[st]);
#pragma unroll
                for (int kk = 0; kk < TT / 16; ++kk)
                    umma_ts(tmem + col_o(g), tmem + col_s(g) + kk * 8, smem_desc(vaddr + kk * 2048, kBoxBytes, 1024),
                            idPV, (j >= 2 || kk > 0) ? 1u : 0u);
                umma_commit(&sm.pv_done[g]);
                umma_commit(&sm.kv_empty[st]);
                ring_next();
                if (g) ++pc1; else ++pc0;
                if (j + 2 < nl && !(ok = issue_s(j + 2))) break;
            }
            ++units_done;
        }
        // drain: all issued MMAs complete before TMEM is released
        umma_commit(&sm.drain);
        drain_phase(&sm.drain, 0, P.status);
    } else if (warp < 8) {
        // ---------------------------------------------------- softmax ---
        // Group g = warp / 4 takes kept tiles j = g, g+2, g+4, ...; warp % 4 is
        // the TMEM lane quarter (thread = query row).  Each group keeps its own
        // running max and sum and accumulates into its own O; the epilogue
        // merges the two groups.
        const int g = warp >> 2, wq = warp & 3;
        const int row = wq * 32 + lane;
        const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
        const float sl2 = P.scale_log2;
        uint32_t sc = 0, uu = 0;          // S tiles consumed by this group; units done
        bool ok = true;
        for (int64_t u = blockIdx.x; u < P.units && ok; u += gridDim.x, ++uu) {
            const UnitRef ur = unit_ref<kSplit>(P, u, n_list);
            const int i = ur.i, h = ur.h, b = ur.b;
            const int nl = kSplit ? ur.nl : n_list, j0 = kSplit ? ur.j0 : 0;
            const int64_t urow = kSplit ? ur.row : u;
            float m_run = -INFINITY, l = 0.f;
            int cnt = 0;
            TileRef r_next = resolve(P, urow, j0 + g);
            for (int j = g; j < nl; j += 2, ++sc, ++cnt) {
                const TileRef r = r_next;
                if (j + 2 < nl) r_next = resolve(P, urow, j0 + j + 2);   // one tile ahead
                if (!(ok = warp_wait(sm, &sm.s_full[g], sc & 1, P.status, P.wait_limit))) break;
                fence_after();
                uint32_t s[128];
                const uint32_t sa = tmem + lane_off + col_s(g);
                TMEM_LD32(sa + 0, (s + 0));
                TMEM_LD32(sa + 32, (s + 32));
                TMEM_LD32(sa + 64, (s + 64));
                TMEM_LD32(sa + 96, (s + 96));
                tmem_wait_ld();

                if (r.valid < TT) {                      // uniform: a short or out-of-range tile
                    if (r.valid == 0 && row == 0) record_status(P.status, VEDA_ERR_BAD_INDEX);
#pragma unroll
                    for (int c = 0; c < 128; ++c)
                        if (c >= r.valid) s[c] = __float_as_uint(-INFINITY);
                }
                // row max: eight independent 3-input chains, then a short tree
                float a8[8];
#pragma unroll
                for (int k = 0; k < 8; ++k) a8[k] = fmaxf(__uint_as_float(s[2 * k]), __uint_as_float(s[2 * k + 1]));
#pragma unroll
                for (int base = 16; base < 128; base += 16)
#pragma unroll
                    for (int k = 0; k < 8; ++k)
                        a8[k] = max3f(a8[k], __uint_as_float(s[base + 2 * k]), __uint_as_float(s[base + 2 * k + 1]));
                const float mx = fmaxf(max3f(a8[0], a8[1], a8[2]), max3f(max3f(a8[3], a8[4], a8[5]), a8[6], a8[7]));
                const float mxs = mx * sl2;
                bool rescale = false;
                float alpha = 1.f;
                if (mxs > m_run + kRescaleThreshold) {
                    if (m_run != -INFINITY) {
                        alpha = fast_exp2(m_run - mxs);
                        rescale = (cnt > 0);
                    }
                    m_run = mxs;
                }
                // a fully masked prefix leaves m_run = -inf; then every logit is -inf and p = 0
                const float neg_m = (m_run == -INFINITY) ? 0.f : -m_run;
                const uint64_t scale2 = pk2(__float_as_uint(sl2), __float_as_uint(sl2));
                const uint64_t negm2 = pk2(__float_as_uint(neg_m), __float_as_uint(neg_m));

                // P over the first 64 columns of the S buffer (S is in registers now;
                // the previous P V of this group finished before this S was written)
                uint64_t lsum[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    uint32_t packed[16];
#pragma unroll
                    for (int c = 0; c < 16; ++c) {
                        const uint64_t y = ffma2(pk2(s[32 * q + 2 * c], s[32 * q + 2 * c + 1]), scale2, negm2);
                        float y0, y1;
                        upk2(y, y0, y1);
                        const float p0 = fast_exp2(y0), p1 = fast_exp2(y1);
                        lsum[c & 3] = fadd2(lsum[c & 3], pk2(__float_as_uint(p0), __float_as_uint(p1)));
                        __nv_bfloat162 pr = __floats2bfloat162_rn(p0, p1);
                        packed[c] = *reinterpret_cast<uint32_t*>(&pr);
                    }
                    TMEM_ST16(sa + 16 * q, packed);
                }
                {
                    const uint64_t t2 = fadd2(fadd2(lsum[0], lsum[1]), fadd2(lsum[2], lsum[3]));
                    float s0, s1;
                    upk2(t2, s0, s1);
                    l = fmaf(l, alpha, s0 + s1);
                }
                tmem_wait_st();
                // This group's O holds its tiles before this one at the old max.
                // tcgen05.ld/st are warp-collective: when any row of the warp needs
                // the rescale, the whole warp waits for the group's previous P V and
                // rewrites its 32 rows of O (factor 1 where the max is kept).
                if (__any_sync(0xffffffffu, rescale)) {
                    if (!(ok = warp_wait(sm, &sm.pv_done[g], (sc - 1) & 1, P.status, P.wait_limit))) break;
                    fence_after();
                    const float a = rescale ? alpha : 1.f;
                    const uint32_t oa = tmem + lane_off + col_o(g);
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        uint32_t o[32];
                        TMEM_LD32(oa + 32 * q, o);
                        tmem_wait_ld();
#pragma unroll
                        for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * a);
                        TMEM_ST32(oa + 32 * q, o);
                    }
                    tmem_wait_st();
                }
                fence_before();
                mbar_arrive(&sm.p_full[g]);
            }
            if (!ok) break;

            // ---- epilogue: merge the two groups; group g stores channels [64g, 64g+64) ----
            if (cnt > 0 && !(ok = warp_wait(sm, &sm.pv_done[g], (sc - 1) & 1, P.status, P.wait_limit))) break;
            const uint32_t up = uu & 1;
            sm.red_m[up][g][row] = m_run;
            sm.red_l[up][g][row] = l;
            mbar_arrive(&sm.xchg[wq]);
            if (!(ok = warp_wait(sm, &sm.xchg[wq], uu & 1, P.status, P.wait_limit))) break;
            fence_after();
            const float m0 = sm.red_m[up][0][row], m1 = sm.red_m[up][1][row];
            const float l0 = sm.red_l[up][0][row], l1 = sm.red_l[up][1][row];
            const float M = fmaxf(m0, m1);
            const float f0 = (m0 == -INFINITY) ? 0.f : fast_exp2(m0 - M);
            const float f1 = (m1 == -INFINITY) ? 0.f : fast_exp2(m1 - M);
            const float L = l0 * f0 + l1 * f1;
            constexpr bool split = kSplit;
            const float inv = split ? 1.f : 1.f / L;   // a split range stays unnormalised for the merge
            const float c0 = f0 * inv, c1 = f1 * inv;
            const int64_t tok = (int64_t)i * TT + row;
            const int64_t prow = kSplit ? (((u % P.n_split) * P.B + b) * (int64_t)P.H + h) * P.n_qtok + tok : 0;
            __nv_bfloat16* dst = P.out + (((int64_t)b * P.n_qtok + tok) * P.H + h) * D + 64 * g;
            const uint64_t o_policy = tc::l2_policy_evict_first();   // O is written once
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                uint32_t o0[32], o1[32];
                TMEM_LD32(tmem + lane_off + col_o(0) + 64 * g + 32 * q, o0);
                TMEM_LD32(tmem + lane_off + col_o(1) + 64 * g + 32 * q, o1);
                tmem_wait_ld();
                if (split && tok < P.n_qtok) {
                    float* po = P.part_o + prow * D + 64 * g + 32 * q;
#pragma unroll
                    for (int c = 0; c < 32; c += 4) {
                        float v[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float a0 = __uint_as_float(o0[c + e]) * c0;
                            v[e] = (c1 != 0.f) ? fmaf(__uint_as_float(o1[c + e]), c1, a0) : a0;
                        }
                        *reinterpret_cast<float4*>(po + c) = make_float4(v[0], v[1], v[2], v[3]);
                    }
                } else if (tok < P.n_qtok) {
#pragma unroll
                    for (int c = 0; c < 32; c += 8) {
                        float v[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            // a group with no tile in this unit contributes nothing
                            // (its O holds stale values: never multiplied in)
                            const float a0 = __uint_as_float(o0[c + e]) * c0;
                            v[e] = (c1 != 0.f) ? fmaf(__uint_as_float(o1[c + e]), c1, a0) : a0;
                        }
                        uint4 w;
                        __nv_bfloat162 v0 = __floats2bfloat162_rn(v[0], v[1]);
                        __nv_bfloat162 v1 = __floats2bfloat162_rn(v[2], v[3]);
                        __nv_bfloat162 v2 = __floats2bfloat162_rn(v[4], v[5]);
                        __nv_bfloat162 v3 = __floats2bfloat162_rn(v[6], v[7]);
                        w.x = *reinterpret_cast<uint32_t*>(&v0);
                        w.y = *reinterpret_cast<uint32_t*>(&v1);
                        w.z = *reinterpret_cast<uint32_t*>(&v2);
                        w.w = *reinterpret_cast<uint32_t*>(&v3);
                        tc::st_global_v4_hint(dst + 32 * q + c, w, o_policy);
                    }
                }
            }
            if (split) {
                if (g == 0 && tok < P.n_qtok) {
                    P.part_ml[2 * prow] = M;
                    P.part_ml[2 * prow + 1] = L;
                }
            } else if (P.lse && g == 0 && tok < P.n_qtok) {
                P.lse[((int64_t)b * P.H + h) * P.n_qtok + tok] = (M + __log2f(L)) * 0.69314718055994531f;
            }
            fence_before();
            mbar_arrive(&sm.o_free);
        }
    }

    // ---------------------------------------------------- teardown ---
    fence_before();
    __syncthreads();
    fence_after();
    if (warp == kMmaWarp) {
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512) : "memory");
    }
}

// Merge of split key ranges: per (b, h, query token) row, with the ranges'
// (max m_s in base-2 units, sum l_s, unnormalised O_s):
//   M = max m_s,  L = sum l_s 2^(m_s - M),  O = sum O_s 2^(m_s - M) / L.
// One warp per row, four channels per lane.
__global__ void __launch_bounds__(256) merge_splits_kernel(const float* __restrict__ part_o,
                                                          const float* __restrict__ part_ml, int n_split,
                                                          int64_t rows, int64_t n_qtok, int H,
                                                          __nv_bfloat16* __restrict__ out, float* __restrict__ lse)
{
    const int64_t r = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    if (r >= rows) return;
    const int lane = threadIdx.x & 31;
    float M = -INFINITY;
    for (int s = 0; s < n_split; ++s) M = fmaxf(M, part_ml[2 * ((int64_t)s * rows + r)]);
    float L = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int s = 0; s < n_split; ++s) {
        const int64_t pr = (int64_t)s * rows + r;
        const float m = part_ml[2 * pr];
        const float w = m == -INFINITY ? 0.f : exp2f(m - M);
        L = fmaf(part_ml[2 * pr + 1], w, L);
        const float4 o = *reinterpret_cast<const float4*>(part_o + pr * D + 4 * lane);
        acc.x = fmaf(o.x, w, acc.x);
        acc.y = fmaf(o.y, w, acc.y);
        acc.z = fmaf(o.z, w, acc.z);
        acc.w = fmaf(o.w, w, acc.w);
    }
    const float inv = 1.f / L;
    const int64_t bh = r / n_qtok, tok = r % n_qtok;
    const int64_t b = bh / H, h = bh % H;
    __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x * inv, acc.y * inv);
    __nv_bfloat162 hi = __floats2bfloat162_rn(acc.z * inv, acc.w * inv);
    uint2 w2;
    w2.x = *reinterpret_cast<uint32_t*>(&lo);
    w2.y = *reinterpret_cast<uint32_t*>(&hi);
    *reinterpret_cast<uint2*>(out + ((b * n_qtok + tok) * H + h) * D + 4 * lane) = w2;
    if (lse && lane == 0) lse[bh * n_qtok + tok] = (M + __log2f(L)) * 0.69314718055994531f;
}

// ------------------------------------------------------------------ host ---
using tc::encode_fn;

// Tensor map over a [B, n, H, 128] bf16 tensor (element strides sb, st, sh),
// box = 64 channels x 128 tokens of one (b, h); dims 1..3 ordered by stride.
bool make_map(PFN_cuTensorMapEncodeTiled_v12000 enc, CUtensorMap* m, int8_t* ph, int8_t* pn, int8_t* pb,
              const void* base, int64_t B, int64_t n, int64_t H, int64_t sb, int64_t st, int64_t sh)
{
    struct Dim { int64_t extent, stride; int which; };   // which: 0 h, 1 n, 2 b
    Dim dims[3] = {{H, sh, 0}, {n, st, 1}, {B, sb, 2}};
    for (auto& d : dims)
        if (d.extent == 1) d.stride = 0;   // extent-1 dims: any legal stride; sort them last
    for (int a = 0; a < 3; ++a)
        for (int c = a + 1; c < 3; ++c) {
            const int64_t sa = dims[a].stride ? dims[a].stride : INT64_MAX;
            const int64_t sc = dims[c].stride ? dims[c].stride : INT64_MAX;
            if (sc < sa) { Dim t = dims[a]; dims[a] = dims[c]; dims[c] = t; }
        }
    cuuint64_t gdim[4] = {128, 0, 0, 0};
    cuuint64_t gstride[3];
    cuuint32_t box[4] = {64, 1, 1, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    int64_t prev_span = 128 * 2;   // bytes spanned by the inner dims so far
    for (int a = 0; a < 3; ++a) {
        gdim[a + 1] = (cuuint64_t)dims[a].extent;
        int64_t bytes = dims[a].stride * 2;
        if (dims[a].extent == 1 || bytes == 0) bytes = (prev_span + 15) / 16 * 16;
        if (bytes % 16 != 0 || bytes <= 0 || bytes >= ((int64_t)1 << 40)) return false;
        gstride[a] = (cuuint64_t)bytes;
        prev_span = bytes * dims[a].extent;
        if (dims[a].which == 1) box[a + 1] = 128;
        if (dims[a].which == 0) *ph = (int8_t)(a + 1);
        if (dims[a].which == 1) *pn = (int8_t)(a + 1);
        if (dims[a].which == 2) *pb = (int8_t)(a + 1);
    }
    const CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), gdim, gstride, box, estr,
                           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

}  // namespace

bool attn_tc_supported(const AttnParams& p)
{
    if (p.dtype != VEDA_BF16 || p.d != 128 || p.T != 128) return false;
    int dev = 0, major = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return false;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return false;
    return major == 10;
}

cudaError_t launch_attn_tc(const AttnParams& a, cudaStream_t s)
{
    const int n_split = a.n_split > 1 ? a.n_split : 1;
    if (n_split > 1 && (!a.part_o || !a.part_ml)) return cudaErrorInvalidValue;
    const int64_t units = (int64_t)a.B * a.H * a.nq * n_split;
    if (units == 0) return cudaSuccess;
    auto enc = encode_fn();
    if (!enc) return cudaErrorNotSupported;
    TcParams P;
    memset(&P, 0, sizeof P);
    bool ok = make_map(enc, &P.tm[0], &P.pos_h[0], &P.pos_n[0], &P.pos_b[0], a.q, a.B, a.n_qtok, a.H, a.qsb,
                       a.qst, a.qsh);
    const Segment* segs[3] = {&a.video, &a.ref, &a.dense};
    for (int g = 0; g < 3 && ok; ++g) {
        const Segment& S = *segs[g];
        P.n_tok[g] = S.n;
        P.n_tiles[g] = S.n_tiles;
        if (S.n == 0) {   // absent segment: never referenced, but keep the maps valid
            ok = make_map(enc, &P.tm[1 + 2 * g], &P.pos_h[1 + 2 * g], &P.pos_n[1 + 2 * g], &P.pos_b[1 + 2 * g],
                          a.video.k, a.B, a.video.n, a.H, a.video.sb, a.video.st, a.video.sh) &&
                 make_map(enc, &P.tm[2 + 2 * g], &P.pos_h[2 + 2 * g], &P.pos_n[2 + 2 * g], &P.pos_b[2 + 2 * g],
                          a.video.v, a.B, a.video.n, a.H, a.video.sb, a.video.st, a.video.sh);
            continue;
        }
        ok = make_map(enc, &P.tm[1 + 2 * g], &P.pos_h[1 + 2 * g], &P.pos_n[1 + 2 * g], &P.pos_b[1 + 2 * g], S.k, a.B,
                      S.n, a.H, S.sb, S.st, S.sh) &&
             make_map(enc, &P.tm[2 + 2 * g], &P.pos_h[2 + 2 * g], &P.pos_n[2 + 2 * g], &P.pos_b[2 + 2 * g], S.v, a.B,
                      S.n, a.H, S.sb, S.st, S.sh);
    }
    if (!ok) return cudaErrorInvalidValue;
    P.idx_v = a.idx_v;
    P.idx_r = a.idx_r;
    P.k_v = a.k_v;
    P.k_r = a.k_r;
    P.n_d = a.dense.n_tiles;
    P.B = a.B;
    P.H = a.H;
    P.nq = a.nq;
    P.n_qtok = a.n_qtok;
    P.units = units;
    P.out = static_cast<__nv_bfloat16*>(a.out);
    P.lse = a.lse;
    P.scale_log2 = a.scale * 1.4426950408889634f;
    P.status = a.status;
    P.wait_limit = a.short_waits ? 64 : kWaitLimit;
    P.n_split = n_split;
    P.part_o = a.part_o;
    P.part_ml = a.part_ml;

    const size_t smem = sizeof(Smem) + 1024;
    auto kern = n_split > 1 ? attn_tc_kernel<true> : attn_tc_kernel<false>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    int64_t grid = num_sms();
    if (grid > units) grid = units;
    kern<<<(unsigned)grid, kThreads, smem, s>>>(P);
    if (n_split > 1) {
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
        const int64_t rows = (int64_t)a.B * a.H * a.n_qtok;
        merge_splits_kernel<<<(unsigned)((rows + 7) / 8), 256, 0, s>>>(a.part_o, a.part_ml, n_split, rows, a.n_qtok,
                                                                       a.H, P.out, a.lse);
    }
    return cudaGetLastError();
}

}  // namespace veda
