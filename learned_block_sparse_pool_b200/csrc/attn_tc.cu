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
//   warp 0      TMA producer: Q tile (double-buffered) and a 4-stage ring of
//               32 KB K/V tiles, loaded in exactly the order the MMA warp
//               consumes them: K0, K1, V0, K2, V1, ..., V(n-1).  Each tile is
//               two 128-row x 128-byte boxes with the 128-byte swizzle.
//   warp 1      MMA issuer (one thread): S(t+1) = Q K(t+1)^T is issued before
//               O += P(t) V(t), so the tensor core works on the next score
//               tile while the softmax warps exponentiate the current one.
//   warp 2      TMEM allocator (all 512 columns).
//   warps 4-7   softmax: thread = query row = TMEM lane.  Loads S from TMEM,
//               masks keys past a segment's end, keeps a running max in
//               base-2 units (rescaling O in TMEM only when the max grows by
//               more than 2^8, otherwise the stale max is kept: the final
//               division by the row sum makes the result exact either way),
//               writes P as packed bf16 into TMEM (the A operand of P V), and
//               finally normalises O and stores the row.
// TMEM columns: S0 [0,128) S1 [128,256) P0 [256,320) P1 [320,384) O [384,512).
// Every mbarrier wait is bounded: on expiry the waiting thread records
// VEDA_ERR_TIMEOUT in the status word and raises a CTA-wide abort flag; all
// roles then leave their loops, outstanding TMA loads and MMAs are drained
// (again with a bound) and TMEM is released before the CTA exits.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include "veda_internal.cuh"

namespace veda {
namespace {

constexpr int D = 128;
constexpr int TT = 128;                   // tile rows (queries / keys)
constexpr int NS = 4;                     // K/V ring stages
constexpr int kTileBytes = TT * D * 2;    // 32 KB
constexpr int kBoxBytes = kTileBytes / 2; // 128 rows x 128 bytes
constexpr int kThreads = 256;
constexpr uint32_t kColS0 = 0, kColS1 = 128, kColP0 = 256, kColP1 = 320, kColO = 384;
constexpr long long kWaitLimit = 1ll << 31;   // clock cycles (~1 s)
constexpr float kRescaleThreshold = 8.0f;     // log2 units: rescale O when the max grows > 2^8

struct TcParams {
    CUtensorMap tm[7];          // Q, Kv, Vv, Kr, Vr, Kd, Vd
    int8_t pos_h[7], pos_n[7], pos_b[7];
    int64_t n_tok[3];           // video, ref, dense tokens
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
};

struct __align__(1024) Smem {
    uint8_t q[2][kTileBytes];
    uint8_t kv[NS][kTileBytes];
    uint64_t q_full[2], q_empty[2], kv_full[NS], kv_empty[NS];
    uint64_t s_full[2], s_free[2], p_full[2], p_free[2], drain;
    uint32_t tmem_base;
    volatile int abort_flag;
};

// ---------------------------------------------------------------- PTX ---
__device__ __forceinline__ uint32_t smem_u32(const void* p)
{
    return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void mbar_init(uint64_t* b, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(b)), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* b)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(b)) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t* b, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(b)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* b, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(b)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Bounded wait: true when the phase completed, false on timeout or abort.
__device__ __forceinline__ bool wait_phase(Smem& sm, uint64_t* b, uint32_t parity, uint32_t* status)
{
    if (mbar_try_wait(b, parity)) return true;
    const long long t0 = clock64();
    for (;;) {
        if (mbar_try_wait(b, parity)) return true;
        if (sm.abort_flag) return false;
        if (clock64() - t0 > kWaitLimit) {
            record_status(status, VEDA_ERR_TIMEOUT);
            sm.abort_flag = 1;
            return false;
        }
    }
}

// Wait by every lane of a warp that next issues warp-collective tcgen05.ld /
// tcgen05.st: reconverges the warp and makes the outcome warp-uniform.
__device__ __forceinline__ bool warp_wait(Smem& sm, uint64_t* b, uint32_t parity, uint32_t* status)
{
    const bool ok = wait_phase(sm, b, parity, status);
    return __all_sync(0xffffffffu, ok);
}

// Drain wait: like wait_phase but ignores the abort flag (used to let copies
// and MMAs already in flight land before the CTA releases its resources).
__device__ __forceinline__ bool drain_phase(uint64_t* b, uint32_t parity, uint32_t* status)
{
    const long long t0 = clock64();
    while (!mbar_try_wait(b, parity)) {
        if (clock64() - t0 > kWaitLimit) {
            record_status(status, VEDA_ERR_TIMEOUT);
            return false;
        }
    }
    return true;
}

__device__ __forceinline__ void tma_load(void* dst, const CUtensorMap* map, uint64_t* bar, int c0, int c1, int c2,
                                         int c3)
{
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4, %5}], "
        "[%6];" ::"r"(smem_u32(dst)),
        "l"((uint64_t)map), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void umma_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                        uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

__device__ __forceinline__ void umma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                        uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

__device__ __forceinline__ void umma_commit(uint64_t* bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

#define TMEM_LD32(taddr, r)                                                                                      \
    asm volatile(                                                                                                \
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17," \
        "%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"                                       \
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),        \
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),  \
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]),             \
          "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]),             \
          "=r"(r[30]), "=r"(r[31])                                                                               \
        : "r"(taddr))

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

__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

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

// Shared-memory matrix descriptor, 128-byte swizzle, sm100 format (version 1).
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo)
{
    return (uint64_t)((addr & 0x3FFFFu) >> 4) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
           ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}

// Instruction descriptor: bf16 x bf16 -> fp32, M = 128, N = 128.
__host__ __device__ constexpr uint32_t idesc_bf16(bool b_mn_major)
{
    return (1u << 4) | (1u << 7) | (1u << 10) | ((b_mn_major ? 1u : 0u) << 16) | ((uint32_t)(128 >> 3) << 17) |
           ((uint32_t)(128 >> 4) << 24);
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
        r.tile = __ldg(P.idx_v + row * P.k_v + j);
    } else if (j < P.k_v + P.k_r) {
        r.seg = 1;
        r.tile = __ldg(P.idx_r + row * P.k_r + (j - P.k_v));
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
    tma_load(dst, &P.tm[m], bar, 0, c1, c2, c3);
    tma_load(dst + kBoxBytes, &P.tm[m], bar, 64, c1, c2, c3);
}

// --------------------------------------------------------------- kernel ---
__global__ void __launch_bounds__(kThreads, 1) attn_tc_kernel(const __grid_constant__ TcParams P)
{
    extern __shared__ uint8_t smem_raw[];
    Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int n_list = P.k_v + P.k_r + P.n_d;

    if (threadIdx.x == 0) {
        for (int i = 0; i < 2; ++i) {
            mbar_init(&sm.q_full[i], 1);
            mbar_init(&sm.q_empty[i], 1);
            mbar_init(&sm.s_full[i], 1);
            mbar_init(&sm.s_free[i], 128);
            mbar_init(&sm.p_full[i], 128);
            mbar_init(&sm.p_free[i], 1);
        }
        for (int i = 0; i < NS; ++i) {
            mbar_init(&sm.kv_full[i], 1);
            mbar_init(&sm.kv_empty[i], 1);
        }
        mbar_init(&sm.drain, 1);
        sm.abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    if (warp == 2) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&sm.tmem_base)),
                     "r"(512)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;

    if (warp == 0 && lane == 0) {
        // ------------------------------------------------ TMA producer ---
        uint32_t uq = 0, f = 0;
        bool ok = true;
        for (int64_t u = blockIdx.x; u < P.units && ok; u += gridDim.x) {
            const int i = (int)(u % P.nq);
            const int64_t bh = u / P.nq;
            const int h = (int)(bh % P.H), b = (int)(bh / P.H);
            const uint32_t qb = uq & 1;
            if (uq >= 2 && !(ok = wait_phase(sm, &sm.q_empty[qb], ((uq >> 1) - 1) & 1, P.status))) break;
            mbar_expect_tx(&sm.q_full[qb], kTileBytes);
            load_box_pair(P, 0, sm.q[qb], &sm.q_full[qb], h, i * TT, b);
            ++uq;
            auto load_kv = [&](int j, int which) -> bool {
                const TileRef r = resolve(P, u, j);
                const uint32_t st = f % NS;
                if (f >= NS && !wait_phase(sm, &sm.kv_empty[st], ((f / NS) - 1) & 1, P.status)) return false;
                mbar_expect_tx(&sm.kv_full[st], kTileBytes);
                const int tok = r.valid > 0 ? r.tile * TT : (int)P.n_tok[r.seg];
                load_box_pair(P, 1 + 2 * r.seg + which, sm.kv[st], &sm.kv_full[st], h, tok, b);
                ++f;
                return true;
            };
            if (!(ok = load_kv(0, 0))) break;
            for (int j = 0; j < n_list && ok; ++j) {
                if (j + 1 < n_list) ok = load_kv(j + 1, 0);
                if (ok) ok = load_kv(j, 1);
            }
        }
        // drain: every issued load must land before the CTA can exit
        for (uint32_t k = (f > NS ? f - NS : 0); k < f; ++k)
            if (!drain_phase(&sm.kv_full[k % NS], (k / NS) & 1, P.status)) break;
        for (uint32_t k = (uq > 2 ? uq - 2 : 0); k < uq; ++k)
            if (!drain_phase(&sm.q_full[k & 1], (k >> 1) & 1, P.status)) break;
    } else if (warp == 1 && lane == 0) {
        // ------------------------------------------------- MMA issuer ---
        constexpr uint32_t idS = idesc_bf16(false), idPV = idesc_bf16(true);
        uint32_t uq = 0, f = 0, ts = 0, tp = 0;
        bool ok = true;
        for (int64_t u = blockIdx.x; u < P.units && ok; u += gridDim.x) {
            const uint32_t qb = uq & 1;
            if (!(ok = wait_phase(sm, &sm.q_full[qb], (uq >> 1) & 1, P.status))) break;
            ++uq;
            tc_fence_after();
            const uint32_t qaddr = smem_u32(sm.q[qb]);
            auto issue_s = [&]() -> bool {
                const uint32_t st = f % NS, sb = ts & 1;
                if (!wait_phase(sm, &sm.kv_full[st], (f / NS) & 1, P.status)) return false;
                if (ts >= 2 && !wait_phase(sm, &sm.s_free[sb], ((ts >> 1) - 1) & 1, P.status)) return false;
                tc_fence_after();
                const uint32_t kaddr = smem_u32(sm.kv[st]);
                const uint32_t d_tmem = tmem + (sb ? kColS1 : kColS0);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * kBoxBytes + (kk & 3) * 32;
                    umma_ss(d_tmem, smem_desc(qaddr + off, 16, 1024), smem_desc(kaddr + off, 16, 1024), idS,
                            kk > 0);
                }
                umma_commit(&sm.s_full[sb]);
                umma_commit(&sm.kv_empty[st]);
                ++f;
                ++ts;
                return true;
            };
            if (!(ok = issue_s())) break;
            for (int j = 0; j < n_list && ok; ++j) {
                if (j + 1 < n_list) {
                    if (!(ok = issue_s())) break;
                } else {
                    umma_commit(&sm.q_empty[qb]);     // every S MMA of this unit has been issued
                }
                const uint32_t st = f % NS, pb = tp & 1;
                if (!(ok = wait_phase(sm, &sm.kv_full[st], (f / NS) & 1, P.status))) break;
                if (!(ok = wait_phase(sm, &sm.p_full[pb], (tp >> 1) & 1, P.status))) break;
                tc_fence_after();
                const uint32_t vaddr = smem_u32(sm.kv[st]);
                const uint32_t p_tmem = tmem + (pb ? kColP1 : kColP0);
#pragma unroll
                for (int kk = 0; kk < TT / 16; ++kk)
                    umma_ts(tmem + kColO, p_tmem + kk * 8, smem_desc(vaddr + kk * 2048, kBoxBytes, 1024), idPV,
                            (j > 0 || kk > 0) ? 1u : 0u);
                umma_commit(&sm.p_free[pb]);
                umma_commit(&sm.kv_empty[st]);
                ++f;
                ++tp;
            }
        }
        // drain: all issued MMAs complete before TMEM is released
        umma_commit(&sm.drain);
        drain_phase(&sm.drain, 0, P.status);
    } else if (warp >= 4) {
        // ---------------------------------------------------- softmax ---
        const int wr = warp - 4;
        const int row = wr * 32 + lane;
        const uint32_t lane_off = (uint32_t)(wr * 32) << 16;
        const float sl2 = P.scale_log2;
        uint32_t t = 0;
        bool ok = true;
        for (int64_t u = blockIdx.x; u < P.units && ok; u += gridDim.x) {
            const int i = (int)(u % P.nq);
            const int64_t bh = u / P.nq;
            const int h = (int)(bh % P.H), b = (int)(bh / P.H);
            float m_run = -INFINITY, l = 0.f;
            for (int j = 0; j < n_list; ++j, ++t) {
                const TileRef r = resolve(P, u, j);      // index load overlaps the wait below
                const uint32_t sb = t & 1;
                if (!(ok = warp_wait(sm, &sm.s_full[sb], (t >> 1) & 1, P.status))) break;
                tc_fence_after();
                uint32_t s[128];
                const uint32_t sa = tmem + lane_off + (sb ? kColS1 : kColS0);
                TMEM_LD32(sa + 0, (s + 0));
                TMEM_LD32(sa + 32, (s + 32));
                TMEM_LD32(sa + 64, (s + 64));
                TMEM_LD32(sa + 96, (s + 96));
                tmem_wait_ld();
                tc_fence_before();
                mbar_arrive(&sm.s_free[sb]);

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
                        rescale = (j > 0);
                    }
                    m_run = mxs;
                }
                // a fully masked prefix leaves m_run = -inf; then every logit is -inf and p = 0
                const float neg_m = (m_run == -INFINITY) ? 0.f : -m_run;
                const uint64_t scale2 = pk2(__float_as_uint(sl2), __float_as_uint(sl2));
                const uint64_t negm2 = pk2(__float_as_uint(neg_m), __float_as_uint(neg_m));

                const uint32_t pb = t & 1;
                if (t >= 2 && !(ok = warp_wait(sm, &sm.p_free[pb], ((t >> 1) - 1) & 1, P.status))) break;
                const uint32_t pa = tmem + lane_off + (pb ? kColP1 : kColP0);
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
                    TMEM_ST16(pa + 16 * q, packed);
                }
                {
                    const uint64_t t2 = fadd2(fadd2(lsum[0], lsum[1]), fadd2(lsum[2], lsum[3]));
                    float s0, s1;
                    upk2(t2, s0, s1);
                    l = fmaf(l, alpha, s0 + s1);
                }
                tmem_wait_st();
                // O holds the sum up to tile t-1 at the old max.  tcgen05.ld/st
                // are warp-collective, so when any row of this warp needs the
                // rescale the whole warp waits for that product and rewrites its
                // 32 rows of O (factor 1 for the rows that keep their max).
                if (__any_sync(0xffffffffu, rescale)) {
                    const uint32_t pp = (t - 1) & 1;
                    if (!(ok = warp_wait(sm, &sm.p_free[pp], ((t - 1) >> 1) & 1, P.status))) break;
                    tc_fence_after();
                    const float a = rescale ? alpha : 1.f;
                    const uint32_t oa = tmem + lane_off + kColO;
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
                tc_fence_before();
                mbar_arrive(&sm.p_full[pb]);
            }
            if (!ok) break;

            // ---- epilogue: O / l, bf16, one row per thread ----
            const uint32_t tl = t - 1;
            if (!(ok = warp_wait(sm, &sm.p_free[tl & 1], (tl >> 1) & 1, P.status))) break;
            tc_fence_after();
            const int64_t tok = (int64_t)i * TT + row;
            const float inv = 1.f / l;
            const uint32_t oa = tmem + lane_off + kColO;
            __nv_bfloat16* dst = P.out + (((int64_t)b * P.n_tok[0] + tok) * P.H + h) * D;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                uint32_t o[32];
                TMEM_LD32(oa + 32 * q, o);
                tmem_wait_ld();
                if (tok < P.n_tok[0]) {
#pragma unroll
                    for (int c = 0; c < 32; c += 8) {
                        uint4 w;
                        __nv_bfloat162 v0 = __floats2bfloat162_rn(__uint_as_float(o[c]) * inv, __uint_as_float(o[c + 1]) * inv);
                        __nv_bfloat162 v1 = __floats2bfloat162_rn(__uint_as_float(o[c + 2]) * inv, __uint_as_float(o[c + 3]) * inv);
                        __nv_bfloat162 v2 = __floats2bfloat162_rn(__uint_as_float(o[c + 4]) * inv, __uint_as_float(o[c + 5]) * inv);
                        __nv_bfloat162 v3 = __floats2bfloat162_rn(__uint_as_float(o[c + 6]) * inv, __uint_as_float(o[c + 7]) * inv);
                        w.x = *reinterpret_cast<uint32_t*>(&v0);
                        w.y = *reinterpret_cast<uint32_t*>(&v1);
                        w.z = *reinterpret_cast<uint32_t*>(&v2);
                        w.w = *reinterpret_cast<uint32_t*>(&v3);
                        *reinterpret_cast<uint4*>(dst + 32 * q + c) = w;
                    }
                }
            }
            if (P.lse && tok < P.n_tok[0])
                P.lse[((int64_t)b * P.H + h) * P.n_tok[0] + tok] = (m_run + __log2f(l)) * 0.69314718055994531f;
            tc_fence_before();
        }
    }

    // ---------------------------------------------------- teardown ---
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 2) {
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512) : "memory");
    }
}

// ------------------------------------------------------------------ host ---
PFN_cuTensorMapEncodeTiled_v12000 encode_fn()
{
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
        return nullptr;
    return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
}

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
    const int64_t units = (int64_t)a.B * a.H * a.nq;
    if (units == 0) return cudaSuccess;
    auto enc = encode_fn();
    if (!enc) return cudaErrorNotSupported;
    TcParams P;
    memset(&P, 0, sizeof P);
    bool ok = make_map(enc, &P.tm[0], &P.pos_h[0], &P.pos_n[0], &P.pos_b[0], a.q, a.B, a.video.n, a.H, a.qsb,
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
    P.units = units;
    P.out = static_cast<__nv_bfloat16*>(a.out);
    P.lse = a.lse;
    P.scale_log2 = a.scale * 1.4426950408889634f;
    P.status = a.status;

    const size_t smem = sizeof(Smem) + 1024;
    cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    int64_t grid = num_sms();
    if (grid > units) grid = units;
    attn_tc_kernel<<<(unsigned)grid, kThreads, smem, s>>>(P);
    return cudaGetLastError();
}

}  // namespace veda
