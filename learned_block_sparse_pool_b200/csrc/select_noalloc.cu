// Tile selection for callers that cannot allocate device memory.
//
// veda_select_tiles() needs a caller-provided workspace (pooled projections
// and the fp32 score matrix, ~140 MB for a 5.17 s clip).  Some callers
// cannot obtain one at call time: a serving engine that plans all device
// memory ahead and forbids allocation once requests flow, a plugin whose
// enqueue hook may not allocate, or a latency-critical loop where
// cudaMalloc's implicit device synchronisation is not acceptable.  This file
// gives them veda_select_tiles_noalloc(): the same pool + project, score
// and top-k kernels, with all scratch in one file-scope __device__ array
// (kScratchBytes) that every GPU loading this code keeps until the process
// exits.  Problems are processed one batch entry and one group of heads at a
// time so the scores of one group fit in the array; a problem whose single
// head does not fit is rejected.
#include <algorithm>
#include <mutex>

#include "veda_internal.cuh"

namespace veda {
namespace {

constexpr size_t kScratchBytes = (size_t)64 << 20;   // 64 MiB per device
constexpr size_t kAlignBytes = 256;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_scratch[kScratchBytes];

// Device address of g_scratch in the current context.  The name g_scratch is
// only a host-side stand-in and must never be passed to a kernel; the device
// address is looked up with cudaGetSymbolAddress once per context and cached
// under the context's unique id, so a context that is destroyed and created
// again (cudaDeviceReset, or the primary context released and retained
// again) gets a fresh lookup instead of a stale address.  A failed lookup is
// not cached: the next call tries again.
struct ScratchCache {
    std::mutex mu;
    bool have = false;
    unsigned long long ctx_id = 0;
    void* addr = nullptr;
};
ScratchCache g_cache[kMaxDevices];

cudaError_t scratch_address(void** out)
{
    int dev = 0;
    unsigned long long id = 0;
    cudaError_t e = current_context(&dev, &id);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    ScratchCache& c = g_cache[dev];
    std::lock_guard<std::mutex> lock(c.mu);
    if (!c.have || c.ctx_id != id) {
        void* a = nullptr;
        if ((e = cudaGetSymbolAddress(&a, g_scratch)) != cudaSuccess) return e;
        c.addr = a;
        c.ctx_id = id;
        c.have = true;
    }
    *out = c.addr;
    return cudaSuccess;
}

size_t align_up(size_t x) { return (x + kAlignBytes - 1) / kAlignBytes * kAlignBytes; }
int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }

}  // namespace
}  // namespace veda

using namespace veda;

extern "C" VEDA_API veda_status veda_select_tiles_noalloc(const veda_problem* p, const void* w_q,
                                                          const void* w_k, int32_t* idx_video,
                                                          int32_t* idx_ref, veda_stream_t stream)
{
    size_t ws_bytes = 0;
    veda_status st = veda_workspace_size(p, &ws_bytes);     // validates the problem
    if (st != VEDA_OK) return st;
    const int64_t nq = cdiv(p->video.n_tokens, p->tile);
    const int64_t nr = p->ref.n_tokens > 0 ? cdiv(p->ref.n_tokens, p->tile) : 0;
    if (!idx_video || (nr > 0) != (idx_ref != nullptr)) return VEDA_ERR_INVALID_ARG;
    if (!w_q || !w_k || ((uintptr_t)w_q & 15u) || ((uintptr_t)w_k & 15u)) return VEDA_ERR_INVALID_ARG;

    // scratch needed by one head: qhat, khat, khat_ref, scores, scores_ref
    const int64_t ld_v = cdiv(nq, 32) * 32, ld_r = cdiv(nr, 32) * 32;
    const size_t per_head = sizeof(float) * (size_t)(2 * nq * p->r + nr * p->r + nq * ld_v + nq * ld_r);
    const size_t fixed = kAlignBytes /* unused head block */ + 5 * kAlignBytes /* region padding */;
    if (per_head + fixed > kScratchBytes) return VEDA_ERR_WORKSPACE;   // one head does not fit
    const int hc_max = (int)std::min<size_t>((size_t)p->H, (kScratchBytes - fixed) / per_head);

    void* base = nullptr;
    if (scratch_address(&base) != cudaSuccess) return VEDA_ERR_CUDA;
    cudaStream_t s = (cudaStream_t)stream;
    char* sb = static_cast<char*>(base);

    const size_t es = p->dtype == VEDA_BF16 ? 2 : 4;
    const char* wq = static_cast<const char*>(w_q);
    const char* wk = static_cast<const char*>(w_k);
    const size_t w_head = es * (size_t)p->d * p->r;

    for (int b = 0; b < p->B; ++b) {
        for (int h0 = 0; h0 < p->H; h0 += hc_max) {
            const int hc = std::min(hc_max, p->H - h0);
            size_t off = kAlignBytes;
            float* qhat = reinterpret_cast<float*>(sb + off);   off = align_up(off + 4 * (size_t)hc * nq * p->r);
            float* khat = reinterpret_cast<float*>(sb + off);   off = align_up(off + 4 * (size_t)hc * nq * p->r);
            float* khat_r = reinterpret_cast<float*>(sb + off); off = align_up(off + 4 * (size_t)hc * nr * p->r);
            float* sc_v = reinterpret_cast<float*>(sb + off);   off = align_up(off + 4 * (size_t)hc * nq * ld_v);
            float* sc_r = reinterpret_cast<float*>(sb + off);

            PoolParams P{};
            P.B = 1; P.H = hc; P.d = p->d; P.T = p->tile; P.r = p->r; P.dtype = p->dtype;
            int64_t items = 0;
            auto add = [&](const void* x, int64_t xsb, int64_t xst, int64_t xsh, int64_t n, const char* w,
                           float* out) {
                PoolJob& J = P.job[P.n_jobs++];
                J.x = static_cast<const char*>(x) + es * ((int64_t)b * xsb + (int64_t)h0 * xsh);
                J.sb = xsb; J.st = xst; J.sh = xsh; J.n_tokens = n;
                J.n_tiles = (int32_t)cdiv(n, p->tile);
                J.first_item = items;
                J.w = w + w_head * h0;
                J.out = out;
                items += (int64_t)hc * J.n_tiles;
            };
            add(p->q, p->q_stride_b, p->q_stride_tok, p->q_stride_h, p->video.n_tokens, wq, qhat);
            add(p->video.k, p->video.stride_b, p->video.stride_tok, p->video.stride_h, p->video.n_tokens, wk,
                khat);
            if (nr > 0)
                add(p->ref.k, p->ref.stride_b, p->ref.stride_tok, p->ref.stride_h, p->ref.n_tokens, wk, khat_r);
            P.total_items = items;
            if (launch_pool_project(P, s) != cudaSuccess) return VEDA_ERR_CUDA;

            ScoreParams S{};
            S.qhat = qhat; S.BH = hc; S.nq = (int32_t)nq; S.r = p->r;
            S.khat = khat; S.scores = sc_v; S.nk = (int32_t)nq; S.ld = ld_v;
            if (launch_score(S, s) != cudaSuccess) return VEDA_ERR_CUDA;
            if (nr > 0) {
                S.khat = khat_r; S.scores = sc_r; S.nk = (int32_t)nr; S.ld = ld_r;
                if (launch_score(S, s) != cudaSuccess) return VEDA_ERR_CUDA;
            }

            const int64_t row0 = ((int64_t)b * p->H + h0) * nq;
            TopkParams T{};
            T.status = nullptr;     // the selection kernels record no device-side errors
            T.rows = (int64_t)hc * nq;
            T.scores = sc_v; T.ld = ld_v; T.n = (int32_t)nq; T.k = p->video.budget;
            T.idx = idx_video + row0 * p->video.budget;
            if (launch_topk(T, s) != cudaSuccess) return VEDA_ERR_CUDA;
            if (nr > 0) {
                T.scores = sc_r; T.ld = ld_r; T.n = (int32_t)nr; T.k = p->ref.budget;
                T.idx = idx_ref + row0 * p->ref.budget;
                if (launch_topk(T, s) != cudaSuccess) return VEDA_ERR_CUDA;
            }
        }
    }
    return VEDA_OK;
}
