// libveda host entry points: argument validation, workspace layout, launches.
//
// Every check here runs on the host before anything is enqueued, so an
// invalid call returns an error code and leaves the device untouched.
#include <cuda.h>
#include <math.h>
#include <string.h>

#include <mutex>

#include "veda_internal.cuh"

namespace veda {

namespace {
typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

template <typename Fn>
Fn driver_fn(const char* name)
{
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint(name, &fn, cudaEnableDefault, &q) != cudaSuccess || q != cudaDriverEntryPointSuccess)
        return nullptr;
    return reinterpret_cast<Fn>(fn);
}
}  // namespace

cudaError_t current_context(int* device, unsigned long long* ctx_id)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    // since CUDA 12, cudaSetDevice initialises the primary context (no-op when current)
    if ((e = cudaSetDevice(dev)) != cudaSuccess) return e;
    static CtxGetCurrentFn get_current = driver_fn<CtxGetCurrentFn>("cuCtxGetCurrent");
    static CtxGetIdFn get_id = driver_fn<CtxGetIdFn>("cuCtxGetId");
    if (!get_current || !get_id) return cudaErrorNotSupported;
    CUcontext ctx = nullptr;
    if (get_current(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, ctx_id) != CUDA_SUCCESS)
        return cudaErrorDeviceUninitialized;
    *device = dev;
    return cudaSuccess;
}

int num_sms()
{
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
    return n;
}

cudaError_t launch_attn_tc(const AttnParams& p, cudaStream_t s);
bool attn_tc_supported(const AttnParams& p);

namespace {

constexpr size_t kAlign = 256;

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

struct Layout {
    int64_t nq, nr;          // query (= video key) tiles, reference tiles
    int64_t ld_v, ld_r;      // score row strides (elements)
    size_t qhat, khat, khat_r, sc_v, sc_r;
    size_t qpl, kpl, kpl_r;  // bf16 planes of the projections (fused scoring), r <= 64
    size_t ksm, ksm_r;       // the planes of the 64 sampled key tiles per head
    size_t fb_v, fb_r;       // fused selection: rows left to the exact top-k (count, then ids)
    size_t total;
};

constexpr int kPlaneWidth = 64;   // columns of a projection plane row

size_t esize(veda_dtype t) { return t == VEDA_BF16 ? 2 : 4; }

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

bool stride_ok(int64_t s, size_t es) { return s >= 0 && ((uint64_t)s * es) % 16 == 0; }

veda_status check_segment(const veda_segment& s, const veda_problem& p, bool sparse, bool required)
{
    if (s.n_tokens < 0 || s.n_tokens > (int64_t)1 << 30) return VEDA_ERR_INVALID_ARG;
    if (s.n_tokens == 0) {
        if (required) return VEDA_ERR_INVALID_ARG;
        return s.budget == 0 ? VEDA_OK : VEDA_ERR_INVALID_ARG;
    }
    if (!s.k || !s.v || !aligned16(s.k) || !aligned16(s.v)) return VEDA_ERR_INVALID_ARG;
    const size_t es = esize(p.dtype);
    if (!stride_ok(s.stride_b, es) || !stride_ok(s.stride_tok, es) || !stride_ok(s.stride_h, es))
        return VEDA_ERR_INVALID_ARG;
    if (s.stride_tok < p.d && s.n_tokens > 1) return VEDA_ERR_INVALID_ARG;
    const int64_t tiles = ceil_div(s.n_tokens, p.tile);
    if (sparse) {
        if (s.budget < 1 || s.budget > tiles) return VEDA_ERR_INVALID_ARG;
        if (tiles > topk_max_tiles()) return VEDA_ERR_UNSUPPORTED;
    } else if (s.budget != 0) {
        return VEDA_ERR_INVALID_ARG;
    }
    return VEDA_OK;
}

veda_status validate(const veda_problem* pp)
{
    if (!pp) return VEDA_ERR_INVALID_ARG;
    const veda_problem& p = *pp;
    if (p.B < 1 || p.H < 1 || (int64_t)p.B * p.H > 65535) return VEDA_ERR_INVALID_ARG;
    if (p.dtype != VEDA_F32 && p.dtype != VEDA_BF16) return VEDA_ERR_INVALID_ARG;
    if (p.d < 1 || p.tile < 1 || p.r < 1) return VEDA_ERR_INVALID_ARG;
    if (p.d != 64 && p.d != 128) return VEDA_ERR_UNSUPPORTED;
    if (p.tile != 64 && p.tile != 128) return VEDA_ERR_UNSUPPORTED;
    if (p.r > 128 || p.r % 4 != 0) return VEDA_ERR_UNSUPPORTED;
    if (!(p.softmax_scale >= 0.f) || !isfinite(p.softmax_scale)) return VEDA_ERR_INVALID_ARG;
    if (p.flags & ~(VEDA_FLAG_SIMT_ATTENTION | VEDA_FLAG_TEST_SHORT_WAITS | VEDA_FLAG_UNFUSED_SELECTION |
                    VEDA_FLAG_ONCHIP_SELECTION))
        return VEDA_ERR_INVALID_ARG;
    if (!p.q || !aligned16(p.q)) return VEDA_ERR_INVALID_ARG;
    const size_t es = esize(p.dtype);
    if (!stride_ok(p.q_stride_b, es) || !stride_ok(p.q_stride_tok, es) || !stride_ok(p.q_stride_h, es))
        return VEDA_ERR_INVALID_ARG;
    veda_status st;
    if ((st = check_segment(p.video, p, true, true)) != VEDA_OK) return st;
    if ((st = check_segment(p.ref, p, true, false)) != VEDA_OK) return st;
    if ((st = check_segment(p.dense, p, false, false)) != VEDA_OK) return st;
    return VEDA_OK;
}

Layout layout(const veda_problem& p)
{
    Layout L;
    L.nq = ceil_div(p.video.n_tokens, p.tile);
    L.nr = p.ref.n_tokens > 0 ? ceil_div(p.ref.n_tokens, p.tile) : 0;
    L.ld_v = (int64_t)align_up((size_t)L.nq, 32);
    L.ld_r = (int64_t)align_up((size_t)L.nr, 32);
    const int64_t BH = (int64_t)p.B * p.H;
    size_t off = kAlign;                                   // status word lives at offset 0
    L.qhat = off;   off = align_up(off + sizeof(float) * BH * L.nq * p.r, kAlign);
    L.khat = off;   off = align_up(off + sizeof(float) * BH * L.nq * p.r, kAlign);
    L.khat_r = off; off = align_up(off + sizeof(float) * BH * L.nr * p.r, kAlign);
    L.sc_v = off;   off = align_up(off + sizeof(float) * BH * L.nq * L.ld_v, kAlign);
    L.sc_r = off;   off = align_up(off + sizeof(float) * BH * L.nq * L.ld_r, kAlign);
    const bool planes = p.r <= kPlaneWidth;
    L.qpl = off;    off = align_up(off + (planes ? 3 * 2 * BH * L.nq * kPlaneWidth : 0), kAlign);
    L.kpl = off;    off = align_up(off + (planes ? 3 * 2 * BH * L.nq * kPlaneWidth : 0), kAlign);
    L.kpl_r = off;  off = align_up(off + (planes ? 3 * 2 * BH * L.nr * kPlaneWidth : 0), kAlign);
    L.ksm = off;    off = align_up(off + (planes ? 3 * 2 * BH * 64 * kPlaneWidth : 0), kAlign);
    L.ksm_r = off;  off = align_up(off + (planes && L.nr > 0 ? 3 * 2 * BH * 64 * kPlaneWidth : 0), kAlign);
    L.fb_v = off;   off = align_up(off + sizeof(int32_t) * (1 + BH * L.nq), kAlign);
    L.fb_r = off;   off = align_up(off + sizeof(int32_t) * (L.nr > 0 ? 1 + BH * L.nq : 0), kAlign);
    L.total = off;
    return L;
}

veda_status check_ws(const veda_problem& p, void* ws, size_t ws_bytes, Layout* L)
{
    *L = layout(p);
    if (!ws || ((uintptr_t)ws % kAlign) != 0 || ws_bytes < L->total) return VEDA_ERR_WORKSPACE;
    return VEDA_OK;
}

template <typename T>
T* at(void* ws, size_t off) { return reinterpret_cast<T*>(static_cast<char*>(ws) + off); }

veda_status from_cuda(cudaError_t e) { return e == cudaSuccess ? VEDA_OK : VEDA_ERR_CUDA; }

Segment to_segment(const veda_segment& s, int tile)
{
    Segment d;
    d.k = s.k;
    d.v = s.v;
    d.n = s.n_tokens;
    d.sb = s.stride_b;
    d.st = s.stride_tok;
    d.sh = s.stride_h;
    d.n_tiles = s.n_tokens > 0 ? (int32_t)ceil_div(s.n_tokens, tile) : 0;
    d.pad = 0;
    return d;
}

veda_status do_pool_project(const veda_problem& p, const Layout& L, const void* w_q, const void* w_k,
                            void* ws, cudaStream_t s)
{
    if (!w_q || !w_k || !aligned16(w_q) || !aligned16(w_k)) return VEDA_ERR_INVALID_ARG;
    PoolParams P;
    memset(&P, 0, sizeof P);
    P.B = p.B; P.H = p.H; P.d = p.d; P.T = p.tile; P.r = p.r; P.dtype = p.dtype;
    int64_t items = 0;
    const bool planes = p.r <= kPlaneWidth;   // bf16 planes for the tensor-core scoring
    auto add = [&](const void* x, int64_t sb, int64_t st, int64_t sh, int64_t n, const void* w, float* out,
                   size_t plane_off, size_t sample_off) {
        PoolJob& J = P.job[P.n_jobs++];
        J.x = x; J.sb = sb; J.st = st; J.sh = sh; J.n_tokens = n;
        J.n_tiles = (int32_t)ceil_div(n, p.tile);
        J.first_item = items;
        J.w = w; J.out = out;
        J.planes = planes ? at<uint16_t>(ws, plane_off) : nullptr;
        J.plane_stride = (int64_t)p.B * p.H * J.n_tiles * kPlaneWidth;
        J.sample_planes = planes && sample_off ? at<uint16_t>(ws, sample_off) : nullptr;
        J.sample_plane_stride = (int64_t)p.B * p.H * 64 * kPlaneWidth;
        items += (int64_t)p.B * p.H * J.n_tiles;
    };
    add(p.q, p.q_stride_b, p.q_stride_tok, p.q_stride_h, p.video.n_tokens, w_q, at<float>(ws, L.qhat), L.qpl, 0);
    add(p.video.k, p.video.stride_b, p.video.stride_tok, p.video.stride_h, p.video.n_tokens, w_k,
        at<float>(ws, L.khat), L.kpl, L.ksm);
    if (p.ref.n_tokens > 0)
        add(p.ref.k, p.ref.stride_b, p.ref.stride_tok, p.ref.stride_h, p.ref.n_tokens, w_k,
            at<float>(ws, L.khat_r), L.kpl_r, L.ksm_r);
    P.total_items = items;
    return from_cuda(launch_pool_project(P, s));
}

veda_status do_score(const veda_problem& p, const Layout& L, void* ws, cudaStream_t s)
{
    ScoreParams S;
    S.qhat = at<float>(ws, L.qhat);
    S.BH = p.B * p.H;
    S.nq = (int32_t)L.nq;
    S.r = p.r;
    S.khat = at<float>(ws, L.khat);
    S.scores = at<float>(ws, L.sc_v);
    S.nk = (int32_t)L.nq;
    S.ld = L.ld_v;
    cudaError_t e = launch_score(S, s);
    if (e == cudaSuccess && L.nr > 0) {
        S.khat = at<float>(ws, L.khat_r);
        S.scores = at<float>(ws, L.sc_r);
        S.nk = (int32_t)L.nr;
        S.ld = L.ld_r;
        e = launch_score(S, s);
    }
    return from_cuda(e);
}

veda_status do_topk(const veda_problem& p, const Layout& L, int32_t* idx_v, int32_t* idx_r, void* ws,
                    cudaStream_t s, uint32_t* status = nullptr)
{
    if (!idx_v || (L.nr > 0) != (idx_r != nullptr)) return VEDA_ERR_INVALID_ARG;
    TopkParams T{};
    T.status = status ? status : at<uint32_t>(ws, 0);
    T.rows = (int64_t)p.B * p.H * L.nq;
    T.scores = at<float>(ws, L.sc_v);
    T.ld = L.ld_v;
    T.n = (int32_t)L.nq;
    T.k = p.video.budget;
    T.idx = idx_v;
    cudaError_t e = launch_topk(T, s);
    if (e == cudaSuccess && L.nr > 0) {
        T.scores = at<float>(ws, L.sc_r);
        T.ld = L.ld_r;
        T.n = (int32_t)L.nr;
        T.k = p.ref.budget;
        T.idx = idx_r;
        e = launch_topk(T, s);
    }
    return from_cuda(e);
}

// Whether the tile scores are computed on the tensor cores (from the bf16
// projection planes) rather than by the fp32 SIMT kernel.
bool use_tensor_scores(const veda_problem& p, const Layout& L)
{
    if (p.flags & VEDA_FLAG_UNFUSED_SELECTION) return false;
    return select_tc_supported(p.r, (int)(L.nq > L.nr ? L.nq : L.nr));
}

// Steps 2-3 on the tensor cores, from the projection planes in the
// workspace: with scores_only the exact scores are written to the
// workspace (then the warp-per-row top-k runs); otherwise each row's top-k
// is selected on chip and no score matrix is written.
veda_status do_select_tc(const veda_problem& p, const Layout& L, int32_t* idx_v, int32_t* idx_r, void* ws,
                         cudaStream_t s, uint32_t* status, bool scores_only)
{
    if (!idx_v || (L.nr > 0) != (idx_r != nullptr)) return VEDA_ERR_INVALID_ARG;
    if (p.r > kPlaneWidth) return VEDA_ERR_UNSUPPORTED;
    SelectParams S{};
    S.scores_only = scores_only ? 1 : 0;
    S.q_planes = at<uint16_t>(ws, L.qpl);
    S.BH = p.B * p.H;
    S.nq = (int32_t)L.nq;
    S.status = status ? status : at<uint32_t>(ws, 0);
    S.short_waits = (p.flags & VEDA_FLAG_TEST_SHORT_WAITS) ? 1 : 0;
    S.n_jobs = L.nr > 0 ? 2 : 1;
    SelectJob& V = S.job[0];
    V.k_planes = at<uint16_t>(ws, L.kpl);
    V.k_sample = at<uint16_t>(ws, L.ksm);
    V.nk = (int32_t)L.nq;
    V.k = p.video.budget;
    V.idx = idx_v;
    V.sc = at<float>(ws, L.sc_v);
    V.ld = L.ld_v;
    V.fb = at<int32_t>(ws, L.fb_v);
    if (L.nr > 0) {
        SelectJob& R = S.job[1];
        R.k_planes = at<uint16_t>(ws, L.kpl_r);
        R.k_sample = at<uint16_t>(ws, L.ksm_r);
        R.nk = (int32_t)L.nr;
        R.k = p.ref.budget;
        R.idx = idx_r;
        R.sc = at<float>(ws, L.sc_r);
        R.ld = L.ld_r;
        R.fb = at<int32_t>(ws, L.fb_r);
    }
    return from_cuda(launch_select_tc(S, s));
}

// Steps 2-3 on the workspace's projections: tensor-core scores and the
// warp-per-row top-k by default, the on-chip selection with
// VEDA_FLAG_ONCHIP_SELECTION, fp32 SIMT scores with VEDA_FLAG_UNFUSED_SELECTION
// (or when the tensor-core path does not apply).
veda_status do_score_topk(const veda_problem& p, const Layout& L, int32_t* idx_v, int32_t* idx_r, void* ws,
                          cudaStream_t s, uint32_t* status = nullptr)
{
    veda_status st;
    if (use_tensor_scores(p, L)) {
        if (p.flags & VEDA_FLAG_ONCHIP_SELECTION) return do_select_tc(p, L, idx_v, idx_r, ws, s, status, false);
        st = do_select_tc(p, L, idx_v, idx_r, ws, s, status, true);
    } else {
        st = do_score(p, L, ws, s);
    }
    if (st != VEDA_OK) return st;
    return do_topk(p, L, idx_v, idx_r, ws, s, status);
}

veda_status do_attn(const veda_problem& p, const Layout& L, const int32_t* idx_v, const int32_t* idx_r,
                    void* out, float* lse, void* ws, cudaStream_t s, uint32_t* status = nullptr)
{
    if (!idx_v || (L.nr > 0) != (idx_r != nullptr)) return VEDA_ERR_INVALID_ARG;
    if (!out || !aligned16(out) || (lse && ((uintptr_t)lse & 3u))) return VEDA_ERR_INVALID_ARG;
    AttnParams A;
    memset(&A, 0, sizeof A);
    A.q = p.q;
    A.qsb = p.q_stride_b; A.qst = p.q_stride_tok; A.qsh = p.q_stride_h;
    A.n_qtok = p.video.n_tokens;
    A.video = to_segment(p.video, p.tile);
    A.ref = to_segment(p.ref, p.tile);
    A.dense = to_segment(p.dense, p.tile);
    A.idx_v = idx_v;
    A.idx_r = L.nr > 0 ? idx_r : nullptr;
    A.k_v = p.video.budget;
    A.k_r = L.nr > 0 ? p.ref.budget : 0;
    A.out = out;
    A.lse = lse;
    A.B = p.B; A.H = p.H; A.d = p.d; A.T = p.tile; A.nq = (int32_t)L.nq;
    A.dtype = p.dtype;
    A.scale = p.softmax_scale > 0.f ? p.softmax_scale : 1.0f / sqrtf((float)p.d);
    A.status = status ? status : at<uint32_t>(ws, 0);
    A.short_waits = (p.flags & VEDA_FLAG_TEST_SHORT_WAITS) ? 1 : 0;
    if (!(p.flags & VEDA_FLAG_SIMT_ATTENTION) && attn_tc_supported(A)) return from_cuda(launch_attn_tc(A, s));
    return from_cuda(launch_attn_simt(A, s));
}

// Key-range split for few (b, h, query tile) units: the number of ranges S
// (1..4) that minimises the waves of the persistent grid per unit of work,
// with a 5% charge for the merge.
int choose_split(int64_t units, int n_list)
{
    const int64_t sms = num_sms();
    int best = 1;
    double best_cost = (double)((units + sms - 1) / sms);
    for (int S = 2; S <= 4 && 2 * S <= n_list; ++S) {
        const double cost = (double)((units * S + sms - 1) / sms) / S * 1.05;
        if (cost < best_cost) {
            best = S;
            best_cost = cost;
        }
    }
    return best;
}

// Dense-query rows: every query row attends to every token of every segment.
veda_status do_dense_query_attn(const veda_problem& p, const void* q_rows, int64_t n_rows, int64_t sb, int64_t st,
                                int64_t sh, void* out, float* lse, void* ws, size_t ws_bytes, cudaStream_t s)
{
    const size_t es = esize(p.dtype);
    if (n_rows < 1 || n_rows > (int64_t)1 << 30 || !q_rows || !aligned16(q_rows)) return VEDA_ERR_INVALID_ARG;
    if (!stride_ok(sb, es) || !stride_ok(st, es) || !stride_ok(sh, es)) return VEDA_ERR_INVALID_ARG;
    if (!out || !aligned16(out) || (lse && ((uintptr_t)lse & 3u))) return VEDA_ERR_INVALID_ARG;
    AttnParams A;
    memset(&A, 0, sizeof A);
    A.q = q_rows;
    A.qsb = sb; A.qst = st; A.qsh = sh;
    A.n_qtok = n_rows;
    A.video = to_segment(p.video, p.tile);
    A.ref = to_segment(p.ref, p.tile);
    A.dense = to_segment(p.dense, p.tile);
    A.idx_v = nullptr;                  // every video tile
    A.idx_r = nullptr;                  // every reference tile
    A.k_v = A.video.n_tiles;
    A.k_r = p.ref.n_tokens > 0 ? A.ref.n_tiles : 0;
    A.out = out;
    A.lse = lse;
    A.B = p.B; A.H = p.H; A.d = p.d; A.T = p.tile;
    A.nq = (int32_t)((n_rows + p.tile - 1) / p.tile);
    A.dtype = p.dtype;
    A.scale = p.softmax_scale > 0.f ? p.softmax_scale : 1.0f / sqrtf((float)p.d);
    A.status = at<uint32_t>(ws, 0);
    A.short_waits = (p.flags & VEDA_FLAG_TEST_SHORT_WAITS) ? 1 : 0;
    if (!(p.flags & VEDA_FLAG_SIMT_ATTENTION) && attn_tc_supported(A)) {
        // few units: split every key list over S CTAs and merge, with the
        // partial results in the workspace past its status block (if they fit)
        const int S = choose_split((int64_t)A.B * A.H * A.nq, A.k_v + A.k_r + A.dense.n_tiles);
        const size_t rows = (size_t)A.B * A.H * (size_t)n_rows;
        const size_t o_bytes = align_up(sizeof(float) * S * rows * p.d, kAlign);
        const size_t ml_bytes = align_up(sizeof(float) * 2 * S * rows, kAlign);
        if (S > 1 && kAlign + o_bytes + ml_bytes <= ws_bytes) {
            A.n_split = S;
            A.part_o = at<float>(ws, kAlign);
            A.part_ml = at<float>(ws, kAlign + o_bytes);
        }
        return from_cuda(launch_attn_tc(A, s));
    }
    return from_cuda(launch_attn_simt(A, s));
}


// ---- host-buffer call: head groups pipelined over three streams ---------
// The caller's device buffer: a 256-byte status block, then two slots, each
// holding one head group's inputs, weights, indices, output and workspace.
struct HostSlot {
    size_t q, kv[6], wq, wk, iv, ir, out, lse, ws, total;   // offsets inside a slot
};

// [B, n, H, d] with nothing between rows: the head range of a group is then a
// 2-D block of B * n rows.
bool packed(const void* base, int64_t B, int64_t n, int64_t H, int64_t d, int64_t sb, int64_t st, int64_t sh)
{
    return base && sh == d && st == H * d && (sb == n * H * d || B == 1);
}

// The hc-head sub-problem of slot `slot` (device pointers, packed [B, n, hc, d]).
veda_problem sub_problem(const veda_problem& p, int hc, char* slot, const HostSlot& S)
{
    veda_problem c = p;
    c.H = hc;
    auto seg = [&](veda_segment& sg, size_t ok, size_t ov) {
        if (sg.n_tokens == 0) return;
        sg.k = slot + ok;
        sg.v = slot + ov;
        sg.stride_h = p.d;
        sg.stride_tok = (int64_t)hc * p.d;
        sg.stride_b = sg.n_tokens * hc * p.d;
    };
    c.q = slot + S.q;
    c.q_stride_h = p.d;
    c.q_stride_tok = (int64_t)hc * p.d;
    c.q_stride_b = p.video.n_tokens * hc * p.d;
    seg(c.video, S.kv[0], S.kv[1]);
    seg(c.ref, S.kv[2], S.kv[3]);
    seg(c.dense, S.kv[4], S.kv[5]);
    return c;
}

HostSlot host_slot(const veda_problem& p, int hc)
{
    HostSlot S;
    const size_t es = esize(p.dtype);
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t at_ = off;
        off = align_up(off + bytes, kAlign);
        return at_;
    };
    const size_t row = (size_t)hc * p.d * es;
    S.q = take((size_t)p.B * p.video.n_tokens * row);
    const veda_segment* segs[3] = {&p.video, &p.ref, &p.dense};
    for (int g = 0; g < 3; ++g) {
        S.kv[2 * g] = take((size_t)p.B * segs[g]->n_tokens * row);
        S.kv[2 * g + 1] = take((size_t)p.B * segs[g]->n_tokens * row);
    }
    S.wq = take((size_t)hc * p.d * p.r * es);
    S.wk = take((size_t)hc * p.d * p.r * es);
    veda_problem c = p;
    c.H = hc;
    const Layout L = layout(c);
    S.iv = take(sizeof(int32_t) * (size_t)p.B * hc * L.nq * p.video.budget);
    S.ir = take(sizeof(int32_t) * (size_t)p.B * hc * L.nq * (L.nr > 0 ? p.ref.budget : 0));
    S.out = take((size_t)p.B * p.video.n_tokens * row);
    S.lse = take(sizeof(float) * (size_t)p.B * hc * p.video.n_tokens);
    S.ws = take(L.total);
    S.total = off;
    return S;
}

// The three streams and nine events veda_attn_host forks its work onto, made
// once per device and context and reused by every call (a call holds the
// device's lock while it enqueues, so concurrent calls take turns on them).
constexpr int kMaxDevices = 64;
struct HostStreams {
    std::mutex mu;
    bool have = false;
    unsigned long long ctx_id = 0;
    cudaStream_t s[3] = {};
    cudaEvent_t ev[9] = {};
};
HostStreams g_host_streams[kMaxDevices];

// Locks and returns the device's streams and events, making them if this
// context has none yet.  nullptr on failure (nothing locked).
HostStreams* host_streams(std::unique_lock<std::mutex>* lock)
{
    int dev = 0;
    unsigned long long id = 0;
    if (current_context(&dev, &id) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    HostStreams& h = g_host_streams[dev];
    std::unique_lock<std::mutex> lk(h.mu);
    if (!h.have || h.ctx_id != id) {
        // a new context: the previous one's handles died with it
        HostStreams fresh_handles;
        bool ok = true;
        for (int i = 0; i < 3 && ok; ++i)
            ok = cudaStreamCreateWithFlags(&fresh_handles.s[i], cudaStreamNonBlocking) == cudaSuccess;
        for (int i = 0; i < 9 && ok; ++i)
            ok = cudaEventCreateWithFlags(&fresh_handles.ev[i], cudaEventDisableTiming) == cudaSuccess;
        if (!ok) {
            for (int i = 0; i < 9; ++i)
                if (fresh_handles.ev[i]) cudaEventDestroy(fresh_handles.ev[i]);
            for (int i = 0; i < 3; ++i)
                if (fresh_handles.s[i]) cudaStreamDestroy(fresh_handles.s[i]);
            return nullptr;
        }
        for (int i = 0; i < 3; ++i) h.s[i] = fresh_handles.s[i];
        for (int i = 0; i < 9; ++i) h.ev[i] = fresh_handles.ev[i];
        h.ctx_id = id;
        h.have = true;
    }
    *lock = std::move(lk);
    return &h;
}

veda_status check_host_problem(const veda_problem& p, int heads_per_group)
{
    if (heads_per_group < 1) return VEDA_ERR_INVALID_ARG;
    if (!packed(p.q, p.B, p.video.n_tokens, p.H, p.d, p.q_stride_b, p.q_stride_tok, p.q_stride_h))
        return VEDA_ERR_UNSUPPORTED;
    const veda_segment* segs[3] = {&p.video, &p.ref, &p.dense};
    for (auto* sg : segs)
        if (sg->n_tokens > 0 &&
            (!packed(sg->k, p.B, sg->n_tokens, p.H, p.d, sg->stride_b, sg->stride_tok, sg->stride_h) ||
             !packed(sg->v, p.B, sg->n_tokens, p.H, p.d, sg->stride_b, sg->stride_tok, sg->stride_h)))
            return VEDA_ERR_UNSUPPORTED;
    return VEDA_OK;
}

}  // namespace
}  // namespace veda

using namespace veda;

extern "C" {

veda_status veda_workspace_size(const veda_problem* p, size_t* bytes)
{
    if (!bytes) return VEDA_ERR_INVALID_ARG;
    veda_status st = validate(p);
    if (st != VEDA_OK) return st;
    *bytes = layout(*p).total;
    return VEDA_OK;
}

veda_status veda_workspace_init(void* ws, size_t ws_bytes, veda_stream_t stream)
{
    if (!ws || ((uintptr_t)ws % kAlign) != 0 || ws_bytes < kAlign) return VEDA_ERR_WORKSPACE;
    return from_cuda(cudaMemsetAsync(ws, 0, kAlign, (cudaStream_t)stream));
}

veda_status veda_pool_project(const veda_problem* p, const void* w_q, const void* w_k, void* ws,
                              size_t ws_bytes, veda_stream_t stream)
{
    veda_status st = validate(p);
    if (st != VEDA_OK) return st;
    Layout L;
    if ((st = check_ws(*p, ws, ws_bytes, &L)) != VEDA_OK) return st;
    return do_pool_project(*p, L, w_q, w_k, ws, (cudaStream_t)stream);
}

veda_status veda_score_tiles(const veda_problem* p, void* ws, size_t ws_bytes, veda_stream_t stream)
{
    veda_status st = validate(p);
    if (st != VEDA_OK) return st;
    Layout L;
    if ((st = check_ws(*p, ws, ws_bytes, &L)) != VEDA_OK) return st;
    return do_score(*p, L, ws, (cudaStream_t)stream);
}

veda_status veda_topk_tiles(const veda_problem* p, int32_t* idx_video, int32_t* idx_ref, void* ws,
                            size_t ws_bytes, veda_stream_t stream)
{
    veda_status st = validate(p);
    if (st != VEDA_OK) return st;
    Layout L;
    if ((st = check_ws(*p, ws, ws_bytes, &L)) != VEDA_OK) return st;
    return do_topk(*p, L, idx_video, idx_ref, ws, (cudaStream_t)stream);
}

veda_status veda_select_tiles(const veda_problem* p, const void* w_q, const void* w_k, int32_t* idx_video,
                              int32_t* idx_ref, void* ws, size_t ws_bytes, veda_stream_t stream)
{
    veda_status st = validate(p);
    if (st != VEDA_OK) return st;
    Layout L;
    if ((st = check_ws(*p, ws, ws_bytes, &L)) != VEDA_OK) return st;
    if (!idx_video || (L.nr > 0) != (idx_ref != nullptr)) return VEDA_ERR_INVALID_ARG;
    cudaStream_t s = (cudaStream_t)stream;
    if ((st = do_pool_project(*p, L, w_q, w_k, ws, s)) != VEDA_OK) return st;
    return do_score_topk(*p, L, idx_video, idx_ref, ws, s);
}

veda_status veda_score_topk_tiles(const veda_problem* p, int32_t* idx_video, int32_t* idx_ref, void* ws,
                                  size_t ws_bytes, veda_stream_t stream)
{
    veda_status st = validate(p);
    if (st != VEDA_OK) return st;
    Layout L;
    if ((st = check_ws(*p, ws, ws_bytes, &L)) != VEDA_OK) return st;
    if (!idx_video || (L.nr > 0) != (idx_ref != nullptr)) return VEDA_ERR_INVALID_ARG;
    return do_score_topk(*p, L, idx_video, idx_ref, ws, (cudaStream_t)stream);
}

veda_status veda_block_sparse_attn(const veda_problem* p, const int32_t* idx_video, const int32_t* idx_ref,
                                   void* out, float* lse, void* ws, size_t ws_bytes, veda_stream_t stream)
{
    veda_status st = validate(p);
    if (st != VEDA_OK) return st;
    if (!ws || ((uintptr_t)ws % kAlign) != 0 || ws_bytes < kAlign) return VEDA_ERR_WORKSPACE;
    const Layout L = layout(*p);
    return do_attn(*p, L, idx_video, idx_ref, out, lse, ws, (cudaStream_t)stream);
}

veda_status veda_dense_query_attn(const veda_problem* p, const void* q_rows, int64_t n_rows, int64_t q_stride_b,
                                  int64_t q_stride_tok, int64_t q_stride_h, void* out, float* lse, void* ws,
                                  size_t ws_bytes, veda_stream_t stream)
{
    veda_status st = validate(p);
    if (st != VEDA_OK) return st;
    if (!ws || ((uintptr_t)ws % kAlign) != 0 || ws_bytes < kAlign) return VEDA_ERR_WORKSPACE;
    return do_dense_query_attn(*p, q_rows, n_rows, q_stride_b, q_stride_tok, q_stride_h, out, lse, ws, ws_bytes,
                               (cudaStream_t)stream);
}

veda_status veda_attn_host_buffer_size(const veda_problem* p, int32_t heads_per_group, size_t* bytes)
{
    if (!bytes) return VEDA_ERR_INVALID_ARG;
    veda_status st = validate(p);
    if (st != VEDA_OK) return st;
    if ((st = check_host_problem(*p, heads_per_group)) != VEDA_OK) return st;
    const int hc = heads_per_group < p->H ? heads_per_group : p->H;
    *bytes = kAlign + 2 * host_slot(*p, hc).total;
    return VEDA_OK;
}

veda_status veda_attn_host(const veda_problem* p, const void* w_q, const void* w_k, int32_t* idx_video,
                           int32_t* idx_ref, void* out, float* lse, int32_t heads_per_group, void* dev_buf,
                           size_t dev_bytes, veda_stream_t stream)
{
    veda_status st = validate(p);
    if (st != VEDA_OK) return st;
    if ((st = check_host_problem(*p, heads_per_group)) != VEDA_OK) return st;
    const veda_problem& P = *p;
    const int hc = heads_per_group < P.H ? heads_per_group : P.H;
    const HostSlot S = host_slot(P, hc);
    if (!dev_buf || ((uintptr_t)dev_buf % kAlign) != 0 || dev_bytes < kAlign + 2 * S.total) return VEDA_ERR_WORKSPACE;
    if (!w_q || !w_k || !out || (lse && ((uintptr_t)lse & 3u))) return VEDA_ERR_INVALID_ARG;
    if ((P.ref.n_tokens > 0) != (idx_ref != nullptr) && idx_video) return VEDA_ERR_INVALID_ARG;
    const size_t es = esize(P.dtype);
    const int64_t nq = (P.video.n_tokens + P.tile - 1) / P.tile;
    uint32_t* status = static_cast<uint32_t*>(dev_buf);
    char* slots[2] = {static_cast<char*>(dev_buf) + kAlign, static_cast<char*>(dev_buf) + kAlign + S.total};
    cudaStream_t caller = (cudaStream_t)stream;

    // three streams (copy in, compute, copy out) forked from and joined back to the caller's stream
    std::unique_lock<std::mutex> hs_lock;
    HostStreams* hs = host_streams(&hs_lock);
    if (!hs) return VEDA_ERR_CUDA;
    cudaStream_t sin = hs->s[0], scomp = hs->s[1], sout = hs->s[2];
    cudaEvent_t* ev = hs->ev;
    cudaEvent_t &e_fork = ev[0], &e_in0 = ev[1], &e_in1 = ev[2], &e_c0 = ev[3], &e_c1 = ev[4], &e_free0 = ev[5],
                &e_free1 = ev[6], &e_comp_end = ev[7], &e_out_end = ev[8];
    cudaEvent_t e_in[2] = {e_in0, e_in1}, e_comp[2] = {e_c0, e_c1}, e_free[2] = {e_free0, e_free1};
    st = VEDA_OK;
    {
        const bool ok = cudaEventRecord(e_fork, caller) == cudaSuccess &&
                        cudaStreamWaitEvent(sin, e_fork, 0) == cudaSuccess &&
                        cudaStreamWaitEvent(scomp, e_fork, 0) == cudaSuccess &&
                        cudaStreamWaitEvent(sout, e_fork, 0) == cudaSuccess;
        if (!ok) st = VEDA_ERR_CUDA;
    }
    const veda_segment* hsegs[3] = {&P.video, &P.ref, &P.dense};
    for (int h0 = 0, c = 0; h0 < P.H && st == VEDA_OK; h0 += hc, ++c) {
        const int g = P.H - h0 < hc ? P.H - h0 : hc;   // heads in this group
        const int sl = c & 1;
        char* slot = slots[sl];
        bool k_ok = true;
        // ---- copy in (after the slot's previous group has been copied out) ----
        if (c >= 2) k_ok = cudaStreamWaitEvent(sin, e_free[sl], 0) == cudaSuccess;
        const size_t row = (size_t)g * P.d * es, hrow = (size_t)P.H * P.d * es, drow = (size_t)hc * P.d * es;
        auto in2d = [&](size_t off, const void* host, int64_t n) {
            if (n > 0 && k_ok)
                k_ok = cudaMemcpy2DAsync(slot + off, drow, static_cast<const char*>(host) + (size_t)h0 * P.d * es,
                                         hrow, row, (size_t)P.B * n, cudaMemcpyHostToDevice, sin) == cudaSuccess;
        };
        in2d(S.q, P.q, P.video.n_tokens);
        for (int s3 = 0; s3 < 3; ++s3) {
            in2d(S.kv[2 * s3], hsegs[s3]->k, hsegs[s3]->n_tokens);
            in2d(S.kv[2 * s3 + 1], hsegs[s3]->v, hsegs[s3]->n_tokens);
        }
        const size_t wbytes = (size_t)g * P.d * P.r * es;
        if (k_ok) k_ok = cudaMemcpyAsync(slot + S.wq, static_cast<const char*>(w_q) + (size_t)h0 * P.d * P.r * es,
                                         wbytes, cudaMemcpyHostToDevice, sin) == cudaSuccess;
        if (k_ok) k_ok = cudaMemcpyAsync(slot + S.wk, static_cast<const char*>(w_k) + (size_t)h0 * P.d * P.r * es,
                                         wbytes, cudaMemcpyHostToDevice, sin) == cudaSuccess;
        if (k_ok) k_ok = cudaEventRecord(e_in[sl], sin) == cudaSuccess;
        // ---- compute the group's selection and attention ----
        veda_problem cp = sub_problem(P, hc, slot, S);
        cp.H = g;
        // the group's tensors are packed for hc heads; a short last group keeps that layout
        cp.q_stride_tok = (int64_t)hc * P.d;
        const Layout L = layout(cp);
        void* ws = slot + S.ws;
        int32_t* iv = reinterpret_cast<int32_t*>(slot + S.iv);
        int32_t* ir = L.nr > 0 ? reinterpret_cast<int32_t*>(slot + S.ir) : nullptr;
        if (k_ok) k_ok = cudaStreamWaitEvent(scomp, e_in[sl], 0) == cudaSuccess;
        if (!k_ok) { st = VEDA_ERR_CUDA; break; }
        if ((st = do_pool_project(cp, L, slot + S.wq, slot + S.wk, ws, scomp)) != VEDA_OK) break;
        if ((st = do_score_topk(cp, L, iv, ir, ws, scomp, status)) != VEDA_OK) break;
        if ((st = do_attn(cp, L, iv, ir, slot + S.out, lse ? reinterpret_cast<float*>(slot + S.lse) : nullptr, ws,
                          scomp, status)) != VEDA_OK)
            break;
        k_ok = cudaEventRecord(e_comp[sl], scomp) == cudaSuccess &&
               cudaStreamWaitEvent(sout, e_comp[sl], 0) == cudaSuccess;
        // ---- copy out: output rows, LSE rows and kept tiles of the group's heads ----
        // the group's output is packed for its own g heads
        if (k_ok) k_ok = cudaMemcpy2DAsync(static_cast<char*>(out) + (size_t)h0 * P.d * es, hrow, slot + S.out, row,
                                           row, (size_t)P.B * P.video.n_tokens, cudaMemcpyDeviceToHost,
                                           sout) == cudaSuccess;
        if (k_ok && lse) {
            const size_t w4 = sizeof(float) * (size_t)g * P.video.n_tokens;
            k_ok = cudaMemcpy2DAsync(lse + (size_t)h0 * P.video.n_tokens, sizeof(float) * (size_t)P.H * P.video.n_tokens,
                                     slot + S.lse, sizeof(float) * (size_t)g * P.video.n_tokens, w4, (size_t)P.B,
                                     cudaMemcpyDeviceToHost, sout) == cudaSuccess;
        }
        if (k_ok && idx_video) {
            const size_t wv = sizeof(int32_t) * (size_t)g * nq * P.video.budget;
            k_ok = cudaMemcpy2DAsync(idx_video + (size_t)h0 * nq * P.video.budget,
                                     sizeof(int32_t) * (size_t)P.H * nq * P.video.budget, iv, wv, wv, (size_t)P.B,
                                     cudaMemcpyDeviceToHost, sout) == cudaSuccess;
            if (k_ok && ir) {
                const size_t wr = sizeof(int32_t) * (size_t)g * nq * P.ref.budget;
                k_ok = cudaMemcpy2DAsync(idx_ref + (size_t)h0 * nq * P.ref.budget,
                                         sizeof(int32_t) * (size_t)P.H * nq * P.ref.budget, ir, wr, wr, (size_t)P.B,
                                         cudaMemcpyDeviceToHost, sout) == cudaSuccess;
            }
        }
        if (k_ok) k_ok = cudaEventRecord(e_free[sl], sout) == cudaSuccess;
        if (!k_ok) st = VEDA_ERR_CUDA;
    }
    // join: the caller's stream waits for every copy and kernel of this call
    // (the join is enqueued on every path, so no stream is left forked)
    cudaEventRecord(e_comp_end, scomp);
    cudaEventRecord(e_out_end, sout);
    cudaStreamWaitEvent(caller, e_comp_end, 0);
    cudaStreamWaitEvent(caller, e_out_end, 0);
    cudaEventRecord(e_fork, sin);               // the copy-in stream's last work
    cudaStreamWaitEvent(caller, e_fork, 0);
    return st;
}

veda_status veda_attn(const veda_problem* p, const void* w_q, const void* w_k, int32_t* idx_video,
                      int32_t* idx_ref, void* out, float* lse, void* ws, size_t ws_bytes, veda_stream_t stream)
{
    veda_status st = validate(p);
    if (st != VEDA_OK) return st;
    Layout L;
    if ((st = check_ws(*p, ws, ws_bytes, &L)) != VEDA_OK) return st;
    if (!idx_video || (L.nr > 0) != (idx_ref != nullptr)) return VEDA_ERR_INVALID_ARG;
    if (!out || !aligned16(out) || (lse && ((uintptr_t)lse & 3u))) return VEDA_ERR_INVALID_ARG;
    if (!w_q || !w_k || !aligned16(w_q) || !aligned16(w_k)) return VEDA_ERR_INVALID_ARG;
    cudaStream_t s = (cudaStream_t)stream;
    if ((st = do_pool_project(*p, L, w_q, w_k, ws, s)) != VEDA_OK) return st;
    if ((st = do_score_topk(*p, L, idx_video, idx_ref, ws, s)) != VEDA_OK) return st;
    return do_attn(*p, L, idx_video, idx_ref, out, lse, ws, s);
}

veda_status veda_workspace_view(const veda_problem* p, void* ws, size_t ws_bytes, int which, const void** ptr,
                                int64_t* ld)
{
    veda_status st = validate(p);
    if (st != VEDA_OK) return st;
    if (!ptr || !ld) return VEDA_ERR_INVALID_ARG;
    Layout L;
    if ((st = check_ws(*p, ws, ws_bytes, &L)) != VEDA_OK) return st;
    const size_t offs[7] = {L.qhat, L.khat, L.khat_r, L.sc_v, L.sc_r, L.fb_v, L.fb_r};
    const int64_t lds[7] = {p->r, p->r, p->r, L.ld_v, L.ld_r, 1, 1};
    if (which < 0 || which > 6) return VEDA_ERR_INVALID_ARG;
    if ((which == 2 || which == 4 || which == 6) && L.nr == 0) return VEDA_ERR_INVALID_ARG;
    *ptr = static_cast<const char*>(ws) + offs[which];
    *ld = lds[which];
    return VEDA_OK;
}

veda_status veda_check_status(void* ws, veda_stream_t stream)
{
    if (!ws || ((uintptr_t)ws % kAlign) != 0) return VEDA_ERR_WORKSPACE;
    cudaStream_t s = (cudaStream_t)stream;
    uint32_t code = 0;
    if (cudaMemcpyAsync(&code, ws, sizeof code, cudaMemcpyDeviceToHost, s) != cudaSuccess) return VEDA_ERR_CUDA;
    if (cudaMemsetAsync(ws, 0, sizeof code, s) != cudaSuccess) return VEDA_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return VEDA_ERR_CUDA;
    return code == 0 ? VEDA_OK : (veda_status)(-(int)code);
}

const char* veda_status_string(veda_status s)
{
    switch (s) {
    case VEDA_OK: return "VEDA_OK";
    case VEDA_ERR_INVALID_ARG: return "VEDA_ERR_INVALID_ARG";
    case VEDA_ERR_UNSUPPORTED: return "VEDA_ERR_UNSUPPORTED";
    case VEDA_ERR_WORKSPACE: return "VEDA_ERR_WORKSPACE";
    case VEDA_ERR_CUDA: return "VEDA_ERR_CUDA";
    case VEDA_ERR_TIMEOUT: return "VEDA_ERR_TIMEOUT";
    case VEDA_ERR_BAD_INDEX: return "VEDA_ERR_BAD_INDEX";
    case VEDA_ERR_FORMAT: return "VEDA_ERR_FORMAT";
    case VEDA_ERR_IO: return "VEDA_ERR_IO";
    }
    return "VEDA_ERR_UNKNOWN";
}

}  // extern "C"
