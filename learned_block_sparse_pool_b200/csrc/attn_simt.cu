// Block-sparse attention on the fp32 SIMT pipe (fp32 problems, and a
// cross-check path for bf16).
//
// Each video query attends to every token of its query tile's kept video
// tiles, kept reference tiles, and every dense (text / VLM / audio) token,
// with one online softmax across the three segments (tao.media, "Affine
// launches MiniMax-H3 video studio...", section "Training the Selector, Not
// the Generator": the predictor picks blocks for a sparse execution kernel;
// veyrul.com, "Veda R2VA for MiniMax-H3", second paragraph: reference and
// video tiles are selected, text / VLM / audio attention stays dense).
// Tokens past a segment's end (a short last tile) are not keys.
//
// One CTA per (b, h, query tile); two threads per query row, each holding
// half of q and of the output accumulator (interleaved 4-element chunks, so
// the two halves read adjacent 16-byte words of the shared K/V tile).
// K and V tiles are staged in shared memory as fp32.  Everything is fp32:
// logits are kept in base-2 units (q pre-scaled by scale * log2 e) and
// exponentials use exp2f.
#include <cuda_bf16.h>

#include "veda_internal.cuh"

namespace veda {
namespace {

__device__ __forceinline__ float4 load4(const float* p) { return *reinterpret_cast<const float4*>(p); }

__device__ __forceinline__ float4 load4(const __nv_bfloat16* p)
{
    const uint2 raw = *reinterpret_cast<const uint2*>(p);
    return make_float4(__uint_as_float(raw.x << 16), __uint_as_float(raw.x & 0xffff0000u),
                       __uint_as_float(raw.y << 16), __uint_as_float(raw.y & 0xffff0000u));
}

__device__ __forceinline__ void store4(float* p, float4 v) { *reinterpret_cast<float4*>(p) = v; }

__device__ __forceinline__ void store4(__nv_bfloat16* p, float4 v)
{
    __nv_bfloat162 a = __floats2bfloat162_rn(v.x, v.y);
    __nv_bfloat162 b = __floats2bfloat162_rn(v.z, v.w);
    uint2 raw;
    raw.x = *reinterpret_cast<uint32_t*>(&a);
    raw.y = *reinterpret_cast<uint32_t*>(&b);
    *reinterpret_cast<uint2*>(p) = raw;
}

template <typename Tin, int D, int TILE>
__global__ void __launch_bounds__(2 * TILE) attn_simt_kernel(const AttnParams P)
{
    constexpr int NC = D / 8;          // 4-element chunks per half row
    constexpr int KC = 16;             // keys per softmax step
    extern __shared__ __align__(16) float sm[];
    float* Ks = sm;                    // [TILE][D]
    float* Vs = sm + TILE * D;         // [TILE][D]

    const int unit = blockIdx.x;
    const int i = unit % P.nq;
    const int bh = unit / P.nq;
    const int h = bh % P.H;
    const int b = bh / P.H;
    const int tid = threadIdx.x;
    const int row = tid >> 1;
    const int half = tid & 1;
    const int64_t t = (int64_t)i * TILE + row;
    const bool valid_q = t < P.n_qtok;
    const float qscale = P.scale * 1.4426950408889634f;   // logits in base-2 units

    float q[4 * NC], o[4 * NC];
    {
        const Tin* qp = static_cast<const Tin*>(P.q) + (int64_t)b * P.qsb + t * P.qst + (int64_t)h * P.qsh;
#pragma unroll
        for (int c = 0; c < NC; ++c) {
            float4 v = valid_q ? load4(qp + 8 * c + 4 * half) : make_float4(0.f, 0.f, 0.f, 0.f);
            q[4 * c + 0] = v.x * qscale;
            q[4 * c + 1] = v.y * qscale;
            q[4 * c + 2] = v.z * qscale;
            q[4 * c + 3] = v.w * qscale;
            o[4 * c + 0] = o[4 * c + 1] = o[4 * c + 2] = o[4 * c + 3] = 0.f;
        }
    }
    float m = -INFINITY, l = 0.f;

    const int64_t idx_row = (int64_t)bh * P.nq + i;
    const int n_list = P.k_v + P.k_r + P.dense.n_tiles;
    for (int jt = 0; jt < n_list; ++jt) {
        const Segment* S;
        int tile;
        if (jt < P.k_v) {
            S = &P.video;
            tile = P.idx_v ? P.idx_v[idx_row * P.k_v + jt] : jt;
        } else if (jt < P.k_v + P.k_r) {
            S = &P.ref;
            tile = P.idx_r ? P.idx_r[idx_row * P.k_r + (jt - P.k_v)] : jt - P.k_v;
        } else {
            S = &P.dense;
            tile = jt - P.k_v - P.k_r;
        }
        if (tile < 0 || tile >= S->n_tiles) {     // uniform over the CTA
            if (tid == 0) record_status(P.status, VEDA_ERR_BAD_INDEX);
            continue;
        }
        const int cnt = (int)min((int64_t)TILE, S->n - (int64_t)tile * TILE);

        __syncthreads();   // everyone is done with the previous tile
        {
            const Tin* kp = static_cast<const Tin*>(S->k) + (int64_t)b * S->sb + (int64_t)h * S->sh;
            const Tin* vp = static_cast<const Tin*>(S->v) + (int64_t)b * S->sb + (int64_t)h * S->sh;
            for (int e = tid; e < cnt * (D / 4); e += 2 * TILE) {
                const int r = e / (D / 4);
                const int c4 = (e % (D / 4)) * 4;
                const int64_t off = ((int64_t)tile * TILE + r) * S->st + c4;
                store4(Ks + r * D + c4, load4(kp + off));
                store4(Vs + r * D + c4, load4(vp + off));
            }
        }
        __syncthreads();

        for (int k0 = 0; k0 < cnt; k0 += KC) {
            float s[KC];
#pragma unroll
            for (int u = 0; u < KC; ++u) {
                const float* kr = Ks + (k0 + u) * D + 4 * half;
                float acc = 0.f;
                if (k0 + u < cnt) {
#pragma unroll
                    for (int c = 0; c < NC; ++c) {
                        const float4 kv = load4(kr + 8 * c);
                        acc = fmaf(q[4 * c + 0], kv.x, acc);
                        acc = fmaf(q[4 * c + 1], kv.y, acc);
                        acc = fmaf(q[4 * c + 2], kv.z, acc);
                        acc = fmaf(q[4 * c + 3], kv.w, acc);
                    }
                }
                s[u] = acc;
            }
            float mx = m;
#pragma unroll
            for (int u = 0; u < KC; ++u) {
                s[u] += __shfl_xor_sync(0xffffffffu, s[u], 1);
                if (k0 + u >= cnt) s[u] = -INFINITY;
                mx = fmaxf(mx, s[u]);
            }
            const float alpha = exp2f(m - mx);    // m = -inf on the first step: alpha = 0
            l *= alpha;
#pragma unroll
            for (int e = 0; e < 4 * NC; ++e) o[e] *= alpha;
#pragma unroll
            for (int u = 0; u < KC; ++u) {
                const float p = exp2f(s[u] - mx);
                l += p;
                if (k0 + u < cnt) {
                    const float* vr = Vs + (k0 + u) * D + 4 * half;
#pragma unroll
                    for (int c = 0; c < NC; ++c) {
                        const float4 vv = load4(vr + 8 * c);
                        o[4 * c + 0] = fmaf(p, vv.x, o[4 * c + 0]);
                        o[4 * c + 1] = fmaf(p, vv.y, o[4 * c + 1]);
                        o[4 * c + 2] = fmaf(p, vv.z, o[4 * c + 2]);
                        o[4 * c + 3] = fmaf(p, vv.w, o[4 * c + 3]);
                    }
                }
            }
            m = mx;
        }
    }

    if (!valid_q) return;
    const float inv = 1.f / l;
    Tin* op = static_cast<Tin*>(P.out) + (((int64_t)b * P.n_qtok + t) * P.H + h) * D;
#pragma unroll
    for (int c = 0; c < NC; ++c)
        store4(op + 8 * c + 4 * half, make_float4(o[4 * c] * inv, o[4 * c + 1] * inv,
                                                  o[4 * c + 2] * inv, o[4 * c + 3] * inv));
    if (P.lse && half == 0)
        P.lse[((int64_t)b * P.H + h) * P.n_qtok + t] = m * 0.6931471805599453f + logf(l);
}

template <typename Tin, int D, int TILE>
cudaError_t launch_typed(const AttnParams& p, cudaStream_t s)
{
    const size_t smem = sizeof(float) * 2 * TILE * D;
    auto kern = attn_simt_kernel<Tin, D, TILE>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int64_t units = (int64_t)p.B * p.H * p.nq;
    kern<<<(unsigned)units, 2 * TILE, smem, s>>>(p);
    return cudaGetLastError();
}

template <typename Tin>
cudaError_t launch_dt(const AttnParams& p, cudaStream_t s)
{
    if (p.d == 64) return p.T == 64 ? launch_typed<Tin, 64, 64>(p, s) : launch_typed<Tin, 64, 128>(p, s);
    return p.T == 64 ? launch_typed<Tin, 128, 64>(p, s) : launch_typed<Tin, 128, 128>(p, s);
}

}  // namespace

cudaError_t launch_attn_simt(const AttnParams& p, cudaStream_t s)
{
    if ((int64_t)p.B * p.H * p.nq == 0) return cudaSuccess;
    return p.dtype == VEDA_BF16 ? launch_dt<__nv_bfloat16>(p, s) : launch_dt<float>(p, s);
}

}  // namespace veda
