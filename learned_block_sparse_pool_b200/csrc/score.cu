// Tile scoring: s[b,h,i,j] = qhat[b,h,i,:] . khat[b,h,j,:] in fp32.
//
// Every key tile is scored for every (query tile, head) (tao.media, "Affine
// launches MiniMax-H3 video studio...", section "Training the Selector, Not
// the Generator": the predictor selects blocks for the sparse kernel).  The
// score is the raw dot product of the projected pooled vectors; a positive
// scale would not change the ranking.
//
// A small SIMT fp32 contraction (r <= 128): 128 x 128 output tiles per CTA,
// 8 x 8 register blocking per thread, operands staged transposed in shared
// memory.  fp32 FMA (not TF32) keeps the ranking within ~1e-6 relative of
// the exact scores.  Output rows use a padded stride `ld` (multiple of 32
// floats) so every row starts 128-byte aligned for the top-k pass.
#include "veda_internal.cuh"

namespace veda {
namespace {

constexpr int BM = 128, BN = 128, BK = 32, kThreads = 256, PAD = 4;

__global__ void __launch_bounds__(kThreads) score_kernel(const ScoreParams P)
{
    __shared__ __align__(16) float As[BK][BM + PAD];
    __shared__ __align__(16) float Bs[BK][BN + PAD];

    const int bh = blockIdx.z;
    const int i0 = blockIdx.y * BM;
    const int j0 = blockIdx.x * BN;
    const int tid = threadIdx.x;
    const int ty = tid / 16, tx = tid % 16;
    const float* qa = P.qhat + (int64_t)bh * P.nq * P.r;
    const float* kb = P.khat + (int64_t)bh * P.nk * P.r;

    float acc[8][8];
#pragma unroll
    for (int a = 0; a < 8; ++a)
#pragma unroll
        for (int c = 0; c < 8; ++c) acc[a][c] = 0.f;

    for (int c0 = 0; c0 < P.r; c0 += BK) {
        // stage a BM x BK slab of qhat and khat, transposed ([c][row])
#pragma unroll
        for (int u = 0; u < (BM * BK / 4) / kThreads; ++u) {
            const int lin = tid + u * kThreads;
            const int row = lin / (BK / 4);
            const int c4 = (lin % (BK / 4)) * 4;
            float4 va = make_float4(0.f, 0.f, 0.f, 0.f), vb = va;
            if (i0 + row < P.nq && c0 + c4 < P.r)
                va = *reinterpret_cast<const float4*>(qa + (int64_t)(i0 + row) * P.r + c0 + c4);
            if (j0 + row < P.nk && c0 + c4 < P.r)
                vb = *reinterpret_cast<const float4*>(kb + (int64_t)(j0 + row) * P.r + c0 + c4);
            As[c4 + 0][row] = va.x; As[c4 + 1][row] = va.y; As[c4 + 2][row] = va.z; As[c4 + 3][row] = va.w;
            Bs[c4 + 0][row] = vb.x; Bs[c4 + 1][row] = vb.y; Bs[c4 + 2][row] = vb.z; Bs[c4 + 3][row] = vb.w;
        }
        __syncthreads();
        const int kmax = min(BK, P.r - c0);
        for (int c = 0; c < kmax; ++c) {
            const float4 a0 = *reinterpret_cast<const float4*>(&As[c][ty * 4]);
            const float4 a1 = *reinterpret_cast<const float4*>(&As[c][64 + ty * 4]);
            const float4 b0 = *reinterpret_cast<const float4*>(&Bs[c][tx * 4]);
            const float4 b1 = *reinterpret_cast<const float4*>(&Bs[c][64 + tx * 4]);
            const float av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
            const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
            for (int a = 0; a < 8; ++a)
#pragma unroll
                for (int q = 0; q < 8; ++q) acc[a][q] = fmaf(av[a], bv[q], acc[a][q]);
        }
        __syncthreads();
    }

    float* out = P.scores + (int64_t)bh * P.nq * P.ld;
#pragma unroll
    for (int a = 0; a < 8; ++a) {
        const int i = i0 + (a < 4 ? ty * 4 + a : 64 + ty * 4 + (a - 4));
        if (i >= P.nq) continue;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            const int j = j0 + half * 64 + tx * 4;
            float* dst = out + (int64_t)i * P.ld + j;
            const float* v = &acc[a][half * 4];
            if (j + 3 < P.nk) {
                *reinterpret_cast<float4*>(dst) = make_float4(v[0], v[1], v[2], v[3]);
            } else {
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    if (j + q < P.nk) dst[q] = v[q];
            }
        }
    }
}

}  // namespace

cudaError_t launch_score(const ScoreParams& p, cudaStream_t s)
{
    if (p.BH == 0 || p.nq == 0 || p.nk == 0) return cudaSuccess;
    dim3 grid((p.nk + BN - 1) / BN, (p.nq + BM - 1) / BM, p.BH);
    score_kernel<<<grid, kThreads, 0, s>>>(p);
    return cudaGetLastError();
}

}  // namespace veda
