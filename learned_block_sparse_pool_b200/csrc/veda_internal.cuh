// Internal declarations of libveda (not part of the ABI).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "veda.h"

namespace veda {

// Device-side status codes are stored as the positive value of the
// veda_status they map to (0 = no error); the first error sticks.
__device__ __forceinline__ void record_status(uint32_t* status, veda_status s)
{
    if (status) atomicCAS(status, 0u, (uint32_t)(-(int)s));
}

struct Segment {            // one key/value segment as device code sees it
    const void* k;
    const void* v;
    int64_t n;              // tokens
    int64_t sb, st, sh;     // element strides
    int32_t n_tiles;
    int32_t pad;
};

// ---- tile pooling + selector projection --------------------------------
struct PoolJob {
    const void* x;          // [B, n, H, d]
    int64_t sb, st, sh;
    int64_t n_tokens;
    int64_t first_item;     // items before this job (item = (b, h, tile))
    const void* w;          // [H, d, r]
    float* out;             // [B, H, n_tiles, r]
    int32_t n_tiles;
    int32_t pad;
    // optional (nullptr: none): the projections again as three bf16 planes
    // [3][B H][n_tiles][64] whose sum is the fp32 value (x = p0 + p1 + p2,
    // p0 = bf16(x), p1 = bf16(x - p0), p2 = bf16(x - p0 - p1)), columns
    // r..63 zero: the operands of the tensor-core tile scoring
    uint16_t* planes;
    int64_t plane_stride;   // elements from one plane to the next
    // optional (nullptr: none): the planes of the kSample tiles the fused
    // selection samples, [3][B H][64][64]: sample m is tile (m n_tiles) / 64
    uint16_t* sample_planes;
    int64_t sample_plane_stride;
};

struct PoolParams {
    PoolJob job[3];
    int32_t n_jobs;
    int32_t B, H, d, T, r;
    int32_t dtype;
    int64_t total_items;
};

cudaError_t launch_pool_project(const PoolParams& p, cudaStream_t s);

// ---- tile scores ----------------------------------------------------------
struct ScoreParams {
    const float* qhat;      // [BH, nq, r]
    const float* khat;      // [BH, nk, r]
    float* scores;          // [BH, nq, ld]
    int32_t BH, nq, nk, r;
    int64_t ld;
};

cudaError_t launch_score(const ScoreParams& p, cudaStream_t s);

// ---- fused tile scoring + top-k on the tensor cores -----------------------
// Scores s[i][j] = qhat_i . khat_j are computed on the tensor cores from the
// bf16 planes written by the pool + project kernel (six plane products: fp32
// accuracy) and never stored; every row's top-k is selected on chip (see
// select_rows.cuh).  Rows whose selection needs the exact fallback get their
// scores written to `sc` and their row id appended to `fb` (fb[0] = count);
// launch_topk_rows then finishes them.
struct SelectJob {
    const uint16_t* k_planes;   // [3][BH][nk][64]
    const uint16_t* k_sample;   // [3][BH][64][64]: the planes of the sampled tiles
    int32_t nk;                 // key tiles
    int32_t k;                  // budget
    int32_t* idx;               // [BH][nq][k]
    float* sc;                  // [BH][nq][ld] fallback scores
    int64_t ld;
    int32_t* fb;                // [1 + BH nq]
};

struct SelectParams {
    const uint16_t* q_planes;   // [3][BH][nq][64]
    SelectJob job[2];
    int32_t n_jobs;
    int32_t BH, nq;
    uint32_t* status;
    int32_t short_waits;
    // 1: only compute the scores (exact, the six plane products) and write
    // them to each job's `sc`; the caller then runs the top-k kernel
    int32_t scores_only;
};

bool select_tc_supported(int r, int n_tiles_max);
cudaError_t launch_select_tc(const SelectParams& p, cudaStream_t s);

// ---- fixed-budget top-k -------------------------------------------------
struct TopkParams {
    const float* scores;    // [rows, ld]
    int64_t ld;
    int64_t rows;
    int32_t n;              // key tiles per row
    int32_t k;              // budget
    int32_t* idx;           // [rows, k]
    uint32_t* status;
    // optional: process only the rows listed in row_list[0 .. *row_count)
    const int32_t* row_list;
    const int32_t* row_count;
};

cudaError_t launch_topk(const TopkParams& p, cudaStream_t s);
int topk_max_tiles();

// ---- attention ----------------------------------------------------------
struct AttnParams {
    const void* q;
    int64_t qsb, qst, qsh;
    int64_t n_qtok;         // query tokens (the video's own, or dense-query rows)
    Segment video, ref, dense;
    const int32_t* idx_v;   // [B, H, nq, k_v]; null: every video tile, in order (k_v = tiles)
    const int32_t* idx_r;   // [B, H, nq, k_r]; null: every reference tile (or no reference)
    int32_t k_v, k_r;
    void* out;              // [B, n_qtok, H, d]
    float* lse;             // [B, H, n_qtok] or null
    int32_t B, H, d, T, nq;
    int32_t dtype;
    float scale;            // softmax scale (natural-log units)
    uint32_t* status;
    int32_t short_waits;    // test hook: bounded waits give up after ~64 clocks
    // tensor-core path only: split each (b, h, query tile) key list into n_split
    // ranges on different CTAs, merged afterwards (scratch: part_o
    // [n_split][B H][n_qtok][d] fp32, part_ml [n_split][B H][n_qtok][2] fp32)
    int32_t n_split;
    float* part_o;
    float* part_ml;
};

cudaError_t launch_attn_simt(const AttnParams& p, cudaStream_t s);

int num_sms();

// The current device and a process-unique id of its current CUDA context
// (the device's primary context is made current first).  Host-side caches of
// per-context objects (a symbol's device address, streams, events) are keyed
// by this id, so a context that is destroyed and created again (for example
// by cudaDeviceReset) gets fresh objects.
cudaError_t current_context(int* device, unsigned long long* ctx_id);

}  // namespace veda
