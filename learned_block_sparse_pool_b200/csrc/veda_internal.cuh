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

// ---- fixed-budget top-k -------------------------------------------------
struct TopkParams {
    const float* scores;    // [rows, ld]
    int64_t ld;
    int64_t rows;
    int32_t n;              // key tiles per row
    int32_t k;              // budget
    int32_t* idx;           // [rows, k]
    uint32_t* status;
};

cudaError_t launch_topk(const TopkParams& p, cudaStream_t s);

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
