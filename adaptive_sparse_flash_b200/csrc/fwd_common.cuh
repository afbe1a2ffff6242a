// fwd_common.cuh - argument block and sweep schedule shared by the two forward kernels.
#pragma once

#include <stdint.h>

#include "entmax_attn.h"
#include "entmax_row.cuh"

namespace eattn {

struct FwdArgs {
    const void* Q;
    const void* K;
    const void* V;
    void* O;
    float* tau;
    uint32_t* mask;    // [B,H,nqb,nw]
    float* obar;       // workspace: U V, fp32 [B,H,n,d]
    float* sum_u;      // workspace: fp32 [B,H,n]
    float* tau_hist;   // optional
    uint8_t* steps;    // optional
    entmax_stats* stats;
    int* status;
    int B, H, n, d;
    int nqb, nkb, nw;  // mask query blocks, key blocks (of mb), words per mask row
    int mb;            // mask block
    int causal;
    int ntiles;        // 128-row query tiles per head
    SolveParams sp;
    // fp16 path (alpha <= 2, d = 64): fp16 copies of Q, K, V and their range exponents (f16.cu)
    const void* Qh;
    const void* Kh;
    const void* Vh;
    const uint32_t* maxbits;  // [3]: Q, K, V
};

enum SweepKind : int { kSweepDense = 0, kSweepRefine = 1, kSweepPV = 2, kSweepDone = 3, kSweepHist = 4, kSweepSupport = 5 };

// Number of allowed keys of query row `row`.
__device__ __forceinline__ int allowed_keys(int row, int n, int causal) {
    return causal ? min(row + 1, n) : n;
}

// Mask blocks (query block, key block) with at least one allowed entry, over query blocks qb0 .. qb0 + nq - 1
// of a tile (causal: key blocks 0 .. qb, since query and key blocks have the same size).
__device__ __forceinline__ uint32_t tile_causal_blocks(int qb0, int nq, int nqb, int nkb, int causal) {
    uint32_t c = 0;
    for (int qb = qb0; qb < qb0 + nq && qb < nqb; ++qb) c += (uint32_t)(causal ? min(qb + 1, nkb) : nkb);
    return c;
}

// Per-CTA statistics, reduced into entmax_stats at the end of a tile.
struct TileStats {
    uint32_t rows, steps, fallbacks, candidate_blocks, nonzero_blocks, causal_blocks, sweeps, overflow_rows;
    uint32_t support;  // nonzero probabilities of the tile's rows
    uint32_t step_hist[kMaxSteps + 1];
};

__device__ __forceinline__ void flush_stats(entmax_stats* g, const TileStats& t) {
    if (!g) return;
    atomicAdd(&g->rows, (unsigned long long)t.rows);
    atomicAdd(&g->steps, (unsigned long long)t.steps);
    atomicAdd(&g->fallbacks, (unsigned long long)t.fallbacks);
    atomicAdd(&g->candidate_blocks, (unsigned long long)t.candidate_blocks);
    atomicAdd(&g->nonzero_blocks, (unsigned long long)t.nonzero_blocks);
    atomicAdd(&g->causal_blocks, (unsigned long long)t.causal_blocks);
    atomicAdd(&g->sweeps, (unsigned long long)t.sweeps);
    if (t.overflow_rows) atomicAdd(&g->overflow_rows, (unsigned long long)t.overflow_rows);
    atomicAdd(&g->support, (unsigned long long)t.support);
    for (int i = 0; i <= kMaxSteps; ++i)
        if (t.step_hist[i]) atomicAdd(&g->step_hist[i], (unsigned long long)t.step_hist[i]);
}

}  // namespace eattn
