// fwd_simt.cu - alpha-entmax attention forward on the FP32 FMA pipes (the fp32 path).
//
// One CTA of 128 threads per (b, h, 128-row query tile); the thread that owns a query row computes its
// scores against key blocks staged in shared memory, keeps the row's histogram ring and solver state,
// and accumulates O = P V and U V in shared memory for the support entries only.
//
// Sweeps over the key blocks of a tile (AdaSplash-2, gist.science (de), section 2):
//   1. dense: running max, left-edge histogram, candidate key blocks (some entry above max - 1);
//   2. refine: solver sums at the current tau over candidate blocks; one hybrid-solver update per row,
//      repeated while a row's last update was larger than one bin width;
//   3. P V: p = [z - tau]_+^k, O, U V, sum u and the exact block mask at the current tau, with the
//      sums doubling as a check of sum p = 1; repeated while any row's tau still moved.
#include <cuda_runtime.h>
#include <math.h>

#include "common.cuh"
#include "fwd_common.cuh"
#include "launch.h"

namespace eattn {
namespace {

constexpr int kKeyBlk = 64;  // keys staged per step (>= the mask block)

template <typename T>
__device__ __forceinline__ float to_f(T v);
template <>
__device__ __forceinline__ float to_f<float>(float v) { return v; }
template <>
__device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 v) { return __bfloat162float(v); }

template <typename T>
__device__ __forceinline__ T from_f(float v);
template <>
__device__ __forceinline__ float from_f<float>(float v) { return v; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float v) { return __float2bfloat16_rn(v); }

// Stage keys [k0, k0 + mb) of one head into dst[mb][D] as float (zeros past n).
template <typename T, int D>
__device__ __forceinline__ void stage(float* dst, const T* src, int k0, int mb, int n) {
    for (int i = threadIdx.x; i < mb * D; i += blockDim.x) {
        const int r = i / D;
        const int key = k0 + r;
        dst[i] = key < n ? to_f<T>(src[(size_t)key * D + (i % D)]) : 0.0f;
    }
}

template <int D>
__device__ __forceinline__ float dot_row(const float* q, const float* k) {
    float acc = 0.0f;
#pragma unroll
    for (int c = 0; c < D; ++c) acc = fmaf(q[c], k[c], acc);
    return acc;
}

template <typename T, int D, int KIND>
__global__ void __launch_bounds__(128, 1) fwd_simt_kernel(const FwdArgs a) {
    extern __shared__ __align__(16) unsigned char smem[];
    const SolveParams sp = a.sp;
    const int mb = a.mb;
    const int B = sp.bins;
    const int cwords = (a.nkb + 31) / 32;
    const int mrows = kTileRows / mb;

    float* sK = reinterpret_cast<float*>(smem);                   // [64][D]
    float* sV = sK + kKeyBlk * D;                                  // [64][D]
    float* uni = sV + kKeyBlk * D;                                 // union: hist | O, U V accumulators
    uint16_t* hist = reinterpret_cast<uint16_t*>(uni);             // [B][128] u16
    float* stash = uni + 256 * kTileRows / 2;                      // [kStashCap][128]
    float* sO = uni;                                               // [D][128]
    float* sOb = uni + D * kTileRows;                              // [D][128]
    const int uni_words = max(256 * kTileRows, 2 * D * kTileRows);
    float* Tk = uni + uni_words;                                   // [B + 1]
    uint32_t* cand = reinterpret_cast<uint32_t*>(Tk + 260);        // [cwords]
    uint32_t* next = cand + cwords;                                // [cwords]
    uint32_t* mrow = next + cwords;                                // [mrows][nw]
    uint32_t* live_all = mrow + mrows * a.nw;                      // [128][kLiveStride]
    __shared__ TileStats st;

    const int tid = threadIdx.x;
    const int qt = a.ntiles - 1 - (int)blockIdx.y;  // grid (B*H, tiles): longest tiles of every head first
    const int bh = blockIdx.x;
    const int row = qt * kTileRows + tid;
    const bool valid = row < a.n;
    const int n_i = valid ? allowed_keys(row, a.n, a.causal) : 1;
    const int kend = a.causal ? min(a.n, qt * kTileRows + kTileRows) : a.n;
    const int nblk = (kend + mb - 1) / mb;
    const size_t head = (size_t)bh * a.n;
    const T* Qh = static_cast<const T*>(a.Q) + head * D;
    const T* Kh = static_cast<const T*>(a.K) + head * D;
    const T* Vh = static_cast<const T*>(a.V) + head * D;

    float q[D];
#pragma unroll
    for (int c = 0; c < D; ++c) q[c] = valid ? to_f<T>(Qh[(size_t)row * D + c]) : 0.0f;

    for (int i = tid; i <= B; i += blockDim.x) Tk[i] = (KIND == kGeneric) ? powf((float)i, sp.k) : 0.0f;
    for (int i = tid; i < cwords; i += blockDim.x) cand[i] = next[i] = 0u;
    if (tid == 0) {
        st = TileStats{};
    }
    __syncthreads();

    auto key_ok = [&](int key) { return valid && key < a.n && (!a.causal || key <= row); };

    // ---- sweep 1: dense scores, running max, histogram, candidate blocks ----
    HistRow h;
    hist_init(h, live_all, tid);
    Stash sh;
    sh.n = 0;
    sh.overflow = false;
    for (int J = 0; J < nblk; ++J) {
        __syncthreads();
        stage<T, D>(sK, Kh, J * mb, mb, a.n);
        __syncthreads();
        float sc[kKeyBlk];
        float amax = -INFINITY;
        for (int jj = 0; jj < mb; ++jj) {
            const int key = J * mb + jj;
            const float s = key_ok(key) ? dot_row<D>(q, sK + jj * D) : -INFINITY;
            sc[jj] = s;
            amax = fmaxf(amax, s);
        }
        bool any = false;
        if (sp.init_mode == 0) {
            hist_raise(h, amax, sp.cbin, sp.inv_cz, sp.bins);
        } else if (amax > h.m_raw) {
            h.m_raw = amax;
            h.thr_raw = amax - sp.inv_cz;
            h.any = true;
        }
        for (int jj = 0; jj < mb; ++jj)
            if (sc[jj] > h.thr_raw) {
                any = true;
                if (sp.init_mode == 0) hist_add(h, sc[jj], sp.cbin, sp.bins, hist, tid);
                stash_add(sh, sc[jj], h.thr_raw, stash, tid);
            }
        if (any) atomicOr(&cand[J >> 5], 1u << (J & 31));
    }

    const float m = sp.cz * h.m_raw;
    float tau_h = m - 1.0f;
    if (valid && sp.init_mode == 0) tau_h = hist_tau<KIND>(h, sp, hist, tid, Tk);
    RowSolve s;
    solve_init(s, tau_h, m, n_i, sp);
    if (!valid) s.done = true;
    if (valid && a.tau_hist) a.tau_hist[head + row] = tau_h;
    int sweeps = 1;
    // rows whose candidates all fit the stash are solved on chip, with no further key sweep
    if (valid && !sh.overflow) {
        for (int it = 0; it < kMaxSweeps && !s.done; ++it) {
            float F0, F1, F2, F0b;
            stash_sums<KIND>(sh, stash, tid, sp.cz, sp.k, s.tau, s.tau2, s.need_two, F0, F1, F2, F0b);
            solve_step(s, F0, F1, F2, F0b, sp);
        }
    }

    // ---- refinement sweep: solver sums only ----
    float last_step = INFINITY;
    int refine = 0, pv = 0;
    auto refine_sweep = [&]() {
        for (int i = tid; i < cwords; i += blockDim.x) next[i] = 0u;
        __syncthreads();
        float F0 = 0.f, F1 = 0.f, F2 = 0.f, F0b = 0.f;
        const float t = s.tau, t2 = s.tau2, lo0 = s.lo;
        const bool two = s.need_two;
        for (int wd = 0; wd < cwords; ++wd) {
            uint32_t bits = cand[wd];
            while (bits) {
                const int J = wd * 32 + __ffs(bits) - 1;
                bits &= bits - 1;
                __syncthreads();
                stage<T, D>(sK, Kh, J * mb, mb, a.n);
                __syncthreads();
                bool keep = false;
                for (int jj = 0; jj < mb; ++jj) {
                    const int key = J * mb + jj;
                    if (!key_ok(key)) continue;
                    const float z = sp.cz * dot_row<D>(q, sK + jj * D);
                    keep |= z > lo0;
                    const float x = z - t;
                    if (x > 0.f) add_sums<KIND>(x, sp.k, F0, F1, F2);
                    if (two) {
                        const float x2 = z - t2;
                        if (x2 > 0.f) F0b += pow_k<KIND>(x2, sp.k);
                    }
                }
                if (keep) atomicOr(&next[J >> 5], 1u << (J & 31));
            }
        }
        const float before = s.tau;
        solve_step(s, F0, F1, F2, F0b, sp);
        last_step = s.tau - before;
        ++refine;
        ++sweeps;
        __syncthreads();
        for (int i = tid; i < cwords; i += blockDim.x) cand[i] = next[i];
    };

    // ---- P V sweep: O, U V, sum u, exact mask; the sums double as the check of sum p = 1 ----
    float Su = 0.f;
    uint32_t nsup = 0;  // nonzero probabilities of this row in the last P V sweep
    auto pv_sweep = [&]() -> bool {
        __syncthreads();
        for (int i = tid; i < cwords; i += blockDim.x) next[i] = 0u;
        for (int i = tid; i < mrows * a.nw; i += blockDim.x) mrow[i] = 0u;
        for (int c = 0; c < D; ++c) sO[c * kTileRows + tid] = sOb[c * kTileRows + tid] = 0.f;
        __syncthreads();
        float Sp = 0.f, F2 = 0.f;
        Su = 0.f;
        nsup = 0;
        const float t = s.tau, lo0 = s.lo;
        for (int wd = 0; wd < cwords; ++wd) {
            uint32_t bits = cand[wd];
            while (bits) {
                const int J = wd * 32 + __ffs(bits) - 1;
                bits &= bits - 1;
                __syncthreads();
                stage<T, D>(sK, Kh, J * mb, mb, a.n);
                stage<T, D>(sV, Vh, J * mb, mb, a.n);
                __syncthreads();
                bool keep = false, nz = false;
                for (int jj = 0; jj < mb; ++jj) {
                    const int key = J * mb + jj;
                    if (!key_ok(key)) continue;
                    const float z = sp.cz * dot_row<D>(q, sK + jj * D);
                    keep |= z > lo0;
                    const float x = z - t;
                    if (x > 0.f) {
                        float u, p;
                        if constexpr (KIND == kAlpha15) { u = x; p = x * x; F2 += 1.f; }
                        else if constexpr (KIND == kAlpha2) { u = 1.f; p = x; }
                        else { u = exp2f((sp.k - 1.f) * __log2f(x)); p = u * x; F2 += __fdividef(u, x); }
                        Sp += p;
                        Su += u;
                        ++nsup;
                        nz = true;
                        const float* v = sV + jj * D;
                        for (int c = 0; c < D; ++c) {
                            sO[c * kTileRows + tid] = fmaf(p, v[c], sO[c * kTileRows + tid]);
                            sOb[c * kTileRows + tid] = fmaf(u, v[c], sOb[c * kTileRows + tid]);
                        }
                    }
                }
                if (keep) atomicOr(&next[J >> 5], 1u << (J & 31));
                if (nz) atomicOr(&mrow[(tid / mb) * a.nw + (J >> 5)], 1u << (J & 31));
            }
        }
        ++sweeps;
        ++pv;
        const float before = s.tau;
        solve_step(s, Sp, Su, F2, 0.f, sp);
        const bool changed = s.tau != before;
        __syncthreads();
        for (int i = tid; i < cwords; i += blockDim.x) cand[i] = next[i];
        return __syncthreads_or(changed) != 0;
    };

    // refine while a row still takes steps wider than one bin; P V (also the check of sum p = 1);
    // if a tau moved, refine until every row stopped and finish with one more P V sweep
    if (__syncthreads_or(!s.done)) {
        do {
            refine_sweep();
        } while (refine < kMaxSweeps && __syncthreads_or(!s.done && fabsf(last_step) > sp.w));
    }
    while (true) {
        const bool changed = pv_sweep();
        if (!changed || pv >= 3) break;
        while (refine < kMaxSweeps && __syncthreads_or(!s.done)) refine_sweep();
    }

    // ---- outputs ----
    if (valid) {
        T* Oh = static_cast<T*>(a.O) + head * D;
        float* Obh = a.obar + head * D;
        for (int c = 0; c < D; ++c) {
            Oh[(size_t)row * D + c] = from_f<T>(sO[c * kTileRows + tid]);
            Obh[(size_t)row * D + c] = sOb[c * kTileRows + tid];
        }
        a.tau[head + row] = s.tau;
        a.sum_u[head + row] = Su;
        if (a.steps) a.steps[head + row] = (uint8_t)s.steps;
        if (sh.overflow) atomicAdd(&st.overflow_rows, 1u);
        atomicAdd(&st.rows, 1u);
        atomicAdd(&st.support, nsup);
        atomicAdd(&st.steps, (uint32_t)s.steps);
        atomicAdd(&st.fallbacks, (uint32_t)s.fallbacks);
        atomicAdd(&st.step_hist[min(s.steps, kMaxSteps)], 1u);
    }
    __syncthreads();
    const int qb0 = qt * mrows;
    for (int i = tid; i < mrows * a.nw; i += blockDim.x) {
        const int rr = i / a.nw;
        if (qb0 + rr < a.nqb) a.mask[((size_t)bh * a.nqb + qb0 + rr) * a.nw + (i % a.nw)] = mrow[i];
    }
    if (a.stats) {
        for (int i = tid; i < mrows * a.nw; i += blockDim.x) atomicAdd(&st.nonzero_blocks, (uint32_t)__popc(mrow[i]));
        for (int i = tid; i < cwords; i += blockDim.x) atomicAdd(&st.candidate_blocks, (uint32_t)__popc(cand[i]));
        __syncthreads();
        if (tid == 0) {
            st.sweeps = (uint32_t)sweeps;
            st.causal_blocks = tile_causal_blocks(qb0, mrows, a.nqb, a.nkb, a.causal);
            flush_stats(a.stats, st);
        }
    }
}

template <typename T, int D, int KIND>
cudaError_t launch_t(const FwdArgs& a, cudaStream_t stream) {
    const int cwords = (a.nkb + 31) / 32;
    const int mrows = kTileRows / a.mb;
    const size_t uni_words = (size_t)max(256 * kTileRows, 2 * D * kTileRows);
    const size_t bytes = (size_t)2 * kKeyBlk * D * 4 + uni_words * 4 + 260 * 4 +
                         (size_t)(2 * cwords + mrows * a.nw) * 4 + (size_t)kTileRows * kLiveStride * 4;
    auto kern = fwd_simt_kernel<T, D, KIND>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (e != cudaSuccess) return e;
    dim3 grid(a.B * a.H, a.ntiles);
    launch_mark(stream);
    kern<<<grid, 128, bytes, stream>>>(a);
    return cudaGetLastError();
}

template <typename T, int D>
cudaError_t launch_d(const FwdArgs& a, cudaStream_t stream) {
    if (a.sp.alpha == 1.5f) return launch_t<T, D, kAlpha15>(a, stream);
    if (a.sp.alpha == 2.0f) return launch_t<T, D, kAlpha2>(a, stream);
    return launch_t<T, D, kGeneric>(a, stream);
}

}  // namespace

// Shared-memory bytes the SIMT forward needs (host-side check before launch).
size_t fwd_simt_smem_bytes(int d, int nkb, int mb, int nw) {
    const int cwords = (nkb + 31) / 32;
    const size_t uni_words = (size_t)max(256 * kTileRows, 2 * d * kTileRows);
    return (size_t)2 * kKeyBlk * d * 4 + uni_words * 4 + 260 * 4 + (size_t)(2 * cwords + (kTileRows / mb) * nw) * 4;
}

cudaError_t launch_fwd_simt(const FwdArgs& a, bool fp32, cudaStream_t stream) {
    if (fp32) {
        if (a.d == 64) return launch_d<float, 64>(a, stream);
        return launch_d<float, 128>(a, stream);
    }
    if (a.d == 64) return launch_d<__nv_bfloat16, 64>(a, stream);
    return launch_d<__nv_bfloat16, 128>(a, stream);
}

}  // namespace eattn
