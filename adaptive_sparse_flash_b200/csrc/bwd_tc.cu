// bwd_tc.cu - backward of alpha-entmax attention (and of the dense softmax baseline) on the sm_100a
// tensor cores: tcgen05 MMAs with TMEM accumulators, TMA-fed shared-memory operands.
//
// With g = dO V^T, u = [z - tau]_+^(k-1) (= p^(2-alpha) on the support) and
// delta = sum(u g) / sum(u) = (dO . U V) / sum(u), the score gradient is dS = u (g - delta); then
// dQ = scale dS K, dK = scale dS^T Q, dV = P^T dO. The softmax baseline has u = p and delta = dO . O.
// Only the (query block, key block) pairs set in the bit-packed mask are visited, found with
// find-first-set over the mask words ("AdaSplash-2", gist.science (de), section 2, "GPU-Optimierung"
// and "Bit-Packed Block Mask"; the largest gain is in the backward, section 4 "Ergebnisse").
//
// Kernels (all 192 threads: warps 0-3 compute, warp 4 MMA issue, warp 5 TMA issue):
//   bwd_pre    delta per query row (from U V; 0 when the caller passes no U V, as the fp16 backward does,
//              whose dQ kernel forms delta itself), and padded copies of the row statistics for bulk copies;
//   bwd_dkdv   one CTA per 128-key tile: walks the tile's query blocks (transposed mask), recomputes
//              S^T = K Q^T and dP^T = V dO^T into TMEM, forms P^T and dS^T (thread = key row) in
//              shared memory, accumulates dV += P^T dO and dK += dS^T Q in TMEM;
//   bwd_dq     one CTA per 128-row query tile: walks the tile's key blocks (row mask), recomputes
//              S and dP, accumulates dQ += dS K in TMEM (deterministic, no atomics).
// With SPLIT, P and dS enter the gradient MMAs as two bf16 terms (high + low part), which keeps the
// products accurate to ~16 mantissa bits; gradients are written in fp32.
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>

#include "common.cuh"
#include "entmax_row.cuh"
#include "launch.h"

namespace eattn {
namespace {

// K-major operands (128-byte rows, 8-row groups 1024 bytes apart) and MN-major operands stored as
// 64-column boxes of 64 rows (next 64 columns 8 KB further; next 8 rows 1024 bytes further)
constexpr uint64_t kDescK = sdesc_sw128_fields(16, 1024);
constexpr uint64_t kDescMN = sdesc_sw128_fields(64 * 128, 1024);

constexpr int kThreads = 192;
constexpr int TM = 128;  // rows of the tile owned by a CTA
constexpr int TB = 64;   // rows of the blocks it walks
constexpr int kModeSoftmax = 3;
constexpr int NST = 4;   // stages of the operand ring that a CTA walks (Q_I/dO_I or K_J/V_J)

__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

// OR over the 128 compute threads (named barrier 1).
__device__ __forceinline__ bool bar_or128(bool pred) {
    uint32_t out;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 q, %1, 0;\n\t"
        "bar.red.or.pred p, 1, 128, q;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(out)
        : "r"((uint32_t)pred)
        : "memory");
    return out != 0;
}

// p and u for one score: MODE is an AlphaKind for entmax, kModeSoftmax for the baseline.
// entmax: x = cz * s - stat; softmax: p = exp2(s * c2 - stat) with stat = lse * log2(e).
template <int MODE>
__device__ __forceinline__ void pointwise(float s, float stat, float cz, float k, bool ok, float& p, float& u) {
    if constexpr (MODE == kModeSoftmax) {
        p = ok ? exp2f(fmaf(s, cz, -stat)) : 0.f;
        u = p;
    } else {
        const float x = ok ? fmaf(s, cz, -stat) : -1.f;
        if constexpr (MODE == kAlpha15) {
            u = fmaxf(x, 0.f);
            p = u * u;
        } else if constexpr (MODE == kAlpha2) {
            p = fmaxf(x, 0.f);
            u = x > 0.f ? 1.f : 0.f;
        } else {
            const bool pos = x > 0.f;
            const float xs = pos ? x : 1.f;
            const float uu = exp2f((k - 1.f) * __log2f(xs));
            u = pos ? uu : 0.f;
            p = u * xs;
        }
    }
}

// Two values as a bf16 pair (high part) and, with SPLIT, the bf16 pair of the remainders (low part).
template <bool SPLIT>
__device__ __forceinline__ void split2(const float* v, uint32_t& hi, uint32_t& lo) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(v[0], v[1]);
    hi = *reinterpret_cast<const uint32_t*>(&h);
    if constexpr (SPLIT) {
        const float2 hf = __bfloat1622float2(h);
        lo = pack_bf16x2(v[0] - hf.x, v[1] - hf.y);
    } else {
        lo = 0u;
    }
}

// ---------------------------------------------------------------------------------------------
// preprocess: delta and padded row statistics
// ---------------------------------------------------------------------------------------------
// One warp per row: lanes split the d columns. Rows past n get zeros in the padded arrays.
template <int D>
__global__ void bwd_pre_kernel(const BwdArgs a, float* __restrict__ delta_pad, float* __restrict__ stat_pad) {
    const int warps = blockDim.x >> 5;
    const int row = blockIdx.x * warps + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    const int bh = blockIdx.y;
    const int npad = a.nqb * TB;
    if (row >= npad) return;
    float dl = 0.f, st = 0.f;
    if (row < a.n) {
        const size_t base = ((size_t)bh * a.n + row) * D;
        const __nv_bfloat16* dO = static_cast<const __nv_bfloat16*>(a.dO) + base;
        float acc = 0.f;
        if (a.softmax) {
            const __nv_bfloat16* O = static_cast<const __nv_bfloat16*>(a.O) + base;
            for (int c = lane; c < D; c += 32) acc = fmaf(__bfloat162float(dO[c]), __bfloat162float(O[c]), acc);
        } else if (a.obar) {
            // the bf16 family's delta from U V; the fp16 backward forms delta in its dQ kernel (obar NULL)
            const float* Ob = a.obar + base;
            for (int c = lane; c < D; c += 32) acc = fmaf(__bfloat162float(dO[c]), Ob[c], acc);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
        const float rs = a.rowstat[(size_t)bh * a.n + row];
        if (a.softmax) {
            dl = acc;
            st = rs * 1.4426950408889634f;  // lse in log2 units
        } else {
            dl = acc / a.sum_u[(size_t)bh * a.n + row];
            st = rs;
        }
    }
    if (lane == 0) {
        delta_pad[(size_t)bh * npad + row] = dl;
        stat_pad[(size_t)bh * npad + row] = st;
    }
}

// ---------------------------------------------------------------------------------------------
// dK / dV
// ---------------------------------------------------------------------------------------------
template <int D>
struct CfgKV {
    static constexpr uint32_t kTile = TM * D * 2;   // K or V tile, 16 / 32 KB
    static constexpr uint32_t kBlk = TB * D * 2;    // Q_I or dO_I block, 8 / 16 KB
    static constexpr uint32_t kStage = 2 * kBlk + 1024;  // Q_I, dO_I, stat[64], delta[64] (+ pad)
    static constexpr uint32_t offK = 0;
    static constexpr uint32_t offV = offK + kTile;
    static constexpr uint32_t offSt = offV + kTile;               // NST stages
    static constexpr uint32_t offBar = offSt + NST * kStage;
    // TMEM: S^T and dP^T (double-buffered at d = 64), dV, dK, and the A operands of the gradient MMAs,
    // read by tcgen05.mma from TMEM: per K step of 16 query rows 32 columns [P^T hi | P^T lo | dS^T hi |
    // dS^T lo], 8 columns (16 bf16) each.
    static constexpr int NSB = (D == 64) ? 2 : 1;
    static constexpr uint32_t colS = 0;
    static constexpr uint32_t colDP = NSB * TB;
    static constexpr uint32_t colDV = 2 * NSB * TB;
    static constexpr uint32_t colDK = colDV + D;
    static constexpr uint32_t colA = colDK + D;
    static constexpr uint32_t tmemCols = 512;
    static_assert(colA + 128 <= tmemCols, "TMEM budget");
};

struct BarsKV {
    uint64_t kv_full;
    uint64_t q_full[NST], q_empty[NST];
    uint64_t s_full[2], s_empty[2];
    uint64_t ds_full, ds_empty;
    uint64_t acc_full;
    uint64_t drain;
    uint32_t tmem_base;
    int abort_flag;
    int nvisit;
};

template <int D, int MODE, bool SPLIT>
__global__ void __launch_bounds__(kThreads, 1)
    bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
                    const BwdArgs a, const float* __restrict__ delta_pad, const float* __restrict__ stat_pad) {
    using C = CfgKV<D>;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char* smem = align_smem_1024(smem_raw);
    BarsKV& bb = *reinterpret_cast<BarsKV*>(smem + C::offBar);
    uint32_t* vis = reinterpret_cast<uint32_t*>(&bb + 1);  // [nwq] query blocks to visit

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int kt = blockIdx.y;  // grid (B*H, key tiles): the longest (first) key tiles of every head first
    const int bh = blockIdx.x;
    const int k0 = kt * TM;
    const int nwq = a.nwq;
    const int npad = a.nqb * TB;
    volatile int* abort_flag = &bb.abort_flag;

    if (tid == 0) {
        mbar_init(&bb.kv_full, 1);
        for (int i = 0; i < NST; ++i) { mbar_init(&bb.q_full[i], 1); mbar_init(&bb.q_empty[i], 1); }
        for (int i = 0; i < 2; ++i) { mbar_init(&bb.s_full[i], 1); mbar_init(&bb.s_empty[i], TM); }
        mbar_init(&bb.ds_full, TM);
        mbar_init(&bb.ds_empty, 1);
        mbar_init(&bb.acc_full, 1);
        mbar_init(&bb.drain, 1);
        bb.abort_flag = 0;
        fence_barrier_init();
    }
    // query blocks to visit: set in either 64-key half of the tile (entmax), or every causal block
    const int J0 = 2 * kt, J1 = 2 * kt + 1;
    for (int w = tid; w < nwq; w += blockDim.x) {
        uint32_t v = 0u;
        if (a.maskT) {
            v = a.maskT[((size_t)bh * a.nkb + J0) * nwq + w];
            if (J1 < a.nkb) v |= a.maskT[((size_t)bh * a.nkb + J1) * nwq + w];
        } else {
            const int ib = a.causal ? 2 * kt : 0;  // first query block with an allowed entry
            for (int b = 0; b < 32; ++b) {
                const int I = w * 32 + b;
                if (I >= ib && I < a.nqb) v |= 1u << b;
            }
        }
        vis[w] = v;
    }
    if (warp == 0) {
        tmem_alloc(&bb.tmem_base, C::tmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bb.tmem_base;
    const uint32_t sK = smem_u32(smem + C::offK);
    const uint32_t sV = smem_u32(smem + C::offV);
    const uint32_t sSt = smem_u32(smem + C::offSt);

    if (warp == 5) {
        if (lane == 0) {
            tma_prefetch_desc(&tmQ); tma_prefetch_desc(&tmK); tma_prefetch_desc(&tmV); tma_prefetch_desc(&tmdO);
            mbar_arrive_expect_tx(&bb.kv_full, 2 * C::kTile);
            for (int c = 0; c < D / 64; ++c) {
                tma_load_3d(smem + C::offK + c * (TM * 128), &tmK, &bb.kv_full, 64 * c, k0, bh);
                tma_load_3d(smem + C::offV + c * (TM * 128), &tmV, &bb.kv_full, 64 * c, k0, bh);
            }
            uint32_t i = 0;
            bool ok = true;
            for (int w = 0; w < nwq && ok; ++w) {
                uint32_t bits = vis[w];
                while (bits && ok) {
                    const int I = w * 32 + __ffs(bits) - 1;
                    bits &= bits - 1;
                    const uint32_t st = i % NST;
                    if (!(ok = wait_bounded(&bb.q_empty[st], ((i / NST) & 1) ^ 1, abort_flag, a.status, true))) break;
                    unsigned char* base = smem + C::offSt + st * C::kStage;
                    mbar_arrive_expect_tx(&bb.q_full[st], 2 * C::kBlk + 512);
                    for (int c = 0; c < D / 64; ++c) {
                        tma_load_3d(base + c * (TB * 128), &tmQ, &bb.q_full[st], 64 * c, I * TB, bh);
                        tma_load_3d(base + C::kBlk + c * (TB * 128), &tmdO, &bb.q_full[st], 64 * c, I * TB, bh);
                    }
                    bulk_load(base + 2 * C::kBlk, stat_pad + (size_t)bh * npad + I * TB, 256, &bb.q_full[st]);
                    bulk_load(base + 2 * C::kBlk + 256, delta_pad + (size_t)bh * npad + I * TB, 256, &bb.q_full[st]);
                    ++i;
                }
            }
            if (!ok) {
                for (uint32_t j = (i > NST ? i - NST : 0); j < i; ++j) wait_drain(&bb.q_full[j % NST], (j / NST) & 1, 100000000ull);
                wait_drain(&bb.kv_full, 0, 100000000ull);
            }
        }
    } else if (warp == 4) {
        if (lane == 0) {
            constexpr uint32_t idS = idesc_bf16_f32(TM, TB, false, false);   // K Q^T, V dO^T
            constexpr uint32_t idG = idesc_bf16_f32(TM, D, false, true);     // P^T dO, dS^T Q (MN-major B)
            bool ok = wait_bounded(&bb.kv_full, 0, abort_flag, a.status, true);
            tc_fence_after();
            uint32_t i = 0;
            auto issue_S = [&](uint32_t idx) -> bool {
                const uint32_t st = idx % NST, sb = idx % C::NSB;
                if (!wait_bounded(&bb.q_full[st], (idx / NST) & 1, abort_flag, a.status, true)) return false;
                if (!wait_bounded(&bb.s_empty[sb], ((idx / C::NSB) & 1) ^ 1, abort_flag, a.status, true)) return false;
                tc_fence_after();
                const uint32_t qb = sSt + st * C::kStage, ob = qb + C::kBlk;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t sub = kk >> 2, off = (kk & 3) * 32;
                    const uint64_t dk = sdesc_at(kDescK, sK + sub * (TM * 128) + off);
                    const uint64_t dq = sdesc_at(kDescK, qb + sub * (TB * 128) + off);
                    const uint64_t dv = sdesc_at(kDescK, sV + sub * (TM * 128) + off);
                    const uint64_t dd = sdesc_at(kDescK, ob + sub * (TB * 128) + off);
                    mma_ss(tmem + C::colS + sb * TB, dk, dq, idS, kk > 0);
                    mma_ss(tmem + C::colDP + sb * TB, dv, dd, idS, kk > 0);
                }
                mma_commit(&bb.s_full[sb]);
                return true;
            };
            auto issue_G = [&](uint32_t idx, bool first) -> bool {
                const uint32_t st = idx % NST;
                if (!wait_bounded(&bb.ds_full, idx & 1, abort_flag, a.status, true)) return false;
                tc_fence_after();
                const uint32_t qb = sSt + st * C::kStage, ob = qb + C::kBlk;
#pragma unroll
                for (int kk = 0; kk < TB / 16; ++kk) {
                    const uint64_t dob = sdesc_at(kDescMN, ob + kk * 2048);
                    const uint64_t dqb = sdesc_at(kDescMN, qb + kk * 2048);
                    const uint32_t ta = tmem + C::colA + 32 * kk;  // this K step's operands
                    const uint32_t acc = (first && kk == 0) ? 0u : 1u;
                    mma_ts(tmem + C::colDV, ta + 0, dob, idG, acc);
                    if constexpr (SPLIT) mma_ts(tmem + C::colDV, ta + 8, dob, idG, 1u);
                    mma_ts(tmem + C::colDK, ta + 16, dqb, idG, acc);
                    if constexpr (SPLIT) mma_ts(tmem + C::colDK, ta + 24, dqb, idG, 1u);
                }
                mma_commit(&bb.ds_empty);
                mma_commit(&bb.q_empty[st]);
                return true;
            };
            uint32_t total = 0;
            for (int w = 0; w < nwq; ++w) total += __popc(vis[w]);
            if (ok && total > 0) ok = issue_S(0);
            for (i = 0; ok && i < total; ++i) {
                if (i + 1 < total && !(ok = issue_S(i + 1))) break;
                if (!(ok = issue_G(i, i == 0))) break;
            }
            if (ok) mma_commit(&bb.acc_full);
            mma_commit(&bb.drain);
            wait_drain(&bb.drain, 0, 200000000ull);
        }
    } else {
        // ------------------------------------------------------------------ compute warps
        const int r = tid;            // key row of the tile == TMEM lane
        const int key = k0 + r;
        const bool kvalid = key < a.n;
        const uint32_t lane_base = tmem + ((uint32_t)(warp * 32) << 16);
        bool ok = true;
        uint32_t i = 0;
        float sv[TB], dpv[TB];
        for (int w = 0; w < nwq && ok; ++w) {
            uint32_t bits = vis[w];
            while (bits) {
                const int I = w * 32 + __ffs(bits) - 1;
                bits &= bits - 1;
                const uint32_t sb = i % C::NSB, st = i % NST;
                ok = __all_sync(0xffffffffu, wait_bounded(&bb.s_full[sb], (i / C::NSB) & 1, abort_flag, a.status));
                if (!ok) break;
                tc_fence_after();
                __syncwarp();
                tmem_ld32(lane_base + C::colS + sb * TB, reinterpret_cast<uint32_t*>(sv));
                tmem_ld32(lane_base + C::colS + sb * TB + 32, reinterpret_cast<uint32_t*>(sv) + 32);
                tmem_ld32(lane_base + C::colDP + sb * TB, reinterpret_cast<uint32_t*>(dpv));
                tmem_ld32(lane_base + C::colDP + sb * TB + 32, reinterpret_cast<uint32_t*>(dpv) + 32);
                tmem_ld_wait();
                tc_fence_before();
                mbar_arrive(&bb.s_empty[sb]);
                // the row statistics of block I arrived with its Q / dO stage
                ok = __all_sync(0xffffffffu, wait_bounded(&bb.q_full[st], (i / NST) & 1, abort_flag, a.status));
                if (!ok) break;
                const float* stat = reinterpret_cast<const float*>(smem + C::offSt + st * C::kStage + 2 * C::kBlk);
                const float* dl = stat + 64;
                const int q0 = I * TB;
                const bool full = kvalid && (q0 + TB <= a.n) && (!a.causal || q0 >= k0 + TM - 1);
                // the A tiles of the previous block's gradient MMAs must have been read
                ok = __all_sync(0xffffffffu, wait_bounded(&bb.ds_empty, (i & 1) ^ 1, abort_flag, a.status));
                if (!ok) break;
                const uint32_t ta = lane_base + C::colA;
                // P^T and dS^T rows for this key against the 64 query rows of block I, 16 columns at a time
#pragma unroll
                for (int gp = 0; gp < 4; ++gp) {
                    uint32_t ks[32];  // [P^T hi 8 | P^T lo 8 | dS^T hi 8 | dS^T lo 8]
                    uint32_t* ph = ks;
                    uint32_t* pl = ks + 8;
                    uint32_t* dh = ks + 16;
                    uint32_t* dlo = ks + 24;
                    float st16[16], dl16[16];
#pragma unroll
                    for (int i4 = 0; i4 < 4; ++i4) {  // broadcast loads of the 16 columns' statistics
                        const float4 a4 = *reinterpret_cast<const float4*>(stat + 16 * gp + 4 * i4);
                        const float4 b4 = *reinterpret_cast<const float4*>(dl + 16 * gp + 4 * i4);
                        st16[4 * i4] = a4.x; st16[4 * i4 + 1] = a4.y; st16[4 * i4 + 2] = a4.z; st16[4 * i4 + 3] = a4.w;
                        dl16[4 * i4] = b4.x; dl16[4 * i4 + 1] = b4.y; dl16[4 * i4 + 2] = b4.z; dl16[4 * i4 + 3] = b4.w;
                    }
                    // entmax: 16 columns with no positive z - tau give P = dS = 0 (the usual case)
                    bool anyx = (MODE == kModeSoftmax);
                    if constexpr (MODE != kModeSoftmax) {
                        float xm = -1.f;
#pragma unroll
                        for (int e = 0; e < 16; ++e) xm = fmaxf(xm, fmaf(sv[16 * gp + e], a.cz, -st16[e]));
                        anyx = xm > 0.f;
                    }
                    if (anyx) {
#pragma unroll
                    for (int q2 = 0; q2 < 8; ++q2) {
                        float pp[2], dd[2];
#pragma unroll
                        for (int e = 0; e < 2; ++e) {
                            const int cc = 2 * q2 + e;
                            const int c = 16 * gp + cc;
                            const int qi = q0 + c;
                            const bool okc = full || (kvalid && qi < a.n && (!a.causal || qi >= key));
                            float p, u;
                            pointwise<MODE>(sv[c], st16[cc], a.cz, a.k, okc, p, u);
                            pp[e] = p;
                            dd[e] = u * (dpv[c] - dl16[cc]);
                        }
                        split2<SPLIT>(pp, ph[q2], pl[q2]);
                        split2<SPLIT>(dd, dh[q2], dlo[q2]);
                    }
                    } else {
#pragma unroll
                        for (int q2 = 0; q2 < 8; ++q2) ph[q2] = pl[q2] = dh[q2] = dlo[q2] = 0u;
                    }
                    tmem_st32(ta + 32 * gp, ks);
                }
                tmem_st_wait();
                tc_fence_before();
                mbar_arrive(&bb.ds_full);
                ++i;
            }
        }
        ok = !bar_or128(!ok || *abort_flag != 0);
        // ---- epilogue: dV and scale * dK to global (fp32) ----
        if (i > 0 && ok)
            ok = __all_sync(0xffffffffu, wait_bounded(&bb.acc_full, 0, abort_flag, a.status));
        ok = !bar_or128(!ok || *abort_flag != 0);
        float* dK = static_cast<float*>(a.dK) + ((size_t)bh * a.n + key) * D;
        float* dV = static_cast<float*>(a.dV) + ((size_t)bh * a.n + key) * D;
        if (ok && i > 0) {
            tc_fence_after();
            __syncwarp();
#pragma unroll
            for (int c0 = 0; c0 < D; c0 += 32) {
                uint32_t vv[32], kk[32];
                tmem_ld32(lane_base + C::colDV + c0, vv);
                tmem_ld32(lane_base + C::colDK + c0, kk);
                tmem_ld_wait();
                if (kvalid) {
#pragma unroll
                    for (int j = 0; j < 32; j += 4) {
                        *reinterpret_cast<float4*>(dV + c0 + j) =
                            make_float4(__uint_as_float(vv[j]), __uint_as_float(vv[j + 1]),
                                        __uint_as_float(vv[j + 2]), __uint_as_float(vv[j + 3]));
                        *reinterpret_cast<float4*>(dK + c0 + j) = make_float4(
                            a.scale * __uint_as_float(kk[j]), a.scale * __uint_as_float(kk[j + 1]),
                            a.scale * __uint_as_float(kk[j + 2]), a.scale * __uint_as_float(kk[j + 3]));
                    }
                }
            }
            tc_fence_before();
        } else if (ok && kvalid) {
            // no query block attends to this key tile
            for (int c = 0; c < D; c += 4) {
                *reinterpret_cast<float4*>(dV + c) = make_float4(0.f, 0.f, 0.f, 0.f);
                *reinterpret_cast<float4*>(dK + c) = make_float4(0.f, 0.f, 0.f, 0.f);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, C::tmemCols);
    }
}

// ---------------------------------------------------------------------------------------------
// dQ
// ---------------------------------------------------------------------------------------------
template <int D>
struct CfgQ {
    static constexpr uint32_t kTile = TM * D * 2;   // Q or dO tile
    static constexpr uint32_t kBlk = TB * D * 2;    // K_J or V_J block
    static constexpr uint32_t kStage = 2 * kBlk;
    static constexpr uint32_t offQ = 0;
    static constexpr uint32_t offO = offQ + kTile;
    static constexpr uint32_t offSt = offO + kTile;  // NST stages of K_J, V_J
    static constexpr uint32_t offBar = offSt + NST * kStage;
    // TMEM: S and dP double buffers, dQ, and the A operands of the dQ MMA: per K step of 16 keys 16
    // columns [dS hi | dS lo], 8 columns each
    static constexpr uint32_t colS = 0;
    static constexpr uint32_t colDP = 128;
    static constexpr uint32_t colDQ = 256;
    static constexpr uint32_t colA = 256 + D;
    static constexpr uint32_t tmemCols = 512;
    static_assert(colA + 64 <= tmemCols, "TMEM budget");
};

template <int D, int MODE, bool SPLIT>
__global__ void __launch_bounds__(kThreads, 1)
    bwd_dq_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
                  const BwdArgs a, const float* __restrict__ delta_pad, const float* __restrict__ stat_pad) {
    using C = CfgQ<D>;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char* smem = align_smem_1024(smem_raw);
    BarsKV& bb = *reinterpret_cast<BarsKV*>(smem + C::offBar);
    uint32_t* vis = reinterpret_cast<uint32_t*>(&bb + 1);  // [nw] key blocks to visit

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int qt = (int)gridDim.y - 1 - (int)blockIdx.y;  // grid (B*H, tiles): longest tiles of every head first
    const int bh = blockIdx.x;
    const int q0 = qt * TM;
    const int nw = a.nw;
    const int npad = a.nqb * TB;
    volatile int* abort_flag = &bb.abort_flag;

    if (tid == 0) {
        mbar_init(&bb.kv_full, 1);
        for (int i = 0; i < NST; ++i) { mbar_init(&bb.q_full[i], 1); mbar_init(&bb.q_empty[i], 1); }
        for (int i = 0; i < 2; ++i) { mbar_init(&bb.s_full[i], 1); mbar_init(&bb.s_empty[i], TM); }
        mbar_init(&bb.ds_full, TM);
        mbar_init(&bb.ds_empty, 1);
        mbar_init(&bb.acc_full, 1);
        mbar_init(&bb.drain, 1);
        bb.abort_flag = 0;
        fence_barrier_init();
    }
    const int I0 = 2 * qt, I1 = 2 * qt + 1;
    for (int w = tid; w < nw; w += blockDim.x) {
        uint32_t v = 0u;
        if (a.mask) {
            v = a.mask[((size_t)bh * a.nqb + I0) * nw + w];
            if (I1 < a.nqb) v |= a.mask[((size_t)bh * a.nqb + I1) * nw + w];
        } else {
            const int je = a.causal ? min(a.nkb, 2 * qt + 2) : a.nkb;  // key blocks with an allowed entry
            for (int b = 0; b < 32; ++b) {
                const int J = w * 32 + b;
                if (J < je) v |= 1u << b;
            }
        }
        vis[w] = v;
    }
    if (warp == 0) {
        tmem_alloc(&bb.tmem_base, C::tmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bb.tmem_base;
    const uint32_t sQ = smem_u32(smem + C::offQ);
    const uint32_t sO = smem_u32(smem + C::offO);
    const uint32_t sSt = smem_u32(smem + C::offSt);

    if (warp == 5) {
        if (lane == 0) {
            tma_prefetch_desc(&tmQ); tma_prefetch_desc(&tmK); tma_prefetch_desc(&tmV); tma_prefetch_desc(&tmdO);
            mbar_arrive_expect_tx(&bb.kv_full, 2 * C::kTile);
            for (int c = 0; c < D / 64; ++c) {
                tma_load_3d(smem + C::offQ + c * (TM * 128), &tmQ, &bb.kv_full, 64 * c, q0, bh);
                tma_load_3d(smem + C::offO + c * (TM * 128), &tmdO, &bb.kv_full, 64 * c, q0, bh);
            }
            uint32_t i = 0;
            bool ok = true;
            for (int w = 0; w < nw && ok; ++w) {
                uint32_t bits = vis[w];
                while (bits && ok) {
                    const int J = w * 32 + __ffs(bits) - 1;
                    bits &= bits - 1;
                    const uint32_t st = i % NST;
                    if (!(ok = wait_bounded(&bb.q_empty[st], ((i / NST) & 1) ^ 1, abort_flag, a.status, true))) break;
                    unsigned char* base = smem + C::offSt + st * C::kStage;
                    mbar_arrive_expect_tx(&bb.q_full[st], 2 * C::kBlk);
                    for (int c = 0; c < D / 64; ++c) {
                        tma_load_3d(base + c * (TB * 128), &tmK, &bb.q_full[st], 64 * c, J * TB, bh);
                        tma_load_3d(base + C::kBlk + c * (TB * 128), &tmV, &bb.q_full[st], 64 * c, J * TB, bh);
                    }
                    ++i;
                }
            }
            if (!ok) {
                for (uint32_t j = (i > NST ? i - NST : 0); j < i; ++j) wait_drain(&bb.q_full[j % NST], (j / NST) & 1, 100000000ull);
                wait_drain(&bb.kv_full, 0, 100000000ull);
            }
        }
    } else if (warp == 4) {
        if (lane == 0) {
            constexpr uint32_t idS = idesc_bf16_f32(TM, TB, false, false);   // Q K^T, dO V^T
            constexpr uint32_t idG = idesc_bf16_f32(TM, D, false, true);     // dS K (MN-major B)
            bool ok = wait_bounded(&bb.kv_full, 0, abort_flag, a.status, true);
            tc_fence_after();
            auto issue_S = [&](uint32_t idx) -> bool {
                const uint32_t st = idx % NST, sb = idx & 1;
                if (!wait_bounded(&bb.q_full[st], (idx / NST) & 1, abort_flag, a.status, true)) return false;
                if (!wait_bounded(&bb.s_empty[sb], ((idx >> 1) & 1) ^ 1, abort_flag, a.status, true)) return false;
                tc_fence_after();
                const uint32_t kb = sSt + st * C::kStage, vb = kb + C::kBlk;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t sub = kk >> 2, off = (kk & 3) * 32;
                    const uint64_t dq = sdesc_at(kDescK, sQ + sub * (TM * 128) + off);
                    const uint64_t dk = sdesc_at(kDescK, kb + sub * (TB * 128) + off);
                    const uint64_t dd = sdesc_at(kDescK, sO + sub * (TM * 128) + off);
                    const uint64_t dv = sdesc_at(kDescK, vb + sub * (TB * 128) + off);
                    mma_ss(tmem + C::colS + sb * TB, dq, dk, idS, kk > 0);
                    mma_ss(tmem + C::colDP + sb * TB, dd, dv, idS, kk > 0);
                }
                mma_commit(&bb.s_full[sb]);
                return true;
            };
            auto issue_G = [&](uint32_t idx, bool first) -> bool {
                const uint32_t st = idx % NST;
                if (!wait_bounded(&bb.ds_full, idx & 1, abort_flag, a.status, true)) return false;
                tc_fence_after();
                const uint32_t kb = sSt + st * C::kStage;
#pragma unroll
                for (int kk = 0; kk < TB / 16; ++kk) {
                    const uint64_t dkb = sdesc_at(kDescMN, kb + kk * 2048);
                    const uint32_t ta = tmem + C::colA + 16 * kk;
                    const uint32_t acc = (first && kk == 0) ? 0u : 1u;
                    mma_ts(tmem + C::colDQ, ta, dkb, idG, acc);
                    if constexpr (SPLIT) mma_ts(tmem + C::colDQ, ta + 8, dkb, idG, 1u);
                }
                mma_commit(&bb.ds_empty);
                mma_commit(&bb.q_empty[st]);
                return true;
            };
            uint32_t total = 0;
            for (int w = 0; w < nw; ++w) total += __popc(vis[w]);
            if (ok && total > 0) ok = issue_S(0);
            for (uint32_t i = 0; ok && i < total; ++i) {
                if (i + 1 < total && !(ok = issue_S(i + 1))) break;
                if (!(ok = issue_G(i, i == 0))) break;
            }
            if (ok) mma_commit(&bb.acc_full);
            mma_commit(&bb.drain);
            wait_drain(&bb.drain, 0, 200000000ull);
        }
    } else {
        // ------------------------------------------------------------------ compute warps
        const int r = tid;
        const int row = q0 + r;
        const bool qvalid = row < a.n;
        const uint32_t lane_base = tmem + ((uint32_t)(warp * 32) << 16);
        const float stat = stat_pad[(size_t)bh * npad + min(row, npad - 1)];
        const float dl = delta_pad[(size_t)bh * npad + min(row, npad - 1)];
        bool ok = true;
        uint32_t i = 0;
        float sv[TB], dpv[TB];
        for (int w = 0; w < nw && ok; ++w) {
            uint32_t bits = vis[w];
            while (bits) {
                const int J = w * 32 + __ffs(bits) - 1;
                bits &= bits - 1;
                const uint32_t sb = i & 1;
                ok = __all_sync(0xffffffffu, wait_bounded(&bb.s_full[sb], (i >> 1) & 1, abort_flag, a.status));
                if (!ok) break;
                tc_fence_after();
                __syncwarp();
                tmem_ld32(lane_base + C::colS + sb * TB, reinterpret_cast<uint32_t*>(sv));
                tmem_ld32(lane_base + C::colS + sb * TB + 32, reinterpret_cast<uint32_t*>(sv) + 32);
                tmem_ld32(lane_base + C::colDP + sb * TB, reinterpret_cast<uint32_t*>(dpv));
                tmem_ld32(lane_base + C::colDP + sb * TB + 32, reinterpret_cast<uint32_t*>(dpv) + 32);
                tmem_ld_wait();
                tc_fence_before();
                mbar_arrive(&bb.s_empty[sb]);
                const int j0 = J * TB;
                const bool full = qvalid && (j0 + TB <= a.n) && (!a.causal || j0 + TB - 1 <= q0);
                ok = __all_sync(0xffffffffu, wait_bounded(&bb.ds_empty, (i & 1) ^ 1, abort_flag, a.status));
                if (!ok) break;
                const uint32_t ta = lane_base + C::colA;
#pragma unroll
                for (int gp = 0; gp < 4; ++gp) {
                    uint32_t ks[16];  // [dS hi 8 | dS lo 8]
                    uint32_t* dh = ks;
                    uint32_t* dlo = ks + 8;
                    bool anyx = (MODE == kModeSoftmax);
                    if constexpr (MODE != kModeSoftmax) {
                        float sm = sv[16 * gp];
#pragma unroll
                        for (int e = 1; e < 16; ++e) sm = fmaxf(sm, sv[16 * gp + e]);
                        anyx = fmaf(sm, a.cz, -stat) > 0.f;
                    }
                    if (anyx) {
#pragma unroll
                    for (int q2 = 0; q2 < 8; ++q2) {
                        float dd[2];
#pragma unroll
                        for (int e = 0; e < 2; ++e) {
                            const int c = 16 * gp + 2 * q2 + e;
                            const int kj = j0 + c;
                            const bool okc = full || (qvalid && kj < a.n && (!a.causal || kj <= row));
                            float p, u;
                            pointwise<MODE>(sv[c], stat, a.cz, a.k, okc, p, u);
                            dd[e] = u * (dpv[c] - dl);
                        }
                        split2<SPLIT>(dd, dh[q2], dlo[q2]);
                    }
                    } else {
#pragma unroll
                        for (int q2 = 0; q2 < 8; ++q2) dh[q2] = dlo[q2] = 0u;
                    }
                    tmem_st16(ta + 16 * gp, ks);
                }
                tmem_st_wait();
                tc_fence_before();
                mbar_arrive(&bb.ds_full);
                ++i;
            }
        }
        ok = !bar_or128(!ok || *abort_flag != 0);
        if (i > 0 && ok) ok = __all_sync(0xffffffffu, wait_bounded(&bb.acc_full, 0, abort_flag, a.status));
        ok = !bar_or128(!ok || *abort_flag != 0);
        float* dQ = static_cast<float*>(a.dQ) + ((size_t)bh * a.n + row) * D;
        if (ok && i > 0) {
            tc_fence_after();
            __syncwarp();
#pragma unroll
            for (int c0 = 0; c0 < D; c0 += 32) {
                uint32_t qq[32];
                tmem_ld32(lane_base + C::colDQ + c0, qq);
                tmem_ld_wait();
                if (qvalid) {
#pragma unroll
                    for (int j = 0; j < 32; j += 4)
                        *reinterpret_cast<float4*>(dQ + c0 + j) = make_float4(
                            a.scale * __uint_as_float(qq[j]), a.scale * __uint_as_float(qq[j + 1]),
                            a.scale * __uint_as_float(qq[j + 2]), a.scale * __uint_as_float(qq[j + 3]));
                }
            }
            tc_fence_before();
        } else if (ok && qvalid) {
            for (int c = 0; c < D; c += 4) *reinterpret_cast<float4*>(dQ + c) = make_float4(0.f, 0.f, 0.f, 0.f);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, C::tmemCols);
    }
}

template <int D, int MODE, bool SPLIT>
cudaError_t launch_t(const BwdArgs& a, float* delta_pad, float* stat_pad, cudaStream_t stream) {
    cudaError_t e;
    const int BH = a.B * a.H;
    {
        const int warps = 8;
        dim3 grid((a.nqb * TB + warps - 1) / warps, BH);
        launch_mark(stream);
        bwd_pre_kernel<D><<<grid, warps * 32, 0, stream>>>(a, delta_pad, stat_pad);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    CUtensorMap tq128, tdo128, tk128, tv128, tq64, tdo64, tk64, tv64;
    if ((e = make_tmap_bf16(&tq128, a.Q, BH, a.n, D, TM)) != cudaSuccess) return e;
    if ((e = make_tmap_bf16(&tdo128, a.dO, BH, a.n, D, TM)) != cudaSuccess) return e;
    if ((e = make_tmap_bf16(&tk128, a.K, BH, a.n, D, TM)) != cudaSuccess) return e;
    if ((e = make_tmap_bf16(&tv128, a.V, BH, a.n, D, TM)) != cudaSuccess) return e;
    if ((e = make_tmap_bf16(&tq64, a.Q, BH, a.n, D, TB)) != cudaSuccess) return e;
    if ((e = make_tmap_bf16(&tdo64, a.dO, BH, a.n, D, TB)) != cudaSuccess) return e;
    if ((e = make_tmap_bf16(&tk64, a.K, BH, a.n, D, TB)) != cudaSuccess) return e;
    if ((e = make_tmap_bf16(&tv64, a.V, BH, a.n, D, TB)) != cudaSuccess) return e;
    const int ntiles = (a.n + TM - 1) / TM;
    {
        using C = CfgKV<D>;
        const size_t bytes = 1024 + C::offBar + sizeof(BarsKV) + (size_t)a.nwq * 4;
        auto kern = bwd_dkdv_kernel<D, MODE, SPLIT>;
        if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes)) != cudaSuccess)
            return e;
        launch_mark(stream);
        kern<<<dim3(BH, ntiles), kThreads, bytes, stream>>>(tq64, tk128, tv128, tdo64, a, delta_pad, stat_pad);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    {
        using C = CfgQ<D>;
        const size_t bytes = 1024 + C::offBar + sizeof(BarsKV) + (size_t)a.nw * 4;
        auto kern = bwd_dq_kernel<D, MODE, SPLIT>;
        if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes)) != cudaSuccess)
            return e;
        launch_mark(stream);
        kern<<<dim3(BH, ntiles), kThreads, bytes, stream>>>(tq128, tk64, tv64, tdo128, a, delta_pad, stat_pad);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    return cudaSuccess;
}

template <int D>
cudaError_t launch_d(const BwdArgs& a, float* dp, float* sp, cudaStream_t s) {
    if (a.softmax) return launch_t<D, kModeSoftmax, false>(a, dp, sp, s);
    if (a.kind == kAlpha15) return launch_t<D, kAlpha15, true>(a, dp, sp, s);
    if (a.kind == kAlpha2) return launch_t<D, kAlpha2, true>(a, dp, sp, s);
    return launch_t<D, kGeneric, true>(a, dp, sp, s);
}

}  // namespace

cudaError_t launch_bwd_pre(const BwdArgs& a, float* delta_pad, float* stat_pad, cudaStream_t stream) {
    const int warps = 8;
    dim3 grid((a.nqb * TB + warps - 1) / warps, a.B * a.H);
    launch_mark(stream);
    if (a.d == 64) bwd_pre_kernel<64><<<grid, warps * 32, 0, stream>>>(a, delta_pad, stat_pad);
    else bwd_pre_kernel<128><<<grid, warps * 32, 0, stream>>>(a, delta_pad, stat_pad);
    return cudaGetLastError();
}

cudaError_t launch_bwd(const BwdArgs& a, float* delta_pad, float* stat_pad, cudaStream_t stream) {
    if (a.d == 64) return launch_d<64>(a, delta_pad, stat_pad, stream);
    return launch_d<128>(a, delta_pad, stat_pad, stream);
}

size_t bwd_smem_bytes(int d, int nw, int nwq) {
    const size_t kv = 1024 + (d == 64 ? CfgKV<64>::offBar : CfgKV<128>::offBar) + sizeof(BarsKV) + (size_t)nwq * 4;
    const size_t q = 1024 + (d == 64 ? CfgQ<64>::offBar : CfgQ<128>::offBar) + sizeof(BarsKV) + (size_t)nw * 4;
    return kv > q ? kv : q;
}

}  // namespace eattn
