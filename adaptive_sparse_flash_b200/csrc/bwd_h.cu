// bwd_h.cu - backward of alpha-entmax attention for alpha <= 2 and d = 64 on the sm_100a tensor cores,
// from fp16 copies of Q, K, V (made by the forward) and dO (f16.cu).
//
// With g = dO V^T, u = [z - tau]_+^(k-1) and delta = sum(u g) / sum(u), the score gradient is
// dS = u (g - delta); dQ = scale dS K, dK = scale dS^T Q, dV = P^T dO. Only the (query block, key block)
// pairs set in the bit-packed mask are visited ("AdaSplash-2", gist.science (de), section 2,
// "GPU-Optimierung" and "Bit-Packed Block Mask").
//
// delta: bwd_pre (bwd_tc.cu) forms an estimate d~ = dO . (U V) / sum u from the forward's U V, whose U was
// one fp16 term. bwd_h_dq runs first and uses that estimate for its dS~ = u (g - d~); while it walks a query
// row's nonzero blocks it also sums dS~ over the row in fp32, which gives the exact delta:
// sum_j u_j (g_j - d~) = sum u (delta - d~), so delta = d~ + sum_j dS~_j / sum u (sum u from the forward,
// over the same u: both passes form x = fma(s, cz, -tau) from the same score tile). It writes that delta
// back for bwd_h_dkdv, which runs second, since dK sums dS against query rows that can be large; in dQ the
// estimate's small error is damped by the unit-scale keys.
//
// The dense softmax baseline uses the same kernels (p = u = softmax probabilities, delta = dO . O, every
// causal block visited).
//
// Both kernels: 352 threads.
//   warps 0-3, 4-7  compute warpgroups 0 and 1 (thread r of a warpgroup owns row r of the CTA's
//                   128-row tile, TMEM lane r); block t of the CTA's walk goes to warpgroup t & 1;
//   warp 8          score issue (one thread): the two score products of a block into that warpgroup's
//                   TMEM buffers;
//   warp 9          TMA issue (one thread): the CTA's fixed tiles once, then a ring of walked blocks
//                   (with their row statistics);
//   warp 10         gradient issue (one thread): the gradient products, with their A operand (P^T, dS^T or
//                   dS) read from TMEM, where the compute warps store it.
// P lies in [0, 1] and enters as one fp16 term. dS enters as two fp16 terms (dS = hi + lo, ~22
// significant bits): the gradients of K and Q sum dS times rows of Q and K that can be large, where a
// single term's 11 bits are not enough. |dS| <= 2 max|g| <= 2 d max|dO| max|V|, and dS is stored scaled
// by 2^-e_ds with e_ds chosen from that bound, so that it stays inside the fp16 range (e_ds = 0 for
// inputs of unit scale). Every power-of-two factor (the copies' range exponents, e_ds) is put back in
// the epilogue.
//
//   bwd_h_dkdv  one CTA per 128-key tile, walking the query blocks of the transposed mask:
//               S^T = K Q^T, dP^T = V dO^T; dV += P^T dO, dK += dS^T Q.
//               TMEM: S^T / dP^T of warpgroup g at 128 g / 128 g + 64 (P^T overwrites the first 32
//               columns of S^T), [dS^T hi | dS^T lo] of g at 256 + 64 g, dV at 384, dK at 448. The dV
//               products of a block go as soon as its P^T is stored and run one block ahead of the dK
//               products; a new S^T goes into a buffer once the dV products that read its P^T completed.
//   bwd_h_dq    one CTA per 128-row query tile, walking the key blocks of the row mask:
//               S = Q K^T, dP = dO V^T; dQ += dS K.
//               TMEM: S / dP of g at 128 g / 128 g + 64, [dS hi | dS lo] of g at 256 + 64 g, dQ at 384.
// Score and dP tiles have their own full / empty barriers and are released as soon as the warpgroup has
// read them, so the next block's products can run while the warpgroup still computes.
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <math.h>

#include "common.cuh"
#include "entmax_row.cuh"
#include "launch.h"

namespace eattn {
namespace {

constexpr uint64_t kDescK = sdesc_sw128_fields(16, 1024);
constexpr uint64_t kDescMN = sdesc_sw128_fields(64 * 128, 1024);

constexpr int kThreads = 352;
constexpr int TM = 128;  // rows of the CTA's tile
constexpr int TB = 64;   // rows of a walked block
constexpr int D = 64;
constexpr int NST = 4;   // walked-block ring stages

constexpr uint32_t kTile = TM * D * 2;            // 16 KB
constexpr uint32_t kBlk = TB * D * 2;             // 8 KB
constexpr uint32_t kStageKV = 2 * kBlk + 1024;    // dkdv: Q_I, dO_I, tau[64], delta[64] (+ pad)
constexpr uint32_t kStageQ = 2 * kBlk;            // dq: K_J, V_J

__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ bool bar_or256(bool pred) {
    uint32_t out;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 q, %1, 0;\n\t"
        "bar.red.or.pred p, 1, 256, q;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(out)
        : "r"((uint32_t)pred)
        : "memory");
    return out != 0;
}

// Mode of the dense softmax baseline: p = 2^(x), x = s scale log2(e) - lse log2(e), u = p, delta = dO . O.
constexpr int kSoftmaxH = 3;

// p and u of one score: x = cz s - tau (x < 0 off the support); softmax: x = c2 s - lse2.
template <int KIND>
__device__ __forceinline__ void entmax_pu(float x, float k, float& p, float& u) {
    if constexpr (KIND == kSoftmaxH) {
        p = exp2f(x);
        u = p;
    } else if constexpr (KIND == kAlpha15) {
        u = fmaxf(x, 0.f);
        p = u * u;
    } else if constexpr (KIND == kAlpha2) {
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

// (a, b) as an fp16 pair (high part) and the fp16 pair of the remainders (low part).
__device__ __forceinline__ void split_half2(float a, float b, uint32_t& hi, uint32_t& lo) {
    const __half2 h = __floats2half2_rn(a, b);
    const float2 hf = __half22float2(h);
    hi = *reinterpret_cast<const uint32_t*>(&h);
    lo = pack_half2(a - hf.x, b - hf.y);
}

__device__ __forceinline__ float4 ld_shared_f4(uint32_t addr) {
    float4 v;
    asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(addr));
    return v;
}

struct Bars {
    uint64_t tile_full;
    uint64_t q_full[NST], q_empty[NST];
    uint64_t s_full[2], s_empty[2];  // score tile: MMA done / buffer free again
    uint64_t d_full[2], d_empty[2];  // dP tile: MMA done / read by the warpgroup
    uint64_t p_full[2], p_empty[2];  // dK / dV: P^T stored / the dV MMAs that read it done
    uint64_t a_full[2], a_empty[2];  // dS operands stored / the MMAs that read them done
    uint64_t acc_full;
    uint64_t drain[2];
    uint32_t tmem_base;
    int abort_flag;
};

// Exponents of the fp16 copies and of dS (see the file comment).
struct Scales {
    float cz;      // (alpha - 1) scale 2^(eQ + eK): raw fp16 score -> z
    float dl;      // 2^-(edO + eV): delta -> the scale of the fp16 dP
    float ds;      // 2^-eds: stored dS = u (dP - delta) 2^-eds
    float dv;      // dV = 2^edO (P^T dO)
    float dk;      // dK = scale 2^(edO + eV + eds + eQ) (dS^T Q)
    float dq;      // dQ = scale 2^(edO + eV + eds + eK) (dS K)
};

__device__ __forceinline__ Scales make_scales(const BwdArgs& a) {
    const int eQ = f16_range_exp(a.maxbits[0]), eK = f16_range_exp(a.maxbits[1]);
    const int eV = f16_range_exp(a.maxbits[2]), edO = f16_range_exp(a.maxbits[3]);
    // max |g| of the scaled copies <= d max|dO'| max|V'|; keep 2 max|g| below 2^15
    const float mdo = ldexpf(__uint_as_float(a.maxbits[3]), -edO);
    const float mv = ldexpf(__uint_as_float(a.maxbits[2]), -eV);
    const float bound = 2.0f * (float)D * mdo * mv;
    int eds = 0;
    if (bound >= 32768.0f && isfinite(bound)) eds = (int)ceilf(log2f(bound / 32768.0f));
    Scales s;
    s.cz = ldexpf(a.cz, eQ + eK);
    s.dl = ldexpf(1.0f, -(edO + eV));
    s.ds = ldexpf(1.0f, -eds);
    s.dv = ldexpf(1.0f, edO);
    s.dk = ldexpf(a.scale, edO + eV + eds + eQ);
    s.dq = ldexpf(a.scale, edO + eV + eds + eK);
    return s;
}

// dQ = scale dS K sums dS against key rows: when every |k| is below 8 (keys of unit scale), one fp16 term of
// dS (relative rounding 2^-11, errors of random sign) keeps dQ far inside the tolerance, and the dQ kernel
// issues one product per K step instead of two. Read from the range word of K, so that the compute warps
// and the issuing thread take the same decision.
__device__ __forceinline__ bool dq_one_term(const BwdArgs& a) { return __uint_as_float(a.maxbits[1]) < 8.0f; }

__device__ __forceinline__ void init_bars(Bars& bb) {
    mbar_init(&bb.tile_full, 1);
    for (int i = 0; i < NST; ++i) { mbar_init(&bb.q_full[i], 1); mbar_init(&bb.q_empty[i], 1); }
    for (int i = 0; i < 2; ++i) {
        mbar_init(&bb.s_full[i], 1);
        mbar_init(&bb.s_empty[i], 4);
        mbar_init(&bb.d_full[i], 1);
        mbar_init(&bb.d_empty[i], 4);
        mbar_init(&bb.p_full[i], 4);
        mbar_init(&bb.p_empty[i], 1);
        mbar_init(&bb.a_full[i], 4);
        mbar_init(&bb.a_empty[i], 1);
    }
    mbar_init(&bb.acc_full, 1);
    mbar_init(&bb.drain[0], 1);
    mbar_init(&bb.drain[1], 1);
    bb.abort_flag = 0;
    fence_barrier_init();
}

// ---------------------------------------------------------------------------------------------
// dK / dV
// ---------------------------------------------------------------------------------------------
constexpr uint32_t kvOffK = 0;
constexpr uint32_t kvOffV = kTile;
constexpr uint32_t kvOffSt = 2 * kTile;
constexpr uint32_t kvOffBar = kvOffSt + NST * kStageKV;

template <int KIND>
__global__ void __launch_bounds__(kThreads, 1)
    bwd_h_dkdv_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
                      const BwdArgs a, const float* __restrict__ delta_pad, const float* __restrict__ stat_pad) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char* smem = align_smem_1024(smem_raw);
    Bars& bb = *reinterpret_cast<Bars*>(smem + kvOffBar);
    uint32_t* vis = reinterpret_cast<uint32_t*>(&bb + 1);  // [nwq] query blocks to visit

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int kt = blockIdx.y;  // grid (B*H, key tiles): the longest (first) key tiles of every head first
    const int bh = blockIdx.x;
    const int k0 = kt * TM;
    const int nwq = a.nwq;
    const int npad = a.nqb * TB;
    volatile int* abort_flag = &bb.abort_flag;

    if (tid == 0) init_bars(bb);
    // query blocks to visit: set in either 64-key half of the tile (entmax), or every block with an
    // allowed entry (softmax baseline)
    const int J0 = 2 * kt, J1 = 2 * kt + 1;
    for (int w = tid; w < nwq; w += blockDim.x) {
        uint32_t v = 0u;
        if (a.maskT) {
            v = a.maskT[((size_t)bh * a.nkb + J0) * nwq + w];
            if (J1 < a.nkb) v |= a.maskT[((size_t)bh * a.nkb + J1) * nwq + w];
        } else {
            const int ib = a.causal ? 2 * kt : 0;
            for (int b = 0; b < 32; ++b) {
                const int I = w * 32 + b;
                if (I >= ib && I < a.nqb) v |= 1u << b;
            }
        }
        vis[w] = v;
    }
    if (warp == 0) {
        tmem_alloc(&bb.tmem_base, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bb.tmem_base;
    const uint32_t sK = smem_u32(smem + kvOffK);
    const uint32_t sV = smem_u32(smem + kvOffV);
    const uint32_t sSt = smem_u32(smem + kvOffSt);
    int T = 0;
    for (int w = 0; w < nwq; ++w) T += __popc(vis[w]);

    if (warp == 9) {
        // ------------------------------------------------------------------ TMA issue
        if (lane == 0) {
            tma_prefetch_desc(&tmQ); tma_prefetch_desc(&tmK); tma_prefetch_desc(&tmV); tma_prefetch_desc(&tmdO);
            mbar_arrive_expect_tx(&bb.tile_full, 2 * kTile);
            tma_load_3d(smem + kvOffK, &tmK, &bb.tile_full, 0, k0, bh);
            tma_load_3d(smem + kvOffV, &tmV, &bb.tile_full, 0, k0, bh);
            uint32_t i = 0;
            bool ok = true;
            for (int w = 0; w < nwq && ok; ++w) {
                uint32_t bits = vis[w];
                while (bits && ok) {
                    const int I = w * 32 + __ffs(bits) - 1;
                    bits &= bits - 1;
                    const uint32_t st = i % NST;
                    if (!(ok = wait_bounded(&bb.q_empty[st], ((i / NST) & 1) ^ 1, abort_flag, a.status, true))) break;
                    unsigned char* base = smem + kvOffSt + st * kStageKV;
                    mbar_arrive_expect_tx(&bb.q_full[st], 2 * kBlk + 512);
                    tma_load_3d(base, &tmQ, &bb.q_full[st], 0, I * TB, bh);
                    tma_load_3d(base + kBlk, &tmdO, &bb.q_full[st], 0, I * TB, bh);
                    bulk_load(base + 2 * kBlk, stat_pad + (size_t)bh * npad + I * TB, 256, &bb.q_full[st]);
                    bulk_load(base + 2 * kBlk + 256, delta_pad + (size_t)bh * npad + I * TB, 256, &bb.q_full[st]);
                    ++i;
                }
            }
            if (!ok) {
                for (uint32_t j = (i > NST ? i - NST : 0); j < i; ++j)
                    wait_drain(&bb.q_full[j % NST], (j / NST) & 1, 100000000ull);
                wait_drain(&bb.tile_full, 0, 100000000ull);
            }
        }
    } else if (warp == 8) {
        // ------------------------------------------------------------------ score issue
        if (lane == 0) {
            constexpr uint32_t idS = idesc_f16_f32(TM, TB, false, false);  // K Q^T, V dO^T
            bool ok = wait_bounded(&bb.tile_full, 0, abort_flag, a.status, true);
            tc_fence_after();
            for (int t = 0; t < T && ok; ++t) {
                const int g = t & 1;
                const uint32_t j = (uint32_t)(t >> 1), st = (uint32_t)t % NST;
                if (!(ok = wait_bounded(&bb.q_full[st], ((uint32_t)t / NST) & 1, abort_flag, a.status, true))) break;
                // S^T buffer: the warpgroup's previous P^T (written over its S^T) read by the dV MMAs
                if (!(ok = wait_bounded(&bb.p_empty[g], (j & 1) ^ 1, abort_flag, a.status, true))) break;
                tc_fence_after();
                const uint32_t qb = sSt + st * kStageKV, ob = qb + kBlk;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk)
                    mma_ss(tmem + 128u * g, sdesc_at(kDescK, sK + kk * 32), sdesc_at(kDescK, qb + kk * 32), idS, kk > 0);
                mma_commit(&bb.s_full[g]);
                // dP^T buffer: read by the warpgroup for its previous block
                if (!(ok = wait_bounded(&bb.d_empty[g], (j & 1) ^ 1, abort_flag, a.status, true))) break;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk)
                    mma_ss(tmem + 128u * g + 64, sdesc_at(kDescK, sV + kk * 32), sdesc_at(kDescK, ob + kk * 32), idS,
                           kk > 0);
                mma_commit(&bb.d_full[g]);
            }
            mma_commit(&bb.drain[0]);
            wait_drain(&bb.drain[0], 0, 200000000ull);
        }
    } else if (warp == 10) {
        // ------------------------------------------------------------------ gradient issue
        // dV of a block as soon as its P^T is stored (that frees the S^T buffer for the next block), dK
        // once its dS^T is: the dV products run one block ahead of the dK products.
        if (lane == 0) {
            constexpr uint32_t idG = idesc_f16_f32(TM, D, false, true);  // P^T dO, dS^T Q (MN-major B)
            bool ok = true;
            auto issue_dv = [&](int t) -> bool {
                const int g = t & 1;
                const uint32_t j = (uint32_t)(t >> 1), st = (uint32_t)t % NST;
                if (!wait_bounded(&bb.p_full[g], j & 1, abort_flag, a.status, true)) return false;
                tc_fence_after();
                const uint32_t ob = sSt + st * kStageKV + kBlk;
                const uint32_t tpt = tmem + 128u * g;  // P^T
#pragma unroll
                for (int kk = 0; kk < TB / 16; ++kk)
                    mma_ts(tmem + 384, tpt + 8 * kk, sdesc_at(kDescMN, ob + kk * 2048), idG, (t == 0 && kk == 0) ? 0u : 1u);
                mma_commit(&bb.p_empty[g]);
                return true;
            };
            auto issue_dk = [&](int t) -> bool {
                const int g = t & 1;
                const uint32_t j = (uint32_t)(t >> 1), st = (uint32_t)t % NST;
                if (!wait_bounded(&bb.a_full[g], j & 1, abort_flag, a.status, true)) return false;
                tc_fence_after();
                const uint32_t qb = sSt + st * kStageKV;
                const uint32_t ta = tmem + 256u + 64u * g;  // dS^T hi, lo
#pragma unroll
                for (int kk = 0; kk < TB / 16; ++kk) {
                    const uint64_t dq = sdesc_at(kDescMN, qb + kk * 2048);
                    mma_ts(tmem + 448, ta + 8 * kk, dq, idG, (t == 0 && kk == 0) ? 0u : 1u);
                    mma_ts(tmem + 448, ta + 32 + 8 * kk, dq, idG, 1u);
                }
                mma_commit(&bb.a_empty[g]);
                mma_commit(&bb.q_empty[st]);  // after the block's dV and dK (and its score MMAs)
                return true;
            };
            for (int t = 0; t < T && ok; ++t) {
                ok = issue_dv(t);
                if (ok && t > 0) ok = issue_dk(t - 1);
            }
            if (ok && T > 0) ok = issue_dk(T - 1);
            if (ok && T > 0) mma_commit(&bb.acc_full);
            mma_commit(&bb.drain[1]);
            wait_drain(&bb.drain[1], 0, 200000000ull);
        }
    } else if (warp < 8) {
        // ------------------------------------------------------------------ compute warpgroups
        const int g = warp >> 2;
        const int r = tid & (TM - 1);  // key row of the tile == TMEM lane
        const int key = k0 + r;
        const bool kvalid = key < a.n;
        const uint32_t lane_base = tmem + ((uint32_t)((warp & 3) * 32) << 16);
        const Scales sc = make_scales(a);
        bool ok = true;
        int t = 0;        // position in the walk
        uint32_t j = 0;   // blocks this warpgroup has done
        for (int w = 0; w < nwq && ok; ++w) {
            uint32_t bits = vis[w];
            while (bits) {
                const int I = w * 32 + __ffs(bits) - 1;
                bits &= bits - 1;
                const int tt = t++;
                if ((tt & 1) != g) continue;
                const uint32_t st = (uint32_t)tt % NST;
                ok = __all_sync(0xffffffffu, wait_bounded(&bb.s_full[g], j & 1, abort_flag, a.status));
                if (!ok) break;
                ok = __all_sync(0xffffffffu, wait_bounded(&bb.q_full[st], ((uint32_t)tt / NST) & 1, abort_flag, a.status));
                if (!ok) break;
                tc_fence_after();
                __syncwarp();
                float sv[TB];
                tmem_ld32(lane_base + 128u * g, reinterpret_cast<uint32_t*>(sv));
                tmem_ld32(lane_base + 128u * g + 32, reinterpret_cast<uint32_t*>(sv) + 32);
                tmem_ld_wait();
                const uint32_t sstat = sSt + st * kStageKV + 2 * kBlk;  // tau[64], then delta[64]
                const int q0 = I * TB;
                const bool full = kvalid && (q0 + TB <= a.n) && (!a.causal || q0 >= k0 + TM - 1);
                // entries outside the causal / valid range get -inf (a partial block is the rare case)
                if (__any_sync(0xffffffffu, !full)) {
#pragma unroll
                    for (int c = 0; c < TB; ++c) {
                        const int qi = q0 + c;
                        if (!(kvalid && qi < a.n && (!a.causal || qi >= key))) sv[c] = -INFINITY;
                    }
                }
                // P^T row of this key against the 64 queries of block I, written over its S^T; u kept in sv
                {
                    uint32_t w32[32];
#pragma unroll
                    for (int c = 0; c < TB; c += 4) {
                        const float4 t4 = ld_shared_f4(sstat + 4 * c);
                        const float tv[4] = {t4.x, t4.y, t4.z, t4.w};
                        float pp[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float x = fmaf(sv[c + e], sc.cz, -tv[e]);
                            float u;
                            entmax_pu<KIND>(x, a.k, pp[e], u);
                            sv[c + e] = u;
                        }
                        w32[c / 2] = pack_half2(pp[0], pp[1]);
                        w32[c / 2 + 1] = pack_half2(pp[2], pp[3]);
                    }
                    tmem_st32(lane_base + 128u * g, w32);
                }
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bb.p_full[g]);
                // dS^T = u (dP^T - delta), formed in place of dP^T
                ok = __all_sync(0xffffffffu, wait_bounded(&bb.d_full[g], j & 1, abort_flag, a.status));
                if (!ok) break;
                tc_fence_after();
                __syncwarp();
                float dp[TB];
                tmem_ld32(lane_base + 128u * g + 64, reinterpret_cast<uint32_t*>(dp));
                tmem_ld32(lane_base + 128u * g + 96, reinterpret_cast<uint32_t*>(dp) + 32);
                tmem_ld_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bb.d_empty[g]);
#pragma unroll
                for (int c = 0; c < TB; c += 4) {
                    const float4 d4 = ld_shared_f4(sstat + 256 + 4 * c);
                    const float dv4[4] = {d4.x, d4.y, d4.z, d4.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) dp[c + e] = sv[c + e] * (dp[c + e] - dv4[e] * sc.dl) * sc.ds;
                }
                // the dS^T buffer is free once this warpgroup's previous dK MMAs completed
                ok = __all_sync(0xffffffffu, wait_bounded(&bb.a_empty[g], (j & 1) ^ 1, abort_flag, a.status));
                if (!ok) break;
                const uint32_t ta = lane_base + 256u + 64u * g;
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    uint32_t whi[16], wlo[16];
#pragma unroll
                    for (int c = 0; c < 32; c += 2) split_half2(dp[32 * h + c], dp[32 * h + c + 1], whi[c / 2], wlo[c / 2]);
                    tmem_st16(ta + 16 * h, whi);
                    tmem_st16(ta + 32 + 16 * h, wlo);
                }
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bb.a_full[g]);
                ++j;
            }
        }
        ok = !bar_or256(!ok || *abort_flag != 0);
        // ---- epilogue: dV (warpgroup 0) and dK (warpgroup 1) to global (fp32) ----
        if (T > 0 && ok) ok = __all_sync(0xffffffffu, wait_bounded(&bb.acc_full, 0, abort_flag, a.status));
        ok = !bar_or256(!ok || *abort_flag != 0);
        float* dst = static_cast<float*>(g == 0 ? a.dV : a.dK) + ((size_t)bh * a.n + key) * D;
        const float f = g == 0 ? sc.dv : sc.dk;
        if (ok && T > 0) {
            tc_fence_after();
            __syncwarp();
#pragma unroll
            for (int c0 = 0; c0 < D; c0 += 32) {
                uint32_t vv[32];
                tmem_ld32(lane_base + (g == 0 ? 384u : 448u) + c0, vv);
                tmem_ld_wait();
                if (kvalid) {
#pragma unroll
                    for (int q = 0; q < 32; q += 4)
                        *reinterpret_cast<float4*>(dst + c0 + q) =
                            make_float4(f * __uint_as_float(vv[q]), f * __uint_as_float(vv[q + 1]),
                                        f * __uint_as_float(vv[q + 2]), f * __uint_as_float(vv[q + 3]));
                }
            }
            tc_fence_before();
        } else if (ok && kvalid) {
            for (int c = 0; c < D; c += 4) *reinterpret_cast<float4*>(dst + c) = make_float4(0.f, 0.f, 0.f, 0.f);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// ---------------------------------------------------------------------------------------------
// dQ
// ---------------------------------------------------------------------------------------------
constexpr uint32_t qOffQ = 0;
constexpr uint32_t qOffO = kTile;
constexpr uint32_t qOffSt = 2 * kTile;
constexpr uint32_t qOffBar = qOffSt + NST * kStageQ;

// Three forms, one launch each in entmax mode, of which the range word of K (dq_one_term) lets exactly the
// needed ones work and the others return at once (uniform over the CTA, before any barrier or TMEM use):
//   MODE kDqAB    - keys of unit scale: dQ = scale (A - delta B) with A = (u g) K and B = u K in two
//                   accumulators, delta from this kernel's own row sums (one fp16 term each);
//   MODE kDqDelta - larger keys, first: the delta pass (row sums only, no dQ product);
//   MODE kDqPlain - larger keys, second, and the softmax baseline: dS = u (g - delta) with delta from the
//                   delta pass (entmax) or from bwd_pre (softmax), one or two fp16 terms.
enum DqMode : int { kDqPlain = 0, kDqAB = 1, kDqDelta = 2 };

template <int KIND, int MODE>
__global__ void __launch_bounds__(kThreads, 1)
    bwd_h_dq_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
                    const BwdArgs a, float* __restrict__ delta_pad, const float* __restrict__ stat_pad) {
    constexpr bool ENT = KIND != kSoftmaxH;
    constexpr bool delta_only = MODE == kDqDelta;
    constexpr bool ab = MODE == kDqAB;
    static_assert(ENT || MODE == kDqPlain, "the softmax baseline takes its delta from bwd_pre");
    const bool one = dq_one_term(a);
    if (ENT && (ab != one)) return;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char* smem = align_smem_1024(smem_raw);
    Bars& bb = *reinterpret_cast<Bars*>(smem + qOffBar);
    float* xsum = reinterpret_cast<float*>(&bb + 1);             // [2][TM]: each warpgroup's row sums of u g
    uint32_t* vis = reinterpret_cast<uint32_t*>(xsum + 2 * TM);  // [nw] key blocks to visit

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int qt = (int)gridDim.y - 1 - (int)blockIdx.y;  // grid (B*H, tiles): longest tiles of every head first
    const int bh = blockIdx.x;
    const int q0 = qt * TM;
    const int nw = a.nw;
    const int npad = a.nqb * TB;
    volatile int* abort_flag = &bb.abort_flag;

    if (tid == 0) init_bars(bb);
    const int I0 = 2 * qt, I1 = 2 * qt + 1;
    for (int w = tid; w < nw; w += blockDim.x) {
        uint32_t v = 0u;
        if (a.mask) {
            v = a.mask[((size_t)bh * a.nqb + I0) * nw + w];
            if (I1 < a.nqb) v |= a.mask[((size_t)bh * a.nqb + I1) * nw + w];
        } else {
            const int je = a.causal ? min(a.nkb, 2 * qt + 2) : a.nkb;
            for (int b = 0; b < 32; ++b) {
                const int J = w * 32 + b;
                if (J < je) v |= 1u << b;
            }
        }
        vis[w] = v;
    }
    if (warp == 0) {
        tmem_alloc(&bb.tmem_base, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bb.tmem_base;
    const uint32_t sQ = smem_u32(smem + qOffQ);
    const uint32_t sO = smem_u32(smem + qOffO);
    const uint32_t sSt = smem_u32(smem + qOffSt);
    int T = 0;
    for (int w = 0; w < nw; ++w) T += __popc(vis[w]);

    if (warp == 9) {
        if (lane == 0) {
            tma_prefetch_desc(&tmQ); tma_prefetch_desc(&tmK); tma_prefetch_desc(&tmV); tma_prefetch_desc(&tmdO);
            mbar_arrive_expect_tx(&bb.tile_full, 2 * kTile);
            tma_load_3d(smem + qOffQ, &tmQ, &bb.tile_full, 0, q0, bh);
            tma_load_3d(smem + qOffO, &tmdO, &bb.tile_full, 0, q0, bh);
            uint32_t i = 0;
            bool ok = true;
            for (int w = 0; w < nw && ok; ++w) {
                uint32_t bits = vis[w];
                while (bits && ok) {
                    const int J = w * 32 + __ffs(bits) - 1;
                    bits &= bits - 1;
                    const uint32_t st = i % NST;
                    if (!(ok = wait_bounded(&bb.q_empty[st], ((i / NST) & 1) ^ 1, abort_flag, a.status, true))) break;
                    unsigned char* base = smem + qOffSt + st * kStageQ;
                    mbar_arrive_expect_tx(&bb.q_full[st], 2 * kBlk);
                    tma_load_3d(base, &tmK, &bb.q_full[st], 0, J * TB, bh);
                    tma_load_3d(base + kBlk, &tmV, &bb.q_full[st], 0, J * TB, bh);
                    ++i;
                }
            }
            if (!ok) {
                for (uint32_t j = (i > NST ? i - NST : 0); j < i; ++j)
                    wait_drain(&bb.q_full[j % NST], (j / NST) & 1, 100000000ull);
                wait_drain(&bb.tile_full, 0, 100000000ull);
            }
        }
    } else if (warp == 8) {
        if (lane == 0) {
            constexpr uint32_t idS = idesc_f16_f32(TM, TB, false, false);  // Q K^T, dO V^T
            bool ok = wait_bounded(&bb.tile_full, 0, abort_flag, a.status, true);
            tc_fence_after();
            for (int t = 0; t < T && ok; ++t) {
                const int g = t & 1;
                const uint32_t j = (uint32_t)(t >> 1), st = (uint32_t)t % NST;
                if (!(ok = wait_bounded(&bb.q_full[st], ((uint32_t)t / NST) & 1, abort_flag, a.status, true))) break;
                if (!(ok = wait_bounded(&bb.s_empty[g], (j & 1) ^ 1, abort_flag, a.status, true))) break;
                tc_fence_after();
                const uint32_t kb = sSt + st * kStageQ, vb = kb + kBlk;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk)
                    mma_ss(tmem + 128u * g, sdesc_at(kDescK, sQ + kk * 32), sdesc_at(kDescK, kb + kk * 32), idS, kk > 0);
                mma_commit(&bb.s_full[g]);
                if (!(ok = wait_bounded(&bb.d_empty[g], (j & 1) ^ 1, abort_flag, a.status, true))) break;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk)
                    mma_ss(tmem + 128u * g + 64, sdesc_at(kDescK, sO + kk * 32), sdesc_at(kDescK, vb + kk * 32), idS,
                           kk > 0);
                mma_commit(&bb.d_full[g]);
                if constexpr (delta_only) mma_commit(&bb.q_empty[st]);  // no dQ product reads this K block
            }
            mma_commit(&bb.drain[0]);
            wait_drain(&bb.drain[0], 0, 200000000ull);
        }
    } else if (warp == 10) {
        if (lane == 0) {
            constexpr uint32_t idG = idesc_f16_f32(TM, D, false, true);  // dS K (MN-major B)
            bool ok = true;
            for (int t = 0; t < T && ok && !delta_only; ++t) {
                const int g = t & 1;
                const uint32_t j = (uint32_t)(t >> 1), st = (uint32_t)t % NST;
                if (!(ok = wait_bounded(&bb.a_full[g], j & 1, abort_flag, a.status, true))) break;
                tc_fence_after();
                const uint32_t kb = sSt + st * kStageQ;
                const uint32_t ta = tmem + 256u + 64u * g;  // [dS hi | dS lo], or [u g | u] (ab)
#pragma unroll
                for (int kk = 0; kk < TB / 16; ++kk) {
                    const uint64_t dk = sdesc_at(kDescMN, kb + kk * 2048);
                    const uint32_t acc = (t == 0 && kk == 0) ? 0u : 1u;
                    mma_ts(tmem + 384, ta + 8 * kk, dk, idG, acc);
                    if (ab) mma_ts(tmem + 448, ta + 32 + 8 * kk, dk, idG, acc);
                    else if (!one) mma_ts(tmem + 384, ta + 32 + 8 * kk, dk, idG, 1u);
                }
                mma_commit(&bb.a_empty[g]);
                mma_commit(&bb.q_empty[st]);
            }
            if (ok && T > 0 && !delta_only) mma_commit(&bb.acc_full);
            mma_commit(&bb.drain[1]);
            wait_drain(&bb.drain[1], 0, 200000000ull);
        }
    } else if (warp < 8) {
        const int g = warp >> 2;
        const int r = tid & (TM - 1);
        const int row = q0 + r;
        const bool qvalid = row < a.n;
        const uint32_t lane_base = tmem + ((uint32_t)((warp & 3) * 32) << 16);
        const Scales sc = make_scales(a);
        const float tau = stat_pad[(size_t)bh * npad + min(row, npad - 1)];
        // delta in dP units: from bwd_pre (softmax) or the delta pass (entmax, larger keys); unused otherwise
        const float dl = (ENT && (ab || delta_only)) ? 0.f : delta_pad[(size_t)bh * npad + min(row, npad - 1)] * sc.dl;
        float rs = 0.f;  // this warpgroup's share of the row sum of u g, in dP units (entmax, ab / delta pass)
        bool ok = true;
        int t = 0;
        uint32_t j = 0;
        for (int w = 0; w < nw && ok; ++w) {
            uint32_t bits = vis[w];
            while (bits) {
                const int J = w * 32 + __ffs(bits) - 1;
                bits &= bits - 1;
                const int tt = t++;
                if ((tt & 1) != g) continue;
                ok = __all_sync(0xffffffffu, wait_bounded(&bb.s_full[g], j & 1, abort_flag, a.status));
                if (!ok) break;
                tc_fence_after();
                __syncwarp();
                float sv[TB];
                tmem_ld32(lane_base + 128u * g, reinterpret_cast<uint32_t*>(sv));
                tmem_ld32(lane_base + 128u * g + 32, reinterpret_cast<uint32_t*>(sv) + 32);
                tmem_ld_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bb.s_empty[g]);  // the score buffer is free for the next block
                const int j0 = J * TB;
                const bool full = qvalid && (j0 + TB <= a.n) && (!a.causal || j0 + TB - 1 <= q0);
                if (__any_sync(0xffffffffu, !full)) {
#pragma unroll
                    for (int c = 0; c < TB; ++c) {
                        const int kj = j0 + c;
                        if (!(qvalid && kj < a.n && (!a.causal || kj <= row))) sv[c] = -INFINITY;
                    }
                }
#pragma unroll
                for (int c = 0; c < TB; ++c) {
                    const float x = fmaf(sv[c], sc.cz, -tau);
                    float p, u;
                    entmax_pu<KIND>(x, a.k, p, u);
                    sv[c] = u;
                }
                ok = __all_sync(0xffffffffu, wait_bounded(&bb.d_full[g], j & 1, abort_flag, a.status));
                if (!ok) break;
                tc_fence_after();
                __syncwarp();
                float dp[TB];
                tmem_ld32(lane_base + 128u * g + 64, reinterpret_cast<uint32_t*>(dp));
                tmem_ld32(lane_base + 128u * g + 96, reinterpret_cast<uint32_t*>(dp) + 32);
                tmem_ld_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bb.d_empty[g]);
                if constexpr (delta_only) {
#pragma unroll
                    for (int c = 0; c < TB; ++c) rs = fmaf(sv[c], dp[c], rs);
                } else {
#pragma unroll
                    for (int c = 0; c < TB; ++c) {
                        const float e = sv[c] * (dp[c] - dl);
                        if (ab) rs += e;
                        dp[c] = e * sc.ds;
                    }
                    ok = __all_sync(0xffffffffu, wait_bounded(&bb.a_empty[g], (j & 1) ^ 1, abort_flag, a.status));
                    if (!ok) break;
                    const uint32_t ta = lane_base + 256u + 64u * g;
                    if (ab) {
                        // [u g | u], one fp16 term each (keys of unit scale), 32 keys at a time
#pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            uint32_t wa[16], wu[16];
#pragma unroll
                            for (int c = 0; c < 32; c += 2) {
                                wa[c / 2] = pack_half2(dp[32 * h + c], dp[32 * h + c + 1]);
                                wu[c / 2] = pack_half2(sv[32 * h + c], sv[32 * h + c + 1]);
                            }
                            tmem_st16(ta + 16 * h, wa);
                            tmem_st16(ta + 32 + 16 * h, wu);
                        }
                    } else if (one) {
                        uint32_t w32[32];
#pragma unroll
                        for (int c = 0; c < TB; c += 2) w32[c / 2] = pack_half2(dp[c], dp[c + 1]);
                        tmem_st32(ta, w32);
                    } else {
#pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            uint32_t whi[16], wlo[16];
#pragma unroll
                            for (int c = 0; c < 32; c += 2)
                                split_half2(dp[32 * h + c], dp[32 * h + c + 1], whi[c / 2], wlo[c / 2]);
                            tmem_st16(ta + 16 * h, whi);
                            tmem_st16(ta + 32 + 16 * h, wlo);
                        }
                    }
                    tmem_st_wait();
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&bb.a_full[g]);
                }
                ++j;
            }
        }
        xsum[g * TM + r] = rs;
        ok = !bar_or256(!ok || *abort_flag != 0);
        // entmax: delta = sum u g / sum u of this row (sum u from the forward, over the same u: both passes
        // form x = fma(s, cz, -tau) from the same score tile), in dP units; written back for the dK / dV kernel
        float dlx = 0.f;
        if (ENT && (ab || delta_only)) {
            const float s_u = qvalid ? a.sum_u[(size_t)bh * a.n + row] : 0.f;
            dlx = s_u > 0.f ? (xsum[r] + xsum[TM + r]) / s_u : 0.f;
            if (ok && g == 0 && qvalid) delta_pad[(size_t)bh * npad + row] = dlx / sc.dl;
        }
        if constexpr (!delta_only) {
            if (T > 0 && ok) ok = __all_sync(0xffffffffu, wait_bounded(&bb.acc_full, 0, abort_flag, a.status));
            ok = !bar_or256(!ok || *abort_flag != 0);
            // warpgroup g writes columns 32 g .. 32 g + 31 of dQ; ab: dQ = scale (A - delta B)
            float* dQ = static_cast<float*>(a.dQ) + ((size_t)bh * a.n + row) * D + 32 * g;
            if (ok && T > 0) {
                tc_fence_after();
                __syncwarp();
                uint32_t qq[32];
                tmem_ld32(lane_base + 384u + 32u * g, qq);
                tmem_ld_wait();
                if (ab) {
                    uint32_t qb[32];
                    tmem_ld32(lane_base + 448u + 32u * g, qb);
                    tmem_ld_wait();
                    const float db = dlx * sc.ds;
#pragma unroll
                    for (int q = 0; q < 32; ++q)
                        qq[q] = __float_as_uint(fmaf(-db, __uint_as_float(qb[q]), __uint_as_float(qq[q])));
                }
                if (qvalid) {
#pragma unroll
                    for (int q = 0; q < 32; q += 4)
                        *reinterpret_cast<float4*>(dQ + q) =
                            make_float4(sc.dq * __uint_as_float(qq[q]), sc.dq * __uint_as_float(qq[q + 1]),
                                        sc.dq * __uint_as_float(qq[q + 2]), sc.dq * __uint_as_float(qq[q + 3]));
                }
                tc_fence_before();
            } else if (ok && qvalid) {
                for (int c = 0; c < 32; c += 4) *reinterpret_cast<float4*>(dQ + c) = make_float4(0.f, 0.f, 0.f, 0.f);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

template <int KIND>
cudaError_t launch_h_t(const BwdArgs& a, float* delta_pad, float* stat_pad, cudaStream_t stream) {
    cudaError_t e;
    const int BH = a.B * a.H;
    CUtensorMap tq128, tdo128, tk128, tv128, tq64, tdo64, tk64, tv64;
    if ((e = make_tmap_f16(&tq128, a.Qh, BH, a.n, D, TM)) != cudaSuccess) return e;
    if ((e = make_tmap_f16(&tdo128, a.dOh, BH, a.n, D, TM)) != cudaSuccess) return e;
    if ((e = make_tmap_f16(&tk128, a.Kh, BH, a.n, D, TM)) != cudaSuccess) return e;
    if ((e = make_tmap_f16(&tv128, a.Vh, BH, a.n, D, TM)) != cudaSuccess) return e;
    if ((e = make_tmap_f16(&tq64, a.Qh, BH, a.n, D, TB)) != cudaSuccess) return e;
    if ((e = make_tmap_f16(&tdo64, a.dOh, BH, a.n, D, TB)) != cudaSuccess) return e;
    if ((e = make_tmap_f16(&tk64, a.Kh, BH, a.n, D, TB)) != cudaSuccess) return e;
    if ((e = make_tmap_f16(&tv64, a.Vh, BH, a.n, D, TB)) != cudaSuccess) return e;
    const int ntiles = (a.n + TM - 1) / TM;
    // dQ first: it writes the exact delta of every row (entmax), which the dK / dV kernel then reads. In entmax
    // mode a delta pass of the same kernel runs before it; it does work only for keys of more than unit scale.
    {
        const size_t bytes = 1024 + qOffBar + sizeof(Bars) + 2 * TM * sizeof(float) + (size_t)a.nw * 4;
        if (bytes > 232448) return cudaErrorInvalidConfiguration;
        using Kern = void (*)(CUtensorMap, CUtensorMap, CUtensorMap, CUtensorMap, BwdArgs, float*, const float*);
        Kern kerns[3];
        int nk = 0;
        if (KIND != kSoftmaxH) {
            kerns[nk++] = bwd_h_dq_kernel<KIND, (KIND != kSoftmaxH ? kDqAB : kDqPlain)>;
            kerns[nk++] = bwd_h_dq_kernel<KIND, (KIND != kSoftmaxH ? kDqDelta : kDqPlain)>;
        }
        kerns[nk++] = bwd_h_dq_kernel<KIND, kDqPlain>;
        for (int i = 0; i < nk; ++i) {
            if ((e = cudaFuncSetAttribute(kerns[i], cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes)) !=
                cudaSuccess)
                return e;
            launch_mark(stream);
            kerns[i]<<<dim3(BH, ntiles), kThreads, bytes, stream>>>(tq128, tk64, tv64, tdo128, a, delta_pad,
                                                                     stat_pad);
            if ((e = cudaGetLastError()) != cudaSuccess) return e;
        }
    }
    {
        const size_t bytes = 1024 + kvOffBar + sizeof(Bars) + (size_t)a.nwq * 4;
        if (bytes > 232448) return cudaErrorInvalidConfiguration;
        auto kern = bwd_h_dkdv_kernel<KIND>;
        if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes)) != cudaSuccess)
            return e;
        launch_mark(stream);
        kern<<<dim3(BH, ntiles), kThreads, bytes, stream>>>(tq64, tk128, tv128, tdo64, a, delta_pad, stat_pad);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace

cudaError_t launch_bwd_h(const BwdArgs& a, float* delta_pad, float* stat_pad, cudaStream_t stream) {
    if (a.d != 64 || (!a.softmax && (!a.mask || !a.maskT))) return cudaErrorInvalidValue;
    cudaError_t e = launch_bwd_pre(a, delta_pad, stat_pad, stream);
    if (e != cudaSuccess) return e;
    if (a.softmax) return launch_h_t<kSoftmaxH>(a, delta_pad, stat_pad, stream);
    if (a.kind == kAlpha15) return launch_h_t<kAlpha15>(a, delta_pad, stat_pad, stream);
    if (a.kind == kAlpha2) return launch_h_t<kAlpha2>(a, delta_pad, stat_pad, stream);
    return launch_h_t<kGeneric>(a, delta_pad, stat_pad, stream);
}

}  // namespace eattn
