// softmax_fwd_h.cu - dense softmax flash-attention forward (the in-library baseline) for d = 64 on fp16
// copies of Q, K, V (f16.cu), in the structure of the entmax forward (fwd_h.cu).
//
// One CTA per (b, h, 128-row query tile), longest causal tiles first, 352 threads:
//   warps 0-3, 4-7  compute warpgroups 0 and 1 (thread r owns query row r, TMEM lane r); they take
//                   alternate key blocks of 64;
//   warp 8          S issue: S = Q K^T (shared-memory operands) into two TMEM buffers per warpgroup;
//   warp 10         P V issue: O_g += P V, P (fp16) written by warpgroup g over the S tile it came from;
//   warp 9          TMA: Q once, then K and V blocks into rings.
// Each warpgroup keeps its own running max m_g and sum l_g per row (base 2) and its own accumulator O_g
// in TMEM. O_g is rescaled lazily: only when m_g grows by more than 2^8 (so P <= 2^8 stays in fp16
// range), after the P V product of the warpgroup's previous block completed. At the end the two partial
// results are merged through shared memory:
//   O = (2^(m_0 - m) O_0 + 2^(m_1 - m) O_1) / (2^(m_0 - m) l_0 + 2^(m_1 - m) l_1),  m = max(m_0, m_1),
//   lse = ln 2 (m + log2 l).
// TMEM columns: S buffer b of warpgroup g at 64 (2 g + b) (P in its first 32), O_g at 256 + 64 g.
// A new S tile enters a buffer only after the P V product that read its P completed. A K ring slot is
// released by the four warps that read the S tile it fed (one commit per tile in the S thread).
// ("faster than FlashAttention-2 above ~60% block sparsity": AdaSplash-2, gist.science (de), section 4.)
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <math.h>

#include "common.cuh"
#include "launch.h"

namespace eattn {
namespace {

constexpr int BM = 128;
constexpr int BN = 64;
constexpr int D = 64;
constexpr int kThreads = 352;
constexpr int kCompute = 256;
constexpr int NKS = 4;
constexpr int NVS = 8;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescale = 8.0f;  // log2 headroom before O_g is rescaled

constexpr uint64_t kDescK = sdesc_sw128_fields(16, 1024);
constexpr uint64_t kDescMN = sdesc_sw128_fields(64 * 128, 1024);

constexpr uint32_t kQBytes = BM * D * 2;
constexpr uint32_t kKBytes = BN * D * 2;
constexpr uint32_t offQ = 0;
constexpr uint32_t offK = offQ + kQBytes;
constexpr uint32_t offV = offK + NKS * kKBytes;
constexpr uint32_t offX = offV + NVS * kKBytes;       // merge: O_1 [64][128] fp32, then m_1, l_1 [128]
constexpr uint32_t offBar = offX + (D + 2) * BM * 4;
constexpr uint32_t kColO = 256;

struct Bars {
    uint64_t q_full;
    uint64_t k_full[NKS], k_empty[NKS];
    uint64_t v_full[NVS], v_empty[NVS];
    uint64_t s_full[2][2], s_empty[2][2];
    uint64_t p_full[2][2], pv_free[2][2];
    uint64_t o_done;
    uint64_t drain[2];
    uint32_t tmem_base;
    int abort_flag;
};

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

__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

__global__ void __launch_bounds__(kThreads, 1)
    softmax_fwd_h_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                         const __grid_constant__ CUtensorMap tmV, const SoftmaxFwdArgs a) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char* smem = align_smem_1024(smem_raw);
    Bars& bb = *reinterpret_cast<Bars*>(smem + offBar);
    float* xo = reinterpret_cast<float*>(smem + offX);  // [64][128]
    float* xm = xo + D * BM;                             // [128]
    float* xl = xm + BM;                                 // [128]

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int qt = a.ntiles - 1 - (int)blockIdx.y;  // grid (B*H, tiles): longest tiles of every head first
    const int bh = blockIdx.x;
    const int row0 = qt * BM;
    const int kend = a.causal ? min(a.n, row0 + BM) : a.n;
    const int T = (kend + BN - 1) / BN;  // key blocks of this tile
    volatile int* abort_flag = &bb.abort_flag;

    if (tid == 0) {
        mbar_init(&bb.q_full, 1);
        for (int i = 0; i < NKS; ++i) { mbar_init(&bb.k_full[i], 1); mbar_init(&bb.k_empty[i], 4); }
        for (int i = 0; i < NVS; ++i) { mbar_init(&bb.v_full[i], 1); mbar_init(&bb.v_empty[i], 1); }
        for (int g = 0; g < 2; ++g)
            for (int b = 0; b < 2; ++b) {
                mbar_init(&bb.s_full[g][b], 1);
                mbar_init(&bb.s_empty[g][b], 4);
                mbar_init(&bb.p_full[g][b], 4);
                mbar_init(&bb.pv_free[g][b], 1);
            }
        mbar_init(&bb.o_done, 1);
        mbar_init(&bb.drain[0], 1);
        mbar_init(&bb.drain[1], 1);
        bb.abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 0) {
        tmem_alloc(&bb.tmem_base, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bb.tmem_base;
    const uint32_t sQ = smem_u32(smem + offQ);
    const uint32_t sK0 = smem_u32(smem + offK);
    const uint32_t sV0 = smem_u32(smem + offV);

    if (warp == 9) {
        // ------------------------------------------------------------------ TMA issue
        if (lane == 0) {
            tma_prefetch_desc(&tmQ); tma_prefetch_desc(&tmK); tma_prefetch_desc(&tmV);
            mbar_arrive_expect_tx(&bb.q_full, kQBytes);
            tma_load_3d(smem + offQ, &tmQ, &bb.q_full, 0, row0, bh);
            uint32_t i = 0;
            bool ok = true;
            for (int J = 0; J < T && ok; ++J, ++i) {
                const uint32_t ks = i % NKS, vs = i % NVS;
                if (!(ok = wait_bounded(&bb.k_empty[ks], ((i / NKS) & 1) ^ 1, abort_flag, a.status, true))) break;
                mbar_arrive_expect_tx(&bb.k_full[ks], kKBytes);
                tma_load_3d(smem + offK + ks * kKBytes, &tmK, &bb.k_full[ks], 0, J * BN, bh);
                if (!(ok = wait_bounded(&bb.v_empty[vs], ((i / NVS) & 1) ^ 1, abort_flag, a.status, true))) break;
                mbar_arrive_expect_tx(&bb.v_full[vs], kKBytes);
                tma_load_3d(smem + offV + vs * kKBytes, &tmV, &bb.v_full[vs], 0, J * BN, bh);
            }
            if (!ok) {
                for (uint32_t k = (i > (uint32_t)NKS ? i - NKS : 0); k <= i && k < (uint32_t)T; ++k)
                    wait_drain(&bb.k_full[k % NKS], (k / NKS) & 1, 100000000ull);
                for (uint32_t k = (i > (uint32_t)NVS ? i - NVS : 0); k <= i && k < (uint32_t)T; ++k)
                    wait_drain(&bb.v_full[k % NVS], (k / NVS) & 1, 100000000ull);
                wait_drain(&bb.q_full, 0, 100000000ull);
            }
        }
    } else if (warp == 8) {
        // ------------------------------------------------------------------ S issue
        if (lane == 0) {
            constexpr uint32_t idS = idesc_f16_f32(BM, BN, false, false);
            uint32_t ppar = 0xfu;  // per buffer: parity of the commit of its last P V (bits start at 1)
            bool ok = wait_bounded(&bb.q_full, 0, abort_flag, a.status, true);
            tc_fence_after();
            for (int t = 0; t < T && ok; ++t) {
                const int g = t & 1;
                const uint32_t sn = (uint32_t)(t >> 1), b = sn & 1u, bi = 2u * g + b;
                const uint32_t ks = (uint32_t)t % NKS;
                if (!(ok = wait_bounded(&bb.k_full[ks], ((uint32_t)t / NKS) & 1, abort_flag, a.status, true))) break;
                if (!(ok = wait_bounded(&bb.s_empty[g][b], ((sn >> 1) & 1) ^ 1, abort_flag, a.status, true))) break;
                // the buffer held block t - 4 (same warpgroup and buffer): its P V must have completed
                if (t >= 4 && !(ok = wait_bounded(&bb.pv_free[g][b], (ppar >> bi) & 1u, abort_flag, a.status, true))) break;
                ppar ^= 1u << bi;
                tc_fence_after();
                const uint32_t kbase = sK0 + ks * kKBytes;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk)
                    mma_ss(tmem + 64u * bi, sdesc_at(kDescK, sQ + kk * 32), sdesc_at(kDescK, kbase + kk * 32), idS,
                           kk > 0 ? 1u : 0u);
                mma_commit(&bb.s_full[g][b]);
            }
            mma_commit(&bb.drain[0]);
            wait_drain(&bb.drain[0], 0, 200000000ull);
        }
    } else if (warp == 10) {
        // ------------------------------------------------------------------ P V issue
        if (lane == 0) {
            constexpr uint32_t idPV = idesc_f16_f32(BM, D, false, true);
            uint32_t ppar = 0xfu;
            bool ok = true;
            for (int t = 0; t < T && ok; ++t) {
                const int g = t & 1;
                const uint32_t sn = (uint32_t)(t >> 1), b = sn & 1u, bi = 2u * g + b;
                const uint32_t vs = (uint32_t)t % NVS;
                if (!(ok = wait_bounded(&bb.p_full[g][b], ((ppar >> bi) & 1u) ^ 1u, abort_flag, a.status, true))) break;
                if (!(ok = wait_bounded(&bb.v_full[vs], ((uint32_t)t / NVS) & 1, abort_flag, a.status, true))) break;
                tc_fence_after();
                const uint32_t vbase = sV0 + vs * kKBytes;
#pragma unroll
                for (int kk = 0; kk < BN / 16; ++kk)
                    mma_ts(tmem + kColO + 64u * g, tmem + 64u * bi + 8 * kk, sdesc_at(kDescMN, vbase + kk * 2048),
                           idPV, (sn == 0 && kk == 0) ? 0u : 1u);
                mma_commit(&bb.pv_free[g][b]);
                mma_commit(&bb.v_empty[vs]);
                ppar ^= 1u << bi;
            }
            if (ok) mma_commit(&bb.o_done);
            mma_commit(&bb.drain[1]);
            wait_drain(&bb.drain[1], 0, 200000000ull);
        }
    } else if (warp < 8) {
        // ------------------------------------------------------------------ compute warpgroups
        const int g = warp >> 2;
        const int r = tid & (BM - 1);
        const int row = row0 + r;
        const bool valid = row < a.n;
        const uint32_t lane_base = tmem + ((uint32_t)((warp & 3) * 32) << 16);
        const int eqk = f16_range_exp(a.maxbits[0]) + f16_range_exp(a.maxbits[1]);
        const float vscale = ldexpf(1.0f, f16_range_exp(a.maxbits[2]));
        const float c2 = ldexpf(a.scale * 1.4426950408889634f, eqk);  // raw fp16 score -> log2 units
        float m_run = -INFINITY, l = 0.f;
        bool ok = true;
        for (int t = g; t < T && ok; t += 2) {
            const uint32_t j = (uint32_t)(t >> 1), b = j & 1u, bi = 2u * g + b;
            ok = __all_sync(0xffffffffu, wait_bounded(&bb.s_full[g][b], (j >> 1) & 1, abort_flag, a.status));
            if (!ok) break;
            tc_fence_after();
            __syncwarp();
            float x[BN];
            tmem_ld32(lane_base + 64u * bi, reinterpret_cast<uint32_t*>(x));
            tmem_ld32(lane_base + 64u * bi + 32, reinterpret_cast<uint32_t*>(x) + 32);
            tmem_ld_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&bb.s_empty[g][b]);
                mbar_arrive(&bb.k_empty[(uint32_t)t % NKS]);  // the MMA that read K block t has completed
            }
            const int k0 = t * BN;
            const bool full = valid && k0 + BN <= a.n && (!a.causal || k0 + BN - 1 <= row0);
            if (__any_sync(0xffffffffu, !full)) {
#pragma unroll
                for (int c = 0; c < BN; ++c) {
                    const int key = k0 + c;
                    if (!(valid && key < a.n && (!a.causal || key <= row))) x[c] = -INFINITY;
                }
            }
            float mb = -INFINITY;
#pragma unroll
            for (int c = 0; c < BN; c += 4) {
#pragma unroll
                for (int e = 0; e < 4; ++e) x[c + e] *= c2;
                mb = fmax3(mb, fmaxf(x[c], x[c + 1]), fmaxf(x[c + 2], x[c + 3]));
            }
            // lazy rescale: only when the row max grows by more than 2^8 over the one P is relative to
            const bool grow = mb > m_run + kRescale || (m_run == -INFINITY && mb > -INFINITY);
            const float m_new = grow ? mb : m_run;
            const float fac = (grow && m_run > -INFINITY) ? exp2f(m_run - m_new) : 1.0f;
            if (__any_sync(0xffffffffu, grow && m_run > -INFINITY && j > 0)) {
                // O_g holds the P V of this warpgroup's earlier blocks: wait for the last one (block j - 1,
                // the other buffer; block j - 2's completed before this S tile was issued), then rescale
                ok = __all_sync(0xffffffffu, wait_bounded(&bb.pv_free[g][b ^ 1u], ((j - 1) >> 1) & 1, abort_flag,
                                                          a.status));
                if (!ok) break;
                tc_fence_after();
                __syncwarp();
#pragma unroll
                for (int c0 = 0; c0 < D; c0 += 32) {
                    uint32_t o[32];
                    tmem_ld32(lane_base + kColO + 64u * g + c0, o);
                    tmem_ld_wait();
#pragma unroll
                    for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * fac);
                    tmem_st32(lane_base + kColO + 64u * g + c0, o);
                }
                tmem_st_wait();
            }
            l *= fac;
            m_run = m_new;
            const float mu = m_run > -INFINITY ? m_run : 0.0f;
            uint32_t w32[32];
#pragma unroll
            for (int c = 0; c < BN; c += 2) {
                const float p0 = exp2f(x[c] - mu), p1 = exp2f(x[c + 1] - mu);
                l += p0 + p1;
                w32[c / 2] = pack_half2(p0, p1);
            }
            tmem_st32(lane_base + 64u * bi, w32);
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bb.p_full[g][b]);
        }
        ok = !bar_or256(!ok || *abort_flag != 0);
        if (ok && T > 0) ok = __all_sync(0xffffffffu, wait_bounded(&bb.o_done, 0, abort_flag, a.status));
        ok = !bar_or256(!ok || *abort_flag != 0);
        // ---- merge the two warpgroups' partial results ----
        const bool has = g < T;  // this warpgroup processed at least one block
        uint32_t o[64];
        if (ok && has) {
            tc_fence_after();
            __syncwarp();
            tmem_ld32(lane_base + kColO + 64u * g, o);
            tmem_ld32(lane_base + kColO + 64u * g + 32, o + 32);
            tmem_ld_wait();
        }
        if (g == 1) {
            xm[r] = m_run;
            xl[r] = l;
            if (has)
                for (int c = 0; c < D; ++c) xo[c * BM + r] = __uint_as_float(o[c]);
        }
        named_bar_sync(1, kCompute);
        if (g == 0 && ok && valid) {
            const float m1 = xm[r], l1 = xl[r];
            const bool has1 = T > 1;
            const float M = fmaxf(m_run, has1 ? m1 : -INFINITY);
            const float w0 = m_run > -INFINITY ? exp2f(m_run - M) : 0.0f;
            const float w1 = (has1 && m1 > -INFINITY) ? exp2f(m1 - M) : 0.0f;
            const float L = w0 * l + w1 * l1;
            const float inv = vscale / L;
            __nv_bfloat16* Oh = static_cast<__nv_bfloat16*>(a.O) + ((size_t)bh * a.n + row) * D;
#pragma unroll
            for (int c = 0; c < D; c += 8) {
                float v[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const float o1 = w1 != 0.0f ? xo[(c + e) * BM + r] : 0.0f;
                    v[e] = (w0 * __uint_as_float(o[c + e]) + w1 * o1) * inv;
                }
                *reinterpret_cast<uint4*>(Oh + c) = make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]),
                                                               pack_bf16x2(v[4], v[5]), pack_bf16x2(v[6], v[7]));
            }
            a.lse[(size_t)bh * a.n + row] = kLn2 * (M + __log2f(L));
        }
        tc_fence_before();
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

}  // namespace

cudaError_t launch_softmax_fwd_h(const SoftmaxFwdArgs& a, cudaStream_t stream) {
    if (a.d != D || !a.Qh || !a.Kh || !a.Vh || !a.maxbits) return cudaErrorInvalidValue;
    CUtensorMap tq, tk, tv;
    cudaError_t e;
    if ((e = make_tmap_f16(&tq, a.Qh, a.B * a.H, a.n, D, BM)) != cudaSuccess) return e;
    if ((e = make_tmap_f16(&tk, a.Kh, a.B * a.H, a.n, D, BN)) != cudaSuccess) return e;
    if ((e = make_tmap_f16(&tv, a.Vh, a.B * a.H, a.n, D, BN)) != cudaSuccess) return e;
    const size_t bytes = 1024 + offBar + sizeof(Bars);
    if ((e = cudaFuncSetAttribute(softmax_fwd_h_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes)) !=
        cudaSuccess)
        return e;
    dim3 grid(a.B * a.H, a.ntiles);
    launch_mark(stream);
    softmax_fwd_h_kernel<<<grid, kThreads, bytes, stream>>>(tq, tk, tv, a);
    return cudaGetLastError();
}

}  // namespace eattn
