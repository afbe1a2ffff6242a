// softmax_fwd.cu - dense softmax flash-attention forward with the same tiling as the entmax kernels:
// the in-library baseline that the sparse path is measured against ("faster than FlashAttention-2
// above ~60% block sparsity": AdaSplash-2, gist.science (de), section 4 "Ergebnisse").
//
// One CTA per (b, h, 128-row query tile), 192 threads: warps 0-3 compute (thread = query row = TMEM
// lane), warp 4 MMA issue, warp 5 TMA issue. One sweep over the causal key blocks of 64: S = Q K^T in
// TMEM (double buffer), online softmax in base 2 with a lazy running max (O in TMEM is rescaled only
// when a row max grows by more than 2^8), P (bf16) to shared memory, O += P V in TMEM. Writes O (bf16)
// and lse (natural log) for the backward.
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>

#include "common.cuh"
#include "launch.h"

namespace eattn {
namespace {

// K-major operands (128-byte rows, 8-row groups 1024 bytes apart) and MN-major operands stored as
// 64-column boxes of 64 rows (next 64 columns 8 KB further; next 8 rows 1024 bytes further)
constexpr uint64_t kDescK = sdesc_sw128_fields(16, 1024);
constexpr uint64_t kDescMN = sdesc_sw128_fields(64 * 128, 1024);

constexpr int BM = 128, BN = 64, kThreads = 192, NST = 3;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescale = 8.0f;  // log2 headroom before O is rescaled

template <int D>
struct CfgS {
    static constexpr uint32_t kQBytes = BM * D * 2;
    static constexpr uint32_t kBlk = BN * D * 2;
    static constexpr uint32_t kStage = 2 * kBlk;  // K_J, V_J
    static constexpr uint32_t kPBytes = BM * BN * 2;
    static constexpr uint32_t offQ = 0;
    static constexpr uint32_t offSt = kQBytes;
    static constexpr uint32_t offP = offSt + NST * kStage;
    static constexpr uint32_t offBar = offP + 2 * kPBytes;
    static constexpr uint32_t colO = 128;
};

struct BarsS {
    uint64_t q_full;
    uint64_t kv_full[NST], kv_empty[NST];
    uint64_t s_full[2], s_empty[2];
    uint64_t p_full[2], p_empty[2];
    uint64_t pv_done[2], o_full, drain;  // pv_done[j & 1]: P V of block j has completed
    uint32_t tmem_base;
    int abort_flag;
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    softmax_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const SoftmaxFwdArgs a) {
    using C = CfgS<D>;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char* smem = align_smem_1024(smem_raw);
    BarsS& bb = *reinterpret_cast<BarsS*>(smem + C::offBar);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int qt = a.ntiles - 1 - (int)blockIdx.y;  // grid (B*H, tiles): longest tiles of every head first
    const int bh = blockIdx.x;
    const int row0 = qt * BM;
    const int kend = a.causal ? min(a.n, row0 + BM) : a.n;
    const int nblk = (kend + BN - 1) / BN;
    volatile int* abort_flag = &bb.abort_flag;

    if (tid == 0) {
        mbar_init(&bb.q_full, 1);
        for (int i = 0; i < NST; ++i) { mbar_init(&bb.kv_full[i], 1); mbar_init(&bb.kv_empty[i], 1); }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&bb.s_full[i], 1); mbar_init(&bb.s_empty[i], BM);
            mbar_init(&bb.p_full[i], BM); mbar_init(&bb.p_empty[i], 1);
        }
        mbar_init(&bb.pv_done[0], 1);
        mbar_init(&bb.pv_done[1], 1);
        mbar_init(&bb.o_full, 1);
        mbar_init(&bb.drain, 1);
        bb.abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 0) {
        tmem_alloc(&bb.tmem_base, 256);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bb.tmem_base;
    const uint32_t sQ = smem_u32(smem + C::offQ);
    const uint32_t sSt = smem_u32(smem + C::offSt);
    const uint32_t sP = smem_u32(smem + C::offP);

    if (warp == 5) {
        if (lane == 0) {
            tma_prefetch_desc(&tmQ); tma_prefetch_desc(&tmK); tma_prefetch_desc(&tmV);
            mbar_arrive_expect_tx(&bb.q_full, C::kQBytes);
            for (int c = 0; c < D / 64; ++c)
                tma_load_3d(smem + C::offQ + c * (BM * 128), &tmQ, &bb.q_full, 64 * c, row0, bh);
            bool ok = true;
            int J = 0;
            for (; J < nblk && ok; ++J) {
                const int st = J % NST;
                if (!(ok = wait_bounded(&bb.kv_empty[st], ((J / NST) & 1) ^ 1, abort_flag, a.status, true))) break;
                unsigned char* base = smem + C::offSt + st * C::kStage;
                mbar_arrive_expect_tx(&bb.kv_full[st], C::kStage);
                for (int c = 0; c < D / 64; ++c) {
                    tma_load_3d(base + c * (BN * 128), &tmK, &bb.kv_full[st], 64 * c, J * BN, bh);
                    tma_load_3d(base + C::kBlk + c * (BN * 128), &tmV, &bb.kv_full[st], 64 * c, J * BN, bh);
                }
            }
            if (!ok) {
                for (int j = (J > NST ? J - NST : 0); j < J; ++j) wait_drain(&bb.kv_full[j % NST], (j / NST) & 1, 100000000ull);
                wait_drain(&bb.q_full, 0, 100000000ull);
            }
        }
    } else if (warp == 4) {
        if (lane == 0) {
            constexpr uint32_t idS = idesc_bf16_f32(BM, BN, false, false);
            constexpr uint32_t idPV = idesc_bf16_f32(BM, D, false, true);
            bool ok = wait_bounded(&bb.q_full, 0, abort_flag, a.status, true);
            tc_fence_after();
            auto issue_S = [&](int J) -> bool {
                const int st = J % NST, sb = J & 1;
                if (!wait_bounded(&bb.kv_full[st], (J / NST) & 1, abort_flag, a.status, true)) return false;
                if (!wait_bounded(&bb.s_empty[sb], ((J >> 1) & 1) ^ 1, abort_flag, a.status, true)) return false;
                tc_fence_after();
                const uint32_t kb = sSt + st * C::kStage;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t sub = kk >> 2, off = (kk & 3) * 32;
                    mma_ss(tmem + sb * BN, sdesc_at(kDescK, sQ + sub * (BM * 128) + off),
                                sdesc_at(kDescK, kb + sub * (BN * 128) + off), idS, kk > 0);
                }
                mma_commit(&bb.s_full[sb]);
                return true;
            };
            auto issue_PV = [&](int J) -> bool {
                const int st = J % NST, pb = J & 1;
                if (!wait_bounded(&bb.p_full[pb], (J >> 1) & 1, abort_flag, a.status, true)) return false;
                tc_fence_after();
                const uint32_t vb = sSt + st * C::kStage + C::kBlk;
#pragma unroll
                for (int kk = 0; kk < BN / 16; ++kk)
                    mma_ss(tmem + C::colO, sdesc_at(kDescK, sP + pb * C::kPBytes + kk * 32),
                                sdesc_at(kDescMN, vb + kk * 2048), idPV, (J > 0 || kk > 0) ? 1u : 0u);
                mma_commit(&bb.p_empty[pb]);
                mma_commit(&bb.kv_empty[st]);
                mma_commit(&bb.pv_done[J & 1]);
                return true;
            };
            if (ok) ok = issue_S(0);
            for (int J = 0; ok && J < nblk; ++J) {
                if (J + 1 < nblk && !(ok = issue_S(J + 1))) break;
                if (!(ok = issue_PV(J))) break;
            }
            if (ok) mma_commit(&bb.o_full);
            mma_commit(&bb.drain);
            wait_drain(&bb.drain, 0, 200000000ull);
        }
    } else {
        const int r = tid;
        const int row = row0 + r;
        const bool valid = row < a.n;
        const uint32_t lane_base = tmem + ((uint32_t)(warp * 32) << 16);
        const float c2 = a.scale * kLog2e;
        float m_used = -INFINITY, l = 0.f;
        bool ok = true;
        float sv[BN];
        for (int J = 0; J < nblk && ok; ++J) {
            const int sb = J & 1;
            ok = __all_sync(0xffffffffu, wait_bounded(&bb.s_full[sb], (J >> 1) & 1, abort_flag, a.status));
            if (!ok) break;
            tc_fence_after();
            __syncwarp();
            tmem_ld32(lane_base + sb * BN, reinterpret_cast<uint32_t*>(sv));
            tmem_ld32(lane_base + sb * BN + 32, reinterpret_cast<uint32_t*>(sv) + 32);
            tmem_ld_wait();
            tc_fence_before();
            mbar_arrive(&bb.s_empty[sb]);
            const int j0 = J * BN;
            const bool full = valid && j0 + BN <= a.n && (!a.causal || j0 + BN - 1 <= row0);
            float bm = -INFINITY;
#pragma unroll
            for (int c = 0; c < BN; ++c) {
                const int kj = j0 + c;
                const bool okc = full || (valid && kj < a.n && (!a.causal || kj <= row));
                sv[c] = okc ? sv[c] * c2 : -INFINITY;
                bm = fmaxf(bm, sv[c]);
            }
            // lazy rescale: only when the max grows past the headroom
            const bool resc = bm > m_used + kRescale;
            if (__any_sync(0xffffffffu, resc)) {
                const float m_new = resc ? bm : m_used;
                const float f = (resc && m_used != -INFINITY) ? exp2f(m_used - m_new) : 1.f;
                if (J > 0 && __any_sync(0xffffffffu, f != 1.f)) {
                    // O holds P V of blocks < J: wait for P V (J-1) (MMAs complete in issue order), then
                    // scale this warp's rows. Each pv_done barrier is at most one phase behind here.
                    ok = __all_sync(0xffffffffu, wait_bounded(&bb.pv_done[(J - 1) & 1], ((J - 1) >> 1) & 1,
                                                              abort_flag, a.status));
                    if (!ok) break;
                    tc_fence_after();
#pragma unroll
                    for (int c0 = 0; c0 < D; c0 += 32) {
                        uint32_t o[32];
                        tmem_ld32(lane_base + C::colO + c0, o);
                        tmem_ld_wait();
#pragma unroll
                        for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * f);
                        tmem_st32(lane_base + C::colO + c0, o);
                    }
                    tmem_st_wait();
                }
                l *= f;
                m_used = m_new;
            }
            const int pb = J & 1;
            ok = __all_sync(0xffffffffu, wait_bounded(&bb.p_empty[pb], ((J >> 1) & 1) ^ 1, abort_flag, a.status));
            if (!ok) break;
            const uint32_t pbase = sP + pb * C::kPBytes;
#pragma unroll
            for (int g = 0; g < 8; ++g) {
                float p[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    p[e] = (m_used == -INFINITY) ? 0.f : exp2f(sv[8 * g + e] - m_used);
                    l += p[e];
                }
                st_shared_v4(pbase + sw128_offset((uint32_t)r, (uint32_t)g), pack_bf16x2(p[0], p[1]),
                             pack_bf16x2(p[2], p[3]), pack_bf16x2(p[4], p[5]), pack_bf16x2(p[6], p[7]));
            }
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(&bb.p_full[pb]);
        }
        if (ok) ok = __all_sync(0xffffffffu, wait_bounded(&bb.o_full, 0, abort_flag, a.status));
        if (ok) {
            tc_fence_after();
            __syncwarp();
            const float inv = l > 0.f ? 1.f / l : 0.f;
            __nv_bfloat16* Oh = static_cast<__nv_bfloat16*>(a.O) + ((size_t)bh * a.n + row) * D;
#pragma unroll
            for (int c0 = 0; c0 < D; c0 += 32) {
                uint32_t o[32];
                tmem_ld32(lane_base + C::colO + c0, o);
                tmem_ld_wait();
                if (valid) {
                    uint4* dst = reinterpret_cast<uint4*>(Oh + c0);
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const float* f = reinterpret_cast<const float*>(o + 8 * i);
                        dst[i] = make_uint4(pack_bf16x2(f[0] * inv, f[1] * inv), pack_bf16x2(f[2] * inv, f[3] * inv),
                                            pack_bf16x2(f[4] * inv, f[5] * inv), pack_bf16x2(f[6] * inv, f[7] * inv));
                    }
                }
            }
            tc_fence_before();
            if (valid) a.lse[(size_t)bh * a.n + row] = (m_used + log2f(l)) * kLn2;
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 256);
    }
}

template <int D>
cudaError_t launch_t(const SoftmaxFwdArgs& a, cudaStream_t stream) {
    using C = CfgS<D>;
    CUtensorMap tq, tk, tv;
    cudaError_t e;
    const int BH = a.B * a.H;
    if ((e = make_tmap_bf16(&tq, a.Q, BH, a.n, D, BM)) != cudaSuccess) return e;
    if ((e = make_tmap_bf16(&tk, a.K, BH, a.n, D, BN)) != cudaSuccess) return e;
    if ((e = make_tmap_bf16(&tv, a.V, BH, a.n, D, BN)) != cudaSuccess) return e;
    const size_t bytes = 1024 + C::offBar + sizeof(BarsS);
    auto kern = softmax_fwd_kernel<D>;
    if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes)) != cudaSuccess)
        return e;
    launch_mark(stream);
    kern<<<dim3(BH, a.ntiles), kThreads, bytes, stream>>>(tq, tk, tv, a);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_softmax_fwd(const SoftmaxFwdArgs& a, cudaStream_t stream) {
    return a.d == 64 ? launch_t<64>(a, stream) : launch_t<128>(a, stream);
}

}  // namespace eattn
