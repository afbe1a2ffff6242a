// fwd_h.cu - alpha-entmax attention forward for alpha <= 2 and d = 64 on the sm_100a tensor cores, from
// fp16 copies of Q, K, V (f16.cu).
//
// One CTA per (b, h, 128-row query tile), 352 threads:
//   warps 0-3, 4-7  compute warpgroups 0 and 1. Thread r of a warpgroup owns query row r of the tile
//                   and reads TMEM lane r; the two warpgroups take alternate key blocks of every sweep;
//   warp 8          S issue (one thread): S = Q K^T from shared memory into three TMEM buffers per
//                   warpgroup;
//   warp 10         P V issue (one thread): O_g += P V with P stored by the compute warps into the TMEM
//                   columns of the S tile it came from, into one accumulator per warpgroup (consecutive
//                   products then never feed one another). Two issuing threads keep the tensor pipe fed:
//                   each waits only on its own barriers, in block order;
//   warp 9          TMA issue (one thread): Q once, K blocks of 64 keys and, in P V sweeps, V blocks.
// A K ring slot is released by the four warps that read the S tile it fed (once they see that S tile
// complete, the MMA that read the slot has completed too), so that the S thread commits once per tile:
// each tcgen05.commit costs the issuing thread tens of cycles.
//
// P lies in [0, 1] for alpha <= 2 and enters P V as one fp16 term (11 significant bits; bf16 would need a
// two-term split). The backward needs no product of u with V from the forward: its dQ kernel forms
// delta = sum u g / sum u itself (bwd_h.cu), so this kernel writes only O, tau, sum u and the mask. P of a
// 64-key block fits the first 32 columns of its S tile. A new S tile goes into a buffer only after the P V
// products that read its previous P have completed (a commit barrier per buffer), and the MMA thread waits
// for all P V products at the end of a P V sweep: MMAs into different accumulators are not ordered by issue
// alone.
//
// TMEM columns (512): S buffer b (of three) of warpgroup g at 64 (3 g + b), holding P in its first 32
// columns (K step kk of 16 keys is columns 8 kk .. 8 kk + 7) in P V sweeps; O_0 at 384, O_1 at 448 (their
// sum is O).
//
// Sweeps follow the plan protocol of the bf16 forward (fwd_tc.cu): before each sweep the compute warps
// publish its kind and its set of key blocks, which the issuing warps follow.
//   dense   - every causal key block: running max and the candidate stash (entries above max - 1); the
//             stash of a row has one half per warpgroup. When the sweep ends both warpgroups bin their
//             halves into the row's histogram (window at the final max), and warpgroup 0 takes tau_h and
//             solves tau on chip from the stash.
//   hist    - only when some row's stash half overflowed: candidate blocks, all on warpgroup 0, which
//             bins those rows' entries into their histograms with the window fixed by the final max;
//   refine  - candidate blocks: solver sums at the current tau (partial sums of the two warpgroups are
//             combined by warpgroup 0, which owns the solver state of each row);
//   P V     - candidate blocks: p to TMEM for the P V MMAs, exact block mask, sum check;
//   support - instead of P V, when every row of the tile was solved on chip from its stash and has at most
//             kElemCap support entries per warpgroup: candidate blocks, S recomputed only to find the
//             support (exact block mask); each warpgroup lists the (key, p) of its blocks' support entries
//             in shared memory, and O = sum p v is then gathered from those rows of V in fp32 (element
//             sparsity: no P V MMAs and no V ring).
// (AdaSplash-2, gist.science (de), section 2: histogram initialisation, hybrid solver, bit-packed block
// mask, only nonzero blocks processed.)
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <math.h>

#include <type_traits>

#include "common.cuh"
#include "fwd_common.cuh"
#include "launch.h"

namespace eattn {
namespace {

constexpr int BM = 128;
constexpr int BN = 64;
constexpr int D = 64;
constexpr int kThreads = 352;
constexpr int kCompute = 256;
constexpr int NKS_MAX = 8;  // K ring stages, at most
constexpr int NVS = 8;
constexpr int NSB = 3;  // S buffers per compute warpgroup

constexpr uint64_t kDescK = sdesc_sw128_fields(16, 1024);
constexpr uint64_t kDescMN = sdesc_sw128_fields(64 * 128, 1024);

constexpr uint32_t kKBytes = BN * D * 2;                 // 8 KB per K or V block
constexpr uint32_t kQBytes = BM * D * 2;                 // 16 KB
constexpr uint32_t offQ = 0;
constexpr uint32_t offK = offQ + kQBytes;

// Shared-memory plan for up to NB histogram bins (256, or 512): the histogram u16 [NB][128] (the V ring of
// P V sweeps reuses it), then the candidate stash fp32 [2][kHalf][128]. At 512 bins the histogram takes
// 128 KB and the stash shrinks to 32 entries per row and warpgroup, so that the CTA still fits. The
// histogram sweep of an overflowed row stages a whole 64-key block in that row's stash slots, from the
// start of warpgroup 0's half: the two halves together must hold 64 entries.
template <int NB>
struct HCfg {
    static constexpr int kNKS = 4;                     // K ring stages
    static constexpr int kHalf = NB == 512 ? 32 : 88;  // stash entries per row and warpgroup
    static constexpr uint32_t offHist = offK + kNKS * kKBytes;
    static_assert(kNKS <= NKS_MAX, "K ring barriers");
    static_assert(2 * kHalf >= BN, "the histogram sweep stages a 64-key block in a row's stash slots");
    static constexpr uint32_t kHistBytes = (uint32_t)NB * BM * 2u;
    static constexpr uint32_t kStashBytes = 2u * kHalf * BM * 4u;
    static constexpr uint32_t offStash = offHist + kHistBytes;
    static constexpr uint32_t offV = offHist;
    static constexpr uint32_t offSmall = offStash + kStashBytes;
    static constexpr int kStride = NB == 512 ? kLiveStride512 : kLiveStride;  // live words per row + 1
    static_assert(NVS * kKBytes <= kHistBytes, "V ring must fit the histogram region");
    // element path: per row and warpgroup a list of up to kElemCap support entries (key u16, p f32) and its
    // length, in the histogram region once tau is solved
    static constexpr int kElemCap = 40;
    static constexpr uint32_t kElemKeys = 2u * kElemCap * BM * 2u;
    static constexpr uint32_t kElemP = 2u * kElemCap * BM * 4u;
    static_assert(kElemKeys + kElemP + 2u * BM * 4u <= kHistBytes, "support lists must fit the histogram region");
};

constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColO = 384;

// exchange rows of Small::xf
enum : int {
    kXMax0 = 0, kXMax1 = 1,  // running max hints of the two warpgroups
    kXCnt1 = 2,              // warpgroup 1: stash count (int bits), -1 when its half overflowed
    kXTau = 3, kXTau2 = 4, kXLo = 5, kXTwo = 6,  // solver state broadcast by warpgroup 0
    kXF0 = 7, kXF1 = 8, kXF2 = 9, kXF0b = 10,    // partial sums of warpgroup 1
    kXOvf = 11,                                  // 1: the row's candidates did not fit the stash
    kXCnt = 12,                                  // partial support count of warpgroup 1 (int bits)
    kXRows = 13,
    kXCnt0 = kXF0b                               // warpgroup 0: stash count (int bits), -1 when its half
                                                 // overflowed; only between the dense sweep and the solve
};

struct Small {
    uint64_t q_full;
    uint64_t k_full[NKS_MAX], k_empty[NKS_MAX];
    uint64_t v_full[NVS], v_empty[NVS];
    uint64_t s_full[2][NSB], s_empty[2][NSB];  // [warpgroup][buffer]
    uint64_t pv_free[2][NSB];                  // P V products that read a buffer's P have completed
    uint64_t pu_full[2][NSB];                  // a buffer's P is stored (one barrier per buffer, so
                                           // that no barrier runs two phases ahead of its waiter)
    uint64_t o_full;
    uint64_t ctrl;
    uint64_t drain[2];
    uint32_t tmem_base;
    int abort_flag;
    int plan_kind[2];
    TileStats st;
    float T[516];  // i^k for i = 0 .. bins (generic alpha)
    float xf[kXRows][BM];
    // followed by: plan_bits[2][W], next[W], mrow[2][W], live[128][stride]
};

// OR of `pred` over the 256 compute threads (named barrier 1); every compute thread gets the result.
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

// Drop the entries of a stash half at or below thr. Returns the new count, or -1 (overflow) when more
// than half of the half stays occupied, so that pruning stays amortised O(1) per entry.
static __device__ __noinline__ int stash_prune(int n, float* st, int r, float thr, int half) {
    int j = 0;
    for (int i = 0; i < n; ++i) {
        const float v = st[i * BM + r];
        if (v > thr) st[(j++) * BM + r] = v;
    }
    return j > half / 2 ? -1 : j;
}

// Start row r's histogram with its window top at the bin of the final max m_raw.
__device__ __forceinline__ void hist_start(HistRow& h, float m_raw, const SolveParams& sp) {
    for (int i = 0; i < h.nlw; ++i) h.live[i] = 0u;
    h.any = m_raw > -INFINITY;
    h.m_raw = m_raw;
    h.thr_raw = m_raw - sp.inv_cz;
    h.top = h.any ? bin_of(m_raw, sp.cbin) : 0;
}

// Bin the entries above the threshold of one staged block (rb[c * 128], c < 64; rb points at the row), groups
// of 8 flagged in gflag.
static __device__ __noinline__ void hist_bin_block(HistRow& h, const float* rb, uint32_t gflag, const SolveParams& sp,
                                                   uint16_t* hist, int r) {
    while (gflag) {
        const int q = __ffs(gflag) - 1;
        gflag &= gflag - 1;
        for (int e = 0; e < 8; ++e) {
            const float v = rb[(8 * q + e) * BM];
            if (v > h.thr_raw) hist_add(h, v, sp.cbin, sp.bins, hist, r);
        }
    }
}

// Solver sums over one stash half, added to F0..F0b.
template <int KIND>
__device__ __forceinline__ void half_sums(const float* st, int n, int r, const SolveParams& sp, float tau, float tau2,
                                          bool two, float& F0, float& F1, float& F2, float& F0b) {
    for (int i = 0; i < n; ++i) {
        const float a = st[i * BM + r];
        const float x = fmaf(a, sp.cz, -tau);
        if (x > 0.f) add_sums<KIND>(x, sp.k, F0, F1, F2);
        if (two) {
            const float x2 = fmaf(a, sp.cz, -tau2);
            if (x2 > 0.f) F0b += pow_k<KIND>(x2, sp.k);
        }
    }
}

// Entries of one stash half above tau (z units): the row's support, when every candidate fit the stash.
__device__ __forceinline__ uint32_t half_count(const float* st, int n, int r, float cz, float tau) {
    uint32_t c = 0;
    for (int i = 0; i < n; ++i) c += fmaf(st[i * BM + r], cz, -tau) > 0.f ? 1u : 0u;
    return c;
}

__device__ __forceinline__ bool block_full(int J, int n, int causal, int row0) {
    const int last = J * BN + BN - 1;
    return last < n && (!causal || last <= row0);
}

template <int KIND, int NB>
__global__ void __launch_bounds__(kThreads, 1)
    fwd_h_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                 const __grid_constant__ CUtensorMap tmV, const FwdArgs a) {
    using HC = HCfg<NB>;
    constexpr int NKS = HC::kNKS;
    constexpr uint32_t offHist = HC::offHist;
    constexpr int kHalf = HC::kHalf;
    constexpr uint32_t offStash = HC::offStash;
    constexpr uint32_t offV = HC::offV;
    constexpr uint32_t offSmall = HC::offSmall;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char* smem = align_smem_1024(smem_raw);
    Small& sm = *reinterpret_cast<Small*>(smem + offSmall);
    const int W = a.nw;
    uint32_t* plan_bits = reinterpret_cast<uint32_t*>(&sm + 1);  // [2][W]
    uint32_t* next = plan_bits + 2 * W;                          // [W]
    uint32_t* mrow = next + W;                                   // [2][W]
    uint32_t* live_all = mrow + 2 * W;                           // [128][HC::kStride]
    uint16_t* hist = reinterpret_cast<uint16_t*>(smem + offHist);
    uint16_t* elem_key = reinterpret_cast<uint16_t*>(smem + offHist);                        // [2][cap][128]
    float* elem_p = reinterpret_cast<float*>(smem + offHist + HC::kElemKeys);                   // [2][cap][128]
    int* elem_cnt = reinterpret_cast<int*>(smem + offHist + HC::kElemKeys + HC::kElemP);        // [2][128]
    float* stash = reinterpret_cast<float*>(smem + offStash);

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    // grid (B*H, tiles): the longest causal tiles of every head first
    const int qt = a.ntiles - 1 - (int)blockIdx.y;
    const int bh = blockIdx.x;
    const int row0 = qt * BM;
    const int kend = a.causal ? min(a.n, row0 + BM) : a.n;
    const int nblk = (kend + BN - 1) / BN;
    volatile int* abort_flag = &sm.abort_flag;

    if (tid == 0) {
        mbar_init(&sm.q_full, 1);
        for (int i = 0; i < NKS; ++i) { mbar_init(&sm.k_full[i], 1); mbar_init(&sm.k_empty[i], 4); }
        for (int i = 0; i < NVS; ++i) { mbar_init(&sm.v_full[i], 1); mbar_init(&sm.v_empty[i], 1); }
        for (int i = 0; i < 2; ++i) {
            for (int b = 0; b < NSB; ++b) {
                mbar_init(&sm.s_full[i][b], 1);
                mbar_init(&sm.s_empty[i][b], 4);
                mbar_init(&sm.pv_free[i][b], 1);
                mbar_init(&sm.pu_full[i][b], 4);
            }
        }
        mbar_init(&sm.o_full, 1);
        mbar_init(&sm.ctrl, kCompute / 32);
        mbar_init(&sm.drain[0], 1);
        mbar_init(&sm.drain[1], 1);
        sm.abort_flag = 0;
        sm.st = TileStats{};
        fence_barrier_init();
    }
    if (warp == 0) {
        tmem_alloc(&sm.tmem_base, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    const uint32_t sQ = smem_u32(smem + offQ);
    const uint32_t sK0 = smem_u32(smem + offK);
    const uint32_t sV0 = smem_u32(smem + offV);

    if (warp == 9) {
        // ------------------------------------------------------------------ TMA issue
        if (lane == 0) {
            tma_prefetch_desc(&tmQ);
            tma_prefetch_desc(&tmK);
            tma_prefetch_desc(&tmV);
            mbar_arrive_expect_tx(&sm.q_full, kQBytes);
            tma_load_3d(smem + offQ, &tmQ, &sm.q_full, 0, row0, bh);
            uint32_t lc = 0, vc = 0;
            bool ok = true;
            for (int sw = 0; ok; ++sw) {
                if (!(ok = wait_bounded(&sm.ctrl, sw & 1, abort_flag, a.status, true))) break;
                const int kind = sm.plan_kind[sw & 1];
                if (kind == kSweepDone) break;
                const uint32_t* bits_p = plan_bits + (sw & 1) * W;
                for (int wd = 0; wd < W && ok; ++wd) {
                    uint32_t bits = bits_p[wd];
                    while (bits && ok) {
                        const int J = wd * 32 + __ffs(bits) - 1;
                        bits &= bits - 1;
                        const uint32_t ks = lc % NKS;
                        if (!(ok = wait_bounded(&sm.k_empty[ks], ((lc / NKS) & 1) ^ 1, abort_flag, a.status, true))) break;
                        mbar_arrive_expect_tx(&sm.k_full[ks], kKBytes);
                        tma_load_3d(smem + offK + ks * kKBytes, &tmK, &sm.k_full[ks], 0, J * BN, bh);
                        ++lc;
                        if (kind == kSweepPV) {
                            const uint32_t vs = vc % NVS;
                            if (!(ok = wait_bounded(&sm.v_empty[vs], ((vc / NVS) & 1) ^ 1, abort_flag, a.status, true))) break;
                            mbar_arrive_expect_tx(&sm.v_full[vs], kKBytes);
                            tma_load_3d(smem + offV + vs * kKBytes, &tmV, &sm.v_full[vs], 0, J * BN, bh);
                            ++vc;
                        }
                    }
                }
            }
            if (!ok) {
                for (uint32_t i = (lc > (uint32_t)NKS ? lc - NKS : 0); i < lc; ++i)
                    wait_drain(&sm.k_full[i % NKS], (i / NKS) & 1, 100000000ull);
                for (uint32_t i = (vc > (uint32_t)NVS ? vc - NVS : 0); i < vc; ++i)
                    wait_drain(&sm.v_full[i % NVS], (i / NVS) & 1, 100000000ull);
                wait_drain(&sm.q_full, 0, 100000000ull);
            }
        }
    } else if (warp == 8) {
        // ------------------------------------------------------------------ S issue
        if (lane == 0) {
            constexpr uint32_t idS = idesc_f16_f32(BM, BN, false, false);
            uint32_t lc = 0;              // K blocks consumed (ring order)
            uint32_t sc0 = 0, sc1 = 0;    // per warpgroup: S tiles issued
            // per buffer (bit 2 g + b): parity of the commit of the P V that last read (or will read) it;
            // after k commits the barrier has completed phase k - 1, so the bits start at 1
            uint32_t ppar = (1u << (2 * NSB)) - 1u;
            bool after_pv = false;
            int npv = 0;
            bool ok = wait_bounded(&sm.q_full, 0, abort_flag, a.status, true);
            tc_fence_after();
            for (int sw = 0; ok; ++sw) {
                if (!(ok = wait_bounded(&sm.ctrl, sw & 1, abort_flag, a.status, true))) break;
                const int kind = sm.plan_kind[sw & 1];
                if (after_pv) {
                    // every P V of the last P V sweep complete before a buffer holding P is overwritten
                    if (!(ok = wait_bounded(&sm.o_full, (npv - 1) & 1, abort_flag, a.status, true))) break;
                    after_pv = false;
                }
                tc_fence_after();
                if (kind == kSweepDone) break;
                const uint32_t* bits_p = plan_bits + (sw & 1) * W;
                int T = 0;
                for (int wd = 0; wd < W; ++wd) T += __popc(bits_p[wd]);
                const bool pvk = kind == kSweepPV;
                for (int ts = 0; ts < T && ok; ++ts) {
                    const int g = (kind == kSweepHist) ? 0 : (ts & 1);
                    const uint32_t sn = g ? sc1 : sc0;
                    const uint32_t b = sn % NSB;
                    const uint32_t bi = NSB * g + b;
                    const uint32_t ks = lc % NKS;
                    if (!(ok = wait_bounded(&sm.k_full[ks], (lc / NKS) & 1, abort_flag, a.status, true))) break;
                    if (!(ok = wait_bounded(&sm.s_empty[g][b], ((sn / NSB) & 1) ^ 1, abort_flag, a.status, true))) break;
                    if (pvk) {
                        // the buffer last held block ts - 2 NSB of this sweep: its P V must have completed
                        if (ts >= 2 * NSB && !(ok = wait_bounded(&sm.pv_free[g][b], (ppar >> bi) & 1u, abort_flag, a.status, true)))
                            break;
                        ppar ^= 1u << bi;  // block ts's own P V, committed later by the P V thread
                    }
                    tc_fence_after();
                    const uint32_t kbase = sK0 + ks * kKBytes;
                    const uint32_t dS = tmem + 64u * bi;
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk)
                        mma_ss(dS, sdesc_at(kDescK, sQ + kk * 32), sdesc_at(kDescK, kbase + kk * 32), idS, kk > 0 ? 1u : 0u);
                    mma_commit(&sm.s_full[g][b]);
                    ++lc;
                    if (g) ++sc1; else ++sc0;
                }
                if (pvk) {
                    after_pv = true;
                    ++npv;
                }
            }
            mma_commit(&sm.drain[0]);
            wait_drain(&sm.drain[0], 0, 200000000ull);
        }
    } else if (warp == 10) {
        // ------------------------------------------------------------------ P V issue
        if (lane == 0) {
            constexpr uint32_t idPV = idesc_f16_f32(BM, D, false, true);
            uint32_t vc = 0;              // V blocks consumed (ring order)
            uint32_t sc0 = 0, sc1 = 0;    // per warpgroup: S tiles issued (followed, not issued here)
            uint32_t ppar = (1u << (2 * NSB)) - 1u;  // per buffer: parity of the last P V commit on its barrier
            bool ok = true;
            for (int sw = 0; ok; ++sw) {
                if (!(ok = wait_bounded(&sm.ctrl, sw & 1, abort_flag, a.status, true))) break;
                tc_fence_after();
                const int kind = sm.plan_kind[sw & 1];
                if (kind == kSweepDone) break;
                const uint32_t* bits_p = plan_bits + (sw & 1) * W;
                int T = 0;
                for (int wd = 0; wd < W; ++wd) T += __popc(bits_p[wd]);
                if (kind != kSweepPV) {
                    if (kind == kSweepHist) sc0 += T;
                    else { sc0 += (T + 1) / 2; sc1 += T / 2; }
                    continue;
                }
                for (int tp = 0; tp < T && ok; ++tp) {
                    const int g = tp & 1;
                    const uint32_t sn = g ? sc1 : sc0;
                    const uint32_t b = sn % NSB;
                    const uint32_t bi = NSB * g + b;
                    const uint32_t vs = vc % NVS;
                    // k P V products on a buffer so far: its P store number k + 1 completes phase k
                    if (!(ok = wait_bounded(&sm.pu_full[g][b], ((ppar >> bi) & 1u) ^ 1u, abort_flag, a.status, true))) break;
                    if (!(ok = wait_bounded(&sm.v_full[vs], (vc / NVS) & 1, abort_flag, a.status, true))) break;
                    tc_fence_after();
                    const uint32_t vbase = sV0 + vs * kKBytes;
                    const uint32_t tpu = tmem + 64u * bi;
#pragma unroll
                    for (int kk = 0; kk < BN / 16; ++kk) {
                        const uint64_t dv = sdesc_at(kDescMN, vbase + kk * 2048);
                        const uint32_t acc = (tp == g && kk == 0) ? 0u : 1u;
                        mma_ts(tmem + kColO + 64u * g, tpu + 8 * kk, dv, idPV, acc);
                    }
                    mma_commit(&sm.pv_free[g][b]);
                    mma_commit(&sm.v_empty[vs]);
                    ppar ^= 1u << bi;
                    ++vc;
                    if (g) ++sc1; else ++sc0;
                }
                if (ok) mma_commit(&sm.o_full);
            }
            mma_commit(&sm.drain[1]);
            wait_drain(&sm.drain[1], 0, 200000000ull);
        }
    } else {
        // ------------------------------------------------------------------ compute warpgroups
        const int g = warp >> 2;
        const int r = tid & (BM - 1);
        const int row = row0 + r;
        const bool valid = row < a.n;
        const int n_i = valid ? allowed_keys(row, a.n, a.causal) : 1;
        const uint32_t lane_base = tmem + ((uint32_t)((warp & 3) * 32) << 16);
        const size_t head = (size_t)bh * a.n;
        const int half = r >> 6;
        float* st_mine = stash + g * (kHalf * BM);

        // range exponents of the fp16 copies: raw scores carry 2^-(eQ + eK), V carries 2^-eV
        SolveParams sp = a.sp;
        const int eqk = f16_range_exp(a.maxbits[0]) + f16_range_exp(a.maxbits[1]);
        const float vscale = ldexpf(1.0f, f16_range_exp(a.maxbits[2]));
        if (eqk) {
            sp.cz = ldexpf(sp.cz, eqk);
            sp.inv_cz = ldexpf(sp.inv_cz, -eqk);
            sp.cbin = ldexpf(sp.cbin, eqk);
        }

        for (int i = tid; i <= sp.bins; i += kCompute) sm.T[i] = (KIND == kGeneric) ? powf((float)i, sp.k) : 0.0f;
        for (int i = tid; i < W; i += kCompute) {
            const int lo = i * 32;
            uint32_t v = 0u;
            if (lo < nblk) v = (nblk - lo >= 32) ? 0xffffffffu : ((1u << (nblk - lo)) - 1u);
            plan_bits[i] = v;  // plan 0: every causal block
            next[i] = 0u;
        }
        sm.xf[kXMax0 + g][r] = -INFINITY;
        if (tid == 0) sm.plan_kind[0] = kSweepDense;

        named_bar_sync(1, kCompute);
        if (lane == 0) mbar_arrive(&sm.ctrl);

        uint32_t sc = 0, pc = 0;
        uint32_t colS = 0;  // TMEM column of the S tile loaded last
        uint32_t curb = 0;  // its buffer index
        int sw = 0;
        bool ok = true;
        float vbuf[BN];

        uint32_t lcs = 0;  // K blocks of the sweeps before this one (ring order)
        auto load_S = [&](uint32_t kidx) -> bool {
            const uint32_t sb = sc % NSB;
            const bool got = wait_bounded(&sm.s_full[g][sb], (sc / NSB) & 1, abort_flag, a.status);
            if (!__all_sync(0xffffffffu, got)) return false;
            tc_fence_after();
            __syncwarp();
            uint32_t* rr = reinterpret_cast<uint32_t*>(vbuf);
            colS = 64u * (NSB * g + sb);
            curb = sb;
            tmem_ld32(lane_base + colS, rr);
            tmem_ld32(lane_base + colS + 32, rr + 32);
            tmem_ld_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&sm.s_empty[g][sb]);
                mbar_arrive(&sm.k_empty[kidx % NKS]);  // the MMA that read this K block has completed
            }
            ++sc;
            return true;
        };
        auto mask_S = [&](int J) {
            if (block_full(J, a.n, a.causal, row0) && valid) return;
#pragma unroll
            for (int c = 0; c < BN; ++c) {
                const int key = J * BN + c;
                if (!(valid && key < a.n && (!a.causal || key <= row))) vbuf[c] = -INFINITY;
            }
        };
        auto publish = [&](int kind) {
            // next[] holds the keep bits of the sweep just finished; the V ring of a P V sweep reuses
            // shared memory that generic loads and stores touched, hence the proxy fence
            fence_proxy_async_smem();
            named_bar_sync(1, kCompute);
            const int nb = (sw + 1) & 1;
            for (int i = tid; i < W; i += kCompute) {
                plan_bits[nb * W + i] = next[i];
                next[i] = 0u;
            }
            if (kind == kSweepPV || kind == kSweepSupport)
                for (int i = tid; i < 2 * W; i += kCompute) mrow[i] = 0u;
            if (tid == 0) sm.plan_kind[nb] = kind;
            named_bar_sync(1, kCompute);
            ++sw;
            if (lane == 0) mbar_arrive(&sm.ctrl);
        };

        float gm[8];
        auto group_max = [&]() -> float {
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const float* v = vbuf + 8 * q;
                gm[q] = fmax3(fmax3(v[0], v[1], v[2]), fmax3(v[3], v[4], v[5]), fmaxf(v[6], v[7]));
            }
            return fmax3(fmax3(gm[0], gm[1], gm[2]), fmax3(gm[3], gm[4], gm[5]), fmaxf(gm[6], gm[7]));
        };

        // ---- sweep 0: dense (warpgroup g takes blocks g, g + 2, ...) ----
        float m_run = -INFINITY, thr = INFINITY;
        int nst = 0;
        bool ovf = false;
        volatile float* xm_other = sm.xf[kXMax0 + (g ^ 1)];
        for (int J = g; J < nblk && ok; J += 2) {
            if (!(ok = load_S(lcs + J))) break;
            mask_S(J);
            const float amax = group_max();
            // the other warpgroup's running max is a valid (tighter) threshold as well
            const float mn = fmaxf(amax, xm_other[r]);
            if (mn > m_run) {
                m_run = mn;
                thr = mn - sp.inv_cz;
                sm.xf[kXMax0 + g][r] = mn;
            }
            const bool any = amax > thr;
            if (__any_sync(0xffffffffu, any)) {
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    bool fl = !ovf && gm[q] > thr;
                    if (__any_sync(0xffffffffu, fl)) {
                        const bool room = fl && nst > kHalf - 8;
                        if (__any_sync(0xffffffffu, room)) {
                            if (room) {
                                nst = stash_prune(nst, st_mine, r, thr, kHalf);
                                if (nst < 0) { ovf = true; nst = 0; }
                            }
                            fl = fl && !ovf;
                        }
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            const float v = vbuf[8 * q + e];
                            const bool put = fl && v > thr;
                            if (put) st_mine[nst * BM + r] = v;
                            nst += put ? 1 : 0;
                        }
                    }
                }
            }
            const uint32_t ball = __ballot_sync(0xffffffffu, any);
            if (lane == 0 && ball) atomicOr(&next[J >> 5], 1u << (J & 31));
        }
        lcs += nblk;
        sm.xf[g ? kXCnt1 : kXCnt0][r] = __int_as_float(ovf ? -1 : nst);
        ok = !bar_or256(!ok || *abort_flag != 0);

        // ---- the rows' histograms, binned from both stash halves at once (window fixed by the final max) ----
        // Counts are u16 [slot][128]; the two warpgroups' threads of a row add into it with 32-bit shared
        // atomics on the word holding the row's count (a count stays below 2^16, so the neighbouring row's
        // half-word is untouched) and set the slot's live bit with an atomic OR.
        {
            const float m_fin = fmaxf(sm.xf[kXMax0][r], sm.xf[kXMax1][r]);
            const bool binit = ok && valid && sp.init_mode == 0 && __float_as_int(sm.xf[kXCnt0][r]) >= 0 &&
                               __float_as_int(sm.xf[kXCnt1][r]) >= 0;
            uint32_t* hist32 = reinterpret_cast<uint32_t*>(hist);
            for (int i = tid; i < NB * BM / 2; i += kCompute) hist32[i] = 0u;
            uint32_t* live_r = live_all + r * HC::kStride;
            if (g == 0)
                for (int i = 0; i < HC::kStride - 1; ++i) live_r[i] = 0u;
            named_bar_sync(1, kCompute);
            if (binit) {
                const int top = bin_of(m_fin, sp.cbin);
                const float thr_raw = m_fin - sp.inv_cz;
                const uint32_t inc = 1u << (16 * (r & 1));
                for (int i = 0; i < nst; ++i) {
                    const float v = st_mine[i * BM + r];
                    if (v > thr_raw) {
                        const int b = bin_of(v, sp.cbin);
                        const int j = top - b;
                        if (j >= 0 && j < sp.bins) {
                            const int sl = b & (sp.bins - 1);
                            atomicAdd(&hist32[(sl * BM + r) >> 1], inc);
                            atomicOr(&live_r[sl >> 5], 1u << (sl & 31));
                        }
                    }
                }
            }
            named_bar_sync(1, kCompute);
        }

        // ---- per-row solve (warpgroup 0 owns the solver state of its row) ----
        HistRow h;
        RowSolve s;
        bool row_ovf = false;
        float Su_stash = 0.f;
        uint32_t nsup = 0;  // the row's support size (warpgroup 0)
        float m_raw = -INFINITY;
        int n1 = 0;
        if (g == 0) {
            // the live words were cleared and set by the binning above
            h.nlw = HC::kStride - 1;
            h.live = live_all + r * HC::kStride;
            const int c1 = __float_as_int(sm.xf[kXCnt1][r]);
            m_raw = fmaxf(m_run, sm.xf[kXMax1][r]);
            row_ovf = ovf || c1 < 0;
            n1 = c1 < 0 ? 0 : c1;
            const float m = sp.cz * m_raw;
            float tau_h = m - 1.0f;
            if (ok && valid && !row_ovf && sp.init_mode == 0) {
                // the window and the counts are in place (binned above); at most 2 kHalf entries per row, so
                // 32-bit moments are exact
                h.any = m_raw > -INFINITY;
                h.m_raw = m_raw;
                h.thr_raw = m_raw - sp.inv_cz;
                h.top = h.any ? bin_of(m_raw, sp.cbin) : 0;
                tau_h = hist_tau<KIND, int>(h, sp, hist, r, sm.T);
            }
            solve_init(s, valid ? tau_h : 0.0f, valid ? m : 1.0f, n_i, sp);
            if (!valid) s.done = true;
            if (valid && !row_ovf && a.tau_hist) a.tau_hist[head + row] = tau_h;
            // rows whose candidates all fit the stash are solved on chip, with no further key sweep; their
            // sum of u comes from the stash too (it holds every entry above tau)
            if (ok && valid && !row_ovf) {
                for (int it = 0; it < kMaxSweeps && !s.done; ++it) {
                    float F0 = 0.f, F1 = 0.f, F2 = 0.f, F0b = 0.f;
                    half_sums<KIND>(st_mine, nst, r, sp, s.tau, s.tau2, s.need_two, F0, F1, F2, F0b);
                    half_sums<KIND>(stash + kHalf * BM, n1, r, sp, s.tau, s.tau2, s.need_two, F0, F1, F2, F0b);
                    solve_step(s, F0, F1, F2, F0b, sp);
                }
                float F0 = 0.f, F1 = 0.f, F2 = 0.f, F0b = 0.f;
                half_sums<KIND>(st_mine, nst, r, sp, s.tau, s.tau, false, F0, F1, F2, F0b);
                half_sums<KIND>(stash + kHalf * BM, n1, r, sp, s.tau, s.tau, false, F0, F1, F2, F0b);
                Su_stash = F1;
                nsup = half_count(st_mine, nst, r, sp.cz, s.tau) + half_count(stash + kHalf * BM, n1, r, sp.cz, s.tau);
            }
            sm.xf[kXOvf][r] = (valid && row_ovf) ? 1.0f : 0.0f;
        }

        // ---- histogram sweep for rows whose stash overflowed (warpgroup 0 only) ----
        if (ok && bar_or256(g == 0 && valid && row_ovf && sp.init_mode == 0)) {
            publish(kSweepHist);
            if (g == 0) {
                const bool mine = valid && row_ovf;
                if (mine) hist_start(h, m_raw, sp);
                const float thr_f = m_raw - sp.inv_cz;
                const uint32_t* bits_p = plan_bits + (sw & 1) * W;
                uint32_t ph = 0;
                for (int wd = 0; wd < W && ok; ++wd) {
                    uint32_t bits = bits_p[wd];
                    while (bits) {
                        const int J = wd * 32 + __ffs(bits) - 1;
                        bits &= bits - 1;
                        if (!(ok = load_S(lcs + ph++))) break;  // warpgroup 0 takes every block
                        mask_S(J);
                        const float amax = group_max();
                        const bool keep = amax > thr_f;
                        if (__any_sync(0xffffffffu, mine && keep)) {
                            if (mine && keep) {
                                // stage the block in the row's stash slots (no longer needed; this is
                                // warpgroup 0, so the slots from the start of the stash, both halves: 2 kHalf
                                // >= 64) and bin it with a rolled loop
                                uint32_t gflag = 0u;
#pragma unroll
                                for (int q = 0; q < 8; ++q) gflag |= (gm[q] > thr_f ? 1u : 0u) << q;
#pragma unroll
                                for (int c = 0; c < BN; ++c) stash[c * BM + r] = vbuf[c];
                                hist_bin_block(h, stash + r, gflag, sp, hist, r);
                            }
                        }
                        const uint32_t ball = __ballot_sync(0xffffffffu, keep);
                        if (lane == 0 && ball) atomicOr(&next[J >> 5], 1u << (J & 31));
                    }
                }
            }
            {
                const uint32_t* bp = plan_bits + (sw & 1) * W;
                for (int wd = 0; wd < W; ++wd) lcs += __popc(bp[wd]);
            }
            ok = !bar_or256(!ok || *abort_flag != 0);
            if (ok && g == 0 && valid && row_ovf) {
                const float tau_h = hist_tau<KIND>(h, sp, hist, r, sm.T);
                solve_init(s, tau_h, sp.cz * m_raw, n_i, sp);
                if (a.tau_hist) a.tau_hist[head + row] = tau_h;
            }
        }
        if (g == 0 && valid && row_ovf && sp.init_mode != 0 && a.tau_hist) a.tau_hist[head + row] = sp.cz * m_raw - 1.0f;

        // ---- refinement sweep: solver sums at the current tau over the candidate blocks ----
        float last_step = INFINITY;
        int refine = 0, pv = 0;
        auto refine_sweep = [&]() {
            if (g == 0) {
                sm.xf[kXTau][r] = s.tau;
                sm.xf[kXTau2][r] = s.tau2;
                sm.xf[kXLo][r] = s.lo;
                sm.xf[kXTwo][r] = s.need_two ? 1.0f : 0.0f;
            }
            publish(kSweepRefine);
            const float t = sm.xf[kXTau][r], t2 = sm.xf[kXTau2][r], lo0 = sm.xf[kXLo][r];
            const bool two = sm.xf[kXTwo][r] != 0.0f;
            float F0 = 0.f, F1 = 0.f, F2 = 0.f, F0b = 0.f;
            const uint32_t* bits_p = plan_bits + (sw & 1) * W;
            int p = 0;
            for (int wd = 0; wd < W && ok; ++wd) {
                uint32_t bits = bits_p[wd];
                while (bits) {
                    const int J = wd * 32 + __ffs(bits) - 1;
                    bits &= bits - 1;
                    if (((p++) & 1) != g) continue;
                    if (!(ok = load_S(lcs + (uint32_t)(p - 1)))) break;
                    mask_S(J);
                    const float amax = group_max();
                    const bool keep = sp.cz * amax > lo0;
                    if (fmaf(amax, sp.cz, -t) > 0.f) {
#pragma unroll
                        for (int q = 0; q < 8; ++q) {
                            if (fmaf(gm[q], sp.cz, -t) > 0.f) {
#pragma unroll
                                for (int e = 0; e < 8; ++e) {
                                    const float x = fmaf(vbuf[8 * q + e], sp.cz, -t);
                                    if constexpr (KIND == kAlpha15) {
                                        const float xp = fmaxf(x, 0.f);
                                        F0 = fmaf(xp, xp, F0);
                                        F1 += xp;
                                        F2 += x > 0.f ? 1.f : 0.f;
                                    } else if constexpr (KIND == kAlpha2) {
                                        F0 += fmaxf(x, 0.f);
                                        F1 += x > 0.f ? 1.f : 0.f;
                                    } else {
                                        if (x > 0.f) add_sums<KIND>(x, sp.k, F0, F1, F2);
                                    }
                                    if (two) {
                                        const float x2 = fmaf(vbuf[8 * q + e], sp.cz, -t2);
                                        if (x2 > 0.f) F0b += pow_k<KIND>(x2, sp.k);
                                    }
                                }
                            }
                        }
                    }
                    const uint32_t ball = __ballot_sync(0xffffffffu, keep);
                    if (lane == 0 && ball) atomicOr(&next[J >> 5], 1u << (J & 31));
                }
            }
            if (g == 1) {
                sm.xf[kXF0][r] = F0;
                sm.xf[kXF1][r] = F1;
                sm.xf[kXF2][r] = F2;
                sm.xf[kXF0b][r] = F0b;
            }
            ok = !bar_or256(!ok || *abort_flag != 0);
            if (g == 0) {
                F0 += sm.xf[kXF0][r];
                F1 += sm.xf[kXF1][r];
                F2 += sm.xf[kXF2][r];
                F0b += sm.xf[kXF0b][r];
                const float before = s.tau;
                solve_step(s, F0, F1, F2, F0b, sp);
                last_step = s.tau - before;
            }
            lcs += (uint32_t)p;
            ++refine;
        };

        // ---- P V sweep: p to TMEM for the P V MMAs, exact mask, sum check ----
        float Su = 0.f;
        int pv_tiles = 0;  // blocks of the last P V sweep
        auto pv_sweep = [&]() -> bool {
            if (g == 0) {
                sm.xf[kXTau][r] = s.tau;
                sm.xf[kXLo][r] = s.lo;
            }
            publish(kSweepPV);
            const float t = sm.xf[kXTau][r], lo0 = sm.xf[kXLo][r];
            const bool need_sums = __any_sync(0xffffffffu, sm.xf[kXOvf][r] != 0.0f);
            float Sp = 0.f, Sq = 0.f, F2 = 0.f;
            uint32_t Sn = 0;
            const uint32_t* bits_p = plan_bits + (sw & 1) * W;
            int p = 0;
            for (int wd = 0; wd < W && ok; ++wd) {
                uint32_t bits = bits_p[wd];
                while (bits) {
                    const int J = wd * 32 + __ffs(bits) - 1;
                    bits &= bits - 1;
                    if (((p++) & 1) != g) continue;
                    if (!(ok = load_S(lcs + (uint32_t)(p - 1)))) break;
                    mask_S(J);
                    const float amax = group_max();
                    const bool keep = sp.cz * amax > lo0;
                    const bool nz = fmaf(amax, sp.cz, -t) > 0.f;
                    // one branch-free pass over the block, 32 keys at a time: p of each key, packed as fp16
                    // pairs into the first 32 columns of the S tile just read (this warpgroup's own buffer).
                    // The solver sums (and u) ride along in warps that hold a row whose tau still needs the
                    // check.
                    const uint32_t tp = lane_base + colS;
                    auto pu_pass = [&](auto with_sums) {
                        constexpr bool SUMS = decltype(with_sums)::value;
#pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            uint32_t wp[16];
#pragma unroll
                            for (int c = 0; c < 32; c += 2) {
                                float p2[2];
#pragma unroll
                                for (int h2 = 0; h2 < 2; ++h2) {
                                    const float x = fmaf(vbuf[32 * h + c + h2], sp.cz, -t);
                                    float pp;
                                    if constexpr (KIND == kAlpha15) {
                                        const float uu = fmaxf(x, 0.f);
                                        pp = uu * uu;
                                        if constexpr (SUMS) {
                                            F2 += x > 0.f ? 1.f : 0.f;
                                            Sq += uu;
                                        }
                                    } else if constexpr (KIND == kAlpha2) {
                                        pp = fmaxf(x, 0.f);
                                        if constexpr (SUMS) Sq += x > 0.f ? 1.f : 0.f;
                                    } else {
                                        const bool pos = x > 0.f;
                                        const float xs = pos ? x : 1.f;
                                        const float u1 = exp2f((sp.k - 1.f) * __log2f(xs));
                                        const float uu = pos ? u1 : 0.f;
                                        pp = uu * xs;
                                        if constexpr (SUMS) {
                                            F2 += pos ? __fdividef(u1, xs) : 0.f;
                                            Sq += uu;
                                        }
                                    }
                                    if constexpr (SUMS) {
                                        Sp += pp;
                                        Sn += x > 0.f ? 1u : 0u;
                                    }
                                    p2[h2] = pp;
                                }
                                wp[c / 2] = pack_half2(p2[0], p2[1]);
                            }
                            tmem_st16(tp + 16 * h, wp);
                        }
                    };
                    if (need_sums) pu_pass(std::true_type{});
                    else pu_pass(std::false_type{});
                    tmem_st_wait();
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&sm.pu_full[g][curb]);
                    ++pc;
                    const uint32_t kb = __ballot_sync(0xffffffffu, keep);
                    const uint32_t nb = __ballot_sync(0xffffffffu, nz);
                    if (lane == 0) {
                        if (kb) atomicOr(&next[J >> 5], 1u << (J & 31));
                        if (nb) atomicOr(&mrow[half * W + (J >> 5)], 1u << (J & 31));
                    }
                }
            }
            if (g == 1) {
                sm.xf[kXF0][r] = Sp;
                sm.xf[kXF1][r] = Sq;
                sm.xf[kXF2][r] = F2;
                sm.xf[kXCnt][r] = __uint_as_float(Sn);
            }
            pv_tiles = p;
            lcs += (uint32_t)p;
            ++pv;
            ok = !bar_or256(!ok || *abort_flag != 0);
            bool changed = false;
            if (g == 0) {
                if (row_ovf) {
                    Sp += sm.xf[kXF0][r];
                    Su = Sq + sm.xf[kXF1][r];
                    F2 += sm.xf[kXF2][r];
                    nsup = Sn + __float_as_uint(sm.xf[kXCnt][r]);
                    const float before = s.tau;
                    solve_step(s, Sp, Su, F2, 0.f, sp);
                    changed = s.tau != before;
                } else {
                    Su = Su_stash;
                }
            }
            return ok && bar_or256(changed);
        };

        // Schedule: refine while some row still takes steps wider than one bin; then P V, whose sums
        // double as the check of sum p = 1. If any tau still moved, refine until every row has
        // stopped and finish with one more P V sweep.
        if (ok && bar_or256(g == 0 && !s.done)) {
            do {
                refine_sweep();
            } while (ok && refine < kMaxSweeps && bar_or256(g == 0 && !s.done && fabsf(last_step) > sp.w));
        }
        // ---- support sweep (element path): list the support entries of each row, then gather O ----
        constexpr int kCap = HC::kElemCap;
        float oacc[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) oacc[i] = 0.f;
        auto support_sweep = [&]() {
            if (g == 0) sm.xf[kXTau][r] = s.tau;
            publish(kSweepSupport);
            const float t = sm.xf[kXTau][r];
            uint16_t* lk = elem_key + g * (kCap * BM) + r;
            float* lp = elem_p + g * (kCap * BM) + r;
            int cnt = 0;
            const uint32_t* bits_p = plan_bits + (sw & 1) * W;
            int p = 0;
            for (int wd = 0; wd < W && ok; ++wd) {
                uint32_t bits = bits_p[wd];
                while (bits) {
                    const int J = wd * 32 + __ffs(bits) - 1;
                    bits &= bits - 1;
                    if (((p++) & 1) != g) continue;
                    if (!(ok = load_S(lcs + (uint32_t)(p - 1)))) break;
                    mask_S(J);
                    const float amax = group_max();
                    const bool nz = fmaf(amax, sp.cz, -t) > 0.f;
                    if (nz) {
                        // the row's support entries in this block (groups of 8 whose max is above tau); the
                        // same S and the same x as the solver's count, so the list never exceeds the row's
                        // support (the cap check only guards the memory)
#pragma unroll
                        for (int q = 0; q < 8; ++q) {
                            if (fmaf(gm[q], sp.cz, -t) > 0.f) {
#pragma unroll
                                for (int e = 0; e < 8; ++e) {
                                    const float x = fmaf(vbuf[8 * q + e], sp.cz, -t);
                                    if (x > 0.f && cnt < kCap) {
                                        lk[cnt * BM] = (uint16_t)(J * BN + 8 * q + e);
                                        lp[cnt * BM] = pow_k<KIND>(x, sp.k);
                                        ++cnt;
                                    }
                                }
                            }
                        }
                    }
                    const uint32_t nb = __ballot_sync(0xffffffffu, nz);
                    if (lane == 0 && nb) atomicOr(&mrow[half * W + (J >> 5)], 1u << (J & 31));
                }
            }
            lcs += (uint32_t)p;
            elem_cnt[g * BM + r] = cnt;
            ++pv;
            ok = !bar_or256(!ok || *abort_flag != 0);  // lists and counts of both warpgroups visible
            if (g == 0) Su = Su_stash;
            // O row r, columns 32 g .. 32 g + 31: sum over both lists of p v_key (fp16 copy of V, fp32 sums)
            if (ok && valid) {
                const __half* Vh = static_cast<const __half*>(a.Vh) + head * D + 32 * g;
                for (int hh = 0; hh < 2; ++hh) {
                    const int nh = elem_cnt[hh * BM + r];
                    const uint16_t* kk = elem_key + hh * (kCap * BM) + r;
                    const float* pk = elem_p + hh * (kCap * BM) + r;
#pragma unroll 4
                    for (int e = 0; e < nh; ++e) {
                        const uint4* src = reinterpret_cast<const uint4*>(Vh + (size_t)kk[e * BM] * D);
                        const float pe = pk[e * BM];
                        uint4 w[4];
#pragma unroll
                        for (int i = 0; i < 4; ++i) w[i] = __ldg(src + i);
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const __half2* h2 = reinterpret_cast<const __half2*>(&w[i]);
#pragma unroll
                            for (int m = 0; m < 4; ++m) {
                                const float2 f = __half22float2(h2[m]);
                                oacc[8 * i + 2 * m] = fmaf(pe, f.x, oacc[8 * i + 2 * m]);
                                oacc[8 * i + 2 * m + 1] = fmaf(pe, f.y, oacc[8 * i + 2 * m + 1]);
                            }
                        }
                    }
                }
            }
        };

        // element path: no row overflowed its stash, every row's tau is final, every support fits a list
        // (and keys fit the u16 lists)
        const bool elem = ok && a.n <= 65536 &&
                          !bar_or256(g == 0 && valid && !(!row_ovf && s.done && nsup <= (uint32_t)kCap));
        if (elem) {
            support_sweep();
        } else {
            while (ok) {
                const bool changed = pv_sweep();
                if (!ok || !changed || pv >= 3) break;
                while (ok && refine < kMaxSweeps && bar_or256(g == 0 && !s.done)) refine_sweep();
            }
        }

        // ---- wait for the last P V MMAs, then write O (warpgroup g: columns 32 g .. 32 g + 31), tau, sum u ----
        if (ok && !elem) ok = __all_sync(0xffffffffu, wait_bounded(&sm.o_full, (pv - 1) & 1, abort_flag, a.status));
        ok = !bar_or256(!ok || *abort_flag != 0);
        if (ok) {
            tc_fence_after();
            __syncwarp();
            uint32_t o[32];
            if (elem) {
#pragma unroll
                for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(oacc[i]);
            } else {
                tmem_ld32(lane_base + kColO + 32u * g, o);
                tmem_ld_wait();
            }
            if (!elem && pv_tiles > 1) {  // the second warpgroup's accumulator holds the odd blocks
                uint32_t o2[32];
                tmem_ld32(lane_base + kColO + 64u + 32u * g, o2);
                tmem_ld_wait();
#pragma unroll
                for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) + __uint_as_float(o2[i]));
            }
            if (valid) {
                uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(a.O) + (head + row) * D + 32 * g);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float* f = reinterpret_cast<const float*>(o + 8 * i);
                    dst[i] = make_uint4(pack_bf16x2(f[0] * vscale, f[1] * vscale),
                                        pack_bf16x2(f[2] * vscale, f[3] * vscale),
                                        pack_bf16x2(f[4] * vscale, f[5] * vscale),
                                        pack_bf16x2(f[6] * vscale, f[7] * vscale));
                }
            }
            tc_fence_before();
            if (g == 0 && valid) {
                a.tau[head + row] = s.tau;
                a.sum_u[head + row] = Su;
                if (a.steps) a.steps[head + row] = (uint8_t)s.steps;
            }
        }
        // tell the issuing warps to stop
        if (tid == 0) sm.plan_kind[(sw + 1) & 1] = kSweepDone;
        named_bar_sync(1, kCompute);
        if (lane == 0) mbar_arrive(&sm.ctrl);

        // mask rows of this tile (two 64-row query blocks)
        named_bar_sync(1, kCompute);
        for (int i = tid; i < 2 * W; i += kCompute) {
            const int qb = qt * 2 + i / W;
            if (qb < a.nqb) a.mask[((size_t)bh * a.nqb + qb) * W + (i % W)] = ok ? mrow[i] : 0u;
        }
        if (a.stats && ok) {
            const uint32_t* cb = plan_bits + (sw & 1) * W;
            uint32_t nzb = 0, cnd = 0;
            for (int i = tid; i < 2 * W; i += kCompute) nzb += __popc(mrow[i]);
            for (int i = tid; i < W; i += kCompute) cnd += __popc(cb[i]);
            if (nzb) atomicAdd(&sm.st.nonzero_blocks, nzb);
            if (cnd) atomicAdd(&sm.st.candidate_blocks, cnd);
            if (g == 0 && valid) {
                if (row_ovf) atomicAdd(&sm.st.overflow_rows, 1u);
                atomicAdd(&sm.st.rows, 1u);
                atomicAdd(&sm.st.support, nsup);
                atomicAdd(&sm.st.steps, (uint32_t)s.steps);
                atomicAdd(&sm.st.fallbacks, (uint32_t)s.fallbacks);
                atomicAdd(&sm.st.step_hist[min(s.steps, kMaxSteps)], 1u);
            }
            named_bar_sync(1, kCompute);
            if (tid == 0) {
                sm.st.sweeps = (uint32_t)(1 + refine + pv);
                sm.st.causal_blocks = tile_causal_blocks(2 * qt, 2, a.nqb, a.nkb, a.causal);
                flush_stats(a.stats, sm.st);
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

template <int KIND, int NB>
cudaError_t launch_fwd_h_t(const FwdArgs& a, cudaStream_t stream) {
    CUtensorMap tq, tk, tv;
    cudaError_t e;
    if ((e = make_tmap_f16(&tq, a.Qh, a.B * a.H, a.n, D, BM)) != cudaSuccess) return e;
    if ((e = make_tmap_f16(&tk, a.Kh, a.B * a.H, a.n, D, BN)) != cudaSuccess) return e;
    if ((e = make_tmap_f16(&tv, a.Vh, a.B * a.H, a.n, D, BN)) != cudaSuccess) return e;
    const size_t bytes = fwd_h_smem_bytes(a.nw, NB);
    if (bytes > 232448) return cudaErrorInvalidConfiguration;
    auto kern = fwd_h_kernel<KIND, NB>;
    if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes)) != cudaSuccess)
        return e;
    dim3 grid(a.B * a.H, a.ntiles);
    launch_mark(stream);
    kern<<<grid, kThreads, bytes, stream>>>(tq, tk, tv, a);
    return cudaGetLastError();
}

template <int NB>
cudaError_t launch_fwd_h_nb(const FwdArgs& a, cudaStream_t stream) {
    if (a.sp.alpha == 1.5f) return launch_fwd_h_t<kAlpha15, NB>(a, stream);
    if (a.sp.alpha == 2.0f) return launch_fwd_h_t<kAlpha2, NB>(a, stream);
    return launch_fwd_h_t<kGeneric, NB>(a, stream);
}

}  // namespace

size_t fwd_h_smem_bytes(int nw, int bins) {
    if (bins > 256) {
        using HC = HCfg<512>;
        return 1024 + HC::offSmall + sizeof(Small) + (size_t)5 * nw * 4 + (size_t)BM * HC::kStride * 4;
    }
    using HC = HCfg<256>;
    return 1024 + HC::offSmall + sizeof(Small) + (size_t)5 * nw * 4 + (size_t)BM * HC::kStride * 4;
}

cudaError_t launch_fwd_h(const FwdArgs& a, cudaStream_t stream) {
    if (a.d != 64 || !(a.sp.alpha <= 2.0f)) return cudaErrorInvalidValue;
    if (a.sp.bins > 256) return launch_fwd_h_nb<512>(a, stream);
    return launch_fwd_h_nb<256>(a, stream);
}

}  // namespace eattn
