// fwd_tc.cu - alpha-entmax attention forward for bf16 on the sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
// One CTA per (b, h, 128-row query tile), 192 threads:
//   warps 0-3  compute: thread r owns query row r of the tile and TMEM lane r (tcgen05.ld 32x32b);
//   warp 4     MMA issue (one thread): S = Q K^T into TMEM, O += P V and U V into TMEM;
//   warp 5     TMA issue (one thread): Q once, K (and V in P V sweeps) blocks of 64 keys into a ring.
// TMEM columns: S double buffer [0, 64) and [64, 128), O [128, 128 + D), U V [128 + D, 128 + 2D).
//
// The key blocks of a tile are swept several times; before each sweep the compute warps publish a
// plan (sweep kind + bit set of key blocks) that the two issuing warps follow:
//   dense  - every causal key block: running max, left-edge histogram (shared memory, one ring of
//            B slots per row), candidate blocks with an entry above max - 1;
//   refine - candidate blocks only: solver sums at the current tau, one hybrid-solver update;
//   P V    - candidate blocks: p = [z - tau]_+^k and u = [z - tau]_+^(k-1) rounded to bf16 into
//            shared memory (128B-swizzled, K-major) for the P V and U V MMAs; exact block mask; the
//            sums check sum p = 1 and the sweep repeats while any row's tau still moved.
// (AdaSplash-2, gist.science (de), section 2: histogram initialisation, hybrid solver, bit-packed
// block mask, only nonzero blocks processed; the histogram lives in on-chip memory, O(B) per row.)
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>

#include "common.cuh"
#include "fwd_common.cuh"
#include "launch.h"

namespace eattn {
namespace {

// K-major operands (128-byte rows, 8-row groups 1024 bytes apart) and MN-major operands stored as
// 64-column boxes of 64 rows (next 64 columns 8 KB further; next 8 rows 1024 bytes further)
constexpr uint64_t kDescK = sdesc_sw128_fields(16, 1024);
constexpr uint64_t kDescMN = sdesc_sw128_fields(64 * 128, 1024);

constexpr int BM = 128;           // query rows per tile
constexpr int BN = 64;            // keys per block (= mask block)
constexpr int kThreads = 192;
// dense sweep: histogram (u16, 64 KB) + stash (64 KB); the V ring after it
constexpr uint32_t kHistBytes = 256u * BM * 2u + kStashCap * BM * 4u;

template <int D>
struct Cfg {
    static constexpr int NKS = (D == 64) ? 4 : 3;          // K ring stages
    static constexpr int NVS = (D == 64) ? 6 : 4;          // V ring stages (inside the union region)
    static constexpr uint32_t kQBytes = BM * D * 2;        // 16 / 32 KB
    static constexpr uint32_t kKBytes = BN * D * 2;        // 8 / 16 KB per stage
    static constexpr uint32_t kPBytes = BM * BN * 2;       // 16 KB
    static constexpr uint32_t offQ = 0;
    static constexpr uint32_t offK = offQ + kQBytes;
    static constexpr int NPB = (D == 64) ? 2 : 1;          // P / U buffer sets in TMEM
    static constexpr uint32_t offU = offK + NKS * kKBytes;  // union region: histogram + stash, then V ring
    static constexpr uint32_t offV = offU;
    static_assert(NVS * kKBytes <= kHistBytes, "V ring must fit the union region");
    static_assert(NVS <= 8, "barrier arrays");
    static constexpr uint32_t offSmall = offU + kHistBytes;
    static constexpr uint32_t tmemCols = 512;
    static constexpr uint32_t colO = 128;
    static constexpr uint32_t colOb = 128 + D;
    // P / U operands of the P V and U V MMAs live in TMEM (A operand from tensor memory): per buffer set
    // 128 columns, one group of 32 per K step of 16 keys: [P high | P low | U high | U low], 8 columns
    // (16 bf16) each, so one 32-column store writes a K step of all four operands.
    static constexpr uint32_t colP = 128 + 2 * D;
    static_assert(colP + NPB * 128 <= tmemCols, "TMEM budget");
};

struct Small {
    uint64_t q_full;
    uint64_t k_full[4], k_empty[4];
    uint64_t v_full[8], v_empty[8];
    uint64_t s_full[2], s_empty[2];
    uint64_t p_full[2], p_empty[2];
    uint64_t o_full;
    uint64_t ctrl;
    uint64_t drain;
    uint32_t tmem_base;
    int abort_flag;
    int pad_;
    int plan_kind[2];
    TileStats st;
    float T[260];
    // followed by: plan_bits[2][W], next[W], mrow[2][W]
};

// OR of `pred` over the 128 compute threads (named barrier 1); every compute thread gets the result.
__device__ __forceinline__ bool bar_or_compute(bool pred) {
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

__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

// Out-of-line path of the dense sweep, taken when a row's stash may not hold another block: drop the
// entries that fell below the threshold; if the stash stays more than half full, the row switches to
// streaming its histogram (its stash is binned now) and is marked overflowed. Returns the new stash
// count, or -1.
static __device__ __noinline__ int stash_room(int n, HistRow& h, float* stash, uint16_t* hist, int r, float m_run,
                                              float thr, float cbin, int bins, int init_mode) {
    int j = 0;
    for (int i = 0; i < n; ++i) {
        const float v = stash[i * kTileRows + r];
        if (v > thr) stash[(j++) * kTileRows + r] = v;
    }
    if (j <= kStashCap / 2) return j;
    if (init_mode == 0) {
        Stash st;
        st.n = j;
        st.overflow = false;
        hist_from_stash(h, st, stash, m_run, thr, cbin, bins, hist, r);
    }
    return -1;
}

// Streaming path for a row whose stash overflowed: bin this block's entries above the threshold
// (rolled loop over the row's scores, staged in the row's now unused stash slots, rb[e * 128]).
static __device__ __noinline__ void stream_block(HistRow& h, const float* rb, uint32_t gflag, float thr, float cbin,
                                                 int bins, int init_mode, uint16_t* hist, int r) {
    if (init_mode != 0) return;
    while (gflag) {
        const int g = __ffs(gflag) - 1;
        gflag &= gflag - 1;
        for (int e = 0; e < 8; ++e) {
            const float v = rb[(8 * g + e) * kTileRows];
            if (v > thr) hist_add(h, v, cbin, bins, hist, r);
        }
    }
}

__device__ __forceinline__ bool block_full(int J, int n, int causal, int row0) {
    const int last = J * BN + BN - 1;
    return last < n && (!causal || last <= row0);
}

template <int D, int KIND>
__global__ void __launch_bounds__(kThreads, 1)
    fwd_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const FwdArgs a) {
    using C = Cfg<D>;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    // 1024-byte alignment for the 128B-swizzled tiles
    unsigned char* smem = align_smem_1024(smem_raw);
    Small& sm = *reinterpret_cast<Small*>(smem + C::offSmall);
    const int W = a.nw;
    uint32_t* plan_bits = reinterpret_cast<uint32_t*>(&sm + 1);  // [2][W]
    uint32_t* next = plan_bits + 2 * W;                          // [W]
    uint32_t* mrow = next + W;                                   // [2][W]
    uint16_t* hist = reinterpret_cast<uint16_t*>(smem + C::offU);                 // [256][128] u16
    float* stash = reinterpret_cast<float*>(smem + C::offU + 256 * BM * 2);        // [kStashCap][128]
    uint32_t* live_all = mrow + 2 * W;                                             // [128][kLiveStride]

    const SolveParams sp = a.sp;
    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const int qt = a.ntiles - 1 - (int)blockIdx.y;  // grid (B*H, tiles): longest tiles of every head first
    const int bh = blockIdx.x;
    const int row0 = qt * BM;
    const int kend = a.causal ? min(a.n, row0 + BM) : a.n;
    const int nblk = (kend + BN - 1) / BN;
    volatile int* abort_flag = &sm.abort_flag;

    if (tid == 0) {
        mbar_init(&sm.q_full, 1);
        for (int i = 0; i < C::NKS; ++i) { mbar_init(&sm.k_full[i], 1); mbar_init(&sm.k_empty[i], 1); }
        for (int i = 0; i < C::NVS; ++i) { mbar_init(&sm.v_full[i], 1); mbar_init(&sm.v_empty[i], 1); }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&sm.s_full[i], 1); mbar_init(&sm.s_empty[i], BM);
            mbar_init(&sm.p_full[i], BM); mbar_init(&sm.p_empty[i], 1);
        }
        mbar_init(&sm.o_full, 1);
        mbar_init(&sm.ctrl, BM);
        mbar_init(&sm.drain, 1);
        sm.abort_flag = 0;
        sm.st = TileStats{};
        fence_barrier_init();
    }
    if (warp == 0) {
        tmem_alloc(&sm.tmem_base, C::tmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    const uint32_t sQ = smem_u32(smem + C::offQ);
    const uint32_t sK0 = smem_u32(smem + C::offK);
    const uint32_t sV0 = smem_u32(smem + C::offV);

    if (warp == 5) {
        // ------------------------------------------------------------------ TMA issue
        if (lane == 0) {
            tma_prefetch_desc(&tmQ);
            tma_prefetch_desc(&tmK);
            tma_prefetch_desc(&tmV);
            mbar_arrive_expect_tx(&sm.q_full, C::kQBytes);
            for (int c = 0; c < D / 64; ++c)
                tma_load_3d(smem + C::offQ + c * (BM * 128), &tmQ, &sm.q_full, 64 * c, row0, bh);
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
                        const uint32_t ks = lc % C::NKS;
                        if (!(ok = wait_bounded(&sm.k_empty[ks], ((lc / C::NKS) & 1) ^ 1, abort_flag, a.status, true))) break;
                        mbar_arrive_expect_tx(&sm.k_full[ks], C::kKBytes);
                        for (int c = 0; c < D / 64; ++c)
                            tma_load_3d(smem + C::offK + ks * C::kKBytes + c * (BN * 128), &tmK, &sm.k_full[ks],
                                        64 * c, J * BN, bh);
                        ++lc;
                        if (kind == kSweepPV) {
                            const uint32_t vs = vc % C::NVS;
                            if (!(ok = wait_bounded(&sm.v_empty[vs], ((vc / C::NVS) & 1) ^ 1, abort_flag, a.status, true))) break;
                            mbar_arrive_expect_tx(&sm.v_full[vs], C::kKBytes);
                            for (int c = 0; c < D / 64; ++c)
                                tma_load_3d(smem + C::offV + vs * C::kKBytes + c * (BN * 128), &tmV,
                                            &sm.v_full[vs], 64 * c, J * BN, bh);
                            ++vc;
                        }
                    }
                }
            }
            if (!ok) {
                // drain copies still in flight before the CTA's shared memory is released
                for (uint32_t i = (lc > (uint32_t)C::NKS ? lc - C::NKS : 0); i < lc; ++i)
                    wait_drain(&sm.k_full[i % C::NKS], (i / C::NKS) & 1, 100000000ull);
                for (uint32_t i = (vc > (uint32_t)C::NVS ? vc - C::NVS : 0); i < vc; ++i)
                    wait_drain(&sm.v_full[i % C::NVS], (i / C::NVS) & 1, 100000000ull);
                wait_drain(&sm.q_full, 0, 100000000ull);
            }
        }
    } else if (warp == 4) {
        // ------------------------------------------------------------------ MMA issue
        if (lane == 0) {
            constexpr uint32_t idS = idesc_bf16_f32(BM, BN, false, false);
            constexpr uint32_t idPV = idesc_bf16_f32(BM, D, false, true);
            uint32_t lc = 0, vc = 0, sc = 0, pc = 0;
            bool ok = wait_bounded(&sm.q_full, 0, abort_flag, a.status, true);
            tc_fence_after();
            auto issue_S = [&](uint32_t ks) -> bool {
                const uint32_t sb = sc & 1;
                if (!wait_bounded(&sm.k_full[ks], (lc / C::NKS) & 1, abort_flag, a.status, true)) return false;
                if (!wait_bounded(&sm.s_empty[sb], ((sc >> 1) & 1) ^ 1, abort_flag, a.status, true)) return false;
                tc_fence_after();
                const uint32_t kbase = sK0 + ks * C::kKBytes;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t sub = kk >> 2, off = (kk & 3) * 32;
                    const uint64_t da = sdesc_at(kDescK, sQ + sub * (BM * 128) + off);
                    const uint64_t db = sdesc_at(kDescK, kbase + sub * (BN * 128) + off);
                    mma_ss(tmem + sb * BN, da, db, idS, kk > 0 ? 1u : 0u);
                }
                mma_commit(&sm.s_full[sb]);
                mma_commit(&sm.k_empty[ks]);
                ++lc;
                ++sc;
                return true;
            };
            auto issue_PV = [&](bool first) -> bool {
                const uint32_t pb = pc % C::NPB;
                const uint32_t vs = vc % C::NVS;
                if (!wait_bounded(&sm.p_full[pb], (pc / C::NPB) & 1, abort_flag, a.status, true)) return false;
                if (!wait_bounded(&sm.v_full[vs], (vc / C::NVS) & 1, abort_flag, a.status, true)) return false;
                tc_fence_after();
                const uint32_t vbase = sV0 + vs * C::kKBytes;
                const uint32_t tp = tmem + C::colP + pb * 128;
#pragma unroll
                for (int kk = 0; kk < BN / 16; ++kk) {
                    const uint64_t dv = sdesc_at(kDescMN, vbase + kk * 2048);
                    const uint32_t acc = (first && kk == 0) ? 0u : 1u;
                    // P = P_hi + P_lo and U = U_hi + U_lo (two bf16 terms each) keep P V and U V accurate
                    // to ~16 mantissa bits; each K step of 16 keys is 8 TMEM columns of the A tile
                    mma_ts(tmem + C::colO, tp + 32 * kk + 0, dv, idPV, acc);
                    mma_ts(tmem + C::colO, tp + 32 * kk + 8, dv, idPV, 1u);
                    mma_ts(tmem + C::colOb, tp + 32 * kk + 16, dv, idPV, acc);
                    mma_ts(tmem + C::colOb, tp + 32 * kk + 24, dv, idPV, 1u);
                }
                mma_commit(&sm.p_empty[pb]);
                mma_commit(&sm.v_empty[vs]);
                ++pc;
                ++vc;
                return true;
            };
            for (int sw = 0; ok; ++sw) {
                if (!(ok = wait_bounded(&sm.ctrl, sw & 1, abort_flag, a.status, true))) break;
                const int kind = sm.plan_kind[sw & 1];
                if (kind == kSweepDone) break;
                const uint32_t* bits_p = plan_bits + (sw & 1) * W;
                bool pending = false, first = true;
                for (int wd = 0; wd < W && ok; ++wd) {
                    uint32_t bits = bits_p[wd];
                    while (bits && ok) {
                        bits &= bits - 1;
                        if (!(ok = issue_S(lc % C::NKS))) break;
                        if (kind == kSweepPV) {
                            if (pending) {
                                if (!(ok = issue_PV(first))) break;
                                first = false;
                            }
                            pending = true;
                        }
                    }
                }
                if (ok && kind == kSweepPV) {
                    if (pending) ok = issue_PV(first);
                    if (ok) mma_commit(&sm.o_full);
                }
            }
            // make sure every MMA has finished before TMEM is released
            mma_commit(&sm.drain);
            wait_drain(&sm.drain, 0, 200000000ull);
        }
    } else {
        // ------------------------------------------------------------------ compute warps
        const int r = tid;  // row within the tile == TMEM lane
        const int row = row0 + r;
        const bool valid = row < a.n;
        const int n_i = valid ? allowed_keys(row, a.n, a.causal) : 1;
        const uint32_t lane_base = tmem + ((uint32_t)(warp * 32) << 16);
        const size_t head = (size_t)bh * a.n;
        const int half = r >> 6;  // which 64-row mask block of the tile

        for (int i = r; i <= sp.bins; i += BM) sm.T[i] = (KIND == kGeneric) ? powf((float)i, sp.k) : 0.0f;
        for (int i = r; i < W; i += BM) {
            const int lo = i * 32;
            uint32_t v = 0u;
            if (lo < nblk) v = (nblk - lo >= 32) ? 0xffffffffu : ((1u << (nblk - lo)) - 1u);
            plan_bits[i] = v;  // plan 0: every causal block
            next[i] = 0u;
        }
        if (r == 0) sm.plan_kind[0] = kSweepDense;
        named_bar_sync(1, BM);
        mbar_arrive(&sm.ctrl);

        uint32_t sc = 0, pc = 0;
        int sw = 0;
        bool ok = true;
        float vbuf[BN];

        // Load this row's S tile of the next block of the current sweep into vbuf (raw q.k).
        auto load_S = [&]() -> bool {
            const uint32_t sb = sc & 1;
            const bool got = wait_bounded(&sm.s_full[sb], (sc >> 1) & 1, abort_flag, a.status);
            if (!__all_sync(0xffffffffu, got)) return false;
            tc_fence_after();
            __syncwarp();
            uint32_t* rr = reinterpret_cast<uint32_t*>(vbuf);
            tmem_ld32(lane_base + sb * BN, rr);
            tmem_ld32(lane_base + sb * BN + 32, rr + 32);
            tmem_ld_wait();
            tc_fence_before();
            mbar_arrive(&sm.s_empty[sb]);
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
            // next[] holds the keep bits of the sweep just finished
            named_bar_sync(1, BM);
            const int nb = (sw + 1) & 1;
            for (int i = r; i < W; i += BM) {
                plan_bits[nb * W + i] = next[i];
                next[i] = 0u;
            }
            if (kind == kSweepPV)
                for (int i = r; i < 2 * W; i += BM) mrow[i] = 0u;
            if (r == 0) sm.plan_kind[nb] = kind;
            named_bar_sync(1, BM);
            ++sw;
            mbar_arrive(&sm.ctrl);
        };

        // 8 groups of 8 scores: group maxima (3-input max), the block max, and per-group tests that
        // skip the rare-path work for groups without a candidate entry.
        float gm[8];
        auto group_max = [&]() -> float {
#pragma unroll
            for (int g = 0; g < 8; ++g) {
                const float* v = vbuf + 8 * g;
                gm[g] = fmax3(fmax3(v[0], v[1], v[2]), fmax3(v[3], v[4], v[5]), fmaxf(v[6], v[7]));
            }
            return fmax3(fmax3(gm[0], gm[1], gm[2]), fmax3(gm[3], gm[4], gm[5]), fmaxf(gm[6], gm[7]));
        };

        // ---- sweep 0: dense ----
        HistRow h;
        hist_init(h, live_all, r);
        Stash sh;
        sh.n = 0;
        sh.overflow = false;
        // Candidates (z > running max - 1) go to the stash; the histogram is built from the stash when
        // the sweep ends (one binning per candidate instead of one window update per block). Rows whose
        // stash overflows stream their histogram from then on.
        float m_run = -INFINITY, thr = INFINITY;
        int nst = 0;           // stash entries
        bool ovf = false;      // stash overflowed: streaming histogram
        for (int J = 0; J < nblk && ok; ++J) {
            if (!(ok = load_S())) break;
            mask_S(J);
            const float amax = group_max();
            if (amax > m_run) {
                m_run = amax;
                thr = amax - sp.inv_cz;
                if (ovf && sp.init_mode == 0) hist_raise(h, amax, sp.cbin, sp.inv_cz, sp.bins);
            }
            const bool any = amax > thr;
            if (__any_sync(0xffffffffu, any)) {
                // make room for a whole block first (at most once per block, out of line)
                const bool room = any && !ovf && nst > kStashCap - BN;
                if (__any_sync(0xffffffffu, room)) {
                    if (room) {
                        nst = stash_room(nst, h, stash, hist, r, m_run, thr, sp.cbin, sp.bins, sp.init_mode);
                        if (nst < 0) { ovf = true; nst = 0; }
                    }
                }
                // stash path, warp-uniform per group; predicated stores inside
#pragma unroll
                for (int g = 0; g < 8; ++g) {
                    const bool fl = !ovf && gm[g] > thr;
                    if (__any_sync(0xffffffffu, fl)) {
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            const float v = vbuf[8 * g + e];
                            const bool q = fl && v > thr;
                            if (q) stash[nst * BM + r] = v;
                            nst += q ? 1 : 0;
                        }
                    }
                }
                // rows that stream their histogram: rolled loop over the block's flagged groups
                const bool strm = any && ovf && sp.init_mode == 0;
                if (__any_sync(0xffffffffu, strm)) {
                    if (strm) {
                        uint32_t gflag = 0u;
#pragma unroll
                        for (int g = 0; g < 8; ++g) gflag |= (gm[g] > thr ? 1u : 0u) << g;
#pragma unroll
                        for (int c = 0; c < BN; ++c) stash[c * BM + r] = vbuf[c];
                        stream_block(h, stash + r, gflag, thr, sp.cbin, sp.bins, sp.init_mode, hist, r);
                    }
                }
            }
            const uint32_t ball = __ballot_sync(0xffffffffu, any);
            if (lane == 0 && ball) atomicOr(&next[J >> 5], 1u << (J & 31));
        }
        ok = !bar_or_compute(!ok || *abort_flag != 0);
        sh.n = nst;
        sh.overflow = ovf;
        if (!ovf) {
            if (sp.init_mode == 0) hist_from_stash(h, sh, stash, m_run, thr, sp.cbin, sp.bins, hist, r);
            h.m_raw = m_run;
            h.thr_raw = thr;
            h.any = m_run > -INFINITY;
        }

        const float m = sp.cz * h.m_raw;
        float tau_h = m - 1.0f;
        if (ok && valid && sp.init_mode == 0) tau_h = hist_tau<KIND>(h, sp, hist, r, sm.T);
        RowSolve s;
        solve_init(s, valid ? tau_h : 0.0f, valid ? m : 1.0f, n_i, sp);
        if (!valid) s.done = true;
        if (valid && a.tau_hist) a.tau_hist[head + row] = tau_h;
        // rows whose candidates all fit the stash are solved on chip, with no further key sweep
        if (ok && valid && !sh.overflow) {
            for (int it = 0; it < kMaxSweeps && !s.done; ++it) {
                float F0, F1, F2, F0b;
                stash_sums<KIND>(sh, stash, r, sp.cz, sp.k, s.tau, s.tau2, s.need_two, F0, F1, F2, F0b);
                solve_step(s, F0, F1, F2, F0b, sp);
            }
        }

        // ---- refinement sweep: solver sums at the current tau over the candidate blocks ----
        float last_step = INFINITY;
        int refine = 0, pv = 0;
        auto refine_sweep = [&]() {
            publish(kSweepRefine);
            float F0 = 0.f, F1 = 0.f, F2 = 0.f, F0b = 0.f;
            const float t = s.tau, t2 = s.tau2, lo0 = s.lo;
            const bool two = s.need_two;
            const uint32_t* bits_p = plan_bits + (sw & 1) * W;
            for (int wd = 0; wd < W && ok; ++wd) {
                uint32_t bits = bits_p[wd];
                while (bits) {
                    const int J = wd * 32 + __ffs(bits) - 1;
                    bits &= bits - 1;
                    if (!(ok = load_S())) break;
                    mask_S(J);
                    const float amax = group_max();
                    const bool keep = sp.cz * amax > lo0;
                    if (sp.cz * amax - t > 0.f) {
#pragma unroll
                        for (int g = 0; g < 8; ++g) {
                            if (sp.cz * gm[g] - t > 0.f) {
#pragma unroll
                                for (int e = 0; e < 8; ++e) {
                                    const float z = sp.cz * vbuf[8 * g + e];
                                    const float x = z - t;
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
                                        const float x2 = z - t2;
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
            const float before = s.tau;
            solve_step(s, F0, F1, F2, F0b, sp);
            last_step = s.tau - before;
            ++refine;
            ok = !bar_or_compute(!ok || *abort_flag != 0);
        };

        // ---- P V sweep: p, u to shared memory for the P V / U V MMAs, exact mask, sum check ----
        float Su = 0.f;
        uint32_t nsup = 0;  // nonzero probabilities of this row in the last P V sweep
        auto pv_sweep = [&]() -> bool {
            publish(kSweepPV);
            float Sp = 0.f, F2 = 0.f;
            Su = 0.f;
            nsup = 0;
            const float t = s.tau, lo0 = s.lo;
            const uint32_t* bits_p = plan_bits + (sw & 1) * W;
            for (int wd = 0; wd < W && ok; ++wd) {
                uint32_t bits = bits_p[wd];
                while (bits) {
                    const int J = wd * 32 + __ffs(bits) - 1;
                    bits &= bits - 1;
                    if (!(ok = load_S())) break;
                    mask_S(J);
                    const float amax = group_max();
                    const bool keep = sp.cz * amax > lo0;
                    const bool nz = sp.cz * amax - t > 0.f;
                    const uint32_t pb = pc % C::NPB;
                    ok = __all_sync(0xffffffffu,
                                    wait_bounded(&sm.p_empty[pb], ((pc / C::NPB) & 1) ^ 1, abort_flag, a.status));
                    if (!ok) break;
                    const uint32_t tp = lane_base + C::colP + pb * 128;
#pragma unroll
                    for (int gp = 0; gp < 4; ++gp) {
                        // two groups of 8 keys = one K step: 8 columns of each of the four operands
                        uint32_t ks[32];  // [P high 8 | P low 8 | U high 8 | U low 8]
                        uint32_t* ph = ks;
                        uint32_t* pl = ks + 8;
                        uint32_t* uh = ks + 16;
                        uint32_t* ul = ks + 24;
#pragma unroll
                        for (int q8 = 0; q8 < 2; ++q8) {
                            const int g = 2 * gp + q8;
                            if (sp.cz * gm[g] - t > 0.f) {
#pragma unroll
                                for (int e = 0; e < 8; e += 2) {
                                    float pv2[2], uv2[2];
#pragma unroll
                                    for (int q = 0; q < 2; ++q) {
                                        const float x = sp.cz * vbuf[8 * g + e + q] - t;
                                        float p, u;
                                        if constexpr (KIND == kAlpha15) {
                                            u = fmaxf(x, 0.f);
                                            p = u * u;
                                            F2 += x > 0.f ? 1.f : 0.f;
                                        } else if constexpr (KIND == kAlpha2) {
                                            p = fmaxf(x, 0.f);
                                            u = x > 0.f ? 1.f : 0.f;
                                        } else {
                                            const bool pos = x > 0.f;
                                            const float xs = pos ? x : 1.f;
                                            const float uu1 = exp2f((sp.k - 1.f) * __log2f(xs));
                                            u = pos ? uu1 : 0.f;
                                            p = u * xs;
                                            F2 += pos ? __fdividef(uu1, xs) : 0.f;
                                        }
                                        Sp += p;
                                        Su += u;
                                        nsup += x > 0.f ? 1u : 0u;
                                        pv2[q] = p;
                                        uv2[q] = u;
                                    }
                                    const int w = q8 * 4 + e / 2;
                                    const __nv_bfloat162 hi = __floats2bfloat162_rn(pv2[0], pv2[1]);
                                    const float2 hf = __bfloat1622float2(hi);
                                    ph[w] = *reinterpret_cast<const uint32_t*>(&hi);
                                    pl[w] = pack_bf16x2(pv2[0] - hf.x, pv2[1] - hf.y);
                                    const __nv_bfloat162 uh2 = __floats2bfloat162_rn(uv2[0], uv2[1]);
                                    const float2 uf = __bfloat1622float2(uh2);
                                    uh[w] = *reinterpret_cast<const uint32_t*>(&uh2);
                                    ul[w] = pack_bf16x2(uv2[0] - uf.x, uv2[1] - uf.y);
                                }
                            } else {
#pragma unroll
                                for (int w = q8 * 4; w < q8 * 4 + 4; ++w) ph[w] = pl[w] = uh[w] = ul[w] = 0u;
                            }
                        }
                        tmem_st32(tp + 32 * gp, ks);
                    }
                    tmem_st_wait();
                    mbar_arrive(&sm.p_full[pb]);
                    ++pc;
                    const uint32_t kb = __ballot_sync(0xffffffffu, keep);
                    const uint32_t nb = __ballot_sync(0xffffffffu, nz);
                    if (lane == 0) {
                        if (kb) atomicOr(&next[J >> 5], 1u << (J & 31));
                        if (nb) atomicOr(&mrow[half * W + (J >> 5)], 1u << (J & 31));
                    }
                }
            }
            ++pv;
            const float before = s.tau;
            solve_step(s, Sp, Su, F2, 0.f, sp);
            const bool changed = s.tau != before;
            ok = !bar_or_compute(!ok || *abort_flag != 0);
            return ok && bar_or_compute(changed);
        };

        // Schedule: refine while some row still takes steps wider than one bin; then P V, whose sums
        // double as the check of sum p = 1. If any tau still moved, refine until every row has
        // stopped (cheaper than repeated P V sweeps) and finish with one more P V sweep.
        if (ok && bar_or_compute(!s.done)) {
            do {
                refine_sweep();
            } while (ok && refine < kMaxSweeps &&
                     bar_or_compute(!s.done && fabsf(last_step) > sp.w));
        }
        while (ok) {
            const bool changed = pv_sweep();
            if (!ok || !changed || pv >= 3) break;
            while (ok && refine < kMaxSweeps && bar_or_compute(!s.done)) refine_sweep();
        }

        // ---- wait for the last P V MMAs, then write O, U V, tau, sum u, mask ----
        if (ok) ok = __all_sync(0xffffffffu, wait_bounded(&sm.o_full, (pv - 1) & 1, abort_flag, a.status));
        ok = !bar_or_compute(!ok || *abort_flag != 0);
        if (ok) {
            tc_fence_after();
            __syncwarp();
            __nv_bfloat16* Oh = static_cast<__nv_bfloat16*>(a.O) + head * D;
            float* Obh = a.obar + head * D;
#pragma unroll
            for (int c0 = 0; c0 < D; c0 += 32) {
                uint32_t o[32], ob[32];
                tmem_ld32(lane_base + C::colO + c0, o);
                tmem_ld32(lane_base + C::colOb + c0, ob);
                tmem_ld_wait();
                if (valid) {
                    uint4* dst = reinterpret_cast<uint4*>(Oh + (size_t)row * D + c0);
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const float* f = reinterpret_cast<const float*>(o + 8 * i);
                        dst[i] = make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]),
                                            pack_bf16x2(f[4], f[5]), pack_bf16x2(f[6], f[7]));
                    }
                    float4* dob = reinterpret_cast<float4*>(Obh + (size_t)row * D + c0);
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const float* f = reinterpret_cast<const float*>(ob + 4 * i);
                        dob[i] = make_float4(f[0], f[1], f[2], f[3]);
                    }
                }
            }
            tc_fence_before();
            if (valid) {
                a.tau[head + row] = s.tau;
                a.sum_u[head + row] = Su;
                if (a.steps) a.steps[head + row] = (uint8_t)s.steps;
            }
        }
        // tell the issuing warps to stop
        if (r == 0) sm.plan_kind[(sw + 1) & 1] = kSweepDone;
        named_bar_sync(1, BM);
        mbar_arrive(&sm.ctrl);

        // mask rows of this tile (two 64-row query blocks)
        named_bar_sync(1, BM);
        for (int i = r; i < 2 * W; i += BM) {
            const int qb = qt * 2 + i / W;
            if (qb < a.nqb) a.mask[((size_t)bh * a.nqb + qb) * W + (i % W)] = ok ? mrow[i] : 0u;
        }
        if (a.stats && ok) {
            const uint32_t* cb = plan_bits + (sw & 1) * W;
            uint32_t nzb = 0, cnd = 0;
            for (int i = r; i < 2 * W; i += BM) nzb += __popc(mrow[i]);
            for (int i = r; i < W; i += BM) cnd += __popc(cb[i]);
            if (nzb) atomicAdd(&sm.st.nonzero_blocks, nzb);
            if (cnd) atomicAdd(&sm.st.candidate_blocks, cnd);
            if (valid) {
                if (sh.overflow) atomicAdd(&sm.st.overflow_rows, 1u);
                atomicAdd(&sm.st.rows, 1u);
                atomicAdd(&sm.st.support, nsup);
                atomicAdd(&sm.st.steps, (uint32_t)s.steps);
                atomicAdd(&sm.st.fallbacks, (uint32_t)s.fallbacks);
                atomicAdd(&sm.st.step_hist[min(s.steps, kMaxSteps)], 1u);
            }
            named_bar_sync(1, BM);
            if (r == 0) {
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
        tmem_dealloc(tmem, C::tmemCols);
    }
}

}  // namespace

// ---------------------------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------------------------
namespace {

using EncodeTiled = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                 const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                 CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiled get_encode() {
    static EncodeTiled fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiled>(p);
    }
    return fn;
}

}  // namespace

// [BH, n, d] tensor of 16-bit elements, boxes of `rows` x 64 columns, 128B swizzle; zero fill past n.
static cudaError_t make_tmap_16(CUtensorMap* map, const void* base, int BH, int n, int d, int rows,
                                CUtensorMapDataType type) {
    EncodeTiled enc = get_encode();
    if (!enc) return cudaErrorNotSupported;
    cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)n, (cuuint64_t)BH};
    cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)n * d * 2};
    cuuint32_t box[3] = {64, (cuuint32_t)rows, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = enc(map, type, 3, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                     CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

cudaError_t make_tmap_bf16(CUtensorMap* map, const void* base, int BH, int n, int d, int rows) {
    return make_tmap_16(map, base, BH, n, d, rows, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16);
}

cudaError_t make_tmap_f16(CUtensorMap* map, const void* base, int BH, int n, int d, int rows) {
    return make_tmap_16(map, base, BH, n, d, rows, CU_TENSOR_MAP_DATA_TYPE_FLOAT16);
}

template <int D, int KIND>
static cudaError_t launch_fwd_tc_t(const FwdArgs& a, cudaStream_t stream) {
    using C = Cfg<D>;
    CUtensorMap tq, tk, tv;
    cudaError_t e;
    if ((e = make_tmap_bf16(&tq, a.Q, a.B * a.H, a.n, D, BM)) != cudaSuccess) return e;
    if ((e = make_tmap_bf16(&tk, a.K, a.B * a.H, a.n, D, BN)) != cudaSuccess) return e;
    if ((e = make_tmap_bf16(&tv, a.V, a.B * a.H, a.n, D, BN)) != cudaSuccess) return e;
    const size_t bytes = 1024 + C::offSmall + sizeof(Small) + (size_t)5 * a.nw * 4 + (size_t)BM * kLiveStride * 4;
    if (bytes > 232448) return cudaErrorInvalidConfiguration;
    auto kern = fwd_tc_kernel<D, KIND>;
    if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes)) != cudaSuccess)
        return e;
    dim3 grid(a.B * a.H, a.ntiles);
    launch_mark(stream);
    kern<<<grid, kThreads, bytes, stream>>>(tq, tk, tv, a);
    return cudaGetLastError();
}

size_t fwd_tc_smem_bytes(int d, int nw) {
    const size_t small = sizeof(Small) + (size_t)5 * nw * 4 + (size_t)BM * kLiveStride * 4;
    return 1024 + (d == 64 ? Cfg<64>::offSmall : Cfg<128>::offSmall) + small;
}

cudaError_t launch_fwd_tc(const FwdArgs& a, cudaStream_t stream) {
    if (a.d == 64) {
        if (a.sp.alpha == 1.5f) return launch_fwd_tc_t<64, kAlpha15>(a, stream);
        if (a.sp.alpha == 2.0f) return launch_fwd_tc_t<64, kAlpha2>(a, stream);
        return launch_fwd_tc_t<64, kGeneric>(a, stream);
    }
    if (a.sp.alpha == 1.5f) return launch_fwd_tc_t<128, kAlpha15>(a, stream);
    if (a.sp.alpha == 2.0f) return launch_fwd_tc_t<128, kAlpha2>(a, stream);
    return launch_fwd_tc_t<128, kGeneric>(a, stream);
}

}  // namespace eattn
