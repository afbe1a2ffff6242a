// entmax_row.cuh - per-query-row pieces of the alpha-entmax normaliser, run by the thread that owns
// the row: the left-edge score histogram, its root tau_h, and the safeguarded hybrid solver step.
//
// Notation: raw score a = q.k (unscaled), z = cz * a with cz = (alpha - 1) * scale, k = 1/(alpha-1),
// f(tau) = sum_j [z_j - tau]_+^k - 1, root tau*.
//
// Histogram ("AdaSplash-2", gist.science (de), section 2, "Streaming & Histogramm-Erstellung" and
// "Theoretische Garantie"): B bins of width w = 1/(B-1) over z, bin b = floor(z / w), left edge
// e_b = b w <= z. The window keeps the B bins top-(B-1) .. top, top = floor(m_run / w) of the running
// max, in a ring of B slots (slot = b mod B); when the max rises, the slots of the bins that fall
// below the window are cleared. Only entries with z > m_run - 1 are binned: everything in the final
// support has z > tau* >= m - 1. Replacing each z by e_b and dropping entries only lowers f, so the
// root tau_h of the binned function is a lower bound on tau*, and tau_h + w is an upper bound.
//
// Solver ("Hybrid Solver & Sparsity-Awareness"; gist.science (hi) technical summary, section 2):
// Halley for alpha <= 1.5, Newton for 1.5 < alpha <= 2, secant above 2, bisection when a step leaves
// the bracket. A row stops when |f| <= ftol, when a step moves tau by <= xtol max(1, |tau|), or after
// kMaxSteps steps.
#pragma once

#include <stdint.h>

namespace eattn {

enum AlphaKind : int { kGeneric = 0, kAlpha2 = 1, kAlpha15 = 2 };
enum Method : int { kHalley = 0, kNewton = 1, kSecant = 2 };

constexpr int kMaxSteps = 8;  // last bin of the step histogram ("8 or more")
constexpr int kMaxSweeps = 30;
constexpr float kFtol = 1e-5f;
constexpr float kXtol = 1e-6f;
constexpr int kTileRows = 128;  // query rows per CTA; hist slot s of row r lives at hist[s * 128 + r]

struct SolveParams {
    float alpha, k, cz, inv_cz, cbin, w;
    int bins;
    int method;
    int init_mode;  // 0: histogram start; 1: plain bracket start
};

__host__ __device__ inline SolveParams make_solve_params(float alpha, float scale, int bins, int init_mode) {
    SolveParams p;
    p.alpha = alpha;
    p.k = 1.0f / (alpha - 1.0f);
    p.cz = (alpha - 1.0f) * scale;
    p.inv_cz = 1.0f / p.cz;
    p.bins = bins;
    p.w = 1.0f / (float)(bins - 1);
    p.cbin = p.cz * (float)(bins - 1);
    p.method = alpha <= 1.5f ? kHalley : (alpha <= 2.0f ? kNewton : kSecant);
    p.init_mode = init_mode;
    return p;
}

// x^k for x > 0.
template <int KIND>
__device__ __forceinline__ float pow_k(float x, float k) {
    if constexpr (KIND == kAlpha15) return x * x;
    else if constexpr (KIND == kAlpha2) return x;
    else return exp2f(k * __log2f(x));
}

// Accumulate x^k, x^(k-1), x^(k-2) for one support entry (x > 0).
template <int KIND>
__device__ __forceinline__ void add_sums(float x, float k, float& F0, float& F1, float& F2) {
    if constexpr (KIND == kAlpha15) {
        F0 = fmaf(x, x, F0);
        F1 += x;
        F2 += 1.0f;
    } else if constexpr (KIND == kAlpha2) {
        F0 += x;
        F1 += 1.0f;
    } else {
        const float l = __log2f(x);
        const float pk1 = exp2f((k - 1.0f) * l);
        F0 = fmaf(pk1, x, F0);
        F1 += pk1;
        F2 += __fdividef(pk1, x);
    }
}

// ---------------------------------------------------------------------------------------------
// Histogram ring (thread-owned row).
//   hist  u16 [B slots][128 rows]; counts saturate at 65535 (a saturated count only drops entries,
//         which keeps the bound);
//   live  u32 [128 rows][stride]: bit s of row r's B / 32 words (8 for B <= 256, 16 for B = 512) marks
//         slot s as holding a counted bin of the current window. Sliding the window clears bits instead
//         of counts, so the histogram needs no zeroing and a slide costs a few word operations.
// ---------------------------------------------------------------------------------------------
constexpr int kLiveStride = 9;      // words per row for B <= 256 (8 used; odd stride: rows on distinct banks)
constexpr int kLiveStride512 = 17;  // words per row for B = 512 (16 used)

struct HistRow {
    float m_raw;     // running max of the raw score
    float thr_raw;   // raw threshold for binning: z > m_run - 1
    int top;         // bin index of the running max
    bool any;        // any entry seen
    int nlw;         // live words per row (stride - 1)
    uint32_t* live;  // this row's live words in shared memory
};

__host__ __device__ __forceinline__ void hist_init(HistRow& h, uint32_t* live_all, int r, int stride = kLiveStride) {
    h.m_raw = -INFINITY;
    h.thr_raw = INFINITY;
    h.top = 0;
    h.any = false;
    h.nlw = stride - 1;
    h.live = live_all + r * stride;
    for (int i = 0; i < h.nlw; ++i) h.live[i] = 0u;
}

__device__ __forceinline__ int bin_of(float a, float cbin) {
    float y = fminf(fmaxf(a * cbin, -1.0e9f), 1.0e9f);
    return __float2int_rd(y);
}

// Word i of the bits [s0, s0 + len) of a B-bit ring (B a power of two, 32 <= B <= 512, len < B; words at
// or beyond B / 32 are 0), host-testable.
__host__ __device__ __forceinline__ uint32_t ring_word_mask(int i, int s0, int len, int B) {
    const int lo = i * 32;
    if (lo >= B) return 0u;
    uint32_t m = 0u;
    const int a0 = (lo - s0) & (B - 1);  // offset of bit 0 of this word from s0
    if (a0 < len) m = (len - a0 >= 32) ? 0xffffffffu : ((1u << (len - a0)) - 1u);
    const int wrap = a0 + 32 - B;  // bits of this word whose offset wrapped past B
    if (wrap > 0) {
        const int cnt = min(wrap, len);
        if (cnt > 0) m |= ((cnt >= 32) ? 0xffffffffu : ((1u << cnt) - 1u)) << (32 - wrap);
    }
    return m;
}

// Raise the running max to `a_max` (raw) and slide the window.
__device__ __forceinline__ void hist_raise(HistRow& h, float a_max, float cbin, float inv_cz, int B) {
    if (!(a_max > h.m_raw)) return;
    const int nt = bin_of(a_max, cbin);
    if (h.any && nt > h.top) {
        const int d = nt - h.top;
        if (d >= B) {
            for (int i = 0; i < h.nlw; ++i) h.live[i] = 0u;
        } else {
            const int s0 = (h.top + 1) & (B - 1);
            for (int i = 0; i < h.nlw; ++i) {
                const uint32_t m = ring_word_mask(i, s0, d, B);
                if (m) h.live[i] &= ~m;
            }
        }
    }
    h.top = h.any ? max(h.top, nt) : nt;
    h.any = true;
    h.m_raw = a_max;
    h.thr_raw = a_max - inv_cz;
}

// Bin one raw score that passed a > thr_raw.
__device__ __forceinline__ void hist_add(const HistRow& h, float a, float cbin, int B, uint16_t* hist, int r) {
    const int b = bin_of(a, cbin);
    const int j = h.top - b;
    if (j >= 0 && j < B) {
        const int s = b & (B - 1);
        uint16_t* c = &hist[s * kTileRows + r];
        const uint32_t w = h.live[s >> 5], bit = 1u << (s & 31);
        if (w & bit) {
            const uint16_t v = *c;
            if (v != 0xffffu) *c = (uint16_t)(v + 1u);
        } else {
            *c = 1u;
            h.live[s >> 5] = w | bit;
        }
    }
}

// ---------------------------------------------------------------------------------------------
// Candidate stash (thread-owned row): raw scores of the entries binned while streaming, in shared
// memory stash[i * 128 + r], i < kStashCap. Every entry of the final support is among them (it lies
// above m - 1 >= m_run - 1), so the solver sums at any tau >= m_run - 1 can be taken over the stash
// instead of another sweep over the keys. When the stash fills up, entries at or below the current
// threshold are dropped; if that leaves it more than half full, the row is marked overflowed (it falls
// back to sweeps) so that the pruning work stays amortised O(1) per entry.
// ---------------------------------------------------------------------------------------------
constexpr int kStashCap = 128;

struct Stash {
    int n;
    bool overflow;
};

__device__ __forceinline__ void stash_add(Stash& st, float a, float thr_raw, float* stash, int r) {
    if (st.overflow) return;
    if (st.n == kStashCap) {
        int j = 0;
        for (int i = 0; i < kStashCap; ++i) {
            const float v = stash[i * kTileRows + r];
            if (v > thr_raw) stash[(j++) * kTileRows + r] = v;
        }
        st.n = j;
        if (j > kStashCap / 2) { st.overflow = true; return; }
    }
    stash[(st.n++) * kTileRows + r] = a;
}

// Bin every stash entry above thr_raw into a histogram whose window top is the bin of m_raw (the row's
// running max so far). Used once per row: at the end of the dense sweep, or when the stash overflows and
// the row switches to streaming the histogram.
__device__ __forceinline__ void hist_from_stash(HistRow& h, const Stash& st, const float* stash, float m_raw,
                                                float thr_raw, float cbin, int B, uint16_t* hist, int r) {
    for (int i = 0; i < h.nlw; ++i) h.live[i] = 0u;
    h.any = m_raw > -INFINITY;
    h.m_raw = m_raw;
    h.thr_raw = thr_raw;
    h.top = h.any ? bin_of(m_raw, cbin) : 0;
    for (int i = 0; i < st.n; ++i) {
        const float v = stash[i * kTileRows + r];
        if (v > thr_raw) hist_add(h, v, cbin, B, hist, r);
    }
}

// Solver sums over the stash at tau (and the secant's second point tau2 when `two`).
template <int KIND>
__device__ __forceinline__ void stash_sums(const Stash& st, const float* stash, int r, float cz, float k, float tau,
                                           float tau2, bool two, float& F0, float& F1, float& F2, float& F0b) {
    F0 = F1 = F2 = F0b = 0.f;
    for (int i = 0; i < st.n; ++i) {
        const float z = cz * stash[i * kTileRows + r];
        const float x = z - tau;
        if (x > 0.f) add_sums<KIND>(x, k, F0, F1, F2);
        if (two) {
            const float x2 = z - tau2;
            if (x2 > 0.f) F0b += pow_k<KIND>(x2, k);
        }
    }
}

// Root tau_h of the left-edge binned function, in z units (a lower bound on tau*).
// For k = 1 and k = 2 the root is found in closed form on its segment (exact integer moments); for
// other k by a search over the bin edges and then bisection inside the segment, keeping the end where
// f >= 0. T[i] = i^k for i = 0..B (generic k only). The result is lowered by a few float32 ulps so that
// rounding cannot lift it above the binned root. I is the integer type of the moments: int is exact while
// the row holds at most a few hundred entries (every moment stays below 2^31 before the crossing: A0 <= 2^9,
// offsets <= 2^9), long long for any count.
template <int KIND, typename I = long long>
__host__ __device__ float hist_tau(const HistRow& h, const SolveParams& sp, const uint16_t* hist, int r, const float* T) {
    const int B = sp.bins;
    float tau_h;
    if constexpr (KIND == kAlpha15 || KIND == kAlpha2) {
        // A0 = sum c_j, A1 = sum c_j (J - j), A2 = sum c_j (J - j)^2 over offsets j < J (exact integers).
        // Only live bins are visited (set bits of the live mask, in order of offset j = top - bin); between
        // them the moments move in closed form, and the first J at which the binned function reaches 0
        // (A2 >= (B-1)^2, or A1 >= B-1 for k = 1) is found by a float estimate corrected in integers.
        I A0 = 0, A1 = 0, A2 = 0;
        const I thr = (KIND == kAlpha15) ? (I)(B - 1) * (B - 1) : (I)(B - 1);
        auto Ak = [&](I t) -> I {  // A_k(J0 + t) from the moments at J0
            return (KIND == kAlpha15) ? A2 + 2 * t * A1 + t * t * A0 : A1 + t * A0;
        };
        auto first_cross = [&]() -> I {  // smallest t >= 1 with A_k(J0 + t) >= thr (A0 > 0)
            float tf;
            if constexpr (KIND == kAlpha15) {
                const float a0 = (float)A0, a1 = (float)A1, d2 = (float)(A2 - thr);
                tf = (-a1 + sqrtf(fmaxf(a1 * a1 - a0 * d2, 0.0f))) / a0;
            } else {
                tf = (float)(thr - A1) / (float)A0;
            }
            I t = (I)fmaxf(1.0f, ceilf(tf));
            while (t > 1 && Ak(t - 1) >= thr) --t;
            while (Ak(t) < thr) ++t;
            return t;
        };
        const int stop = h.top & (B - 1);
        const int nw = B >= 32 ? B / 32 : 1;
        int J = B - 1, J0 = 0;  // moments are evaluated at J0 (bins with offset < J0)
        bool found = false;
        // visit slots stop, stop-1, ..., 0, B-1, ..., stop+1: word by word from the word holding `stop`
        for (int step = 0; step <= nw && !found; ++step) {
            const int wi = ((stop >> 5) - step + 2 * nw) % nw;
            uint32_t bits = h.live[wi];
            if (B < 32) bits &= (1u << B) - 1u;
            if (step == 0) bits &= (stop & 31) == 31 ? 0xffffffffu : ((2u << (stop & 31)) - 1u);   // slots <= stop
            if (step == nw) bits &= (stop & 31) == 31 ? 0u : ~((2u << (stop & 31)) - 1u);        // slots > stop
            while (bits && !found) {
#ifdef __CUDA_ARCH__
                const int bpos = 31 - __clz(bits);
#else
                const int bpos = 31 - __builtin_clz(bits);
#endif
                bits &= ~(1u << bpos);
                const int sl = wi * 32 + bpos;
                const I c = hist[sl * kTileRows + r];
                if (c == 0) continue;
                const int jn = (stop - sl) & (B - 1);  // offset of this bin below the top
                const int J1 = jn + 1;                 // first J at which the bin counts
                if (A0 > 0) {
                    const I T = J1 - J0;
                    // crosses before this bin starts to count iff A_k(J1 - 1) reaches thr (A_k is
                    // nondecreasing in J); only then is the crossing located
                    if (T >= 2 && Ak(T - 1) >= thr) {
                        const I t = first_cross();
                        A2 = (KIND == kAlpha15) ? Ak(t) : A2;
                        A1 += t * A0;
                        J = J0 + (int)t;
                        found = true;
                        break;
                    }
                    A2 += 2 * T * A1 + T * T * A0;
                    A1 += T * A0;
                }
                A0 += c;
                A1 += c;
                A2 += c;
                J0 = J1;
                if (((KIND == kAlpha15) ? A2 : A1) >= thr) { J = J1; found = true; }
            }
        }
        if (!found && A0 > 0) {
            const I t = first_cross();
            A2 = (KIND == kAlpha15) ? Ak(t) : A2;
            A1 += t * A0;
            J = J0 + (int)t;
        }
        if (J >= B) J = B - 1;
        float u;  // tau_h = (top - J + u) w, u in [0, 1)
        const float a0 = (float)A0, a1 = (float)A1, a2 = (float)A2;
        if constexpr (KIND == kAlpha15) {
            const float disc = fmaxf(a1 * a1 - a0 * (a2 - (float)thr), 0.0f);
            u = (a1 - sqrtf(disc)) / a0;
        } else {
            u = (a1 - (float)thr) / a0;
        }
        u = fminf(fmaxf(u, 0.0f), 1.0f);
        tau_h = ((float)(h.top - J) + u) * sp.w;
    } else {
        const float thr = T[B - 1];
        // visit the nonzero bins at offsets j < J in ascending j (live slots stop, stop - 1, ..., 0, B - 1, ...,
        // stop + 1, word by word), so that each evaluation costs the row's nonzero bins, not J
        const int stop = h.top & (B - 1);
        const int nw = B >= 32 ? B / 32 : 1;
        auto for_nonzero = [&](int J, auto&& fn) {
            for (int step = 0; step <= nw; ++step) {
                const int wi = ((stop >> 5) - step + 2 * nw) % nw;
                uint32_t bits = h.live[wi];
                if (B < 32) bits &= (1u << B) - 1u;
                if (step == 0) bits &= (stop & 31) == 31 ? 0xffffffffu : ((2u << (stop & 31)) - 1u);
                if (step == nw) bits &= (stop & 31) == 31 ? 0u : ~((2u << (stop & 31)) - 1u);
                while (bits) {
#ifdef __CUDA_ARCH__
                    const int bpos = 31 - __clz(bits);
#else
                    const int bpos = 31 - __builtin_clz(bits);
#endif
                    bits &= ~(1u << bpos);
                    const int sl = wi * 32 + bpos;
                    const int j = (stop - sl) & (B - 1);
                    if (j >= J) return;
                    const uint32_t c = hist[sl * kTileRows + r];
                    if (c) fn(j, c);
                }
            }
        };
        auto F = [&](int J) -> float {
            float s = 0.0f;
            for_nonzero(J, [&](int j, uint32_t c) { s = fmaf((float)c, T[J - j], s); });
            return s;
        };
        // smallest J in [1, B-1] with F(J) >= thr (F is nondecreasing in J)
        int lo = 1, hi = B - 1;
        while (lo < hi) {
            const int mid = (lo + hi) >> 1;
            if (F(mid) >= thr) hi = mid; else lo = mid + 1;
        }
        const int J = lo;
        // bisection on u in [0, 1): g(u) = sum_{j<J} c_j (J - j - u)^k, keep g(u_lo) >= thr
        float ulo = 0.0f, uhi = 1.0f;
        for (int it = 0; it < 6; ++it) {
            const float um = 0.5f * (ulo + uhi);
            float s = 0.0f;
            for_nonzero(J, [&](int j, uint32_t c) {
                const float x = (float)(J - j) - um;
#ifdef __CUDA_ARCH__
                if (x > 0.0f) s = fmaf((float)c, exp2f(sp.k * __log2f(x)), s);
#else
                if (x > 0.0f) s = fmaf((float)c, exp2f(sp.k * log2f(x)), s);
#endif
            });
            if (s >= thr) ulo = um; else uhi = um;
        }
        tau_h = ((float)(h.top - J) + ulo) * sp.w;
    }
    return tau_h - 4.0f * 1.1920929e-7f * fmaxf(1.0f, fabsf(tau_h));
}

// ---------------------------------------------------------------------------------------------
// Solver state and step
//
// Halley / Newton: open steps from the current tau, kept inside the bracket [lo, hi] (bisection
// otherwise); stop at |f| <= ftol, a step <= xtol max(1, |tau|), or the step cap.
// Secant (alpha > 2): bracketing (Illinois) secant. The first sweep evaluates f at both bracket
// ends; each step takes the secant through the current ends and the new point replaces the end of
// the same sign, halving the f value of an end kept twice in a row. Stop at |f| <= ftol, a bracket
// narrower than ~4 float32 ulps of tau, or the step cap.
// ---------------------------------------------------------------------------------------------
constexpr float kXtolBracket = 4.8e-7f;

struct RowSolve {
    float tau, lo, hi;
    float flo, fhi;  // secant: f at the bracket ends
    float tau2;      // secant: the second point evaluated in the first refinement sweep
    int side;        // secant: which end the last point replaced (+1 lo, -1 hi)
    int steps, fallbacks, max_steps;
    bool done;
    bool need_two;   // secant: the next sweep also evaluates f at tau2
};

// Initial bracket from the histogram bound (or the plain bracket), for a row with max z `m` and
// `n_i` allowed keys.
__device__ __forceinline__ void solve_init(RowSolve& s, float tau_h, float m, int n_i, const SolveParams& sp) {
    const float lo0 = m - 1.0f;
    const float hi0 = m - exp2f((1.0f - sp.alpha) * __log2f((float)n_i));
    float lo = lo0, hi = hi0;
    if (sp.init_mode == 0) {
        lo = fmaxf(tau_h, lo0);
        hi = fminf(tau_h + sp.w, hi0);
        if (lo > hi) { lo = lo0; hi = hi0; }
    }
    s.lo = lo;
    s.hi = hi;
    s.tau = lo;
    s.tau2 = hi;
    s.flo = 0.0f;
    s.fhi = 0.0f;
    s.side = 0;
    s.steps = 0;
    s.fallbacks = 0;
    s.max_steps = sp.init_mode == 0 ? 12 : 24;
    s.done = false;
    s.need_two = (sp.method == kSecant);
}

__device__ __forceinline__ void secant_next(RowSolve& s) {
    const float cand = s.hi - s.fhi * (s.hi - s.lo) / (s.fhi - s.flo);
    const bool ok = isfinite(cand) && cand > s.lo && cand < s.hi;
    s.tau = ok ? cand : 0.5f * (s.lo + s.hi);
    s.fallbacks += ok ? 0 : 1;
    s.steps += 1;
    if (s.hi - s.lo <= kXtolBracket * fmaxf(1.0f, fabsf(s.tau)) || s.steps >= s.max_steps) s.done = true;
}

// One solver update from the sums at the current tau (F0 = sum x^k, F1 = sum x^(k-1),
// F2 = sum x^(k-2)); F0b = sum (z - tau2)_+^k when the secant's second point was evaluated.
__device__ __forceinline__ void solve_step(RowSolve& s, float F0, float F1, float F2, float F0b,
                                           const SolveParams& sp) {
    if (s.done) return;
    if (sp.method == kSecant) {
        if (s.need_two) {
            s.need_two = false;
            const float fa = F0 - 1.0f, fb = F0b - 1.0f;
            // an end whose sign contradicts the bracket is off only by rounding: accept it
            if (fabsf(fa) <= kFtol || fa < 0.0f) { s.done = true; return; }
            if (fabsf(fb) <= kFtol || fb > 0.0f) { s.tau = s.tau2; s.done = true; return; }
            s.flo = fa;
            s.fhi = fb;
            secant_next(s);
            return;
        }
        const float fc = F0 - 1.0f;
        if (fabsf(fc) <= kFtol) { s.done = true; return; }
        if (fc > 0.0f) {
            s.lo = s.tau; s.flo = fc;
            if (s.side == 1) s.fhi *= 0.5f;
            s.side = 1;
        } else {
            s.hi = s.tau; s.fhi = fc;
            if (s.side == -1) s.flo *= 0.5f;
            s.side = -1;
        }
        secant_next(s);
        return;
    }
    const float f = F0 - 1.0f;
    if (fabsf(f) <= kFtol) { s.done = true; return; }
    if (f > 0.0f) s.lo = fmaxf(s.lo, s.tau); else s.hi = fminf(s.hi, s.tau);
    const float k = sp.k;
    const float fp = -k * F1;
    float cand;
    if (sp.method == kHalley) {
        const float fpp = k * (k - 1.0f) * F2;
        cand = s.tau - 2.0f * f * fp / (2.0f * fp * fp - f * fpp);
    } else {
        cand = s.tau - f / fp;
    }
    const bool ok = isfinite(cand) && cand > s.lo && cand < s.hi;
    const float nt = ok ? cand : 0.5f * (s.lo + s.hi);
    s.fallbacks += ok ? 0 : 1;
    s.steps += 1;
    const bool small = fabsf(nt - s.tau) <= kXtol * fmaxf(1.0f, fabsf(s.tau));
    s.tau = nt;
    if (small || s.steps >= s.max_steps) s.done = true;
}

}  // namespace eattn
