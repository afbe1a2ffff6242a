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

constexpr int kMaxSteps = 8;
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
// Histogram ring (thread-owned row). hist: u32 [B slots][128 rows].
// ---------------------------------------------------------------------------------------------
struct HistRow {
    float m_raw;    // running max of the raw score
    float thr_raw;  // raw threshold for binning: z > m_run - 1
    int top;        // bin index of the running max
    bool any;       // any entry seen
};

__device__ __forceinline__ int bin_of(float a, float cbin) {
    float y = fminf(fmaxf(a * cbin, -1.0e9f), 1.0e9f);
    return __float2int_rd(y);
}

// Raise the running max to `a_max` (raw) and slide the window.
__device__ __forceinline__ void hist_raise(HistRow& h, float a_max, const SolveParams& sp, uint32_t* hist, int r) {
    if (!(a_max > h.m_raw)) return;
    const int nt = bin_of(a_max, sp.cbin);
    const int B = sp.bins;
    if (h.any && nt > h.top) {
        const int steps = min(nt - h.top, B);
        for (int t = 1; t <= steps; ++t) hist[((h.top + t) & (B - 1)) * kTileRows + r] = 0u;
    }
    h.top = h.any ? max(h.top, nt) : nt;
    h.any = true;
    h.m_raw = a_max;
    h.thr_raw = a_max - sp.inv_cz;
}

// Bin one raw score that passed a > thr_raw.
__device__ __forceinline__ void hist_add(const HistRow& h, float a, const SolveParams& sp, uint32_t* hist, int r) {
    const int b = bin_of(a, sp.cbin);
    const int j = h.top - b;
    if (j >= 0 && j < sp.bins) hist[(b & (sp.bins - 1)) * kTileRows + r] += 1u;
}

// Root tau_h of the left-edge binned function, in z units (a lower bound on tau*).
// For k = 1 and k = 2 the root is found in closed form on its segment; for other k by a search over
// the bin edges and then bisection inside the segment, keeping the end where f >= 0.
// T[i] = i^k for i = 0..B (generic k only).
template <int KIND>
__device__ float hist_tau(const HistRow& h, const SolveParams& sp, const uint32_t* hist, int r, const float* T) {
    const int B = sp.bins;
    const float Bm1 = (float)(B - 1);
    auto cnt = [&](int j) -> float { return (float)hist[((h.top - j) & (B - 1)) * kTileRows + r]; };
    if constexpr (KIND == kAlpha15 || KIND == kAlpha2) {
        // A0 = sum c_j, A1 = sum c_j (J - j), A2 = sum c_j (J - j)^2 over offsets j < J (exact integers)
        double A0 = 0.0, A1 = 0.0, A2 = 0.0;
        const double thr = (KIND == kAlpha15) ? (double)Bm1 * (double)Bm1 : (double)Bm1;
        int J = 1;
        for (; J < B; ++J) {
            if (J > 1) {
                A2 += 2.0 * A1 + A0;
                A1 += A0;
            }
            const double c = (double)cnt(J - 1);
            A0 += c;
            A1 += c;
            A2 += c;
            const double F = (KIND == kAlpha15) ? A2 : A1;
            if (F >= thr) break;
        }
        if (J >= B) J = B - 1;
        double u;  // tau_h = (top - J + u) w, u in [0, 1)
        if constexpr (KIND == kAlpha15) {
            const double disc = fmax(A1 * A1 - A0 * (A2 - thr), 0.0);
            u = (A1 - sqrt(disc)) / A0;
        } else {
            u = (A1 - thr) / A0;
        }
        u = fmin(fmax(u, 0.0), 1.0);
        return (float)(((double)(h.top - J) + u) * (double)sp.w);
    } else {
        const float thr = T[B - 1];
        auto F = [&](int J) -> float {
            float s = 0.0f;
            for (int j = 0; j < J; ++j) {
                const float c = cnt(j);
                if (c != 0.0f) s = fmaf(c, T[J - j], s);
            }
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
            for (int j = 0; j < J; ++j) {
                const float c = cnt(j);
                const float x = (float)(J - j) - um;
                if (c != 0.0f && x > 0.0f) s = fmaf(c, exp2f(sp.k * __log2f(x)), s);
            }
            if (s >= thr) ulo = um; else uhi = um;
        }
        return ((float)(h.top - J) + ulo) * sp.w;
    }
}

// ---------------------------------------------------------------------------------------------
// Solver state and step
// ---------------------------------------------------------------------------------------------
struct RowSolve {
    float tau, lo, hi;
    float prev_t, prev_f;  // secant: the other point
    float tau2;            // secant: second point evaluated in the first refinement sweep
    int steps, fallbacks;
    bool done;
    bool need_two;  // secant: the next sweep also evaluates f at tau2
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
    s.prev_t = hi;
    s.prev_f = 0.0f;
    s.tau2 = hi;
    s.steps = 0;
    s.fallbacks = 0;
    s.done = false;
    s.need_two = (sp.method == kSecant);
}

// One solver update from the sums at the current tau (F0 = sum x^k, F1 = sum x^(k-1),
// F2 = sum x^(k-2)); F0b = sum (z - tau2)_+^k when the secant's second point was evaluated.
__device__ __forceinline__ void solve_step(RowSolve& s, float F0, float F1, float F2, float F0b,
                                           const SolveParams& sp) {
    if (s.done) return;
    if (s.need_two) {
        // secant start: (tau2, f(tau2)) is the other point; it is a bracket end if its sign says so
        s.need_two = false;
        const float fb = F0b - 1.0f;
        s.prev_t = s.tau2;
        s.prev_f = fb;
        if (fb <= 0.0f) s.hi = fminf(s.hi, s.tau2);
        else s.lo = fmaxf(s.lo, s.tau2);
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
    } else if (sp.method == kNewton) {
        cand = s.tau - f / fp;
    } else {
        cand = s.tau - f * (s.tau - s.prev_t) / (f - s.prev_f);
        s.prev_t = s.tau;
        s.prev_f = f;
    }
    const bool ok = isfinite(cand) && cand > s.lo && cand < s.hi;
    const float nt = ok ? cand : 0.5f * (s.lo + s.hi);
    s.fallbacks += ok ? 0 : 1;
    s.steps += 1;
    const bool small = fabsf(nt - s.tau) <= kXtol * fmaxf(1.0f, fabsf(s.tau));
    s.tau = nt;
    if (small || s.steps >= kMaxSteps) s.done = true;
}

}  // namespace eattn
