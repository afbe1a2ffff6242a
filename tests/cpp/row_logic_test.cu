// Host-side check of the per-row histogram logic of the kernels (entmax_row.cuh) against brute force:
// the window ring masks and the root tau_h of the binned function (a lower bound, exact for k = 1, 2).
#include <cstdio>
#include <cmath>
#include <cstdlib>
#include <vector>
#include "entmax_row.cuh"
using namespace eattn;
// brute force: root of f_h(tau) = sum_j c_j ((top - j) w - tau)_+^k - 1 by bisection in double
double brute(const std::vector<int>& c, int top, int B, double k) {
  double w = 1.0 / (B - 1), lo = top * w - 1.0, hi = top * w;
  for (int it = 0; it < 200; ++it) {
    double mid = 0.5 * (lo + hi), f = -1.0;
    for (int j = 0; j < B; ++j) if (c[j]) { double x = (top - j) * w - mid; if (x > 0) f += c[j] * pow(x, k); }
    if (f >= 0) lo = mid; else hi = mid;
  }
  return lo;
}
template <int KIND> int run(double k, float alpha) {
  int bad = 0;
  srand(3);
  for (int trial = 0; trial < 3000; ++trial) {
    const int B = (trial % 4 == 0) ? 64 : (trial % 4 == 1) ? 512 : (trial % 4 == 2) ? 128 : 256;
    std::vector<uint16_t> hist(512 * 128, 0);
    uint32_t live_all[6 * 17] = {0};
    HistRow h;
    hist_init(h, live_all, 5, B > 256 ? kLiveStride512 : kLiveStride);
    uint32_t* live = h.live;
    h.top = 1000 + rand() % 500; h.any = true;
    std::vector<int> c(B, 0);
    c[0] = 1 + rand() % 3;
    const int nb = rand() % 40;
    for (int i = 0; i < nb; ++i) { int j = (trial % 5 == 0) ? rand() % 6 : rand() % B; c[j] += 1 + rand() % (trial % 7 == 0 ? 5000 : 4); }
    const int r = 5;
    for (int j = 0; j < B; ++j) if (c[j]) { int sl = (h.top - j) & (B - 1); hist[sl * 128 + r] = c[j]; live[sl >> 5] |= 1u << (sl & 31); }
    // some dead slots with garbage counts
    for (int i = 0; i < 5; ++i) { int j = rand() % B; if (!c[j]) { int sl = (h.top - j) & (B - 1); hist[sl * 128 + r] = 77; } }
    SolveParams sp = make_solve_params(alpha, 0.125f, B, 0);
    float T[516]; for (int i = 0; i <= B; ++i) T[i] = powf((float)i, sp.k);
    const float got = hist_tau<KIND>(h, sp, hist.data(), r, T);
    // 32-bit moments (the forward's stash rows): the same result wherever the row holds few entries
    int total = 0;
    for (int j = 0; j < B; ++j) total += c[j];
    if (total <= 512 && hist_tau<KIND, int>(h, sp, hist.data(), r, T) != got) {
      if (bad < 5) printf("KIND %d trial %d: 32-bit moments differ\n", KIND, trial);
      ++bad;
    }
    const double ref = brute(c, h.top, B, k);
    const double tol = 1e-5 * fmax(1.0, fabs(ref)) + (KIND == kGeneric ? sp.w / 64 + 1e-5 : 0);
    if (!(got <= ref + 1e-6 * fmax(1.0, fabs(ref))) || ref - got > tol) {
      if (bad < 5) printf("KIND %d trial %d B=%d got %.9f ref %.9f diff %.3e\n", KIND, trial, B, got, ref, got - ref);
      ++bad;
    }
  }
  return bad;
}
int ring_masks() {
  int bad = 0;
  for (int B : {64, 128, 256, 512})
    for (int s0 = 0; s0 < B; ++s0)
      for (int len = 0; len < B; ++len) {
        uint32_t live[16];
        for (int i = 0; i < 16; ++i) live[i] = 0xffffffffu & ~ring_word_mask(i, s0, len, B);
        for (int p = 0; p < 512; ++p) {
          const bool cleared = p < B && ((p - s0) % B + B) % B < len;
          const bool bit = (live[p >> 5] >> (p & 31)) & 1u;
          if (bit == cleared) ++bad;
        }
      }
  printf("ring mask mismatches %d\n", bad);
  return bad;
}
int main() {
  int bad = ring_masks();
  bad += run<kAlpha15>(2.0, 1.5) + run<kAlpha2>(1.0, 2.0) + run<kGeneric>(4.0, 1.25) + run<kGeneric>(0.5, 3.0);
  printf("hist_tau mismatches %d\n", bad);
  return bad != 0;
}
