// Host-side check of the row-range schedule in sa_internal.h (the code the
// kernels run), on random ragged batches: the ranges are ordered and start
// at a user's first row or a whole number of tiles into the user; every row
// of every user is covered by exactly one segment; cta_of_row names the CTA
// that covered each row; users inside one CTA range go straight to the
// outputs; split users use distinct partial slots below 2G; the finalize
// pass (one unit per user, from the user's offsets and one range search)
// reduces every split user exactly once, over exactly the slots that the
// partial pass wrote for it, in ascending CTA order.  The 32-way search
// the kernels use (warp_range_begin) is replayed here step by step and must
// agree with the serial search.
#include <cstdio>
#include <cstdlib>
#include <map>
#include <random>
#include <set>
#include <vector>

#include "sa_internal.h"

using namespace sa;

static int fail(const char* what, long long a, long long b) {
  std::printf("FAIL %s (%lld, %lld)\n", what, a, b);
  return 1;
}

// Host replay of warp_range_begin (sa_ptx.cuh): 32 lanes test evenly
// spaced users, the highest lane whose user's start cost is <= tau narrows
// the range, until one user is left.
static int64_t warp_search_replay(const int64_t* off, int64_t B, int64_t N, int64_t c, int64_t G,
                                  int64_t* user) {
  if (c <= 0 || B <= 0 || c >= G) {
    *user = (c <= 0 || B <= 0) ? 0 : B;
    return c <= 0 ? 0 : N;
  }
  const int64_t tau = range_target(B, N, c, G);
  int64_t lo = 0, hi = B - 1;
  while (lo < hi) {
    const int64_t step = (hi - lo + 32) / 32;
    int last = -1;
    for (int lane = 0; lane < 32; ++lane) {
      const int64_t b = lo + lane * step;
      if (b <= hi && cost_before_user(off, b) <= tau) last = lane;
    }
    const int64_t nlo = lo + (last < 0 ? 0 : last) * step;
    hi = (nlo + step - 1) < hi ? (nlo + step - 1) : hi;
    lo = nlo;
  }
  *user = lo;
  return range_row(off, lo, N, tau);
}

static int check(const std::vector<int64_t>& off, int64_t sms) {
  const int64_t B = static_cast<int64_t>(off.size()) - 1, N = off.back();
  const int64_t T = tiles_of(N);
  int64_t G = T < sms ? T : sms;
  if (G < 1) G = 1;
  std::vector<int> covered(N, 0);
  std::vector<int64_t> owner(N, -1);
  std::map<int64_t, std::set<int64_t>> written;  // user -> slots
  std::map<int64_t, int64_t> slot_owner;          // slot -> user
  std::vector<int> direct(B, 0);
  for (int64_t c = 0; c < G; ++c) {
    int64_t bu, bw, bu1;
    const int64_t R0 = range_begin(off.data(), B, N, c, G, &bu);
    const int64_t R1 = range_begin(off.data(), B, N, c + 1, G, &bu1);
    if (warp_search_replay(off.data(), B, N, c, G, &bw) != R0 || bw != bu)
      return fail("warp search != serial search", c, R0);
    if (R0 > R1) return fail("ranges out of order", c, R0);
    if (R0 < R1 && B > 0) {
      const int64_t u = user_at_or_before(off.data(), B, R0);
      if (off[u] < R0 && (R0 - off[u]) % kTileRows) return fail("range not tile-aligned in its user", c, R0);
      if (off[bu] > R0) return fail("walker start after R0", c, bu);
    }
    const int64_t b0 = (B > 0 && R0 < R1) ? bu : B;
    SegmentWalker w{off.data(), B, R0, R1, b0};
    int64_t u, s, e, lo, hi;
    while (w.next(u, s, e, lo, hi)) {
      if (s < R0 || e > R1 || s < lo || e > hi) return fail("segment bounds", s, e);
      for (int64_t r = s; r < e; ++r) {
        covered[r]++;
        owner[r] = c;
      }
      const int64_t slot = segment_slot(c, lo, hi, R0, R1);
      if (slot < 0) {
        direct[u]++;
        continue;
      }
      if (slot >= 2 * G) return fail("slot range", slot, 2 * G);
      if (slot_owner.count(slot)) return fail("slot reused", slot, u);
      slot_owner[slot] = u;
      written[u].insert(slot);
    }
  }
  for (int64_t r = 0; r < N; ++r)
    if (covered[r] != 1) return fail("row coverage", r, covered[r]);
  // cta_of_row against the owner of every row (a sample of rows for big N)
  const int64_t stride = N > 200000 ? 97 : 1;
  for (int64_t r = 0, u = 0; r < N; r += stride) {
    while (off[u + 1] <= r) ++u;
    if (cta_of_row(off.data(), u, B, N, G, r) != owner[r]) return fail("cta_of_row", r, owner[r]);
  }
  // finalize ownership, same arithmetic as finalize_kernel: per user, the
  // CTAs holding its first and last rows; split if they differ; the first
  // CTA's slot by whether that CTA's range starts at the user's first row
  // (in closed form after a non-empty user, else found with the warp search
  // the kernel uses), then 2c for later CTAs.
  std::map<int64_t, std::vector<int64_t>> reduced;
  for (int64_t b = 0; b < B; ++b) {
    const int64_t lo = off[b], hi = off[b + 1];
    if (lo >= hi) continue;
    const int64_t c_lo = cta_of_row(off.data(), b, B, N, G, lo);
    const int64_t c_hi = cta_of_row(off.data(), b, B, N, G, hi - 1 < N - 1 ? hi - 1 : N - 1);
    if (c_hi <= c_lo) continue;
    bool first;
    const int64_t prev = b > 0 ? off[b - 1] : -1;
    if (prev < lo) {  // closed form, as in finalize_kernel
      const int64_t tau = c_lo > 0 ? range_target(B, N, c_lo, G) : 0;
      const int64_t cb = lo + kUserStartCost * b;
      first = c_lo > 0 ? (tau >= cb && tau < cb + kUserStartCost + kTileRows) : lo == 0;
      // and it agrees with the range start the partial pass uses
      int64_t ub0;
      if (first != (lo <= range_begin(off.data(), B, N, c_lo, G, &ub0)))
        return fail("closed-form first slot", b, c_lo);
    } else {
      int64_t ub;
      first = lo <= warp_search_replay(off.data(), B, N, c_lo, G, &ub);
    }
    std::vector<int64_t> slots{2 * c_lo + (first ? 0 : 1)};
    for (int64_t cc = c_lo + 1; cc <= c_hi; ++cc) slots.push_back(2 * cc);
    reduced[b] = slots;
  }
  for (int64_t b = 0; b < B; ++b) {
    const bool split = written.count(b) > 0;
    const bool empty = off[b] == off[b + 1];
    if (empty && (split || direct[b])) return fail("empty user written", b, 0);
    if (!empty && split == (direct[b] == 1)) return fail("user both/neither direct+split", b, direct[b]);
    if (direct[b] > 1) return fail("direct twice", b, direct[b]);
    if (split) {
      if (!reduced.count(b)) return fail("split user never reduced", b, 0);
      std::set<int64_t> want(reduced[b].begin(), reduced[b].end());
      if (want != written[b]) return fail("reduced slots != written slots", b, (long long)want.size());
      for (size_t i = 1; i < reduced[b].size(); ++i)
        if (reduced[b][i] <= reduced[b][i - 1]) return fail("slot order", b, i);
    } else if (reduced.count(b)) {
      return fail("unsplit user reduced", b, 0);
    }
  }
  return 0;
}

int main() {
  std::mt19937_64 rng(12345);
  long long cases = 0;
  // Range counts: tiny grids, one per SM (148), and the cluster passes' counts on a
  // B200 (74 pairs, 45 clusters of 3, 33 of 4, 15 of 8).
  const int64_t sms_list[] = {1, 2, 3, 7, 15, 33, 45, 74, 148};
  const int n_sms = static_cast<int>(sizeof(sms_list) / sizeof(sms_list[0]));
  for (int iter = 0; iter < 4500; ++iter) {
    const int64_t sms = sms_list[iter % n_sms];
    const int B = 1 + static_cast<int>(rng() % 40);
    std::vector<int64_t> off{0};
    const int mode = iter % 4;
    for (int b = 0; b < B; ++b) {
      int64_t n;
      switch (mode) {
        case 0: n = rng() % 300; break;                          // small, many empties possible
        case 1: n = (rng() % 4 == 0) ? 0 : 1 + rng() % 5000; break;
        case 2: n = 127 + rng() % 3; break;                      // around one tile
        default: n = 1 + rng() % 40000; break;
      }
      off.push_back(off.back() + n);
    }
    if (check(off, sms)) {
      std::printf("case iter=%d B=%d N=%lld sms=%lld\n", iter, B, (long long)off.back(), (long long)sms);
      return 1;
    }
    ++cases;
  }
  // large batches: several rounds of the 32-way search
  for (int iter = 0; iter < 40; ++iter) {
    const int B = 1000 + static_cast<int>(rng() % 40000);
    std::vector<int64_t> off{0};
    for (int b = 0; b < B; ++b) off.push_back(off.back() + ((rng() % 3 == 0) ? 0 : 1 + rng() % 900));
    if (check(off, iter % 2 ? 148 : 15)) {
      std::printf("case large iter=%d B=%d\n", iter, B);
      return 1;
    }
    ++cases;
  }
  // the benchmark shapes
  std::vector<int64_t> u16{0};
  for (int b = 0; b < 16; ++b) u16.push_back(u16.back() + 100000);
  if (check(u16, 148) || check(u16, 15)) return 1;  // one CTA per SM; clusters of 8
  std::vector<int64_t> zero{0, 0, 0};
  if (check(zero, 148)) return 1;
  std::printf("OK %lld cases\n", cases + 2);
  return 0;
}
