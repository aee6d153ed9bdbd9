// Host-only check of the split-K W4A16 work partition (w4_unit0 / w4_cta_of in
// w4a16_kernel.cuh, the same inline functions the kernel runs). For each
// (tiles, slices per tile, CTAs): the runs [w4_unit0(c), w4_unit0(c + 1)) cover
// every unit once, in order, none empty; w4_cta_of inverts them; a tile shared
// by several runs gets one partial slot per run (2c for a run's first tile,
// 2c + 1 for its last), no slot serves two tiles, and every tile strictly inside
// a run is whole. Prints "ok" and exits 0, else prints the first failure.
#include <cstdio>
#include <set>
#include <vector>

#include "w4a16_kernel.cuh"

static int fail(const char* what, long long T, long long G, int C, long long x) {
  std::printf("FAIL %s: T=%lld G=%lld C=%d at %lld\n", what, T, G, C, x);
  return 1;
}

static int check(long long T, long long G, int C) {
  const long long U = T * G;
  if (C < 1 || C > U) return fail("C out of range", T, G, C, C);
  if (attn::w4_unit0(0, U, C) != 0 || attn::w4_unit0(C, U, C) != U) return fail("ends", T, G, C, 0);
  for (int c = 0; c < C; ++c) {
    const long long a = attn::w4_unit0(c, U, C), b = attn::w4_unit0(c + 1, U, C);
    if (b <= a) return fail("empty run", T, G, C, c);
    if (attn::w4_cta_of(a, U, C) != c || attn::w4_cta_of(b - 1, U, C) != c) return fail("cta_of", T, G, C, c);
    // tiles strictly inside the run are whole
    const long long t0 = a / G, t1 = (b - 1) / G;
    for (long long t = t0 + 1; t < t1; ++t) {
      if (attn::w4_cta_of(t * G, U, C) != c || attn::w4_cta_of(t * G + G - 1, U, C) != c)
        return fail("middle tile not whole", T, G, C, t);
    }
  }
  std::set<long long> slots;
  for (long long t = 0; t < T; ++t) {
    const int lo = attn::w4_cta_of(t * G, U, C), hi = attn::w4_cta_of(t * G + G - 1, U, C);
    if (lo > hi) return fail("segment order", T, G, C, t);
    if (lo == hi) continue;                    // whole: written straight to Y
    for (int c = lo; c <= hi; ++c) {
      const long long tile0 = attn::w4_unit0(c, U, C) / G;
      const long long slot = 2ll * c + (tile0 == t ? 0 : 1);
      if (slot >= 2ll * C) return fail("slot range", T, G, C, slot);
      if (!slots.insert(slot).second) return fail("slot reused", T, G, C, slot);
      // a run's last-tile slot is only used when that tile is not also its first
      if (tile0 != t && (attn::w4_unit0(c + 1, U, C) - 1) / G != t) return fail("tail slot", T, G, C, c);
    }
  }
  return 0;
}

int main() {
  int bad = 0, cases = 0;
  const long long tiles[] = {1, 2, 3, 7, 8, 9, 24, 36, 112, 148, 224, 296, 300, 448, 897};
  const long long gs[] = {1, 2, 3, 10, 17, 32, 64, 65, 128};
  for (long long T : tiles)
    for (long long G : gs) {
      const long long U = T * G;
      // the CTA counts the library launches: one per tile, and split-K with a
      // 148-SM device (min(296, 2 * 148, max(1, U / 8))), plus every C up to 40
      std::vector<int> cs = {static_cast<int>(T)};
      long long k = U / 8;
      k = k < 1 ? 1 : (k > 296 ? 296 : k);
      cs.push_back(static_cast<int>(k));
      for (int c = 1; c <= 40 && c <= U; ++c) cs.push_back(c);
      for (int C : cs) {
        ++cases;
        if (check(T, G, C)) bad = 1;
      }
    }
  if (!bad) std::printf("ok %d cases\n", cases);
  return bad;
}
