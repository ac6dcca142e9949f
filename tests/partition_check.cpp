// Host check of the stream-K partition the attention launcher uses (sk_partition): for many
// frame shapes and grid sizes, the CTA starts begin at 0, end at the frame's work, strictly
// increase (every CTA gets work), and no CTA's modelled cost exceeds the even share by more
// than one unit's start plus a step.  And of the key-order rotations (sk_rotations): each in
// [0, n_tiles); the CTA holding the larger part of a unit (of the first two CTAs on it) reads
// key tile tau mod n_tiles at its step tau throughout that part; each unit still visits every
// key tile once.  And the multiply-high division of tile indices (tile_div_magic): exact for
// every index below the tile count it is enabled for, off where it could fail.
// Built and run by tests/test_partition_host.py.
#include <cstdio>
#include <algorithm>
#include "../rope_paged_kv_02_b200/csrc/lbm_internal.h"

using namespace lbm;

static AttnParams p;  // large: static storage

int main() {
  long long checked = 0;
  for (int T : {7, 22, 128, 129, 256, 300, 774, 1005, 4102})
    for (int H : {1, 2, 8, 16, 40})
      for (int nt : {1, 2, 3, 7, 153, 1090})
        for (int want : {1, 2, 3, 16, 100, 148, 592, 1024}) {
          p.tokens = T;
          p.heads = H;
          p.n_tiles = nt;
          p.n_pairs = ((T + 127) / 128 + 1) / 2;
          p.work = (long long)p.n_pairs * H * nt;
          p.grid = (int)std::min<long long>(std::min<long long>(want, p.work), kMaxGrid);
          sk_partition(p);
          if (p.sk_start[0] != 0 || p.sk_start[p.grid] != p.work) {
            std::printf("FAIL ends T=%d H=%d nt=%d grid=%d\n", T, H, nt, p.grid);
            return 1;
          }
          const bool single_last = ((T + 127) / 128) % 2 == 1;
          long long total = 0, worst = 0;
          for (int c = 0; c < p.grid; ++c) {
            if (p.sk_start[c + 1] <= p.sk_start[c]) {
              std::printf("FAIL empty share T=%d H=%d nt=%d grid=%d c=%d\n", T, H, nt, p.grid, c);
              return 1;
            }
            long long cost = 0;
            for (int x = p.sk_start[c]; x < p.sk_start[c + 1]; ++x) {
              const int unit = x / nt;
              const bool single = single_last && unit % p.n_pairs == p.n_pairs - 1;
              if (x == p.sk_start[c] || x % nt == 0) cost += kCostSegment;
              cost += single ? kCostSingleStep : kCostPairStep;
            }
            total += cost;
            worst = std::max(worst, cost);
          }
          // the even share plus what one boundary can add: a segment start and a step, plus
          // the steps the non-empty rule may move onto a CTA when shares are tiny
          const long long even = (total + p.grid - 1) / p.grid;
          const long long slack = kCostSegment + 2 * kCostPairStep;
          if (p.work >= 4LL * p.grid && worst > even + slack) {
            std::printf("FAIL balance T=%d H=%d nt=%d grid=%d worst=%lld even=%lld\n", T, H, nt,
                        p.grid, worst, even);
            return 1;
          }
          sk_rotations(p);
          const long long units = (long long)p.n_pairs * H;
          if (units <= kMaxUnits) {
            for (int c = 0; c < p.grid; ++c) {
              for (long long x = p.sk_start[c]; x < p.sk_start[c + 1]; ++x) {
                const long long u = x / nt, i = x % nt;
                const int r = p.rot[u];
                if (r < 0 || r >= nt) {
                  std::printf("FAIL rot range u=%lld r=%d nt=%d\n", u, r, nt);
                  return 1;
                }
                const long long tile = (i + r) % nt, step = x - p.sk_start[c];
                // the CTA holding the larger part of the unit (of the first two) reads it in
                // phase with its own steps
                const long long first = u * nt, end = first + nt;
                int c0 = 0;
                while (c0 + 1 < p.grid && p.sk_start[c0 + 1] <= first) ++c0;
                const long long own = std::min<long long>(p.sk_start[c0 + 1], end) - first;
                const long long next =
                    c0 + 1 < p.grid ? std::min<long long>(p.sk_start[c0 + 2], end) -
                                          std::min<long long>(p.sk_start[c0 + 1], end)
                                    : 0;
                const int phased = next > own ? c0 + 1 : c0;
                if (c == phased && tile != step % nt) {
                  std::printf("FAIL phase T=%d H=%d nt=%d grid=%d c=%d u=%lld\n", T, H, nt,
                              p.grid, c, u);
                  return 1;
                }
              }
            }
            // a rotation is a bijection of the unit's tiles (every key tile read once)
            for (long long u = 0; u < units && nt <= 1090; ++u) {
              static bool seen[1090];
              std::fill(seen, seen + nt, false);
              for (int i = 0; i < nt; ++i) seen[(i + p.rot[u]) % nt] = true;
              if (!std::all_of(seen, seen + nt, [](bool b) { return b; })) {
                std::printf("FAIL cover u=%lld\n", u);
                return 1;
              }
            }
          }
          ++checked;
        }
  // the multiply-high division of tile indices by tiles per page (tile_div_magic)
  for (int d : {2, 3, 5, 6, 7, 8, 9, 17, 63, 64, 65, 127, 1000, 2047, 4095, 16384, 65535}) {
    for (long long n : {100LL, 70000LL, 1LL << 17, 1LL << 20, 1LL << 24}) {
      const uint32_t m = tile_div_magic(d, n);
      if ((unsigned long long)n * d > (1ull << 32)) {
        if (m != 0) {
          std::printf("FAIL magic should be off d=%d n=%lld\n", d, n);
          return 1;
        }
        continue;
      }
      const long long step = n > (1LL << 20) ? 7 : 1;
      for (long long t = 0; t < n; t += step) {
        const long long q = (long long)(((unsigned long long)t * m) >> 32);
        if (q != t / d) {
          std::printf("FAIL magic d=%d t=%lld\n", d, t);
          return 1;
        }
      }
      for (long long t = n - 1; t >= 0 && t > n - 4096; --t) {   // the largest indices
        if ((long long)(((unsigned long long)t * m) >> 32) != t / d) {
          std::printf("FAIL magic top d=%d t=%lld\n", d, t);
          return 1;
        }
      }
    }
  }
  std::printf("ok %lld\n", checked);
  return 0;
}
