// Host-side check of the GEMM work schedule (zi_gemm.cuh): the tile walk, the split
// of a ragged last wave along K, and the partial-slot and counter indices, run with
// the same functions the kernels call (tile_origin, WorkWalker are host-callable),
// for the single-CTA (128 x 256 tiles, 148 units) and CTA-pair (256 x 256 tiles,
// 74 units) kernels over a grid of shapes.  Built and run by tests/test_gemm_schedule.py;
// prints one line per failure and "schedule ok <cases>" on success.
#include <cstdio>
#include <vector>

#include "zi_gemm.cuh"

using namespace zi;

static int failures = 0;
#define CHECK(cond, ...)                       \
  do {                                         \
    if (!(cond)) {                             \
      if (failures < 20) {                     \
        std::printf("FAIL %s: ", #cond);       \
        std::printf(__VA_ARGS__);              \
        std::printf("\n");                     \
      }                                        \
      ++failures;                              \
    }                                          \
  } while (0)

static void check_case(bool pair, int M, int N, int K, int bk, bool split) {
  const int BM = pair ? 256 : 128, BN = 256, G = pair ? 74 : 148;
  const int num_m = (M + BM - 1) / BM, num_n = N / BN, tiles = num_m * num_n, kb = K / bk;
  int group, group_n;
  choose_raster(num_m, num_n, double(BM) * K * 2, double(BN) * K * 2, group, group_n);
  const TailSched s = make_tail_sched(tiles, G, kb, split, num_n, group, group_n);
  const int units = sched_units(s, tiles);
  CHECK(group >= 1, "M=%d N=%d K=%d group %d", M, N, K, group);
  // the walk visits every (m, n) tile once
  std::vector<int> seen(size_t(tiles), 0);
  for (int t = 0; t < tiles; ++t) {
    int m0, n0;
    if (pair)
      tile_origin<256, 256>(s, num_m, t, m0, n0);
    else
      tile_origin<128, 256>(s, num_m, t, m0, n0);
    const bool ok = m0 % BM == 0 && n0 % BN == 0 && m0 >= 0 && m0 < num_m * BM && n0 >= 0 && n0 < N;
    CHECK(ok, "pair=%d M=%d N=%d tile %d -> (%d, %d)", pair, M, N, t, m0, n0);
    if (ok) ++seen[size_t(m0 / BM) * num_n + n0 / BN];
  }
  for (int i = 0; i < tiles; ++i) CHECK(seen[size_t(i)] == 1, "pair=%d M=%d N=%d tile (%d) seen %d", pair, M, N, i, seen[size_t(i)]);
  // every k-block of every tile is computed once; split pieces are well formed
  std::vector<int> kcover(size_t(tiles) * kb, 0);
  std::vector<int> pieces(size_t(tiles), 0);
  CHECK(units >= 1 && units <= G, "pair=%d M=%d N=%d K=%d units %d", pair, M, N, K, units);
  for (int u = 0; u < units; ++u) {
    WorkWalker w(s, u);
    WorkItem wi;
    int n_items = 0;
    while (w.next(wi)) {
      ++n_items;
      CHECK(wi.tile >= 0 && wi.tile < tiles, "tile %d of %d", wi.tile, tiles);
      if (wi.tile < 0 || wi.tile >= tiles) break;
      CHECK(wi.kb0 >= 0 && wi.kb0 < wi.kb1 && wi.kb1 <= kb, "k range [%d, %d) of %d", wi.kb0, wi.kb1, kb);
      for (int k = wi.kb0; k < wi.kb1 && k < kb; ++k) ++kcover[size_t(wi.tile) * kb + k];
      if (wi.piece >= 0) {
        CHECK(wi.tile >= s.dp_tiles, "piece of a whole tile %d (dp %d)", wi.tile, s.dp_tiles);
        CHECK(wi.kb1 - wi.kb0 >= kMinSplitKb, "piece of %d k-blocks", wi.kb1 - wi.kb0);
        CHECK(wi.piece < s.tail_s, "piece %d of %d", wi.piece, s.tail_s);
        ++pieces[size_t(wi.tile)];
        // partial slots: one per CTA (a pair's two CTAs use 2u and 2u + 1); counters per tile and rank
        const int slot_max = pair ? 2 * u + 1 : u;
        CHECK(slot_max < kSplitSlots, "slot %d", slot_max);
        const int cnt_max = pair ? 2 * (wi.tile - s.dp_tiles) + 1 : wi.tile - s.dp_tiles;
        CHECK(cnt_max < kSplitSlots, "counter %d", cnt_max);
        // the finisher reads piece j's partial at slot (u - piece + j) (pairs: per rank)
        CHECK(u - wi.piece >= 0 && u - wi.piece + s.tail_s - 1 < units, "piece slots of unit %d", u);
      } else {
        CHECK(wi.kb0 == 0 && wi.kb1 == kb, "whole tile with k range [%d, %d)", wi.kb0, wi.kb1);
      }
      if (n_items > tiles + 4) break;
    }
  }
  for (int t = 0; t < tiles; ++t)
    for (int k = 0; k < kb; ++k)
      CHECK(kcover[size_t(t) * kb + k] == 1, "pair=%d M=%d N=%d K=%d split=%d tile %d k-block %d covered %d times", pair,
            M, N, K, split, t, k, kcover[size_t(t) * kb + k]);
  for (int t = s.dp_tiles; t < tiles; ++t)
    if (s.tail_s > 1) CHECK(pieces[size_t(t)] == s.tail_s, "tile %d has %d of %d pieces", t, pieces[size_t(t)], s.tail_s);
}

int main() {
  int cases = 0;
  const int Ms[] = {1, 32, 96, 128, 200, 256, 288, 456, 512, 1152, 4096, 4128, 4224, 16896, 33792};
  const int NKs[][2] = {{256, 64}, {256, 3840}, {11520, 3840}, {3840, 3840}, {20480, 3840}, {3840, 10240}, {64 * 4, 640}};
  for (int pair = 0; pair < 2; ++pair)
    for (int split = 0; split < 2; ++split)
      for (int M : Ms)
        for (const auto& nk : NKs)
          for (int bk : {64, 128}) {
            if (nk[1] % bk) continue;
            check_case(pair != 0, M, nk[0], nk[1], bk, split != 0);
            ++cases;
          }
  if (failures) {
    std::printf("schedule FAILED %d checks\n", failures);
    return 1;
  }
  std::printf("schedule ok %d\n", cases);
  return 0;
}
