// Host-side check of the stream-K partition arithmetic shared by the
// tensor-core GEMMs (gemm_tc.cuh, gemm_tokm.cuh) and the epilogue kernels
// that reduce their parts (epilogue.cuh).  Compiled with nvcc and run on the
// CPU: no device code is launched.
//
// For a launch of n_tiles output tiles of KBt k-units each, split over
// `grid` contiguous unit ranges [sk_start(i), sk_start(i + 1)):
//  - the ranges cover every unit once and none is empty (grid <= units);
//  - sk_owner(u) is the range that holds u;
//  - a tile's contributors are exactly sk_owner(first unit) ..
//    sk_owner(last unit), as the fix-up and the epilogue read them;
//  - per contributor, only its first and its last part can be cut; the
//    fix-up slot rule (slot 0 iff the range starts inside the tile) agrees
//    with the producer's (slot 0 for its first part, 1 for any later one);
//  - the DUMP-mode part slots (tile + contributor) are distinct and below
//    n_tiles + grid, the count the host allocates;
//  - with m-tile groups, the CTA indices (which pick the fix-up slots) are
//    distinct, below the grid and the SM count, and each CTA's units map to
//    tiles of its own m-tile;
//  - the epilogue's row groups (epi_groups_per_tile) cover every row of an
//    m-tile once and never straddle two.
// Prints "ok" and exits 0, or prints the first failures and exits 1.

#include <cstdio>
#include <cstdlib>
#include <set>
#include <vector>

#include "../lossless_diffusion_draft_b200/csrc/epilogue.cuh"
#include "../lossless_diffusion_draft_b200/csrc/gemm_tc.cuh"

using namespace uno;

static long long g_fail = 0, g_cases = 0;

#define CHECK(cond, ...)                                          \
  do {                                                            \
    if (!(cond)) {                                                \
      if (g_fail < 20) {                                          \
        std::printf("FAIL %s: ", #cond);                          \
        std::printf(__VA_ARGS__);                                 \
        std::printf("\n");                                        \
      }                                                           \
      ++g_fail;                                                   \
    }                                                             \
  } while (0)

static void check_partition(int n_tiles, int KBt, int grid) {
  ++g_cases;
  const int units = n_tiles * KBt;
  CHECK(sk_start(0, units, grid) == 0, "units %d grid %d", units, grid);
  CHECK(sk_start(grid, units, grid) == units, "units %d grid %d", units, grid);
  for (int i = 0; i < grid; ++i)
    CHECK(sk_start(i + 1, units, grid) > sk_start(i, units, grid), "empty range %d of %d (units %d)", i,
          grid, units);
  for (int u = 0; u < units; ++u) {
    const int o = sk_owner(u, units, grid);
    CHECK(o >= 0 && o < grid && sk_start(o, units, grid) <= u && u < sk_start(o + 1, units, grid),
          "owner of unit %d (units %d grid %d) is %d", u, units, grid, o);
  }
  // contributors of each tile, from the ranges themselves
  std::vector<int> lo(n_tiles, grid), hi(n_tiles, -1);
  std::set<long long> dump_slots;
  for (int i = 0; i < grid; ++i) {
    const int u0 = sk_start(i, units, grid), u1 = sk_start(i + 1, units, grid);
    int part = 0;
    for (int u = u0; u < u1; ++part) {
      // the producer's walk over its range (gemm_tc.cuh, epilogue warps)
      const int t = u / KBt, kb0 = u % KBt;
      const int kb1 = kb0 + (u1 - u) < KBt ? kb0 + (u1 - u) : KBt;
      u += kb1 - kb0;
      const bool whole = kb0 == 0 && kb1 == KBt;
      const bool last_part = u >= u1;
      lo[t] = lo[t] < i ? lo[t] : i;
      hi[t] = hi[t] > i ? hi[t] : i;
      CHECK(whole || part == 0 || last_part, "cut middle part: range %d tile %d", i, t);
      if (!whole) {
        const int producer_slot = part == 0 ? 0 : 1;
        const int reducer_slot = sk_start(i, units, grid) >= t * KBt ? 0 : 1;
        CHECK(producer_slot == reducer_slot, "slot of range %d in tile %d: %d vs %d", i, t, producer_slot,
              reducer_slot);
      }
      const long long slot = (long long)t + i;
      CHECK(dump_slots.insert(slot).second, "DUMP slot %lld used twice", slot);
      CHECK(slot < (long long)n_tiles + grid, "DUMP slot %lld past %d", slot, n_tiles + grid);
    }
  }
  for (int t = 0; t < n_tiles; ++t) {
    const int first = sk_owner(t * KBt, units, grid);
    const int last = sk_owner(t * KBt + KBt - 1, units, grid);
    CHECK(first == lo[t] && last == hi[t], "tile %d contributors %d..%d, ranges say %d..%d", t, first,
          last, lo[t], hi[t]);
  }
}

// m-tile groups (several token m-tiles, not DUMP): g = min(SMs / m_tiles,
// units / 8) splits of the n-tiles' units, repeated for every m-tile; CTA
// i * m_tiles + mt works on m-tile mt.  The CTA indices, which select the
// fix-up slots of the workspace (two per SM), stay below the grid and the SM
// count, and every (n-tile, m-tile) tile is reduced from its own m-tile's
// CTAs only.
static void check_grouped(int n_tiles, int m_tiles, int KBt, int sm) {
  ++g_cases;
  const int vunits = n_tiles * KBt;
  int g = sm / m_tiles < vunits / 8 ? sm / m_tiles : vunits / 8;
  if (g < 1) return;   // the host then takes the ungrouped form
  const int grid = g * m_tiles;
  CHECK(grid <= sm, "grid %d over %d SMs", grid, sm);
  std::set<int> ctas;
  for (int mt = 0; mt < m_tiles; ++mt)
    for (int i = 0; i < g; ++i) {
      const int cta = i * m_tiles + mt;
      CHECK(cta >= 0 && cta < grid && ctas.insert(cta).second, "CTA %d (split %d, m-tile %d)", cta, i, mt);
      const int u0 = sk_start(i, vunits, g), u1 = sk_start(i + 1, vunits, g);
      for (int u = u0; u < u1; ++u) {
        const int t = (u / KBt) * m_tiles + mt;   // the kernel's tile_of
        CHECK(t % m_tiles == mt && t / m_tiles < n_tiles, "unit %d of CTA %d maps to tile %d", u, cta, t);
      }
    }
  CHECK((int)ctas.size() == grid, "%d CTAs for a grid of %d", (int)ctas.size(), grid);
}

static void check_row_groups(int M, int NT, int RG) {
  ++g_cases;
  const int m_tiles = (M + NT - 1) / NT;
  const int gpt = epi_groups_per_tile(NT, M, RG);
  std::vector<int> seen(M, 0);
  for (int y = 0; y < m_tiles * gpt; ++y) {
    // row_group(): blockIdx.y = m-tile * groups_per_tile + group
    const int mt = y / gpt, g = y % gpt;
    const int m0 = mt * NT + g * RG;
    const int end = M < (mt + 1) * NT ? M : (mt + 1) * NT;
    const int nrows = RG < end - m0 ? RG : end - m0;
    for (int j = 0; j < nrows; ++j) {
      CHECK(m0 + j < M && (m0 + j) / NT == mt, "row %d of group %d outside its m-tile", m0 + j, y);
      if (m0 + j < M) ++seen[m0 + j];
    }
  }
  for (int m = 0; m < M; ++m) CHECK(seen[m] == 1, "row %d covered %d times (M %d NT %d RG %d)", m, seen[m], M, NT, RG);
}

int main() {
  // the host's launch shapes: grid = min(SMs, units / 8) (gemm_tc) or the
  // m-tile groups' split count, over the projections of the three model
  // shapes (k-units of 2 k-blocks of 64: K / 128) and odd sizes
  const int sms[] = {148, 132, 100, 17};
  const int kbts[] = {1, 2, 8, 16, 32, 96};
  for (int sm : sms)
    for (int KBt : kbts)
      for (int n_tiles = 1; n_tiles <= 1200; n_tiles += (n_tiles < 64 ? 1 : 37)) {
        const int units = n_tiles * KBt;
        int grid = units / 8 < sm ? units / 8 : sm;
        if (grid < 1) grid = 1;
        check_partition(n_tiles, KBt, grid);
      }
  // every split count up to the units, for small launches
  for (int KBt : {1, 3, 32})
    for (int n_tiles = 1; n_tiles <= 12; ++n_tiles)
      for (int grid = 1; grid <= n_tiles * KBt && grid <= 300; ++grid) check_partition(n_tiles, KBt, grid);
  // the LM head of the Qwen3-8B shape (151936 / 128 tiles, K 4096 / 128)
  check_partition(1187, 32, 148);
  // m-tile groups: max batch (1360 / 1280 rows in 128-row token tiles),
  // prefill chunks, the tokens-in-M form's 256-wide weight tiles
  for (int sm : {148, 132})
    for (int m_tiles : {2, 3, 8, 11, 16, 64})
      for (int KBt : {32, 96})
        for (int n_tiles : {2, 16, 17, 33, 48, 96, 194, 594, 1187}) {
          check_grouped(n_tiles, m_tiles, KBt, sm);
          const int g = sm / m_tiles < n_tiles * KBt / 8 ? sm / m_tiles : n_tiles * KBt / 8;
          if (g >= 1) check_partition(n_tiles, KBt, g);
        }
  // row groups: the draft and verify passes, max batch, prefill chunks
  for (int M : {1, 9, 16, 17, 18, 33, 100, 128, 129, 136, 1280, 1360, 1361})
    for (int NT : {16, 32, 64, 128})
      for (int RG : {1, 8, 9, 16}) check_row_groups(M, NT, RG);
  if (g_fail) {
    std::printf("%lld failures in %lld cases\n", g_fail, g_cases);
    return 1;
  }
  std::printf("ok (%lld cases)\n", g_cases);
  return 0;
}
