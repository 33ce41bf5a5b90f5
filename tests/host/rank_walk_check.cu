// Host check of the grouped rank-r kernel's schedule (rank_gemm.cuh): for
// problem lists of the shapes the library launches (the LLaMA-7B and -65B
// backward groups at 8192 tokens, single linears, ragged and tiny shapes),
// the planner's splits and the launch order are laid out as the launcher lays
// them out, and the kernel's own unit decoding (rank_unit) and boustrophedon
// walk (rank_unit_at) are replayed for every CTA of the grid.  Checked: every
// unit is visited by exactly one CTA; every (problem, row tile, n-tile) is
// covered by its splits exactly once, in contiguous non-empty k-block ranges
// that end at the reduction's end; and each CTA's units keep the order of the
// list.  Prints "<n> problem lists, 0 wrong" on success.
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <vector>

#include "rank_gemm.cuh"

using namespace qlora;

static int wrong = 0;
#define CHECK(c, ...)                       \
  do {                                      \
    if (!(c)) {                             \
      if (wrong < 20) std::printf(__VA_ARGS__); \
      ++wrong;                              \
    }                                       \
  } while (0)

struct P {
  int64_t rows, kext;
  int n_tiles;
};

static void check(const std::vector<P> &ps, int sms) {
  const int n = (int)ps.size();
  RankShape sh[kRankMaxProbs];
  int splits[kRankMaxProbs], order[kRankMaxProbs];
  int64_t kbps[kRankMaxProbs];
  for (int i = 0; i < n; ++i) {
    sh[i].m_tiles = (ps[i].rows + kBM - 1) / kBM;
    sh[i].tiles = sh[i].m_tiles * ps[i].n_tiles;
    sh[i].nkb = (ps[i].kext + kBK - 1) / kBK;
  }
  plan_rank(sh, n, sms, splits);
  rank_order(sh, splits, n, kbps, order);
  // lay the problems out as the launcher does
  static RankArgs a;
  std::memset(&a, 0, sizeof(a));
  int64_t units = 0;
  for (int oi = 0; oi < n; ++oi) {
    const int i = order[oi];
    RankProb &q = a.prob[a.nprob++];
    q.rows = (int)ps[i].rows;
    q.m_tiles = (int)sh[i].m_tiles;
    q.n_tiles = ps[i].n_tiles;
    q.nkb = (int)sh[i].nkb;
    q.splits = splits[i];
    q.kb_per_split = (int)kbps[i];
    q.unit0 = (int)units;
    units += sh[i].tiles * splits[i];
    CHECK(splits[i] >= 1 && (int64_t)(splits[i] - 1) * kbps[i] < sh[i].nkb,
          "problem %d: split %d of %lld k-blocks (%lld per split) is empty\n", i, splits[i], (long long)sh[i].nkb,
          (long long)kbps[i]);
  }
  a.units = (int)units;
  const int G = (int)std::min<int64_t>(units, sms);
  std::vector<int> seen((size_t)units, 0);
  // coverage[p][tile][kb]
  std::vector<std::vector<std::vector<int>>> cov(n);
  for (int p = 0; p < n; ++p)
    cov[p].assign((size_t)(a.prob[p].m_tiles * a.prob[p].n_tiles), std::vector<int>((size_t)a.prob[p].nkb, 0));
  for (int b = 0; b < G; ++b) {
    int last = -1;
    for (int k = 0; k * G < a.units; ++k) {
      const int u = rank_unit_at(k, G, b);
      if (u >= a.units) continue;
      CHECK(u > last, "CTA %d: unit %d after unit %d\n", b, u, last);
      last = u;
      ++seen[(size_t)u];
      const RankUnit ru = rank_unit(a, u);
      CHECK(ru.p >= 0 && ru.p < n, "unit %d: problem %d\n", u, ru.p);
      if (ru.p < 0 || ru.p >= n) continue;
      const RankProb &q = a.prob[ru.p];
      const bool in = ru.mt >= 0 && ru.mt < q.m_tiles && ru.nt >= 0 && ru.nt < q.n_tiles && ru.split >= 0 &&
                      ru.split < q.splits;
      CHECK(in, "unit %d: tile (%d, %d) split %d out of range\n", u, ru.mt, ru.nt, ru.split);
      if (!in) continue;
      const int kb0 = ru.split * q.kb_per_split, kb1 = std::min(q.nkb, kb0 + q.kb_per_split);
      CHECK(kb0 < kb1, "unit %d: empty k range [%d, %d)\n", u, kb0, kb1);
      for (int kb = kb0; kb < kb1; ++kb) ++cov[ru.p][(size_t)(ru.mt * q.n_tiles + ru.nt)][(size_t)kb];
    }
  }
  for (int64_t u = 0; u < units; ++u) CHECK(seen[(size_t)u] == 1, "unit %lld visited %d times\n", (long long)u, seen[(size_t)u]);
  for (int p = 0; p < n; ++p)
    for (auto &t : cov[p])
      for (int c : t) CHECK(c == 1, "problem %d: a k-block covered %d times\n", p, c);
}

int main() {
  std::vector<std::vector<P>> lists;
  const int64_t M = 8192;
  // LLaMA-7B backward groups: G (rows M, reduction N) and dL2 (rows N, reduction M), then dL1 sets
  auto g_dl2 = [&](std::vector<P> &v, int64_t N) {
    v.push_back({M, N, 1});
    v.push_back({N, M, 1});
  };
  {
    std::vector<P> v;
    g_dl2(v, 4096);
    lists.push_back(v);   // o or down alone
  }
  {
    std::vector<P> v;
    g_dl2(v, 11008);
    g_dl2(v, 11008);
    lists.push_back(v);   // gate, up
  }
  {
    std::vector<P> v;
    for (int i = 0; i < 3; ++i) g_dl2(v, 4096);
    lists.push_back(v);   // q, k, v
  }
  lists.push_back({{4096, M, 3}});     // dL1 of q, k, v on H
  lists.push_back({{4096, M, 2}});     // dL1 of gate, up
  lists.push_back({{11008, M, 1}});    // dL1 of down
  lists.push_back({{M, 4096, 5}});     // T of q, k, v, gate, up
  lists.push_back({{M, 11008, 1}});    // T of down
  {
    std::vector<P> v;                  // LLaMA-65B gate, up
    g_dl2(v, 22016);
    g_dl2(v, 22016);
    lists.push_back(v);
  }
  // ragged and tiny: few tokens, odd widths, a full list of 16 problems
  lists.push_back({{1, 72, 1}, {72, 1, 1}});
  lists.push_back({{129, 520, 1}, {520, 129, 1}, {333, 64, 1}});
  {
    std::vector<P> v;
    for (int i = 0; i < 16; ++i) v.push_back({(int64_t)(97 * (i + 1)), (int64_t)(64 * (i % 5 + 1) + 8 * i), 1 + i % 3});
    lists.push_back(v);
  }
  srand(7);
  for (int t = 0; t < 200; ++t) {
    std::vector<P> v;
    const int n = 1 + rand() % kRankMaxProbs;
    for (int i = 0; i < n; ++i) v.push_back({1 + rand() % 20000, 1 + rand() % 20000, 1 + rand() % 4});
    lists.push_back(v);
  }
  for (auto &l : lists)
    for (int sms : {148, 132, 7, 1}) check(l, sms);
  std::printf("%zu problem lists, %d wrong\n", lists.size(), wrong);
  return wrong ? 1 : 0;
}
