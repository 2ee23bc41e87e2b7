// Host-side check of the forward kernel's work schedule, using the kernel's
// own decode functions (compiled for the host here).  Run by
// tests/test_scheduler.py; exit status 0 and "sched ok" when every check holds.
#include <cuda.h>

#include <cstdio>
#include <utility>
#include <vector>

#include "fa_fwd_short.cuh"
#include "fa_fwd_short_wg.cuh"
#include "fa_fwd_tc.cuh"

using fa::TcParams;
using fa::Unit;

static int fails = 0;
#define CHECK(cond, ...)                  \
  do {                                    \
    if (!(cond)) {                        \
      if (fails < 20) {                   \
        std::printf(__VA_ARGS__);         \
        std::printf("\n");                \
      }                                   \
      ++fails;                            \
    }                                     \
  } while (0)

static int cdiv(int a, int b) { return (a + b - 1) / b; }

static TcParams params(int B, int H, int Nq, int Nkv, int causal, int chunk) {
  TcParams p{};
  p.B = B; p.H = H; p.Nq = Nq; p.Nkv = Nkv; p.causal = causal;
  p.n_pairs = (cdiv(Nq, 128) + 1) / 2;
  p.n_units = B * H * p.n_pairs;
  p.chunk_heads = chunk;
  p.kv_group = 1;
  return p;
}

// KV tiles with a visible key for some row of Q tile qt (all 128 rows of the
// tile, as the kernel computes them): brute force over the rows.
static int tiles_needed(int qt, int Nkv, int causal) {
  int lim = 0;
  for (int r = qt * 128; r < qt * 128 + 128; ++r) {
    const int l = causal ? (r + 1 < Nkv ? r + 1 : Nkv) : Nkv;
    if (l > lim) lim = l;
  }
  return cdiv(lim, 128);
}

static void check_plain(int B, int H, int Nq, int Nkv, int causal, int chunk) {
  TcParams p = params(B, H, Nq, Nkv, causal, chunk);
  const int qtiles = cdiv(Nq, 128);
  std::vector<int> seen((size_t)B * H * qtiles, 0);
  int prev_chunk = -1, prev_pair = 1 << 30;
  for (int t = 0; t < p.n_units; ++t) {
    int sp = 0;
    const Unit w = fa::decode_unit_t<false, false>(t, p, sp);
    CHECK(w.b >= 0 && w.b < B && w.h >= 0 && w.h < H && w.qt0 % 2 == 0 && w.qt0 < qtiles,
          "plain B%d H%d Nq%d: ticket %d decodes outside the problem", B, H, Nq, t);
    if (!(w.b >= 0 && w.b < B && w.h >= 0 && w.h < H && w.qt0 >= 0 && w.qt0 < qtiles)) continue;
    seen[((size_t)w.b * H + w.h) * qtiles + w.qt0]++;
    CHECK(w.n0 == tiles_needed(w.qt0, Nkv, causal), "plain: n0 %d for tile %d", w.n0, w.qt0);
    if (w.qt0 + 1 < qtiles) {
      CHECK(w.active1 == 1, "plain: second tile %d inactive", w.qt0 + 1);
      seen[((size_t)w.b * H + w.h) * qtiles + w.qt0 + 1]++;
      CHECK(w.n1 == tiles_needed(w.qt0 + 1, Nkv, causal), "plain: n1 %d for tile %d", w.n1, w.qt0 + 1);
    } else {
      CHECK(w.active1 == 0 && w.n1 == 0, "plain: a second tile past the last (%d)", w.qt0 + 1);
    }
    // within a chunk of (batch, head) pairs the heaviest Q-tile pairs come first
    const int ch = t / (chunk * p.n_pairs);
    const int pair = w.qt0 / 2;
    if (ch == prev_chunk) CHECK(pair <= prev_pair, "plain: pair %d after pair %d in one chunk", pair, prev_pair);
    prev_chunk = ch;
    prev_pair = pair;
  }
  for (size_t i = 0; i < seen.size(); ++i)
    CHECK(seen[i] == 1, "plain B%d H%d Nq%d Nkv%d causal%d chunk%d: tile %zu scheduled %d times", B, H, Nq, Nkv,
          causal, chunk, i, seen[i]);
}

static void check_band(int B, int H, int Nq, int Nkv, int pre, int next, int chunk) {
  TcParams p = params(B, H, Nq, Nkv, 0, chunk);
  p.band.pre_tokens = pre;
  p.band.next_tokens = next;
  const int qtiles = cdiv(Nq, 128);
  std::vector<int> seen((size_t)B * H * qtiles, 0);
  for (int t = 0; t < p.n_units; ++t) {
    int sp = 0;
    const Unit w = fa::decode_unit_t<true, false>(t, p, sp);
    CHECK(w.s1 >= 0, "band: tile 1 starts before tile 0 (s1 = %d)", w.s1);
    for (int i = 0; i < 2; ++i) {
      const int qt = w.qt0 + i;
      if (qt >= qtiles) continue;
      seen[((size_t)w.b * H + w.h) * qtiles + qt]++;
      const int lo = w.lo0 + (i ? w.s1 : 0), n = i ? w.n1 : w.n0;
      // every visible key of every valid row lies in [lo, lo + n)
      bool lo_used = false, hi_used = false;
      for (int r = qt * 128; r < qt * 128 + 128; ++r) {
        const int k0 = r - pre < 0 ? 0 : r - pre;
        const int k1 = r + next + 1 < Nkv ? r + next + 1 : Nkv;  // visible keys [k0, k1)
        if (k0 >= k1) continue;
        if (r < Nq)
          CHECK(k0 / 128 >= lo && (k1 - 1) / 128 < lo + n, "band pre%d next%d: row %d's keys [%d, %d) outside tiles [%d, %d)",
                pre, next, r, k0, k1, lo, lo + n);
        if (k0 / 128 <= lo && (k1 - 1) / 128 >= lo) lo_used = true;
        if (k0 / 128 <= lo + n - 1 && (k1 - 1) / 128 >= lo + n - 1) hi_used = true;
      }
      CHECK(n >= 1 && lo_used && hi_used, "band pre%d next%d: tile %d's range [%d, %d) has an unused end", pre, next,
            qt, lo, lo + n);
    }
  }
  for (size_t i = 0; i < seen.size(); ++i) CHECK(seen[i] == 1, "band: tile %zu scheduled %d times", i, seen[i]);
}

static void check_split(int B, int H, int Nq, int Nkv, int S_req, int chunk) {
  TcParams p = params(B, H, Nq, Nkv, 0, chunk);
  const int nt = cdiv(Nkv, 128);
  const int st = cdiv(nt, S_req < nt ? S_req : nt);
  p.split.split_tiles = st;
  p.split.n_splits = cdiv(nt, st);
  p.n_units = B * H * p.n_pairs * p.split.n_splits;
  std::vector<int> covered((size_t)B * H * p.n_pairs * nt, 0);
  for (int t = 0; t < p.n_units; ++t) {
    int sp = -1;
    const Unit w = fa::decode_unit_t<false, true>(t, p, sp);
    CHECK(sp >= 0 && sp < p.split.n_splits && w.n0 >= 1, "split: ticket %d slice %d with %d tiles", t, sp, w.n0);
    if (!(sp >= 0 && sp < p.split.n_splits)) continue;
    CHECK(w.lo0 == sp * st && w.lo0 + w.n0 <= nt, "split: slice %d at [%d, %d)", sp, w.lo0, w.lo0 + w.n0);
    for (int k = w.lo0; k < w.lo0 + w.n0 && k < nt; ++k)
      covered[(((size_t)w.b * H + w.h) * p.n_pairs + w.qt0 / 2) * nt + k]++;
  }
  for (size_t i = 0; i < covered.size(); ++i)
    CHECK(covered[i] == 1, "split B%d H%d Nq%d Nkv%d S%d: key tile %zu covered %d times", B, H, Nq, Nkv, S_req, i,
          covered[i]);
}

// The short-key kernel's static schedule: CTA c of G takes query tiles
// [t0, t1); the ranges tile [0, n_tiles) exactly, none is empty and their
// sizes differ by at most one; every tile decodes to a distinct (b, h, qt)
// inside the problem with the K/V head h / (H / Hkv).
static void check_short(int B, int H, int Hkv, int Nq, int G) {
  fa::ShParams p{};
  p.B = B; p.H = H; p.Nq = Nq;
  p.qtiles = cdiv(Nq, 128);
  p.n_tiles = B * H * p.qtiles;
  p.kv_group = H / Hkv;
  if (G > p.n_tiles) G = p.n_tiles;
  std::vector<int> seen((size_t)p.n_tiles, 0);
  int expect = 0, lo = 1 << 30, hi = 0;
  for (int c = 0; c < G; ++c) {
    int t0, t1;
    fa::sh_range(c, G, p.n_tiles, t0, t1);
    CHECK(t0 == expect && t1 > t0, "short B%d H%d Nq%d G%d: CTA %d range [%d, %d)", B, H, Nq, G, c, t0, t1);
    expect = t1;
    lo = t1 - t0 < lo ? t1 - t0 : lo;
    hi = t1 - t0 > hi ? t1 - t0 : hi;
    for (int t = t0; t < t1; ++t) {
      const fa::ShTile x = fa::sh_decode(t, p);
      CHECK(x.b >= 0 && x.b < B && x.h >= 0 && x.h < H && x.qt >= 0 && x.qt < p.qtiles,
            "short: tile %d decodes outside the problem", t);
      CHECK(x.kv == x.b * Hkv + x.h / (H / Hkv), "short: tile %d K/V key %d", t, x.kv);
      if (x.b >= 0 && x.b < B && x.h >= 0 && x.h < H && x.qt >= 0 && x.qt < p.qtiles)
        seen[((size_t)x.b * H + x.h) * p.qtiles + x.qt]++;
    }
  }
  CHECK(expect == p.n_tiles && hi - lo <= 1, "short B%d H%d Nq%d G%d: ranges end at %d, sizes %d..%d", B, H, Nq, G,
        expect, lo, hi);
  for (size_t i = 0; i < seen.size(); ++i) CHECK(seen[i] == 1, "short: tile %zu scheduled %d times", i, seen[i]);
}

// The four-pipeline short-key kernel: the same contiguous CTA ranges, and
// warpgroup w of a CTA with n tiles takes tiles w, w + 4, ... (its count
// `mine`, as the kernel computes it), so the four warpgroups cover the range
// exactly once; every tile decodes inside the problem.
static void check_short_wg(int B, int H, int Hkv, int Nq, int G) {
  fa::SwParams p{};
  p.B = B; p.H = H; p.Nq = Nq;
  p.qtiles = cdiv(Nq, 128);
  p.n_tiles = B * H * p.qtiles;
  p.kv_group = H / Hkv;
  if (G > p.n_tiles) G = p.n_tiles;
  std::vector<int> seen((size_t)p.n_tiles, 0);
  int expect = 0;
  for (int c = 0; c < G; ++c) {
    int t0, t1;
    fa::sw_range(c, G, p.n_tiles, t0, t1);
    CHECK(t0 == expect && t1 > t0, "short-wg B%d H%d Nq%d G%d: CTA %d range [%d, %d)", B, H, Nq, G, c, t0, t1);
    expect = t1;
    const int n = t1 - t0;
    for (int wg = 0; wg < fa::SW_WGS; ++wg) {
      const int mine = n > wg ? (n - wg + fa::SW_WGS - 1) / fa::SW_WGS : 0;
      for (int j = 0; j < mine; ++j) {
        const int t = t0 + wg + fa::SW_WGS * j;
        CHECK(t < t1, "short-wg: warpgroup %d tile %d past its CTA's range", wg, t);
        const fa::SwTile x = fa::sw_decode(t, p);
        CHECK(x.b >= 0 && x.b < B && x.h >= 0 && x.h < H && x.qt >= 0 && x.qt < p.qtiles,
              "short-wg: tile %d decodes outside the problem", t);
        CHECK(x.kv == x.b * Hkv + x.h / (H / Hkv), "short-wg: tile %d K/V key %d", t, x.kv);
        if (t >= 0 && t < p.n_tiles) seen[(size_t)t]++;
      }
    }
  }
  CHECK(expect == p.n_tiles, "short-wg B%d H%d Nq%d G%d: ranges end at %d", B, H, Nq, G, expect);
  for (size_t i = 0; i < seen.size(); ++i) CHECK(seen[i] == 1, "short-wg: tile %zu scheduled %d times", i, seen[i]);
}

int main() {
  const int short_shapes[][4] = {{1, 1, 1, 1}, {2, 8, 8, 4096}, {4, 32, 32, 4096}, {5, 200, 100, 100},
                                 {1, 8, 2, 2000}, {3, 7, 7, 129}};
  for (const auto& s : short_shapes)
    for (int G : {1, 7, 148, 1 << 20}) {
      check_short(s[0], s[1], s[2], s[3], G);
      check_short_wg(s[0], s[1], s[2], s[3], G);
    }

  const int shapes[][4] = {{1, 1, 1, 1}, {1, 2, 300, 333}, {2, 3, 129, 127}, {1, 40, 1024, 1024},
                           {2, 5, 777, 2000}, {3, 7, 4096, 77}, {1, 1, 8192, 8192}};
  for (const auto& s : shapes) {
    for (int chunk : {1, 3, s[0] * s[1]}) {
      if (chunk > s[0] * s[1]) continue;
      for (int causal = 0; causal < 2; ++causal) check_plain(s[0], s[1], s[2], s[3], causal, chunk);
      // bands the entry point accepts: pre_tokens >= Nq - Nkv, so that every row sees a key
      for (const auto& pn : {std::pair<int, int>{200, 17}, {2047, 0}, {s[2] + s[3], 0}})
        if (pn.first >= s[2] - s[3]) check_band(s[0], s[1], s[2], s[3], pn.first, pn.second, chunk);
      for (int S : {1, 3, 7, 64}) check_split(s[0], s[1], s[2], s[3], S, chunk);
    }
  }
  if (fails == 0) std::printf("sched ok\n");
  return fails == 0 ? 0 : 1;
}
