// Host-side check of the window tiling plan (csrc/plan.cpp). Reads geometries
// "T H W wt wh ww st sy sx" from stdin, one per line, and for each prints
// "ok <tiles> <pieces>" or "fail <reason>" (or "unsupported"). For every window of
// the shifted grid it checks that the window type's pieces cover the window's
// tokens exactly once, that every piece is one in-bounds box of the original grid
// (it does not wrap), that pieces sit at 8-row aligned offsets inside their 128-row
// tile without overlap, and that each tile's row mask and valid-row count match.
#include <cstdio>
#include <vector>

#include "../../sparse_window_attention_b200/csrc/basa_internal.h"

using namespace basa;

static const char *check(const basa_params &p, const WindowPlan &plan) {
  const Geo g = make_geo(p);
  std::vector<int> seen(size_t(g.N), -1);
  for (int w = 0; w < g.nWin; ++w) {
    int ot, oy, ox, ty;
    window_origin(g, w, &ot, &oy, &ox, &ty);
    const PlanType &pt = plan.type[ty];
    if (pt.n_tiles == 0) return "window type without tiles";
    long count = 0;
    for (int t = 0; t < pt.n_tiles; ++t) {
      const PlanTile &tile = plan.tile[pt.first_tile + t];
      int used[kTileRows] = {0};
      int valid = 0;
      for (int i = 0; i < tile.n_pieces; ++i) {
        const PlanPiece &pc = plan.piece[tile.first_piece + i];
        const PlanShape &sh = plan.shape[pc.shape];
        if (pc.dest % 8) return "piece not 8-row aligned";
        if (pc.dest + sh.rows > kTileRows) return "piece overflows its tile";
        if (sh.rows != sh.ct * sh.cy * sh.cx) return "shape rows";
        for (int r = pc.dest; r < pc.dest + sh.rows; ++r) {
          if (used[r]++) return "pieces overlap";
          if (!((tile.mask[r >> 5] >> (r & 31)) & 1u)) return "mask misses a row";
        }
        valid += sh.rows;
        if (pc.lt + sh.ct > p.wt || pc.ly + sh.cy > p.wh || pc.lx + sh.cx > p.ww) return "piece leaves the window";
        const int t0 = (ot + pc.lt) % p.T, y0 = (oy + pc.ly) % p.H, x0 = (ox + pc.lx) % p.W;
        if (t0 + sh.ct > p.T || y0 + sh.cy > p.H || x0 + sh.cx > p.W) return "box wraps around the grid";
        for (int a = 0; a < sh.ct; ++a)
          for (int b = 0; b < sh.cy; ++b)
            for (int c = 0; c < sh.cx; ++c) {
              const int tt = (ot + pc.lt + a) % p.T, yy = (oy + pc.ly + b) % p.H, xx = (ox + pc.lx + c) % p.W;
              if (tt != t0 + a || yy != y0 + b || xx != x0 + c) return "box is not the window's tokens";
              const long n = (long(tt) * p.H + yy) * p.W + xx;
              if (seen[size_t(n)] != -1) return "token covered twice";
              seen[size_t(n)] = w;
              ++count;
            }
      }
      if (valid != tile.valid_rows) return "valid_rows";
      int pop = 0;
      for (int i = 0; i < 4; ++i) pop += __builtin_popcount(tile.mask[i]);
      if (pop != valid) return "mask population";
    }
    if (count != long(p.wt) * p.wh * p.ww) return "window not fully covered";
  }
  for (int v : seen)
    if (v < 0) return "token in no window";
  return nullptr;
}

int main() {
  basa_params p{};
  p.B = 1;
  p.heads = 1;
  p.head_dim = 128;
  while (std::scanf("%d %d %d %d %d %d %d %d %d", &p.T, &p.H, &p.W, &p.wt, &p.wh, &p.ww, &p.st, &p.sy, &p.sx) == 9) {
    WindowPlan plan;
    if (build_window_plan(p, &plan) != BASA_OK) {
      std::printf("unsupported\n");
      continue;
    }
    const char *err = check(p, plan);
    if (err) std::printf("fail %s\n", err);
    else std::printf("ok %d %d\n", plan.n_tiles, plan.n_pieces);
  }
  return 0;
}
