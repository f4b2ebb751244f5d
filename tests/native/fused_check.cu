// Host check of the fused pre-pass index arithmetic (csrc/pool_route_fused.cu): the
// real plan_fused, build_runs and build_cells, compiled into this file. Reads
// geometries "T H W wt wh ww st sy sx pt ph pw head_dim dtype" (dtype 0 = bf16,
// 1 = f32) from stdin and prints "ok <boxes> <max_cells>", "unsupported" or
// "fail <reason>" per line. Checks, over every box of the grid: box extents are
// whole pool patches dividing the grid; each axis's cells tile the box exactly,
// each inside the window of its run and the pool patch it names; cell and run
// counts stay within the kernel's limits; every pool patch is summed by exactly one
// box; every window's slots (box positions along its run of boxes) are distinct,
// inside the slot grid, cover the window's tokens exactly once in total, and are
// exactly the slots the reduction kernel reads.
#include <cstdio>
#include <set>
#include <vector>

#include "../../sparse_window_attention_b200/csrc/pool_route_fused.cu"

namespace basa {
// the top-k launch is not exercised here
basa_status launch_topk(const float *, const float *, int32_t *, float *, const basa_params &, cudaStream_t) {
  return BASA_OK;
}
}  // namespace basa

using namespace basa;

static const char *check(const basa_params &p, const FusedPlan &fp, long *boxes) {
  const int G[3] = {p.T, p.H, p.W}, P[3] = {p.pt, p.ph, p.pw}, w[3] = {p.wt, p.wh, p.ww}, s[3] = {p.st, p.sy, p.sx};
  const int nw[3] = {G[0] / w[0], G[1] / w[1], G[2] / w[2]};
  for (int a = 0; a < 3; ++a) {
    if (fp.e[a] % P[a] || G[a] % fp.e[a] || fp.nb[a] != G[a] / fp.e[a]) return "box extents";
    if (fp.e[a] > 256) return "box extent above 256";
  }
  if (fp.max_cells > kMaxCells) return "max_cells above the kernel limit";
  if (cell_smem_bytes(fp.max_cells, p.head_dim, p.dtype) > 227 * 1024) return "shared memory";
  const long nwin = long(nw[0]) * nw[1] * nw[2];
  std::vector<std::set<long>> win_slots(static_cast<size_t>(nwin));
  std::vector<long> cover(size_t(nwin), 0);
  const long npool = long(G[0] / P[0]) * (G[1] / P[1]) * (G[2] / P[2]);
  std::vector<int> pooled(size_t(npool), 0);
  *boxes = 0;
  for (int bt = 0; bt < fp.nb[0]; ++bt)
    for (int by = 0; by < fp.nb[1]; ++by)
      for (int bx = 0; bx < fp.nb[2]; ++bx) {
        ++*boxes;
        const int box[3] = {bt, by, bx};
        AxisRun runs[3][kMaxAxisRuns];
        AxisCell cells[3][kMaxAxisCells];
        int nr[3], nc[3];
        for (int a = 0; a < 3; ++a) {
          build_runs(box[a] * fp.e[a], fp.e[a], w[a], s[a], G[a], runs[a], &nr[a]);
          build_cells(runs[a], nr[a], P[a], cells[a], &nc[a]);
          if (nr[a] >= kMaxAxisRuns || nc[a] >= kMaxAxisCells) return "run or cell table full";
          std::vector<int> seen(size_t(fp.e[a]), 0);
          for (int i = 0; i < nc[a]; ++i) {
            const AxisCell &c = cells[a][i];
            if (c.lo >= c.hi || c.run < 0 || c.run >= nr[a]) return "cell bounds";
            for (int x = c.lo; x < c.hi; ++x) {
              ++seen[size_t(x)];
              const int g = box[a] * fp.e[a] + x;
              if (((g - s[a]) % G[a] + G[a]) % G[a] / w[a] != runs[a][c.run].j) return "cell outside its window";
              if (x / P[a] != c.patch) return "cell outside its patch";
            }
          }
          for (int v : seen)
            if (v != 1) return "cells do not tile the box";
        }
        if (long(nc[0]) * nc[1] * nc[2] > fp.max_cells) return "more cells than planned";
        // pool patches of the box
        const int np[3] = {fp.e[0] / P[0], fp.e[1] / P[1], fp.e[2] / P[2]};
        for (int a0 = 0; a0 < np[0]; ++a0)
          for (int a1 = 0; a1 < np[1]; ++a1)
            for (int a2 = 0; a2 < np[2]; ++a2) {
              const long gp = ((long(bt * np[0] + a0) * (G[1] / P[1])) + by * np[1] + a1) * (G[2] / P[2]) + bx * np[2] + a2;
              ++pooled[size_t(gp)];
            }
        // window partial sums of the box
        for (int it = 0; it < nr[0]; ++it)
          for (int iy = 0; iy < nr[1]; ++iy)
            for (int ix = 0; ix < nr[2]; ++ix) {
              const int j[3] = {runs[0][it].j, runs[1][iy].j, runs[2][ix].j};
              const int ri[3] = {it, iy, ix};
              long k = 0, tokens = 1;
              for (int a = 0; a < 3; ++a) {
                const int o = (j[a] * w[a] + s[a]) % G[a];
                const int ka = (box[a] - o / fp.e[a] + fp.nb[a]) % fp.nb[a];
                if (ka >= fp.K[a]) return "slot outside the slot grid";
                k = k * fp.K[a] + ka;
                long len = 0;
                for (int i = 0; i < nc[a]; ++i)
                  if (cells[a][i].run == ri[a]) len += cells[a][i].hi - cells[a][i].lo;
                tokens *= len;
              }
              const long win = (long(j[0]) * nw[1] + j[1]) * nw[2] + j[2];
              if (!win_slots[size_t(win)].insert(k).second) return "two boxes write one slot";
              cover[size_t(win)] += tokens;
            }
      }
  for (int v : pooled)
    if (v != 1) return "pool patch not summed exactly once";
  for (long win = 0; win < nwin; ++win) {
    if (cover[size_t(win)] != long(w[0]) * w[1] * w[2]) return "window not covered exactly once";
    const int j[3] = {int(win / (nw[1] * nw[2])), int((win / nw[2]) % nw[1]), int(win % nw[2])};
    std::set<long> reads;
    int n[3];
    for (int a = 0; a < 3; ++a) {
      const int o = (j[a] * w[a] + s[a]) % G[a];
      n[a] = std::min((o + w[a] - 1) / fp.e[a] - o / fp.e[a] + 1, fp.nb[a]);
    }
    for (int a = 0; a < n[0]; ++a)
      for (int b = 0; b < n[1]; ++b)
        for (int c = 0; c < n[2]; ++c) reads.insert((long(a) * fp.K[1] + b) * fp.K[2] + c);
    if (reads != win_slots[size_t(win)]) return "reduction reads other slots than were written";
  }
  return nullptr;
}

int main() {
  basa_params p{};
  p.B = 1;
  p.heads = 1;
  p.routed_k = 1;
  int dt = 0;
  while (std::scanf("%d %d %d %d %d %d %d %d %d %d %d %d %d %d", &p.T, &p.H, &p.W, &p.wt, &p.wh, &p.ww, &p.st, &p.sy,
                    &p.sx, &p.pt, &p.ph, &p.pw, &p.head_dim, &dt) == 14) {
    p.dtype = dt ? BASA_F32 : BASA_BF16;
    FusedPlan fp;
    if (plan_fused(p, &fp) != BASA_OK) {
      std::printf("unsupported\n");
      continue;
    }
    long boxes = 0;
    const char *err = check(p, fp, &boxes);
    if (err) std::printf("fail %s\n", err);
    else std::printf("ok %ld %d\n", boxes, fp.max_cells);
  }
  return 0;
}
