// Host-side tiling plan for the tensor-core attention kernel (see basa_internal.h).
#include <algorithm>
#include <cstring>
#include <vector>

#include "basa_internal.h"

namespace basa {
namespace {

struct Part {
  int start, len;  // window-local start and length along one axis
};

// Parts of a window along one axis: one part, or two when the window wraps.
std::vector<Part> axis_parts(int w, int s, bool wraps) {
  if (!wraps) return {{0, w}};
  const int a = w - (s % w);  // tokens before the grid edge
  return {{0, a}, {a, w - a}};
}

struct RawPiece {
  int lt, ly, lx, ct, cy, cx;
  int rows() const { return ct * cy * cx; }
  int padded() const { return (rows() + 7) / 8 * 8; }
};

struct TypePlan {
  std::vector<RawPiece> pieces;        // in tile order
  std::vector<std::vector<int>> tiles;  // indices into pieces
  std::vector<int> dest;                // per piece
};

// Cut every sub-box of a window type into boxes of <= 128 tokens, then pack them
// into 128-row tiles (first fit, largest first) at 8-row aligned offsets.
TypePlan plan_type(const basa_params &p, int type, int ct_cap, int cy_cap) {
  TypePlan tp;
  const auto pt = axis_parts(p.wt, p.st, type & 1);
  const auto py = axis_parts(p.wh, p.sy, type & 2);
  const auto px = axis_parts(p.ww, p.sx, type & 4);
  std::vector<RawPiece> raw;
  for (const Part &a : pt)
    for (const Part &b : py)
      for (const Part &c : px) {
        const int cx = std::min(c.len, kTileRows);
        const int cy = std::min({cy_cap, b.len, std::max(1, kTileRows / cx)});
        const int ct = std::min({ct_cap, a.len, std::max(1, kTileRows / (cy * cx))});
        for (int t0 = 0; t0 < a.len; t0 += ct)
          for (int y0 = 0; y0 < b.len; y0 += cy)
            for (int x0 = 0; x0 < c.len; x0 += cx)
              raw.push_back({a.start + t0, b.start + y0, c.start + x0, std::min(ct, a.len - t0),
                             std::min(cy, b.len - y0), std::min(cx, c.len - x0)});
      }
  std::vector<int> order(raw.size());
  for (size_t i = 0; i < order.size(); ++i) order[i] = int(i);
  std::stable_sort(order.begin(), order.end(), [&](int i, int j) { return raw[i].padded() > raw[j].padded(); });
  std::vector<int> used;
  std::vector<std::vector<int>> bins;
  std::vector<int> dest(raw.size());
  for (int i : order) {
    const int need = raw[i].padded();
    size_t b = 0;
    while (b < bins.size() && used[b] + need > kTileRows) ++b;
    if (b == bins.size()) {
      bins.emplace_back();
      used.push_back(0);
    }
    dest[i] = used[b];
    used[b] += need;
    bins[b].push_back(i);
  }
  for (auto &bin : bins) {
    std::vector<int> ids;
    for (int i : bin) {
      ids.push_back(int(tp.pieces.size()));
      tp.pieces.push_back(raw[i]);
      tp.dest.push_back(dest[i]);
    }
    tp.tiles.push_back(ids);
  }
  return tp;
}

// Number of windows of each type.
long long type_count(const basa_params &p, int type) {
  const int nw[3] = {p.T / p.wt, p.H / p.wh, p.W / p.ww};
  const int w[3] = {p.wt, p.wh, p.ww};
  const int s[3] = {p.st, p.sy, p.sx};
  long long c = 1;
  for (int a = 0; a < 3; ++a) {
    const bool wraps = (s[a] % w[a]) != 0;
    const bool bit = (type >> a) & 1;
    if (bit) c *= wraps ? 1 : 0;
    else c *= wraps ? nw[a] - 1 : nw[a];
  }
  return c;
}

}  // namespace

basa_status build_window_plan(const basa_params &p, WindowPlan *plan) {
  std::memset(plan, 0, sizeof(*plan));
  long long best_cost = -1, best_pieces = 0;
  int best_shapes = 0, best_ct = 1, best_cy = 1;
  for (int ct_cap = 1; ct_cap <= p.wt; ++ct_cap)
    for (int cy_cap = 1; cy_cap <= p.wh; ++cy_cap) {
      long long cost = 0, pieces = 0;
      std::vector<long long> shapes;
      int tiles = 0, npieces = 0;
      for (int type = 0; type < 8; ++type) {
        const long long cnt = type_count(p, type);
        if (cnt == 0) continue;
        TypePlan tp = plan_type(p, type, ct_cap, cy_cap);
        cost += cnt * (long long)tp.tiles.size();
        pieces += cnt * (long long)tp.pieces.size();
        tiles += int(tp.tiles.size());
        npieces += int(tp.pieces.size());
        for (auto &rp : tp.pieces) {
          long long key = (long long)rp.ct << 40 | (long long)rp.cy << 20 | rp.cx;
          if (std::find(shapes.begin(), shapes.end(), key) == shapes.end()) shapes.push_back(key);
        }
      }
      if (int(shapes.size()) > kMaxShapes || tiles > kMaxTiles || npieces > kMaxPieces) continue;
      const bool better = best_cost < 0 || cost < best_cost || (cost == best_cost && pieces < best_pieces) ||
                          (cost == best_cost && pieces == best_pieces && int(shapes.size()) < best_shapes);
      if (better) {
        best_cost = cost;
        best_pieces = pieces;
        best_shapes = int(shapes.size());
        best_ct = ct_cap;
        best_cy = cy_cap;
      }
    }
  if (best_cost < 0) return BASA_ERR_UNSUPPORTED;

  for (int type = 0; type < 8; ++type) {
    plan->type[type].first_tile = uint16_t(plan->n_tiles);
    plan->type[type].n_tiles = 0;
    if (type_count(p, type) == 0) continue;
    TypePlan tp = plan_type(p, type, best_ct, best_cy);
    for (auto &ids : tp.tiles) {
      PlanTile &t = plan->tile[plan->n_tiles++];
      t.first_piece = uint16_t(plan->n_pieces);
      t.n_pieces = uint16_t(ids.size());
      t.valid_rows = 0;
      for (int id : ids) {
        const RawPiece &rp = tp.pieces[id];
        int shape = -1;
        for (int s = 0; s < plan->n_shapes; ++s)
          if (plan->shape[s].ct == rp.ct && plan->shape[s].cy == rp.cy && plan->shape[s].cx == rp.cx) shape = s;
        if (shape < 0) {
          shape = plan->n_shapes++;
          plan->shape[shape] = {int16_t(rp.ct), int16_t(rp.cy), int16_t(rp.cx), int16_t(rp.rows())};
        }
        PlanPiece &pc = plan->piece[plan->n_pieces++];
        pc.lt = int16_t(rp.lt);
        pc.ly = int16_t(rp.ly);
        pc.lx = int16_t(rp.lx);
        pc.shape = uint8_t(shape);
        pc.dest = uint8_t(tp.dest[id]);
        for (int r = tp.dest[id]; r < tp.dest[id] + rp.rows(); ++r) t.mask[r >> 5] |= 1u << (r & 31);
        t.valid_rows = uint16_t(t.valid_rows + rp.rows());
      }
      if (t.valid_rows < kTileRows) plan->zero_fill = 1;
    }
    plan->type[type].n_tiles = uint16_t(tp.tiles.size());
    plan->max_pairs = std::max(plan->max_pairs, int((tp.tiles.size() + 1) / 2));
  }
  return BASA_OK;
}

}  // namespace basa
