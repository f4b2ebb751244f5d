// Host-side tiling plan for the tensor-core attention kernel (see basa_internal.h).
#include <algorithm>
#include <cstring>
#include <deque>
#include <memory>
#include <mutex>
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

// Cut every sub-box of a window type into boxes of <= 128 tokens (at most ct_cap x
// cy_cap x cx_cap), then pack them into 128-row tiles (first fit, largest first) at
// 8-row aligned offsets.
struct Caps {
  int ct, cy, cx;
};

struct Extent {
  int ct, cy, cx;
};

// Box extents used for one (t, y, x) combination of parts.
Extent piece_extent(const Caps &cap, const Part &a, const Part &b, const Part &c) {
  const int cx = std::min({cap.cx, c.len, kTileRows});
  const int cy = std::min({cap.cy, b.len, std::max(1, kTileRows / cx)});
  const int ct = std::min({cap.ct, a.len, std::max(1, kTileRows / (cy * cx))});
  return {ct, cy, cx};
}

struct TypeParts {
  std::vector<Part> t, y, x;
};

TypeParts type_parts(const basa_params &p, int type) {
  return {axis_parts(p.wt, p.st, type & 1), axis_parts(p.wh, p.sy, type & 2), axis_parts(p.ww, p.sx, type & 4)};
}

int ceil_div(int a, int b) { return (a + b - 1) / b; }

// Number of pieces a type is cut into (no packing needed).
long long count_pieces(const TypeParts &tp, const Caps &cap) {
  long long n = 0;
  for (const Part &a : tp.t)
    for (const Part &b : tp.y)
      for (const Part &c : tp.x) {
        const Extent e = piece_extent(cap, a, b, c);
        n += (long long)ceil_div(a.len, e.ct) * ceil_div(b.len, e.cy) * ceil_div(c.len, e.cx);
      }
  return n;
}

TypePlan plan_type(const basa_params &p, int type, const Caps &cap) {
  TypePlan tp;
  const TypeParts parts = type_parts(p, type);
  std::vector<RawPiece> raw;
  for (const Part &a : parts.t)
    for (const Part &b : parts.y)
      for (const Part &c : parts.x) {
        const Extent e = piece_extent(cap, a, b, c);
        for (int t0 = 0; t0 < a.len; t0 += e.ct)
          for (int y0 = 0; y0 < b.len; y0 += e.cy)
            for (int x0 = 0; x0 < c.len; x0 += e.cx)
              raw.push_back({a.start + t0, b.start + y0, c.start + x0, std::min(e.ct, a.len - t0),
                             std::min(e.cy, b.len - y0), std::min(e.cx, c.len - x0)});
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

// Distinct values ceil(L / k) over the part lengths L of one axis: the box
// extents that cut some part into k nearly equal boxes.
std::vector<int> cap_candidates(const std::vector<int> &lens) {
  std::vector<int> c;
  for (int L : lens)
    for (int k = 1; k <= L; ++k) {
      const int v = ceil_div(L, k);
      if (v <= kTileRows && std::find(c.begin(), c.end(), v) == c.end()) c.push_back(v);
    }
  return c;
}

// Sum over a type's pieces of their 8-row padded heights: tiles >= ceil(sum / 128).
long long padded_rows(const TypeParts &tp, const Caps &cap) {
  long long rows = 0;
  for (const Part &a : tp.t)
    for (const Part &b : tp.y)
      for (const Part &c : tp.x) {
        const Extent e = piece_extent(cap, a, b, c);
        for (int t0 = 0; t0 < a.len; t0 += e.ct)
          for (int y0 = 0; y0 < b.len; y0 += e.cy) {
            const int full = c.len / e.cx, rest = c.len % e.cx;
            const int hw = std::min(e.ct, a.len - t0) * std::min(e.cy, b.len - y0);
            rows += (long long)full * ((hw * e.cx + 7) / 8 * 8);
            if (rest) rows += (hw * rest + 7) / 8 * 8;
          }
      }
  return rows;
}

basa_status search_window_plan(const basa_params &p, WindowPlan *plan) {
  std::memset(plan, 0, sizeof(*plan));
  std::vector<int> types;
  std::vector<TypeParts> parts;
  std::vector<int> lt, ly, lx;
  for (int type = 0; type < 8; ++type) {
    if (type_count(p, type) == 0) continue;
    types.push_back(type);
    parts.push_back(type_parts(p, type));
    for (const Part &a : parts.back().t) lt.push_back(a.len);
    for (const Part &a : parts.back().y) ly.push_back(a.len);
    for (const Part &a : parts.back().x) lx.push_back(a.len);
  }
  const std::vector<int> ct_c = cap_candidates(lt), cy_c = cap_candidates(ly), cx_c = cap_candidates(lx);
  long long best_cost = -1, best_pieces = 0;
  int best_shapes = 0;
  Caps best{1, 1, 1};
  for (int cx : cx_c)
    for (int cy : cy_c)
      for (int ct : ct_c) {
        const Caps cap{ct, cy, cx};
        long long npieces = 0, lb = 0;
        for (size_t i = 0; i < types.size(); ++i) {
          npieces += count_pieces(parts[i], cap);
          lb += type_count(p, types[i]) * ((padded_rows(parts[i], cap) + kTileRows - 1) / kTileRows);
        }
        if (npieces > kMaxPieces) continue;
        if (best_cost >= 0 && lb > best_cost) continue;  // cannot beat the best plan so far
        long long cost = 0, pieces = 0;
        std::vector<long long> shapes;
        int tiles = 0;
        for (size_t i = 0; i < types.size(); ++i) {
          const long long cnt = type_count(p, types[i]);
          TypePlan tp = plan_type(p, types[i], cap);
          cost += cnt * (long long)tp.tiles.size();
          pieces += cnt * (long long)tp.pieces.size();
          tiles += int(tp.tiles.size());
          for (auto &rp : tp.pieces) {
            const long long key = (long long)rp.ct << 40 | (long long)rp.cy << 20 | rp.cx;
            if (std::find(shapes.begin(), shapes.end(), key) == shapes.end()) shapes.push_back(key);
          }
        }
        if (int(shapes.size()) > kMaxShapes || tiles > kMaxTiles) continue;
        const bool better = best_cost < 0 || cost < best_cost || (cost == best_cost && pieces < best_pieces) ||
                            (cost == best_cost && pieces == best_pieces && int(shapes.size()) < best_shapes);
        if (better) {
          best_cost = cost;
          best_pieces = pieces;
          best_shapes = int(shapes.size());
          best = cap;
        }
      }
  if (best_cost < 0) return BASA_ERR_UNSUPPORTED;

  for (int type = 0; type < 8; ++type) {
    plan->type[type].first_tile = uint16_t(plan->n_tiles);
    plan->type[type].n_tiles = 0;
    if (type_count(p, type) == 0) continue;
    TypePlan tp = plan_type(p, type, best);
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

}  // namespace

// Plans depend only on the grid, window and shift; the search above takes up to a
// few milliseconds for large windows, so plans are kept in a small cache.
basa_status build_window_plan(const basa_params &p, WindowPlan *plan) {
  struct Entry {
    int key[9];
    basa_status status;
    std::unique_ptr<WindowPlan> plan;
  };
  static std::mutex mu;
  static std::deque<Entry> cache;
  constexpr size_t kCacheEntries = 32;
  const int key[9] = {p.T, p.H, p.W, p.wt, p.wh, p.ww, p.st, p.sy, p.sx};
  {
    std::lock_guard<std::mutex> lock(mu);
    for (const Entry &e : cache)
      if (std::equal(key, key + 9, e.key)) {
        if (e.status == BASA_OK) *plan = *e.plan;
        return e.status;
      }
  }
  Entry e;
  std::copy(key, key + 9, e.key);
  e.plan.reset(new WindowPlan);
  e.status = search_window_plan(p, e.plan.get());
  if (e.status == BASA_OK) *plan = *e.plan;
  std::lock_guard<std::mutex> lock(mu);
  if (cache.size() >= kCacheEntries) cache.pop_front();
  cache.push_back(std::move(e));
  return cache.back().status;
}

}  // namespace basa
