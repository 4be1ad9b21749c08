// Host-side planning: shape groups, launch classes and workspace layout.
//
// Grouping by (rows, cols, dtype), ids in order of first appearance, members
// ascending: many same-shape matrices (every layer's q_proj, or all MoE
// experts) then run as one batched launch.  Groups whose oriented shape
// (min, max) and dtype agree (e.g. gate_proj R x C and down_proj C x R) share a
// launch class, because the Newton-Schulz chain only sees the oriented m x n
// matrix.
#include <algorithm>
#include <cstdlib>
#include <map>
#include <tuple>

#include "internal.h"

namespace dmuon {

std::vector<Group> plan_groups(const dmuon_shape_t* shapes, int32_t count) {
  std::vector<Group> groups;
  std::map<std::tuple<int64_t, int64_t, int32_t>, size_t> ids;
  for (int32_t i = 0; i < count; ++i) {
    auto key = std::make_tuple(shapes[i].rows, shapes[i].cols, shapes[i].dtype);
    auto it = ids.find(key);
    if (it == ids.end()) {
      it = ids.emplace(key, groups.size()).first;
      groups.push_back(Group{shapes[i].rows, shapes[i].cols, shapes[i].dtype, {}});
    }
    groups[it->second].members.push_back(i);
  }
  return groups;
}

std::vector<LaunchClass> plan_classes(const std::vector<Group>& groups) {
  std::vector<LaunchClass> classes;
  std::map<std::tuple<int64_t, int64_t, int32_t>, size_t> ids;
  for (const Group& g : groups) {
    const int64_t m = std::min(g.rows, g.cols), n = std::max(g.rows, g.cols);
    auto key = std::make_tuple(m, n, g.dtype);
    auto it = ids.find(key);
    if (it == ids.end()) {
      it = ids.emplace(key, classes.size()).first;
      classes.push_back(LaunchClass{m, n, g.dtype, {}});
    }
    auto& mem = classes[it->second].members;
    mem.insert(mem.end(), g.members.begin(), g.members.end());
  }
  return classes;
}

static int64_t round_up(int64_t v, int64_t a) { return (v + a - 1) / a * a; }

// DMUON_GRAM_BLOCKS: "0" per-iteration form only; unset/"1" the last two
// iterations in Gram space; "2" blocks of 2, 3, 3, ... (fewest flops, least
// accurate on ill-conditioned matrices).
static int gram_block_mode() {
  const char* e = std::getenv("DMUON_GRAM_BLOCKS");
  if (e && e[0] == '0') return 0;
  if (e && e[0] == '2') return 2;
  return 1;
}

ChunkLayout chunk_layout(int64_t m, int64_t n, int32_t dtype, bool allow_blocked) {
  ChunkLayout L{};
  if (dtype == DMUON_F32)
    L.path = Path::kF32;
  else if (m <= kSmallM)
    L.path = Path::kSmallBf16;
  else if (m < kF32XBelowM && n < kNearSquare * m)
    L.path = Path::kBf16F32;
  else
    L.path = Path::kTensorBf16;
  // Gram-space blocks cost 3 m^2 n + (4L - 3) m^3 per block of L iterations
  // against L (3 m^2 n + m^3) iteration by iteration: fewer flops once n > m,
  // but Gram space squares the singular values, so bf16 rounding there costs
  // accuracy, the more the closer to square the matrix is and the smaller it
  // is (measured 1.5-1.8e-2 against 1.0-1.2e-2 at n = 1.25 m, m = 256..384, for
  // 3 % fewer flops).  Used where n >= 2 m (8.6 % fewer flops or more), or
  // n >= 1.25 m once m >= 512.
  const bool wide = n >= 2 * m || (m >= 512 && 4 * n >= 5 * m);
  L.blocked = allow_blocked && gram_block_mode() != 0 && L.path == Path::kTensorBf16 && wide;
  L.gslots = L.blocked ? 5 : 2;
  const int64_t xs = (dtype == DMUON_BF16 && L.path != Path::kBf16F32) ? 2 : 4;
  const int64_t gs = L.path == Path::kTensorBf16 ? 2 : 4;
  // 16-byte row pitch: the TMA descriptors need it, vector loads like it
  L.ldn = round_up(n, 8);
  L.ldm = round_up(m, 8);
  L.xbytes = m * L.ldn * xs;
  L.gbytes = m * L.ldm * gs;
  L.tiles_per_mat = ((m + kElemTile - 1) / kElemTile) * ((n + kElemTile - 1) / kElemTile);
  L.per_matrix = 2 * L.xbytes + L.gslots * L.gbytes + L.tiles_per_mat * 4 + 8 + 7 * 256;
  return L;
}

int64_t workspace_cap_bytes() {
  const char* e = std::getenv("DMUON_WS_CAP_MB");
  if (e && *e) {
    long long mb = std::atoll(e);
    if (mb > 0) return (int64_t)mb << 20;
  }
  return (int64_t)8 << 30;
}

// Largest chunk that fits the cap, then evened out over the chunks needed so
// that no chunk is left with a small remainder.
int64_t chunk_size(const ChunkLayout& L, int64_t members, int64_t cap) {
  int64_t c = cap / std::max<int64_t>(1, L.per_matrix);
  c = std::min<int64_t>(c, kMaxTable);
  c = std::max<int64_t>(1, std::min<int64_t>(c, members));
  const int64_t chunks = (members + c - 1) / c;
  return std::max<int64_t>(1, (members + chunks - 1) / chunks);
}

StepPlan make_step_plan(const dmuon_shape_t* shapes, int32_t count) {
  StepPlan P;
  P.classes = plan_classes(plan_groups(shapes, count));
  for (const LaunchClass& c : P.classes) P.layouts.push_back(chunk_layout(c.m, c.n, c.dtype));
  const char* ov = std::getenv("DMUON_OVERLAP");
  const bool allow = !(ov && ov[0] == '0');
  const int64_t cap = workspace_cap_bytes();
  StepPlan serial;
  for (int pass = 0; pass < 2; ++pass) {
    // pass 0: one buffer with the whole cap; pass 1: two buffers of half the cap
    const int64_t cap_b = pass == 0 ? cap : cap / 2;
    P.chunks.clear();
    P.buffer_bytes = 0;
    for (size_t k = 0; k < P.classes.size(); ++k) {
      const int64_t mem = (int64_t)P.classes[k].members.size();
      const int64_t cs = chunk_size(P.layouts[k], mem, cap_b);
      for (int64_t start = 0; start < mem; start += cs) {
        const int b = (int)std::min<int64_t>(cs, mem - start);
        P.chunks.push_back(ChunkRef{k, (size_t)start, b});
        P.buffer_bytes = std::max(P.buffer_bytes, chunk_offsets(P.layouts[k], b).total);
      }
    }
    P.overlap = pass == 1;
    if (pass == 0 && (!allow || P.chunks.size() < 2)) break;
    if (pass == 0) serial = P;
  }
  // a matrix whose workspace alone exceeds half the cap would make the two
  // overlapped buffers exceed the cap: run serially in one buffer instead
  if (P.overlap && 2 * P.buffer_bytes > cap) return serial;
  return P;
}

std::vector<int> chain_blocks(const ChunkLayout& L, int32_t steps) {
  std::vector<int> b;
  const int mode = L.blocked ? gram_block_mode() : 0;
  if (mode == 0 || steps < 2) {
    b.assign(steps, 1);
  } else if (mode == 1) {
    // Gram space squares the singular values, so bf16 rounding there hurts
    // small ones; by the last two iterations they have grown by a^(steps-2).
    b.assign(steps - 2, 1);
    b.push_back(2);
  } else {
    for (int k = 0, first = 1; k < steps; first = 0) {
      const int len = std::min(first ? 2 : 3, steps - k);
      b.push_back(len);
      k += len;
    }
  }
  return b;
}

ChunkOffsets chunk_offsets(const ChunkLayout& L, int64_t b) {
  ChunkOffsets o{};
  int64_t at = 0;
  o.x0 = at; at += round_up(b * L.xbytes, 256);
  o.x1 = at; at += round_up(b * L.xbytes, 256);
  o.g = at; at += round_up(b * L.gbytes, 256);
  o.p = at; at += round_up(b * L.gbytes, 256) * (L.gslots - 1);
  o.partials = at; at += round_up(b * L.tiles_per_mat * 4, 256);
  o.scale = at; at += round_up(b * 4, 256);
  o.counters = at; at += round_up((b + 1) * 4, 256);  // one per matrix, then the tile counter
  o.total = at;
  return o;
}

// Dedicated ownership (every matrix to one rank): longest processing time
// first over the Newton-Schulz flops of one iteration, 3 m^2 n + m^3; equal
// costs in index order, equal loads to the lower rank.
void assign_owners(const dmuon_shape_t* shapes, int32_t count, int32_t world, int32_t* owner_of,
                   double* loads) {
  std::vector<double> cost((size_t)count);
  std::vector<int32_t> order((size_t)count);
  for (int32_t i = 0; i < count; ++i) {
    const double m = (double)std::min(shapes[i].rows, shapes[i].cols);
    const double n = (double)std::max(shapes[i].rows, shapes[i].cols);
    cost[(size_t)i] = 3.0 * m * m * n + m * m * m;
    order[(size_t)i] = i;
  }
  std::stable_sort(order.begin(), order.end(), [&](int32_t a, int32_t b) { return cost[a] > cost[b]; });
  for (int32_t r = 0; r < world; ++r) loads[r] = 0.0;
  for (int32_t i : order) {
    int32_t best = 0;
    for (int32_t r = 1; r < world; ++r)
      if (loads[r] < loads[best]) best = r;
    owner_of[i] = best;
    loads[best] += cost[(size_t)i];
  }
}

}  // namespace dmuon
