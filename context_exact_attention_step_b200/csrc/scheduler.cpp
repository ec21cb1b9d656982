// Host ring-step scheduler (plain C++, no CUDA).
//
// Ring Attention ("序列並行（Sequence Parallelism）" concept page (compassingai),
// "Ring Attention 的不同思路" steps 1-4; "Context Parallelism" write-up
// (pwwt.cn) §2.2): rank r keeps its query shard and at step t holds the
// key/value shard j = (r - t) mod P; each step yields a partial result that is
// folded into the rank's output.  With P virtual ranks on one GPU the steps
// are independent, so the scheduler enumerates every (r, t), decides which
// block pairs the mask leaves non-empty (the causal mask must follow each
// received block's global positions: pwwt.cn §3.3), trims the query rows of a
// pair that see none of its keys, orders the pairs heaviest first for the
// launch, and lays out the partials and the merge tasks.
#include "scheduler.h"

#include <algorithm>
#include <climits>

namespace cp {

int Docs::start_of(int pos) const {
  // largest i < n with cu[i] <= pos
  int lo = 0, hi = n - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) / 2;
    if (cu[mid] <= pos) lo = mid; else hi = mid - 1;
  }
  return cu[lo];
}

int Docs::end_of(int pos) const {
  int lo = 0, hi = n - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) / 2;
    if (cu[mid] <= pos) lo = mid; else hi = mid - 1;
  }
  return cu[lo + 1];
}

std::vector<Seg> shard_segments(int S, int P, Layout layout, int r) {
  std::vector<Seg> s;
  if (layout == Layout::Contiguous) {
    const int n = S / P;
    s.push_back({r * n, r * n, n, 0});
  } else if (layout == Layout::Striped) {
    const int n = S / P;
    s.push_back({r * n, 0, n, 0});
  } else {
    const int c = S / (2 * P);
    const int base = r * 2 * c;
    s.push_back({base, r * c, c, 0});
    s.push_back({base + c, (2 * P - 1 - r) * c, c, c});
  }
  return s;
}

// admitted pairs between positions [qa, qb] and [ka, kb], one document
static int64_t count_range(int64_t qa, int64_t qb, int64_t ka, int64_t kb, bool causal) {
  if (qa > qb || ka > kb) return 0;
  if (!causal) return (qb - qa + 1) * (kb - ka + 1);
  int64_t total = 0;
  const int64_t lo = std::max(qa, ka), hi = std::min(qb, kb);
  if (lo <= hi) total += (hi - lo + 1) * ((lo - ka + 1) + (hi - ka + 1)) / 2;
  const int64_t lo2 = std::max(qa, kb + 1);
  if (lo2 <= qb) total += (qb - lo2 + 1) * (kb - ka + 1);
  return total;
}

int64_t count_admitted(int qa, int ql, int ka, int kl, bool causal, const Docs& docs) {
  if (ql <= 0 || kl <= 0) return 0;
  const int qb = qa + ql - 1, kb = ka + kl - 1;
  if (!docs.any()) return count_range(qa, qb, ka, kb, causal);
  int64_t total = 0;
  int pos = std::min(qa, ka);
  const int last = std::max(qb, kb);
  while (pos <= last) {
    const int s = docs.start_of(pos), e = docs.end_of(pos);  // [s, e)
    total += count_range(std::max(qa, s), std::min(qb, e - 1), std::max(ka, s), std::min(kb, e - 1), causal);
    pos = e;
  }
  return total;
}

// Query rows (positions) of [qa, qb] with at least one admitted key in
// [ka, kb]; returns an empty range as lo > hi.
static void live_rows(int qa, int qb, int ka, int kb, bool causal, const Docs& docs, int& lo, int& hi) {
  lo = qa;
  hi = qb;
  if (causal) lo = std::max(lo, ka);
  if (docs.any()) {
    hi = std::min(hi, docs.end_of(kb) - 1);
    if (!causal) lo = std::max(lo, docs.start_of(ka));
  }
}

int64_t pair_tile_cost(const std::vector<Seg>& q, const std::vector<Seg>& k, bool causal, const Docs& docs) {
  int64_t cost = 0;
  for (const Seg& qs : q) {
    for (int off = 0; off < qs.len; off += CP_Q_TILE) {
      const int valid = std::min(CP_Q_TILE, qs.len - off);
      for (int t = 0; t < 2; ++t) {
        const int vt = std::min(128, valid - t * 128);
        if (vt <= 0) continue;
        const int qa = qs.pos + off + t * 128, qb = qa + vt - 1;
        const int vis_lo = docs.any() ? docs.start_of(qa) : INT_MIN;
        const int vis_hi = causal ? qb : (docs.any() ? docs.end_of(qb) - 1 : INT_MAX);
        for (const Seg& ks : k)
          for (int ko = 0; ko < ks.len; ko += CP_KV_TILE) {
            const int ka = ks.pos + ko, kb = ka + std::min(CP_KV_TILE, ks.len - ko) - 1;
            if (kb >= vis_lo && ka <= vis_hi) ++cost;
          }
      }
    }
  }
  return cost;
}

RingPlan build_ring_plan(int S, int P, Layout layout, bool causal, const Docs& docs, int hq, int dh) {
  RingPlan plan;
  plan.S = S;
  plan.P = P;
  plan.n = S / P;
  plan.layout = layout;
  plan.causal = causal;
  plan.src.assign((size_t)P * P, 0);
  plan.launched.assign((size_t)P * P, 0);
  plan.q_rows.assign((size_t)P * P, 0);
  plan.live_all.assign((size_t)P * P, 0);

  for (int r = 0; r < P; ++r) {
    const std::vector<Seg> qsegs = shard_segments(S, P, layout, r);
    for (int t = 0; t < P; ++t) {
      const int j = ((r - t) % P + P) % P;
      const size_t idx = (size_t)r * P + t;
      plan.src[idx] = j;
      PairPlan pp;
      pp.r = r;
      pp.t = t;
      pp.j = j;
      pp.k = shard_segments(S, P, layout, j);
      if (layout == Layout::Striped && j > r) {
        // Striped: rank r holds positions r + P*a, shard j positions j + P*b.
        // k <= q  <=>  b <= a for j <= r and b <= a - 1 for j > r, i.e. a
        // local causal mask whose key positions are shifted by one for j > r.
        pp.k[0].pos = 1;
      }
      int out_row = 0;
      for (const Seg& qs : qsegs) {
        int lo = INT_MAX, hi = INT_MIN;
        for (const Seg& ks : pp.k) {
          int a, b;
          live_rows(qs.pos, qs.pos + qs.len - 1, ks.pos, ks.pos + ks.len - 1, causal, docs, a, b);
          if (a <= b) {
            lo = std::min(lo, a);
            hi = std::max(hi, b);
          }
        }
        if (lo > hi) continue;
        Seg s;
        s.buf_row = qs.buf_row + (lo - qs.pos);
        s.pos = lo;
        s.len = hi - lo + 1;
        s.out_row = out_row;
        out_row += s.len;
        pp.q.push_back(s);
      }
      for (const Seg& qs : pp.q)
        for (const Seg& ks : pp.k) pp.live += count_admitted(qs.pos, qs.len, ks.pos, ks.len, causal, docs);
      plan.live_all[idx] = pp.live;
      if (pp.live == 0) continue;
      pp.rows = out_row;
      for (const Seg& qs : pp.q) pp.qtiles += (qs.len + CP_Q_TILE - 1) / CP_Q_TILE;
      pp.cost = pair_tile_cost(pp.q, pp.k, causal, docs);
      plan.launched[idx] = 1;
      plan.q_rows[idx] = pp.rows;
      plan.pairs.push_back(std::move(pp));
    }
  }

  // heaviest CTAs first: sort by mean tile cost per query tile
  std::stable_sort(plan.pairs.begin(), plan.pairs.end(), [](const PairPlan& a, const PairPlan& b) {
    return a.cost * b.qtiles > b.cost * a.qtiles;
  });

  // workspace layout of the partials
  size_t off = 0;
  auto align = [](size_t x) { return (x + 255) & ~size_t(255); };
  for (PairPlan& pp : plan.pairs) {
    pp.o_off = off;
    off = align(off + (size_t)pp.rows * hq * dh * sizeof(float));
    pp.lse_off = off;
    off = align(off + (size_t)hq * pp.rows * sizeof(float));
  }
  plan.partial_bytes = off;

  // merge tasks: per rank, split the shard rows where the covering set of
  // partials changes
  for (int r = 0; r < P; ++r) {
    const int base = r * plan.n;
    std::vector<int> cuts = {0, plan.n};
    for (const PairPlan& pp : plan.pairs)
      if (pp.r == r)
        for (const Seg& s : pp.q) {
          cuts.push_back(s.buf_row - base);
          cuts.push_back(s.buf_row - base + s.len);
        }
    std::sort(cuts.begin(), cuts.end());
    cuts.erase(std::unique(cuts.begin(), cuts.end()), cuts.end());
    for (size_t c = 0; c + 1 < cuts.size(); ++c) {
      const int a = cuts[c], b = cuts[c + 1];
      if (a >= b) continue;
      MergeTaskPlan task;
      task.rank = r;
      task.row0 = base + a;
      task.rows = b - a;
      for (size_t pi = 0; pi < plan.pairs.size(); ++pi) {
        const PairPlan& pp = plan.pairs[pi];
        if (pp.r != r) continue;
        for (const Seg& s : pp.q) {
          const int sa = s.buf_row - base, sb = sa + s.len;
          if (sa <= a && b <= sb) task.inputs.push_back({(int)pi, s.out_row + (a - sa)});
        }
      }
      plan.tasks.push_back(std::move(task));
    }
  }
  return plan;
}

}  // namespace cp
