// Host ring-step scheduler: which block pairs a ring of P virtual ranks
// computes, which of their rows are live, how many (q, k) pairs each admits,
// in what order their CTAs launch, and how the partials fold back per rank.
#pragma once
#include <stdint.h>

#include <vector>

#include "plan.h"

namespace cp {

enum class Layout { Contiguous = 0, Zigzag = 1, Striped = 2 };

// Document table on the host (prefix sums; n docs, n + 1 entries), or none.
struct Docs {
  const int32_t* cu = nullptr;
  int n = 0;
  bool any() const { return cu != nullptr && n > 0; }
  int start_of(int pos) const;  // first position of pos's document
  int end_of(int pos) const;    // one past the last position of pos's document
};

// Rows of one side of a block pair.  buf_row is absolute in the sharded
// buffer; out_row is the row in the pair's partial output.
struct Seg {
  int buf_row, pos, len, out_row;
};

struct PairPlan {
  int r = 0, t = 0, j = 0;
  std::vector<Seg> q, k;
  int rows = 0;           // computed query rows (sum of q lens)
  int64_t live = 0;       // admitted (q, k) pairs
  int64_t cost = 0;       // live 128x128 tiles summed over the pair's query tiles
  int qtiles = 0;
  size_t o_off = 0, lse_off = 0;  // workspace offsets of the partial
};

struct MergeTaskPlan {
  int rank = 0;
  int row0 = 0;           // first row of the task, absolute in the sharded output
  int rows = 0;
  std::vector<std::pair<int, int>> inputs;  // (pair index, first row in that partial)
};

struct RingPlan {
  int S = 0, P = 0, n = 0;
  Layout layout = Layout::Contiguous;
  bool causal = true;
  std::vector<PairPlan> pairs;        // live pairs, in launch order
  std::vector<MergeTaskPlan> tasks;
  size_t partial_bytes = 0;           // workspace bytes for the partials
  std::vector<int32_t> src, launched, q_rows;
  std::vector<int64_t> live_all;      // per (r, t)
};

// Segments of rank r's shard, buf_row absolute (rank-major storage).  For the
// striped layout the positions are per-pair virtual positions (see
// build_ring_plan), and this returns the shard's rows at position 0.
std::vector<Seg> shard_segments(int S, int P, Layout layout, int r);

// Admitted (q, k) pairs between position ranges [qa, qa+ql) and [ka, ka+kl).
int64_t count_admitted(int qa, int ql, int ka, int kl, bool causal, const Docs& docs);

// Build the full ring plan; hq and dh size the partial buffers.
RingPlan build_ring_plan(int S, int P, Layout layout, bool causal, const Docs& docs, int hq, int dh);

// Count live 128-row key tiles for every 256-row query tile, mirroring the
// kernel's tile classification (for launch ordering).
int64_t pair_tile_cost(const std::vector<Seg>& q, const std::vector<Seg>& k, bool causal, const Docs& docs);

}  // namespace cp
