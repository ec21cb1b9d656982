// Block attention forward for one launch of ring-step block pairs (sm_100a).
//
// For every block pair of the plan, every query head and every 256-row query
// tile, one CTA computes the partial result of those queries against the
// pair's key/value rows:
//     S = Q K^T * scale, masked by global position (causal: k <= q;
//     document mask: same document), online softmax over the key tiles,
//     O = softmax(S) V normalised within the pair, LSE = ln sum exp(S).
// This is the per-block recurrence of the "序列並行（Sequence Parallelism）"
// concept page (compassingai), 技術原理 §二 "Ring Attention 的塊級線上
// Softmax" (running max m, running denominator l, rescaled O; S = Q K^T /
// sqrt(d_k)), with the mask offsets of the "Context Parallelism" write-up
// (pwwt.cn) §3.3 taken from each block's global positions.
//
// CTA layout (384 threads, one CTA per SM):
//   warp 0      TMA producer: Q tile once, then K/V tiles into a 4-stage ring
//               (the whole warp runs the loop, an elected lane issues copies)
//   warp 1      tcgen05.mma issuer (whole warp converged, an elected lane
//               issues each MMA and commit) and TMEM owner
//   warps 2-3   no work: they complete the control warpgroup, whose four
//               warps give back registers together (setmaxnreg)
//   warps 4-7   softmax and epilogue of query sub-tile 0 (rows 0-127; one
//               row per thread)
//   warps 8-11  softmax and epilogue of query sub-tile 1 (rows 128-255)
// TMEM (512 columns): S0 | S1 (128 fp32 columns each; P is written back over
// S as packed bf16) | O0 | O1 (dh columns each).
// Tensor-pipe order per key tile j: PV0(j), S0(j+1), PV1(j), S1(j+1), so
// each sub-tile's softmax overlaps the other sub-tile's MMAs.
// Rescaling of O is lazy: the running max used for P only moves when the tile
// max exceeds it by more than 2^8, which keeps P <= 256 and the result exact.
#include <cuda.h>
#include <cuda_runtime.h>
#include <math_constants.h>

#include <atomic>
#include <climits>

#include "plan.h"
#include "sm100_ptx.cuh"

namespace cp {

std::atomic<uint64_t>& launch_counter();

__device__ uint32_t g_attn_err = 0;

constexpr int kThreads = 384;
constexpr int kLoNone = -(1 << 30);
// Document tables with fewer entries than this are copied into shared memory
// at CTA start, so the per-CTA and per-row document lookups (binary searches)
// do not wait on global-memory latency.
constexpr int kCuSmem = 1024;
constexpr int kHiNone = (1 << 30);

template <int DH>
struct AttnCfg {
  static constexpr int kBoxes = DH / 64;            // 128-byte column boxes per row
  static constexpr int kBoxBytes = 128 * 128;       // 128 rows x 128 bytes
  static constexpr int kTileBytes = kBoxes * kBoxBytes;
  static constexpr int kStages = DH == 128 ? 4 : 8;
  static constexpr int kQBytes = 2 * kTileBytes;
  static constexpr int kBarBytes = 256;
  static constexpr int kSmemBytes = 1024 + kQBytes + kStages * kTileBytes + kBarBytes + kCuSmem * 4;
  static_assert(kSmemBytes <= kMaxSmemPerCta, "forward kernel exceeds the shared memory of a CTA");
  static constexpr uint32_t kTmemCols = 512;
  // TMEM column of the S/P tile and of the O accumulator of sub-tile t
  __device__ static constexpr uint32_t col_s(int t) { return (uint32_t)t * 128u; }
  __device__ static constexpr uint32_t col_o(int t) { return 256u + (uint32_t)t * DH; }
};

struct KTile {
  int buf_row, pos, valid;
  bool live0, live1;
};

// Enumerates the key tiles of a block pair that are not fully masked for at
// least one of the two query sub-tiles.  Every role of the CTA runs its own
// copy, so all of them see the same sequence without communicating.
struct KIter {
  const cp_pair_desc* pd;
  int seg, t, nk;
  int len, pos, row;  // the current segment, read from the plan once per segment
  int vis_lo[2], vis_hi[2];
  int lo_min;  // first position visible to either live sub-tile
  bool alive[2];

  __device__ void enter(int s) {
    seg = s;
    t = 0;
    if (s < nk) {
      len = pd->k[s].len;
      pos = pd->k[s].pos;
      row = pd->k[s].buf_row;
    }
  }

  __device__ bool next(KTile& out) {
    while (seg < nk) {
      const int off = t * CP_KV_TILE;
      if (off >= len) {
        enter(seg + 1);
        continue;
      }
      const int ka = pos + off;
      // Positions grow along a segment: once past both causal limits, the
      // rest of the segment is masked.
      if ((!alive[0] || ka > vis_hi[0]) && (!alive[1] || ka > vis_hi[1])) {
        enter(seg + 1);
        continue;
      }
      // Tiles that end before both windows start (keys of earlier documents)
      // are jumped over in one step, to the tile holding the first visible
      // position.
      if (ka + CP_KV_TILE - 1 < lo_min) {
        t = (lo_min - pos) / CP_KV_TILE;
        continue;
      }
      ++t;
      const int valid = min(CP_KV_TILE, len - off);
      const int kb = ka + valid - 1;
      const bool l0 = alive[0] && kb >= vis_lo[0] && ka <= vis_hi[0];
      const bool l1 = alive[1] && kb >= vis_lo[1] && ka <= vis_hi[1];
      if (l0 || l1) {
        out.buf_row = row + off;
        out.pos = ka;
        out.valid = valid;
        out.live0 = l0;
        out.live1 = l1;
        return true;
      }
    }
    return false;
  }
};

// Index of the document holding position x (cu = prefix sums, n_docs docs).
// cu is the CTA's shared-memory copy of the table, or the global table when
// it is too long to copy (generic loads serve both).
__device__ __forceinline__ int doc_index(const int32_t* cu, int n_docs, int x) {
  int lo = 0, hi = n_docs - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (cu[mid] <= x) lo = mid; else hi = mid - 1;
  }
  return lo;
}
__device__ __forceinline__ int doc_start(const int32_t* cu, int n_docs, int x) {
  return cu[doc_index(cu, n_docs, x)];
}
// Last position of the document holding x.
__device__ __forceinline__ int doc_last(const int32_t* cu, int n_docs, int x) {
  return cu[doc_index(cu, n_docs, x) + 1] - 1;
}

struct Item {
  const cp_pair_desc* pd;
  int h, hk;
  int q_buf_row0, q_pos0, q_valid, out_row0;
  // per query sub-tile: visible window hull and the fully-visible window
  int vis_lo[2], vis_hi[2], full_lo[2], full_hi[2];
  bool alive[2];
};

// CTA -> (block, head, pair, query tile): head-major inside each block.
__device__ __forceinline__ void decode_item(const cp_attn_plan& plan, const int32_t* cu, Item& it) {
  const int cta = blockIdx.x;
  int b = 0;  // at most CP_MAX_BLOCKS entries, adjacent in the parameter block
  while (b + 1 < plan.n_blocks && plan.blk_cta_begin[b + 1] <= cta) ++b;
  const int local = cta - plan.blk_cta_begin[b];
  const int nqt = plan.blk_qtiles[b];
  it.h = local / nqt;
  int qt = local - it.h * nqt;
  // the last pair of the block whose first tile is <= qt (binary search: a
  // linear scan would touch a new line of the parameter block per pair)
  int p = plan.blk_pair_begin[b];
  int p_hi = plan.blk_pair_begin[b + 1] - 1;
  while (p < p_hi) {
    const int mid = (p + p_hi + 1) >> 1;
    if (plan.pairs[mid].qt_begin <= qt) p = mid; else p_hi = mid - 1;
  }
  const cp_pair_desc* pd = &plan.pairs[p];
  qt -= pd->qt_begin;
  it.pd = pd;
  it.hk = it.h / (plan.hq / plan.hkv);
  if (pd->reverse) qt = pd->qtiles - 1 - qt;
  int s = 0;
  for (; s < pd->nq; ++s) {
    const int nt = (pd->q[s].len + CP_Q_TILE - 1) / CP_Q_TILE;
    if (qt < nt) break;
    qt -= nt;
  }
  const int off = qt * CP_Q_TILE;
  it.q_buf_row0 = pd->q[s].buf_row + off;
  it.q_pos0 = pd->q[s].pos + off;
  it.q_valid = min(CP_Q_TILE, pd->q[s].len - off);
  it.out_row0 = pd->q[s].out_row + off;
  for (int t = 0; t < 2; ++t) {
    const int vt = min(128, it.q_valid - t * 128);
    it.alive[t] = vt > 0;
    const int qa = it.q_pos0 + t * 128;
    const int qb = qa + max(vt, 1) - 1;
    const bool varlen = plan.n_docs > 0;
    it.vis_lo[t] = varlen ? doc_start(cu, plan.n_docs, qa) : kLoNone;
    it.full_lo[t] = varlen ? doc_start(cu, plan.n_docs, qb) : kLoNone;
    // upper key limit of a row: itself (causal) or its document's end
    it.vis_hi[t] = plan.causal ? qb : (varlen ? doc_last(cu, plan.n_docs, qb) : kHiNone);
    it.full_hi[t] = plan.causal ? qa : (varlen ? doc_last(cu, plan.n_docs, qa) : kHiNone);
  }
}

__device__ __forceinline__ void make_iter(const Item& it, KIter& ki) {
  ki.pd = it.pd;
  ki.nk = it.pd->nk;
  for (int t = 0; t < 2; ++t) {
    ki.vis_lo[t] = it.vis_lo[t];
    ki.vis_hi[t] = it.vis_hi[t];
    ki.alive[t] = it.alive[t];
  }
  ki.lo_min = min(it.alive[0] ? it.vis_lo[0] : INT_MAX, it.alive[1] ? it.vis_lo[1] : INT_MAX);
  ki.enter(0);
}

template <int DH>
__global__ void __launch_bounds__(kThreads, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ cp_attn_plan plan) {
  using C = AttnCfg<DH>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sKV = smem + C::kQBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sKV + C::kStages * C::kTileBytes);
  // barrier indices
  const int B_Q = 0, B_FULL = 1, B_EMPTY = 1 + C::kStages, B_S = 1 + 2 * C::kStages, B_P = B_S + 2,
            B_O = B_P + 4, B_DRAIN = B_O + 2, B_COUNT = B_DRAIN + 1;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + B_COUNT);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  int32_t* s_cu = reinterpret_cast<int32_t*>(reinterpret_cast<uint8_t*>(bars) + C::kBarBytes);
  auto bar = [&](int i) { return smem_addr(bars + i); };

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  uint32_t* err = plan.err;
  const int32_t* cu = plan.cu_seqlens;
  if (plan.n_docs > 0 && plan.n_docs < kCuSmem) {
    for (int i = threadIdx.x; i <= plan.n_docs; i += kThreads) s_cu[i] = __ldg(plan.cu_seqlens + i);
    cu = s_cu;  // read after the __syncthreads below
  }

  if (threadIdx.x == 0) {
    mbar_init(bar(B_Q), 1);
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(bar(B_FULL + s), 1);
      mbar_init(bar(B_EMPTY + s), 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(bar(B_S + t), 1);
      mbar_init(bar(B_P + 2 * t + 0), 4);  // one arrive per softmax warp
      mbar_init(bar(B_P + 2 * t + 1), 4);
      mbar_init(bar(B_O + t), 1);
    }
    mbar_init(bar(B_DRAIN), 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  if (warp == 1) {
    tmem_alloc(smem_addr(tmem_holder), C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  Item it;
  decode_item(plan, cu, it);

  // Registers: launched at 168 per thread (384 threads); inside its own
  // branch the control warpgroup (warps 0-3) drops to 80 and the two softmax
  // warpgroups rise to 192: 128 * 80 + 256 * 192 = 59392 <= 384 * 168 = 64512.
  if (warp < 4) {
    regs_dec<80>();

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    // The whole warp runs the loop; one elected lane issues each copy.
    mbar_arrive_expect_tx_elect(bar(B_Q), C::kQBytes);
    for (int t = 0; t < 2; ++t)
      for (int b = 0; b < C::kBoxes; ++b)
        tma_load_2d_elect(smem_addr(sQ + (t * C::kBoxes + b) * C::kBoxBytes), &tm_q, it.h * DH + b * 64,
                          it.q_buf_row0 + t * 128, bar(B_Q));
    KIter ki;
    make_iter(it, ki);
    KTile kt;
    uint32_t c = 0;
    bool ok = true;
    while (ok && ki.next(kt)) {
      for (int w = 0; w < 2 && ok; ++w) {
        const int slot = c % C::kStages;
        const uint32_t ph = (c / C::kStages) & 1u;
        ok = mbar_wait_warp(bar(B_EMPTY + slot), ph ^ 1u, abort_flag, err);
        if (!ok) break;
        mbar_arrive_expect_tx_elect(bar(B_FULL + slot), C::kTileBytes);
        const CUtensorMap* m = w == 0 ? &tm_k : &tm_v;
        for (int b = 0; b < C::kBoxes; ++b)
          tma_load_2d_elect(smem_addr(sKV + slot * C::kTileBytes + b * C::kBoxBytes), m, it.hk * DH + b * 64,
                            kt.buf_row, bar(B_FULL + slot));
        ++c;
      }
    }
    // Drain: make sure every copy issued here has landed before the CTA can
    // exit (only matters after an abort).
    const uint32_t first = c > (uint32_t)C::kStages ? c - C::kStages : 0u;
    for (uint32_t i = first; i < c; ++i)
      mbar_wait_warp(bar(B_FULL + i % C::kStages), (i / C::kStages) & 1u, abort_flag, nullptr, 1000000000ull);
    mbar_wait_warp(bar(B_Q), 0, abort_flag, nullptr, 1000000000ull);
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp runs the loop (operands stay warp-uniform); one elected
    // lane issues each tcgen05.mma / tcgen05.commit.
    constexpr uint32_t idesc_qk = idesc_bf16_f32(128, 128, false);
    constexpr uint32_t idesc_pv = idesc_bf16_f32(128, DH, true);
    uint32_t pc[2] = {0u, 0u};  // P hand-offs consumed per sub-tile
    const uint32_t sq_base = smem_addr(sQ);
    const uint32_t skv_base = smem_addr(sKV);
    auto issue_s = [&](int t, int slot) {
      const uint64_t a0 = sdesc_sw128(sq_base + t * C::kBoxes * C::kBoxBytes, 16, 1024);
      const uint64_t b0 = sdesc_sw128(skv_base + slot * C::kTileBytes, 16, 1024);
#pragma unroll
      for (int kk = 0; kk < DH / 16; ++kk) {
        const uint32_t off = (kk >> 2) * C::kBoxBytes + (kk & 3) * 32;
        tc_mma_ss_elect(tmem + C::col_s(t), sdesc_add(a0, off), sdesc_add(b0, off), idesc_qk, kk > 0 ? 1u : 0u);
      }
    };
    // O_t += P_t V over the 64 keys of half h of the tile
    auto issue_pv_half = [&](int t, int slot, int h, bool acc) {
      const uint64_t b0 = sdesc_sw128(skv_base + slot * C::kTileBytes, C::kBoxBytes, 1024);
#pragma unroll
      for (int k4 = 0; k4 < CP_KV_TILE / 32; ++k4) {
        const int kk = h * (CP_KV_TILE / 32) + k4;
        tc_mma_ts_elect(tmem + C::col_o(t), tmem + C::col_s(t) + kk * 8, sdesc_add(b0, kk * 2048), idesc_pv,
                        (acc || kk > 0) ? 1u : 0u);
      }
    };
    // P_t is released in two halves: the first half's MMAs run while the
    // softmax computes the second half.
    auto issue_pv = [&](int t, int slot, bool acc) -> bool {
      for (int h = 0; h < 2; ++h) {
        if (!mbar_wait_warp(bar(B_P + 2 * t + h), pc[t] & 1u, abort_flag, err)) return false;
        tc_fence_after();
        issue_pv_half(t, slot, h, acc);
      }
      ++pc[t];
      return true;
    };
    auto kslot = [&](int j) { return (2 * j) % C::kStages; };
    auto kph = [&](int j) { return (uint32_t)(((2 * j) / C::kStages) & 1); };
    auto vslot = [&](int j) { return (2 * j + 1) % C::kStages; };
    auto vph = [&](int j) { return (uint32_t)(((2 * j + 1) / C::kStages) & 1); };

    bool ok = mbar_wait_warp(bar(B_Q), 0, abort_flag, err);
    KIter ki;
    make_iter(it, ki);
    KTile cur, nxt;
    bool have = ok && ki.next(cur);
    bool acc[2] = {false, false};
    int j = 0;
    if (have) {
      ok = mbar_wait_warp(bar(B_FULL + kslot(0)), kph(0), abort_flag, err);
      if (ok) {
        tc_fence_after();
        if (cur.live0) { issue_s(0, kslot(0)); tc_commit_elect(bar(B_S + 0)); }
        if (cur.live1) { issue_s(1, kslot(0)); tc_commit_elect(bar(B_S + 1)); }
        tc_commit_elect(bar(B_EMPTY + kslot(0)));
      }
      have = ok;
    }
    while (have) {
      const bool hn = ki.next(nxt);
      if (!(ok = mbar_wait_warp(bar(B_FULL + vslot(j)), vph(j), abort_flag, err))) break;
      if (cur.live0) {
        if (!(ok = issue_pv(0, vslot(j), acc[0]))) break;
        acc[0] = true;
      }
      if (hn) {
        if (!(ok = mbar_wait_warp(bar(B_FULL + kslot(j + 1)), kph(j + 1), abort_flag, err))) break;
        if (nxt.live0) { issue_s(0, kslot(j + 1)); tc_commit_elect(bar(B_S + 0)); }
      }
      if (cur.live1) {
        if (!(ok = issue_pv(1, vslot(j), acc[1]))) break;
        acc[1] = true;
      }
      tc_commit_elect(bar(B_EMPTY + vslot(j)));
      if (hn) {
        if (nxt.live1) { issue_s(1, kslot(j + 1)); tc_commit_elect(bar(B_S + 1)); }
        tc_commit_elect(bar(B_EMPTY + kslot(j + 1)));
      }
      cur = nxt;
      have = hn;
      ++j;
    }
    tc_commit_elect(bar(B_O + 0));
    tc_commit_elect(bar(B_O + 1));
    // Wait for every MMA issued here before TMEM and shared memory go away.
    tc_commit_elect(bar(B_DRAIN));
    mbar_wait_warp(bar(B_DRAIN), 0, abort_flag, nullptr, 1000000000ull);
  }
  } else {
    regs_inc<192>();
    // ------------------------------------------------------------ softmax
    const int t = (warp - 4) >> 2;
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    const uint32_t tS = tmem + lane_base + C::col_s(t);
    const uint32_t tO = tmem + lane_base + C::col_o(t);
    const int grow = t * 128 + row;
    const bool rvalid = grow < it.q_valid;
    const int qpos = it.q_pos0 + grow;
    const bool varlen = plan.n_docs > 0;
    const int row_lo = rvalid ? (varlen ? doc_start(cu, plan.n_docs, qpos) : kLoNone) : kHiNone;
    const int row_hi =
        rvalid ? (plan.causal ? qpos : (varlen ? doc_last(cu, plan.n_docs, qpos) : kHiNone)) : kLoNone;
    const float scale_log2 = plan.scale_log2;
    const int full_lo = t == 0 ? it.full_lo[0] : it.full_lo[1];
    const int full_hi = t == 0 ? it.full_hi[0] : it.full_hi[1];

    // Running state of this row (log2 domain, scores already scaled):
    //   m_used  reference the accumulated O and l are relative to
    //   l       sum of 2^(x - m_used) over the keys seen so far
    //   pend    factor O still has to be multiplied by (lazy rescale)
    float m_used = -CUDART_INF_F;
    float l = 0.f;
    float pend = 1.f;
    uint32_t n_tiles = 0;
    bool ok = true;
    KIter ki;
    make_iter(it, ki);
    KTile kt;
    const uint64_t c2 = f2_pack(scale_log2, scale_log2);
    // O <- O * f for this warp's 32 rows (warp-collective)
    auto rescale_o = [&](float f) {
#pragma unroll 1
      for (int ch = 0; ch < DH / 32; ++ch) {
        uint32_t o[32];
        tmem_ld32(tO + ch * 32, o);
        tc_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * f);
        tmem_st32(tO + ch * 32, o);
      }
    };
    while (ki.next(kt)) {
      if (!(t == 0 ? kt.live0 : kt.live1)) continue;
      ok = mbar_wait(bar(B_S + t), n_tiles & 1u, abort_flag, err);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      uint32_t s[128];
      tmem_ld32(tS + 0, *reinterpret_cast<uint32_t(*)[32]>(&s[0]));
      tmem_ld32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(&s[32]));
      tmem_ld32(tS + 64, *reinterpret_cast<uint32_t(*)[32]>(&s[64]));
      tmem_ld32(tS + 96, *reinterpret_cast<uint32_t(*)[32]>(&s[96]));
      tc_wait_ld();
      const bool full = kt.valid == CP_KV_TILE && kt.pos >= full_lo && kt.pos + CP_KV_TILE - 1 <= full_hi;
      const int clo = row_lo - kt.pos;
      const int chi = min(row_hi - kt.pos, kt.valid - 1);
      // -inf outside this row's visible keys, for columns [c0, c1)
      auto mask_cols = [&](int c0, int c1) {
#pragma unroll
        for (int c = 0; c < 128; ++c)
          if (c >= c0 && c < c1 && (c < clo || c > chi)) s[c] = __float_as_uint(-CUDART_INF_F);
      };
      if (!full) mask_cols(0, 128);
      // S(j) is complete, hence so is PV(j-1): apply a pending rescale of O
      // before P(j) is released.
      if (__any_sync(0xffffffffu, pend != 1.f)) {
        rescale_o(pend);
        pend = 1.f;
      }
      // Reference for this tile: the running one.  A row that has seen no
      // admitted key yet takes the exact maximum of this tile first.
      float ref = m_used;
      if (__any_sync(0xffffffffu, ref == -CUDART_INF_F)) {
        float a = -CUDART_INF_F, b = -CUDART_INF_F;
#pragma unroll
        for (int c = 0; c < 128; c += 4) {
          a = max3f(a, __uint_as_float(s[c]), __uint_as_float(s[c + 1]));
          b = max3f(b, __uint_as_float(s[c + 2]), __uint_as_float(s[c + 3]));
        }
        if (ref == -CUDART_INF_F) ref = fmaxf(a, b) * scale_log2;
      }
      uint32_t pk[32];
      uint64_t lsum = f2_pack(0.f, 0.f);
      float ma = -CUDART_INF_F;
      // P = 2^(x - ref) for columns [64h, 64h + 64), packed to bf16 pairs;
      // with fold_max the maximum of those columns is taken on the way, so
      // each score register dies as soon as its exponential is formed.
      auto exp_half = [&](int h, bool fold_max) {
        const float nr = ref == -CUDART_INF_F ? 0.f : -ref;
        const uint64_t nr2 = f2_pack(nr, nr);
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          const float s0 = __uint_as_float(s[h * 64 + 2 * c]), s1 = __uint_as_float(s[h * 64 + 2 * c + 1]);
          if (fold_max) ma = max3f(ma, s0, s1);
          const uint64_t x = f2_fma(f2_pack(s0, s1), c2, nr2);
          float x0, x1;
          f2_unpack(x, x0, x1);
          const float p0 = ex2_approx(x0);
          const float p1 = ex2_approx(x1);
          lsum = f2_add(lsum, f2_pack(p0, p1));
          pk[c] = pack_bf16x2(p0, p1);
        }
      };
      exp_half(0, true);
      // Tile maximum, checked before the first half of P is released.
      float mb = -CUDART_INF_F, mc = -CUDART_INF_F;
#pragma unroll
      for (int c = 64; c < 128; c += 4) {
        mb = max3f(mb, __uint_as_float(s[c]), __uint_as_float(s[c + 1]));
        mc = max3f(mc, __uint_as_float(s[c + 2]), __uint_as_float(s[c + 3]));
      }
      const float mt = fmaxf(ma, fmaxf(mb, mc)) * scale_log2;
      // Guard: P must stay far from the bf16 / fp32 range limits.  A row whose
      // tile maximum exceeds the reference by more than 2^64 re-bases now
      // (rescaling what O and l hold) and recomputes its P; the first half of
      // the scores is read again from TMEM, where P has not yet replaced it.
      const bool over = mt > ref + 64.f;
      if (__any_sync(0xffffffffu, over)) {
        float f = 1.f;
        if (over) {
          f = ex2_approx(ref - mt);
          ref = mt;
          l *= f;
        }
        if (n_tiles > 0) rescale_o(f);
        tmem_ld32(tS + 0, *reinterpret_cast<uint32_t(*)[32]>(&s[0]));
        tmem_ld32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(&s[32]));
        tc_wait_ld();
        if (!full) mask_cols(0, 64);
        lsum = f2_pack(0.f, 0.f);
        exp_half(0, false);
      }
      tmem_st32(tS + 0, pk);
      tc_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(B_P + 2 * t + 0));
      exp_half(1, false);
      tmem_st32(tS + 32, pk);
      tc_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(B_P + 2 * t + 1));
      float l0, l1;
      f2_unpack(lsum, l0, l1);
      l += l0 + l1;
      m_used = ref;
      // Lazy re-basing: move the reference only when the tile maximum is
      // more than 2^8 above it; O follows at the start of the next tile.
      if (mt > m_used + 8.f) {
        const float f = ex2_approx(m_used - mt);
        pend = f;
        l *= f;
        m_used = mt;
      }
      ++n_tiles;
    }
    if (ok) {
      ok = mbar_wait(bar(B_O + t), 0, abort_flag, err);
      ok = __all_sync(0xffffffffu, ok);
    }
    if (ok) {
      tc_fence_after();
      // Epilogue.  O leaves TMEM one row per thread; stored from there, one
      // warp instruction would touch 32 rows 16 KB apart.  Instead each
      // 32-column slab goes through a 4 KB shared-memory tile per warp (in the
      // K/V stage buffers, idle once every MMA has completed), 16-byte chunks
      // XOR-swizzled by row so that both the row-wise writes and the
      // column-wise reads take the minimum of four wavefronts, and leaves as
      // four whole 128-byte row segments per store instruction.
      const cp_pair_desc* pd = it.pd;
      const int orow = it.out_row0 + grow;
      const float inv_l = l > 0.f ? pend / l : 0.f;
      float4* stile = reinterpret_cast<float4*>(sKV + (warp - 4) * 4096);
      const int wrow0 = t * 128 + quarter * 32;  // CTA row of lane 0 of this warp
      const int cc = lane & 7;
      fence_proxy_async_smem();
#pragma unroll 1
      for (int ch = 0; ch < DH / 32; ++ch) {
        uint32_t o[32];
        if (n_tiles > 0) {
          tmem_ld32(tO + ch * 32, o);
          tc_wait_ld();
        }
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
          if (n_tiles > 0 && l > 0.f) {
            v.x = __uint_as_float(o[4 * c + 0]) * inv_l;
            v.y = __uint_as_float(o[4 * c + 1]) * inv_l;
            v.z = __uint_as_float(o[4 * c + 2]) * inv_l;
            v.w = __uint_as_float(o[4 * c + 3]) * inv_l;
          }
          stile[lane * 8 + (c ^ (lane & 7))] = v;
        }
        __syncwarp();
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int rr = 4 * i + (lane >> 3);  // lanes 8k..8k+7 write one row's 128 bytes
          const float4 v = stile[rr * 8 + (cc ^ (rr & 7))];
          if (wrow0 + rr < it.q_valid) {
            float* dst = pd->o + ((size_t)(it.out_row0 + wrow0 + rr) * plan.hq + it.h) * DH + ch * 32;
            reinterpret_cast<float4*>(dst)[cc] = v;
          }
        }
        __syncwarp();
      }
      if (rvalid) {
        const float lse = l > 0.f ? (m_used + __log2f(l)) * 0.69314718055994531f : -CUDART_INF_F;
        pd->lse[(size_t)it.h * pd->lse_ld + orow] = lse;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

// ------------------------------------------------------------------ host side
template <int DH>
static cudaError_t launch_attn_dh(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                                  const cp_attn_plan& plan, cudaStream_t stream) {
  using C = AttnCfg<DH>;
  static bool configured = false;  // per process; attribute is per function
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(attn_fwd_kernel<DH>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         C::kSmemBytes);
    if (e != cudaSuccess) return e;
    configured = true;
  }
  if (plan.total_ctas <= 0) return cudaSuccess;
  attn_fwd_kernel<DH><<<plan.total_ctas, kThreads, C::kSmemBytes, stream>>>(tq, tk, tv, plan);
  launch_counter()++;
  return cudaGetLastError();
}

cudaError_t launch_attn(int dh, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                        const cp_attn_plan& plan, cudaStream_t stream) {
  if (dh == 128) return launch_attn_dh<128>(tq, tk, tv, plan, stream);
  return launch_attn_dh<64>(tq, tk, tv, plan, stream);
}

cudaError_t attn_err_word(uint32_t** dev_ptr) {
  return cudaGetSymbolAddress(reinterpret_cast<void**>(dev_ptr), g_attn_err);
}

}  // namespace cp
