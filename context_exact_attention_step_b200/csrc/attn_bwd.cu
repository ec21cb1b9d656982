// Backward of the ring-step block attention (sm_100a).
//
// The pages define the forward only; the backward is the gradient of that
// exact attention for an upstream dO.  Ring form: the forward's merged O and
// LSE of every rank are kept, and at ring step t rank r, holding key/value
// shard j = (r - t) mod P, contributes with
//     P_rj  = exp(scale Q_r K_j^T - LSE_r)      (the merged LSE, so P_rj is
//                                               the true slice of softmax)
//     D_r   = rowsum(dO_r * O_r)
//     dS_rj = P_rj * (dO_r V_j^T - D_r)
//     dQ_r += scale dS_rj K_j,  dK_j += scale dS_rj^T Q_r,  dV_j += P_rj^T dO_r.
// Differentiating the LSE merge ("序列並行（Sequence Parallelism）" concept
// page (compassingai), 技術原理 §二, the block recurrence) together with each
// pair's own normalisation gives exactly this, so the merge needs no backward
// kernel of its own.  Masks follow each block's global positions as in the
// forward ("Context Parallelism" write-up (pwwt.cn) §3.3).
//
// With the P ranks on one GPU the contributions are summed on chip instead
// of travelling around the ring:
//   * bwd_prep_kernel: D and LSE * log2(e) for every (row, head)   (HBM-bound)
//   * attn_bwd_dq_kernel: one CTA per (128-row query tile of rank r, query
//     head) walks the key/value tiles of shards (r - t) mod P, t = 0..P-1,
//     and accumulates dQ in tensor memory;
//   * attn_bwd_dkdv_kernel: one CTA per (128-row key/value tile of shard j,
//     KV head) walks the query tiles of ranks (j + t) mod P and every query
//     head of the group, and accumulates dK and dV in tensor memory.
// No atomics: every output row is written once by one CTA.
//
// Across GPUs the same kernels run one block pair per launch (the plan's ring
// steps narrowed to the one partner, and `accumulate` set so each launch adds
// to dQ and to the dK/dV that travel with their shard).
//
// CTA layout of both tensor-core kernels (384 threads, one CTA per SM):
//   warp 0      TMA producer
//   warp 1      tcgen05.mma issuer (whole warp converged, an elected lane
//               issues each MMA and commit) and TMEM owner
//   warps 2-3   no work: they complete the control warpgroup, whose four
//               warps give back registers together (setmaxnreg)
//   warps 4-7   element-wise stage, columns 0-63 of every tile, one own row
//               per thread (TMEM lane)
//   warps 8-11  element-wise stage, columns 64-127 of the same rows
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math_constants.h>

#include <atomic>

#include "plan.h"
#include "sm100_ptx.cuh"

namespace cp {

std::atomic<uint64_t>& launch_counter();

namespace {

constexpr int kBwdThreads = 384;
constexpr int kNoLo = -(1 << 30);
constexpr int kNoHi = (1 << 30);
constexpr float kLog2e = 1.4426950408889634f;
// Every wait of these kernels is on the CTA's own pipeline and lasts
// microseconds; half a second means the CTA is stuck, so it gives up.
constexpr uint64_t kWaitNs = 500000000ull;

__device__ __forceinline__ int bdoc_index(const int32_t* __restrict__ cu, int n_docs, int x) {
  int lo = 0, hi = n_docs - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (__ldg(cu + mid) <= x) lo = mid; else hi = mid - 1;
  }
  return lo;
}
__device__ __forceinline__ int bdoc_start(const int32_t* __restrict__ cu, int n_docs, int x) {
  return __ldg(cu + bdoc_index(cu, n_docs, x));
}
__device__ __forceinline__ int bdoc_last(const int32_t* __restrict__ cu, int n_docs, int x) {
  return __ldg(cu + bdoc_index(cu, n_docs, x) + 1) - 1;
}

template <int DH>
struct BwdTile {
  static constexpr int kBoxes = DH / 64;       // 128-byte column boxes per row
  static constexpr int kBoxBytes = 128 * 128;  // 128 rows x 128 bytes
  static constexpr int kTileBytes = kBoxes * kBoxBytes;
};

struct Own {
  int rank, grp, grp_row0, buf_row0, pos0, valid;
};

__device__ __forceinline__ void decode_own(const cp_bwd_plan& pl, uint32_t item, Own& o) {
  o.rank = (int)(item >> 26);
  const int sg = (int)((item >> 25) & 1u);
  o.grp = (int)((item >> 19) & 63u);
  const int tile = (int)(item & 0x7FFFFu);
  const cp_seg& s = pl.seg[o.rank][sg];
  o.grp_row0 = o.grp * pl.group_rows;
  o.buf_row0 = o.grp_row0 + s.buf_row + tile * 128;
  o.pos0 = s.pos + tile * 128;
  o.valid = min(128, s.len - tile * 128);
}

// One warp stores 32 rows (row = lane) x 32 fp32 columns, o[] * f (zeros when
// `zero`): the values pass through the warp's 4 KB shared tile, 16-byte chunks
// XOR-swizzled by row so that the row-wise writes and the column-wise reads
// both take the minimum of four wavefronts, and leave as four whole 128-byte
// row segments per store instruction (stored straight from the TMEM layout,
// one warp instruction would touch 32 rows far apart).  Row r goes to
// dst_row0 + r * pitch; rows >= n_rows are skipped; with accumulate the
// destination is read and added.
__device__ __forceinline__ void warp_store_32x32(float4* stile, const uint32_t (&o)[32], float f, bool zero,
                                                 float* dst_row0, size_t pitch, int n_rows, bool accumulate) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (!zero) {
      v.x = __uint_as_float(o[4 * c + 0]) * f;
      v.y = __uint_as_float(o[4 * c + 1]) * f;
      v.z = __uint_as_float(o[4 * c + 2]) * f;
      v.w = __uint_as_float(o[4 * c + 3]) * f;
    }
    stile[lane * 8 + (c ^ (lane & 7))] = v;
  }
  __syncwarp();
  const int cc = lane & 7;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int rr = 4 * i + (lane >> 3);  // lanes 8k..8k+7 take one row's 128 bytes
    float4 v = stile[rr * 8 + (cc ^ (rr & 7))];
    if (rr < n_rows) {
      float4* d = reinterpret_cast<float4*>(dst_row0 + (size_t)rr * pitch) + cc;
      if (accumulate) {
        const float4 a = *d;
        v.x += a.x;
        v.y += a.y;
        v.z += a.z;
        v.w += a.w;
      }
      *d = v;
    }
  }
  __syncwarp();
}

// ------------------------------------------------------------------ dQ side
struct KvTile {
  int buf_row, pos, valid;
  bool full;
};

// Key/value tiles seen by one query tile of rank r, in ring-step order.
// Every role of the CTA runs its own copy and sees the same sequence.
struct DqIter {
  const cp_bwd_plan* pl;
  int r, t, sg, tl, row0;
  int P, t_end;
  bool striped;
  // the current ring step's shard j = (r - t) mod P, its segment count and
  // the current segment, read from the plan once per step / segment
  int j, n_seg, s_pos, s_len, s_row, shift;
  int vis_lo, vis_hi, full_lo, full_hi;

  __device__ void enter_seg() {
    if (sg < n_seg) {
      s_pos = pl->seg[j][sg].pos;
      s_len = pl->seg[j][sg].len;
      s_row = pl->seg[j][sg].buf_row;
    }
  }
  __device__ void enter_step() {
    j = r - t;
    if (j < 0) j += P;
    n_seg = pl->nseg[j];
    shift = (striped && j > r) ? 1 : 0;
    sg = tl = 0;
    enter_seg();
  }

  __device__ void init(const cp_bwd_plan& p, const Own& own) {
    pl = &p;
    r = own.rank;
    row0 = own.grp_row0;
    P = p.P;
    t_end = p.t_end;
    striped = p.striped != 0;
    t = p.t_begin;
    if (t < t_end) enter_step();
    const int qa = own.pos0, qb = own.pos0 + own.valid - 1;
    const bool docs = p.n_docs > 0;
    vis_lo = docs ? bdoc_start(p.cu_seqlens, p.n_docs, qa) : kNoLo;
    full_lo = docs ? bdoc_start(p.cu_seqlens, p.n_docs, qb) : kNoLo;
    vis_hi = p.causal ? qb : (docs ? bdoc_last(p.cu_seqlens, p.n_docs, qb) : kNoHi);
    full_hi = p.causal ? qa : (docs ? bdoc_last(p.cu_seqlens, p.n_docs, qa) : kNoHi);
  }

  __device__ bool next(KvTile& out) {
    while (t < t_end) {
      if (sg >= n_seg) {
        if (++t < t_end) enter_step();
        continue;
      }
      const int off = tl * 128;
      if (off >= s_len) {
        ++sg;
        tl = 0;
        enter_seg();
        continue;
      }
      const int ka = s_pos + shift + off;
      if (ka > vis_hi) {  // positions grow along a segment
        ++sg;
        tl = 0;
        enter_seg();
        continue;
      }
      if (ka + 127 < vis_lo) {  // keys of earlier documents: jump to the first visible tile
        tl = (vis_lo - s_pos - shift) / 128;
        continue;
      }
      ++tl;
      const int valid = min(128, s_len - off);
      const int kb = ka + valid - 1;
      if (kb >= vis_lo && ka <= vis_hi) {
        out.buf_row = row0 + s_row + off;
        out.pos = ka;
        out.valid = valid;
        out.full = valid == 128 && ka >= full_lo && kb <= full_hi;
        return true;
      }
    }
    return false;
  }
};

template <int DH>
struct DqCfg {
  using T = BwdTile<DH>;
  static constexpr int kStages = DH == 128 ? 4 : 8;
  static constexpr int kSmemBytes = 1024 + 2 * T::kTileBytes + kStages * T::kTileBytes + 256;
  static_assert(kSmemBytes <= kMaxSmemPerCta, "dQ kernel exceeds the shared memory of a CTA");
  // TMEM: S | dP (dS is written over it) | dQ | Q and dO as the A operands of
  // S = Q K^T and dP = dO V^T, copied in once so that these MMAs read only
  // K and V from shared memory
  static constexpr uint32_t kColS = 0, kColD = 128, kColQ = 256, kColQA = 256 + DH, kColDOA = kColQA + DH / 2;
};

template <int DH>
__global__ void __launch_bounds__(kBwdThreads, 1)
    attn_bwd_dq_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
                       const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                       const __grid_constant__ cp_bwd_plan plan) {
  using C = DqCfg<DH>;
  using T = BwdTile<DH>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sDO = smem + T::kTileBytes;
  uint8_t* sKV = smem + 2 * T::kTileBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sKV + C::kStages * T::kTileBytes);
  const int B_QD = 0, B_FULL = 1, B_EMPTY = 1 + C::kStages, B_S = 1 + 2 * C::kStages, B_DP = B_S + 1,
            B_SC = B_DP + 1, B_DS = B_SC + 1, B_ACC = B_DS + 1, B_A = B_ACC + 1, B_DRAIN = B_A + 1,
            B_COUNT = B_DRAIN + 1;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + B_COUNT);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  auto bar = [&](int i) { return smem_addr(bars + i); };
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  uint32_t* err = plan.err;

  if (threadIdx.x == 0) {
    mbar_init(bar(B_QD), 1);
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(bar(B_FULL + s), 1);
      mbar_init(bar(B_EMPTY + s), 1);
    }
    mbar_init(bar(B_S), 1);
    mbar_init(bar(B_DP), 1);
    mbar_init(bar(B_SC), 8);  // one arrive per element-wise warp
    mbar_init(bar(B_DS), 8);
    mbar_init(bar(B_ACC), 1);
    mbar_init(bar(B_A), 8);   // Q and dO copied into TMEM by the element-wise warps
    mbar_init(bar(B_DRAIN), 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_do);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  if (warp == 1) {
    tmem_alloc(smem_addr(tmem_holder), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  // Head-major: consecutive CTAs take the items of one head (heaviest first),
  // so the CTAs running together stream the same head's K and V through L2.
  const int h = blockIdx.x / plan.n_items;
  const int hk = h / (plan.hq / plan.hkv);
  Own own;
  decode_own(plan, plan.items[blockIdx.x % plan.n_items], own);
  auto col_d = [](int) { return C::kColD; };

  // Registers: launched at 168 per thread (384 threads); inside its own
  // branch the control warpgroup (warps 0-3) drops to 64 and the two
  // element-wise warpgroups rise to 216: 128 * 64 + 256 * 216 <= 384 * 168.
  if (warp < 4) {
    regs_dec<64>();
  if (warp == 0) {
    // ------------------------------------------------------------ producer
    mbar_arrive_expect_tx_elect(bar(B_QD), 2 * T::kTileBytes);
    for (int b = 0; b < T::kBoxes; ++b) {
      tma_load_2d_elect(smem_addr(sQ + b * T::kBoxBytes), &tm_q, h * DH + b * 64, own.buf_row0, bar(B_QD));
      tma_load_2d_elect(smem_addr(sDO + b * T::kBoxBytes), &tm_do, h * DH + b * 64, own.buf_row0, bar(B_QD));
    }
    DqIter it;
    it.init(plan, own);
    KvTile kt;
    uint32_t c = 0;
    bool ok = true;
    while (ok && it.next(kt)) {
      for (int w = 0; w < 2 && ok; ++w) {
        const int slot = c % C::kStages;
        const uint32_t ph = (c / C::kStages) & 1u;
        ok = mbar_wait_warp(bar(B_EMPTY + slot), ph ^ 1u, abort_flag, err, kWaitNs);
        if (!ok) break;
        mbar_arrive_expect_tx_elect(bar(B_FULL + slot), T::kTileBytes);
        const CUtensorMap* m = w == 0 ? &tm_k : &tm_v;
        for (int b = 0; b < T::kBoxes; ++b)
          tma_load_2d_elect(smem_addr(sKV + slot * T::kTileBytes + b * T::kBoxBytes), m, hk * DH + b * 64,
                            kt.buf_row, bar(B_FULL + slot));
        ++c;
      }
    }
    const uint32_t first = c > (uint32_t)C::kStages ? c - C::kStages : 0u;
    for (uint32_t i = first; i < c; ++i)
      mbar_wait_warp(bar(B_FULL + i % C::kStages), (i / C::kStages) & 1u, abort_flag, nullptr, 1000000000ull);
    mbar_wait_warp(bar(B_QD), 0, abort_flag, nullptr, 1000000000ull);
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    constexpr uint32_t idesc_ss = idesc_bf16_f32(128, 128, false);
    constexpr uint32_t idesc_dq = idesc_bf16_f32(128, DH, true);
    const uint32_t skv = smem_addr(sKV);
    const uint32_t sq = C::kColQA, sdo = C::kColDOA;  // A operands, in TMEM
    // D[col] = A B^T over dh: A (Q or dO, bf16 in TMEM at column acol, 8
    // columns per K-step of 16) times a K-major 128-row key/value tile
    auto issue_ss = [&](uint32_t dcol, uint32_t acol, uint32_t b_base) {
      const uint64_t b0 = sdesc_sw128(b_base, 16, 1024);
#pragma unroll
      for (int kk = 0; kk < DH / 16; ++kk) {
        const uint32_t off = (kk >> 2) * T::kBoxBytes + (kk & 3) * 32;
        tc_mma_ts_elect(tmem + dcol, tmem + acol + kk * 8, sdesc_add(b0, off), idesc_ss, kk > 0 ? 1u : 0u);
      }
    };
    // dQ += dS K: A = dS (bf16 in TMEM, 128 keys as 8 K-steps of 16; keys
    // 0-63 at dcol, keys 64-127 at dcol + 64), B = the K tile read MN-major
    auto issue_dq = [&](uint32_t dcol, uint32_t kbase, bool acc) {
      const uint64_t b0 = sdesc_sw128(kbase, T::kBoxBytes, 1024);
#pragma unroll
      for (int kk = 0; kk < 128 / 16; ++kk) {
        const uint32_t acol = kk < 4 ? dcol + kk * 8 : dcol + 64 + (kk - 4) * 8;
        tc_mma_ts_elect(tmem + C::kColQ, tmem + acol, sdesc_add(b0, kk * 2048), idesc_dq, (acc || kk > 0) ? 1u : 0u);
      }
    };
    auto kslot = [&](int j) { return (2 * j) % C::kStages; };
    auto kph = [&](int j) { return (uint32_t)(((2 * j) / C::kStages) & 1); };
    auto vslot = [&](int j) { return (2 * j + 1) % C::kStages; };
    auto vph = [&](int j) { return (uint32_t)(((2 * j + 1) / C::kStages) & 1); };
    auto slot_addr = [&](int s) { return skv + (uint32_t)s * T::kTileBytes; };

    bool ok = mbar_wait_warp(bar(B_A), 0, abort_flag, err, kWaitNs);
    DqIter it;
    it.init(plan, own);
    KvTile cur, nxt;
    bool have = ok && it.next(cur);
    if (have) {
      ok = mbar_wait_warp(bar(B_FULL + kslot(0)), kph(0), abort_flag, err, kWaitNs);
      if (ok) {
        tc_fence_after();
        issue_ss(C::kColS, sq, slot_addr(kslot(0)));
        tc_commit_elect(bar(B_S));
        ok = mbar_wait_warp(bar(B_FULL + vslot(0)), vph(0), abort_flag, err, kWaitNs);
      }
      if (ok) {
        tc_fence_after();
        issue_ss(col_d(0), sdo, slot_addr(vslot(0)));
        tc_commit_elect(bar(B_DP));
        tc_commit_elect(bar(B_EMPTY + vslot(0)));
      }
      have = ok;
    }
    int j = 0;
    while (have) {
      const bool hn = it.next(nxt);
      // S(j) has been read: S(j+1) may overwrite it
      if (!(ok = mbar_wait_warp(bar(B_SC), j & 1u, abort_flag, err, kWaitNs))) break;
      if (hn) {
        if (!(ok = mbar_wait_warp(bar(B_FULL + kslot(j + 1)), kph(j + 1), abort_flag, err, kWaitNs))) break;
        tc_fence_after();
        issue_ss(C::kColS, sq, slot_addr(kslot(j + 1)));
        tc_commit_elect(bar(B_S));
      }
      if (!(ok = mbar_wait_warp(bar(B_DS), j & 1u, abort_flag, err, kWaitNs))) break;
      tc_fence_after();
      issue_dq(col_d(j), slot_addr(kslot(j)), j > 0);
      tc_commit_elect(bar(B_EMPTY + kslot(j)));
      if (hn) {
        if (!(ok = mbar_wait_warp(bar(B_FULL + vslot(j + 1)), vph(j + 1), abort_flag, err, kWaitNs))) break;
        tc_fence_after();
        issue_ss(col_d(j + 1), sdo, slot_addr(vslot(j + 1)));
        tc_commit_elect(bar(B_DP));
        tc_commit_elect(bar(B_EMPTY + vslot(j + 1)));
      }
      cur = nxt;
      have = hn;
      ++j;
    }
    tc_commit_elect(bar(B_ACC));
    tc_commit_elect(bar(B_DRAIN));
    mbar_wait_warp(bar(B_DRAIN), 0, abort_flag, nullptr, 1000000000ull);
  }
  } else {
    regs_inc<216>();
    // ------------------------------------------------------------ element-wise
    // Two warpgroups share each query row (TMEM lane): warpgroup hh owns key
    // columns [64 hh, 64 hh + 64) of every tile, so two warps per scheduler
    // hide each other's latency.  dS is written over dP columns the same
    // warpgroup has read: hh = 0 -> [0, 32), hh = 1 -> [64, 96).
    const int hh = (warp - 4) >> 2;
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    const bool rvalid = row < own.valid;
    const int qpos = own.pos0 + row;
    const bool docs = plan.n_docs > 0;
    const size_t vec = (size_t)h * plan.S + own.buf_row0 + row;
    const float neg_lg = rvalid ? -__ldg(plan.lg + vec) : 0.f;
    const float dd = rvalid ? __ldg(plan.dd + vec) : 0.f;
    const int row_lo = rvalid ? (docs ? bdoc_start(plan.cu_seqlens, plan.n_docs, qpos) : kNoLo) : kNoHi;
    const int row_hi =
        rvalid ? (plan.causal ? qpos : (docs ? bdoc_last(plan.cu_seqlens, plan.n_docs, qpos) : kNoHi)) : kNoLo;
    const uint64_t c2 = f2_pack(plan.scale_log2, plan.scale_log2);
    const uint64_t nl2 = f2_pack(neg_lg, neg_lg);
    const uint64_t nd2 = f2_pack(-dd, -dd);
    const int c0 = hh * 64;
    const uint32_t ds_off = hh ? 64u : 0u;
    bool ok = true;
    {
      // copy this row of Q (warpgroup 0) or dO (warpgroup 1) from its
      // 128-byte-swizzled shared tile (16-byte chunk c of row r stored at
      // chunk c ^ (r & 7)) into TMEM, two bf16 per column
      ok = mbar_wait(bar(B_QD), 0, abort_flag, err, kWaitNs);
      ok = __all_sync(0xffffffffu, ok);
      if (ok) {
        const uint8_t* src = (hh == 0 ? sQ : sDO) + row * 128;
        const uint32_t dst = tmem + lane_base + (hh == 0 ? C::kColQA : C::kColDOA);
#pragma unroll
        for (int b = 0; b < T::kBoxes; ++b) {
          uint32_t w[32];
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const uint4 v = *reinterpret_cast<const uint4*>(src + b * T::kBoxBytes + ((c ^ (row & 7)) << 4));
            w[4 * c + 0] = v.x;
            w[4 * c + 1] = v.y;
            w[4 * c + 2] = v.z;
            w[4 * c + 3] = v.w;
          }
          tmem_st32(dst + b * 32, w);
        }
        tc_wait_st();
        tc_fence_before();
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(B_A));
    }
    DqIter it;
    it.init(plan, own);
    KvTile kt;
    int j = 0;
    while (ok && it.next(kt)) {
      ok = mbar_wait(bar(B_S), j & 1u, abort_flag, err, kWaitNs);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      uint32_t s[64];
      const uint32_t tS = tmem + lane_base + C::kColS + c0;
      tmem_ld32(tS + 0, *reinterpret_cast<uint32_t(*)[32]>(&s[0]));
      tmem_ld32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(&s[32]));
      tc_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(B_SC));
      if (!kt.full) {
        const int clo = row_lo - kt.pos - c0;
        const int chi = min(row_hi - kt.pos, kt.valid - 1) - c0;
#pragma unroll
        for (int c = 0; c < 64; ++c)
          if (c < clo || c > chi) s[c] = __float_as_uint(-CUDART_INF_F);
      }
      // P = 2^(S * scale * log2(e) - LSE * log2(e)), in place
#pragma unroll
      for (int c = 0; c < 64; c += 2) {
        float x0, x1;
        f2_unpack(f2_fma(f2_pack(__uint_as_float(s[c]), __uint_as_float(s[c + 1])), c2, nl2), x0, x1);
        s[c] = __float_as_uint(ex2_approx(x0));
        s[c + 1] = __float_as_uint(ex2_approx(x1));
      }
      ok = mbar_wait(bar(B_DP), j & 1u, abort_flag, err, kWaitNs);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      const uint32_t tD = tmem + lane_base + col_d(j);
      uint32_t w[32];
#pragma unroll
      for (int ch = 0; ch < 2; ++ch) {
        uint32_t d[32];
        tmem_ld32(tD + c0 + ch * 32, d);
        tc_wait_ld();
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int c = ch * 32 + 2 * i;
          const uint64_t t = f2_add(f2_pack(__uint_as_float(d[2 * i]), __uint_as_float(d[2 * i + 1])), nd2);
          float a, b;
          f2_unpack(f2_mul(f2_pack(__uint_as_float(s[c]), __uint_as_float(s[c + 1])), t), a, b);
          w[ch * 16 + i] = pack_bf16x2(a, b);
        }
      }
      tmem_st32(tD + ds_off, w);
      tc_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(B_DS));
      ++j;
    }
    if (ok) {
      ok = mbar_wait(bar(B_ACC), 0, abort_flag, err, kWaitNs);
      ok = __all_sync(0xffffffffu, ok);
    }
    if (ok) {
      // warpgroup hh writes dQ columns [hh DH/2, (hh + 1) DH/2), staged in
      // the K/V stage buffers (idle once every MMA has completed)
      tc_fence_after();
      const size_t orow0 = (size_t)(own.buf_row0 - own.grp_row0 + quarter * 32);
      const size_t pitch = (size_t)plan.out_hq * DH;
      float* dst = plan.dq + orow0 * pitch + (size_t)(own.grp * plan.hq + h) * DH + hh * (DH / 2);
      float4* stile = reinterpret_cast<float4*>(sKV + (warp - 4) * 4096);
      fence_proxy_async_smem();
#pragma unroll 1
      for (int ch = 0; ch < DH / 64; ++ch) {
        uint32_t o[32];
        if (j > 0) {
          tmem_ld32(tmem + lane_base + C::kColQ + hh * (DH / 2) + ch * 32, o);
          tc_wait_ld();
        }
        warp_store_32x32(stile, o, plan.scale, j == 0, dst + ch * 32, pitch, own.valid - quarter * 32,
                         plan.accumulate != 0);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc(tmem, 512);
  }
}

// ------------------------------------------------------------------ dK/dV side
struct QTile {
  int buf_row, pos, valid, h, r;
  bool full;
};

// Query tiles seen by one key/value tile of shard j: every query head of the
// KV head's group, then the ranks (j + t) mod P that hold shard j at ring
// step t, then their tiles.
struct KvIter {
  const cp_bwd_plan* pl;
  int j, hk, g, t, sg, tl, row0;
  int P, t_begin, t_end, group;
  bool striped_causal;
  // the current ring step's rank r = (j + t) mod P, its segment count and
  // the current segment, read from the plan once per step / segment
  int r, n_seg, s_pos, s_len, s_row, shift;
  int ka0, kb0;                    // own positions without the striped shift
  int lo0, hi0, flo0, fhi0;        // windows of admitted query positions

  __device__ void enter_seg() {
    if (sg < n_seg) {
      s_pos = pl->seg[r][sg].pos;
      s_len = pl->seg[r][sg].len;
      s_row = pl->seg[r][sg].buf_row;
    }
  }
  __device__ void enter_step() {
    r = j + t;
    if (r >= P) r -= P;
    n_seg = pl->nseg[r];
    shift = (striped_causal && j > r) ? 1 : 0;
    sg = tl = 0;
    enter_seg();
  }

  __device__ void init(const cp_bwd_plan& p, const Own& own, int kv_head) {
    pl = &p;
    j = own.rank;
    hk = kv_head;
    row0 = own.grp_row0;
    P = p.P;
    t_begin = p.t_begin;
    t_end = p.t_end;
    group = p.hq / p.hkv;
    striped_causal = p.striped && p.causal;
    g = sg = tl = 0;
    t = p.t_begin;
    if (t < t_end) enter_step();
    ka0 = own.pos0;
    kb0 = own.pos0 + own.valid - 1;
    const bool docs = p.n_docs > 0;
    // a key k admits queries q >= k (causal) inside its document
    lo0 = p.causal ? ka0 : (docs ? bdoc_start(p.cu_seqlens, p.n_docs, ka0) : kNoLo);
    hi0 = docs ? bdoc_last(p.cu_seqlens, p.n_docs, kb0) : kNoHi;
    flo0 = p.causal ? kb0 : (docs ? bdoc_start(p.cu_seqlens, p.n_docs, kb0) : kNoLo);
    fhi0 = docs ? bdoc_last(p.cu_seqlens, p.n_docs, ka0) : kNoHi;
  }

  __device__ bool next(QTile& out) {
    while (g < group) {
      if (t >= t_end) {
        ++g;
        t = t_begin;
        if (t < t_end) enter_step();
        continue;
      }
      if (sg >= n_seg) {
        if (++t < t_end) enter_step();
        continue;
      }
      const int off = tl * 128;
      if (off >= s_len) {
        ++sg;
        tl = 0;
        enter_seg();
        continue;
      }
      const int qa = s_pos + off;
      if (qa > hi0) {  // positions grow along a segment
        ++sg;
        tl = 0;
        enter_seg();
        continue;
      }
      if (qa + 127 < lo0 + shift) {  // queries before the key (or its document): jump over them
        tl = (lo0 + shift - s_pos) / 128;
        continue;
      }
      ++tl;
      const int valid = min(128, s_len - off);
      const int qb = qa + valid - 1;
      if (qb >= lo0 + shift && qa <= hi0) {
        out.buf_row = row0 + s_row + off;
        out.pos = qa;
        out.valid = valid;
        out.h = hk * group + g;
        out.r = r;
        out.full = valid == 128 && qa >= flo0 + shift && qb <= fhi0;
        return true;
      }
    }
    return false;
  }
};

template <int DH>
struct DkvCfg {
  using T = BwdTile<DH>;
  static constexpr int kStages = DH == 128 ? 2 : 4;
  static constexpr int kStageBytes = 2 * T::kTileBytes;  // Q and dO tiles
  static constexpr int kVecBytes = 2 * 128 * 4;          // -LSE*log2(e) and D of the 128 query rows
  static constexpr int kSmemBytes =
      1024 + 2 * T::kTileBytes + kStages * kStageBytes + kStages * kVecBytes + 256;
  static_assert(kSmemBytes <= kMaxSmemPerCta, "dK/dV kernel exceeds the shared memory of a CTA");
  // TMEM: two 128-column buffers (S^T with P^T and dS^T written over it, and
  // dP^T, alternating per query tile) | dV | dK
  static constexpr uint32_t kColDV = 256, kColDK = 256 + DH;
};

template <int DH>
__global__ void __launch_bounds__(kBwdThreads, 1)
    attn_bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
                         const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                         const __grid_constant__ cp_bwd_plan plan) {
  using C = DkvCfg<DH>;
  using T = BwdTile<DH>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sK = smem;
  uint8_t* sV = smem + T::kTileBytes;
  uint8_t* sStage = smem + 2 * T::kTileBytes;
  float* sVec = reinterpret_cast<float*>(sStage + C::kStages * C::kStageBytes);
  uint64_t* bars = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(sVec) + C::kStages * C::kVecBytes);
  const int B_KV = 0, B_FULL = 1, B_EMPTY = 1 + C::kStages, B_S = 1 + 2 * C::kStages, B_DP = B_S + 1,
            B_P = B_DP + 1, B_DS = B_P + 1, B_DPR = B_DS + 1, B_ACC = B_DPR + 1, B_DRAIN = B_ACC + 1,
            B_COUNT = B_DRAIN + 1;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + B_COUNT);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  auto bar = [&](int i) { return smem_addr(bars + i); };
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  uint32_t* err = plan.err;

  if (threadIdx.x == 0) {
    mbar_init(bar(B_KV), 1);
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(bar(B_FULL + s), 1 + 32);  // the copy's expect_tx plus one arrive per producer lane
      mbar_init(bar(B_EMPTY + s), 1);
    }
    mbar_init(bar(B_S), 1);
    mbar_init(bar(B_DP), 1);
    mbar_init(bar(B_P), 8);  // one arrive per element-wise warp
    mbar_init(bar(B_DS), 8);
    mbar_init(bar(B_DPR), 8);  // dP^T read out of TMEM by every element-wise warp
    mbar_init(bar(B_ACC), 1);
    mbar_init(bar(B_DRAIN), 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_do);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  if (warp == 1) {
    tmem_alloc(smem_addr(tmem_holder), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  // Head-major, as in the dQ kernel: the CTAs running together share the
  // query heads whose Q and dO tiles they stream.
  const int hk = blockIdx.x / plan.n_items;
  Own own;
  decode_own(plan, plan.items[blockIdx.x % plan.n_items], own);
  auto col_r = [](int i) { return (i & 1) ? 128u : 0u; };
  auto stage_q = [&](int s) { return sStage + s * C::kStageBytes; };
  auto stage_do = [&](int s) { return sStage + s * C::kStageBytes + T::kTileBytes; };

  // Registers: launched at 168 per thread (384 threads); inside its own
  // branch the control warpgroup (warps 0-3) drops to 64 and the two
  // element-wise warpgroups rise to 216: 128 * 64 + 256 * 216 <= 384 * 168.
  if (warp < 4) {
    regs_dec<64>();
  if (warp == 0) {
    // ------------------------------------------------------------ producer
    mbar_arrive_expect_tx_elect(bar(B_KV), 2 * T::kTileBytes);
    for (int b = 0; b < T::kBoxes; ++b) {
      tma_load_2d_elect(smem_addr(sK + b * T::kBoxBytes), &tm_k, hk * DH + b * 64, own.buf_row0, bar(B_KV));
      tma_load_2d_elect(smem_addr(sV + b * T::kBoxBytes), &tm_v, hk * DH + b * 64, own.buf_row0, bar(B_KV));
    }
    KvIter it;
    it.init(plan, own, hk);
    QTile qt;
    uint32_t c = 0;
    bool ok = true;
    // -LSE*log2(e) and D of a tile's query rows (0 past the tile's end).  The
    // loads for the next tile are issued as soon as the current tile's values
    // are stored, so their latency hides behind the wait for a free stage.
    float nl[4], nd[4];
    auto load_vec = [&](const QTile& x) {
      const size_t base = (size_t)x.h * plan.S + x.buf_row;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int cidx = lane + 32 * i;
        const bool in = cidx < x.valid;
        nl[i] = in ? -__ldg(plan.lg + base + cidx) : 0.f;
        nd[i] = in ? __ldg(plan.dd + base + cidx) : 0.f;
      }
    };
    bool have = it.next(qt);
    if (have) load_vec(qt);
    while (ok && have) {
      const int slot = c % C::kStages;
      const uint32_t ph = (c / C::kStages) & 1u;
      ok = mbar_wait_warp(bar(B_EMPTY + slot), ph ^ 1u, abort_flag, err, kWaitNs);
      if (!ok) break;
      mbar_arrive_expect_tx_elect(bar(B_FULL + slot), 2 * T::kTileBytes);
      for (int b = 0; b < T::kBoxes; ++b) {
        tma_load_2d_elect(smem_addr(stage_q(slot) + b * T::kBoxBytes), &tm_q, qt.h * DH + b * 64, qt.buf_row,
                          bar(B_FULL + slot));
        tma_load_2d_elect(smem_addr(stage_do(slot) + b * T::kBoxBytes), &tm_do, qt.h * DH + b * 64, qt.buf_row,
                          bar(B_FULL + slot));
      }
      float* vl = sVec + slot * (C::kVecBytes / 4);
      float* vd = vl + 128;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        vl[lane + 32 * i] = nl[i];
        vd[lane + 32 * i] = nd[i];
      }
      QTile nx;
      have = it.next(nx);
      if (have) load_vec(nx);
      mbar_arrive(bar(B_FULL + slot));  // release: the stores above are visible to the waiters
      qt = nx;
      ++c;
    }
    const uint32_t first = c > (uint32_t)C::kStages ? c - C::kStages : 0u;
    for (uint32_t i = first; i < c; ++i)
      mbar_wait_warp(bar(B_FULL + i % C::kStages), (i / C::kStages) & 1u, abort_flag, nullptr, 1000000000ull);
    mbar_wait_warp(bar(B_KV), 0, abort_flag, nullptr, 1000000000ull);
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    constexpr uint32_t idesc_ss = idesc_bf16_f32(128, 128, false);
    constexpr uint32_t idesc_acc = idesc_bf16_f32(128, DH, true);
    const uint32_t sk = smem_addr(sK), sv = smem_addr(sV);
    auto issue_ss = [&](uint32_t dcol, uint32_t a_base, uint32_t b_base) {
      const uint64_t a0 = sdesc_sw128(a_base, 16, 1024);
      const uint64_t b0 = sdesc_sw128(b_base, 16, 1024);
#pragma unroll
      for (int kk = 0; kk < DH / 16; ++kk) {
        const uint32_t off = (kk >> 2) * T::kBoxBytes + (kk & 3) * 32;
        tc_mma_ss_elect(tmem + dcol, sdesc_add(a0, off), sdesc_add(b0, off), idesc_ss, kk > 0 ? 1u : 0u);
      }
    };
    // D[dcol] += A (bf16 in TMEM, 128 query rows as 8 K-steps of 16) x B (a
    // 128-row query-side tile read MN-major).  The A columns of K-steps 0-3
    // (queries 0-63) start at lo_col, those of K-steps 4-7 at hi_col.
    auto issue_acc = [&](uint32_t dcol, uint32_t lo_col, uint32_t hi_col, uint32_t b_base, bool acc) {
      const uint64_t b0 = sdesc_sw128(b_base, T::kBoxBytes, 1024);
#pragma unroll
      for (int kk = 0; kk < 128 / 16; ++kk) {
        const uint32_t acol = kk < 4 ? lo_col + kk * 8 : hi_col + (kk - 4) * 8;
        tc_mma_ts_elect(tmem + dcol, tmem + acol, sdesc_add(b0, kk * 2048), idesc_acc, (acc || kk > 0) ? 1u : 0u);
      }
    };
    auto slot_of = [&](int i) { return i % C::kStages; };
    auto ph_of = [&](int i) { return (uint32_t)((i / C::kStages) & 1); };

    bool ok = mbar_wait_warp(bar(B_KV), 0, abort_flag, err, kWaitNs);
    KvIter it;
    it.init(plan, own, hk);
    QTile cur, nxt;
    bool have = ok && it.next(cur);
    if (have) {
      ok = mbar_wait_warp(bar(B_FULL + slot_of(0)), ph_of(0), abort_flag, err, kWaitNs);
      if (ok) {
        tc_fence_after();
        issue_ss(col_r(0), sk, smem_addr(stage_q(slot_of(0))));
        tc_commit_elect(bar(B_S));
        issue_ss(col_r(1), sv, smem_addr(stage_do(slot_of(0))));
        tc_commit_elect(bar(B_DP));
      }
      have = ok;
    }
    int i = 0;
    while (have) {
      const bool hn = it.next(nxt);
      const int s = slot_of(i);
      if (!(ok = mbar_wait_warp(bar(B_P), i & 1u, abort_flag, err, kWaitNs))) break;
      tc_fence_after();
      issue_acc(C::kColDV, col_r(i) + 0, col_r(i) + 96, smem_addr(stage_do(s)), i > 0);
      if (hn) {
        // S^T(i+1) goes where dP^T(i) lives: issued as soon as every
        // element-wise warp has read dP^T(i), while they still form dS^T(i)
        if (!(ok = mbar_wait_warp(bar(B_DPR), i & 1u, abort_flag, err, kWaitNs))) break;
        if (!(ok = mbar_wait_warp(bar(B_FULL + slot_of(i + 1)), ph_of(i + 1), abort_flag, err, kWaitNs))) break;
        tc_fence_after();
        issue_ss(col_r(i + 1), sk, smem_addr(stage_q(slot_of(i + 1))));
        tc_commit_elect(bar(B_S));
      }
      if (!(ok = mbar_wait_warp(bar(B_DS), i & 1u, abort_flag, err, kWaitNs))) break;
      tc_fence_after();
      issue_acc(C::kColDK, col_r(i) + 32, col_r(i) + 64, smem_addr(stage_q(s)), i > 0);
      tc_commit_elect(bar(B_EMPTY + s));
      if (hn) {
        // dP^T(i+1) goes where P^T(i) / dS^T(i) live: issued after the two
        // MMAs that read them
        issue_ss(col_r(i), sv, smem_addr(stage_do(slot_of(i + 1))));
        tc_commit_elect(bar(B_DP));
      }
      cur = nxt;
      have = hn;
      ++i;
    }
    tc_commit_elect(bar(B_ACC));
    tc_commit_elect(bar(B_DRAIN));
    mbar_wait_warp(bar(B_DRAIN), 0, abort_flag, nullptr, 1000000000ull);
  }
  } else {
    regs_inc<216>();
    // ------------------------------------------------------------ element-wise
    // Two warpgroups share each key row (TMEM lane): warpgroup hh owns query
    // columns [64 hh, 64 hh + 64) of every tile, so two warps per scheduler
    // hide each other's latency.  Each writes its packed P^T and dS^T only
    // over S^T columns it has itself read:
    //   hh = 0: P^T(q 0-63) -> cols [0, 32),   dS^T(q 0-63) -> cols [32, 64)
    //   hh = 1: dS^T(q 64-127) -> cols [64, 96), P^T(q 64-127) -> cols [96, 128)
    const int hh = (warp - 4) >> 2;
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    const bool rvalid = row < own.valid;
    const int kpos = own.pos0 + row;
    const bool docs = plan.n_docs > 0;
    // admitted query positions of this key: [col_lo, col_hi]
    const int lo0 = rvalid ? (plan.causal ? kpos : (docs ? bdoc_start(plan.cu_seqlens, plan.n_docs, kpos) : kNoLo))
                           : kNoHi;
    const int col_hi = rvalid ? (docs ? bdoc_last(plan.cu_seqlens, plan.n_docs, kpos) : kNoHi) : kNoLo;
    const uint64_t c2 = f2_pack(plan.scale_log2, plan.scale_log2);
    const int c0 = hh * 64;                    // first query column of this warpgroup
    const uint32_t p_col = hh ? 96u : 0u;      // where its P^T goes
    const uint32_t ds_col = hh ? 64u : 32u;    // where its dS^T goes
    KvIter it;
    it.init(plan, own, hk);
    QTile qt;
    int i = 0;
    bool ok = true;
    while (it.next(qt)) {
      const int s = i % C::kStages;
      const float* vl = sVec + s * (C::kVecBytes / 4) + c0;
      const float* vd = sVec + s * (C::kVecBytes / 4) + 128 + c0;
      ok = mbar_wait(bar(B_S), i & 1u, abort_flag, err, kWaitNs);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      // P^T = 2^(S^T * scale * log2(e) - LSE_q * log2(e)), kept only as the
      // bf16 pairs the dV MMA reads
      const uint32_t tR = tmem + lane_base + col_r(i);
      const int shift = (plan.striped && plan.causal && own.rank > qt.r && rvalid) ? 1 : 0;
      const int clo = lo0 + shift - qt.pos - c0;
      const int chi = min(col_hi - qt.pos, qt.valid - 1) - c0;
      uint32_t pk[32];
      {
        uint32_t sv[64];
        tmem_ld32(tR + c0, *reinterpret_cast<uint32_t(*)[32]>(&sv[0]));
        tmem_ld32(tR + c0 + 32, *reinterpret_cast<uint32_t(*)[32]>(&sv[32]));
        tc_wait_ld();
        if (!qt.full) {
#pragma unroll
          for (int cc = 0; cc < 64; ++cc)
            if (cc < clo || cc > chi) sv[cc] = __float_as_uint(-CUDART_INF_F);
        }
#pragma unroll
        for (int i4 = 0; i4 < 16; ++i4) {
          const float4 l4 = *reinterpret_cast<const float4*>(vl + 4 * i4);
          float x0, x1, x2, x3;
          f2_unpack(f2_fma(f2_pack(__uint_as_float(sv[4 * i4]), __uint_as_float(sv[4 * i4 + 1])), c2,
                           f2_pack(l4.x, l4.y)),
                    x0, x1);
          f2_unpack(f2_fma(f2_pack(__uint_as_float(sv[4 * i4 + 2]), __uint_as_float(sv[4 * i4 + 3])), c2,
                           f2_pack(l4.z, l4.w)),
                    x2, x3);
          pk[2 * i4] = pack_bf16x2(ex2_approx(x0), ex2_approx(x1));
          pk[2 * i4 + 1] = pack_bf16x2(ex2_approx(x2), ex2_approx(x3));
        }
      }
      tmem_st32(tR + p_col, pk);
      tc_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(B_P));
      ok = mbar_wait(bar(B_DP), i & 1u, abort_flag, err, kWaitNs);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      // dS^T = P^T * (dP^T - D_q) from the bf16 P^T
      {
        const uint32_t tD = tmem + lane_base + col_r(i + 1) + c0;
        uint32_t d[64];
        tmem_ld32(tD, *reinterpret_cast<uint32_t(*)[32]>(&d[0]));
        tmem_ld32(tD + 32, *reinterpret_cast<uint32_t(*)[32]>(&d[32]));
        tc_wait_ld();
        // dP^T(i) is in registers: its TMEM columns may take S^T(i+1)
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(B_DPR));
        uint32_t w[32];
#pragma unroll
        for (int i4 = 0; i4 < 16; ++i4) {
          const float4 d4 = *reinterpret_cast<const float4*>(vd + 4 * i4);
          const uint32_t pw0 = pk[2 * i4], pw1 = pk[2 * i4 + 1];
          const uint64_t t0 = f2_add(f2_pack(__uint_as_float(d[4 * i4]), __uint_as_float(d[4 * i4 + 1])),
                                     f2_pack(-d4.x, -d4.y));
          const uint64_t t1 = f2_add(f2_pack(__uint_as_float(d[4 * i4 + 2]), __uint_as_float(d[4 * i4 + 3])),
                                     f2_pack(-d4.z, -d4.w));
          float a0, a1, a2, a3;
          f2_unpack(f2_mul(f2_pack(__uint_as_float(pw0 << 16), __uint_as_float(pw0 & 0xFFFF0000u)), t0), a0, a1);
          f2_unpack(f2_mul(f2_pack(__uint_as_float(pw1 << 16), __uint_as_float(pw1 & 0xFFFF0000u)), t1), a2, a3);
          w[2 * i4] = pack_bf16x2(a0, a1);
          w[2 * i4 + 1] = pack_bf16x2(a2, a3);
        }
        tmem_st32(tR + ds_col, w);
      }
      tc_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(B_DS));
      ++i;
    }
    if (ok) {
      ok = mbar_wait(bar(B_ACC), 0, abort_flag, err, kWaitNs);
      ok = __all_sync(0xffffffffu, ok);
    }
    if (ok) {
      // warpgroup 0 writes dV, warpgroup 1 writes dK * scale, staged in the
      // Q/dO stage buffers (idle once every MMA has completed)
      tc_fence_after();
      const size_t pitch = (size_t)plan.out_hkv * DH;
      const size_t orow0 = (size_t)(own.buf_row0 - own.grp_row0 + quarter * 32);
      float* dst = (hh == 0 ? plan.dv : plan.dk) + orow0 * pitch + (size_t)(own.grp * plan.hkv + hk) * DH;
      const uint32_t col = hh == 0 ? C::kColDV : C::kColDK;
      const float f = hh == 0 ? 1.f : plan.scale;
      float4* stile = reinterpret_cast<float4*>(sStage + (warp - 4) * 4096);
      fence_proxy_async_smem();
#pragma unroll 1
      for (int ch = 0; ch < DH / 32; ++ch) {
        uint32_t o[32];
        if (i > 0) {
          tmem_ld32(tmem + lane_base + col + ch * 32, o);
          tc_wait_ld();
        }
        warp_store_32x32(stile, o, f, i == 0, dst + ch * 32, pitch, own.valid - quarter * 32, plan.accumulate != 0);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc(tmem, 512);
  }
}

// ------------------------------------------------------------------ prep
// D = rowsum(dO * O) and LSE * log2(e) per (row, head), one warp per pair.
// The outputs are [hg][groups * G] (plan rows: group g's rows start at g G);
// O, dO are read in their final [G][groups * hg][dh] layout and LSE in its
// final [groups * hg][G] layout, group g holding heads [g hg, (g + 1) hg).
template <int DH>
__global__ void __launch_bounds__(256) bwd_prep_kernel(const float* __restrict__ o, const uint16_t* __restrict__ dout,
                                                       const float* __restrict__ lse, int rows, int G, int hg,
                                                       int groups, float* __restrict__ lg, float* __restrict__ dd) {
  constexpr int E = DH / 32;
  const long long item = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  if (item >= (long long)rows * hg) return;
  const int lane = threadIdx.x & 31;
  const int row = (int)(item / hg);
  const int h = (int)(item - (long long)row * hg);
  const int g = row / G, x = row - g * G;
  const int hq = groups * hg;
  const size_t base = ((size_t)x * hq + g * hg + h) * DH + (size_t)lane * E;
  float acc = 0.f;
  if constexpr (E == 4) {
    const float4 a = __ldcs(reinterpret_cast<const float4*>(o + base));
    const uint2 b = __ldcs(reinterpret_cast<const uint2*>(dout + base));
    acc = a.x * __uint_as_float(b.x << 16) + a.y * __uint_as_float(b.x & 0xFFFF0000u) +
          a.z * __uint_as_float(b.y << 16) + a.w * __uint_as_float(b.y & 0xFFFF0000u);
  } else {
    const float2 a = __ldcs(reinterpret_cast<const float2*>(o + base));
    const uint32_t b = __ldcs(reinterpret_cast<const unsigned int*>(dout + base));
    acc = a.x * __uint_as_float(b << 16) + a.y * __uint_as_float(b & 0xFFFF0000u);
  }
#pragma unroll
  for (int m = 16; m > 0; m >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, m);
  if (lane == 0) {
    const size_t v = (size_t)h * rows + row;
    const float l = lse[((size_t)g * hg + h) * G + x];
    dd[v] = acc;
    lg[v] = l == -CUDART_INF_F ? 0.f : l * kLog2e;
  }
}

template <int DH>
cudaError_t launch_bwd_dh(const CUtensorMap& tq, const CUtensorMap& tdo, const CUtensorMap& tk,
                          const CUtensorMap& tv, const cp_bwd_plan& plan, bool dq_side, cudaStream_t st) {
  static bool configured = false;
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(attn_bwd_dq_kernel<DH>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         DqCfg<DH>::kSmemBytes);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(attn_bwd_dkdv_kernel<DH>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             DkvCfg<DH>::kSmemBytes);
    if (e != cudaSuccess) return e;
    configured = true;
  }
  if (plan.n_items <= 0) return cudaSuccess;
  if (dq_side)
    attn_bwd_dq_kernel<DH><<<plan.n_items * plan.hq, kBwdThreads, DqCfg<DH>::kSmemBytes, st>>>(tq, tdo, tk, tv, plan);
  else
    attn_bwd_dkdv_kernel<DH>
        <<<plan.n_items * plan.hkv, kBwdThreads, DkvCfg<DH>::kSmemBytes, st>>>(tq, tdo, tk, tv, plan);
  launch_counter()++;
  return cudaGetLastError();
}

}  // namespace

// rows = groups * G plan rows, hg heads per group.
cudaError_t launch_bwd_prep(int dh, const float* o, const void* dout, const float* lse, int G, int hg, int groups,
                            float* lg, float* dd, cudaStream_t st) {
  const int rows = G * groups;
  const long long items = (long long)rows * hg;
  if (items <= 0) return cudaSuccess;
  const unsigned grid = (unsigned)((items + 7) / 8);
  if (dh == 128)
    bwd_prep_kernel<128><<<grid, 256, 0, st>>>(o, static_cast<const uint16_t*>(dout), lse, rows, G, hg, groups, lg, dd);
  else
    bwd_prep_kernel<64><<<grid, 256, 0, st>>>(o, static_cast<const uint16_t*>(dout), lse, rows, G, hg, groups, lg, dd);
  launch_counter()++;
  return cudaGetLastError();
}

// dq_side: the dQ kernel (CTAs = items x hq); otherwise the dK/dV kernel
// (CTAs = items x hkv).
cudaError_t launch_bwd(int dh, const CUtensorMap& tq, const CUtensorMap& tdo, const CUtensorMap& tk,
                       const CUtensorMap& tv, const cp_bwd_plan& plan, bool dq_side, cudaStream_t st) {
  if (dh == 128) return launch_bwd_dh<128>(tq, tdo, tk, tv, plan, dq_side, st);
  return launch_bwd_dh<64>(tq, tdo, tk, tv, plan, dq_side, st);
}

}  // namespace cp
