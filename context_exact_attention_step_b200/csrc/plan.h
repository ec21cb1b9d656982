// Launch plans shared by the host scheduler and the sm_100a kernels.
//
// A plan is a small POD passed by value as a __grid_constant__ kernel
// parameter, so every launch is self-describing (no host->device copy of a
// work list, nothing to allocate, capturable in a CUDA graph).
#pragma once
#include <stdint.h>

#define CP_MAX_SEGS 4        // row segments per side of one block pair
#define CP_MAX_PAIRS 64      // block pairs per attention launch
#define CP_MAX_BLOCKS 16     // pair blocks per attention launch (see cp_attn_plan)
#define CP_MAX_TASKS 128     // merge tasks per merge launch
#define CP_MAX_INPUTS 512    // merge inputs per merge launch
#define CP_Q_TILE 256        // query rows per CTA (two 128-row MMA tiles)
#define CP_KV_TILE 128       // key/value rows per pipeline stage (and per S tile)

// A run of consecutive buffer rows whose global token positions are also
// consecutive.  buf_row: first row in the Q/K/V buffer; pos: global position
// of that row; len: number of rows; out_row: first row in the output buffer
// (Q side only).
struct cp_seg {
  int32_t buf_row;
  int32_t pos;
  int32_t len;
  int32_t out_row;
};

// One block pair of a ring step: some query rows of rank r against the
// key/value rows of shard j.
struct cp_pair_desc {
  int32_t nq, nk;
  cp_seg q[CP_MAX_SEGS];
  cp_seg k[CP_MAX_SEGS];
  int32_t qtiles;     // sum over q segments of ceil(len / CP_Q_TILE)
  int32_t qt_begin;   // first query tile of this pair among its block's tiles of one head
  int32_t reverse;    // visit the query tiles last-first (heaviest first under causal)
  int32_t lse_ld;     // row pitch of the LSE output ([hq][lse_ld])
  float* o;           // O output, [rows][hq][dh] fp32
  float* lse;         // LSE output, [hq][lse_ld] fp32
};

// The pairs of a launch come in blocks: the pairs of one block read the same
// Q/K/V rows (all ring steps of one ring), different blocks read different
// rows (the head groups of Ulysses, the head blocks of the hybrid).  Inside a
// block the CTAs run head-major -- every query tile of every pair of head 0,
// then head 1, ... -- so the CTAs resident at one time share one head's Q and
// K/V through L2 instead of streaming every head's side by side.
struct cp_attn_plan {
  int32_t n_pairs;
  int32_t total_ctas;
  int32_t n_blocks;
  int32_t blk_cta_begin[CP_MAX_BLOCKS + 1];   // CTAs of block b: [blk_cta_begin[b], blk_cta_begin[b + 1])
  int32_t blk_pair_begin[CP_MAX_BLOCKS + 1];  // pairs of block b: [blk_pair_begin[b], blk_pair_begin[b + 1])
  int32_t blk_qtiles[CP_MAX_BLOCKS];          // query tiles per head of block b
  int32_t hq, hkv;
  int32_t causal;
  int32_t n_docs;               // 0: no document mask
  const int32_t* cu_seqlens;    // device, n_docs + 1 entries
  float scale_log2;             // softmax_scale * log2(e)
  uint32_t* err;                // device error word (bounded-wait timeouts)
  cp_pair_desc pairs[CP_MAX_PAIRS];
};

// Merge: rows [out_row0, out_row0 + rows) of the output are the LSE-weighted
// fold of n_in partial results; input i supplies row (row0 + x) for output
// row (out_row0 + x).  A task covers h heads of its inputs and writes them as
// heads [head_off, head_off + h) of an output whose rows hold o_heads heads,
// so a merge can scatter head blocks straight into a wider output.
struct cp_merge_input {
  const float* o;      // [.][h][dh]
  const float* lse;    // [h][lse_ld]
  int32_t row0;
  int32_t lse_ld;
};

struct cp_merge_task {
  int32_t out_row0;
  int32_t rows;
  int32_t n_in;
  int32_t in_begin;
  int32_t head_off;      // first output head of the task's h heads
  int32_t cta_begin;     // first CTA of the task in the launch (tasks in CTA order)
};

struct cp_merge_plan {
  int32_t n_tasks;
  int32_t h, dh;
  int32_t lse_out_ld;
  int32_t o_heads;       // heads per output row of O (>= head_off + h)
  float* o_out;          // [.][o_heads][dh]
  float* lse_out;        // [o_heads][lse_out_ld]
  uint16_t* o_out_bf16;  // optional bf16 copy of O (nullable)
  cp_merge_task tasks[CP_MAX_TASKS];
  cp_merge_input inputs[CP_MAX_INPUTS];
};

// ------------------------------------------------------------------ backward
#define CP_BWD_MAX_RANKS 16
#define CP_BWD_MAX_ITEMS 2048   // own 128-row tiles per backward launch

// Backward of the ring over P ranks, run as two kernels: one CTA per
// (own 128-row tile, head).  For the dQ kernel the own rows are a query tile
// of rank r and the partners are the key/value shards j = (r - t) mod P of
// the ring steps t = 0..P-1; for the dK/dV kernel the own rows are a key/value
// tile of shard j and the partners are the ranks (j + t) mod P that hold it at
// step t (and every query head of its group).
//
// item: (rank << 26) | (segment << 25) | (group << 19) | tile, tile =
// 128-row tile index inside the segment.  A group is a block of heads whose
// rows start at group * group_rows in the Q/K/V/dO buffers (the head-major
// layout of the Ulysses transpose; one group for the plain ring).  Striped
// layouts carry local row indices as positions; a key of shard j seen from
// rank r then sits one position later when j > r.
#define CP_BWD_MAX_GROUPS 64
struct cp_bwd_plan {
  int32_t P;
  int32_t hq, hkv;
  int32_t causal;
  int32_t striped;
  int32_t n_docs;
  const int32_t* cu_seqlens;
  float scale_log2;             // softmax_scale * log2(e)
  float scale;
  int32_t S;                    // rows of every buffer (row pitch of lg, dd)
  int32_t group_rows;           // rows per head group in the buffers
  int32_t out_hq, out_hkv;      // heads per row of dq and of dk, dv (all groups)
  int32_t nseg[CP_BWD_MAX_RANKS];
  cp_seg seg[CP_BWD_MAX_RANKS][2];
  const float* lg;              // [hq][S]: LSE * log2(e) (0 where LSE = -inf)
  const float* dd;              // [hq][S]: rowsum(dO * O)
  float* dq;                    // [group_rows][out_hq][dh]: group g holds heads [g hq, (g + 1) hq)
  float* dk;                    // [group_rows][out_hkv][dh]
  float* dv;                    // [group_rows][out_hkv][dh]
  uint32_t* err;
  int32_t t_begin, t_end;       // ring steps every own tile visits: [t_begin, t_end) of 0..P-1
  int32_t accumulate;           // 1: add to dq / dk / dv instead of overwriting them
  int32_t n_items;
  uint32_t items[CP_BWD_MAX_ITEMS];
};
