/*
 * cp_attn.h -- C ABI of the B200 (sm_100a) context-parallel exact attention
 * library: ring-step block attention producing partial (O, LSE), the fp32 LSE
 * merge, the zigzag and striped reorders, the Ulysses sequence<->head
 * transpose and head-block split, the ring / Ulysses / hybrid (USP)
 * composites with the P ranks of a context-parallel group held as virtual
 * ranks on one GPU, their backward, and the backward of one block pair (the
 * per-GPU step of a ring that spans GPUs).
 *
 * Conventions shared by every call
 * --------------------------------
 *  - Tensor arguments are DEVICE pointers owned by the caller (allocate them
 *    however you like, e.g. through PyTorch).  The library allocates no device
 *    memory; calls that need scratch space take a caller workspace.
 *  - Host arrays (chunk lists, pointer lists, cu_seqlens_host) are read during
 *    the call only and may be freed when it returns.
 *  - Every call is asynchronous on `stream` (a cudaStream_t passed as void*;
 *    NULL = legacy default stream) and returns before the GPU work finishes.
 *  - Layouts are row-major, token-major: a Q/K/V/O tensor is [rows][heads][dh]
 *    (the pages' [batch, seq_len, heads, head_dim] with batch = 1 and no
 *    padding between heads), an LSE tensor is [heads][rows].
 *  - Every device pointer must be 16-byte aligned, and row pitches follow from
 *    the shapes (no strides).
 *  - Errors: every call returns a cp_status.  Arguments are validated before
 *    anything is launched; on error nothing is launched, nothing is written,
 *    and cp_last_error_string() (thread-local) describes the problem.  The
 *    library never aborts the process and never prints.
 *  - Kernels that wait on hardware barriers give up after a bounded time and
 *    record it in a device error word read by cp_device_error(); they never
 *    trap.
 */
#ifndef CP_ATTN_H
#define CP_ATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  CP_OK = 0,
  CP_ERR_INVALID_ARG = 1,  /* a size, count or pointer is out of range       */
  CP_ERR_UNSUPPORTED = 2,  /* valid request outside what the library supports */
  CP_ERR_ALIGNMENT = 3,    /* a device pointer is not 16-byte aligned        */
  CP_ERR_WORKSPACE = 4,    /* workspace missing or smaller than required      */
  CP_ERR_CUDA = 5          /* the CUDA runtime reported an error              */
} cp_status;

typedef enum { CP_BF16 = 0, CP_FP32 = 1 } cp_dtype;
typedef enum { CP_MASK_NONE = 0, CP_MASK_CAUSAL = 1 } cp_mask;
typedef enum { CP_LAYOUT_CONTIGUOUS = 0, CP_LAYOUT_ZIGZAG = 1, CP_LAYOUT_STRIPED = 2 } cp_layout;
typedef enum { CP_SEQ_TO_HEAD = 0, CP_HEAD_TO_SEQ = 1 } cp_dir;

/* A run of consecutive rows of a Q or K/V buffer whose global token
 * positions are consecutive: rows [row, row + len) of the buffer (in list
 * order) hold positions [start, start + len). */
typedef struct {
  int32_t start;
  int32_t len;
} cp_chunk;

#define CP_MAX_CHUNKS 4

/* Description of the last error returned on the calling thread. */
const char* cp_last_error_string(void);

/* Library version string. */
const char* cp_version(void);

/*
 * cp_block_attn_fwd -- one ring step for one virtual rank: the rank's query
 * shard against one key/value block, with that block pair's mask offsets.
 *
 * Computes, for every query row i and query head h (kv head g = h / (hq/hkv)),
 *   s_j = softmax_scale * q_i . k_j over the admitted keys j,
 *   O_i = sum_j softmax(s)_j v_j  (normalised within this block pair),
 *   LSE_i = ln sum_j exp(s_j)     (natural log of the scaled scores),
 * where key j is admitted iff (mask == CP_MASK_CAUSAL ? pos(j) <= pos(i) : 1)
 * and (n_docs > 0 ? doc(pos(i)) == doc(pos(j)) : 1).  Rows with no admitted
 * key get O = 0 and LSE = -inf.  This is the block step of Ring Attention
 * ("序列並行（Sequence Parallelism）" concept page (compassingai), "Ring
 * Attention 的不同思路" steps 1-4 and 技術原理 §二, S = Q K^T / sqrt(d_k)),
 * with the per-block mask offsets of the "Context Parallelism" write-up
 * (pwwt.cn) §3.3, and packed documents through cu_seqlens (XTuner tutorial
 * ch09 §9.5).
 *
 *   q            [n_q][hq][dh] bf16 (dtype must be CP_BF16)
 *   k, v         [n_k][hkv][dh] bf16
 *   q_chunks     host, nq_chunks (1..CP_MAX_CHUNKS) entries covering the n_q
 *                rows in order; positions of the query rows
 *   k_chunks     host, nk_chunks entries covering the n_k rows; key positions
 *   mask         CP_MASK_NONE or CP_MASK_CAUSAL (by global position)
 *   cu_seqlens_dev  device int32 [n_docs + 1], 0 = first, strictly increasing
 *                (document lengths > 0), covering every position used; NULL
 *                with n_docs = 0 for no document mask
 *   softmax_scale  > 0, or <= 0 for 1/sqrt(dh)
 *   o            out, [n_q][hq][dh] fp32
 *   lse          out, [hq][n_q] fp32
 * Supported: dh in {64, 128}; hq % hkv == 0; 1 <= n_q, n_k < 2^30.
 */
cp_status cp_block_attn_fwd(const void* q, const void* k, const void* v, cp_dtype dtype, int n_q, int n_k,
                            int hq, int hkv, int dh, const cp_chunk* q_chunks, int nq_chunks,
                            const cp_chunk* k_chunks, int nk_chunks, cp_mask mask,
                            const int32_t* cu_seqlens_dev, int n_docs, float softmax_scale, float* o,
                            float* lse, void* stream);

/*
 * cp_lse_merge -- fold n_parts partial results over the same rows:
 *   LSE = ln sum_i exp(LSE_i),  O = sum_i exp(LSE_i - LSE) * O_i,
 * in fp32; partials with LSE_i = -inf for a row contribute nothing there (their
 * O is never combined, so it may hold anything, NaN included); rows where every
 * LSE_i is -inf get O = 0, LSE = -inf.  The
 * block-granular form of the online-softmax recurrence ("序列並行" concept page
 * (compassingai), 技術原理 §二).
 *
 *   o_parts      host array of n_parts device pointers, each [rows][h][dh] fp32
 *   lse_parts    host array of n_parts device pointers, each [h][rows] fp32
 *   o_out        out, [rows][h][dh] fp32 (may not alias an input)
 *   lse_out      out, [h][rows] fp32
 *   o_out_bf16   optional out, [rows][h][dh] bf16 copy of O (NULL to skip)
 * Supported: 1 <= n_parts <= 64, dh in {64, 128}.
 */
cp_status cp_lse_merge(int n_parts, const float* const* o_parts, const float* const* lse_parts, int rows, int h,
                       int dh, float* o_out, float* lse_out, void* o_out_bf16, void* stream);

/*
 * cp_ring_attn_workspace_size -- bytes of workspace cp_ring_attn_fwd needs for
 * these arguments (partials of every live block pair, plus bf16 copies of Q,
 * K, V when dtype is CP_FP32).  cu_seqlens_host may be NULL; when given, the
 * same array must be passed to cp_ring_attn_fwd.
 */
cp_status cp_ring_attn_workspace_size(int S, int hq, int hkv, int dh, int P, cp_layout layout, cp_mask mask,
                                      cp_dtype dtype, const int32_t* cu_seqlens_host, int n_docs, size_t* bytes);

/*
 * cp_ring_attn_fwd -- exact attention of a whole sequence split over P
 * virtual ranks, computed as Ring Attention does it: rank r keeps its query
 * shard, at step t = 0..P-1 it holds key/value shard j = (r - t) mod P, every
 * live block pair yields a partial (O, LSE) (cp_block_attn_fwd semantics) and
 * the partials of each rank are folded by the LSE merge.  Block pairs the mask
 * leaves empty are skipped, as are the query rows of a pair that see none of
 * its keys.  ("序列並行" concept page (compassingai), Ring Attention steps 1-4;
 * "Context Parallelism" write-up (pwwt.cn) §2.2, §3.3; zigzag balancing:
 * "长上下文序列并行训练深度解析" (mooersco) timeline, Striped / zigzag.)
 *
 *   q            [S][hq][dh], k, v [S][hkv][dh], bf16 or fp32 (fp32 inputs are
 *                rounded to bf16, nearest-even, before use) ALREADY in the
 *                rank-major sharded order of `layout`: rank r holds rows
 *                [r*S/P, (r+1)*S/P).  CP_LAYOUT_CONTIGUOUS: rank r holds
 *                positions [r*S/P, (r+1)*S/P).  CP_LAYOUT_ZIGZAG: rank r holds
 *                chunk r then chunk 2P-1-r of the 2P chunks of S/(2P) tokens
 *                (cp_zigzag_reorder produces this order).  CP_LAYOUT_STRIPED:
 *                rank r holds positions r, r+P, r+2P, ... (Striped Attention,
 *                same timeline; cp_striped_reorder produces this order); not
 *                combinable with documents (CP_ERR_UNSUPPORTED).
 *   cu_seqlens_host, cu_seqlens_dev  the same document table on host and device
 *                (n_docs + 1 entries; both NULL and n_docs = 0 for none); the
 *                host copy lets the scheduler skip pairs across documents
 *   o            out, [S][hq][dh] fp32, in the same sharded order as q
 *   lse          out, [hq][S] fp32, same order
 *   workspace    device scratch of at least cp_ring_attn_workspace_size bytes,
 *                256-byte aligned; its contents are overwritten
 * Supported: 1 <= P <= 16, S % P == 0 (S % 2P == 0 for zigzag), dh in {64,128},
 * hq % hkv == 0.
 */
cp_status cp_ring_attn_fwd(const void* q, const void* k, const void* v, cp_dtype dtype, int S, int hq, int hkv,
                           int dh, int P, cp_layout layout, cp_mask mask, const int32_t* cu_seqlens_host,
                           const int32_t* cu_seqlens_dev, int n_docs, float softmax_scale, float* o, float* lse,
                           void* workspace, size_t ws_bytes, void* stream);

/*
 * cp_ulysses_permute -- the DeepSpeed-Ulysses all-to-all transpose as a local
 * permute ("序列並行" concept page (compassingai), 技術原理 §三 "Ulysses 的
 * AllToAll 轉置"; "Context Parallelism" write-up (pwwt.cn) §2.3), with n = S/P:
 *   CP_SEQ_TO_HEAD: in [P][n][h][dh] -> out [P][S][h/P][dh],
 *                   out[r][p*n + s][h'] = in[p][s][r*h/P + h']
 *   CP_HEAD_TO_SEQ: the inverse.
 * Bit-exact copy of elem_bytes-sized elements (2 for bf16, 4 for fp32).
 * For GQA call it on Q with h = hq and on K, V with h = hkv.
 * Supported: P | S, P | h; in and out must not overlap.
 */
cp_status cp_ulysses_permute(const void* in, void* out, int P, int S, int h, int dh, int elem_bytes, cp_dir dir,
                             void* stream);

/*
 * cp_zigzag_reorder -- natural token order <-> rank-major zigzag order
 * (rank i holds chunks i and 2P-1-i of 2P chunks of S/(2P) rows), the load
 * balancing of causal Ring Attention: pairing an early chunk with a late one
 * gives every rank the same share of the causal mask ("长上下文序列并行训练
 * 深度解析" (mooersco) timeline, Striped / zigzag 负载均衡重排; the pages name
 * the scheme without fixing the chunk pairing, which is taken as i with
 * 2P-1-i, in that order inside the shard).  in/out are
 * [batch][S][row_bytes] byte arrays: use batch = 1, row_bytes = h*dh*elem for
 * Q/K/V/O, and batch = h, row_bytes = 4 for an fp32 LSE [h][S].
 * inverse = 0: natural -> zigzag; 1: zigzag -> natural.  Bit-exact.
 * Supported: S % (2P) == 0; in and out must not overlap.
 */
cp_status cp_zigzag_reorder(const void* in, void* out, int P, int S, int batch, int row_bytes, int inverse,
                            void* stream);

/*
 * cp_head_block_split -- the local half of the Ulysses all-to-all when every
 * rank is its own GPU ("序列並行" concept page (compassingai), 技術原理 §三;
 * "Context Parallelism" write-up (pwwt.cn) §2.3): one rank's rows in [n][h][dh]
 * are regrouped by head block, out [P][n][h/P][dh], out[r][s][h'] =
 * in[s][r*h/P + h'], so that block r can be sent to rank r; inverse = 1 undoes
 * it after the exchange.  Bit-exact copy of elem_bytes-sized elements.
 * Supported: P | h; in and out must not overlap.
 */
cp_status cp_head_block_split(const void* in, void* out, int n, int h, int dh, int P, int elem_bytes, int inverse,
                              void* stream);

/*
 * cp_striped_reorder -- natural token order <-> rank-major striped order
 * (token t on rank t mod P, rank r's rows in position order: row r*S/P + a
 * holds position a*P + r), the Striped Attention balancing of causal Ring
 * Attention: every rank holds positions spread evenly over the sequence, so
 * every block pair is a (possibly one-key-shifted) local causal block
 * ("长上下文序列并行训练深度解析" (mooersco) timeline, Striped / zigzag
 * 负载均衡重排).  in/out are [batch][S][row_bytes] byte arrays as
 * for cp_zigzag_reorder.  inverse = 0: natural -> striped; 1: back.  Bit-exact.
 * Supported: S % P == 0; in and out must not overlap.
 */
cp_status cp_striped_reorder(const void* in, void* out, int P, int S, int batch, int row_bytes, int inverse,
                             void* stream);

/*
 * cp_ulysses_attn_workspace_size / cp_ulysses_attn_fwd -- the Ulysses path:
 * seq->head transpose of Q (hq heads) and K, V (hkv heads), local attention of
 * every head group over the whole sequence (P = 1 ring, GQA inside the group),
 * head->seq transpose of O back.  Inputs q [P][S/P][hq][dh], k, v
 * [P][S/P][hkv][dh] bf16 (sequence-sharded, natural position order); outputs o
 * [P][S/P][hq][dh] fp32 and lse [hq][S] fp32 (natural positions).
 * Supported: P | hkv (the Ulysses head limit; KV heads are not replicated),
 * P | S, dh in {64, 128}.
 */
cp_status cp_ulysses_attn_workspace_size(int S, int hq, int hkv, int dh, int P, size_t* bytes);
cp_status cp_ulysses_attn_fwd(const void* q, const void* k, const void* v, int S, int hq, int hkv, int dh, int P,
                              cp_mask mask, float softmax_scale, float* o, float* lse, void* workspace,
                              size_t ws_bytes, void* stream);

/*
 * cp_usp_attn_workspace_size / cp_usp_attn_fwd -- the two-dimensional hybrid
 * of the two methods: P = Pr * Pu virtual ranks, DeepSpeed-Ulysses inside
 * each group of Pu ranks and Ring Attention across the Pr groups ("序列並行"
 * concept page (compassingai), closing section: Ulysses all-to-all inside the
 * NVLink domain, Ring P2P across it, which lifts the head-count limit;
 * "Context Parallelism" write-up (pwwt.cn) §6: Ulysses head regrouping inside
 * the CP group, then the Ring passes the sequence).
 *
 * Layout: group g is ring shard g of `layout` over Pr ranks (contiguous,
 * zigzag or striped, exactly the rank-major buffer cp_ring_attn_fwd takes
 * with P = Pr); its S/Pr rows are split into Pu consecutive sub-shards, sub-
 * rank u of group g being rank g*Pu + u.  Inputs q [S][hq][dh], k, v
 * [S][hkv][dh] bf16 in that storage order; outputs o [S][hq][dh] fp32 and
 * lse [hq][S] fp32 in the same order (row i of o is row i of q).
 *
 * Steps: Ulysses seq->head transpose of Q, K, V over Pu (every group at
 * once); one attention launch for every live ring block pair of every head
 * block (the ring schedule of cp_ring_attn_fwd with P = Pr); one merge launch
 * that folds each head block's partials and writes them directly as heads
 * [u*hq/Pu, (u+1)*hq/Pu) of o and lse, which is the head->seq transpose.
 *
 * Workspace (caller-owned, 256-byte aligned, size from
 * cp_usp_attn_workspace_size with the same arguments): head-major bf16 copies
 * of Q, K, V plus Pu sets of ring partials.
 * Supported: Pu | hkv (KV heads are not replicated), 1 <= Pr <= 16,
 * S % (Pr*Pu) == 0 (and S % (2*Pr) == 0 for zigzag), dh in {64, 128}; documents
 * (cu_seqlens, as for cp_ring_attn_fwd) with the contiguous and zigzag
 * layouts.  Errors as for cp_ring_attn_fwd; nothing is launched on error.
 */
cp_status cp_usp_attn_workspace_size(int S, int hq, int hkv, int dh, int Pr, int Pu, cp_layout layout, cp_mask mask,
                                     const int32_t* cu_seqlens_host, int n_docs, size_t* bytes);
cp_status cp_usp_attn_fwd(const void* q, const void* k, const void* v, int S, int hq, int hkv, int dh, int Pr, int Pu,
                          cp_layout layout, cp_mask mask, const int32_t* cu_seqlens_host,
                          const int32_t* cu_seqlens_dev, int n_docs, float softmax_scale, float* o, float* lse,
                          void* workspace, size_t ws_bytes, void* stream);

/*
 * cp_ring_attn_bwd_workspace_size / cp_ring_attn_bwd -- gradients of the ring
 * attention forward (cp_ring_attn_fwd) for an upstream gradient dO.  The pages
 * define the forward; training also runs the backward (the DeepSpeed-Ulysses /
 * ring-flash-attention how-to (2kiu.com), §4, checks memory after forward and
 * backward), and this is the gradient of that exact attention in ring form:
 * at step t rank r holds key/value shard j = (r - t) mod P and, with the
 * forward's merged LSE_r and D_r = rowsum(dO_r * O_r),
 *   P_rj = exp(scale Q_r K_j^T - LSE_r),  dS_rj = P_rj * (dO_r V_j^T - D_r),
 *   dQ_r += scale dS_rj K_j,  dK_j += scale dS_rj^T Q_r,  dV_j += P_rj^T dO_r
 * (masks by global position as in the forward; the LSE merge needs no
 * separate backward because P_rj already uses the merged LSE).
 *
 * Inputs (device, in the rank-major order of `layout`, as given to and
 * returned by cp_ring_attn_fwd): q [S][hq][dh], k, v [S][hkv][dh] bf16;
 * o [S][hq][dh] fp32 and lse [hq][S] fp32 from the forward; dout [S][hq][dh]
 * bf16.  Outputs (device, same order, fp32, fully overwritten): dq
 * [S][hq][dh], dk and dv [S][hkv][dh].  GQA sums dk, dv over the query heads
 * of each KV head.
 *
 * Runs a prep kernel (D and LSE*log2(e) into the workspace), a dQ kernel and
 * a dK/dV kernel (tcgen05, accumulators in tensor memory, no atomics; the
 * result does not depend on the launch order).  Workspace: caller-owned,
 * 256-byte aligned, size from cp_ring_attn_bwd_workspace_size.
 * Supported: bf16 only, everything else as cp_ring_attn_fwd.  Errors: as
 * cp_ring_attn_fwd; nothing is launched on error.
 */
cp_status cp_ring_attn_bwd_workspace_size(int S, int hq, int hkv, int dh, int P, cp_layout layout, cp_mask mask,
                                          const int32_t* cu_seqlens_host, int n_docs, size_t* bytes);
cp_status cp_ring_attn_bwd(const void* q, const void* k, const void* v, const float* o, const float* lse,
                           const void* dout, int S, int hq, int hkv, int dh, int P, cp_layout layout, cp_mask mask,
                           const int32_t* cu_seqlens_host, const int32_t* cu_seqlens_dev, int n_docs,
                           float softmax_scale, float* dq, float* dk, float* dv, void* workspace, size_t ws_bytes,
                           void* stream);

/*
 * cp_attn_bwd_prep -- the per-row vectors of the backward for n query rows:
 *   lg[h][i] = LSE[h][i] * log2(e)  (0 where LSE = -inf: the row saw no key),
 *   dd[h][i] = sum_c dO[i][h][c] * O[i][h][c]   (D of the gradient of softmax).
 *   o     [n][hq][dh] fp32 and lse [hq][n] fp32: the forward's merged result
 *   dout  [n][hq][dh] bf16, the upstream gradient
 *   lg, dd  out, [hq][n] fp32 (caller-owned device buffers)
 * Supported: dh in {64, 128}, 1 <= n < 2^30.  Errors: CP_ERR_INVALID_ARG /
 * CP_ERR_ALIGNMENT for NULL or unaligned pointers; nothing launched on error.
 *
 * cp_block_attn_bwd -- the gradient contribution of one block pair: the
 * query rows of one rank against one key/value shard, with the merged LSE of
 * those query rows, i.e. one step of the ring backward of cp_ring_attn_bwd
 * (the step a rank takes between two exchanges of the travelling K/V and
 * dK/dV when the ranks are separate GPUs):
 *   P  = exp(scale Q K^T - LSE) over the admitted (q, k) pairs (0 elsewhere),
 *   dS = P * (dO V^T - D),
 *   dq (+)= scale dS K,   dk (+)= scale dS^T Q,   dv (+)= P^T dO.
 * The admitted pairs follow the chunk positions, mask and documents exactly as
 * in cp_block_attn_fwd (a striped key shift belongs in k_chunks).
 *   q, dout      [n_q][hq][dh] bf16;  k, v [n_k][hkv][dh] bf16
 *   lg, dd       [hq][n_q] fp32 from cp_attn_bwd_prep on the same rows
 *   q_chunks, k_chunks  host, 1..CP_BWD_MAX_CHUNKS entries per side covering
 *                the rows in order
 *   parts        CP_BWD_DQ, CP_BWD_DKDV or both: which outputs to compute
 *                (the dQ kernel and the dK/dV kernel, one launch each)
 *   accumulate   0: dq (or dk, dv) are overwritten, rows with no admitted
 *                pair get 0; 1: the contribution is added to what they hold
 *   dq           [n_q][hq][dh] fp32 (may be NULL without CP_BWD_DQ)
 *   dk, dv       [n_k][hkv][dh] fp32, summed over the query heads of each KV
 *                head (may be NULL without CP_BWD_DKDV)
 * The pages define only the forward; this is the gradient of its exact
 * attention, in the ring form the LSE merge of the "序列並行" concept page
 * (compassingai), 技術原理 §二, leads to when differentiated.  No atomics:
 * each output row is written by one CTA, so concurrent calls on different
 * streams must not share an output buffer.  Supported: dh in {64, 128},
 * hq % hkv == 0, 1 <= n_q, n_k < 2^30.  Errors as cp_block_attn_fwd;
 * nothing is launched on error.
 */
#define CP_BWD_DQ 1
#define CP_BWD_DKDV 2
#define CP_BWD_MAX_CHUNKS 2
cp_status cp_attn_bwd_prep(const float* o, const void* dout, const float* lse, int n, int hq, int dh, float* lg,
                           float* dd, void* stream);
cp_status cp_block_attn_bwd(const void* q, const void* k, const void* v, const void* dout, const float* lg,
                            const float* dd, int n_q, int n_k, int hq, int hkv, int dh, const cp_chunk* q_chunks,
                            int nq_chunks, const cp_chunk* k_chunks, int nk_chunks, cp_mask mask,
                            const int32_t* cu_seqlens_dev, int n_docs, float softmax_scale, float* dq, float* dk,
                            float* dv, int parts, int accumulate, void* stream);

/*
 * cp_usp_attn_bwd_workspace_size / cp_usp_attn_bwd -- gradients of
 * cp_usp_attn_fwd (the Ulysses-inside / Ring-across hybrid) for an upstream
 * gradient dO, with the same rank grid, layouts and support as the forward.
 * Inputs (device, in the forward's storage order): q [S][hq][dh], k, v
 * [S][hkv][dh], dout [S][hq][dh] bf16; o [S][hq][dh] fp32 and lse [hq][S]
 * fp32 from the forward.  Outputs (fp32, fully overwritten, same order): dq
 * [S][hq][dh], dk and dv [S][hkv][dh].
 * Steps: Ulysses seq->head transpose of Q, K, V and dO over Pu; for every
 * head block, the ring backward of cp_ring_attn_bwd over the Pr groups (one
 * dQ launch and one dK/dV launch cover all head blocks); the kernels read O
 * and LSE and write dq, dk, dv directly in the final layouts, which is the
 * head->seq transpose of the gradients.
 * Workspace: caller-owned, 256-byte aligned, size from
 * cp_usp_attn_bwd_workspace_size (head-major Q, dO, K, V and two fp32
 * [hq][S] vectors).  Errors as cp_usp_attn_fwd; nothing is launched on error.
 */
cp_status cp_usp_attn_bwd_workspace_size(int S, int hq, int hkv, int dh, int Pr, int Pu, cp_layout layout,
                                         cp_mask mask, const int32_t* cu_seqlens_host, int n_docs, size_t* bytes);
cp_status cp_usp_attn_bwd(const void* q, const void* k, const void* v, const float* o, const float* lse,
                          const void* dout, int S, int hq, int hkv, int dh, int Pr, int Pu, cp_layout layout,
                          cp_mask mask, const int32_t* cu_seqlens_host, const int32_t* cu_seqlens_dev, int n_docs,
                          float softmax_scale, float* dq, float* dk, float* dv, void* workspace, size_t ws_bytes,
                          void* stream);

/*
 * cp_ulysses_attn_bwd_workspace_size / cp_ulysses_attn_bwd -- gradients of
 * cp_ulysses_attn_fwd: the hybrid backward with Pr = 1 and Pu = P (every
 * rank's head group attends over the whole sequence).  Inputs and outputs
 * in the forward's natural sequence order, dtypes as cp_usp_attn_bwd.
 * Supported: P | hkv, P | S, dh in {64, 128}.
 */
cp_status cp_ulysses_attn_bwd_workspace_size(int S, int hq, int hkv, int dh, int P, size_t* bytes);
cp_status cp_ulysses_attn_bwd(const void* q, const void* k, const void* v, const float* o, const float* lse,
                              const void* dout, int S, int hq, int hkv, int dh, int P, cp_mask mask,
                              float softmax_scale, float* dq, float* dk, float* dv, void* workspace, size_t ws_bytes,
                              void* stream);

/*
 * Host-only inspection of the ring-step schedule (no GPU needed).  For every
 * rank r and step t (index r*P + t):
 *   src[r*P+t]        the key/value shard j = (r - t) mod P held at that step
 *   launched[r*P+t]   1 if the block pair is computed, 0 if skipped as empty
 *   q_rows[r*P+t]     query rows of the pair that are computed
 *   live_pairs[r*P+t] number of admitted (query, key) pairs in the block pair
 * Any output pointer may be NULL.  cu_seqlens_host as in cp_ring_attn_fwd.
 */
cp_status cp_ring_schedule(int S, int P, cp_layout layout, cp_mask mask, const int32_t* cu_seqlens_host,
                           int n_docs, int32_t* src, int32_t* launched, int32_t* q_rows, int64_t* live_pairs);

/* Number of admitted (query, key) pairs of the whole sequence: the unit of
 * the causal-effective FLOP count 4 * dh * hq * pairs.  Host only. */
cp_status cp_count_live_pairs(int S, cp_mask mask, const int32_t* cu_seqlens_host, int n_docs, int64_t* pairs);

/* Self-test of failure detection: launches one CTA that waits on a barrier
 * nothing ever arrives on.  The bounded wait gives up after timeout_ns
 * (0 < timeout_ns <= 10 s), sets bit 0 of the device error word (read it with
 * cp_device_error after synchronising) and returns; the CUDA context stays
 * usable.  Used by the tests; the pages have no counterpart. */
cp_status cp_selftest_wait_timeout(uint64_t timeout_ns, void* stream);

/* Reads (and, if clear != 0, resets) the device error word of the current
 * device: 0 = no kernel gave up waiting; bit 0 = a bounded wait timed out.
 * Synchronous. */
cp_status cp_device_error(uint32_t* bits, int clear);

/*
 * cp_ring_attn_fwd_noalloc -- cp_ring_attn_fwd for callers that may not
 * allocate device memory (for example a plugin whose host application owns
 * the whole device-memory budget and forbids allocation while it runs, or a
 * latency-critical loop in which an allocation would stall the device).  The
 * pages have no counterpart: this is a property of the library, not of the
 * method.
 *
 * Same arguments and results as cp_ring_attn_fwd, without the workspace: the
 * partial results live in a scratch array of CP_NOALLOC_SCRATCH_BYTES bytes
 * compiled into the library, which every GPU that uses the library keeps
 * until the process exits.  The call allocates nothing.
 *  - Problems whose cp_ring_attn_workspace_size exceeds the scratch are
 *    rejected with CP_ERR_WORKSPACE and a message giving both sizes.
 *  - The first call on each device looks up the scratch address of that
 *    device (cudaGetSymbolAddress); make that first call before any stream
 *    capture begins.  The address is kept for the life of the process, so
 *    the entry point must not be used after cudaDeviceReset (or any other
 *    teardown of the device's primary context) in the same process.
 *  - All calls share the one scratch array per device and it keeps whatever
 *    the last call left there.  Calls whose GPU work overlaps in time (on
 *    different streams, or from different threads) race on it: order them on
 *    one stream or synchronise between them.
 */
#define CP_NOALLOC_SCRATCH_BYTES ((size_t)64 << 20)
cp_status cp_ring_attn_fwd_noalloc(const void* q, const void* k, const void* v, cp_dtype dtype, int S, int hq,
                                   int hkv, int dh, int P, cp_layout layout, cp_mask mask,
                                   const int32_t* cu_seqlens_host, const int32_t* cu_seqlens_dev, int n_docs,
                                   float softmax_scale, float* o, float* lse, void* stream);

/* Total number of kernels this library has launched in the process (all
 * devices, all threads).  Host only. */
cp_status cp_kernel_launch_count(uint64_t* count);

/* Profiling hook: when non-NULL, the composite calls (cp_ring_attn_fwd,
 * cp_ulysses_attn_fwd, cp_usp_attn_fwd) made afterwards on the calling thread
 * record `attn_begin` / `attn_end` (cudaEvent_t passed as void*) on their
 * stream immediately before their first and after their last block-attention
 * launch, and `merge_end` after their last merge launch.  cp_ring_attn_bwd
 * records `attn_begin` before its dQ kernel, `merge_end` between the dQ and
 * the dK/dV kernels, and `attn_end` after the dK/dV kernel.  Pass NULLs to
 * turn it off. */
cp_status cp_set_profile_events(void* attn_begin, void* attn_end, void* merge_end);

#ifdef __cplusplus
}
#endif

#endif /* CP_ATTN_H */
