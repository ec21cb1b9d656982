// C ABI of the library (see include/cp_attn.h): argument validation, TMA
// tensor maps, the ring / Ulysses / hybrid composites forward and backward,
// the block-pair entry points and the host-only schedule queries.  Host code
// only; the kernels live in attn_fwd.cu, attn_bwd.cu, merge.cu and
// permute.cu.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <climits>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#include "cp_attn.h"
#include "plan.h"
#include "scheduler.h"

namespace cp {
cudaError_t launch_attn(int dh, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                        const cp_attn_plan& plan, cudaStream_t stream);
cudaError_t attn_err_word(uint32_t** dev_ptr);
cudaError_t launch_merge(const cp_merge_plan& plan, int total_ctas, cudaStream_t stream);
int merge_task_ctas(int rows, int h);
cudaError_t launch_ulysses(const void* in, void* out, int P, int n, size_t chunk_bytes, int dir, cudaStream_t st);
cudaError_t launch_zigzag(const void* in, void* out, int P, int batch, size_t chunk_bytes, int inverse,
                          cudaStream_t st);
cudaError_t launch_f32_to_bf16(const float* in, void* out, size_t n, cudaStream_t st);
cudaError_t launch_head_blocks(const void* in, void* out, int P, int n, size_t chunk_bytes, int inverse,
                               cudaStream_t st);
cudaError_t launch_striped(const void* in, void* out, int P, int S, int batch, size_t row_bytes, int inverse,
                           cudaStream_t st);
cudaError_t launch_bwd_prep(int dh, const float* o, const void* dout, const float* lse, int G, int hg, int groups,
                            float* lg, float* dd, cudaStream_t st);
cudaError_t launch_bwd(int dh, const CUtensorMap& tq, const CUtensorMap& tdo, const CUtensorMap& tk,
                       const CUtensorMap& tv, const cp_bwd_plan& plan, bool dq_side, cudaStream_t st);
std::atomic<uint64_t>& launch_counter();
}  // namespace cp

namespace {
thread_local std::string g_err;
}  // namespace

namespace cp {
// Lets other translation units of the library report an error message.
void set_error_message(const char* msg) { g_err = msg ? msg : ""; }
}  // namespace cp

using namespace cp;

namespace {

thread_local cudaEvent_t g_ev_attn_begin = nullptr, g_ev_attn_end = nullptr, g_ev_merge_end = nullptr;

void record(cudaEvent_t ev, cudaStream_t st) {
  if (ev) cudaEventRecord(ev, st);
}

cp_status fail(cp_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_err = buf;
  return s;
}

cp_status ok() {
  g_err.clear();
  return CP_OK;
}

cp_status cuda_fail(cudaError_t e, const char* what) {
  return fail(CP_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

#define CP_CHECK_PTR(p)                                                             \
  do {                                                                              \
    if (!(p)) return fail(CP_ERR_INVALID_ARG, "%s is NULL", #p);                   \
    if (!aligned16(p)) return fail(CP_ERR_ALIGNMENT, "%s is not 16-byte aligned", #p); \
  } while (0)

// --------------------------------------------------------------- TMA maps
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// bf16 matrix of `rows` rows x `row_elems` elements, box_rows-row x 64-column
// boxes with 128-byte swizzle (the canonical K-major tcgen05 operand layout).
cp_status make_map(CUtensorMap* m, const void* base, int64_t rows, int64_t row_elems, uint32_t box_rows) {
  auto fn = encode_fn();
  if (!fn) return fail(CP_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  cuuint64_t dims[2] = {(cuuint64_t)row_elems, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)row_elems * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(CP_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return CP_OK;
}

// --------------------------------------------------------------- error word
cp_status err_word(uint32_t** p) {
  static uint32_t* words[64] = {nullptr};
  static std::mutex mu;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= 64) return fail(CP_ERR_UNSUPPORTED, "device index %d", dev);
  std::lock_guard<std::mutex> lk(mu);
  if (!words[dev]) {
    e = attn_err_word(&words[dev]);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(error word)");
  }
  *p = words[dev];
  return CP_OK;
}

// --------------------------------------------------------------- attention
struct PairIn {
  std::vector<Seg> q, k;
  int qtiles;
  float* o;
  float* lse;
  int lse_ld;
  bool reverse;
  int block = 0;  // pairs with equal block read the same Q/K/V rows (cp_attn_plan)
};

cp_status run_pairs(const void* q, const void* k, const void* v, int64_t q_rows, int64_t k_rows, int hq, int hkv,
                    int dh, bool causal, const int32_t* cu_dev, int n_docs, float scale,
                    const std::vector<PairIn>& pairs, cudaStream_t st) {
  CUtensorMap tq, tk, tv;
  cp_status s;
  // query boxes: one 128-row MMA tile; key/value boxes: one CP_KV_TILE-row tile
  if ((s = make_map(&tq, q, q_rows, (int64_t)hq * dh, 128)) != CP_OK) return s;
  if ((s = make_map(&tk, k, k_rows, (int64_t)hkv * dh, CP_KV_TILE)) != CP_OK) return s;
  if ((s = make_map(&tv, v, k_rows, (int64_t)hkv * dh, CP_KV_TILE)) != CP_OK) return s;
  uint32_t* err = nullptr;
  if ((s = err_word(&err)) != CP_OK) return s;

  // Pairs of one block run together (stable: the heaviest-first order of the
  // caller is kept inside each block).
  std::vector<const PairIn*> order;
  order.reserve(pairs.size());
  for (const PairIn& pi : pairs) order.push_back(&pi);
  std::stable_sort(order.begin(), order.end(), [](const PairIn* a, const PairIn* b) { return a->block < b->block; });

  static cp_attn_plan plan;  // large POD: keep it off the stack
  static std::mutex plan_mu;
  std::lock_guard<std::mutex> lk(plan_mu);
  size_t i = 0;
  while (i < order.size()) {
    memset(&plan, 0, sizeof(plan));
    plan.hq = hq;
    plan.hkv = hkv;
    plan.causal = causal ? 1 : 0;
    plan.n_docs = n_docs;
    plan.cu_seqlens = cu_dev;
    plan.scale_log2 = scale * 1.4426950408889634f;
    plan.err = err;
    int ctas = 0, qt = 0;
    int cur_block = -1;
    // fill one launch: at most CP_MAX_PAIRS pairs in at most CP_MAX_BLOCKS blocks
    while (i < order.size() && plan.n_pairs < CP_MAX_PAIRS) {
      const PairIn& pi = *order[i];
      if (pi.block != cur_block) {
        if (plan.n_blocks == CP_MAX_BLOCKS) break;
        if (plan.n_blocks > 0) ctas += qt * hq;  // close the previous block
        plan.blk_cta_begin[plan.n_blocks] = ctas;
        plan.blk_pair_begin[plan.n_blocks] = plan.n_pairs;
        ++plan.n_blocks;
        cur_block = pi.block;
        qt = 0;
      }
      cp_pair_desc& d = plan.pairs[plan.n_pairs++];
      d.nq = (int)pi.q.size();
      d.nk = (int)pi.k.size();
      for (int x = 0; x < d.nq; ++x) d.q[x] = {pi.q[x].buf_row, pi.q[x].pos, pi.q[x].len, pi.q[x].out_row};
      for (int x = 0; x < d.nk; ++x) d.k[x] = {pi.k[x].buf_row, pi.k[x].pos, pi.k[x].len, 0};
      d.qtiles = pi.qtiles;
      d.qt_begin = qt;
      d.reverse = pi.reverse ? 1 : 0;
      d.lse_ld = pi.lse_ld;
      d.o = pi.o;
      d.lse = pi.lse;
      qt += pi.qtiles;
      plan.blk_qtiles[plan.n_blocks - 1] = qt;
      ++i;
    }
    ctas += qt * hq;
    plan.blk_cta_begin[plan.n_blocks] = ctas;
    plan.blk_pair_begin[plan.n_blocks] = plan.n_pairs;
    plan.total_ctas = ctas;
    cudaError_t e = launch_attn(dh, tq, tk, tv, plan, st);
    if (e != cudaSuccess) return cuda_fail(e, "attention launch");
  }
  return CP_OK;
}

int qtiles_of(const std::vector<Seg>& q) {
  int t = 0;
  for (const Seg& s : q) t += (s.len + CP_Q_TILE - 1) / CP_Q_TILE;
  return t;
}

cp_status check_docs_host(const int32_t* cu, int n_docs, int S) {
  if (n_docs < 0) return fail(CP_ERR_INVALID_ARG, "n_docs < 0");
  if (n_docs == 0) return CP_OK;
  if (!cu) return CP_OK;
  if (cu[0] != 0) return fail(CP_ERR_INVALID_ARG, "cu_seqlens[0] must be 0");
  for (int i = 0; i < n_docs; ++i)
    if (cu[i + 1] <= cu[i]) return fail(CP_ERR_INVALID_ARG, "cu_seqlens must be strictly increasing");
  if (cu[n_docs] != S) return fail(CP_ERR_INVALID_ARG, "cu_seqlens[n_docs] = %d, expected S = %d", cu[n_docs], S);
  return CP_OK;
}

cp_status check_common(int hq, int hkv, int dh) {
  if (dh != 64 && dh != 128) return fail(CP_ERR_UNSUPPORTED, "dh = %d (supported: 64, 128)", dh);
  if (hq <= 0 || hkv <= 0) return fail(CP_ERR_INVALID_ARG, "head counts must be positive");
  if (hq % hkv != 0) return fail(CP_ERR_INVALID_ARG, "hq (%d) must be a multiple of hkv (%d)", hq, hkv);
  return CP_OK;
}

struct Merge {
  const float* o;
  const float* lse;
  int row0;
  int lse_ld;
};
struct MergeTaskIn {
  int out_row0, rows;
  int head_off = 0;
  std::vector<Merge> in;
};

// o_heads: heads per output row of O (h unless tasks scatter head blocks
// into a wider output through head_off).
cp_status run_merge(const std::vector<MergeTaskIn>& tasks_in, int h, int dh, float* o_out, float* lse_out,
                    int lse_out_ld, void* o_bf16, cudaStream_t st, int o_heads = 0) {
  static cp_merge_plan plan;
  static std::mutex mu;
  std::lock_guard<std::mutex> lk(mu);
  // Tasks with more partials per row first: CTAs start in task order and a
  // CTA's time grows with its task's partial count, so the slow CTAs do not
  // form the tail of the launch.
  std::vector<const MergeTaskIn*> order;
  order.reserve(tasks_in.size());
  for (const MergeTaskIn& t : tasks_in) order.push_back(&t);
  std::stable_sort(order.begin(), order.end(), [](const MergeTaskIn* a, const MergeTaskIn* b) {
    return a->in.size() > b->in.size();
  });
  std::vector<MergeTaskIn> tasks;
  tasks.reserve(order.size());
  for (const MergeTaskIn* t : order) tasks.push_back(*t);
  size_t i = 0;
  while (i < tasks.size()) {
    memset(&plan, 0, sizeof(plan));
    plan.h = h;
    plan.dh = dh;
    plan.lse_out_ld = lse_out_ld;
    plan.o_heads = o_heads > 0 ? o_heads : h;
    plan.o_out = o_out;
    plan.lse_out = lse_out;
    plan.o_out_bf16 = static_cast<uint16_t*>(o_bf16);
    int n_in = 0;
    long long ctas = 0;
    while (i < tasks.size() && plan.n_tasks < CP_MAX_TASKS &&
           n_in + (int)tasks[i].in.size() <= CP_MAX_INPUTS) {
      const MergeTaskIn& t = tasks[i];
      const long long task_ctas = merge_task_ctas(t.rows, h);
      if (ctas + task_ctas > INT32_MAX) break;
      cp_merge_task& d = plan.tasks[plan.n_tasks++];
      d.out_row0 = t.out_row0;
      d.rows = t.rows;
      d.n_in = (int)t.in.size();
      d.in_begin = n_in;
      d.head_off = t.head_off;
      d.cta_begin = (int)ctas;
      for (const Merge& m : t.in) plan.inputs[n_in++] = {m.o, m.lse, m.row0, m.lse_ld};
      ctas += task_ctas;
      ++i;
    }
    if (plan.n_tasks == 0) return fail(CP_ERR_UNSUPPORTED, "merge task with more than %d inputs", CP_MAX_INPUTS);
    cudaError_t e = launch_merge(plan, (int)ctas, st);
    if (e != cudaSuccess) return cuda_fail(e, "merge launch");
  }
  return CP_OK;
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

}  // namespace

extern "C" {

const char* cp_last_error_string(void) { return g_err.c_str(); }

const char* cp_version(void) { return "cp_attn 0.1 (sm_100a)"; }

cp_status cp_block_attn_fwd(const void* q, const void* k, const void* v, cp_dtype dtype, int n_q, int n_k, int hq,
                            int hkv, int dh, const cp_chunk* q_chunks, int nq_chunks, const cp_chunk* k_chunks,
                            int nk_chunks, cp_mask mask, const int32_t* cu_seqlens_dev, int n_docs,
                            float softmax_scale, float* o, float* lse, void* stream) {
  cp_status s;
  if ((s = check_common(hq, hkv, dh)) != CP_OK) return s;
  if (dtype != CP_BF16) return fail(CP_ERR_UNSUPPORTED, "cp_block_attn_fwd takes bf16 inputs");
  if (n_q <= 0 || n_k <= 0 || n_q >= (1 << 30) || n_k >= (1 << 30))
    return fail(CP_ERR_INVALID_ARG, "n_q, n_k must be in [1, 2^30)");
  CP_CHECK_PTR(q);
  CP_CHECK_PTR(k);
  CP_CHECK_PTR(v);
  CP_CHECK_PTR(o);
  CP_CHECK_PTR(lse);
  if (mask != CP_MASK_NONE && mask != CP_MASK_CAUSAL) return fail(CP_ERR_INVALID_ARG, "unknown mask %d", (int)mask);
  if (!q_chunks || !k_chunks) return fail(CP_ERR_INVALID_ARG, "chunk lists are NULL");
  if (nq_chunks < 1 || nq_chunks > CP_MAX_CHUNKS || nk_chunks < 1 || nk_chunks > CP_MAX_CHUNKS)
    return fail(CP_ERR_UNSUPPORTED, "1..%d chunks per side", CP_MAX_CHUNKS);
  if (n_docs < 0 || (n_docs > 0 && !cu_seqlens_dev))
    return fail(CP_ERR_INVALID_ARG, "n_docs > 0 needs cu_seqlens_dev");
  PairIn pi;
  int rows = 0;
  for (int i = 0; i < nq_chunks; ++i) {
    if (q_chunks[i].len <= 0 || q_chunks[i].start < 0) return fail(CP_ERR_INVALID_ARG, "bad q chunk %d", i);
    pi.q.push_back({rows, q_chunks[i].start, q_chunks[i].len, rows});
    rows += q_chunks[i].len;
  }
  if (rows != n_q) return fail(CP_ERR_INVALID_ARG, "q chunks cover %d rows, n_q = %d", rows, n_q);
  rows = 0;
  for (int i = 0; i < nk_chunks; ++i) {
    if (k_chunks[i].len <= 0 || k_chunks[i].start < 0) return fail(CP_ERR_INVALID_ARG, "bad k chunk %d", i);
    pi.k.push_back({rows, k_chunks[i].start, k_chunks[i].len, 0});
    rows += k_chunks[i].len;
  }
  if (rows != n_k) return fail(CP_ERR_INVALID_ARG, "k chunks cover %d rows, n_k = %d", rows, n_k);
  pi.qtiles = qtiles_of(pi.q);
  pi.o = o;
  pi.lse = lse;
  pi.lse_ld = n_q;
  pi.reverse = mask == CP_MASK_CAUSAL;
  const float scale = softmax_scale > 0.f ? softmax_scale : 1.0f / std::sqrt((float)dh);
  std::vector<PairIn> pairs{pi};
  if ((s = run_pairs(q, k, v, n_q, n_k, hq, hkv, dh, mask == CP_MASK_CAUSAL, cu_seqlens_dev, n_docs, scale, pairs,
                     static_cast<cudaStream_t>(stream))) != CP_OK)
    return s;
  return ok();
}

cp_status cp_lse_merge(int n_parts, const float* const* o_parts, const float* const* lse_parts, int rows, int h,
                       int dh, float* o_out, float* lse_out, void* o_out_bf16, void* stream) {
  if (n_parts < 1 || n_parts > 64) return fail(CP_ERR_UNSUPPORTED, "n_parts = %d (supported 1..64)", n_parts);
  if (dh != 64 && dh != 128) return fail(CP_ERR_UNSUPPORTED, "dh = %d (supported: 64, 128)", dh);
  if (rows <= 0 || h <= 0) return fail(CP_ERR_INVALID_ARG, "rows and h must be positive");
  if (!o_parts || !lse_parts) return fail(CP_ERR_INVALID_ARG, "part lists are NULL");
  CP_CHECK_PTR(o_out);
  CP_CHECK_PTR(lse_out);
  if (o_out_bf16 && !aligned16(o_out_bf16)) return fail(CP_ERR_ALIGNMENT, "o_out_bf16 is not 16-byte aligned");
  MergeTaskIn t;
  t.out_row0 = 0;
  t.rows = rows;
  for (int i = 0; i < n_parts; ++i) {
    if (!o_parts[i] || !lse_parts[i]) return fail(CP_ERR_INVALID_ARG, "part %d is NULL", i);
    if (!aligned16(o_parts[i])) return fail(CP_ERR_ALIGNMENT, "o_parts[%d] is not 16-byte aligned", i);
    if (o_parts[i] == o_out) return fail(CP_ERR_INVALID_ARG, "o_out aliases o_parts[%d]", i);
    t.in.push_back({o_parts[i], lse_parts[i], 0, rows});
  }
  std::vector<MergeTaskIn> tasks{t};
  cp_status s = run_merge(tasks, h, dh, o_out, lse_out, rows, o_out_bf16, static_cast<cudaStream_t>(stream));
  if (s != CP_OK) return s;
  return ok();
}

static cp_status ring_check(int S, int hq, int hkv, int dh, int P, cp_layout layout, cp_mask mask, cp_dtype dtype,
                            const int32_t* cu_host, int n_docs) {
  cp_status s;
  if ((s = check_common(hq, hkv, dh)) != CP_OK) return s;
  if (P < 1 || P > 16) return fail(CP_ERR_UNSUPPORTED, "P = %d (supported 1..16)", P);
  if (S <= 0 || S >= (1 << 30)) return fail(CP_ERR_INVALID_ARG, "S = %d", S);
  if (layout != CP_LAYOUT_CONTIGUOUS && layout != CP_LAYOUT_ZIGZAG && layout != CP_LAYOUT_STRIPED)
    return fail(CP_ERR_INVALID_ARG, "unknown layout %d", (int)layout);
  if (layout == CP_LAYOUT_STRIPED && n_docs > 0)
    return fail(CP_ERR_UNSUPPORTED, "the striped layout does not take a document mask");
  if (mask != CP_MASK_NONE && mask != CP_MASK_CAUSAL) return fail(CP_ERR_INVALID_ARG, "unknown mask %d", (int)mask);
  if (dtype != CP_BF16 && dtype != CP_FP32) return fail(CP_ERR_INVALID_ARG, "unknown dtype %d", (int)dtype);
  const int div = layout == CP_LAYOUT_ZIGZAG ? 2 * P : P;
  if (S % div != 0) return fail(CP_ERR_INVALID_ARG, "S = %d is not a multiple of %d", S, div);
  return check_docs_host(cu_host, n_docs, S);
}

static RingPlan make_ring_plan(int S, int hq, int dh, int P, cp_layout layout, cp_mask mask,
                               const int32_t* cu_host, int n_docs) {
  Docs docs;
  if (cu_host && n_docs > 0) {
    docs.cu = cu_host;
    docs.n = n_docs;
  }
  const Layout lay = layout == CP_LAYOUT_ZIGZAG ? Layout::Zigzag
                     : layout == CP_LAYOUT_STRIPED ? Layout::Striped
                                                   : Layout::Contiguous;
  return build_ring_plan(S, P, lay, mask == CP_MASK_CAUSAL, docs, hq, dh);
}

cp_status cp_ring_attn_workspace_size(int S, int hq, int hkv, int dh, int P, cp_layout layout, cp_mask mask,
                                      cp_dtype dtype, const int32_t* cu_seqlens_host, int n_docs, size_t* bytes) {
  cp_status s;
  if (!bytes) return fail(CP_ERR_INVALID_ARG, "bytes is NULL");
  if ((s = ring_check(S, hq, hkv, dh, P, layout, mask, dtype, cu_seqlens_host, n_docs)) != CP_OK) return s;
  RingPlan plan = make_ring_plan(S, hq, dh, P, layout, mask, cu_seqlens_host, n_docs);
  size_t b = plan.partial_bytes;
  if (dtype == CP_FP32)
    b += align256((size_t)S * hq * dh * 2) + 2 * align256((size_t)S * hkv * dh * 2);
  *bytes = b;
  return ok();
}

cp_status cp_ring_attn_fwd(const void* q, const void* k, const void* v, cp_dtype dtype, int S, int hq, int hkv,
                           int dh, int P, cp_layout layout, cp_mask mask, const int32_t* cu_seqlens_host,
                           const int32_t* cu_seqlens_dev, int n_docs, float softmax_scale, float* o, float* lse,
                           void* workspace, size_t ws_bytes, void* stream) {
  cp_status s;
  if ((s = ring_check(S, hq, hkv, dh, P, layout, mask, dtype, cu_seqlens_host, n_docs)) != CP_OK) return s;
  CP_CHECK_PTR(q);
  CP_CHECK_PTR(k);
  CP_CHECK_PTR(v);
  CP_CHECK_PTR(o);
  CP_CHECK_PTR(lse);
  if (n_docs > 0 && !cu_seqlens_dev) return fail(CP_ERR_INVALID_ARG, "n_docs > 0 needs cu_seqlens_dev");
  RingPlan plan = make_ring_plan(S, hq, dh, P, layout, mask, cu_seqlens_host, n_docs);
  size_t need = plan.partial_bytes;
  if (dtype == CP_FP32) need += align256((size_t)S * hq * dh * 2) + 2 * align256((size_t)S * hkv * dh * 2);
  if (need > 0 && (!workspace || ws_bytes < need))
    return fail(CP_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", need, ws_bytes);
  if (workspace && (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return fail(CP_ERR_ALIGNMENT, "workspace is not 256-byte aligned");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const void *qb = q, *kb = k, *vb = v;
  size_t off = 0;
  if (dtype == CP_FP32) {
    void* q16 = ws + off;
    off += align256((size_t)S * hq * dh * 2);
    void* k16 = ws + off;
    off += align256((size_t)S * hkv * dh * 2);
    void* v16 = ws + off;
    off += align256((size_t)S * hkv * dh * 2);
    cudaError_t e;
    if ((e = launch_f32_to_bf16(static_cast<const float*>(q), q16, (size_t)S * hq * dh, st)) != cudaSuccess ||
        (e = launch_f32_to_bf16(static_cast<const float*>(k), k16, (size_t)S * hkv * dh, st)) != cudaSuccess ||
        (e = launch_f32_to_bf16(static_cast<const float*>(v), v16, (size_t)S * hkv * dh, st)) != cudaSuccess)
      return cuda_fail(e, "fp32 -> bf16 conversion");
    qb = q16;
    kb = k16;
    vb = v16;
  }
  uint8_t* parts = ws + off;
  std::vector<PairIn> pairs;
  pairs.reserve(plan.pairs.size());
  for (const PairPlan& pp : plan.pairs) {
    PairIn pi;
    pi.q = pp.q;
    pi.k = pp.k;
    pi.qtiles = pp.qtiles;
    pi.o = reinterpret_cast<float*>(parts + pp.o_off);
    pi.lse = reinterpret_cast<float*>(parts + pp.lse_off);
    pi.lse_ld = pp.rows;
    pi.reverse = mask == CP_MASK_CAUSAL;
    pairs.push_back(std::move(pi));
  }
  const float scale = softmax_scale > 0.f ? softmax_scale : 1.0f / std::sqrt((float)dh);
  record(g_ev_attn_begin, st);
  if ((s = run_pairs(qb, kb, vb, S, S, hq, hkv, dh, mask == CP_MASK_CAUSAL, cu_seqlens_dev, n_docs, scale, pairs,
                     st)) != CP_OK)
    return s;
  record(g_ev_attn_end, st);
  std::vector<MergeTaskIn> tasks;
  for (const MergeTaskPlan& tp : plan.tasks) {
    MergeTaskIn t;
    t.out_row0 = tp.row0;
    t.rows = tp.rows;
    for (const auto& in : tp.inputs) {
      const PairPlan& pp = plan.pairs[in.first];
      t.in.push_back({reinterpret_cast<const float*>(parts + pp.o_off),
                      reinterpret_cast<const float*>(parts + pp.lse_off), in.second, pp.rows});
    }
    tasks.push_back(std::move(t));
  }
  if ((s = run_merge(tasks, hq, dh, o, lse, S, nullptr, st)) != CP_OK) return s;
  record(g_ev_merge_end, st);
  return ok();
}

cp_status cp_ulysses_permute(const void* in, void* out, int P, int S, int h, int dh, int elem_bytes, cp_dir dir,
                             void* stream) {
  if (!in || !out) return fail(CP_ERR_INVALID_ARG, "in/out is NULL");
  if (P < 1 || S <= 0 || h <= 0 || dh <= 0) return fail(CP_ERR_INVALID_ARG, "sizes must be positive");
  if (elem_bytes != 1 && elem_bytes != 2 && elem_bytes != 4 && elem_bytes != 8)
    return fail(CP_ERR_INVALID_ARG, "elem_bytes = %d", elem_bytes);
  if (S % P != 0) return fail(CP_ERR_INVALID_ARG, "S = %d is not a multiple of P = %d", S, P);
  if (h % P != 0) return fail(CP_ERR_UNSUPPORTED, "heads (%d) must be a multiple of P (%d)", h, P);
  if (dir != CP_SEQ_TO_HEAD && dir != CP_HEAD_TO_SEQ) return fail(CP_ERR_INVALID_ARG, "unknown direction");
  const size_t bytes = (size_t)S * h * dh * elem_bytes;
  const uint8_t *a = static_cast<const uint8_t*>(in), *b = static_cast<const uint8_t*>(out);
  if (a < b + bytes && b < a + bytes) return fail(CP_ERR_INVALID_ARG, "in and out overlap");
  const size_t chunk = (size_t)(h / P) * dh * elem_bytes;
  cudaError_t e = launch_ulysses(in, out, P, S / P, chunk, dir == CP_SEQ_TO_HEAD ? 0 : 1,
                                 static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "ulysses permute launch");
  return ok();
}

cp_status cp_zigzag_reorder(const void* in, void* out, int P, int S, int batch, int row_bytes, int inverse,
                            void* stream) {
  if (!in || !out) return fail(CP_ERR_INVALID_ARG, "in/out is NULL");
  if (P < 1 || S <= 0 || batch <= 0 || row_bytes <= 0) return fail(CP_ERR_INVALID_ARG, "sizes must be positive");
  if (S % (2 * P) != 0) return fail(CP_ERR_INVALID_ARG, "S = %d is not a multiple of 2P = %d", S, 2 * P);
  const size_t bytes = (size_t)batch * S * row_bytes;
  const uint8_t *a = static_cast<const uint8_t*>(in), *b = static_cast<const uint8_t*>(out);
  if (a < b + bytes && b < a + bytes) return fail(CP_ERR_INVALID_ARG, "in and out overlap");
  const size_t chunk = (size_t)(S / (2 * P)) * row_bytes;
  cudaError_t e = launch_zigzag(in, out, P, batch, chunk, inverse ? 1 : 0, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "zigzag reorder launch");
  return ok();
}

cp_status cp_head_block_split(const void* in, void* out, int n, int h, int dh, int P, int elem_bytes, int inverse,
                              void* stream) {
  if (!in || !out) return fail(CP_ERR_INVALID_ARG, "in/out is NULL");
  if (P < 1 || n <= 0 || h <= 0 || dh <= 0) return fail(CP_ERR_INVALID_ARG, "sizes must be positive");
  if (elem_bytes != 1 && elem_bytes != 2 && elem_bytes != 4 && elem_bytes != 8)
    return fail(CP_ERR_INVALID_ARG, "elem_bytes = %d", elem_bytes);
  if (h % P != 0) return fail(CP_ERR_UNSUPPORTED, "heads (%d) must be a multiple of P (%d)", h, P);
  const size_t bytes = (size_t)n * h * dh * elem_bytes;
  const uint8_t *a = static_cast<const uint8_t*>(in), *b = static_cast<const uint8_t*>(out);
  if (a < b + bytes && b < a + bytes) return fail(CP_ERR_INVALID_ARG, "in and out overlap");
  cudaError_t e = launch_head_blocks(in, out, P, n, (size_t)(h / P) * dh * elem_bytes, inverse ? 1 : 0,
                                     static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "head-block split launch");
  return ok();
}

cp_status cp_striped_reorder(const void* in, void* out, int P, int S, int batch, int row_bytes, int inverse,
                             void* stream) {
  if (!in || !out) return fail(CP_ERR_INVALID_ARG, "in/out is NULL");
  if (P < 1 || S <= 0 || batch <= 0 || row_bytes <= 0) return fail(CP_ERR_INVALID_ARG, "sizes must be positive");
  if (S % P != 0) return fail(CP_ERR_INVALID_ARG, "S = %d is not a multiple of P = %d", S, P);
  const size_t bytes = (size_t)batch * S * row_bytes;
  const uint8_t *a = static_cast<const uint8_t*>(in), *b = static_cast<const uint8_t*>(out);
  if (a < b + bytes && b < a + bytes) return fail(CP_ERR_INVALID_ARG, "in and out overlap");
  cudaError_t e = launch_striped(in, out, P, S, batch, (size_t)row_bytes, inverse ? 1 : 0,
                                 static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "striped reorder launch");
  return ok();
}

cp_status cp_ulysses_attn_workspace_size(int S, int hq, int hkv, int dh, int P, size_t* bytes) {
  cp_status s;
  if (!bytes) return fail(CP_ERR_INVALID_ARG, "bytes is NULL");
  if ((s = check_common(hq, hkv, dh)) != CP_OK) return s;
  if (P < 1 || S <= 0 || S % P != 0) return fail(CP_ERR_INVALID_ARG, "S = %d, P = %d", S, P);
  if (hkv % P != 0) return fail(CP_ERR_UNSUPPORTED, "P (%d) must divide the KV head count (%d)", P, hkv);
  *bytes = align256((size_t)S * hq * dh * 2) + 2 * align256((size_t)S * hkv * dh * 2) +
           align256((size_t)S * hq * dh * 4);
  return ok();
}

cp_status cp_ulysses_attn_fwd(const void* q, const void* k, const void* v, int S, int hq, int hkv, int dh, int P,
                              cp_mask mask, float softmax_scale, float* o, float* lse, void* workspace,
                              size_t ws_bytes, void* stream) {
  size_t need = 0;
  cp_status s = cp_ulysses_attn_workspace_size(S, hq, hkv, dh, P, &need);
  if (s != CP_OK) return s;
  CP_CHECK_PTR(q);
  CP_CHECK_PTR(k);
  CP_CHECK_PTR(v);
  CP_CHECK_PTR(o);
  CP_CHECK_PTR(lse);
  if (mask != CP_MASK_NONE && mask != CP_MASK_CAUSAL) return fail(CP_ERR_INVALID_ARG, "unknown mask %d", (int)mask);
  if (!workspace || ws_bytes < need)
    return fail(CP_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", need, ws_bytes);
  if (reinterpret_cast<uintptr_t>(workspace) & 255u) return fail(CP_ERR_ALIGNMENT, "workspace is not 256-byte aligned");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  size_t off = 0;
  void* qh = ws + off;
  off += align256((size_t)S * hq * dh * 2);
  void* kh = ws + off;
  off += align256((size_t)S * hkv * dh * 2);
  void* vh = ws + off;
  off += align256((size_t)S * hkv * dh * 2);
  float* oh = reinterpret_cast<float*>(ws + off);
  const int n = S / P, hg = hq / P, hkg = hkv / P;
  cudaError_t e;
  if ((e = launch_ulysses(q, qh, P, n, (size_t)hg * dh * 2, 0, st)) != cudaSuccess ||
      (e = launch_ulysses(k, kh, P, n, (size_t)hkg * dh * 2, 0, st)) != cudaSuccess ||
      (e = launch_ulysses(v, vh, P, n, (size_t)hkg * dh * 2, 0, st)) != cudaSuccess)
    return cuda_fail(e, "ulysses seq->head");
  // One pair per head group r: rows [r*S, (r+1)*S) of the head-sharded
  // buffers hold every position of that group's heads.
  std::vector<PairIn> pairs;
  for (int r = 0; r < P; ++r) {
    PairIn pi;
    pi.q.push_back({r * S, 0, S, r * S});
    pi.k.push_back({r * S, 0, S, 0});
    pi.qtiles = qtiles_of(pi.q);
    pi.o = oh;
    // LSE of group r, local head h', position x lives at lse[(r*hg + h')*S + x];
    // the kernel addresses lse[h'*lse_ld + out_row] with out_row = r*S + x.
    pi.lse = lse + (ptrdiff_t)r * hg * S - (ptrdiff_t)r * S;
    pi.lse_ld = S;
    pi.reverse = mask == CP_MASK_CAUSAL;
    pi.block = r;
    pairs.push_back(std::move(pi));
  }
  const float scale = softmax_scale > 0.f ? softmax_scale : 1.0f / std::sqrt((float)dh);
  record(g_ev_attn_begin, st);
  if ((s = run_pairs(qh, kh, vh, (int64_t)P * S, (int64_t)P * S, hg, hkg, dh, mask == CP_MASK_CAUSAL, nullptr, 0,
                     scale, pairs, st)) != CP_OK)
    return s;
  record(g_ev_attn_end, st);
  if ((e = launch_ulysses(oh, o, P, n, (size_t)hg * dh * 4, 1, st)) != cudaSuccess)
    return cuda_fail(e, "ulysses head->seq");
  return ok();
}

static cp_status usp_check(int S, int hq, int hkv, int dh, int Pr, int Pu, cp_layout layout, cp_mask mask,
                           const int32_t* cu_host, int n_docs) {
  cp_status s;
  if ((s = check_common(hq, hkv, dh)) != CP_OK) return s;
  if (Pu < 1 || Pu > 64) return fail(CP_ERR_UNSUPPORTED, "Pu = %d (supported 1..64)", Pu);
  if (hkv % Pu != 0) return fail(CP_ERR_UNSUPPORTED, "Pu (%d) must divide the KV head count (%d)", Pu, hkv);
  if ((s = ring_check(S, hq / Pu, hkv / Pu, dh, Pr, layout, mask, CP_BF16, cu_host, n_docs)) != CP_OK) return s;
  if (S % (Pr * Pu) != 0) return fail(CP_ERR_INVALID_ARG, "S = %d is not a multiple of Pr*Pu = %d", S, Pr * Pu);
  if ((int64_t)Pu * S >= (1 << 30)) return fail(CP_ERR_UNSUPPORTED, "Pu * S = %lld rows", (long long)Pu * S);
  return CP_OK;
}

// Workspace of the hybrid: head-major Q [Pu][S][hq/Pu][dh], K and V
// [Pu][S][hkv/Pu][dh] (bf16), then Pu copies of the ring partials.
static size_t usp_workspace(int S, int hq, int hkv, int dh, int Pu, const RingPlan& plan) {
  return align256((size_t)S * hq * dh * 2) + 2 * align256((size_t)S * hkv * dh * 2) +
         (size_t)Pu * align256(plan.partial_bytes);
}

cp_status cp_usp_attn_workspace_size(int S, int hq, int hkv, int dh, int Pr, int Pu, cp_layout layout, cp_mask mask,
                                     const int32_t* cu_seqlens_host, int n_docs, size_t* bytes) {
  cp_status s;
  if (!bytes) return fail(CP_ERR_INVALID_ARG, "bytes is NULL");
  if ((s = usp_check(S, hq, hkv, dh, Pr, Pu, layout, mask, cu_seqlens_host, n_docs)) != CP_OK) return s;
  RingPlan plan = make_ring_plan(S, hq / Pu, dh, Pr, layout, mask, cu_seqlens_host, n_docs);
  *bytes = usp_workspace(S, hq, hkv, dh, Pu, plan);
  return ok();
}

cp_status cp_usp_attn_fwd(const void* q, const void* k, const void* v, int S, int hq, int hkv, int dh, int Pr, int Pu,
                          cp_layout layout, cp_mask mask, const int32_t* cu_seqlens_host,
                          const int32_t* cu_seqlens_dev, int n_docs, float softmax_scale, float* o, float* lse,
                          void* workspace, size_t ws_bytes, void* stream) {
  cp_status s;
  if ((s = usp_check(S, hq, hkv, dh, Pr, Pu, layout, mask, cu_seqlens_host, n_docs)) != CP_OK) return s;
  CP_CHECK_PTR(q);
  CP_CHECK_PTR(k);
  CP_CHECK_PTR(v);
  CP_CHECK_PTR(o);
  CP_CHECK_PTR(lse);
  if (n_docs > 0 && !cu_seqlens_dev) return fail(CP_ERR_INVALID_ARG, "n_docs > 0 needs cu_seqlens_dev");
  const int hg = hq / Pu, hkg = hkv / Pu;
  RingPlan plan = make_ring_plan(S, hg, dh, Pr, layout, mask, cu_seqlens_host, n_docs);
  const size_t need = usp_workspace(S, hq, hkv, dh, Pu, plan);
  if (!workspace || ws_bytes < need)
    return fail(CP_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", need, ws_bytes);
  if (reinterpret_cast<uintptr_t>(workspace) & 255u) return fail(CP_ERR_ALIGNMENT, "workspace is not 256-byte aligned");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  size_t off = 0;
  void* qh = ws + off;
  off += align256((size_t)S * hq * dh * 2);
  void* kh = ws + off;
  off += align256((size_t)S * hkv * dh * 2);
  void* vh = ws + off;
  off += align256((size_t)S * hkv * dh * 2);
  uint8_t* parts = ws + off;
  const size_t part_stride = align256(plan.partial_bytes);

  // Ulysses seq->head inside every group at once: on one device the groups'
  // sub-shards are consecutive rows, so the transpose over Pu with n = S/Pu
  // gives head block u all S rows in storage order, out[u][row] = in[row][u].
  cudaError_t e;
  const int n = S / Pu;
  if ((e = launch_ulysses(q, qh, Pu, n, (size_t)hg * dh * 2, 0, st)) != cudaSuccess ||
      (e = launch_ulysses(k, kh, Pu, n, (size_t)hkg * dh * 2, 0, st)) != cudaSuccess ||
      (e = launch_ulysses(v, vh, Pu, n, (size_t)hkg * dh * 2, 0, st)) != cudaSuccess)
    return cuda_fail(e, "usp seq->head");

  // Ring across the groups for every head block: head block u's rows start
  // at u*S in the head-major buffers.  Each head block is one block of the
  // launch (its pairs read rows [u*S, (u+1)*S)); inside it the pairs keep the
  // heaviest-first order of the ring plan.
  std::vector<PairIn> pairs;
  pairs.reserve(plan.pairs.size() * Pu);
  for (const PairPlan& pp : plan.pairs)
    for (int u = 0; u < Pu; ++u) {
      PairIn pi;
      pi.q = pp.q;
      pi.k = pp.k;
      for (Seg& x : pi.q) x.buf_row += u * S;
      for (Seg& x : pi.k) x.buf_row += u * S;
      pi.qtiles = pp.qtiles;
      uint8_t* pu = parts + (size_t)u * part_stride;
      pi.o = reinterpret_cast<float*>(pu + pp.o_off);
      pi.lse = reinterpret_cast<float*>(pu + pp.lse_off);
      pi.lse_ld = pp.rows;
      pi.reverse = mask == CP_MASK_CAUSAL;
      pi.block = u;
      pairs.push_back(std::move(pi));
    }
  const float scale = softmax_scale > 0.f ? softmax_scale : 1.0f / std::sqrt((float)dh);
  record(g_ev_attn_begin, st);
  if ((s = run_pairs(qh, kh, vh, (int64_t)Pu * S, (int64_t)Pu * S, hg, hkg, dh, mask == CP_MASK_CAUSAL,
                     cu_seqlens_dev, n_docs, scale, pairs, st)) != CP_OK)
    return s;
  record(g_ev_attn_end, st);

  // Merge per head block, writing heads [u*hg, (u+1)*hg) of every output
  // row: the head->seq transpose happens in the merge's stores.
  std::vector<MergeTaskIn> tasks;
  for (int u = 0; u < Pu; ++u) {
    const uint8_t* pu = parts + (size_t)u * part_stride;
    for (const MergeTaskPlan& tp : plan.tasks) {
      MergeTaskIn t;
      t.out_row0 = tp.row0;
      t.rows = tp.rows;
      t.head_off = u * hg;
      for (const auto& in : tp.inputs) {
        const PairPlan& pp = plan.pairs[in.first];
        t.in.push_back({reinterpret_cast<const float*>(pu + pp.o_off),
                        reinterpret_cast<const float*>(pu + pp.lse_off), in.second, pp.rows});
      }
      tasks.push_back(std::move(t));
    }
  }
  if ((s = run_merge(tasks, hg, dh, o, lse, S, nullptr, st, hq)) != CP_OK) return s;
  record(g_ev_merge_end, st);
  return ok();
}

// ------------------------------------------------------------------ backward
static size_t bwd_workspace(int S, int hq) { return 2 * align256((size_t)S * hq * sizeof(float)); }

cp_status cp_ring_attn_bwd_workspace_size(int S, int hq, int hkv, int dh, int P, cp_layout layout, cp_mask mask,
                                          const int32_t* cu_seqlens_host, int n_docs, size_t* bytes) {
  cp_status s;
  if (!bytes) return fail(CP_ERR_INVALID_ARG, "bytes is NULL");
  if ((s = ring_check(S, hq, hkv, dh, P, layout, mask, CP_BF16, cu_seqlens_host, n_docs)) != CP_OK) return s;
  *bytes = bwd_workspace(S, hq);
  return ok();
}

namespace {
struct BwdItem {
  uint32_t code;
  int64_t cost;
};

// Own 128-row tiles of every rank (dq_side) or shard and every head group,
// ordered by the number of (q, k) pairs they admit over the plan's ring steps,
// heaviest first.  only >= 0 keeps the tiles of that rank alone.
std::vector<uint32_t> bwd_items(const cp_bwd_plan& pl, int groups, bool dq_side, const Docs& docs, int only = -1) {
  std::vector<BwdItem> v;
  for (int a = 0; a < pl.P; ++a) {
    if (only >= 0 && a != only) continue;
    for (int sg = 0; sg < pl.nseg[a]; ++sg) {
      const cp_seg& own = pl.seg[a][sg];
      for (int t = 0; t * 128 < own.len; ++t) {
        const int pos = own.pos + t * 128, len = std::min(128, own.len - t * 128);
        int64_t cost = 0;
        for (int step = pl.t_begin; step < pl.t_end; ++step) {
          const int b = dq_side ? ((a - step) % pl.P + pl.P) % pl.P : (a + step) % pl.P;
          for (int x = 0; x < pl.nseg[b]; ++x) {
            const cp_seg& other = pl.seg[b][x];
            // striped: a key of shard j sits one position later for rank r < j
            if (dq_side) {
              const int shift = (pl.striped && b > a) ? 1 : 0;
              cost += count_admitted(pos, len, other.pos + shift, other.len, pl.causal != 0, docs);
            } else {
              const int shift = (pl.striped && a > b) ? 1 : 0;
              cost += count_admitted(other.pos, other.len, pos + shift, len, pl.causal != 0, docs);
            }
          }
        }
        for (int g = 0; g < groups; ++g)
          v.push_back({((uint32_t)a << 26) | ((uint32_t)sg << 25) | ((uint32_t)g << 19) | (uint32_t)t, cost});
      }
    }
  }
  std::stable_sort(v.begin(), v.end(), [](const BwdItem& x, const BwdItem& y) { return x.cost > y.cost; });
  std::vector<uint32_t> out;
  out.reserve(v.size());
  for (const BwdItem& x : v) out.push_back(x.code);
  return out;
}

// The ring backward over P ranks for `groups` blocks of heads.  qh, kh, vh,
// doh are the head-major bf16 buffers ([groups][S][hg | hkg][dh]; one group:
// the plain sharded buffers) the tensor cores read; dout, o, lse, dq, dk, dv
// are in the final [S][groups * h][dh] / [groups * hq][S] layouts; lg, dd
// are fp32 [hg][groups * S].
cp_status run_bwd(const void* qh, const void* kh, const void* vh, const void* doh, const void* dout, const float* o,
                  const float* lse, int S, int groups, int hg, int hkg, int dh, int P, cp_layout layout, cp_mask mask,
                  const int32_t* cu_host, const int32_t* cu_dev, int n_docs, float softmax_scale, float* dq,
                  float* dk, float* dv, float* lg, float* dd, cudaStream_t st) {
  cp_status s;
  const int64_t rows = (int64_t)groups * S;
  CUtensorMap tq, tdo, tk, tv;
  if ((s = make_map(&tq, qh, rows, (int64_t)hg * dh, 128)) != CP_OK) return s;
  if ((s = make_map(&tdo, doh, rows, (int64_t)hg * dh, 128)) != CP_OK) return s;
  if ((s = make_map(&tk, kh, rows, (int64_t)hkg * dh, 128)) != CP_OK) return s;
  if ((s = make_map(&tv, vh, rows, (int64_t)hkg * dh, 128)) != CP_OK) return s;
  uint32_t* err = nullptr;
  if ((s = err_word(&err)) != CP_OK) return s;

  static cp_bwd_plan plan;  // large POD: keep it off the stack
  static std::mutex plan_mu;
  std::lock_guard<std::mutex> lk(plan_mu);
  memset(&plan, 0, sizeof(plan));
  const Layout lay = layout == CP_LAYOUT_ZIGZAG ? Layout::Zigzag
                     : layout == CP_LAYOUT_STRIPED ? Layout::Striped
                                                   : Layout::Contiguous;
  plan.P = P;
  plan.hq = hg;
  plan.hkv = hkg;
  plan.causal = mask == CP_MASK_CAUSAL ? 1 : 0;
  plan.striped = lay == Layout::Striped ? 1 : 0;
  plan.n_docs = n_docs;
  plan.cu_seqlens = cu_dev;
  const float scale = softmax_scale > 0.f ? softmax_scale : 1.0f / std::sqrt((float)dh);
  plan.scale = scale;
  plan.scale_log2 = scale * 1.4426950408889634f;
  plan.S = (int32_t)rows;
  plan.group_rows = S;
  plan.out_hq = groups * hg;
  plan.out_hkv = groups * hkg;
  for (int r = 0; r < P; ++r) {
    const std::vector<Seg> segs = shard_segments(S, P, lay, r);
    plan.nseg[r] = (int)segs.size();
    for (size_t x = 0; x < segs.size(); ++x) plan.seg[r][x] = {segs[x].buf_row, segs[x].pos, segs[x].len, 0};
  }
  plan.lg = lg;
  plan.dd = dd;
  plan.dq = dq;
  plan.dk = dk;
  plan.dv = dv;
  plan.err = err;
  plan.t_begin = 0;
  plan.t_end = P;
  plan.accumulate = 0;
  Docs docs;
  if (cu_host && n_docs > 0) {
    docs.cu = cu_host;
    docs.n = n_docs;
  }
  cudaError_t e = launch_bwd_prep(dh, o, dout, lse, S, hg, groups, lg, dd, st);
  if (e != cudaSuccess) return cuda_fail(e, "backward prep launch");
  record(g_ev_attn_begin, st);
  for (int side = 0; side < 2; ++side) {
    const bool dq_side = side == 0;
    const std::vector<uint32_t> items = bwd_items(plan, groups, dq_side, docs);
    for (size_t base = 0; base < items.size(); base += CP_BWD_MAX_ITEMS) {
      const size_t cnt = std::min(items.size() - base, (size_t)CP_BWD_MAX_ITEMS);
      plan.n_items = (int)cnt;
      std::copy(items.begin() + base, items.begin() + base + cnt, plan.items);
      e = launch_bwd(dh, tq, tdo, tk, tv, plan, dq_side, st);
      if (e != cudaSuccess) return cuda_fail(e, dq_side ? "backward dQ launch" : "backward dK/dV launch");
    }
    if (dq_side) record(g_ev_merge_end, st);
  }
  record(g_ev_attn_end, st);
  return CP_OK;
}

cp_status bwd_check_ptrs(const void* q, const void* k, const void* v, const float* o, const float* lse,
                         const void* dout, float* dq, float* dk, float* dv) {
  CP_CHECK_PTR(q);
  CP_CHECK_PTR(k);
  CP_CHECK_PTR(v);
  CP_CHECK_PTR(o);
  CP_CHECK_PTR(lse);
  CP_CHECK_PTR(dout);
  CP_CHECK_PTR(dq);
  CP_CHECK_PTR(dk);
  CP_CHECK_PTR(dv);
  return CP_OK;
}
}  // namespace

cp_status cp_ring_attn_bwd(const void* q, const void* k, const void* v, const float* o, const float* lse,
                           const void* dout, int S, int hq, int hkv, int dh, int P, cp_layout layout, cp_mask mask,
                           const int32_t* cu_seqlens_host, const int32_t* cu_seqlens_dev, int n_docs,
                           float softmax_scale, float* dq, float* dk, float* dv, void* workspace, size_t ws_bytes,
                           void* stream) {
  cp_status s;
  if ((s = ring_check(S, hq, hkv, dh, P, layout, mask, CP_BF16, cu_seqlens_host, n_docs)) != CP_OK) return s;
  if ((s = bwd_check_ptrs(q, k, v, o, lse, dout, dq, dk, dv)) != CP_OK) return s;
  if (P > CP_BWD_MAX_RANKS) return fail(CP_ERR_UNSUPPORTED, "P = %d (backward supports 1..%d)", P, CP_BWD_MAX_RANKS);
  if (n_docs > 0 && !cu_seqlens_dev) return fail(CP_ERR_INVALID_ARG, "n_docs > 0 needs cu_seqlens_dev");
  const size_t need = bwd_workspace(S, hq);
  if (!workspace || ws_bytes < need)
    return fail(CP_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", need, ws_bytes);
  if (reinterpret_cast<uintptr_t>(workspace) & 255u) return fail(CP_ERR_ALIGNMENT, "workspace is not 256-byte aligned");
  float* lg = static_cast<float*>(workspace);
  float* dd = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + align256((size_t)S * hq * sizeof(float)));
  if ((s = run_bwd(q, k, v, dout, dout, o, lse, S, 1, hq, hkv, dh, P, layout, mask, cu_seqlens_host, cu_seqlens_dev,
                   n_docs, softmax_scale, dq, dk, dv, lg, dd, static_cast<cudaStream_t>(stream))) != CP_OK)
    return s;
  return ok();
}

cp_status cp_attn_bwd_prep(const float* o, const void* dout, const float* lse, int n, int hq, int dh, float* lg,
                           float* dd, void* stream) {
  if (dh != 64 && dh != 128) return fail(CP_ERR_UNSUPPORTED, "dh = %d (supported: 64, 128)", dh);
  if (n <= 0 || n >= (1 << 30) || hq <= 0) return fail(CP_ERR_INVALID_ARG, "n must be in [1, 2^30), hq > 0");
  CP_CHECK_PTR(o);
  CP_CHECK_PTR(dout);
  CP_CHECK_PTR(lse);
  CP_CHECK_PTR(lg);
  CP_CHECK_PTR(dd);
  cudaError_t e = launch_bwd_prep(dh, o, dout, lse, n, hq, 1, lg, dd, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "backward prep launch");
  return ok();
}

// One block pair as a two-rank plan: rank 0 holds the query rows (buffer rows
// of q, dout, dq), rank 1 the key/value rows (buffer rows of k, v, dk, dv),
// and the ring is narrowed to step 1, at which each sees only the other.
// Positions come from the chunks as given (a striped key shift is already
// part of them), so the plan's striped flag stays off.
cp_status cp_block_attn_bwd(const void* q, const void* k, const void* v, const void* dout, const float* lg,
                            const float* dd, int n_q, int n_k, int hq, int hkv, int dh, const cp_chunk* q_chunks,
                            int nq_chunks, const cp_chunk* k_chunks, int nk_chunks, cp_mask mask,
                            const int32_t* cu_seqlens_dev, int n_docs, float softmax_scale, float* dq, float* dk,
                            float* dv, int parts, int accumulate, void* stream) {
  cp_status s;
  if ((s = check_common(hq, hkv, dh)) != CP_OK) return s;
  if (n_q <= 0 || n_k <= 0 || n_q >= (1 << 30) || n_k >= (1 << 30))
    return fail(CP_ERR_INVALID_ARG, "n_q, n_k must be in [1, 2^30)");
  if (parts < 1 || parts > (CP_BWD_DQ | CP_BWD_DKDV)) return fail(CP_ERR_INVALID_ARG, "parts = %d", parts);
  if (accumulate != 0 && accumulate != 1) return fail(CP_ERR_INVALID_ARG, "accumulate must be 0 or 1");
  CP_CHECK_PTR(q);
  CP_CHECK_PTR(k);
  CP_CHECK_PTR(v);
  CP_CHECK_PTR(dout);
  CP_CHECK_PTR(lg);
  CP_CHECK_PTR(dd);
  if (parts & CP_BWD_DQ) CP_CHECK_PTR(dq);
  if (parts & CP_BWD_DKDV) {
    CP_CHECK_PTR(dk);
    CP_CHECK_PTR(dv);
  }
  if (mask != CP_MASK_NONE && mask != CP_MASK_CAUSAL) return fail(CP_ERR_INVALID_ARG, "unknown mask %d", (int)mask);
  if (!q_chunks || !k_chunks) return fail(CP_ERR_INVALID_ARG, "chunk lists are NULL");
  if (nq_chunks < 1 || nq_chunks > CP_BWD_MAX_CHUNKS || nk_chunks < 1 || nk_chunks > CP_BWD_MAX_CHUNKS)
    return fail(CP_ERR_UNSUPPORTED, "1..%d chunks per side", CP_BWD_MAX_CHUNKS);
  if (n_docs < 0 || (n_docs > 0 && !cu_seqlens_dev))
    return fail(CP_ERR_INVALID_ARG, "n_docs > 0 needs cu_seqlens_dev");
  const cp_chunk* side_chunks[2] = {q_chunks, k_chunks};
  const int side_n[2] = {nq_chunks, nk_chunks}, side_rows[2] = {n_q, n_k};
  cp_seg segs[2][2];
  for (int a = 0; a < 2; ++a) {
    int rows = 0;
    for (int i = 0; i < side_n[a]; ++i) {
      const cp_chunk& c = side_chunks[a][i];
      if (c.len <= 0 || c.start < 0) return fail(CP_ERR_INVALID_ARG, "bad %s chunk %d", a ? "k" : "q", i);
      segs[a][i] = {rows, c.start, c.len, 0};
      rows += c.len;
    }
    if (rows != side_rows[a])
      return fail(CP_ERR_INVALID_ARG, "%s chunks cover %d rows, expected %d", a ? "k" : "q", rows, side_rows[a]);
  }
  CUtensorMap tq, tdo, tk, tv;
  if ((s = make_map(&tq, q, n_q, (int64_t)hq * dh, 128)) != CP_OK) return s;
  if ((s = make_map(&tdo, dout, n_q, (int64_t)hq * dh, 128)) != CP_OK) return s;
  if ((s = make_map(&tk, k, n_k, (int64_t)hkv * dh, 128)) != CP_OK) return s;
  if ((s = make_map(&tv, v, n_k, (int64_t)hkv * dh, 128)) != CP_OK) return s;
  uint32_t* err = nullptr;
  if ((s = err_word(&err)) != CP_OK) return s;

  static cp_bwd_plan plan;
  static std::mutex plan_mu;
  std::lock_guard<std::mutex> lk(plan_mu);
  memset(&plan, 0, sizeof(plan));
  plan.P = 2;
  plan.hq = hq;
  plan.hkv = hkv;
  plan.causal = mask == CP_MASK_CAUSAL ? 1 : 0;
  plan.striped = 0;
  plan.n_docs = n_docs;
  plan.cu_seqlens = cu_seqlens_dev;
  const float scale = softmax_scale > 0.f ? softmax_scale : 1.0f / std::sqrt((float)dh);
  plan.scale = scale;
  plan.scale_log2 = scale * 1.4426950408889634f;
  plan.S = n_q;  // row pitch of lg and dd
  plan.group_rows = 0;
  plan.out_hq = hq;
  plan.out_hkv = hkv;
  for (int a = 0; a < 2; ++a) {
    plan.nseg[a] = side_n[a];
    for (int i = 0; i < side_n[a]; ++i) plan.seg[a][i] = segs[a][i];
  }
  plan.lg = lg;
  plan.dd = dd;
  plan.dq = dq;
  plan.dk = dk;
  plan.dv = dv;
  plan.err = err;
  plan.t_begin = 1;
  plan.t_end = 2;
  plan.accumulate = accumulate;
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  for (int side = 0; side < 2; ++side) {
    const bool dq_side = side == 0;
    if (!(parts & (dq_side ? CP_BWD_DQ : CP_BWD_DKDV))) continue;
    const std::vector<uint32_t> items = bwd_items(plan, 1, dq_side, Docs{}, dq_side ? 0 : 1);
    for (size_t base = 0; base < items.size(); base += CP_BWD_MAX_ITEMS) {
      const size_t cnt = std::min(items.size() - base, (size_t)CP_BWD_MAX_ITEMS);
      plan.n_items = (int)cnt;
      std::copy(items.begin() + base, items.begin() + base + cnt, plan.items);
      cudaError_t e = launch_bwd(dh, tq, tdo, tk, tv, plan, dq_side, st);
      if (e != cudaSuccess) return cuda_fail(e, dq_side ? "block backward dQ launch" : "block backward dK/dV launch");
    }
  }
  return ok();
}

// Workspace of the hybrid backward: head-major bf16 Q, dO [Pu][S][hq/Pu][dh],
// K, V [Pu][S][hkv/Pu][dh], then D and LSE*log2(e).
static size_t usp_bwd_workspace(int S, int hq, int hkv, int dh) {
  return 2 * align256((size_t)S * hq * dh * 2) + 2 * align256((size_t)S * hkv * dh * 2) + bwd_workspace(S, hq);
}

cp_status cp_usp_attn_bwd_workspace_size(int S, int hq, int hkv, int dh, int Pr, int Pu, cp_layout layout,
                                         cp_mask mask, const int32_t* cu_seqlens_host, int n_docs, size_t* bytes) {
  cp_status s;
  if (!bytes) return fail(CP_ERR_INVALID_ARG, "bytes is NULL");
  if ((s = usp_check(S, hq, hkv, dh, Pr, Pu, layout, mask, cu_seqlens_host, n_docs)) != CP_OK) return s;
  *bytes = usp_bwd_workspace(S, hq, hkv, dh);
  return ok();
}

cp_status cp_usp_attn_bwd(const void* q, const void* k, const void* v, const float* o, const float* lse,
                          const void* dout, int S, int hq, int hkv, int dh, int Pr, int Pu, cp_layout layout,
                          cp_mask mask, const int32_t* cu_seqlens_host, const int32_t* cu_seqlens_dev, int n_docs,
                          float softmax_scale, float* dq, float* dk, float* dv, void* workspace, size_t ws_bytes,
                          void* stream) {
  cp_status s;
  if ((s = usp_check(S, hq, hkv, dh, Pr, Pu, layout, mask, cu_seqlens_host, n_docs)) != CP_OK) return s;
  if ((s = bwd_check_ptrs(q, k, v, o, lse, dout, dq, dk, dv)) != CP_OK) return s;
  if (Pr > CP_BWD_MAX_RANKS) return fail(CP_ERR_UNSUPPORTED, "Pr = %d (backward supports 1..%d)", Pr, CP_BWD_MAX_RANKS);
  if (Pu > CP_BWD_MAX_GROUPS) return fail(CP_ERR_UNSUPPORTED, "Pu = %d (backward supports 1..%d)", Pu, CP_BWD_MAX_GROUPS);
  if (n_docs > 0 && !cu_seqlens_dev) return fail(CP_ERR_INVALID_ARG, "n_docs > 0 needs cu_seqlens_dev");
  const size_t need = usp_bwd_workspace(S, hq, hkv, dh);
  if (!workspace || ws_bytes < need)
    return fail(CP_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", need, ws_bytes);
  if (reinterpret_cast<uintptr_t>(workspace) & 255u) return fail(CP_ERR_ALIGNMENT, "workspace is not 256-byte aligned");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  size_t off = 0;
  void* qh = ws + off;
  off += align256((size_t)S * hq * dh * 2);
  void* doh = ws + off;
  off += align256((size_t)S * hq * dh * 2);
  void* kh = ws + off;
  off += align256((size_t)S * hkv * dh * 2);
  void* vh = ws + off;
  off += align256((size_t)S * hkv * dh * 2);
  float* lg = reinterpret_cast<float*>(ws + off);
  float* dd = reinterpret_cast<float*>(ws + off + align256((size_t)S * hq * sizeof(float)));
  const int hg = hq / Pu, hkg = hkv / Pu, n = S / Pu;
  // Ulysses seq->head of Q, K, V and dO (every group at once); the gradients
  // and the LSE are read and written in their final layouts by the kernels.
  cudaError_t e;
  if ((e = launch_ulysses(q, qh, Pu, n, (size_t)hg * dh * 2, 0, st)) != cudaSuccess ||
      (e = launch_ulysses(dout, doh, Pu, n, (size_t)hg * dh * 2, 0, st)) != cudaSuccess ||
      (e = launch_ulysses(k, kh, Pu, n, (size_t)hkg * dh * 2, 0, st)) != cudaSuccess ||
      (e = launch_ulysses(v, vh, Pu, n, (size_t)hkg * dh * 2, 0, st)) != cudaSuccess)
    return cuda_fail(e, "usp backward seq->head");
  if ((s = run_bwd(qh, kh, vh, doh, dout, o, lse, S, Pu, hg, hkg, dh, Pr, layout, mask, cu_seqlens_host,
                   cu_seqlens_dev, n_docs, softmax_scale, dq, dk, dv, lg, dd, st)) != CP_OK)
    return s;
  return ok();
}

cp_status cp_ulysses_attn_bwd_workspace_size(int S, int hq, int hkv, int dh, int P, size_t* bytes) {
  return cp_usp_attn_bwd_workspace_size(S, hq, hkv, dh, 1, P, CP_LAYOUT_CONTIGUOUS, CP_MASK_CAUSAL, nullptr, 0, bytes);
}

cp_status cp_ulysses_attn_bwd(const void* q, const void* k, const void* v, const float* o, const float* lse,
                              const void* dout, int S, int hq, int hkv, int dh, int P, cp_mask mask,
                              float softmax_scale, float* dq, float* dk, float* dv, void* workspace, size_t ws_bytes,
                              void* stream) {
  return cp_usp_attn_bwd(q, k, v, o, lse, dout, S, hq, hkv, dh, 1, P, CP_LAYOUT_CONTIGUOUS, mask, nullptr, nullptr, 0,
                         softmax_scale, dq, dk, dv, workspace, ws_bytes, stream);
}


cp_status cp_ring_schedule(int S, int P, cp_layout layout, cp_mask mask, const int32_t* cu_seqlens_host, int n_docs,
                           int32_t* src, int32_t* launched, int32_t* q_rows, int64_t* live_pairs) {
  cp_status s = ring_check(S, 1, 1, 128, P, layout, mask, CP_BF16, cu_seqlens_host, n_docs);
  if (s != CP_OK) return s;
  RingPlan plan = make_ring_plan(S, 1, 128, P, layout, mask, cu_seqlens_host, n_docs);
  for (int i = 0; i < P * P; ++i) {
    if (src) src[i] = plan.src[i];
    if (launched) launched[i] = plan.launched[i];
    if (q_rows) q_rows[i] = plan.q_rows[i];
    if (live_pairs) live_pairs[i] = plan.live_all[i];
  }
  return ok();
}

cp_status cp_count_live_pairs(int S, cp_mask mask, const int32_t* cu_seqlens_host, int n_docs, int64_t* pairs) {
  if (!pairs) return fail(CP_ERR_INVALID_ARG, "pairs is NULL");
  if (S <= 0) return fail(CP_ERR_INVALID_ARG, "S = %d", S);
  cp_status s = check_docs_host(cu_seqlens_host, n_docs, S);
  if (s != CP_OK) return s;
  Docs docs;
  if (cu_seqlens_host && n_docs > 0) {
    docs.cu = cu_seqlens_host;
    docs.n = n_docs;
  }
  *pairs = count_admitted(0, S, 0, S, mask == CP_MASK_CAUSAL, docs);
  return ok();
}

cp_status cp_kernel_launch_count(uint64_t* count) {
  if (!count) return fail(CP_ERR_INVALID_ARG, "count is NULL");
  *count = cp::launch_counter().load();
  return ok();
}

cp_status cp_set_profile_events(void* attn_begin, void* attn_end, void* merge_end) {
  g_ev_attn_begin = static_cast<cudaEvent_t>(attn_begin);
  g_ev_attn_end = static_cast<cudaEvent_t>(attn_end);
  g_ev_merge_end = static_cast<cudaEvent_t>(merge_end);
  return ok();
}

cp_status cp_device_error(uint32_t* bits, int clear) {
  if (!bits) return fail(CP_ERR_INVALID_ARG, "bits is NULL");
  uint32_t* w = nullptr;
  cp_status s = err_word(&w);
  if (s != CP_OK) return s;
  cudaError_t e = cudaMemcpy(bits, w, sizeof(uint32_t), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "read error word");
  if (clear) {
    e = cudaMemset(w, 0, sizeof(uint32_t));
    if (e != cudaSuccess) return cuda_fail(e, "clear error word");
  }
  return ok();
}

}  // extern "C"
