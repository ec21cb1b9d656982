// LSE merge of partial attention results (sm_100a, HBM-bound).
//
// For each output row and head:  LSE = ln sum_i exp(LSE_i),
//                                 O   = sum_i exp(LSE_i - LSE) * O_i,
// the block-granular form of the online-softmax recurrence of the
// "序列並行（Sequence Parallelism）" concept page (compassingai), 技術原理 §二:
// each partial carries its own max and denominator folded into LSE_i, and the
// fold rescales each partial's normalised O by its share of the total
// denominator.  Partials whose LSE_i is -inf hold no admitted key for that row;
// they get weight 0 and their O is never combined.  All arithmetic is fp32.
//
// One group of dh/4 threads handles one (row, head): every thread owns four
// consecutive columns and moves them with 16-byte loads and stores, so a warp
// touches 512 contiguous bytes per input row (dh = 128).
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math_constants.h>

#include <atomic>

#include "plan.h"

namespace cp {

std::atomic<uint64_t>& launch_counter();

template <int DH>
__global__ void __launch_bounds__(256) lse_merge_kernel(const __grid_constant__ cp_merge_plan plan) {
  constexpr int TPI = DH / 4;        // threads per (row, head)
  constexpr int IPB = 256 / TPI;     // (row, head) items per block
  constexpr int U = 4;               // partials whose loads are in flight together
  const cp_merge_task& task = plan.tasks[blockIdx.y];
  const int item = blockIdx.x * IPB + threadIdx.x / TPI;
  const int sub = threadIdx.x % TPI;
  const int h = plan.h;
  const int row = item / h;
  const int head = item - row * h;
  if (row >= task.rows) return;

  const cp_merge_input* in = plan.inputs + task.in_begin;
  const int n = task.n_in;
  // Single pass with a running maximum: the LSE and O loads of U partials
  // are issued together (no load waits on another), then folded.
  float m = -CUDART_INF_F, tot = 0.f;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int i0 = 0; i0 < n; i0 += U) {
    float li[U];
    float4 o[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      li[u] = -CUDART_INF_F;
      o[u] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (i0 + u < n) {
        const cp_merge_input& x = in[i0 + u];
        li[u] = __ldg(x.lse + (size_t)head * x.lse_ld + x.row0 + row);
        o[u] = __ldcs(reinterpret_cast<const float4*>(x.o + ((size_t)(x.row0 + row) * h + head) * DH) + sub);
      }
    }
    float mr = m;
#pragma unroll
    for (int u = 0; u < U; ++u) mr = fmaxf(mr, li[u]);
    if (mr != -CUDART_INF_F) {
      if (mr > m) {
        const float f = m == -CUDART_INF_F ? 0.f : expf(m - mr);
        tot *= f;
        acc.x *= f;
        acc.y *= f;
        acc.z *= f;
        acc.w *= f;
        m = mr;
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        // a partial with LSE = -inf has no admitted key: weight 0, and its O
        // (possibly not a number) is never combined
        if (li[u] != -CUDART_INF_F) {
          const float w = expf(li[u] - m);
          tot += w;
          acc.x = fmaf(w, o[u].x, acc.x);
          acc.y = fmaf(w, o[u].y, acc.y);
          acc.z = fmaf(w, o[u].z, acc.z);
          acc.w = fmaf(w, o[u].w, acc.w);
        }
      }
    }
  }
  const float inv = tot > 0.f ? 1.f / tot : 0.f;
  acc.x *= inv;
  acc.y *= inv;
  acc.z *= inv;
  acc.w *= inv;
  const size_t orow = (size_t)(task.out_row0 + row);
  const size_t ohead = (size_t)task.head_off + head;
  const size_t oidx = (orow * plan.o_heads + ohead) * DH;
  __stcs(reinterpret_cast<float4*>(plan.o_out + oidx) + sub, acc);
  if (plan.o_out_bf16) {
    const __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x, acc.y);
    const __nv_bfloat162 hi = __floats2bfloat162_rn(acc.z, acc.w);
    uint2 pk;
    pk.x = *reinterpret_cast<const uint32_t*>(&lo);
    pk.y = *reinterpret_cast<const uint32_t*>(&hi);
    reinterpret_cast<uint2*>(plan.o_out_bf16 + oidx)[sub] = pk;
  }
  if (sub == 0) {
    const float lse = tot > 0.f ? m + logf(tot) : -CUDART_INF_F;
    plan.lse_out[ohead * plan.lse_out_ld + orow] = lse;
  }
}

cudaError_t launch_merge(const cp_merge_plan& plan, int max_rows, cudaStream_t stream) {
  if (plan.n_tasks <= 0 || max_rows <= 0) return cudaSuccess;
  const int tpi = plan.dh / 4;
  const int ipb = 256 / tpi;
  const long long items = (long long)max_rows * plan.h;
  dim3 grid((unsigned)((items + ipb - 1) / ipb), (unsigned)plan.n_tasks);
  if (plan.dh == 128) lse_merge_kernel<128><<<grid, 256, 0, stream>>>(plan);
  else lse_merge_kernel<64><<<grid, 256, 0, stream>>>(plan);
  launch_counter()++;
  return cudaGetLastError();
}

}  // namespace cp
