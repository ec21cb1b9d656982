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
// A CTA takes a block of 8 rows x 8 heads of one task; warp w folds row w,
// two (row, head) items at a time with all their loads (LSE and O of two
// partials each) issued together, the 8 warps' LSE loads of one head and
// partial falling in one sector:
// dh/4 threads per (row, head), each owning four consecutive columns moved
// with 16-byte loads and stores, so a warp instruction covers 512 contiguous
// bytes of a row (dh = 128) and a warp's eight heads cover 4 KB.  The tasks of
// a launch own consecutive ranges of CTAs in one flat grid (no CTA without
// work).
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math_constants.h>

#include <atomic>

#include "plan.h"

namespace cp {

std::atomic<uint64_t>& launch_counter();

constexpr int kMergeRows = 8;    // rows per CTA (one per warp)
constexpr int kMergeHeads = 8;   // heads per CTA

template <int DH>
__global__ void __launch_bounds__(256, 5) lse_merge_kernel(const __grid_constant__ cp_merge_plan plan) {
  constexpr int TPI = DH / 4;     // threads per (row, head)
  constexpr int IPW = 32 / TPI;   // (row, head) items per warp instruction
  constexpr int U = 2;            // partials per item whose loads are in flight together
  __shared__ float s_out[kMergeHeads][kMergeRows];

  const int cta = blockIdx.x;
  int lo = 0, hi = plan.n_tasks - 1;  // the last task whose first CTA is <= cta
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (plan.tasks[mid].cta_begin <= cta) lo = mid; else hi = mid - 1;
  }
  const cp_merge_task& task = plan.tasks[lo];
  const int h = plan.h;
  const int n_hb = (h + kMergeHeads - 1) / kMergeHeads;
  const int local = cta - task.cta_begin;
  const int rb = local / n_hb;
  const int row0 = rb * kMergeRows;
  const int h0 = (local - rb * n_hb) * kMergeHeads;
  const cp_merge_input* in = plan.inputs + task.in_begin;
  const int n = task.n_in;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int sub = lane % TPI;
  const int row = row0 + warp;
  if (row < task.rows) {
    // Two (row, head) items per pass, heads hh and hh + IPW, folded side by
    // side: the loads of both items' partials [i0, i0 + U) are issued
    // together, so even a row with one or two partials keeps several 16-byte
    // loads per thread in flight.
    for (int hh0 = 0; hh0 < kMergeHeads; hh0 += 2 * IPW) {
      int hh[2], head[2];
      float m[2], tot[2];
      float4 acc[2];
#pragma unroll
      for (int a = 0; a < 2; ++a) {
        hh[a] = hh0 + lane / TPI + a * IPW;
        head[a] = h0 + hh[a];
        m[a] = -CUDART_INF_F;
        tot[a] = 0.f;
        acc[a] = make_float4(0.f, 0.f, 0.f, 0.f);
      }
      for (int i0 = 0; i0 < n; i0 += U) {
        float li[2][U];
        float4 o[2][U];
#pragma unroll
        for (int a = 0; a < 2; ++a)
#pragma unroll
          for (int u = 0; u < U; ++u) {
            li[a][u] = -CUDART_INF_F;
            o[a][u] = make_float4(0.f, 0.f, 0.f, 0.f);
            if (head[a] < h && i0 + u < n) {
              const cp_merge_input& x = in[i0 + u];
              // the 8 warps read 8 consecutive rows of this head: one sector
              li[a][u] = __ldg(x.lse + (size_t)head[a] * x.lse_ld + x.row0 + row);
              o[a][u] = __ldcs(reinterpret_cast<const float4*>(x.o + ((size_t)(x.row0 + row) * h + head[a]) * DH) + sub);
            }
          }
#pragma unroll
        for (int a = 0; a < 2; ++a) {
          // running maximum over the groups of partials
          float mr = m[a];
#pragma unroll
          for (int u = 0; u < U; ++u) mr = fmaxf(mr, li[a][u]);
          if (mr == -CUDART_INF_F) continue;
          if (mr > m[a]) {
            const float f = m[a] == -CUDART_INF_F ? 0.f : expf(m[a] - mr);
            tot[a] *= f;
            acc[a].x *= f;
            acc[a].y *= f;
            acc[a].z *= f;
            acc[a].w *= f;
            m[a] = mr;
          }
#pragma unroll
          for (int u = 0; u < U; ++u) {
            // a partial with LSE = -inf has no admitted key: weight 0, and
            // its O (possibly not a number) is never combined
            if (li[a][u] != -CUDART_INF_F) {
              const float w = expf(li[a][u] - m[a]);
              tot[a] += w;
              acc[a].x = fmaf(w, o[a][u].x, acc[a].x);
              acc[a].y = fmaf(w, o[a][u].y, acc[a].y);
              acc[a].z = fmaf(w, o[a][u].z, acc[a].z);
              acc[a].w = fmaf(w, o[a][u].w, acc[a].w);
            }
          }
        }
      }
#pragma unroll
      for (int a = 0; a < 2; ++a) {
        if (head[a] >= h) continue;
        const float inv = tot[a] > 0.f ? 1.f / tot[a] : 0.f;
        float4 r = acc[a];
        r.x *= inv;
        r.y *= inv;
        r.z *= inv;
        r.w *= inv;
        const size_t orow = (size_t)(task.out_row0 + row);
        const size_t ohead = (size_t)task.head_off + head[a];
        const size_t oidx = (orow * plan.o_heads + ohead) * DH;
        __stcs(reinterpret_cast<float4*>(plan.o_out + oidx) + sub, r);
        if (plan.o_out_bf16) {
          const __nv_bfloat162 lo2 = __floats2bfloat162_rn(r.x, r.y);
          const __nv_bfloat162 hi2 = __floats2bfloat162_rn(r.z, r.w);
          uint2 pk;
          pk.x = *reinterpret_cast<const uint32_t*>(&lo2);
          pk.y = *reinterpret_cast<const uint32_t*>(&hi2);
          reinterpret_cast<uint2*>(plan.o_out_bf16 + oidx)[sub] = pk;
        }
        if (sub == 0) s_out[hh[a]][warp] = tot[a] > 0.f ? m[a] + logf(tot[a]) : -CUDART_INF_F;
      }
    }
  }
  __syncthreads();
  // LSE out: 8 consecutive rows of each head, one sector per head
  if (threadIdx.x < kMergeHeads * kMergeRows) {
    const int hh = threadIdx.x / kMergeRows, rr = threadIdx.x % kMergeRows;
    const int r = row0 + rr, head = h0 + hh;
    if (r < task.rows && head < h)
      plan.lse_out[((size_t)task.head_off + head) * plan.lse_out_ld + task.out_row0 + r] = s_out[hh][rr];
  }
}

// CTAs of a merge task of `rows` rows and h heads.
int merge_task_ctas(int rows, int h) {
  return ((rows + kMergeRows - 1) / kMergeRows) * ((h + kMergeHeads - 1) / kMergeHeads);
}

// total_ctas: the sum of merge_task_ctas over the tasks, the tasks'
// cta_begin being the running prefix of that sum.
cudaError_t launch_merge(const cp_merge_plan& plan, int total_ctas, cudaStream_t stream) {
  if (plan.n_tasks <= 0 || total_ctas <= 0) return cudaSuccess;
  if (plan.dh == 128) lse_merge_kernel<128><<<total_ctas, 256, 0, stream>>>(plan);
  else lse_merge_kernel<64><<<total_ctas, 256, 0, stream>>>(plan);
  launch_counter()++;
  return cudaGetLastError();
}

}  // namespace cp
