// Layout kernels (sm_100a, HBM-bound, bit-exact copies):
//
//  * Ulysses sequence<->head transpose, the local form of the all-to-all of
//    the "序列並行（Sequence Parallelism）" concept page (compassingai), 技術原理
//    §三 "Ulysses 的 AllToAll 轉置" ([S/N, H, d_h] -> [S, H/N, d_h], device i
//    taking head block i) and of the "Context Parallelism" write-up (pwwt.cn)
//    §2.3:  out[r][p*n + s][h'] = in[p][s][r*H/P + h'] and its inverse.
//  * Zigzag reorder: rank-major layout in which rank i holds chunks i and
//    2P-1-i of the 2P equal chunks ("长上下文序列并行训练深度解析" (mooersco),
//    timeline: Striped / zigzag load-balancing reorder), and its inverse.
//  * Striped reorder: token t on rank t mod P (same timeline, Striped
//    Attention), and its inverse.
//  * Head-block split of one rank's rows for the Ulysses all-to-all:
//    out[r][s][h'] = in[s][r*H/P + h'] (the send buffer whose block r goes
//    to rank r), and its inverse after the exchange.
//  * fp32 -> bf16 round-to-nearest-even conversion of input tensors.
//
// Both layout changes move whole runs of >= 256 contiguous bytes (one head
// block of one token, or one chunk of rows), so every kernel below is a
// strided block copy with the widest vector the run length and the pointers
// allow (16 bytes for every configuration in use), several loads in flight
// per thread, streaming cache hints, and a grid of whole waves over the SMs.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

namespace cp {

std::atomic<uint64_t>& launch_counter();

template <typename U>
__device__ __forceinline__ U ld_stream(const U* p) { return *p; }
template <>
__device__ __forceinline__ uint4 ld_stream<uint4>(const uint4* p) { return __ldcs(p); }
template <typename U>
__device__ __forceinline__ void st_stream(U* p, const U& v) { *p = v; }
template <>
__device__ __forceinline__ void st_stream<uint4>(uint4* p, const uint4& v) { __stcs(p, v); }

// Copy block (r, p) of the Ulysses transpose.  cu = units per (token, head
// block) chunk; S = P * n tokens.  dir 0: seq->head, 1: head->seq.
template <typename U, int ILP>
__global__ void __launch_bounds__(256) ulysses_kernel(const U* __restrict__ in, U* __restrict__ out, int P, int n,
                                                      uint32_t cu, int dir) {
  const int r = blockIdx.y / P;
  const int p = blockIdx.y % P;
  const uint32_t total = (uint32_t)n * cu;
  const size_t S = (size_t)P * n;
  const size_t head_base = ((size_t)r * S + (size_t)p * n) * cu;  // contiguous side
  const size_t stride = gridDim.x * blockDim.x;
  for (size_t u0 = (size_t)blockIdx.x * blockDim.x + threadIdx.x; u0 < total; u0 += stride * ILP) {
    U v[ILP];
    size_t dst[ILP];
#pragma unroll
    for (int i = 0; i < ILP; ++i) {
      const size_t u = u0 + i * stride;
      if (u < total) {
        const uint32_t s = (uint32_t)u / cu;
        const uint32_t c = (uint32_t)u - s * cu;
        const size_t seq_off = (((size_t)p * n + s) * P + r) * cu + c;
        const size_t src = dir == 0 ? seq_off : head_base + u;
        dst[i] = dir == 0 ? head_base + u : seq_off;
        v[i] = ld_stream(in + src);
      }
    }
#pragma unroll
    for (int i = 0; i < ILP; ++i) {
      const size_t u = u0 + i * stride;
      if (u < total) st_stream(out + dst[i], v[i]);
    }
  }
}

// Chunk oc of the rank-major zigzag layout is natural chunk nat(oc).
__device__ __forceinline__ int zigzag_natural_chunk(int oc, int P) {
  const int r = oc >> 1;
  return (oc & 1) ? 2 * P - 1 - r : r;
}

template <typename U, int ILP>
__global__ void __launch_bounds__(256) zigzag_kernel(const U* __restrict__ in, U* __restrict__ out, int P,
                                                     size_t chunk_units, int inverse) {
  const int chunks = 2 * P;
  const int b = blockIdx.y / chunks;
  const int oc = blockIdx.y % chunks;
  const int nc = zigzag_natural_chunk(oc, P);
  const size_t batch_base = (size_t)b * chunks * chunk_units;
  const size_t src_base = batch_base + (size_t)(inverse ? oc : nc) * chunk_units;
  const size_t dst_base = batch_base + (size_t)(inverse ? nc : oc) * chunk_units;
  const size_t stride = (size_t)gridDim.x * blockDim.x;
  for (size_t u0 = (size_t)blockIdx.x * blockDim.x + threadIdx.x; u0 < chunk_units; u0 += stride * ILP) {
    U v[ILP];
#pragma unroll
    for (int i = 0; i < ILP; ++i) {
      const size_t u = u0 + i * stride;
      if (u < chunk_units) v[i] = ld_stream(in + src_base + u);
    }
#pragma unroll
    for (int i = 0; i < ILP; ++i) {
      const size_t u = u0 + i * stride;
      if (u < chunk_units) st_stream(out + dst_base + u, v[i]);
    }
  }
}

// Striped layout: rank r holds positions r, r + P, ...; rank-major row
// r * n + a holds natural row a * P + r (n = S / P).  One CTA row-loop per
// batch entry; every row is copied with `upr` units.
template <typename U>
__global__ void __launch_bounds__(256) striped_kernel(const U* __restrict__ in, U* __restrict__ out, int P, int n,
                                                      uint32_t upr, int inverse) {
  const size_t S = (size_t)P * n;
  const size_t base = (size_t)blockIdx.y * S * upr;
  const uint32_t total = (uint32_t)(S * upr);
  for (uint32_t u = blockIdx.x * blockDim.x + threadIdx.x; u < total; u += gridDim.x * blockDim.x) {
    const uint32_t orow = u / upr;
    const uint32_t c = u - orow * upr;
    uint32_t irow;
    if (!inverse) {  // out row r*n + a <- natural row a*P + r
      const uint32_t r = orow / n, a = orow - r * n;
      irow = a * P + r;
    } else {         // out row a*P + r <- rank-major row r*n + a
      const uint32_t a = orow / P, r = orow - a * P;
      irow = r * n + a;
    }
    st_stream(out + base + (size_t)orow * upr + c, ld_stream(in + base + (size_t)irow * upr + c));
  }
}

// Head blocks: in [n][P][cu] <-> out [P][n][cu] (cu units per head block).
template <typename U, int ILP>
__global__ void __launch_bounds__(256) head_block_kernel(const U* __restrict__ in, U* __restrict__ out, int P, int n,
                                                         uint32_t cu, int inverse) {
  const int r = blockIdx.y;
  const uint32_t total = (uint32_t)n * cu;
  const size_t stride = (size_t)gridDim.x * blockDim.x;
  for (size_t u0 = (size_t)blockIdx.x * blockDim.x + threadIdx.x; u0 < total; u0 += stride * ILP) {
    U v[ILP];
    size_t dst[ILP];
#pragma unroll
    for (int i = 0; i < ILP; ++i) {
      const size_t u = u0 + i * stride;
      if (u < total) {
        const uint32_t s = (uint32_t)u / cu;
        const uint32_t c = (uint32_t)u - s * cu;
        const size_t seq_major = ((size_t)s * P + r) * cu + c;
        const size_t block_major = (size_t)r * total + u;
        dst[i] = inverse ? seq_major : block_major;
        v[i] = ld_stream(in + (inverse ? block_major : seq_major));
      }
    }
#pragma unroll
    for (int i = 0; i < ILP; ++i) {
      const size_t u = u0 + i * stride;
      if (u < total) st_stream(out + dst[i], v[i]);
    }
  }
}

__global__ void __launch_bounds__(256) f32_to_bf16_kernel(const float* __restrict__ in, __nv_bfloat16* __restrict__ out,
                                                          size_t n) {
  const size_t stride = (size_t)gridDim.x * blockDim.x;
  const size_t n8 = n / 8;
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n8; i += stride) {
    const float4 a = __ldcs(reinterpret_cast<const float4*>(in) + 2 * i);
    const float4 b = __ldcs(reinterpret_cast<const float4*>(in) + 2 * i + 1);
    __nv_bfloat162 o0 = __floats2bfloat162_rn(a.x, a.y), o1 = __floats2bfloat162_rn(a.z, a.w);
    __nv_bfloat162 o2 = __floats2bfloat162_rn(b.x, b.y), o3 = __floats2bfloat162_rn(b.z, b.w);
    uint4 pk;
    pk.x = *reinterpret_cast<uint32_t*>(&o0);
    pk.y = *reinterpret_cast<uint32_t*>(&o1);
    pk.z = *reinterpret_cast<uint32_t*>(&o2);
    pk.w = *reinterpret_cast<uint32_t*>(&o3);
    reinterpret_cast<uint4*>(out)[i] = pk;
  }
  for (size_t i = n8 * 8 + (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride)
    out[i] = __float2bfloat16_rn(in[i]);
}

// ------------------------------------------------------------------ host side
static int num_sms() {
  static int sms = 0;
  if (!sms) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (sms <= 0) sms = 148;
  }
  return sms;
}

// Widest unit (16/8/4/2/1 bytes) dividing the run length and both pointers.
static int unit_bytes(size_t run_bytes, const void* a, const void* b) {
  const uintptr_t al = reinterpret_cast<uintptr_t>(a) | reinterpret_cast<uintptr_t>(b);
  for (int u = 16; u > 1; u >>= 1)
    if (run_bytes % u == 0 && al % u == 0) return u;
  return 1;
}

// Grid x so that grid.x * grid.y covers a whole number of waves (8 blocks of
// 256 threads per SM) without exceeding the work.
static unsigned grid_x(size_t units_per_block_row, int ilp, unsigned gy) {
  const size_t need = (units_per_block_row + 256ull * ilp - 1) / (256ull * ilp);
  const size_t wave = (size_t)num_sms() * 8;
  size_t gx = (wave + gy - 1) / gy;
  if (gx > need) gx = need;
  if (gx < 1) gx = 1;
  return (unsigned)gx;
}

template <typename U>
static cudaError_t ulysses_t(const void* in, void* out, int P, int n, size_t chunk_bytes, int dir, cudaStream_t st) {
  constexpr int ILP = 4;
  const uint32_t cu = (uint32_t)(chunk_bytes / sizeof(U));
  const unsigned gy = (unsigned)(P * P);
  dim3 grid(grid_x((size_t)n * cu, ILP, gy), gy);
  ulysses_kernel<U, ILP><<<grid, 256, 0, st>>>(static_cast<const U*>(in), static_cast<U*>(out), P, n, cu, dir);
  launch_counter()++;
  return cudaGetLastError();
}

cudaError_t launch_ulysses(const void* in, void* out, int P, int n, size_t chunk_bytes, int dir, cudaStream_t st) {
  switch (unit_bytes(chunk_bytes, in, out)) {
    case 16: return ulysses_t<uint4>(in, out, P, n, chunk_bytes, dir, st);
    case 8: return ulysses_t<uint2>(in, out, P, n, chunk_bytes, dir, st);
    case 4: return ulysses_t<uint32_t>(in, out, P, n, chunk_bytes, dir, st);
    case 2: return ulysses_t<uint16_t>(in, out, P, n, chunk_bytes, dir, st);
    default: return ulysses_t<uint8_t>(in, out, P, n, chunk_bytes, dir, st);
  }
}

template <typename U>
static cudaError_t zigzag_t(const void* in, void* out, int P, int batch, size_t chunk_bytes, int inverse,
                            cudaStream_t st) {
  constexpr int ILP = 4;
  const size_t units = chunk_bytes / sizeof(U);
  const unsigned gy = (unsigned)(batch * 2 * P);
  dim3 grid(grid_x(units, ILP, gy), gy);
  zigzag_kernel<U, ILP><<<grid, 256, 0, st>>>(static_cast<const U*>(in), static_cast<U*>(out), P, units, inverse);
  launch_counter()++;
  return cudaGetLastError();
}

cudaError_t launch_zigzag(const void* in, void* out, int P, int batch, size_t chunk_bytes, int inverse,
                          cudaStream_t st) {
  switch (unit_bytes(chunk_bytes, in, out)) {
    case 16: return zigzag_t<uint4>(in, out, P, batch, chunk_bytes, inverse, st);
    case 8: return zigzag_t<uint2>(in, out, P, batch, chunk_bytes, inverse, st);
    case 4: return zigzag_t<uint32_t>(in, out, P, batch, chunk_bytes, inverse, st);
    case 2: return zigzag_t<uint16_t>(in, out, P, batch, chunk_bytes, inverse, st);
    default: return zigzag_t<uint8_t>(in, out, P, batch, chunk_bytes, inverse, st);
  }
}

template <typename U>
static cudaError_t striped_t(const void* in, void* out, int P, int n, int batch, size_t row_bytes, int inverse,
                            cudaStream_t st) {
  const uint32_t upr = (uint32_t)(row_bytes / sizeof(U));
  const size_t total = (size_t)P * n * upr;
  size_t gx = (total + 255) / 256;
  const size_t wave = (size_t)num_sms() * 8;
  if (gx > wave) gx = wave;
  dim3 grid((unsigned)gx, (unsigned)batch);
  striped_kernel<U><<<grid, 256, 0, st>>>(static_cast<const U*>(in), static_cast<U*>(out), P, n, upr, inverse);
  launch_counter()++;
  return cudaGetLastError();
}

cudaError_t launch_striped(const void* in, void* out, int P, int S, int batch, size_t row_bytes, int inverse,
                           cudaStream_t st) {
  const int n = S / P;
  switch (unit_bytes(row_bytes, in, out)) {
    case 16: return striped_t<uint4>(in, out, P, n, batch, row_bytes, inverse, st);
    case 8: return striped_t<uint2>(in, out, P, n, batch, row_bytes, inverse, st);
    case 4: return striped_t<uint32_t>(in, out, P, n, batch, row_bytes, inverse, st);
    case 2: return striped_t<uint16_t>(in, out, P, n, batch, row_bytes, inverse, st);
    default: return striped_t<uint8_t>(in, out, P, n, batch, row_bytes, inverse, st);
  }
}

template <typename U>
static cudaError_t head_block_t(const void* in, void* out, int P, int n, size_t chunk_bytes, int inverse,
                                cudaStream_t st) {
  constexpr int ILP = 4;
  const uint32_t cu = (uint32_t)(chunk_bytes / sizeof(U));
  dim3 grid(grid_x((size_t)n * cu, ILP, (unsigned)P), (unsigned)P);
  head_block_kernel<U, ILP><<<grid, 256, 0, st>>>(static_cast<const U*>(in), static_cast<U*>(out), P, n, cu,
                                                   inverse);
  launch_counter()++;
  return cudaGetLastError();
}

cudaError_t launch_head_blocks(const void* in, void* out, int P, int n, size_t chunk_bytes, int inverse,
                               cudaStream_t st) {
  switch (unit_bytes(chunk_bytes, in, out)) {
    case 16: return head_block_t<uint4>(in, out, P, n, chunk_bytes, inverse, st);
    case 8: return head_block_t<uint2>(in, out, P, n, chunk_bytes, inverse, st);
    case 4: return head_block_t<uint32_t>(in, out, P, n, chunk_bytes, inverse, st);
    case 2: return head_block_t<uint16_t>(in, out, P, n, chunk_bytes, inverse, st);
    default: return head_block_t<uint8_t>(in, out, P, n, chunk_bytes, inverse, st);
  }
}

cudaError_t launch_f32_to_bf16(const float* in, void* out, size_t n, cudaStream_t st) {
  if (n == 0) return cudaSuccess;
  const size_t need = (n / 8 + 255) / 256 + 1;
  size_t g = (size_t)num_sms() * 8;
  if (g > need) g = need;
  f32_to_bf16_kernel<<<(unsigned)g, 256, 0, st>>>(in, static_cast<__nv_bfloat16*>(out), n);
  launch_counter()++;
  return cudaGetLastError();
}

}  // namespace cp
