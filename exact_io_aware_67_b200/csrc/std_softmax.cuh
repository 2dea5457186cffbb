// std_softmax.cuh -- the softmax step of *standard* attention, for the
// comparator that measures what the tiled kernels avoid.
//
// Standard attention (tutorial 「注意力机制基础」 2.1, 2.2.2) materialises
// S = Q K^T in HBM, reads it back for a row softmax that writes P to HBM,
// and reads P again for O = P V: 2 (4 N^2 + 4 N d) bytes per head at 16-bit
// elements.  The two products run in a library GEMM; this kernel is the
// middle step: read one bf16 row of S, write the bf16 row of P and the row's
// log-sum-exp.  It is bound by HBM bandwidth (2 bytes read + 2 written per
// element), so the design is about coalescing and a single pass over HBM:
//  * one CTA per row (one warp per row when a row has at most 1024 values),
//    each thread holding up to 32 values in registers, loaded and stored as
//    16-byte vectors with consecutive threads on consecutive vectors;
//  * the row max and the row sum are reduced in registers, then across the
//    warp with shuffles and across warps through shared memory;
//  * with the causal mask, entries j > i of row i read as -inf and P_ij = 0.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace fa {

struct StdSoftmaxParams {
  const __nv_bfloat16* s;   // [rows][n]
  __nv_bfloat16* p;         // [rows][n]
  float* lse;               // [rows]
  long rows;
  int n;                    // row length; also the query count per head (square S)
  int causal;
  float scale_log2;         // scale * log2(e)
};

constexpr int STD_VPT = 32;   // values per thread (four 16-byte vectors)

__device__ __forceinline__ float std_warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float std_warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// One row per group of G threads (G = blockDim.x for a CTA per row, 32 for a
// warp per row).  Vector c of the row (8 values) belongs to thread c mod G.
template <bool WARP_ROW>
__global__ void std_softmax_kernel(const StdSoftmaxParams p) {
  __shared__ float red[32];
  const int G = WARP_ROW ? 32 : (int)blockDim.x;
  const int tid = WARP_ROW ? (int)(threadIdx.x & 31) : (int)threadIdx.x;
  const long row = WARP_ROW ? (long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5)
                            : (long)blockIdx.x;
  if (row >= p.rows) return;   // whole warps (warp per row) or whole CTAs leave
  const int i = (int)(row % p.n);                  // query index within its head
  const int lim = p.causal ? i + 1 : p.n;          // allowed columns [0, lim)
  const int nvec = p.n / 8;
  const uint4* src = reinterpret_cast<const uint4*>(p.s + row * (long)p.n);
  uint4* dst = reinterpret_cast<uint4*>(p.p + row * (long)p.n);

  float x[STD_VPT];
  float mx = -INFINITY;
#pragma unroll
  for (int k = 0; k < STD_VPT / 8; ++k) {
    const int c = tid + k * G;
    uint4 u = make_uint4(0u, 0u, 0u, 0u);
    if (c < nvec) u = __ldcs(src + c);   // streamed once: do not keep in L1
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const uint32_t half = (e & 1) ? (w[e >> 1] >> 16) : (w[e >> 1] & 0xffffu);
      const float v = __uint_as_float(half << 16) * p.scale_log2;
      const int col = 8 * c + e;
      x[8 * k + e] = (c < nvec && col < lim) ? v : -INFINITY;
      mx = fmaxf(mx, x[8 * k + e]);
    }
  }
  // row max
  mx = std_warp_max(mx);
  if (!WARP_ROW) {
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = mx;
    __syncthreads();
    float m2 = -INFINITY;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) m2 = fmaxf(m2, red[w]);
    mx = m2;
    __syncthreads();
  }
  float sum = 0.f;
#pragma unroll
  for (int k = 0; k < STD_VPT; ++k) {
    x[k] = exp2f(x[k] - mx);   // masked and padding entries: exp2(-inf) = 0
    sum += x[k];
  }
  sum = std_warp_sum(sum);
  if (!WARP_ROW) {
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = sum;
    __syncthreads();
    float s2 = 0.f;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) s2 += red[w];
    sum = s2;
  }
  const float inv = 1.f / sum;
#pragma unroll
  for (int k = 0; k < STD_VPT / 8; ++k) {
    const int c = tid + k * G;
    if (c < nvec) {
      uint32_t w[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const __nv_bfloat162 h = __floats2bfloat162_rn(x[8 * k + 2 * e] * inv,
                                                       x[8 * k + 2 * e + 1] * inv);
        w[e] = *reinterpret_cast<const uint32_t*>(&h);
      }
      __stcs(dst + c, make_uint4(w[0], w[1], w[2], w[3]));
    }
  }
  if (tid == 0) p.lse[row] = (mx + log2f(sum)) * 0.69314718055994530942f;
}

// Largest row the kernel takes: 1024 threads x 32 values.
constexpr int STD_MAX_N = 1024 * STD_VPT;

inline cudaError_t launch_std_softmax(const StdSoftmaxParams& p, cudaStream_t stream) {
  const int nvec = p.n / 8;
  const int threads_needed = (nvec + STD_VPT / 8 - 1) / (STD_VPT / 8);
  if (threads_needed <= 32) {
    const int rows_per_cta = 8;   // one warp per row
    const long grid = (p.rows + rows_per_cta - 1) / rows_per_cta;
    std_softmax_kernel<true><<<(unsigned)grid, 32 * rows_per_cta, 0, stream>>>(p);
  } else {
    const int threads = (threads_needed + 31) / 32 * 32;
    std_softmax_kernel<false><<<(unsigned)p.rows, threads, 0, stream>>>(p);
  }
  return cudaGetLastError();
}

}  // namespace fa
