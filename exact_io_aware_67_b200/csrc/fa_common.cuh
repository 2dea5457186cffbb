// fa_common.cuh -- parameter blocks, error codes and small helpers shared by
// the kernels of libfa.so.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>

#include "sm100.cuh"

namespace fa {

// Codes written to the device error word when a bounded wait gives up:
// 0x1xx forward kernel, 0x2xx backward kernels, 0x3xx self-test, 0x4xx decode.
enum : int {
  ERR_FWD_KV_EMPTY = 0x101,
  ERR_FWD_Q_FULL = 0x102,
  ERR_FWD_KV_FULL = 0x103,
  ERR_FWD_P_FULL = 0x104,
  ERR_FWD_S_FULL = 0x105,
  ERR_FWD_O_DONE = 0x106,
  ERR_FWD_S_FREE = 0x107,
  ERR_FWD_P_FREE = 0x108,
  ERR_BWD_LOAD_EMPTY = 0x201,
  ERR_BWD_KV_FULL = 0x202,
  ERR_BWD_Q_FULL = 0x203,
  ERR_BWD_S_FULL = 0x204,
  ERR_BWD_P_FULL = 0x205,
  ERR_BWD_DS_FULL = 0x206,
  ERR_BWD_DQ_FULL = 0x207,
  ERR_BWD_DQ_EMPTY = 0x208,
  ERR_BWD_DKV_DONE = 0x209,
  ERR_BWD_DP_FULL = 0x20a,
  ERR_BWD_STATS = 0x20b,
  ERR_BWD_SMEM_ALIGN = 0x20c,
  ERR_SELFTEST = 0x301,
  ERR_DEC_KV_FULL = 0x401,
  ERR_DEC_KV_EMPTY = 0x402,
  // cu_seqlens validation (validate_cu_kernel): the lowest failing rule wins
  ERR_CU_FIRST = 0x501,        // cu[0] != 0
  ERR_CU_DECREASING = 0x502,   // cu[b + 1] < cu[b]
  ERR_CU_TOO_LONG = 0x503,     // a sequence longer than N
  ERR_CU_TOTAL = 0x504,        // cu[B] > total_tokens
};

struct FwdParams {
  __nv_bfloat16* o;
  __nv_bfloat16* o_lo;     // optional: O - bf16(O), rounded to bf16 (nullptr: not written)
  float* lse;
  const int* cu_seqlens;   // nullptr for dense inputs
  int B, Hq, Hkv, N, group;
  int total;               // token rows of a varlen batch
  int num_qblocks;         // ceil(N / 256)
  int order_chunk;         // (sequence, kv head) pairs per dispatch chunk
  float scale_log2;        // scale * log2(e)
  unsigned long long wait_limit_ns;
  // block-sparse mode only: tile (qt, kt) of sequence b and kv head hk is
  // allowed iff bmask[b * bm_sb + hk * bm_sh + qt * bm_nt + kt] != 0
  const uint8_t* bmask;
  long bm_sb, bm_sh;
  int bm_nt;
};

// Largest N of the block-sparse kernels: the per-CTA tile lists live in
// shared memory.
constexpr int FA_SPARSE_MAX_TILES = 512;

// Device error word of the library (first error wins; 0 = none).  All
// kernels live in one translation unit, so one definition serves them all.
__device__ int g_fa_error = 0;

// Token range [*start, *start + *len) of sequence b of a variable-length
// batch, clamped to [0, total]: whatever cu_seqlens holds (decreasing,
// negative, past the caller's allocation), every row a kernel derives from
// it lies inside the buffers.  The results of such a batch are undefined;
// validate_cu_kernel reports it.
__device__ __forceinline__ void seq_range(const int* cu, int b, int total, int* start,
                                          int* len) {
  const int s = min(max(cu[b], 0), total);
  const int e = min(max(cu[b + 1], s), total);
  *start = s;
  *len = e - s;
}

// Checks a cu_seqlens array with one block: cu[0] == 0, non-decreasing,
// every length at most N, cu[B] <= total.  The lowest failing rule's code
// goes to the error word (first error wins there).  Reads cu[0..B] only.
__global__ void __launch_bounds__(256) validate_cu_kernel(const int* cu, int B, int N,
                                                           int total) {
  __shared__ int worst;
  if (threadIdx.x == 0) worst = 0x7fffffff;
  __syncthreads();
  int code = 0x7fffffff;
  for (int b = threadIdx.x; b <= B; b += blockDim.x) {
    const int c = cu[b];
    if (b == 0 && c != 0) code = min(code, (int)ERR_CU_FIRST);
    if (b < B) {
      const int nxt = cu[b + 1];
      if (nxt < c) code = min(code, (int)ERR_CU_DECREASING);
      else if ((long)nxt - c > (long)N) code = min(code, (int)ERR_CU_TOO_LONG);
    } else if (c > total) {
      code = min(code, (int)ERR_CU_TOTAL);
    }
  }
  atomicMin(&worst, code);
  __syncthreads();
  if (threadIdx.x == 0 && worst != 0x7fffffff) atomicCAS(&g_fa_error, 0, worst);
}

__device__ __forceinline__ uint8_t* align_1024(uint8_t* p) {
  const uint32_t a = smem_u32(p);
  return p + (((a + 1023u) & ~1023u) - a);
}

// Bounded wait that ignores the abort flag: used while winding down, to let
// asynchronous copies and MMAs that were already issued complete.
__device__ __forceinline__ bool mbar_wait_drain(uint64_t* bar, uint32_t parity,
                                                unsigned long long limit_ns) {
  const uint32_t a = smem_u32(bar);
  if (mbar_try_wait(a, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(a, parity)) return true;
    if ((it & 15u) == 0 && globaltimer_ns() - t0 > limit_ns) return false;
  }
}

}  // namespace fa
