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
};

struct FwdParams {
  __nv_bfloat16* o;
  float* lse;
  const int* cu_seqlens;   // nullptr for dense inputs
  int B, Hq, Hkv, N, group;
  int total;               // token rows of a varlen batch
  int num_qblocks;         // ceil(N / 256)
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
