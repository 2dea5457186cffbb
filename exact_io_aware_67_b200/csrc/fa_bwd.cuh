// fa_bwd.cuh -- backward kernels (work in progress: launcher only).
#pragma once
#include "fa_common.cuh"
#include "sm100.cuh"

namespace fa {

struct BwdParams {
  const __nv_bfloat16* q;
  const __nv_bfloat16* o;
  const __nv_bfloat16* dout;
  const float* lse;
  __nv_bfloat16* dq;
  __nv_bfloat16* dk;
  __nv_bfloat16* dv;
  float* dpsum;      // D = rowsum(dO o O), layout of lse
  float* dq_acc;     // fp32 dQ accumulator
  const int* cu_seqlens;
  int B, Hq, Hkv, N, group, total;
  float scale, scale_log2;
  unsigned long long wait_limit_ns;
};

inline size_t bwd_workspace_bytes(int Hq, int d, long tokens) {
  const size_t dsum = ((size_t)Hq * (size_t)tokens * 4 + 255) & ~(size_t)255;
  const size_t acc = (size_t)tokens * Hq * d * 4;
  return dsum + acc + 256 * 128;   // slack so the accumulator covers whole tiles
}

inline void bwd_carve_workspace(BwdParams& p, void* ws, long tokens, int d) {
  uint8_t* base = static_cast<uint8_t*>(ws);
  const size_t dsum = ((size_t)p.Hq * (size_t)tokens * 4 + 255) & ~(size_t)255;
  p.dpsum = reinterpret_cast<float*>(base);
  p.dq_acc = reinterpret_cast<float*>(base + dsum);
  (void)d;
}

inline cudaError_t launch_bwd(const CUtensorMap&, const CUtensorMap&, const CUtensorMap&,
                              const CUtensorMap&, const BwdParams&, int, bool, cudaStream_t) {
  return cudaErrorNotSupported;
}

// One warp waits on an mbarrier that nothing arrives on; the bounded wait
// must give up, record ERR_SELFTEST and return.
__global__ void watchdog_selftest_kernel(unsigned long long limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  const Watchdog wd{&g_fa_error, &abort_flag, limit_ns};
  if (threadIdx.x == 0) mbar_wait(&bar, 0, wd, ERR_SELFTEST);
  __syncwarp();
}

}  // namespace fa
