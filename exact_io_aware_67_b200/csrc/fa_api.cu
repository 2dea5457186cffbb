// fa_api.cu -- host side of libfa.so: argument validation, TMA descriptor
// encoding, launch configuration, and the C entry points declared in
// include/fa.h.  The library allocates no device memory (the one exception
// is the fixed scratch array behind fa_bwd_noalloc, a file-scope device
// variable) and never synchronises the caller's stream.
#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <cstdint>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include "fa.h"
#include "fa_bwd.cuh"
#include "fa_decode.cuh"
#include "fa_fwd.cuh"
#include "std_softmax.cuh"

namespace {

std::atomic<unsigned long long> g_wait_limit_ns{2000000000ull};
thread_local int t_last_cuda_error = 0;
// Optional events recorded around the main kernel of the next calls made by
// this thread (see fa_set_profile_events).
thread_local cudaEvent_t t_prof_begin = nullptr;
thread_local cudaEvent_t t_prof_end = nullptr;

// Record a failed CUDA call for fa_last_cuda_error() and map it to a status;
// with FA_DEBUG set in the environment the failing site is printed.
fa_status cuda_fail(cudaError_t e, const char* site) {
  t_last_cuda_error = (int)e;
  if (std::getenv("FA_DEBUG") != nullptr)
    std::fprintf(stderr, "libfa: %s failed: %s\n", site, cudaGetErrorString(e));
  return FA_ERR_CUDA;
}

// With FA_DEBUG_VALIDATE set in the environment, every varlen fa_fwd /
// fa_bwd call first enqueues validate_cu_kernel on its stream.
bool debug_validate() {
  static const bool on = std::getenv("FA_DEBUG_VALIDATE") != nullptr;
  return on;
}

cudaError_t launch_validate_cu(const int* cu, int B, int N, int total, cudaStream_t stream) {
  fa::validate_cu_kernel<<<1, 256, 0, stream>>>(cu, B, N, total);
  return cudaGetLastError();
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static std::atomic<PFN_cuTensorMapEncodeTiled_v12000> fn{nullptr};
  PFN_cuTensorMapEncodeTiled_v12000 f = fn.load();
  if (f == nullptr) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess && ptr != nullptr) {
      f = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
      fn.store(f);
    }
  }
  return f;
}

// Tensor map over a token-major 16-bit tensor [batches][rows][heads][d]
// (bf16 by default; the backward's fp16 operand copies use the same shape):
// box = 64 d-elements (128 B, 128-byte swizzle) x 1 head x 128 rows.
// Rows past `rows` read as zeros.
bool encode_rows_map(CUtensorMap* m, const void* base, int d, int heads, long rows,
                     int batches,
                     CUtensorMapDataType dtype = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = encode_fn();
  if (enc == nullptr) return false;
  const cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)heads, (cuuint64_t)rows,
                              (cuuint64_t)batches};
  const cuuint64_t strides[3] = {(cuuint64_t)d * 2, (cuuint64_t)heads * d * 2,
                                 (cuuint64_t)rows * heads * d * 2};
  const cuuint32_t box[4] = {64, 1, 128, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  const CUresult r =
      enc(m, dtype, 4, const_cast<void*>(base), dims, strides, box,
          estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Make the device that owns `ptr` current for the calling thread.  A thread
// that has not touched CUDA yet (autograd's worker, a user thread) has no
// current context, and tensor-map encoding needs one.  Host pointers are
// rejected.
fa_status bind_device_of(const void* ptr) {
  cudaPointerAttributes a{};
  cudaError_t e = cudaPointerGetAttributes(&a, ptr);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return FA_ERR_INVALID_ARG;
  }
  if (a.type != cudaMemoryTypeDevice && a.type != cudaMemoryTypeManaged)
    return FA_ERR_INVALID_ARG;
  // cudaSetDevice also binds the device's primary context to this thread;
  // cudaGetDevice alone would report device 0 without binding anything.
  e = cudaSetDevice(a.device);
  if (e != cudaSuccess) return cuda_fail(e, "select device");
  return FA_OK;
}

struct Dims {
  int B, Hq, Hkv, N, d, total;
  bool varlen;
  long rows() const { return varlen ? (long)total : (long)N; }
  int batches() const { return varlen ? 1 : B; }
  long tokens() const { return varlen ? (long)total : (long)B * N; }
};

// Shared validation of the size arguments.  Returns FA_OK and sets *empty
// when there is nothing to compute.
fa_status check_dims(const Dims& s, float scale, bool* empty) {
  *empty = false;
  if (s.d != 64 && s.d != 128) return FA_ERR_UNSUPPORTED;
  if (s.B < 0 || s.Hq < 1 || s.Hkv < 1 || s.Hq % s.Hkv != 0) return FA_ERR_INVALID_ARG;
  if (!(scale > 0.f) || !std::isfinite(scale)) return FA_ERR_INVALID_ARG;
  if (s.N < 1 || s.N > (1 << 24)) return FA_ERR_INVALID_ARG;
  if (s.varlen && s.total < 0) return FA_ERR_INVALID_ARG;
  if (s.Hq > 65535) return FA_ERR_INVALID_ARG;
  if (s.B == 0 || (s.varlen && s.total == 0)) {
    *empty = true;
    return FA_OK;
  }
  const long long qblocks = (s.N + 255) / 256;
  if (qblocks * s.Hq * s.B > 0x7fffffffLL) return FA_ERR_INVALID_ARG;
  if (s.tokens() * s.Hq * (long long)s.d > (1LL << 40)) return FA_ERR_INVALID_ARG;
  return FA_OK;
}

template <int D, bool CAUSAL, bool SPARSE = false>
cudaError_t launch_fwd(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                       const fa::FwdParams& p, cudaStream_t stream) {
  auto kern = fa::fwd_kernel<D, CAUSAL, SPARSE>;
  const int smem = fa::FwdLayout<D>::ALLOC;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  // dispatch chunks (see the kernel): one chunk of every (sequence, kv head)
  // pair unless K and V together are at least twice the L2; then the fewest
  // pairs whose blocks make at least two waves (one block per SM)
  fa::FwdParams pc = p;
  {
    int dev = 0, sms = 0, l2 = 0;
    e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&l2, cudaDevAttrL2CacheSize, dev);
    if (e != cudaSuccess) return e;
    const long npairs = (long)p.B * p.Hkv;
    const long per_pair = (long)p.group * p.num_qblocks;
    const double kv_bytes = 2.0 * (double)p.total * p.Hkv * D * 2.0;
    const long want = (2L * sms + per_pair - 1) / per_pair;
    pc.order_chunk = (kv_bytes >= 2.0 * l2) ? (int)std::max(1L, std::min(npairs, want))
                                            : (int)npairs;
  }
  const unsigned grid = (unsigned)p.num_qblocks * p.Hq * p.B;
  if (t_prof_begin != nullptr) cudaEventRecord(t_prof_begin, stream);
  kern<<<grid, fa::FWD_THREADS, smem, stream>>>(mq, mk, mv, pc);
  e = cudaGetLastError();
  if (e == cudaSuccess && t_prof_end != nullptr) e = cudaEventRecord(t_prof_end, stream);
  return e;
}

// Fixed scratch for fa_bwd_noalloc(): file-scope device memory, so that
// callers who cannot allocate still get a working backward.  In host code
// this name is only a stand-in for the symbol; its device address comes
// from cudaGetSymbolAddress, looked up once per device and cached.
static __device__ __align__(256) unsigned char g_fa_bwd_scratch[FA_BWD_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::atomic<void*> g_scratch_addr[kMaxDevices];

// Device address of g_fa_bwd_scratch on the current device (nullptr and a
// recorded error on failure).
void* scratch_on_current_device() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  void* ptr = g_scratch_addr[dev].load();
  if (ptr == nullptr) {
    const cudaError_t e = cudaGetSymbolAddress(&ptr, g_fa_bwd_scratch);
    if (e != cudaSuccess) {
      cuda_fail(e, "scratch symbol address");
      return nullptr;
    }
    g_scratch_addr[dev].store(ptr);
  }
  return ptr;
}

// Block mask of the block-sparse entry points: bytes [*][*][nt][nt] with
// nt = ceil(N / 128), strides (in elements) per sequence and per kv head.
struct BlockMask {
  const unsigned char* m;
  long sb, sh;
};

fa_status check_mask(const BlockMask& bm, const void* cu_seqlens, int N) {
  if (bm.m == nullptr) return FA_OK;
  if (cu_seqlens != nullptr) return FA_ERR_UNSUPPORTED;   // dense batches only
  if ((N + 127) / 128 > fa::FA_SPARSE_MAX_TILES) return FA_ERR_UNSUPPORTED;
  if (bm.sb < 0 || bm.sh < 0) return FA_ERR_INVALID_ARG;
  return FA_OK;
}

fa_status fwd_impl(const void* q, const void* k, const void* v, void* o, float* lse, void* o_lo,
                   int B, int Hq, int Hkv, int N, int d, float scale, int causal,
                   const int* cu_seqlens, int total_tokens, const BlockMask& bm,
                   cudaStream_t stream) {
  const Dims s{B, Hq, Hkv, N, d, total_tokens, cu_seqlens != nullptr};
  bool empty = false;
  fa_status st = check_dims(s, scale, &empty);
  if (st != FA_OK) return st;
  if (!q || !k || !v || !o || !lse) return FA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse) ||
      !aligned16(o_lo))
    return FA_ERR_INVALID_ARG;
  if (o_lo != nullptr && o_lo == o) return FA_ERR_INVALID_ARG;
  st = check_mask(bm, cu_seqlens, N);
  if (st != FA_OK) return st;
  if (empty) return FA_OK;
  st = bind_device_of(q);
  if (st != FA_OK) return st;

  CUtensorMap mq, mk, mv;
  if (!encode_rows_map(&mq, q, d, Hq, s.rows(), s.batches()) ||
      !encode_rows_map(&mk, k, d, Hkv, s.rows(), s.batches()) ||
      !encode_rows_map(&mv, v, d, Hkv, s.rows(), s.batches()))
    return cuda_fail(cudaErrorInvalidValue, "tensor map encode");

  fa::FwdParams p{};
  p.o = static_cast<__nv_bfloat16*>(o);
  p.o_lo = static_cast<__nv_bfloat16*>(o_lo);
  p.lse = lse;
  p.cu_seqlens = cu_seqlens;
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.N = N;
  p.group = Hq / Hkv;
  p.total = s.varlen ? total_tokens : B * N;
  p.num_qblocks = (N + 255) / 256;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.wait_limit_ns = g_wait_limit_ns.load();
  p.bmask = bm.m;
  p.bm_sb = bm.sb;
  p.bm_sh = bm.sh;
  p.bm_nt = (N + 127) / 128;

  cudaError_t e;
  if (cu_seqlens != nullptr && debug_validate()) {
    e = launch_validate_cu(cu_seqlens, B, N, total_tokens, stream);
    if (e != cudaSuccess) return cuda_fail(e, "cu_seqlens validation launch");
  }
  if (bm.m == nullptr) {
    if (d == 64)
      e = causal ? launch_fwd<64, true>(mq, mk, mv, p, stream)
                 : launch_fwd<64, false>(mq, mk, mv, p, stream);
    else
      e = causal ? launch_fwd<128, true>(mq, mk, mv, p, stream)
                 : launch_fwd<128, false>(mq, mk, mv, p, stream);
  } else {
    if (d == 64)
      e = causal ? launch_fwd<64, true, true>(mq, mk, mv, p, stream)
                 : launch_fwd<64, false, true>(mq, mk, mv, p, stream);
    else
      e = causal ? launch_fwd<128, true, true>(mq, mk, mv, p, stream)
                 : launch_fwd<128, false, true>(mq, mk, mv, p, stream);
  }
  return e == cudaSuccess ? FA_OK : cuda_fail(e, "forward launch");
}



fa_status bwd_impl(const void* q, const void* k, const void* v, const void* o, const float* lse,
                   const void* o_lo, const void* dO, void* dq, void* dk, void* dv, void* workspace,
                   size_t workspace_bytes, int B, int Hq, int Hkv, int N, int d, float scale,
                   int causal, const int* cu_seqlens, int total_tokens, const BlockMask& bm,
                   cudaStream_t stream) {
  const Dims s{B, Hq, Hkv, N, d, total_tokens, cu_seqlens != nullptr};
  bool empty = false;
  fa_status st = check_dims(s, scale, &empty);
  if (st != FA_OK) return st;
  if (!q || !k || !v || !o || !lse || !dO || !dq || !dk || !dv) return FA_ERR_INVALID_ARG;
  const void* ptrs[] = {q, k, v, o, lse, dO, dq, dk, dv, o_lo};
  for (const void* ptr : ptrs)
    if (!aligned16(ptr)) return FA_ERR_INVALID_ARG;
  if (o_lo != nullptr && o_lo == o) return FA_ERR_INVALID_ARG;
  st = check_mask(bm, cu_seqlens, N);
  if (st != FA_OK) return st;
  if (empty) return FA_OK;
  const size_t need = fa::bwd_workspace_bytes(B, Hq, Hkv, N, d, s.tokens(), s.varlen);
  if (workspace == nullptr || workspace_bytes < need ||
      (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return FA_ERR_WORKSPACE;
  st = bind_device_of(q);
  if (st != FA_OK) return st;

  fa::BwdParams p{};
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.k = static_cast<const __nv_bfloat16*>(k);
  p.v = static_cast<const __nv_bfloat16*>(v);
  p.o = static_cast<const __nv_bfloat16*>(o);
  p.o_lo = static_cast<const __nv_bfloat16*>(o_lo);
  p.dout = static_cast<const __nv_bfloat16*>(dO);
  p.lse = lse;
  p.dq = static_cast<__nv_bfloat16*>(dq);
  p.dk = static_cast<__nv_bfloat16*>(dk);
  p.dv = static_cast<__nv_bfloat16*>(dv);
  p.cu_seqlens = cu_seqlens;
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.N = N;
  p.group = Hq / Hkv;
  p.total = s.varlen ? total_tokens : B * N;
  p.scale = scale;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.wait_limit_ns = g_wait_limit_ns.load();
  p.bmask = bm.m;
  p.bm_sb = bm.sb;
  p.bm_sh = bm.sh;
  p.bm_nt = (N + 127) / 128;
  fa::bwd_carve_workspace(p, workspace, s.tokens(), d);
  // the main kernel's products read the fp16 copies the preprocess writes
  CUtensorMap mq, mk, mv, mdo;
  const CUtensorMapDataType f16 = CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  if (!encode_rows_map(&mq, p.q16, d, Hq, s.rows(), s.batches(), f16) ||
      !encode_rows_map(&mk, p.k16, d, Hkv, s.rows(), s.batches(), f16) ||
      !encode_rows_map(&mv, p.v16, d, Hkv, s.rows(), s.batches(), f16) ||
      !encode_rows_map(&mdo, p.do16, d, Hq, s.rows(), s.batches(), f16))
    return cuda_fail(cudaErrorInvalidValue, "tensor map encode");
  if (cu_seqlens != nullptr && debug_validate()) {
    const cudaError_t ev = launch_validate_cu(cu_seqlens, B, N, total_tokens, stream);
    if (ev != cudaSuccess) return cuda_fail(ev, "cu_seqlens validation launch");
  }

  const cudaError_t e =
      fa::launch_bwd(mq, mk, mv, mdo, p, d, causal != 0, stream, t_prof_begin, t_prof_end);
  return e == cudaSuccess ? FA_OK : cuda_fail(e, "backward launch");
}

}  // namespace

extern "C" {

fa_status fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, void* o_lo,
                 int B, int Hq, int Hkv, int N, int d, float scale, int causal,
                 const int* cu_seqlens, int total_tokens, cudaStream_t stream) {
  return fwd_impl(q, k, v, o, lse, o_lo, B, Hq, Hkv, N, d, scale, causal, cu_seqlens,
                  total_tokens, BlockMask{nullptr, 0, 0}, stream);
}

fa_status fa_fwd_blockmask(const void* q, const void* k, const void* v, void* o, float* lse,
                           void* o_lo, int B, int Hq, int Hkv, int N, int d, float scale,
                           int causal, const unsigned char* block_mask, long mask_batch_stride,
                           long mask_head_stride, cudaStream_t stream) {
  if (block_mask == nullptr) return FA_ERR_INVALID_ARG;
  return fwd_impl(q, k, v, o, lse, o_lo, B, Hq, Hkv, N, d, scale, causal, nullptr, B * N,
                  BlockMask{block_mask, mask_batch_stride, mask_head_stride}, stream);
}

size_t fa_bwd_workspace_size(int B, int Hq, int N, int d, int total_tokens) {
  if (B < 0 || Hq < 1 || N < 1 || (d != 64 && d != 128) || total_tokens < 0) return 0;
  // the size must serve a dense call (total_tokens = B * N) and a varlen
  // call with the same numbers, so take the larger of the two layouts; the
  // key/value head count is not an argument, so the K and V copies are sized
  // for Hkv = Hq, an upper bound for every grouping
  const size_t a = fa::bwd_workspace_bytes(B, Hq, Hq, N, d, (long)total_tokens, false);
  const size_t v = fa::bwd_workspace_bytes(B, Hq, Hq, N, d, (long)total_tokens, true);
  return a > v ? a : v;
}

fa_status fa_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse,
                 const void* o_lo, const void* dO, void* dq, void* dk, void* dv,
                 void* workspace, size_t workspace_bytes, int B, int Hq, int Hkv, int N, int d,
                 float scale, int causal, const int* cu_seqlens, int total_tokens,
                 cudaStream_t stream) {
  return bwd_impl(q, k, v, o, lse, o_lo, dO, dq, dk, dv, workspace, workspace_bytes, B, Hq, Hkv, N, d,
                  scale, causal, cu_seqlens, total_tokens, BlockMask{nullptr, 0, 0}, stream);
}

fa_status fa_bwd_blockmask(const void* q, const void* k, const void* v, const void* o,
                           const float* lse, const void* o_lo, const void* dO, void* dq,
                           void* dk, void* dv, void* workspace, size_t workspace_bytes, int B,
                           int Hq, int Hkv, int N, int d, float scale, int causal,
                           const unsigned char* block_mask, long mask_batch_stride,
                           long mask_head_stride, cudaStream_t stream) {
  if (block_mask == nullptr) return FA_ERR_INVALID_ARG;
  return bwd_impl(q, k, v, o, lse, o_lo, dO, dq, dk, dv, workspace, workspace_bytes, B, Hq, Hkv, N, d,
                  scale, causal, nullptr, B * N,
                  BlockMask{block_mask, mask_batch_stride, mask_head_stride}, stream);
}

fa_status fa_bwd_noalloc(const void* q, const void* k, const void* v, const void* o,
                         const float* lse, const void* o_lo, const void* dO, void* dq, void* dk,
                         void* dv, int B, int Hq, int Hkv, int N, int d, float scale, int causal,
                         const int* cu_seqlens, int total_tokens, cudaStream_t stream) {
  const Dims s{B, Hq, Hkv, N, d, total_tokens, cu_seqlens != nullptr};
  bool empty = false;
  fa_status st = check_dims(s, scale, &empty);
  if (st != FA_OK) return st;
  if (!q || !k || !v || !o || !lse || !dO || !dq || !dk || !dv) return FA_ERR_INVALID_ARG;
  if (empty) return FA_OK;
  const size_t need = fa::bwd_workspace_bytes(B, Hq, Hkv, N, d, s.tokens(), s.varlen);
  if (need > (size_t)FA_BWD_NOALLOC_SCRATCH_BYTES) return FA_ERR_WORKSPACE;
  st = bind_device_of(q);
  if (st != FA_OK) return st;
  void* scratch = scratch_on_current_device();
  if (scratch == nullptr) return FA_ERR_CUDA;
  return fa_bwd(q, k, v, o, lse, o_lo, dO, dq, dk, dv, scratch, FA_BWD_NOALLOC_SCRATCH_BYTES, B, Hq,
                Hkv, N, d, scale, causal, cu_seqlens, total_tokens, stream);
}

size_t fa_decode_workspace_size(int B, int Hq, int Lmax, int d) {
  if (B < 0 || Hq < 1 || Lmax < 1 || Lmax > (1 << 24) || (d != 64 && d != 128)) return 0;
  return fa::decode_workspace_bytes(B, Hq, Lmax, d);
}

fa_status fa_decode(const void* q, const void* k_cache, const void* v_cache, void* o,
                    float* lse, const int* cache_seqlens, int B, int Hq, int Hkv, int Lmax,
                    int d, float scale, void* workspace, size_t workspace_bytes,
                    cudaStream_t stream) {
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  if (B < 0 || Hq < 1 || Hkv < 1 || Hq % Hkv != 0) return FA_ERR_INVALID_ARG;
  if (Hq / Hkv > fa::DEC_GMAX) return FA_ERR_UNSUPPORTED;
  if (Lmax < 1 || Lmax > (1 << 24) || B > 65535 || Hkv > 65535) return FA_ERR_INVALID_ARG;
  if ((long long)B * Hq > 0x7fffffffLL) return FA_ERR_INVALID_ARG;
  if (!(scale > 0.f) || !std::isfinite(scale)) return FA_ERR_INVALID_ARG;
  if (B == 0) return FA_OK;
  if (!q || !k_cache || !v_cache || !o || !lse) return FA_ERR_INVALID_ARG;
  const void* ptrs[] = {q, k_cache, v_cache, o, lse};
  for (const void* ptr : ptrs)
    if (!aligned16(ptr)) return FA_ERR_INVALID_ARG;
  if (cache_seqlens != nullptr && (reinterpret_cast<uintptr_t>(cache_seqlens) & 3u) != 0)
    return FA_ERR_INVALID_ARG;
  const size_t need = fa::decode_workspace_bytes(B, Hq, Lmax, d);
  if (workspace == nullptr || workspace_bytes < need ||
      (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return FA_ERR_WORKSPACE;
  fa_status st = bind_device_of(q);
  if (st != FA_OK) return st;
  int dev = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return cuda_fail(e, "device attribute");

  CUtensorMap mk, mv;
  if (!encode_rows_map(&mk, k_cache, d, Hkv, Lmax, B) ||
      !encode_rows_map(&mv, v_cache, d, Hkv, Lmax, B))
    return cuda_fail(cudaErrorInvalidValue, "tensor map encode");
  fa::DecodeParams p{};
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.o = static_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  p.seqlens = cache_seqlens;
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.Lmax = Lmax;
  p.group = Hq / Hkv;
  // one CTA per SM (at most the number of tiles when every cache is full;
  // with device-side lengths some CTAs may get empty ranges)
  const long long tiles_full = (long long)B * Hkv * ((Lmax + 127) / 128);
  p.grid = (int)std::min<long long>(std::min(sms, fa::DEC_MAX_GRID), tiles_full);
  char* wsp = static_cast<char*>(workspace);
  p.boff = reinterpret_cast<long long*>(wsp);
  wsp += ((size_t)(B + 1) * 8 + 255) & ~(size_t)255;
  const size_t rows = (size_t)B * Hq + (size_t)fa::DEC_MAX_GRID * fa::DEC_GMAX;
  p.o_part = reinterpret_cast<float*>(wsp);
  wsp += (rows * d * 4 + 255) & ~(size_t)255;
  p.lse_part = reinterpret_cast<float*>(wsp);
  p.scale_log2 = scale * 1.4426950408889634f;
  p.wait_limit_ns = g_wait_limit_ns.load();
  e = fa::launch_decode(mk, mv, p, d, stream);
  return e == cudaSuccess ? FA_OK : cuda_fail(e, "decode launch");
}

fa_status fa_std_softmax(const void* s, void* p, float* lse, int BH, int N, float scale,
                         int causal, cudaStream_t stream) {
  if (BH < 0 || N < 1) return FA_ERR_INVALID_ARG;
  if (N % 8 != 0 || N > fa::STD_MAX_N) return FA_ERR_UNSUPPORTED;
  if (!(scale > 0.f) || !std::isfinite(scale)) return FA_ERR_INVALID_ARG;
  if ((long long)BH * N > 0x7fffffffLL) return FA_ERR_INVALID_ARG;
  if (BH == 0) return FA_OK;
  if (!s || !p || !lse || !aligned16(s) || !aligned16(p) || !aligned16(lse))
    return FA_ERR_INVALID_ARG;
  const fa_status st = bind_device_of(s);
  if (st != FA_OK) return st;
  fa::StdSoftmaxParams prm{};
  prm.s = static_cast<const __nv_bfloat16*>(s);
  prm.p = static_cast<__nv_bfloat16*>(p);
  prm.lse = lse;
  prm.rows = (long)BH * N;
  prm.n = N;
  prm.causal = causal != 0;
  prm.scale_log2 = scale * 1.4426950408889634f;
  const cudaError_t e = fa::launch_std_softmax(prm, stream);
  return e == cudaSuccess ? FA_OK : cuda_fail(e, "standard softmax launch");
}

fa_status fa_validate_cu_seqlens(const int* cu_seqlens, int B, int N, int total_tokens,
                                 cudaStream_t stream) {
  if (cu_seqlens == nullptr || B < 0 || N < 1 || total_tokens < 0) return FA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(cu_seqlens) & 3u) != 0) return FA_ERR_INVALID_ARG;
  const fa_status st = bind_device_of(cu_seqlens);
  if (st != FA_OK) return st;
  const cudaError_t e = launch_validate_cu(cu_seqlens, B, N, total_tokens, stream);
  return e == cudaSuccess ? FA_OK : cuda_fail(e, "cu_seqlens validation launch");
}

int fa_device_error(void) {
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, fa::g_fa_error, sizeof(int)) != cudaSuccess) return -1;
  return v;
}

fa_status fa_clear_device_error(void) {
  const int z = 0;
  return cudaMemcpyToSymbol(fa::g_fa_error, &z, sizeof(int)) == cudaSuccess ? FA_OK
                                                                             : FA_ERR_CUDA;
}

void fa_set_wait_limit_ns(unsigned long long ns) {
  g_wait_limit_ns.store(ns < 1000ull ? 1000ull : ns);
}

fa_status fa_watchdog_selftest(cudaStream_t stream) {
  fa::watchdog_selftest_kernel<<<1, 32, 0, stream>>>(g_wait_limit_ns.load());
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? FA_OK : cuda_fail(e, "self-test launch");
}

int fa_last_cuda_error(void) { return t_last_cuda_error; }

void fa_set_profile_events(cudaEvent_t main_begin, cudaEvent_t main_end) {
  t_prof_begin = main_begin;
  t_prof_end = main_end;
}

const char* fa_status_string(fa_status s) {
  switch (s) {
    case FA_OK: return "FA_OK";
    case FA_ERR_INVALID_ARG: return "FA_ERR_INVALID_ARG";
    case FA_ERR_UNSUPPORTED: return "FA_ERR_UNSUPPORTED";
    case FA_ERR_WORKSPACE: return "FA_ERR_WORKSPACE";
    case FA_ERR_CUDA: return "FA_ERR_CUDA";
  }
  return "FA_UNKNOWN_STATUS";
}

}  // extern "C"
