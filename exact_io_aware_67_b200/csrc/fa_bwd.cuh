// fa_bwd.cuh -- backward attention kernels for sm_100a.
//
// The backward recomputes S and P from Q, K and the forward's LSE instead of
// reading stored N x N matrices (paper review "FlashAttention: Fast and
// Memory-Efficient Exact Attention with IO-Awareness", 方法 item 3).  The
// gradient formulas are the derivative of O = softmax(scale Q K^T + mask) V:
//     P = exp(scale S - LSE),  dV = P^T dO,  dP = dO V^T,
//     D_i = sum_c dO_ic O_ic (= sum_j P_ij dP_ij),  dS = P o (dP - D),
//     dQ = scale dS K,  dK = scale dS^T Q.
//
// Three kernels run in stream order:
//   bwd_pre_kernel     D = rowsum(dO o O) in fp32 and zero the fp32 dQ
//                      accumulator (HBM-bound, grid-stride).  O is the bf16
//                      output plus, when the forward wrote it, its bf16
//                      rounding residual: with bf16 O alone the rounding
//                      error of D reaches dK through -scale P_ij D_i Q_i.
//   bwd_main_kernel    one CTA per 128-row K/V tile of one (sequence, kv
//                      head).  It loops over the query heads of its group and
//                      over the query tiles (only those on or below the
//                      diagonal when causal).  dK and dV accumulate in TMEM
//                      for the whole loop; each tile's dQ partial goes to the
//                      fp32 accumulator by vector atomic addition.
//   bwd_dq_kernel      dQ = scale * accumulator -> bf16, transposed back to
//                      the token-major layout.
//
// Orientation in bwd_main_kernel (kv rows are the MMA M dimension, so the
// per-thread row owned by the elementwise warps is a kv row):
//   S^T  = K Q^T        SS, A = K (K-major), B = Q (K-major)      -> TMEM
//   dP^T = V dO^T       SS, A = V (K-major), B = dO (K-major)     -> TMEM
//   dV  += P^T dO       TS, A = P^T (bf16 in TMEM), B = dO (N-major)
//   dK  += dS^T Q       SS, A = dS^T (smem, K-major), B = Q (N-major)
//   dQ_i = dS K         SS, A = dS (same smem, M-major), B = K (N-major)
// One 128 x 128 bf16 dS tile in shared memory serves both dK and dQ: as
// [kv row][q] it is K-major for dK and M-major for dQ.
//
// dQ accumulator layout (fp32, tile-major): query tile i of sequence b has
// its own 128-row block at tile slot  tb(b) + i,  where
//   tb(b) = b * ceil(N / 128)                 (dense batches)
//   tb(b) = ceil(start(b) / 128) + b          (variable-length batches; start(b)
//                                             is cu_seqlens[b] clamped to
//                                             [0, total]),
// which never overlaps the next sequence's slots.  Inside a slot the layout
// is [head][column group of 4][row 0..127][4], so the 32 threads of a warp
// (32 consecutive rows) add one contiguous 512-byte run per vector atomic.
// Rows of a tile past the end of its sequence are never added and never read.
// (Measured alternative: staging the tile in shared memory and adding it with
// bulk asynchronous reductions was slower -- the reductions from one issuing
// thread proceed nearly one after another.)
#pragma once
#include <algorithm>
#include <atomic>
#include <cstdio>
#include <cstdlib>

#include "fa_common.cuh"
#include "sm100.cuh"

namespace fa {

// Power-of-two scales of the backward's fp16 operands and the factors that
// undo them (written by bwd_pre_kernel, read by the main and dQ kernels).
struct BwdScales {
  float sq, sk, sv, sdo;   // Q, K, V, dO copies = fp16(x * s_x)
  float sds;               // dS operand = fp16(dS * s_ds)
  float c2p;               // scale * log2(e) / (s_q s_k): S of the fp16 product -> log2 units
  float vdo_sds;           // s_ds / (s_v s_do): dP of the fp16 product -> s_ds units
  float dv_mul;            // 1 / s_do
  float dk_mul;            // scale / (s_ds s_q)
  float dq_mul;            // scale / (s_ds s_k)
};

struct BwdParams {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  const __nv_bfloat16* v;
  const __nv_bfloat16* o;
  const __nv_bfloat16* o_lo;   // optional bf16 rounding residual of O (nullptr: none)
  const __nv_bfloat16* dout;
  const float* lse;
  __nv_bfloat16* dq;
  __nv_bfloat16* dk;
  __nv_bfloat16* dv;
  float* dpsum;      // D, same layout as lse
  float* dq_acc;     // fp32 dQ accumulator (layout above)
  // fp16 copies of the product operands (token-major, like the originals)
  __half* q16;
  __half* k16;
  __half* v16;
  __half* do16;
  float* absmax_part;   // [nabs][4]: per-block max |Q|, |K|, |V|, |dO|
  int nabs;             // blocks of bwd_absmax_kernel
  BwdScales* scales;
  long tile_slots;   // tile slots of the accumulator per head
  int order_chunk;   // (sequence, kv head) pairs per dispatch chunk (causal grid order)
  const int* cu_seqlens;
  int B, Hq, Hkv, N, group, total;
  float scale, scale_log2;
  unsigned long long wait_limit_ns;
  // block-sparse mode only: tile (qt, kt) of sequence b and kv head hk is
  // allowed iff bmask[b * bm_sb + hk * bm_sh + qt * bm_nt + kt] != 0
  const uint8_t* bmask;
  long bm_sb, bm_sh;
  int bm_nt;
};

constexpr int ABSMAX_MAX_BLOCKS = 2048;

inline size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

// number of 128-row tile slots of the dQ accumulator
inline long bwd_tile_slots(int B, int N, long tokens, bool varlen) {
  return varlen ? (tokens + 127) / 128 + B : (long)B * ((N + 127) / 128);
}

// Workspace layout: D, the max-abs partials, the scale record, the fp16
// copies of Q, K, V, dO, and the fp32 dQ accumulator, each 256-byte aligned.
struct BwdWsLayout {
  size_t dsum, part, scales, q16, k16, v16, do16, acc, total;
};

inline BwdWsLayout bwd_ws_layout(int B, int Hq, int Hkv, int N, int d, long tokens,
                                 bool varlen) {
  BwdWsLayout w{};
  size_t off = 0;
  w.dsum = off;
  off += align256((size_t)Hq * (size_t)tokens * 4);
  w.part = off;
  off += align256((size_t)ABSMAX_MAX_BLOCKS * 4 * 4);
  w.scales = off;
  off += 256;
  w.q16 = off;
  off += align256((size_t)tokens * Hq * d * 2);
  w.k16 = off;
  off += align256((size_t)tokens * Hkv * d * 2);
  w.v16 = off;
  off += align256((size_t)tokens * Hkv * d * 2);
  w.do16 = off;
  off += align256((size_t)tokens * Hq * d * 2);
  w.acc = off;
  off += (size_t)bwd_tile_slots(B, N, tokens, varlen) * Hq * 128 * d * 4;
  w.total = off;
  return w;
}

inline size_t bwd_workspace_bytes(int B, int Hq, int Hkv, int N, int d, long tokens,
                                  bool varlen) {
  return bwd_ws_layout(B, Hq, Hkv, N, d, tokens, varlen).total;
}

inline void bwd_carve_workspace(BwdParams& p, void* ws, long tokens, int d) {
  const BwdWsLayout w =
      bwd_ws_layout(p.B, p.Hq, p.Hkv, p.N, d, tokens, p.cu_seqlens != nullptr);
  uint8_t* base = static_cast<uint8_t*>(ws);
  p.dpsum = reinterpret_cast<float*>(base + w.dsum);
  p.absmax_part = reinterpret_cast<float*>(base + w.part);
  p.scales = reinterpret_cast<BwdScales*>(base + w.scales);
  p.q16 = reinterpret_cast<__half*>(base + w.q16);
  p.k16 = reinterpret_cast<__half*>(base + w.k16);
  p.v16 = reinterpret_cast<__half*>(base + w.v16);
  p.do16 = reinterpret_cast<__half*>(base + w.do16);
  p.dq_acc = reinterpret_cast<float*>(base + w.acc);
  p.tile_slots = bwd_tile_slots(p.B, p.N, tokens, p.cu_seqlens != nullptr);
}

// first tile slot of sequence b (from its clamped start, so that a corrupt
// cu_seqlens still keeps every slot below tile_slots)
__device__ __forceinline__ long tile_base(const BwdParams& p, int b) {
  if (p.cu_seqlens == nullptr) return (long)b * ((p.N + 127) / 128);
  int start, len;
  seq_range(p.cu_seqlens, b, p.total, &start, &len);
  return (long)((start + 127) / 128) + b;
}

// fp32 offset of (head h, tile slot ts, column group 0, row 0)
template <int D>
__device__ __forceinline__ long acc_tile_offset(const BwdParams& p, int h, long ts) {
  return ((long)h * p.tile_slots + ts) * (long)(128 * D);
}

// statistic index (lse / D) of token row `row` of sequence b, head h
__device__ __forceinline__ long stat_index(const BwdParams& p, int b, int h, int seq_start,
                                           int row) {
  return (p.cu_seqlens != nullptr) ? (long)h * p.total + seq_start + row
                                   : ((long)b * p.Hq + h) * p.N + row;
}

// ============================================================================
// K1: per-block max |x| of Q, K, V and dO
// ============================================================================
// The backward's five products run on fp16 operands: 11 significant bits for
// P and dS instead of bf16's 8, which keeps dV and dK within 2e-2 of the
// exact gradient where their magnitude reaches 4-8 (there bf16 output
// rounding alone takes up to 1.6e-2 of that).  Each input gets an fp16 copy
// scaled by a power of two that puts its largest magnitude just below 2^14,
// so the copy is exact for every bf16 value in fp16's normal range and the
// scales cancel exactly.  This kernel finds the largest magnitudes; the
// preprocess combines the per-block partials.
template <int D>
__global__ void __launch_bounds__(256) bwd_absmax_kernel(const BwdParams p, long tokens) {
  __shared__ float red[8][4];
  const long gtid = blockIdx.x * (long)blockDim.x + threadIdx.x;
  const long gstride = (long)gridDim.x * blockDim.x;
  float mx[4];
#pragma unroll
  for (int t = 0; t < 4; ++t) {
    const __nv_bfloat16* src = t == 0 ? p.q : t == 1 ? p.k : t == 2 ? p.v : p.dout;
    const int heads = (t == 0 || t == 3) ? p.Hq : p.Hkv;
    const long n8 = tokens * heads * (D / 8);
    const uint4* s4 = reinterpret_cast<const uint4*>(src);
    float m = 0.f;
    auto take = [&](const uint4 a) {
      const uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 x = unpack_bf16(w[e]);
        m = fmaxf(m, fmaxf(fabsf(x.x), fabsf(x.y)));
      }
    };
    // four independent 16-byte loads in flight per thread: one at a time
    // left HBM about half idle (2.9 TB/s on 50 MB)
    long i = gtid;
    for (; i + 3 * gstride < n8; i += 4 * gstride) {
      uint4 a[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) a[u] = s4[i + u * gstride];
#pragma unroll
      for (int u = 0; u < 4; ++u) take(a[u]);
    }
    for (; i < n8; i += gstride) take(s4[i]);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    mx[t] = m;
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0)
    for (int t = 0; t < 4; ++t) red[warp][t] = mx[t];
  __syncthreads();
  if (threadIdx.x < 4) {
    float m = 0.f;
    for (int w = 0; w < 8; ++w) m = fmaxf(m, red[w][threadIdx.x]);
    p.absmax_part[blockIdx.x * 4 + threadIdx.x] = m;
  }
}

// 2^(14 - e) for m < 2^e: the power of two that puts m just below 2^14
// (1 for m = 0 or a non-finite m; the exponent is clamped to stay normal).
__device__ __forceinline__ float fp16_pow2_scale(float m) {
  if (!(m > 0.f) || !isfinite(m)) return 1.f;
  int e;
  frexpf(m, &e);
  return ldexpf(1.f, max(-100, min(100, 14 - e)));
}

// The scales from the four maxima (every caller computes the same values).
__device__ __forceinline__ BwdScales bwd_make_scales(const BwdParams& p, const float mx[4],
                                                     int d) {
  BwdScales sc;
  sc.sq = fp16_pow2_scale(mx[0]);
  sc.sk = fp16_pow2_scale(mx[1]);
  sc.sv = fp16_pow2_scale(mx[2]);
  sc.sdo = fp16_pow2_scale(mx[3]);
  // |dS| <= P (|dP| + |D|) <= 2 d max|dO| max|V| (|O| <= max|V| row by row)
  sc.sds = fp16_pow2_scale(2.f * (float)d * mx[3] * mx[2]);
  sc.c2p = p.scale_log2 / (sc.sq * sc.sk);
  sc.vdo_sds = sc.sds / (sc.sv * sc.sdo);
  sc.dv_mul = 1.f / sc.sdo;
  sc.dk_mul = p.scale / (sc.sds * sc.sq);
  sc.dq_mul = p.scale / (sc.sds * sc.sk);
  return sc;
}

// ============================================================================
// K2: scales, fp16 operand copies, D = rowsum(dO o O), zeroed dQ accumulator
// ============================================================================
// Grid-stride; every block first combines the max-abs partials into the
// scales (block 0 also stores them for the later kernels), then writes its
// share of the four fp16 copies, D and the zeroed accumulator.
template <int D>
__global__ void __launch_bounds__(256, 6) bwd_pre_kernel(const BwdParams p, long tokens) {
  __shared__ float red[8][4];
  __shared__ BwdScales s_sc;
  {
    float mx[4] = {0.f, 0.f, 0.f, 0.f};
    for (int i = threadIdx.x; i < p.nabs; i += blockDim.x)
#pragma unroll
      for (int t = 0; t < 4; ++t) mx[t] = fmaxf(mx[t], p.absmax_part[i * 4 + t]);
#pragma unroll
    for (int t = 0; t < 4; ++t)
#pragma unroll
      for (int off = 16; off > 0; off >>= 1)
        mx[t] = fmaxf(mx[t], __shfl_xor_sync(0xffffffffu, mx[t], off));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0)
      for (int t = 0; t < 4; ++t) red[warp][t] = mx[t];
    __syncthreads();
    if (threadIdx.x == 0) {
      float m[4];
      for (int t = 0; t < 4; ++t) {
        m[t] = 0.f;
        for (int w = 0; w < 8; ++w) m[t] = fmaxf(m[t], red[w][t]);
      }
      s_sc = bwd_make_scales(p, m, D);
      if (blockIdx.x == 0) *p.scales = s_sc;
    }
    __syncthreads();
  }
  const long gtid = blockIdx.x * (long)blockDim.x + threadIdx.x;
  const long gstride = (long)gridDim.x * blockDim.x;
  // the fp16 copies of Q, K, V (dO's is written by the D pass below, which
  // reads every dO row anyway)
#pragma unroll 1
  for (int t = 0; t < 3; ++t) {
    const __nv_bfloat16* src = t == 0 ? p.q : t == 1 ? p.k : t == 2 ? p.v : p.dout;
    __half* dst = t == 0 ? p.q16 : t == 1 ? p.k16 : t == 2 ? p.v16 : p.do16;
    const float sx = t == 0 ? s_sc.sq : t == 1 ? s_sc.sk : t == 2 ? s_sc.sv : s_sc.sdo;
    const int heads = (t == 0 || t == 3) ? p.Hq : p.Hkv;
    const long n8 = tokens * heads * (D / 8);
    const uint4* s4 = reinterpret_cast<const uint4*>(src);
    uint4* d4 = reinterpret_cast<uint4*>(dst);
    auto conv = [&](const uint4 a) {
      const float2 x0 = unpack_bf16(a.x), x1 = unpack_bf16(a.y);
      const float2 x2 = unpack_bf16(a.z), x3 = unpack_bf16(a.w);
      return make_uint4(pack_f16(x0.x * sx, x0.y * sx), pack_f16(x1.x * sx, x1.y * sx),
                        pack_f16(x2.x * sx, x2.y * sx), pack_f16(x3.x * sx, x3.y * sx));
    };
    // two independent loads in flight per thread
    long i = gtid;
    for (; i + gstride < n8; i += 2 * gstride) {
      const uint4 a0 = s4[i], a1 = s4[i + gstride];
      d4[i] = conv(a0);
      d4[i + gstride] = conv(a1);
    }
    if (i < n8) d4[i] = conv(s4[i]);
  }
  // zero the accumulator
  {
    float4* acc = reinterpret_cast<float4*>(p.dq_acc);
    const long n4 = p.tile_slots * p.Hq * 128 * (D / 4);
    for (long i = gtid; i < n4; i += gstride) acc[i] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
  // one group of D/8 lanes per (token, head) row; each lane reads 8 bf16
  constexpr int LPR = D / 8;            // lanes per row
  constexpr int RPW = 32 / LPR;         // rows per warp pass
  const int lane = threadIdx.x & 31;
  const int sub = lane / LPR;
  const int li = lane % LPR;
  const long rows = tokens * p.Hq;
  const long warp_global = gtid >> 5;
  const long nwarps = gstride >> 5;
  for (long base = warp_global * RPW; base < rows; base += nwarps * RPW) {
    const long row = base + sub;
    float s = 0.f;
    if (row < rows) {
      const uint4 a = *reinterpret_cast<const uint4*>(p.o + row * D + li * 8);
      const uint4 b = *reinterpret_cast<const uint4*>(p.dout + row * D + li * 8);
      uint4 c = make_uint4(0u, 0u, 0u, 0u);
      if (p.o_lo != nullptr) c = *reinterpret_cast<const uint4*>(p.o_lo + row * D + li * 8);
      const uint32_t av[4] = {a.x, a.y, a.z, a.w};
      const uint32_t bv[4] = {b.x, b.y, b.z, b.w};
      const uint32_t cv[4] = {c.x, c.y, c.z, c.w};
      uint32_t h16[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        // O = bf16(O) + residual: exact in fp32 (about 16 significant bits)
        const float2 x = unpack_bf16(av[e]);
        const float2 xr = unpack_bf16(cv[e]);
        const float2 y = unpack_bf16(bv[e]);
        s = fmaf(x.x + xr.x, y.x, s);
        s = fmaf(x.y + xr.y, y.y, s);
        h16[e] = pack_f16(y.x * s_sc.sdo, y.y * s_sc.sdo);
      }
      *reinterpret_cast<uint4*>(p.do16 + row * D + li * 8) =
          make_uint4(h16[0], h16[1], h16[2], h16[3]);
    }
#pragma unroll
    for (int off = LPR / 2; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    if (li == 0 && row < rows) {
      const long t = row / p.Hq;
      const int h = (int)(row % p.Hq);
      long idx;
      if (p.cu_seqlens != nullptr) {
        idx = (long)h * p.total + t;
      } else {
        const long b = t / p.N, n = t % p.N;
        idx = (b * p.Hq + h) * p.N + n;
      }
      p.dpsum[idx] = s;
    }
  }
}

// ============================================================================
// K4: dQ = scale * accumulator / (s_ds s_k) -> bf16 [token][head][d]
// ============================================================================
// Persistent: a few blocks per SM stride over the (query tile, head,
// sequence) items, item = (b * Hq + h) * nq + i; 256 threads turn one
// 128-row tile (two halves of 64 rows) back into token-major bf16.  Each
// thread issues all its loads of a half before its shared-memory stores.
// The staging rows are D + 4 floats apart, so the float4 stores (eight
// consecutive rows per phase) hit eight different 16-byte bank groups, and
// so do the two float4 loads of a row's 8-column chunk when every other
// group of four chunks takes its two halves in swapped order.
template <int D>
__global__ void __launch_bounds__(256) bwd_dq_kernel(const BwdParams p, long items, int nq) {
  constexpr int RH = 64;                       // rows per half
  constexpr int LD = (D / 4) * RH / 256;       // float4 loads per thread and half
  __shared__ __align__(16) float tile[RH][D + 4];
  const int tid = threadIdx.x;
  // the accumulator holds sum dS16 K16 = s_ds s_k sum dS K
  const float mul = p.scales->dq_mul;
  for (long it = blockIdx.x; it < items; it += gridDim.x) {
    const int i = (int)(it % nq);
    const long bh = it / nq;
    const int h = (int)(bh % p.Hq), b = (int)(bh / p.Hq);
    int seq_start = 0, len = p.N;
    if (p.cu_seqlens != nullptr) seq_range(p.cu_seqlens, b, p.total, &seq_start, &len);
    if (128 * i >= len) continue;   // the same for the whole block
    const long tok0 = ((p.cu_seqlens != nullptr) ? (long)seq_start : (long)b * p.N) + 128 * i;
    const float4* src =
        reinterpret_cast<const float4*>(p.dq_acc + acc_tile_offset<D>(p, h, tile_base(p, b) + i));
    for (int half = 0; half < 2; ++half) {
      const int r0 = half * RH;
      if (128 * i + r0 >= len) break;
      float4 v[LD];
#pragma unroll
      for (int k = 0; k < LD; ++k) {
        const int idx = tid + 256 * k;
        v[k] = src[(idx / RH) * 128 + r0 + idx % RH];
      }
#pragma unroll
      for (int k = 0; k < LD; ++k) {
        const int idx = tid + 256 * k;
        *reinterpret_cast<float4*>(&tile[idx % RH][4 * (idx / RH)]) = v[k];
      }
      __syncthreads();
      for (int idx = tid; idx < RH * (D / 8); idx += 256) {
        const int rr = idx / (D / 8), ch = idx % (D / 8);
        if (128 * i + r0 + rr >= len) continue;
        const int sw = (ch >> 2) & 1;
        const float4 x = *reinterpret_cast<const float4*>(&tile[rr][8 * ch + 4 * sw]);
        const float4 y = *reinterpret_cast<const float4*>(&tile[rr][8 * ch + 4 - 4 * sw]);
        const float4 lo = sw ? y : x, hi = sw ? x : y;
        uint4 w;
        w.x = pack_bf16(lo.x * mul, lo.y * mul);
        w.y = pack_bf16(lo.z * mul, lo.w * mul);
        w.z = pack_bf16(hi.x * mul, hi.y * mul);
        w.w = pack_bf16(hi.z * mul, hi.w * mul);
        *reinterpret_cast<uint4*>(p.dq + ((tok0 + r0 + rr) * p.Hq + h) * D + 8 * ch) = w;
      }
      __syncthreads();
    }
  }
}

// ============================================================================
// K3: main backward kernel
// ============================================================================
template <int D>
struct BwdLayout {
  static constexpr int TILE = 128 * D * 2;   // one 128 x D bf16 tile
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = OFF_K + TILE;
  static constexpr int DO_STAGES = 2;
  static constexpr int OFF_Q = OFF_V + TILE;            // 2 stages
  static constexpr int OFF_DO = OFF_Q + 2 * TILE;       // DO_STAGES stages
  static constexpr int OFF_DS = OFF_DO + DO_STAGES * TILE;   // 128 x 128 bf16
  static constexpr int OFF_STATS = OFF_DS + 32768;      // 2 stages x (lse2[128], D[128])
  static constexpr int OFF_BAR = OFF_STATS + 2 * 1024;
  // kv_full q_full[2] q_empty[2] st_full[2] do_full[2] do_empty[2] s_full dp_full
  // p_full ds_full ds_empty dq_full dq_empty dkv_done drain
  static constexpr int NBAR = 20;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  // block-sparse mode: which query tiles the CTA's K/V tile meets (bits
  // [FA_SPARSE_MAX_TILES / 32]) and how many
  static constexpr int OFF_QBITS = OFF_MISC + 16;
  static constexpr int OFF_NQ = OFF_QBITS + (FA_SPARSE_MAX_TILES / 32) * 4;
  static constexpr int BYTES = OFF_NQ + 16;
  static_assert(BYTES <= 232448, "shared memory per block");
  // The d = 128 layout uses all but ~0.8 KB of the 227 KB a CTA may have, so
  // it relies on the dynamic shared memory window starting 1024-byte aligned
  // (checked at run time; a misaligned base reports ERR_BWD_SMEM_ALIGN).
  static constexpr bool SLACK = (BYTES + 1024 <= 232448);
  static constexpr int ALLOC = SLACK ? BYTES + 1024 : BYTES;
  // TMEM columns
  static constexpr uint32_t T_DV = 0;
  static constexpr uint32_t T_DK = D;
  static constexpr uint32_t T_S = 2 * D;
  static constexpr uint32_t T_DP = 2 * D + 128;
  static constexpr uint32_t T_DQ = (D == 128) ? T_DP : 2 * D + 256;   // aliases dP at d = 128
};

// warps 0-7: elementwise (two warpgroups, 64 query columns each)
// warps 8-11: dQ drain;  warp 12: TMA producer;  warp 13: MMA issuer;
// warps 14-15: idle (they only give their registers to the drain warps)
constexpr int BWD_THREADS = 512;
constexpr int BWD_REGS_DRAIN = 176;   // warpgroup 2 after setmaxnreg.inc
constexpr int BWD_REGS_CTRL = 80;     // warpgroup 3 after setmaxnreg.dec
static_assert(128 * (128 + 128 + BWD_REGS_DRAIN + BWD_REGS_CTRL) == 65536, "register split");

// First set bit at or after position `from` of a bit list, or `limit`.
__device__ __forceinline__ int next_set_bit(const uint32_t* bits, int from, int limit) {
  for (int w = from >> 5; (w << 5) < limit; ++w) {
    uint32_t x = bits[w];
    if (w == (from >> 5)) x &= ~0u << (from & 31);
    if (x != 0u) return min(limit, (w << 5) + __ffs(x) - 1);
  }
  return limit;
}

template <int D, bool CAUSAL, bool SPARSE = false>
__global__ void __launch_bounds__(BWD_THREADS, 1)
    bwd_main_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                    const BwdParams p) {
  using L = BwdLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  if (!L::SLACK && (smem_u32(smem_raw) & 1023u) != 0) {
    if (threadIdx.x == 0) atomicCAS(&g_fa_error, 0, ERR_BWD_SMEM_ALIGN);
    return;
  }
  uint8_t* smem = L::SLACK ? align_1024(smem_raw) : smem_raw;

  // ---------------------------------------------------------------- work item
  // Blocks are dispatched roughly in index order.  Causal: the (sequence, kv
  // head) pairs are cut into chunks of order_chunk pairs; within a chunk the
  // K/V tile index is slowest, so the longest blocks (tile j has nq - j query
  // tiles) start first and the short ones fill the chunk's tail -- at B=2,
  // Hkv=8, N=4096 (one chunk) this took the main kernel from 737 to 912
  // TFLOP/s on B200.  A chunk holds at least four waves of blocks, so the
  // tails still interleave, while the blocks in flight touch only the chunk's
  // Q, dO and dQ-accumulator tiles, which then stay in L2 between the blocks
  // that share them (at N = 65536 the accumulator is four times the L2).
  // Without the mask every tile of a sequence has the same work, and the
  // tiles of one (sequence, kv head) stay adjacent to share Q and dO in L2.
  const unsigned nkv_blocks = (unsigned)(p.N + 127) / 128;
  const unsigned bh = (unsigned)p.Hkv * p.B;
  unsigned u;
  int j;
  if (CAUSAL) {
    const unsigned chunk = (unsigned)p.order_chunk;
    const unsigned c = blockIdx.x / (chunk * nkv_blocks);
    const unsigned r = blockIdx.x - c * chunk * nkv_blocks;
    const unsigned pairs = min(chunk, bh - c * chunk);
    u = c * chunk + r % pairs;
    j = (int)(r / pairs);
  } else {
    u = blockIdx.x / nkv_blocks;
    j = (int)(blockIdx.x % nkv_blocks);
  }
  const int hk = (int)(u % p.Hkv);
  const int b = (int)(u / p.Hkv);
  int seq_start = 0, len = p.N, bcoord = b;
  if (p.cu_seqlens != nullptr) {
    seq_range(p.cu_seqlens, b, p.total, &seq_start, &len);
    bcoord = 0;
  }
  if (128 * j >= len) return;
  const int nq = (len + 127) / 128;
  const int i0 = CAUSAL ? j : 0;
  // Block-sparse: the query tiles this K/V tile meets are those the block
  // mask of its kv head allows (on or below the diagonal when causal); every
  // query head of the group walks the same list, found once here.
  uint32_t* s_qbits = reinterpret_cast<uint32_t*>(smem + L::OFF_QBITS);
  int* s_nq = reinterpret_cast<int*>(smem + L::OFF_NQ);
  if (SPARSE && warp == 14) {
    const uint8_t* mcol = p.bmask + (long)b * p.bm_sb + (long)hk * p.bm_sh + j;
    int cnt = 0;
    for (int c0 = 0; c0 < FA_SPARSE_MAX_TILES; c0 += 32) {
      const int i = c0 + lane;
      const bool a = i >= i0 && i < nq && mcol[(long)i * p.bm_nt] != 0;
      const uint32_t bal = __ballot_sync(0xffffffffu, a);
      if (lane == 0) s_qbits[c0 >> 5] = bal;
      cnt += __popc(bal);
    }
    if (lane == 0) *s_nq = cnt;
  }

  uint8_t* sK = smem + L::OFF_K;
  uint8_t* sV = smem + L::OFF_V;
  uint8_t* sQ = smem + L::OFF_Q;
  uint8_t* sDO = smem + L::OFF_DO;
  uint8_t* sDS = smem + L::OFF_DS;
  float* stats = reinterpret_cast<float*>(smem + L::OFF_STATS);   // [2][2][128]
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);
  uint64_t* kv_full = bars + 0;
  uint64_t* q_full = bars + 1;      // [2]
  uint64_t* q_empty = bars + 3;     // [2]
  uint64_t* st_full = bars + 5;     // [2]  statistics of the Q stage
  uint64_t* do_full = bars + 7;     // [2]
  uint64_t* do_empty = bars + 9;    // [2]
  uint64_t* s_full = bars + 11;
  uint64_t* dp_full = bars + 12;
  uint64_t* p_full = bars + 13;
  uint64_t* ds_full = bars + 14;
  uint64_t* ds_empty = bars + 15;
  uint64_t* dq_full = bars + 16;
  uint64_t* dq_empty = bars + 17;
  uint64_t* dkv_done = bars + 18;
  uint64_t* drain = bars + 19;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::OFF_MISC + 4);

  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(q_full + s, 1);
      mbar_init(q_empty + s, 1);
      mbar_init(st_full + s, 32);
      mbar_init(do_full + s, 1);
      mbar_init(do_empty + s, 1);
    }
    mbar_init(s_full, 1);
    mbar_init(dp_full, 1);
    mbar_init(p_full, 256);
    mbar_init(ds_full, 256);
    mbar_init(ds_empty, 1);
    mbar_init(dq_full, 1);
    mbar_init(dq_empty, 128);
    mbar_init(dkv_done, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 13) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  if (warp == 12 && lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
    tma_prefetch_desc(&tmDO);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const Watchdog wd{&g_fa_error, abort_flag, p.wait_limit_ns};
  const int n_i = SPARSE ? *s_nq : nq - i0;   // query tiles per head
  const int T = p.group * n_i;                // iterations of this CTA
  // query tile of iteration n (iterations run head by head over the list);
  // `cur` carries the previous answer, so each role calls it with n = 0, 1, ...
  auto qtile = [&](int n, int& cur) -> int {
    if (!SPARSE) return i0 + n % n_i;
    cur = next_set_bit(s_qbits, (n % n_i == 0) ? 0 : cur + 1, nq);
    return cur;
  };

  if (SPARSE && n_i == 0) {
    // no query tile meets this K/V tile: dK = dV = 0 for its rows
    for (int e = threadIdx.x; e < 128 * (D / 8); e += BWD_THREADS) {
      const int r = e / (D / 8), c8 = e % (D / 8);
      const int kv_row = 128 * j + r;
      if (kv_row < len) {
        const long t = (long)b * p.N + kv_row;
        reinterpret_cast<uint4*>(p.dk + (t * p.Hkv + hk) * (long)D)[c8] = make_uint4(0u, 0u, 0u, 0u);
        reinterpret_cast<uint4*>(p.dv + (t * p.Hkv + hk) * (long)D)[c8] = make_uint4(0u, 0u, 0u, 0u);
      }
    }
  } else if (warp >= 12) {
  // ============================================================== warpgroup 3
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;\n" ::"n"(BWD_REGS_CTRL));
  if (warp == 12) {
    // ============================================================ producer
    const float kLog2e = 1.4426950408889634f;
    const float sds = p.scales->sds;
    if (lane == 0) {
      mbar_arrive_expect_tx(kv_full, 2 * L::TILE);
#pragma unroll
      for (int c = 0; c < D / 64; ++c) {
        tma_load_4d(sK + c * 16384, &tmK, kv_full, c * 64, hk, seq_start + 128 * j, bcoord);
        tma_load_4d(sV + c * 16384, &tmV, kv_full, c * 64, hk, seq_start + 128 * j, bcoord);
      }
    }
    int q_issued = 0, do_issued = 0;
    bool ok = true;
    int qcur = 0;
    for (int n = 0; n < T && ok; ++n) {
      const int h = hk * p.group + n / n_i;
      const int i = qtile(n, qcur);
      const int s = n & 1;
      const uint32_t ph_empty = ((n >> 1) & 1) ^ 1;
      // Q_n (stage s) and dO_n (stage s) by TMA
      ok = __all_sync(0xffffffffu, mbar_wait(q_empty + s, ph_empty, wd, ERR_BWD_LOAD_EMPTY));
      if (!ok) break;
      if (lane == 0) {
        mbar_arrive_expect_tx(q_full + s, L::TILE);
#pragma unroll
        for (int c = 0; c < D / 64; ++c)
          tma_load_4d(sQ + s * L::TILE + c * 16384, &tmQ, q_full + s, c * 64, h,
                      seq_start + 128 * i, bcoord);
      }
      q_issued = n + 1;
      const int sd = n % L::DO_STAGES;
      ok = __all_sync(0xffffffffu, mbar_wait(do_empty + sd, ((n / L::DO_STAGES) & 1) ^ 1, wd,
                                             ERR_BWD_LOAD_EMPTY));
      if (!ok) break;
      if (lane == 0) {
        mbar_arrive_expect_tx(do_full + sd, L::TILE);
#pragma unroll
        for (int c = 0; c < D / 64; ++c)
          tma_load_4d(sDO + sd * L::TILE + c * 16384, &tmDO, do_full + sd, c * 64, h,
                      seq_start + 128 * i, bcoord);
      }
      do_issued = n + 1;
      // statistics of the 128 query rows, negated for the packed elementwise
      // math: -LSE * log2(e) and -D * s_ds (dS goes to fp16 scaled by s_ds);
      // rows past the sequence end get -inf / 0 so that their P and dS
      // vanish.  The stage's previous readers are
      // done: they finished before dK of iteration n-2, which released
      // q_empty[s].
      float lv[4], dv[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int row = 128 * i + lane + 32 * e;
        const long si = stat_index(p, b, h, seq_start, min(row, len - 1));
        lv[e] = p.lse[si];
        dv[e] = p.dpsum[si];
      }
      float* st = stats + s * 256;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int r = lane + 32 * e;
        const bool valid = 128 * i + r < len;
        st[r] = valid ? -lv[e] * kLog2e : -INFINITY;
        st[128 + r] = valid ? -dv[e] * sds : 0.f;
      }
      mbar_arrive(st_full + s);
    }
    if (lane == 0 && *abort_flag) {
      mbar_wait_drain(kv_full, 0, p.wait_limit_ns);
      for (int n = max(0, q_issued - 2); n < q_issued; ++n)
        mbar_wait_drain(q_full + (n & 1), (n >> 1) & 1, p.wait_limit_ns);
      for (int n = max(0, do_issued - L::DO_STAGES); n < do_issued; ++n)
        mbar_wait_drain(do_full + n % L::DO_STAGES, (n / L::DO_STAGES) & 1, p.wait_limit_ns);
    }
    __syncwarp();
  } else if (warp == 13) {
    // ============================================================ MMA issuer
    if (lane == 0) {
      // every product takes both operands in fp16 (the scaled copies of Q, K,
      // V, dO, and P and dS written as fp16 by the elementwise warps)
      constexpr uint32_t id_sq = idesc_f16_f32(128, 128, false, false);   // S^T, dP^T
      constexpr uint32_t id_kn = idesc_f16_f32(128, D, false, true);      // dV, dK
      constexpr uint32_t id_mn = idesc_f16_f32(128, D, true, true);       // dQ
      // descriptors built once; K-major views (LBO unused) and N/M-major
      // views (LBO = distance between 64-element blocks)
      const SDesc kK = sdesc_make(smem_u32(sK), 16, 1024);     // K, A of S^T
      const SDesc kV = sdesc_make(smem_u32(sV), 16, 1024);     // V, A of dP^T
      const SDesc kQ = sdesc_make(smem_u32(sQ), 16, 1024);     // Q, B of S^T
      const SDesc kDO = sdesc_make(smem_u32(sDO), 16, 1024);   // dO, B of dP^T
      const SDesc kDS = sdesc_make(smem_u32(sDS), 16, 1024);   // dS^T, A of dK
      const SDesc nDO = sdesc_make(smem_u32(sDO), 16384, 1024);  // dO, B of dV
      const SDesc nQ = sdesc_make(smem_u32(sQ), 16384, 1024);    // Q, B of dK
      const SDesc nK = sdesc_make(smem_u32(sK), 16384, 1024);    // K, B of dQ
      const SDesc mDS = sdesc_make(smem_u32(sDS), 16384, 1024);  // dS, A of dQ
      // D[128 x 128] = A[128 x D] B[128 x D]^T, both K-major
      auto mma_nt = [&](uint32_t dcol, SDesc a, SDesc bq, uint32_t boff) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
          mma_ss(tmem + dcol, sdesc_at(a, off), sdesc_at(bq, boff + off), id_sq, kk > 0 ? 1u : 0u);
        }
      };
      bool ok = mbar_wait(kv_full, 0, wd, ERR_BWD_KV_FULL);
      // prologue: S_0 and dP_0
      if (ok) ok = mbar_wait(q_full + 0, 0, wd, ERR_BWD_Q_FULL);
      if (ok) {
        tc_fence_after();
        mma_nt(L::T_S, kK, kQ, 0);
        mma_commit(s_full);
        ok = mbar_wait(do_full + 0, 0, wd, ERR_BWD_Q_FULL);
      }
      if (ok) {
        tc_fence_after();
        mma_nt(L::T_DP, kV, kDO, 0);
        mma_commit(dp_full);
      }
      // Steady state, iteration n (issue order; the tensor pipe runs them in
      // this order):  dV_n, S_{n+1}, dQ_n, dK_n, dP_{n+1}.  S_{n+1} goes out
      // right after the last reader of P_n so that the elementwise warps can
      // build P_{n+1} while dQ_n and dK_n run; dQ_n precedes dK_n so that its
      // TMEM drain overlaps dK_n.
      for (int n = 0; ok && n < T; ++n) {
        const int s = n & 1;
        const uint32_t ph = n & 1;
        const bool has_next = n + 1 < T;
        // dV += P^T dO  (A = P^T in TMEM: q columns 0-63 at T_S + 0..31,
        // 64-127 at T_S + 64..95)
        if (!(ok = mbar_wait(p_full, ph, wd, ERR_BWD_P_FULL))) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t acol = L::T_S + (kk < 4 ? 8 * kk : 64 + 8 * (kk - 4));
          mma_ts(tmem + L::T_DV, tmem + acol,
                 sdesc_at(nDO, (n % L::DO_STAGES) * L::TILE + kk * 2048), id_kn,
                 (n > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(do_empty + n % L::DO_STAGES);
        if (has_next) {
          const int s1 = (n + 1) & 1;
          if (!(ok = mbar_wait(q_full + s1, ((n + 1) >> 1) & 1, wd, ERR_BWD_Q_FULL))) break;
          tc_fence_after();
          mma_nt(L::T_S, kK, kQ, s1 * L::TILE);
          mma_commit(s_full);
        }
        if (!(ok = mbar_wait(ds_full, ph, wd, ERR_BWD_DS_FULL))) break;
        tc_fence_after();
        // dQ_n = dS K  (A = dS M-major in smem, B = K N-major)
        if (D != 128 && n > 0) {
          if (!(ok = mbar_wait(dq_empty, (n - 1) & 1, wd, ERR_BWD_DQ_EMPTY))) break;
          tc_fence_after();
        }
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ss(tmem + L::T_DQ, sdesc_at(mDS, kk * 2048), sdesc_at(nK, kk * 2048), id_mn,
                 kk > 0 ? 1u : 0u);
        mma_commit(dq_full);
        // dK += dS^T Q  (A = dS^T K-major in smem, B = Q N-major)
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t aoff = (kk >> 2) * 16384 + (kk & 3) * 32;
          mma_ss(tmem + L::T_DK, sdesc_at(kDS, aoff), sdesc_at(nQ, s * L::TILE + kk * 2048), id_kn,
                 (n > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(q_empty + s);
        mma_commit(ds_empty);
        if (has_next) {
          const int sd1 = (n + 1) % L::DO_STAGES;
          if (!(ok = mbar_wait(do_full + sd1, ((n + 1) / L::DO_STAGES) & 1, wd, ERR_BWD_Q_FULL)))
            break;
          if (D == 128) {
            // the dP columns hold dQ_n until the dQ warps have read it
            if (!(ok = mbar_wait(dq_empty, n & 1, wd, ERR_BWD_DQ_EMPTY))) break;
          }
          tc_fence_after();
          mma_nt(L::T_DP, kV, kDO, sd1 * L::TILE);
          mma_commit(dp_full);
        }
      }
      mma_commit(dkv_done);
      mma_commit(drain);
      mbar_wait_drain(drain, 0, p.wait_limit_ns);
    }
    __syncwarp();
  }
  } else if (warp >= 8) {
    // ============================================================ dQ drain
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;\n" ::"n"(BWD_REGS_DRAIN));
    // Each thread owns one query row of the tile (its TMEM lane).  The whole
    // row is read out of TMEM first so the columns can be released early;
    // then the row is added into the fp32 accumulator with vector atomics.
    // In the tile-major accumulator the 32 lanes of a warp cover 32
    // consecutive rows of one column group: one 512-byte run per instruction.
    const int r = (warp & 3) * 32 + lane;                  // query row within tile
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t tq = tmem + lane_off + L::T_DQ;
    const long tb = tile_base(p, b);
    int qcur = 0;
    for (int n = 0; n < T; ++n) {
      const int h = hk * p.group + n / n_i;
      const int i = qtile(n, qcur);
      if (!__all_sync(0xffffffffu, mbar_wait(dq_full, n & 1, wd, ERR_BWD_DQ_FULL))) break;
      tc_fence_after();
      uint32_t v[D];
#pragma unroll
      for (int c = 0; c < D / 32; ++c) tmem_ld32(tq + 32 * c, v + 32 * c);
#pragma unroll
      for (int c = 0; c < D / 32; ++c) tmem_wait_ld32(v + 32 * c);
      tc_fence_before();
      mbar_arrive(dq_empty);
      // rows past the end of the sequence hold exact zeros: skip them
      if (128 * i + r < len) {
        float4* acc = reinterpret_cast<float4*>(p.dq_acc + acc_tile_offset<D>(p, h, tb + i)) + r;
#pragma unroll
        for (int g = 0; g < D / 4; ++g)
          atomicAdd(acc + g * 128, make_float4(__uint_as_float(v[4 * g]), __uint_as_float(v[4 * g + 1]),
                                               __uint_as_float(v[4 * g + 2]),
                                               __uint_as_float(v[4 * g + 3])));
      }
    }
  } else {
    // ============================================================ elementwise
    // warp w owns kv rows 32 (w % 4) .. +31 (its TMEM lanes); warpgroup
    // wg = w / 4 owns query columns 64 wg .. 64 wg + 63 of the tile.
    const int wg = warp >> 2;
    const int r = (warp & 3) * 32 + lane;                 // kv row within tile
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lane_off + L::T_S + 64 * wg;
    const uint32_t tDP = tmem + lane_off + L::T_DP + 64 * wg;
    const int kv_row = 128 * j + r;
    const bool kv_ok = kv_row < len;
    // S and dP of the fp16 products carry the operand scales: c2 maps S to
    // log2 units, vdo_sds maps dP to the s_ds units of the stored -D s_ds
    const float c2 = p.scales->c2p;
    const float vdo_sds = p.scales->vdo_sds;
    // byte offset of this thread's row inside its 64-column dS region
    uint8_t* ds_row = sDS + wg * 16384 + (r >> 3) * 1024 + (r & 7) * 128;
    bool ok = true;
    int qcur = 0;
    for (int n = 0; n < T; ++n) {
      const int i = qtile(n, qcur);
      const int s = n & 1;
      const float* st = stats + s * 256;
      ok = __all_sync(0xffffffffu, mbar_wait(s_full, n & 1, wd, ERR_BWD_S_FULL) &&
                                       mbar_wait(st_full + s, (n >> 1) & 1, wd, ERR_BWD_STATS));
      if (!ok) break;
      tc_fence_after();
      float P[64];
      {
        uint32_t sv[64];
        tmem_ld32(tS, sv);
        tmem_ld32(tS + 32, sv + 32);
        tmem_wait_ld32(sv);
        tmem_wait_ld32(sv + 32);
        // x = s c2 - LSE log2(e) in packed pairs (the stats hold -LSE log2 e)
        const float2 c22 = make_float2(c2, c2);
#pragma unroll
        for (int c4 = 0; c4 < 16; ++c4) {
          const float4 l4 = *reinterpret_cast<const float4*>(st + 64 * wg + 4 * c4);
          const float2 x01 = ffma2(make_float2(__uint_as_float(sv[4 * c4 + 0]),
                                               __uint_as_float(sv[4 * c4 + 1])),
                                   c22, make_float2(l4.x, l4.y));
          const float2 x23 = ffma2(make_float2(__uint_as_float(sv[4 * c4 + 2]),
                                               __uint_as_float(sv[4 * c4 + 3])),
                                   c22, make_float2(l4.z, l4.w));
          P[4 * c4 + 0] = ex2(x01.x);
          P[4 * c4 + 1] = ex2(x01.y);
          P[4 * c4 + 2] = ex2(x23.x);
          P[4 * c4 + 3] = ex2(x23.y);
        }
        // masks (warp-uniform test first): causal diagonal tile -- key row
        // kv_row is masked for query q < kv_row -- and key rows past the end
        // of the sequence
        const bool diag = CAUSAL && i == j;
        if (__any_sync(0xffffffffu, diag || !kv_ok)) {
          const int qlim = diag ? (kv_row - 128 * i - 64 * wg) : 0;
#pragma unroll
          for (int c = 0; c < 64; ++c)
            if (!kv_ok || c < qlim) P[c] = 0.f;
        }
        uint32_t pk[32];
#pragma unroll
        for (int c = 0; c < 32; ++c) pk[c] = pack_f16(P[2 * c], P[2 * c + 1]);
        tmem_st32(tS, pk);      // P^T (fp16) over the S columns just read
        tmem_wait_st();
      }
      tc_fence_before();
      mbar_arrive(p_full);
      // dS = P o (dP - D)
      ok = __all_sync(0xffffffffu, mbar_wait(dp_full, n & 1, wd, ERR_BWD_DP_FULL));
      if (!ok) break;
      tc_fence_after();
      uint32_t dsp[32];
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        uint32_t dv[32];
        tmem_ld32(tDP + 32 * hh, dv);
        tmem_wait_ld32(dv);
#pragma unroll
        for (int c4 = 0; c4 < 8; ++c4) {
          // dS s_ds = P (dP vdo_sds - D s_ds) (the stats hold -D s_ds)
          const float4 d4 = *reinterpret_cast<const float4*>(st + 128 + 64 * wg + 32 * hh + 4 * c4);
          const int c = 32 * hh + 4 * c4;
          const float2 ds01 = make_float2(
              P[c] * fmaf(__uint_as_float(dv[4 * c4 + 0]), vdo_sds, d4.x),
              P[c + 1] * fmaf(__uint_as_float(dv[4 * c4 + 1]), vdo_sds, d4.y));
          const float2 ds23 = make_float2(
              P[c + 2] * fmaf(__uint_as_float(dv[4 * c4 + 2]), vdo_sds, d4.z),
              P[c + 3] * fmaf(__uint_as_float(dv[4 * c4 + 3]), vdo_sds, d4.w));
          dsp[16 * hh + 2 * c4] = pack_f16(ds01.x, ds01.y);
          dsp[16 * hh + 2 * c4 + 1] = pack_f16(ds23.x, ds23.y);
        }
      }
      // the previous dS tile must have been consumed by its dK and dQ products
      if (n > 0) {
        ok = __all_sync(0xffffffffu, mbar_wait(ds_empty, (n - 1) & 1, wd, ERR_BWD_DS_FULL));
        if (!ok) break;
      }
#pragma unroll
      for (int ch = 0; ch < 8; ++ch) {
        const int pos = ch ^ (r & 7);       // 128-byte swizzle
        *reinterpret_cast<uint4*>(ds_row + pos * 16) =
            make_uint4(dsp[4 * ch], dsp[4 * ch + 1], dsp[4 * ch + 2], dsp[4 * ch + 3]);
      }
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      tc_fence_before();
      mbar_arrive(ds_full);
    }
    // ---------------------------------------------------------- epilogue
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(dkv_done, 0, wd, ERR_BWD_DKV_DONE));
    if (ok) {
      tc_fence_after();
      const uint32_t tcol = tmem + lane_off + (wg == 0 ? L::T_DV : L::T_DK);
      // undo the operand scales: dV carries s_do, dK carries s_ds s_q
      const float mul = (wg == 0) ? p.scales->dv_mul : p.scales->dk_mul;
      __nv_bfloat16* dst = (wg == 0) ? p.dv : p.dk;
      const long t = (p.cu_seqlens != nullptr) ? (long)seq_start + kv_row : (long)b * p.N + kv_row;
      __nv_bfloat16* row_ptr = dst + (t * p.Hkv + hk) * (long)D;
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        uint32_t v[32];
        tmem_ld32(tcol + 32 * c, v);
        tmem_wait_ld32(v);
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e)
          pk[e] = pack_bf16(__uint_as_float(v[2 * e]) * mul, __uint_as_float(v[2 * e + 1]) * mul);
        if (kv_ok) {
          uint4* d4 = reinterpret_cast<uint4*>(row_ptr + 32 * c);
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4)
            d4[q4] = make_uint4(pk[4 * q4], pk[4 * q4 + 1], pk[4 * q4 + 2], pk[4 * q4 + 3]);
        }
      }
    }
  }

  // ---------------------------------------------------------------- teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 13) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <int D, bool CAUSAL, bool SPARSE>
cudaError_t launch_bwd_t(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                         const CUtensorMap& mdo, const BwdParams& p, cudaStream_t stream,
                         cudaEvent_t ev_begin, cudaEvent_t ev_end) {
  const long tokens = (p.cu_seqlens != nullptr) ? (long)p.total : (long)p.B * p.N;
  int dev = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  // K1: max-abs partials (one per block), K2: scales, fp16 copies, D, zeroed
  // accumulator
  BwdParams pp = p;
  pp.nabs = std::min(sms * 4, ABSMAX_MAX_BLOCKS);
  bwd_absmax_kernel<D><<<pp.nabs, 256, 0, stream>>>(pp, tokens);
  e = cudaGetLastError();
  if (e != cudaSuccess) {
    if (std::getenv("FA_DEBUG")) std::fprintf(stderr, "libfa: absmax kernel launch\n");
    return e;
  }
  bwd_pre_kernel<D><<<sms * 6, 256, 0, stream>>>(pp, tokens);
  e = cudaGetLastError();
  if (e != cudaSuccess) {
    if (std::getenv("FA_DEBUG")) std::fprintf(stderr, "libfa: pre kernel launch\n");
    return e;
  }
  auto kern = bwd_main_kernel<D, CAUSAL, SPARSE>;
  const int smem = BwdLayout<D>::ALLOC;
  // causal dispatch chunks: one chunk of every pair unless the fp32 dQ
  // accumulator is at least twice the L2; then the fewest (sequence, kv head)
  // pairs whose blocks make at least four waves (one block per SM).  Measured
  // on B200: at B=1, H=16, N=65536, d=128 (512 MiB accumulator, chunks of 2)
  // the step went from 910 to 951 TFLOP/s, mostly through a higher sustained
  // clock; at N=16384, d=64 (64 MiB, in L2 anyway) chunks of 5 were 3% slower
  // than one chunk.
  BwdParams pc = pp;
  {
    const long nkv = (p.N + 127) / 128;
    const long bh = (long)p.Hkv * p.B;
    int l2 = 0;
    if (cudaDeviceGetAttribute(&l2, cudaDevAttrL2CacheSize, dev) != cudaSuccess) l2 = 0;
    const double acc_bytes = (double)p.tile_slots * p.Hq * 128.0 * D * 4.0;
    const long want = (4L * sms + nkv - 1) / nkv;
    pc.order_chunk = (l2 > 0 && acc_bytes >= 2.0 * l2) ? (int)std::max(1L, std::min(bh, want))
                                                         : (int)bh;
  }
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) {
    if (std::getenv("FA_DEBUG")) std::fprintf(stderr, "libfa: set smem attribute\n");
    return e;
  }
  const unsigned grid = (unsigned)((p.N + 127) / 128) * p.Hkv * p.B;
  if (ev_begin != nullptr) cudaEventRecord(ev_begin, stream);
  kern<<<grid, BWD_THREADS, smem, stream>>>(mq, mk, mv, mdo, pc);
  e = cudaGetLastError();
  if (e == cudaSuccess && ev_end != nullptr) e = cudaEventRecord(ev_end, stream);
  if (e != cudaSuccess) {
    if (std::getenv("FA_DEBUG")) std::fprintf(stderr, "libfa: main kernel launch\n");
    return e;
  }
  const int nq = (p.N + 127) / 128;
  const long items = (long)nq * p.Hq * p.B;
  // resident blocks per SM of the convert kernel: per instantiation, the same
  // on every B200; callers on several host threads may race to fill it, so
  // it is an atomic (relaxed: any thread's answer is the same number)
  static std::atomic<int> dq_blocks_cache{0};
  int dq_blocks_per_sm = dq_blocks_cache.load(std::memory_order_relaxed);
  if (dq_blocks_per_sm == 0) {
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&dq_blocks_per_sm, bwd_dq_kernel<D>, 256, 0);
    if (e != cudaSuccess) return e;
    if (dq_blocks_per_sm < 1) dq_blocks_per_sm = 1;
    dq_blocks_cache.store(dq_blocks_per_sm, std::memory_order_relaxed);
  }
  const long g2 = std::min<long>(items, (long)sms * dq_blocks_per_sm);
  bwd_dq_kernel<D><<<(unsigned)g2, 256, 0, stream>>>(pp, items, nq);
  return cudaGetLastError();
}

template <bool SPARSE>
inline cudaError_t launch_bwd_s(const CUtensorMap& mq, const CUtensorMap& mk,
                                const CUtensorMap& mv, const CUtensorMap& mdo,
                                const BwdParams& p, int d, bool causal, cudaStream_t stream,
                                cudaEvent_t ev_begin, cudaEvent_t ev_end) {
  if (d == 64)
    return causal ? launch_bwd_t<64, true, SPARSE>(mq, mk, mv, mdo, p, stream, ev_begin, ev_end)
                  : launch_bwd_t<64, false, SPARSE>(mq, mk, mv, mdo, p, stream, ev_begin, ev_end);
  return causal ? launch_bwd_t<128, true, SPARSE>(mq, mk, mv, mdo, p, stream, ev_begin, ev_end)
                : launch_bwd_t<128, false, SPARSE>(mq, mk, mv, mdo, p, stream, ev_begin, ev_end);
}

inline cudaError_t launch_bwd(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                              const CUtensorMap& mdo, const BwdParams& p, int d, bool causal,
                              cudaStream_t stream, cudaEvent_t ev_begin, cudaEvent_t ev_end) {
  return p.bmask != nullptr
             ? launch_bwd_s<true>(mq, mk, mv, mdo, p, d, causal, stream, ev_begin, ev_end)
             : launch_bwd_s<false>(mq, mk, mv, mdo, p, d, causal, stream, ev_begin, ev_end);
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
