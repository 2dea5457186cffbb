// fa_decode.cuh -- decode attention over a KV cache for sm_100a: one new
// query token per sequence attends to the L_b cached keys and values of its
// sequence.
//
// What is computed is the forward of the same definition (tutorial
// 「注意力机制基础」 2.1) for a single query row: o = softmax(scale q K^T) V
// over keys 0..L_b-1, and lse = ln sum_j exp(scale q.k_j).  The tutorial's
// 2.3.1 and the blog post's 4.2 describe this decode step: every generated
// token re-reads the whole cache, so the step is bound by HBM bandwidth,
// not by arithmetic -- about 2 FLOP per byte of K and V per query head.
//
// B200 design:
//  * Split-KV, balanced.  The 128-key tiles of every (sequence, kv head)
//    pair, laid end to end, are cut into one contiguous range per CTA of
//    equal length (to one tile), so that a few long caches or many short
//    ones fill the 148 SMs alike.  A CTA serves all g = Hq/Hkv query heads
//    of a kv head, so each K and V element leaves HBM once.  For every pair
//    its range touches it writes a partial (o_s normalised by its own sum,
//    lse_s); the merge kernel combines each pair's partials exactly:
//    lse = ln sum_s e^(lse_s) and o = sum_s e^(lse_s - lse) o_s (the
//    online-softmax merge rule of the blog post's 3.2.1, applied to chunk
//    results).
//  * One TMA producer warp streams the range's K and V tiles through a
//    shared-memory ring, across pair boundaries; eight consumer warps take
//    16 keys of every tile each, with S = Q K^T and O += P V as m16n8k16
//    bf16 tensor-core products (the g query heads are the 16 MMA rows, q
//    stays in registers, and the fp32 S fragment is P's A fragment).
//  * Keys at or past L_b are masked (their cache rows may hold anything).
//  * Launches: [prefix kernel, when the lengths live on the device,] split
//    kernel, merge kernel.  The split and merge kernels are programmatic
//    dependent launches: their CTAs become resident and run their set-up
//    while the previous kernel finishes, then wait for it (griddep_wait)
//    before their first read or write of global memory.
#pragma once
#include "fa_common.cuh"
#include "sm100.cuh"

namespace fa {

struct DecodeParams {
  const __nv_bfloat16* q;   // [B][Hq][D]
  __nv_bfloat16* o;         // [B][Hq][D]
  float* lse;               // [B][Hq]
  const int* seqlens;       // [B] cached keys per sequence, or null (all Lmax)
  long long* boff;          // [B + 1] tiles of the sequences before b (with seqlens)
  float* o_part;            // [B * Hkv + grid][g][D] range partials, normalised
  float* lse_part;          // [B * Hkv + grid][g]    their LSE (natural log)
  int B, Hq, Hkv, Lmax, group;
  int grid;                 // CTAs of the split kernel
  float scale_log2;
  unsigned long long wait_limit_ns;
};

constexpr int DEC_MAX_GRID = 1024;   // bound used by the workspace size

constexpr int DEC_CONSUMERS = 8;                     // warps that compute
constexpr int DEC_THREADS = 32 * (DEC_CONSUMERS + 1);  // + one TMA producer warp
constexpr int DEC_TILE = 16 * DEC_CONSUMERS;         // keys per TMA tile, 16 per warp
constexpr int DEC_GMAX = 16;                         // largest Hq / Hkv (MMA rows)
constexpr int DEC_MERGE_REGS = 8;                    // partials a merge holds in registers

template <int D>
struct DecodeLayout {
  static constexpr int TILE = DEC_TILE * D * 2;            // one K or V tile, bf16
  static constexpr int STAGES = (D == 128) ? 3 : 6;        // K+V tile pairs in flight
  static constexpr int OFF_KV = 0;                         // [stage][K, V]
  static constexpr int OFF_R = STAGES * 2 * TILE;          // fp32 [GMAX][D] output sums
  static constexpr int OFF_M = OFF_R + DEC_GMAX * D * 4;   // fp32 [warps][GMAX] maxima
  static constexpr int OFF_L = OFF_M + DEC_CONSUMERS * DEC_GMAX * 4;   // fp32 [GMAX] sums
  static constexpr int OFF_BAR = OFF_L + DEC_GMAX * 4;     // full[STAGES], empty[STAGES]
  static constexpr int OFF_MISC = OFF_BAR + 2 * STAGES * 8;
  static constexpr int BYTES = OFF_MISC + 16;
  static constexpr int ALLOC = BYTES + 1024;
  static_assert(ALLOC <= 227 * 1024, "shared memory per block");
};

// Tiles of sequence b, and the tiles of the sequences before it (per kv
// head): the flattened tile space is pair-major, pair = b * Hkv + hk.
__device__ __forceinline__ int dec_len(const DecodeParams& p, int b) {
  return p.seqlens != nullptr ? min(max(p.seqlens[b], 0), p.Lmax) : p.Lmax;
}
__device__ __forceinline__ int dec_ntiles(const DecodeParams& p, int b) {
  return (dec_len(p, b) + DEC_TILE - 1) / DEC_TILE;
}
__device__ __forceinline__ long long dec_boff(const DecodeParams& p, int b) {
  return p.seqlens != nullptr ? p.boff[b]
                              : (long long)b * ((p.Lmax + DEC_TILE - 1) / DEC_TILE);
}
__device__ __forceinline__ long long dec_total(const DecodeParams& p) {
  return (long long)p.Hkv * dec_boff(p, p.B);
}
// first flattened tile of CTA c's range: floor(c T / grid)
__device__ __forceinline__ long long dec_range_start(long long c, long long T, int grid) {
  return c * T / grid;
}
// the CTA whose range holds flattened tile x
__device__ __forceinline__ int dec_cta_of(long long x, long long T, int grid) {
  return (int)(((x + 1) * grid - 1) / T);
}

// One contiguous piece of a CTA's range inside one (sequence, kv head) pair.
struct DecodeSeg {
  int b, hk, k0, k1, ntiles;
  long long slot;   // partial slot: pair + CTA (unique, increasing along the ranges)
};

// Walks a CTA's range [pos, end) pair by pair.
struct DecodeWalker {
  int b, hk, tile;
  long long pos, end;

  __device__ void init(const DecodeParams& p, long long t0, long long t1) {
    pos = t0;
    end = t1;
    if (pos >= end) return;
    // the sequence whose tiles hold t0: largest b with Hkv * boff(b) <= t0
    int lo = 0, hi = p.B - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if ((long long)p.Hkv * dec_boff(p, mid) <= t0) lo = mid;
      else hi = mid - 1;
    }
    b = lo;
    const int nt = dec_ntiles(p, b);
    if (nt == 0) {   // only if the offsets disagreed with the lengths
      pos = end;
      return;
    }
    const long long r = t0 - (long long)p.Hkv * dec_boff(p, b);
    hk = (int)(r / nt);
    tile = (int)(r % nt);
  }
  __device__ bool next(const DecodeParams& p, DecodeSeg& sg) {
    if (pos >= end) return false;
    const int nt = dec_ntiles(p, b);
    const int n = (int)min((long long)(nt - tile), end - pos);
    sg.b = b;
    sg.hk = hk;
    sg.k0 = tile * DEC_TILE;
    sg.k1 = min((tile + n) * DEC_TILE, dec_len(p, b));
    sg.ntiles = n;
    sg.slot = (long long)b * p.Hkv + hk + blockIdx.x;
    pos += n;
    tile = 0;
    if (++hk == p.Hkv) {
      hk = 0;
      do {
        ++b;
      } while (b < p.B && dec_ntiles(p, b) == 0);
    }
    return true;
  }
};

// Programmatic dependent launch.  griddep_wait blocks until the grids this
// one depends on have completed and their writes are visible; launched
// without the attribute, stream order has already done that and it returns
// at once.  griddep_launch_dependents lets the next kernel's CTAs start
// their own set-up (they wait in the same way before touching memory).
__device__ __forceinline__ void griddep_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void griddep_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// 16 x 8 x 16 bf16 MMA with fp32 accumulation (sm_80+ warp-level form; the
// query heads of one kv head are at most 16 rows, the M of this shape).
__device__ __forceinline__ void mma_16816(float* c, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
      "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t* r) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t* r) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
// byte address of the 8 elements (16 bytes) at row r, column c (c % 8 == 0)
// of a 128-byte-swizzled TMA tile made of 64-column boxes of DEC_TILE rows
__device__ __forceinline__ uint32_t sw128_addr(uint32_t base, int r, int c) {
  return base + (uint32_t)((c >> 6) * (DEC_TILE * 128) + r * 128 +
                           ((((c & 63) >> 3) ^ (r & 7)) << 4));
}

// Persistent: gridDim.x CTAs (at most one per SM), each with one contiguous
// range of the flattened tiles.  Warp 8 streams the range's K and V tiles
// through the TMA ring, across pair boundaries; warps 0-7 each take 16 keys
// of every tile with their own online-softmax state (running max and sum
// per query head, and a 16 x D output fragment), and merge the eight states
// at the end of each pair's piece.
//
// Per warp and tile: S^T = Q K^T as (heads x 16 keys), Q held in registers
// as MMA A-fragments for the whole item and K^T fragments read with
// ldmatrix from the swizzled tile; p = 2^(S scale log2e - m); the fp32
// S fragment is exactly the A-fragment layout of P for O += P V, whose
// V fragments come from ldmatrix.trans.  Heads past g are zero rows.
template <int D>
__global__ void __launch_bounds__(DEC_THREADS, 1)
    decode_split_kernel(const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmV, const DecodeParams p) {
  using L = DecodeLayout<D>;
  constexpr int ST = L::STAGES;
  constexpr int KS = D / 16;   // k-steps of S (over d)
  constexpr int NB = D / 8;    // n-blocks of O (over d)
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align_1024(smem_raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = p.group;

  uint8_t* ring = smem + L::OFF_KV;
  float* sr = reinterpret_cast<float*>(smem + L::OFF_R);
  float* smx = reinterpret_cast<float*>(smem + L::OFF_M);
  float* sl = reinterpret_cast<float*>(smem + L::OFF_L);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);
  uint64_t* empty = full + ST;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::OFF_MISC);
  const Watchdog wd{&g_fa_error, abort_flag, p.wait_limit_ns};

  if (tid == 0) {
    for (int s = 0; s < ST; ++s) {
      mbar_init(full + s, 1);
      mbar_init(empty + s, DEC_CONSUMERS);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  for (int i = tid; i < DEC_GMAX * D; i += DEC_THREADS) sr[i] = 0.f;
  for (int i = tid; i < DEC_GMAX; i += DEC_THREADS) sl[i] = 0.f;
  if (warp == DEC_CONSUMERS && lane == 0) {
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
  }
  __syncthreads();
  if (tid == 0) griddep_launch_dependents();
  // Nothing above touched global memory.  From here on the kernel reads
  // the lengths, the tile offsets, q and the caches, and writes the
  // partials that the previous call's merge kernel may still be reading.
  griddep_wait();
  const long long T = dec_total(p);   // tiles of the whole batch, per kv head summed

  if (warp == DEC_CONSUMERS) {
    // ============================================================ producer
    if (lane == 0) {
      long c = 0;   // stream position
      bool pok = true;
      DecodeWalker wk;
      DecodeSeg it;
      wk.init(p, dec_range_start(blockIdx.x, T, gridDim.x),
              dec_range_start(blockIdx.x + 1, T, gridDim.x));
      while (pok && wk.next(p, it)) {
        for (int t = 0; pok && t < it.ntiles; ++t, ++c) {
          const int st = (int)(c % ST);
          if (c >= ST && !(pok = mbar_wait(empty + st, (uint32_t)((c / ST - 1) & 1), wd,
                                           ERR_DEC_KV_EMPTY)))
            break;
          uint8_t* kt = ring + (2 * st) * L::TILE;
          uint8_t* vt = kt + L::TILE;
          mbar_arrive_expect_tx(full + st, 2 * L::TILE);
          const int row = it.k0 + DEC_TILE * t;
#pragma unroll
          for (int cb = 0; cb < D / 64; ++cb) {
            tma_load_4d(kt + cb * (DEC_TILE * 128), &tmK, full + st, cb * 64, it.hk, row, it.b);
            tma_load_4d(vt + cb * (DEC_TILE * 128), &tmV, full + st, cb * 64, it.hk, row, it.b);
          }
        }
      }
      if (!pok) {
        // the last fills may still be landing: they must before the CTA exits
        for (long x = (c > ST ? c - ST : 0); x < c; ++x)
          mbar_wait_drain(full + x % ST, (uint32_t)((x / ST) & 1), p.wait_limit_ns);
      }
    }
    return;
  }

  // ============================================================== consumers
  const int qr = lane >> 2;          // fragment row: heads qr and qr + 8
  const int qc = 2 * (lane & 3);     // fragment column pair
  const float c2 = p.scale_log2;
  const uint32_t ring_u = smem_u32(ring);
  long c = 0;                        // stream position
  bool ok = true;

  DecodeWalker wk;
  DecodeSeg it;
  wk.init(p, dec_range_start(blockIdx.x, T, gridDim.x),
          dec_range_start(blockIdx.x + 1, T, gridDim.x));
  while (wk.next(p, it)) {
    const int h0 = it.hk * g;
    float* opart = p.o_part + it.slot * g * D;
    float* lpart = p.lse_part + it.slot * g;
    // Q of the group as A-fragments (rows = heads, zero past g)
    uint32_t qa[KS][4];
    {
      const __nv_bfloat16* qg = p.q + ((long)it.b * p.Hq + h0) * D;
      const bool r0 = qr < g, r1 = qr + 8 < g;
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) {
        const int d0 = 16 * ks + qc;
        qa[ks][0] = r0 ? *reinterpret_cast<const uint32_t*>(qg + qr * D + d0) : 0u;
        qa[ks][1] = r1 ? *reinterpret_cast<const uint32_t*>(qg + (qr + 8) * D + d0) : 0u;
        qa[ks][2] = r0 ? *reinterpret_cast<const uint32_t*>(qg + qr * D + d0 + 8) : 0u;
        qa[ks][3] = r1 ? *reinterpret_cast<const uint32_t*>(qg + (qr + 8) * D + d0 + 8) : 0u;
      }
    }
    float m0 = -INFINITY, m1 = -INFINITY;   // running max of rows qr, qr + 8 (log2 units)
    float l0 = 0.f, l1 = 0.f;               // this lane's share of their sums
    float o[NB][4];
#pragma unroll
    for (int nb = 0; nb < NB; ++nb) o[nb][0] = o[nb][1] = o[nb][2] = o[nb][3] = 0.f;

    for (int t = 0; t < it.ntiles; ++t, ++c) {
      const int st = (int)(c % ST);
      if (ok) ok = mbar_wait(full + st, (uint32_t)((c / ST) & 1), wd, ERR_DEC_KV_FULL);
      if (ok) {
        const uint32_t kt = ring_u + (uint32_t)((2 * st) * L::TILE);
        const uint32_t vt = kt + (uint32_t)L::TILE;
        const int kb = 16 * warp;                                  // this warp's keys
        const int nvalid = min(DEC_TILE, it.k1 - (it.k0 + DEC_TILE * t));
        // ---- S^T (heads x 16 keys) = Q K^T: two 8-key n-blocks
        float s[2][4];
#pragma unroll
        for (int nb = 0; nb < 2; ++nb) {
          s[nb][0] = s[nb][1] = s[nb][2] = s[nb][3] = 0.f;
          const int key = kb + 8 * nb + (lane & 7);
#pragma unroll
          for (int kq = 0; kq < KS / 2; ++kq) {     // 4 matrices: d0 .. d0 + 31
            uint32_t r[4];
            ldsm_x4(sw128_addr(kt, key, 32 * kq + 8 * (lane >> 3)), r);
            mma_16816(s[nb], qa[2 * kq], r[0], r[1]);
            mma_16816(s[nb], qa[2 * kq + 1], r[2], r[3]);
          }
        }
        // ---- online softmax on the fragments (rows qr, qr + 8)
        float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
        for (int nb = 0; nb < 2; ++nb)
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const bool valid = kb + 8 * nb + qc + e < nvalid;
            s[nb][e] = valid ? s[nb][e] * c2 : -INFINITY;
            s[nb][2 + e] = valid ? s[nb][2 + e] * c2 : -INFINITY;
            mx0 = fmaxf(mx0, s[nb][e]);
            mx1 = fmaxf(mx1, s[nb][2 + e]);
          }
#pragma unroll
        for (int x = 1; x <= 2; x <<= 1) {
          mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, x));
          mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, x));
        }
        const float n0 = fmaxf(m0, mx0), n1 = fmaxf(m1, mx1);
        const float r0 = (n0 == -INFINITY) ? 0.f : n0;   // all keys so far masked
        const float r1 = (n1 == -INFINITY) ? 0.f : n1;
        const float a0 = ex2(m0 - r0), a1 = ex2(m1 - r1);
        m0 = n0;
        m1 = n1;
        uint32_t pa[4];   // P as the A-fragment of O += P V
        float ps0 = 0.f, ps1 = 0.f;
#pragma unroll
        for (int nb = 0; nb < 2; ++nb) {
          const float p0 = ex2(s[nb][0] - r0), p1 = ex2(s[nb][1] - r0);
          const float p2 = ex2(s[nb][2] - r1), p3 = ex2(s[nb][3] - r1);
          ps0 += p0 + p1;
          ps1 += p2 + p3;
          pa[2 * nb] = pack_bf16(p0, p1);
          pa[2 * nb + 1] = pack_bf16(p2, p3);
        }
        l0 = l0 * a0 + ps0;
        l1 = l1 * a1 + ps1;
        // ---- O = O * alpha + P V: V fragments by ldmatrix.trans, two
        // 8-column n-blocks per load.  A cache row past the sequence's end
        // may hold anything (inf, NaN), and 0 * inf is not 0: in a warp's
        // partial tile the V halves of masked keys are zeroed in registers
        // (b0 holds keys kb + qc, kb + qc + 1; b1 the same plus 8).
        const bool partial = kb + 16 > nvalid;
        uint32_t vm0 = 0xffffffffu, vm1 = 0xffffffffu;
        if (partial) {
          vm0 = (kb + qc < nvalid ? 0x0000ffffu : 0u) | (kb + qc + 1 < nvalid ? 0xffff0000u : 0u);
          vm1 = (kb + 8 + qc < nvalid ? 0x0000ffffu : 0u) |
                (kb + 9 + qc < nvalid ? 0xffff0000u : 0u);
        }
#pragma unroll
        for (int nb = 0; nb < NB; nb += 2) {
          uint32_t r[4];
          const int key = kb + 8 * ((lane >> 3) & 1) + (lane & 7);
          ldsm_x4_trans(sw128_addr(vt, key, 8 * nb + 8 * (lane >> 4)), r);
          r[0] &= vm0;
          r[1] &= vm1;
          r[2] &= vm0;
          r[3] &= vm1;
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            o[nb + e][0] *= a0;
            o[nb + e][1] *= a0;
            o[nb + e][2] *= a1;
            o[nb + e][3] *= a1;
            mma_16816(o[nb + e], pa, r[2 * e], r[2 * e + 1]);
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(empty + st);   // this warp is done with the stage
    }

    // ---- merge the eight warps' states: common max per head, rescaled sums
    l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
    l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
    if ((lane & 3) == 0) {
      smx[warp * DEC_GMAX + qr] = m0;
      smx[warp * DEC_GMAX + qr + 8] = m1;
    }
    asm volatile("bar.sync 1, %0;" ::"n"(32 * DEC_CONSUMERS));
    float M0 = -INFINITY, M1 = -INFINITY;
#pragma unroll
    for (int w = 0; w < DEC_CONSUMERS; ++w) {
      M0 = fmaxf(M0, smx[w * DEC_GMAX + qr]);
      M1 = fmaxf(M1, smx[w * DEC_GMAX + qr + 8]);
    }
    const float f0 = (m0 == -INFINITY) ? 0.f : ex2(m0 - M0);
    const float f1 = (m1 == -INFINITY) ? 0.f : ex2(m1 - M1);
    if (ok) {
      if ((lane & 3) == 0) {
        if (qr < g) atomicAdd(sl + qr, f0 * l0);
        if (qr + 8 < g) atomicAdd(sl + qr + 8, f1 * l1);
      }
#pragma unroll
      for (int nb = 0; nb < NB; ++nb) {
        const int col = 8 * nb + qc;
        if (qr < g) {
          atomicAdd(sr + qr * D + col, f0 * o[nb][0]);
          atomicAdd(sr + qr * D + col + 1, f0 * o[nb][1]);
        }
        if (qr + 8 < g) {
          atomicAdd(sr + (qr + 8) * D + col, f1 * o[nb][2]);
          atomicAdd(sr + (qr + 8) * D + col + 1, f1 * o[nb][3]);
        }
      }
    }
    asm volatile("bar.sync 1, %0;" ::"n"(32 * DEC_CONSUMERS));
    if (ok) {
      for (int e = tid; e < g * D; e += 32 * DEC_CONSUMERS) {
        const int h = e / D;
        opart[e] = sr[e] / sl[h];
        if (e % D == 0) {
          float mh = -INFINITY;
          for (int w = 0; w < DEC_CONSUMERS; ++w) mh = fmaxf(mh, smx[w * DEC_GMAX + h]);
          lpart[h] = (mh + log2f(sl[h])) * 0.69314718055994530942f;
        }
      }
    }
    asm volatile("bar.sync 1, %0;" ::"n"(32 * DEC_CONSUMERS));
    for (int e = tid; e < g * D; e += 32 * DEC_CONSUMERS) sr[e] = 0.f;
    if (tid < DEC_GMAX) sl[tid] = 0.f;
    asm volatile("bar.sync 1, %0;" ::"n"(32 * DEC_CONSUMERS));
  }
}

// Merge the partials of one (sequence, query head): grid B * Hq, D threads
// (one output column each).  The pair's partials sit in the slots pair + c
// of the CTAs c whose ranges overlap its tiles.  Up to DEC_MERGE_REGS of
// them are loaded at once into registers (one memory round trip); more go
// through shared memory D at a time, so that every thread's sum is a run of
// independent loads.
template <int D>
__global__ void __launch_bounds__(D) decode_merge_kernel(const DecodeParams p) {
  __shared__ float wsh[D];
  __shared__ float red[D / 32];
  const int bh = blockIdx.x;   // b * Hq + h
  const int b = bh / p.Hq, h = bh % p.Hq;
  const int g = p.group, hk = h / g, hg = h - hk * g;
  const int tid = threadIdx.x;
  // The pair's slot range.  With every cache full it follows from the
  // launch parameters alone and is worked out while the split kernel runs;
  // device-side lengths need the prefix kernel's offsets first.
  int nt = 0, c0 = 0, c1 = -1;
  long long T = 0;
  auto slot_range = [&]() {
    nt = dec_ntiles(p, b);
    if (nt == 0) return;
    T = dec_total(p);
    const long long off = (long long)p.Hkv * dec_boff(p, b) + (long long)hk * nt;
    c0 = dec_cta_of(off, T, p.grid);
    c1 = dec_cta_of(off + nt - 1, T, p.grid);
  };
  if (p.seqlens == nullptr) slot_range();
  griddep_wait();   // the split kernel's partials (and, before it, the offsets)
  if (p.seqlens != nullptr) slot_range();
  float acc = 0.f, wsum = 0.f, M = -INFINITY;
  if (nt > 0) {
    const int ns = c1 - c0 + 1;
    const long long s0 = (long long)b * p.Hkv + hk + c0;   // first slot
    // a CTA between c0 and c1 with an empty range wrote no partial: it is
    // skipped.  Empty ranges exist only with more CTAs than tiles.
    const bool all_ranges = T >= p.grid;
    auto has_range = [&](int c) {
      return all_ranges || dec_range_start(c, T, p.grid) < dec_range_start(c + 1, T, p.grid);
    };
    if (ns <= DEC_MERGE_REGS) {
      // the usual case: every partial of this thread's column and every
      // partial LSE loaded at once, then weighed in registers
      float l[DEC_MERGE_REGS], v[DEC_MERGE_REGS];
#pragma unroll
      for (int k = 0; k < DEC_MERGE_REGS; ++k) {
        l[k] = -INFINITY;
        v[k] = 0.f;
        if (k < ns && has_range(c0 + k)) {
          l[k] = p.lse_part[(s0 + k) * g + hg];
          v[k] = p.o_part[((s0 + k) * g + hg) * D + tid];
        }
      }
#pragma unroll
      for (int k = 0; k < DEC_MERGE_REGS; ++k) M = fmaxf(M, l[k]);
#pragma unroll
      for (int k = 0; k < DEC_MERGE_REGS; ++k) {
        const float w = (l[k] == -INFINITY) ? 0.f : expf(l[k] - M);
        wsum += w;
        acc = fmaf(w, v[k], acc);
      }
      p.o[(long long)bh * D + tid] = __float2bfloat16_rn(acc / wsum);
      if (tid == 0) p.lse[bh] = M + logf(wsum);
      return;
    }
    float mx = -INFINITY;
    for (int s = tid; s < ns; s += D)
      if (has_range(c0 + s)) mx = fmaxf(mx, p.lse_part[(s0 + s) * g + hg]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    if ((tid & 31) == 0) red[tid >> 5] = mx;
    __syncthreads();
#pragma unroll
    for (int w = 0; w < D / 32; ++w) M = fmaxf(M, red[w]);
    for (int sb = 0; sb < ns; sb += D) {
      const int n = min(D, ns - sb);
      __syncthreads();
      if (tid < n)
        wsh[tid] = has_range(c0 + sb + tid) ? expf(p.lse_part[(s0 + sb + tid) * g + hg] - M)
                                            : -1.f;   // no partial
      __syncthreads();
      const float* op = p.o_part + ((s0 + sb) * g + hg) * D + tid;
#pragma unroll 8
      for (int k = 0; k < n; ++k) {
        const float w = wsh[k];
        if (w >= 0.f) {
          wsum += w;
          acc = fmaf(w, op[(long long)k * g * D], acc);
        }
      }
    }
    acc /= wsum;
  }
  p.o[(long long)bh * D + tid] = __float2bfloat16_rn(acc);
  if (tid == 0) p.lse[bh] = (nt == 0) ? -INFINITY : M + logf(wsum);
}

// Tiles before each sequence (exclusive prefix sum of ceil(L_b / 128)), one
// block: needed when the cache lengths live on the device.
__global__ void __launch_bounds__(1024) decode_prefix_kernel(const DecodeParams p) {
  __shared__ long long part[1024];
  const int tid = threadIdx.x;
  if (tid == 0) griddep_launch_dependents();   // the split kernel waits for our writes
  const int per = (p.B + 1023) / 1024;
  const int b0 = min(p.B, tid * per), b1 = min(p.B, b0 + per);
  long long sum = 0;
  for (int b = b0; b < b1; ++b) sum += dec_ntiles(p, b);
  part[tid] = sum;
  __syncthreads();
  for (int o = 1; o < 1024; o <<= 1) {   // inclusive scan
    const long long v = tid >= o ? part[tid - o] : 0;
    __syncthreads();
    part[tid] += v;
    __syncthreads();
  }
  long long run = part[tid] - sum;   // exclusive
  for (int b = b0; b < b1; ++b) {
    p.boff[b] = run;
    run += dec_ntiles(p, b);
  }
  if (tid == 1023) p.boff[p.B] = part[1023];
}

inline size_t decode_workspace_bytes(int B, int Hq, int Lmax, int d) {
  (void)Lmax;
  const size_t boff = ((size_t)(B + 1) * 8 + 255) & ~(size_t)255;
  // slots (B * Hkv + grid) x g heads <= B * Hq + grid * 16
  const size_t rows = (size_t)B * Hq + (size_t)DEC_MAX_GRID * DEC_GMAX;
  const size_t o = (rows * d * 4 + 255) & ~(size_t)255;
  return boff + o + ((rows * 4 + 255) & ~(size_t)255);
}

template <int D>
cudaError_t launch_decode_d(const CUtensorMap& mk, const CUtensorMap& mv, const DecodeParams& p,
                            cudaStream_t stream) {
  auto kern = decode_split_kernel<D>;
  const int smem = DecodeLayout<D>::ALLOC;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  if (p.seqlens != nullptr) {
    decode_prefix_kernel<<<1, 1024, 0, stream>>>(p);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  cudaLaunchAttribute pdl[1];
  pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  pdl[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.stream = stream;
  cfg.attrs = pdl;
  cfg.numAttrs = 1;
  if (p.grid > 0) {
    cfg.gridDim = dim3((unsigned)p.grid);
    cfg.blockDim = dim3(DEC_THREADS);
    cfg.dynamicSmemBytes = (size_t)smem;
    e = cudaLaunchKernelEx(&cfg, kern, mk, mv, p);
    if (e != cudaSuccess) return e;
  }
  cfg.gridDim = dim3((unsigned)(p.B * p.Hq));
  cfg.blockDim = dim3(D);
  cfg.dynamicSmemBytes = 0;
  return cudaLaunchKernelEx(&cfg, decode_merge_kernel<D>, p);
}

inline cudaError_t launch_decode(const CUtensorMap& mk, const CUtensorMap& mv,
                                 const DecodeParams& p, int d, cudaStream_t stream) {
  return d == 64 ? launch_decode_d<64>(mk, mv, p, stream) : launch_decode_d<128>(mk, mv, p, stream);
}

}  // namespace fa
